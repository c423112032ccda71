"""The oracle's pins catch plausible mistakes in it.

One mistake at a time is planted in a copy of the oracle's C source -- a
wrong exponent bias, rounding direction, tie rule, sign, index, constant or
dropped term of the kind a hand-written encoder or generator could carry --
and the copy is compiled with the oracle's own flags.  The oracle pin tests
then run against it in a child process (the oracle loads the copy through
FP4_ORACLE_LIB); every mutant must make at least one pin fail, while the
unmodified source, compiled the same way, passes them all.  The oracle's own
source file is never modified.  The Python-level GEMM reference is mutated
in process the same way.
"""
import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

import pytest

import oracle as O
from oracle import build as ob
from conftest import ROOT

PINS = [os.path.join(ROOT, "tests", f) for f in
        ("test_oracle_formats.py", "test_oracle_quant.py", "test_oracle_rht.py",
         "test_oracle_sr_philox.py", "test_oracle_quest.py")]

# (name, text in fp4_oracle.c, replacement, which occurrence to replace)
MUTANTS = [
    ("e2m1 exponent bias", "ldexp(1.0 + 0.5 * m, e - 1)", "ldexp(1.0 + 0.5 * m, e)", 0),
    ("e2m1 ties away from even",
     "double d = fabs(a - orc_e2m1_value((uint8_t)c));\n"
     "    if (d < bestd || (d == bestd && (c & 1) == 0 && (best & 1) == 1)) {",
     "double d = fabs(a - orc_e2m1_value((uint8_t)c));\n    if (d <= bestd) {", 0),
    ("e2m1 sign of a negative zero lost", "return (uint8_t)(best | (signbit(v) ? 8 : 0));",
     "return (uint8_t)(best | (v < 0 ? 8 : 0));", 0),
    ("SR carry test off by one", "code = (k + (uint32_t)u >= 65536u) ? hi : lo;",
     "code = (k + (uint32_t)u > 65536u) ? hi : lo;", 0),
    ("SR fraction rounded up", "(uint32_t)floor(ldexp(p, 16))", "(uint32_t)ceil(ldexp(p, 16))", 0),
    ("SR fraction to 15 bits", "(uint32_t)floor(ldexp(p, 16))", "(uint32_t)floor(ldexp(p, 15))", 0),
    ("SR decided on the complemented draw", "code = (k + (uint32_t)u >= 65536u) ? hi : lo;",
     "code = (k + (uint32_t)(65535u - u) >= 65536u) ? hi : lo;", 0),
    ("16-bit draw halves swapped", "return (uint16_t)((i & 1) ? (w >> 16) : (w & 0xFFFFu));",
     "return (uint16_t)((i & 1) ? (w & 0xFFFFu) : (w >> 16));", 0),
    ("16-bit draw from 32-bit draw i, not i / 2", "uint32_t w = orc_draw(seed, stream, i >> 1);",
     "uint32_t w = orc_draw(seed, stream, i);", 0),
    ("E4M3 exponent bias", "ldexp(1.0 + (double)m / 8.0, e - 7)",
     "ldexp(1.0 + (double)m / 8.0, e - 8)", 0),
    ("E4M3 saturates to NaN", "if (a > 448.0) return 0x7E;", "if (a > 448.0) return 0x7F;", 0),
    ("tensor scale without the E2M1 maximum", "float e = 2688.0f / A;",
     "float e = 448.0f / A;", 0),
    ("decode scale inverted", "*s_dec = A / 2688.0f;", "*s_dec = 2688.0f / A;", 0),
    ("block scale divides by 4, not 6", "float t = (bmax * q->s_enc) / 6.0f;",
     "float t = (bmax * q->s_enc) / 4.0f;", 0),
    ("block reciprocal inverted", "float inv = (sf == 0) ? 0.0f : q->s_enc / sfv;",
     "float inv = (sf == 0) ? 0.0f : sfv / q->s_enc;", 0),
    ("nibble order swapped",
     "if ((c & 1) == 0) *byte = (uint8_t)((*byte & 0xF0) | code);",
     "if ((c & 1) == 1) *byte = (uint8_t)((*byte & 0xF0) | code);", 0),
    ("SR draw index transposed",
     "uint64_t idx = (uint64_t)(q->row_offset + r) * (uint64_t)C + (uint64_t)c;",
     "uint64_t idx = (uint64_t)c * (uint64_t)C + (uint64_t)(q->row_offset + r);", 0),
    ("MXFP4 SR draw index without the row offset",
     "uint64_t idx = (uint64_t)(q->row_offset + r) * (uint64_t)C + (uint64_t)c;",
     "uint64_t idx = (uint64_t)r * (uint64_t)C + (uint64_t)c;", 1),
    ("Philox with 9 rounds", "for (int round = 0; round < 10; ++round)",
     "for (int round = 0; round < 9; ++round)", 0),
    ("Philox Weyl constants swapped", "if (round > 0) { k0 += PHILOX_W0; k1 += PHILOX_W1; }",
     "if (round > 0) { k0 += PHILOX_W1; k1 += PHILOX_W0; }", 0),
    ("Philox key bumped before the first round",
     "if (round > 0) { k0 += PHILOX_W0; k1 += PHILOX_W1; }",
     "{ k0 += PHILOX_W0; k1 += PHILOX_W1; }", 0),
    ("Philox output words reversed", "return out[i & 3];", "return out[3 - (i & 3)];", 0),
    ("Philox stream in the wrong counter word",
     "uint32_t ctr[4] = {(uint32_t)c, (uint32_t)(c >> 32), stream, 0u};",
     "uint32_t ctr[4] = {(uint32_t)c, (uint32_t)(c >> 32), 0u, stream};", 0),
    ("Hadamard scale 1/n", "return (float)(1.0 / sqrt((double)n));",
     "return (float)(1.0 / (double)n);", 0),
    ("Hadamard butterfly sign", "v[j + h] = a - b;", "v[j + h] = b - a;", 0),
    ("Hadamard random signs dropped", "for (int j = 0; j < n; ++j) v[j] = v[j] * d[j];",
     "for (int j = 0; j < n; ++j) v[j] = v[j];", 0),
    ("MXFP4 exponent offset", "orc_floor_log2(top) - 2;", "orc_floor_log2(top) - 1;", 0),
    ("MXFP4 scale byte bias", "(uint8_t)(e + 127);", "(uint8_t)(e + 128);", 0),
    ("E8M0 decode bias", "return ldexp(1.0, (int)b - 127);", "return ldexp(1.0, (int)b - 126);", 0),
    ("amax of signed values", "float a = fabsf(x[i]);", "float a = x[i];", 0),
    ("2-D tile max over its first row only",
     "float v = fabsf(q->x[(i * 16 + a) * C + j * 16 + b]);",
     "float v = fabsf(q->x[(i * 16) * C + j * 16 + b]);", 0),
    ("floor(log2) of subnormals", "return k - 149;", "return k - 150;", 0),
    ("floor(log2) of normals", "if (E > 0) return E - 127;", "if (E > 0) return E - 126;", 0),
    ("E4M3 subnormal exponent", "ldexp((double)m / 8.0, -6)", "ldexp((double)m / 8.0, -7)", 0),
    ("E2M1 RTN clamps at 5", "if (a > 8.0) a = 8.0;", "if (a > 5.0) a = 5.0;", 0),
    ("2-D block scale divides by 4, not 6", "float t = (bmax * q->s_enc) / 6.0f;",
     "float t = (bmax * q->s_enc) / 4.0f;", 1),
    ("2-D block reciprocal inverted", "float inv = (sf == 0) ? 0.0f : q->s_enc / sfv;",
     "float inv = (sf == 0) ? 0.0f : sfv / q->s_enc;", 1),
    ("dequantize with the other scale format",
     "double sv = is_e8m0 ? orc_e8m0_value(s) : orc_e4m3_value(s);",
     "double sv = is_e8m0 ? orc_e4m3_value(s) : orc_e8m0_value(s);", 0),
    ("MXFP4 exponent clamp at -126", "if (e < -127) e = -127;", "if (e < -126) e = -126;", 0),
    ("zero tensor decodes with scale 0", "if (A == 0.0f) { *s_enc = 1.0f; *s_dec = 1.0f; return; }",
     "if (A == 0.0f) { *s_enc = 1.0f; *s_dec = 0.0f; return; }", 0),
    ("reciprocal of a zero scale not zero", "float inv = (sf == 0) ? 0.0f : q->s_enc / sfv;",
     "float inv = (sf == 0) ? 1.0f : q->s_enc / sfv;", 0),
    ("QuEST alpha of 3", "#define QUEST_ALPHA 2.9224751f", "#define QUEST_ALPHA 3.0f", 0),
    ("QuEST mean over 31", "float rms = sqrtf(sum / 32.0f);", "float rms = sqrtf(sum / 31.0f);", 0),
    ("QuEST without the square root", "float rms = sqrtf(sum / 32.0f);", "float rms = sum / 32.0f;", 0),
    ("QuEST last group dropped", "float sum = (g[0] + g[1]) + (g[2] + g[3]);",
     "float sum = (g[0] + g[1]) + g[2];", 0),
    ("QuEST scale from the block max", "float top = (q->round_mode == 2) ? orc_quest_threshold(row + b * 32) : bmax;",
     "float top = bmax;", 0),
    ("QuEST rounds stochastically", "        if (q->round_mode != 1) {\n          code = orc_e2m1_rtn(v);",
     "        if (q->round_mode == 0) {\n          code = orc_e2m1_rtn(v);", 0),
]


def _mutated_source(old: str, new: str, occurrence: int) -> str:
    src = open(ob.SRC).read()
    pos, start = -1, 0
    for _ in range(occurrence + 1):
        pos = src.find(old, start)
        assert pos >= 0, f"mutation site not found: {old!r}"
        start = pos + 1
    return src[:pos] + new + src[pos + len(old):]


def _pins_pass(lib_path: str) -> bool:
    env = dict(os.environ, FP4_ORACLE_LIB=lib_path, PYTHONPATH=ROOT)
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        *PINS], cwd=ROOT, env=env, capture_output=True, timeout=600)
    return r.returncode == 0


def _build_and_check(tmp, tag, text):
    src = os.path.join(tmp, f"oracle_{tag}.c")
    with open(src, "w") as f:
        f.write(text)
    lib = ob.compile_to(src, os.path.join(tmp, f"liboracle_{tag}.so"))
    return _pins_pass(lib)


def test_every_mutant_is_caught(tmp_path):
    tmp = str(tmp_path)
    jobs = [("clean", open(ob.SRC).read())]
    jobs += [(f"m{i}", _mutated_source(old, new, occ))
             for i, (_name, old, new, occ) in enumerate(MUTANTS)]
    with ThreadPoolExecutor(max_workers=max(1, min(8, os.cpu_count() or 1))) as ex:
        passed = list(ex.map(lambda j: _build_and_check(tmp, *j), jobs))
    assert passed[0], "the unmodified oracle, compiled the same way, must pass its pins"
    survivors = [MUTANTS[i][0] for i, ok in enumerate(passed[1:]) if ok]
    assert not survivors, f"mutants no pin catches: {survivors}"


def test_gemm_reference_mutants_are_caught(monkeypatch):
    """The float64 GEMM reference with a dropped tensor scale, or with alpha
    applied twice, fails the exact small-case pin."""
    import test_oracle_quant as Q
    orig = O.gemm

    def drop_sdec_b(a_hat, b_hat, alpha=1.0, s_dec_a=1.0, s_dec_b=1.0):
        return orig(a_hat, b_hat, alpha, s_dec_a, 1.0)

    def alpha_twice(a_hat, b_hat, alpha=1.0, s_dec_a=1.0, s_dec_b=1.0):
        return orig(a_hat, b_hat, alpha * alpha, s_dec_a, s_dec_b)

    for mutant in (drop_sdec_b, alpha_twice):
        monkeypatch.setattr(O, "gemm", mutant)
        with pytest.raises(AssertionError):
            Q.test_gemm_reference_exact_on_small_case()
    monkeypatch.setattr(O, "gemm", orig)
    Q.test_gemm_reference_exact_on_small_case()


def _fails(fn) -> bool:
    try:
        fn()
    except AssertionError:
        return True
    return False


def test_quant_noise_mutants_are_caught(monkeypatch):
    """The noise diagnostic's reference without the tensor decode scale, with
    |error| summed instead of its square, or with the dequantized signal in
    place of the input's, fails one of its pins."""
    import numpy as np
    import test_oracle_quant as Q
    orig = O.quant_noise
    pins = (Q.test_quant_noise_closed_form_mxfp4_block,
            Q.test_quant_noise_zero_for_representable_blocks,
            Q.test_quant_noise_matches_independent_decode_nvfp4)

    def no_sdec(x, codes, scales, s_dec, block=(1, 16), e8m0=False):
        return orig(x, codes, scales, 1.0, block, e8m0)

    def abs_error(x, codes, scales, s_dec, block=(1, 16), e8m0=False):
        x = np.asarray(x, dtype=np.float64)
        d = O.dequantize(codes, scales, block, e8m0) * float(s_dec) - x
        return float(np.sum(x * x)), float(np.sum(np.abs(d)))

    def signal_of_deq(x, codes, scales, s_dec, block=(1, 16), e8m0=False):
        deq = O.dequantize(codes, scales, block, e8m0) * float(s_dec)
        d = deq - np.asarray(x, dtype=np.float64)
        return float(np.sum(deq * deq)), float(np.sum(d * d))

    for mutant in (no_sdec, abs_error, signal_of_deq):
        monkeypatch.setattr(O, "quant_noise", mutant)
        assert any(_fails(p) for p in pins), mutant.__name__
    monkeypatch.setattr(O, "quant_noise", orig)
    for p in pins:
        p()
