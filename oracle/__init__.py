"""CPU oracle for the FP4 fully-quantized linear layer (TEST INFRASTRUCTURE).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path never does: it has
its own CUDA implementation and shares no code with this one.

The arithmetic lives in ``fp4_oracle.c`` (plain C, IEEE binary32, no FMA
contraction); this module only marshals numpy arrays through ctypes.  The
GEMM reference is a float64 matrix product (numpy ``@``) of the exactly
dequantized operands, scaled afterwards by ``alpha * s_dec(a) * s_dec(b)``
(the "FP4" page of Robots Atlas, How it works: the products are formed from
FP4 operands and summed at a wider precision).

Parity status of each function is recorded in the repository's design notes;
the Philox generator is pinned block for block against an independent
Philox4x32-10, cuRAND's host generator, besides its statistical checks.
"""
from __future__ import annotations

import ctypes as C
import os

import numpy as np

from . import build as _build

RHT_STREAM = 0x48414441

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = C.CDLL(path)
        f32p = np.ctypeslib.ndpointer(np.float32, flags="C_CONTIGUOUS")
        u8p = np.ctypeslib.ndpointer(np.uint8, flags="C_CONTIGUOUS")
        u32p = np.ctypeslib.ndpointer(np.uint32, flags="C_CONTIGUOUS")
        f64p = np.ctypeslib.ndpointer(np.float64, flags="C_CONTIGUOUS")
        u16p = np.ctypeslib.ndpointer(np.uint16, flags="C_CONTIGUOUS")
        i64, u64, u32, i32 = C.c_int64, C.c_uint64, C.c_uint32, C.c_int
        L.orc_e2m1_value.restype = C.c_double
        L.orc_e2m1_value.argtypes = [C.c_uint8]
        L.orc_e4m3_value.restype = C.c_double
        L.orc_e4m3_value.argtypes = [C.c_uint8]
        L.orc_e8m0_value.restype = C.c_double
        L.orc_e8m0_value.argtypes = [C.c_uint8]
        L.orc_e2m1_rtn.restype = C.c_uint8
        L.orc_e2m1_rtn.argtypes = [C.c_float]
        L.orc_e2m1_sr.restype = C.c_uint8
        L.orc_e2m1_sr.argtypes = [C.c_float, C.c_uint16]
        L.orc_e4m3_rne_sat.restype = C.c_uint8
        L.orc_e4m3_rne_sat.argtypes = [C.c_float]
        L.orc_floor_log2.restype = C.c_int
        L.orc_floor_log2.argtypes = [C.c_float]
        L.orc_philox4x32_10.restype = None
        L.orc_philox4x32_10.argtypes = [u32p, u32p, u32p]
        L.orc_draw.restype = u32
        L.orc_draw.argtypes = [u64, u32, u64]
        L.orc_draw_n.restype = None
        L.orc_draw_n.argtypes = [u64, u32, u64, i64, u32p]
        L.orc_draw16.restype = C.c_uint16
        L.orc_draw16.argtypes = [u64, u32, u64]
        L.orc_draw16_n.restype = None
        L.orc_draw16_n.argtypes = [u64, u32, u64, i64, u16p]
        L.orc_e2m1_rtn_n.restype = None
        L.orc_e2m1_rtn_n.argtypes = [f32p, i64, u8p]
        L.orc_e2m1_sr_n.restype = None
        L.orc_e2m1_sr_n.argtypes = [f32p, u16p, i64, u8p]
        L.orc_e4m3_rne_sat_n.restype = None
        L.orc_e4m3_rne_sat_n.argtypes = [f32p, i64, u8p]
        L.orc_rht_signs.restype = None
        L.orc_rht_signs.argtypes = [u64, i32, f32p]
        L.orc_rht_scale.restype = C.c_float
        L.orc_rht_scale.argtypes = [i32]
        L.orc_rht_block.restype = None
        L.orc_rht_block.argtypes = [f32p, i32, f32p]
        L.orc_rht_rows.restype = None
        L.orc_rht_rows.argtypes = [f32p, i64, i64, i32, u64]
        L.orc_amax.restype = C.c_float
        L.orc_amax.argtypes = [f32p, i64]
        L.orc_nvfp4_global_scales.restype = None
        L.orc_nvfp4_global_scales.argtypes = [C.c_float, C.POINTER(C.c_float),
                                              C.POINTER(C.c_float)]
        L.orc_nvfp4_quantize_1d.restype = i32
        L.orc_nvfp4_quantize_1d.argtypes = [f32p, i64, i64, i64, i32, i32, u64, u64, u32,
                                            C.c_void_p, u8p, u8p, C.POINTER(C.c_float),
                                            C.POINTER(C.c_float)]
        L.orc_nvfp4_quantize_2d.restype = i32
        L.orc_nvfp4_quantize_2d.argtypes = [f32p, i64, i64, C.c_void_p, u8p, u8p,
                                            C.POINTER(C.c_float), C.POINTER(C.c_float)]
        L.orc_mxfp4_quantize.restype = i32
        L.orc_mxfp4_quantize.argtypes = [f32p, i64, i64, i64, i32, i32, u64, u64, u32,
                                         u8p, u8p]
        L.orc_dequantize.restype = None
        L.orc_dequantize.argtypes = [u8p, u8p, i64, i64, i32, i32, i32, f64p]
        L.orc_quest_threshold.restype = C.c_float
        L.orc_quest_threshold.argtypes = [f32p]
        L.orc_quest_alpha.restype = C.c_float
        L.orc_quest_alpha.argtypes = []
        L.orc_set_threads.restype = i32
        L.orc_set_threads.argtypes = [i32]
        L.orc_num_threads.restype = i32
        L.orc_num_threads.argtypes = []
        _lib = L
    return _lib


def _f32(x) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(x, dtype=np.float32))


# --------------------------------------------------------------------------
# scalar / elementwise definitions
# --------------------------------------------------------------------------
def e2m1_value(code: int) -> float:
    return lib().orc_e2m1_value(int(code) & 0xFF)


def e4m3_value(code: int) -> float:
    return lib().orc_e4m3_value(int(code) & 0xFF)


def e8m0_value(code: int) -> float:
    return lib().orc_e8m0_value(int(code) & 0xFF)


def floor_log2(b: float) -> int:
    return lib().orc_floor_log2(float(np.float32(b)))


def e2m1_rtn(v) -> np.ndarray:
    v = _f32(v).reshape(-1)
    out = np.empty(v.size, np.uint8)
    lib().orc_e2m1_rtn_n(v, v.size, out)
    return out


def e2m1_sr(v, u) -> np.ndarray:
    """Stochastic E2M1 codes of v with 16-bit draws u (0 .. 65535)."""
    v = _f32(v).reshape(-1)
    u = np.asarray(u)
    assert u.size == 0 or (u.min() >= 0 and u.max() <= 0xFFFF), "draws are 16-bit"
    u = np.ascontiguousarray(u.astype(np.uint16).reshape(-1))
    assert u.size == v.size
    out = np.empty(v.size, np.uint8)
    lib().orc_e2m1_sr_n(v, u, v.size, out)
    return out


def e4m3_rne_sat(t) -> np.ndarray:
    t = _f32(t).reshape(-1)
    out = np.empty(t.size, np.uint8)
    lib().orc_e4m3_rne_sat_n(t, t.size, out)
    return out


def philox4x32_10(ctr, key) -> np.ndarray:
    c = np.ascontiguousarray(np.asarray(ctr, dtype=np.uint32))
    k = np.ascontiguousarray(np.asarray(key, dtype=np.uint32))
    out = np.empty(4, np.uint32)
    lib().orc_philox4x32_10(c, k, out)
    return out


def draws(seed: int, stream: int, i0: int, n: int) -> np.ndarray:
    """32-bit draws i0 .. i0 + n - 1 of a stream (word i mod 4 of block i / 4)."""
    out = np.empty(n, np.uint32)
    lib().orc_draw_n(seed, stream, i0, n, out)
    return out


def draws16(seed: int, stream: int, i0: int, n: int) -> np.ndarray:
    """16-bit stochastic-rounding draws i0 .. i0 + n - 1 of a stream."""
    out = np.empty(n, np.uint16)
    lib().orc_draw16_n(seed, stream, i0, n, out)
    return out


def rht_signs(seed: int, n: int) -> np.ndarray:
    d = np.empty(n, np.float32)
    lib().orc_rht_signs(seed, n, d)
    return d


def rht_scale(n: int) -> float:
    return lib().orc_rht_scale(n)


def rht_block(v, n: int, signs) -> np.ndarray:
    v = _f32(v).copy()
    lib().orc_rht_block(v, n, _f32(signs))
    return v


def rht_rows(x, n: int, seed: int) -> np.ndarray:
    y = _f32(x).copy()
    R, Cc = y.shape
    lib().orc_rht_rows(y, R, Cc, n, seed)
    return y


def amax(x) -> float:
    x = _f32(x).reshape(-1)
    return float(lib().orc_amax(x, x.size))


def nvfp4_global_scales(A: float):
    e, d = C.c_float(), C.c_float()
    lib().orc_nvfp4_global_scales(float(np.float32(A)), C.byref(e), C.byref(d))
    return np.float32(e.value), np.float32(d.value)


# --------------------------------------------------------------------------
# quantizers
# --------------------------------------------------------------------------
def _amax_arg(amax_in):
    if amax_in is None:
        return None, None
    buf = np.array([amax_in], dtype=np.float32)
    return buf.ctypes.data_as(C.c_void_p), buf


def nvfp4_quantize_1d(x, round_mode: str = "rtn", rht_n: int = 0, rht_seed: int = 0,
                      sr_seed: int = 0, sr_stream: int = 0, amax_in=None,
                      row_offset: int = 0) -> dict:
    """NVFP4 1x16 quantization of the rows of x (float32 [R, C])."""
    x = _f32(x)
    R, Cc = x.shape
    codes = np.zeros((R, Cc // 2), np.uint8)
    scales = np.zeros((R, Cc // 16), np.uint8)
    a, d = C.c_float(), C.c_float()
    ptr, _keep = _amax_arg(amax_in)
    rc = lib().orc_nvfp4_quantize_1d(x, R, Cc, row_offset, 0 if round_mode == "rtn" else 1,
                                     rht_n, rht_seed, sr_seed, sr_stream, ptr, codes, scales,
                                     C.byref(a), C.byref(d))
    if rc != 0:
        raise ValueError(f"oracle nvfp4_quantize_1d rejected shape {x.shape} rht_n={rht_n}")
    return {"codes": codes, "scales": scales, "amax": np.float32(a.value),
            "s_dec": np.float32(d.value)}


def nvfp4_quantize_2d(x, amax_in=None) -> dict:
    """NVFP4 16x16 2-D quantization (round to nearest) of x (float32 [R, C])."""
    x = _f32(x)
    R, Cc = x.shape
    codes = np.zeros((R, Cc // 2), np.uint8)
    scales = np.zeros((R // 16, Cc // 16), np.uint8)
    a, d = C.c_float(), C.c_float()
    ptr, _keep = _amax_arg(amax_in)
    rc = lib().orc_nvfp4_quantize_2d(x, R, Cc, ptr, codes, scales, C.byref(a), C.byref(d))
    if rc != 0:
        raise ValueError(f"oracle nvfp4_quantize_2d rejected shape {x.shape}")
    return {"codes": codes, "scales": scales, "amax": np.float32(a.value),
            "s_dec": np.float32(d.value)}


def quest_threshold(block) -> float:
    """The QuEST-style clipping threshold RN(alpha * RMS) of one 32-value
    block (binary32 tree sum of squares)."""
    b = _f32(block).reshape(-1)
    assert b.size == 32
    return float(lib().orc_quest_threshold(b))


def quest_alpha() -> float:
    return float(lib().orc_quest_alpha())


_MODES = {"rtn": 0, "sr": 1, "quest": 2}


def mxfp4_quantize(x, round_mode: str = "rtn", rht_n: int = 0, rht_seed: int = 0,
                   sr_seed: int = 0, sr_stream: int = 0, row_offset: int = 0) -> dict:
    """MXFP4 1x32 quantization of the rows of x (float32 [R, C]); round_mode
    "rtn", "sr", or "quest" (RMS-based clipping scale, then round to nearest)."""
    x = _f32(x)
    R, Cc = x.shape
    codes = np.zeros((R, Cc // 2), np.uint8)
    scales = np.zeros((R, Cc // 32), np.uint8)
    rc = lib().orc_mxfp4_quantize(x, R, Cc, row_offset, _MODES[round_mode],
                                  rht_n, rht_seed, sr_seed, sr_stream, codes, scales)
    if rc != 0:
        raise ValueError(f"oracle mxfp4_quantize rejected shape {x.shape} rht_n={rht_n}")
    return {"codes": codes, "scales": scales, "s_dec": np.float32(1.0)}


def dequantize(codes, scales, block=(1, 16), e8m0: bool = False) -> np.ndarray:
    """Exact float64 values e2m1(code) * scale (tensor scale NOT applied)."""
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint8)
    R, half = codes.shape
    out = np.empty((R, half * 2), np.float64)
    lib().orc_dequantize(codes, scales, R, half * 2, block[0], block[1], int(e8m0), out)
    return out


def quant_noise(x, codes, scales, s_dec: float, block=(1, 16), e8m0: bool = False):
    """(sum x^2, sum (deq - x)^2) in float64 for a tensor x and its
    quantization (codes, logical scales, per-tensor decode scale s_dec):
    deq = e2m1(code) * block scale * s_dec.  The gradient-norm and
    quantization-noise pair of the "FP4 All the Way" page (Summary), which
    states a threshold between them without giving its form."""
    x = np.asarray(x, dtype=np.float64)
    deq = dequantize(codes, scales, block, e8m0) * float(s_dec)
    d = deq - x
    return float(np.sum(x * x)), float(np.sum(d * d))


def gemm(a_hat: np.ndarray, b_hat: np.ndarray, alpha: float = 1.0, s_dec_a: float = 1.0,
         s_dec_b: float = 1.0) -> np.ndarray:
    """C = alpha * s_dec_a * s_dec_b * A_hat @ B_hat^T in float64.

    A_hat [M, K] and B_hat [N, K] are dequantized operands without their
    tensor scales (products of two such values are exact in float64)."""
    return (a_hat @ b_hat.T) * (float(alpha) * float(s_dec_a) * float(s_dec_b))


def set_threads(n: int) -> int:
    return lib().orc_set_threads(n)


def num_threads() -> int:
    return lib().orc_num_threads()
