/*
 * fp4_oracle.c -- plain CPU oracle for the FP4 fully-quantized linear layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this library.  It shares no code,
 * header, table or constant generator with the CUDA path; every definition
 * below is written out from the format and method descriptions it cites.
 *
 * Sources (page title, section):
 *   [FP4]      "FP4" (Robots Atlas): How it works; Components (E2M1 format,
 *              NVFP4, MXFP4, Block scaling); Hyperparameters (format variant,
 *              scaling block size, scale factor format); Execution paradigm.
 *   [FQT]      "FP4 All the Way: Fully Quantized Training of LLMs": Key points
 *              and Summary (NVFP4; round-to-nearest forward, stochastic
 *              rounding in backward and update passes).
 *   [Quartet]  "Quartet: Native FP4 Training Can Be Optimal for Large Language
 *              Models": Approach (block-wise Hadamard rotations, RTN backward).
 *   Philox4x32-10: Salmon, Moraes, Dror, Shaw, "Parallel Random Numbers: As
 *              Easy as 1, 2, 3", SC'11 (the published counter-based generator).
 *
 * Points where the pages are silent are resolved by the readings listed in
 * the repository's design notes; each is marked "reading:" below.
 *
 * Arithmetic rules: every float operation written as `float` is one IEEE-754
 * binary32 operation rounded to nearest-even (built with -ffp-contract=off, no
 * fast-math, SSE arithmetic).  Searches over code tables are done in double,
 * where every compared quantity is exact.
 *
 * Slow and obvious on purpose: encoders search the whole code table.
 */
#include <math.h>
#include <float.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

/* ------------------------------------------------------------------------ */
/* Threading: split a row range over worker threads (no arithmetic here).   */
/* ------------------------------------------------------------------------ */
static int g_threads = 0;

int orc_set_threads(int n) { g_threads = n; return n; }

int orc_num_threads(void) {
  if (g_threads > 0) return g_threads;
  long n = sysconf(_SC_NPROCESSORS_ONLN);
  return n > 0 ? (int)n : 1;
}

typedef void (*row_fn)(void* ctx, int64_t r0, int64_t r1);
typedef struct { row_fn fn; void* ctx; int64_t r0, r1; } job_t;

static void* job_main(void* p) {
  job_t* j = (job_t*)p;
  j->fn(j->ctx, j->r0, j->r1);
  return NULL;
}

static void parallel_rows(row_fn fn, void* ctx, int64_t nrows) {
  int nt = orc_num_threads();
  if (nt > 64) nt = 64;
  if ((int64_t)nt > nrows) nt = (int)(nrows > 0 ? nrows : 1);
  if (nt <= 1) { fn(ctx, 0, nrows); return; }
  pthread_t th[64];
  job_t jobs[64];
  int64_t per = (nrows + nt - 1) / nt;
  int started = 0;
  for (int t = 0; t < nt; ++t) {
    int64_t a = (int64_t)t * per, b = a + per;
    if (a >= nrows) break;
    if (b > nrows) b = nrows;
    jobs[t].fn = fn; jobs[t].ctx = ctx; jobs[t].r0 = a; jobs[t].r1 = b;
    if (pthread_create(&th[t], NULL, job_main, &jobs[t]) != 0) {
      fn(ctx, a, b);             /* could not start a thread: do it inline */
      jobs[t].fn = NULL;
    }
    started = t + 1;
  }
  for (int t = 0; t < started; ++t)
    if (jobs[t].fn) pthread_join(th[t], NULL);
}

/* ------------------------------------------------------------------------ */
/* E2M1: sign in bit 3, a two-bit exponent in bits 2-1, mantissa in bit 0.  */
/* [FP4] Components, "E2M1 format": eight magnitudes 0, 0.5, 1, 1.5, 2, 3, */
/* 4, 6, each with either sign, so the format spans +-6.                    */
/* ------------------------------------------------------------------------ */
double orc_e2m1_value(uint8_t code) {
  int s = (code >> 3) & 1, e = (code >> 1) & 3, m = code & 1;
  double mag = (e == 0) ? 0.5 * m : ldexp(1.0 + 0.5 * m, e - 1);
  return s ? -mag : mag;
}

/* Round to nearest E2M1 level.  Ties go to the level whose mantissa bit is 0
 * (ties-to-even).  Magnitudes beyond 6 saturate to 6 (E2M1 has no Inf/NaN).
 * reading: a negative input that rounds to zero keeps its sign (code 8). */
uint8_t orc_e2m1_rtn(float v) {
  double a = fabs((double)v);
  /* Saturate first: beyond 6 the answer is 6, and below 8 every distance
   * computed in the search is exact in double. */
  if (a > 8.0) a = 8.0;
  int best = 0;
  double bestd = INFINITY;
  for (int c = 0; c < 8; ++c) {
    double d = fabs(a - orc_e2m1_value((uint8_t)c));
    if (d < bestd || (d == bestd && (c & 1) == 0 && (best & 1) == 1)) {
      bestd = d; best = c;
    }
  }
  return (uint8_t)(best | (signbit(v) ? 8 : 0));
}

/* Stochastic rounding to E2M1 with one 16-bit uniform draw u (0 .. 65535).
 * [FQT] stochastic rounding in the backward and update passes;
 * [FP4] "stochastic rounding of gradients".
 * reading: with lo <= |v| <= hi the neighbouring levels (|v| first clamped to
 * 6) and p = (|v| - lo) / (hi - lo), round up iff floor(p * 2^16) + u >= 2^16.
 * Over the 2^16 equally likely draws the value rounds up with probability
 * floor(p * 2^16) / 2^16: p truncated to 16 bits, so the expected result
 * lies within (hi - lo) * 2^-16 below |v| (never above it). */
uint8_t orc_e2m1_sr(float v, uint16_t u) {
  double a = fabs((double)v);
  if (a > 6.0) a = 6.0;
  int lo = 0, hi = 7;
  for (int c = 0; c < 8; ++c) {
    double lv = orc_e2m1_value((uint8_t)c);
    if (lv <= a) lo = c;
  }
  for (int c = 7; c >= 0; --c) {
    double lv = orc_e2m1_value((uint8_t)c);
    if (lv >= a) hi = c;
  }
  int code;
  if (lo == hi) {
    code = lo;
  } else {
    double l = orc_e2m1_value((uint8_t)lo), h = orc_e2m1_value((uint8_t)hi);
    double p = (a - l) / (h - l);                 /* exact: power-of-two gap */
    uint32_t k = (uint32_t)floor(ldexp(p, 16));   /* exact: p has <= 26 bits */
    code = (k + (uint32_t)u >= 65536u) ? hi : lo;
  }
  return (uint8_t)(code | (signbit(v) ? 8 : 0));
}

/* ------------------------------------------------------------------------ */
/* E4M3 (FP8, bias 7, no infinities, S.1111.111 is NaN; max 448), the NVFP4 */
/* block scale.  [FP4] Components, "NVFP4": E4M3 FP8 scale per 16 values.   */
/* ------------------------------------------------------------------------ */
double orc_e4m3_value(uint8_t code) {
  int s = (code >> 7) & 1, e = (code >> 3) & 15, m = code & 7;
  double mag;
  if (e == 15 && m == 7) return NAN;
  if (e == 0) mag = ldexp((double)m / 8.0, -6);
  else mag = ldexp(1.0 + (double)m / 8.0, e - 7);
  return s ? -mag : mag;
}

/* Encode a non-negative value: nearest of the 127 finite non-negative codes,
 * ties to the code with an even mantissa, anything above 448 saturates to
 * 448 (satfinite).  reading: the scale is rounded to nearest-even. */
uint8_t orc_e4m3_rne_sat(float t) {
  if (isnan(t)) return 0x7F;
  double a = (double)t;
  if (a < 0) a = 0;                 /* scales are magnitudes */
  if (a > 448.0) return 0x7E;       /* satfinite; below it the search is exact */
  int best = 0;
  double bestd = INFINITY;
  for (int c = 0; c < 0x7F; ++c) {
    double d = fabs(a - orc_e4m3_value((uint8_t)c));
    if (d < bestd || (d == bestd && (c & 1) == 0 && (best & 1) == 1)) {
      bestd = d; best = c;
    }
  }
  return (uint8_t)best;
}

/* ------------------------------------------------------------------------ */
/* E8M0: unsigned power-of-two scale 2^(b-127); 0xFF is NaN.                */
/* [FP4] Components, "MXFP4": one E8M0 scale per 32-value block, which can  */
/* only be a power of two.                                                  */
/* ------------------------------------------------------------------------ */
double orc_e8m0_value(uint8_t b) {
  if (b == 0xFF) return NAN;
  return ldexp(1.0, (int)b - 127);
}

/* floor(log2 b) for finite b > 0, read exactly from the binary32 encoding
 * (subnormals normalised). */
int orc_floor_log2(float b) {
  uint32_t bits;
  memcpy(&bits, &b, 4);
  int E = (int)((bits >> 23) & 0xFF);
  uint32_t man = bits & 0x7FFFFF;
  if (E > 0) return E - 127;
  int k = 31;
  while (k >= 0 && !((man >> k) & 1u)) --k;   /* man > 0 for b > 0 */
  return k - 149;
}

/* ------------------------------------------------------------------------ */
/* Philox4x32-10 (Salmon et al., SC'11).                                    */
/* Round: two 32x32->64 products of counter words 0 and 2 with the round    */
/* multipliers; outputs mix the high halves with the other two counter      */
/* words and the key; the key is bumped by the Weyl constants between       */
/* rounds.                                                                  */
/* ------------------------------------------------------------------------ */
#define PHILOX_M0 0xD2511F53u
#define PHILOX_M1 0xCD9E8D57u
#define PHILOX_W0 0x9E3779B9u
#define PHILOX_W1 0xBB67AE85u

void orc_philox4x32_10(const uint32_t ctr_in[4], const uint32_t key_in[2],
                       uint32_t out[4]) {
  uint32_t c0 = ctr_in[0], c1 = ctr_in[1], c2 = ctr_in[2], c3 = ctr_in[3];
  uint32_t k0 = key_in[0], k1 = key_in[1];
  for (int round = 0; round < 10; ++round) {
    if (round > 0) { k0 += PHILOX_W0; k1 += PHILOX_W1; }
    uint64_t p0 = (uint64_t)PHILOX_M0 * (uint64_t)c0;
    uint64_t p1 = (uint64_t)PHILOX_M1 * (uint64_t)c2;
    uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
    uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
    uint32_t n0 = hi1 ^ c1 ^ k0;
    uint32_t n1 = lo1;
    uint32_t n2 = hi0 ^ c3 ^ k1;
    uint32_t n3 = lo0;
    c0 = n0; c1 = n1; c2 = n2; c3 = n3;
  }
  out[0] = c0; out[1] = c1; out[2] = c2; out[3] = c3;
}

/* The draw for element i of a stream: reading: key = (seed lo, seed hi),
 * counter = (c lo, c hi, stream, 0) with c = i / 4; word i mod 4. */
uint32_t orc_draw(uint64_t seed, uint32_t stream, uint64_t i) {
  uint64_t c = i >> 2;
  uint32_t ctr[4] = {(uint32_t)c, (uint32_t)(c >> 32), stream, 0u};
  uint32_t key[2] = {(uint32_t)seed, (uint32_t)(seed >> 32)};
  uint32_t out[4];
  orc_philox4x32_10(ctr, key, out);
  return out[i & 3];
}

/* The 16-bit draw of element i of a stream, for stochastic rounding.
 * reading: the low (i even) or high (i odd) half of the 32-bit draw i / 2,
 * so one Philox block (counter i / 8) serves eight consecutive elements. */
uint16_t orc_draw16(uint64_t seed, uint32_t stream, uint64_t i) {
  uint32_t w = orc_draw(seed, stream, i >> 1);
  return (uint16_t)((i & 1) ? (w >> 16) : (w & 0xFFFFu));
}

/* ------------------------------------------------------------------------ */
/* Block-wise random Hadamard transform.                                    */
/* [FP4] How it works / pitfalls: random Hadamard transforms tame outliers; */
/* [Quartet] Approach: block-wise Hadamard rotations.                       */
/* reading: y = c_n * (x .* d) * H_n on each n-block of the contraction     */
/* dimension; H_n the Sylvester +-1 matrix (natural order); d_j = -1 iff    */
/* bit 31 of draw j of stream RHT_STREAM is set; c_n = RN(1/sqrt(n)).       */
/* ------------------------------------------------------------------------ */
#define RHT_STREAM 0x48414441u

void orc_rht_signs(uint64_t seed, int n, float* d) {
  for (int j = 0; j < n; ++j)
    d[j] = (orc_draw(seed, RHT_STREAM, (uint64_t)j) >> 31) ? -1.0f : 1.0f;
}

float orc_rht_scale(int n) { return (float)(1.0 / sqrt((double)n)); }

/* In place on one block of n values: sign flip, then the butterfly
 * (a, b) -> (a + b, a - b) over strides 1, 2, 4, ..., n/2, then scale. */
void orc_rht_block(float* v, int n, const float* d) {
  for (int j = 0; j < n; ++j) v[j] = v[j] * d[j];
  for (int h = 1; h < n; h <<= 1) {
    for (int j = 0; j < n; ++j) {
      if (j & h) continue;
      float a = v[j], b = v[j + h];
      v[j] = a + b;
      v[j + h] = a - b;
    }
  }
  float c = orc_rht_scale(n);
  for (int j = 0; j < n; ++j) v[j] = v[j] * c;
}

/* Rotate every n-block of every row of x[R, C] (row-major) in place. */
void orc_rht_rows(float* x, int64_t R, int64_t C, int n, uint64_t seed) {
  float d[64];
  orc_rht_signs(seed, n, d);
  for (int64_t r = 0; r < R; ++r)
    for (int64_t c0 = 0; c0 < C; c0 += n) orc_rht_block(x + r * C + c0, n, d);
}

/* ------------------------------------------------------------------------ */
/* Tensor amax (exact: max is exact).                                       */
/* ------------------------------------------------------------------------ */
float orc_amax(const float* x, int64_t n) {
  float m = 0.0f;
  for (int64_t i = 0; i < n; ++i) {
    float a = fabsf(x[i]);
    if (a > m) m = a;
  }
  return m;
}

/* ------------------------------------------------------------------------ */
/* NVFP4 two-level scaling.  [FP4] How it works + Components "NVFP4":       */
/* 16-value blocks with an E4M3 scale, plus one FP32 scale per tensor.      */
/* reading: the tensor amax maps to the top of the two-level range          */
/* 6 * 448 = 2688: s_enc = RN(2688 / A) (largest finite float if that       */
/* overflows), s_dec = RN(A / 2688); A = 0 gives s_enc = s_dec = 1.         */
/* Block: t = RN(RN(b * s_enc) / 6), sf = E4M3(t), inv = RN(s_enc / sf)     */
/* (0 when sf = 0; the largest finite float if it overflows, which only a   */
/* block whose max is below ~1.8e-38 can cause), element v = RN(x * inv)    */
/* rounded to E2M1.                                                         */
/* ------------------------------------------------------------------------ */
void orc_nvfp4_global_scales(float A, float* s_enc, float* s_dec) {
  if (A == 0.0f) { *s_enc = 1.0f; *s_dec = 1.0f; return; }
  float e = 2688.0f / A;
  if (isinf(e)) e = FLT_MAX;
  *s_enc = e;
  *s_dec = A / 2688.0f;
}

typedef struct {
  const float* y;          /* values to quantize (already rotated) [R, C] */
  int64_t R, C, row_offset, bs;
  int round_mode;          /* 0 = RTN, 1 = SR */
  uint64_t sr_seed;
  uint32_t sr_stream;
  float s_enc;
  uint8_t* codes;          /* [R, C/2] */
  uint8_t* scales;         /* [R, C/bs] */
} q1d_ctx;

static void nvfp4_rows_worker(void* p, int64_t r0, int64_t r1) {
  q1d_ctx* q = (q1d_ctx*)p;
  const int64_t C = q->C, nb = C / 16;
  for (int64_t r = r0; r < r1; ++r) {
    const float* row = q->y + r * C;
    for (int64_t b = 0; b < nb; ++b) {
      float bmax = 0.0f;
      for (int j = 0; j < 16; ++j) {
        float a = fabsf(row[b * 16 + j]);
        if (a > bmax) bmax = a;
      }
      float t = (bmax * q->s_enc) / 6.0f;
      uint8_t sf = orc_e4m3_rne_sat(t);
      float sfv = (float)orc_e4m3_value(sf);
      float inv = (sf == 0) ? 0.0f : q->s_enc / sfv;
      if (isinf(inv)) inv = FLT_MAX;   /* reading: the reciprocal saturates */
      q->scales[r * nb + b] = sf;
      for (int j = 0; j < 16; ++j) {
        int64_t c = b * 16 + j;
        float v = row[c] * inv;
        uint8_t code;
        if (q->round_mode == 0) {
          code = orc_e2m1_rtn(v);
        } else {
          uint64_t idx = (uint64_t)(q->row_offset + r) * (uint64_t)C + (uint64_t)c;
          code = orc_e2m1_sr(v, orc_draw16(q->sr_seed, q->sr_stream, idx));
        }
        uint8_t* byte = &q->codes[r * (C / 2) + c / 2];
        if ((c & 1) == 0) *byte = (uint8_t)((*byte & 0xF0) | code);
        else *byte = (uint8_t)((*byte & 0x0F) | (code << 4));
      }
    }
  }
}

/* NVFP4 1x16 quantization of x[R, C] (rows R of a tensor whose first row is
 * row `row_offset`; the stochastic-rounding draw of element (r, c) is
 * draw(sr_seed, sr_stream, (row_offset + r) * C + c)).
 * rht_n in {0, 16}: rotate each 16-block of each row first.
 * amax_in: if non-NULL, the tensor amax to use (otherwise computed here).
 * Returns 0, or -1 for bad sizes. */
int orc_nvfp4_quantize_1d(const float* x, int64_t R, int64_t C, int64_t row_offset,
                          int round_mode, int rht_n, uint64_t rht_seed,
                          uint64_t sr_seed, uint32_t sr_stream, const float* amax_in,
                          uint8_t* codes, uint8_t* scales, float* amax_out,
                          float* s_dec_out) {
  if (R < 0 || C < 0 || C % 16) return -1;
  if (!(rht_n == 0 || rht_n == 16 || rht_n == 32) || (rht_n && C % rht_n)) return -1;
  float* y = (float*)malloc(sizeof(float) * (size_t)(R * C > 0 ? R * C : 1));
  if (!y) return -2;
  memcpy(y, x, sizeof(float) * (size_t)(R * C));
  if (rht_n) orc_rht_rows(y, R, C, rht_n, rht_seed);
  float A = amax_in ? *amax_in : orc_amax(y, R * C);
  float s_enc, s_dec;
  orc_nvfp4_global_scales(A, &s_enc, &s_dec);
  memset(codes, 0, (size_t)(R * C / 2));
  q1d_ctx q = {y, R, C, row_offset, 16, round_mode, sr_seed, sr_stream, s_enc,
               codes, scales};
  parallel_rows(nvfp4_rows_worker, &q, R);
  if (amax_out) *amax_out = A;
  if (s_dec_out) *s_dec_out = s_dec;
  free(y);
  return 0;
}

/* NVFP4 16x16 2-D quantization (weights, round to nearest).
 * [FP4] How it works: "two-dimensional quantization" as a stabiliser; the
 * 16x16 tile is the 2-D analogue of the 16-value block.  One E4M3 scale per
 * 16x16 tile, scales laid out [R/16, C/16]; codes [R, C/2] as in 1-D. */
typedef struct {
  const float* x;
  int64_t R, C;
  float s_enc;
  uint8_t* codes;
  uint8_t* scales;
} q2d_ctx;

/* Tile rows [t0, t1) of the 16x16 grid. */
static void nvfp4_2d_worker(void* p, int64_t t0, int64_t t1) {
  q2d_ctx* q = (q2d_ctx*)p;
  const int64_t C = q->C, tc = C / 16;
  for (int64_t i = t0; i < t1; ++i) {
    for (int64_t j = 0; j < tc; ++j) {
      float bmax = 0.0f;
      for (int a = 0; a < 16; ++a)
        for (int b = 0; b < 16; ++b) {
          float v = fabsf(q->x[(i * 16 + a) * C + j * 16 + b]);
          if (v > bmax) bmax = v;
        }
      float t = (bmax * q->s_enc) / 6.0f;
      uint8_t sf = orc_e4m3_rne_sat(t);
      float sfv = (float)orc_e4m3_value(sf);
      float inv = (sf == 0) ? 0.0f : q->s_enc / sfv;
      if (isinf(inv)) inv = FLT_MAX;   /* reading: the reciprocal saturates */
      q->scales[i * tc + j] = sf;
      for (int a = 0; a < 16; ++a)
        for (int b = 0; b < 16; ++b) {
          int64_t r = i * 16 + a, c = j * 16 + b;
          uint8_t code = orc_e2m1_rtn(q->x[r * C + c] * inv);
          uint8_t* byte = &q->codes[r * (C / 2) + c / 2];
          if ((c & 1) == 0) *byte = (uint8_t)((*byte & 0xF0) | code);
          else *byte = (uint8_t)((*byte & 0x0F) | (code << 4));
        }
    }
  }
}

/* NVFP4 16x16 2-D quantization (weights, round to nearest).
 * [FP4] How it works: "two-dimensional quantization" as a stabiliser; the
 * 16x16 tile is the 2-D analogue of the 16-value block.  One E4M3 scale per
 * 16x16 tile, scales laid out [R/16, C/16]; codes [R, C/2] as in 1-D. */
int orc_nvfp4_quantize_2d(const float* x, int64_t R, int64_t C, const float* amax_in,
                          uint8_t* codes, uint8_t* scales, float* amax_out,
                          float* s_dec_out) {
  if (R < 0 || C < 0 || R % 16 || C % 16) return -1;
  float A = amax_in ? *amax_in : orc_amax(x, R * C);
  float s_enc, s_dec;
  orc_nvfp4_global_scales(A, &s_enc, &s_dec);
  memset(codes, 0, (size_t)(R * C / 2));
  q2d_ctx q = {x, R, C, s_enc, codes, scales};
  parallel_rows(nvfp4_2d_worker, &q, R / 16);
  if (amax_out) *amax_out = A;
  if (s_dec_out) *s_dec_out = s_dec;
  return 0;
}

/* ------------------------------------------------------------------------ */
/* MXFP4: 32-value blocks, one E8M0 scale, no tensor scale.                 */
/* [FP4] Components "MXFP4" and Hyperparameters (block 32, E8M0).           */
/* reading (OCP MX rule): e = floor(log2 b) - 2 (2 = E2M1's largest         */
/* exponent), clamped to [-127, 127]; scale byte e + 127; v = x * 2^-e,     */
/* then E2M1 rounding (values in (6, 8) saturate); b = 0 gives scale byte 0 */
/* and zero codes.                                                          */
/* ------------------------------------------------------------------------ */
/* ------------------------------------------------------------------------ */
/* QuEST-style MXFP4 forward block scale.  [Quartet] Approach and Measured  */
/* effects (ablations): the forward pass uses a QuEST-style quantizer --     */
/* Hadamard rotation, then clipping -- instead of plain round-to-nearest.   */
/* The pages give no clipping rule.  reading: the block's scale comes from  */
/* its root-mean-square instead of its maximum: T = RN(alpha * RMS), with   */
/* alpha the clipping multiple that minimises the mean squared error of     */
/* E2M1 round-to-nearest for a unit Gaussian (values beyond alpha clip to   */
/* the top level), and the OCP MX power-of-two rule applied to T in place   */
/* of the block max: e = floor(log2 T) - 2, clamped to [-127, 127]; values  */
/* whose scaled magnitude exceeds 6 saturate (the clipping).  T = 0 gives   */
/* scale byte 0 and zero codes, as a zero block does.                       */
/* The mean square of the 32 values is summed in binary32 in a fixed tree:  */
/* four groups of 8 consecutive values, each ((y0^2 + y1^2) + (y2^2 +       */
/* y3^2)) + ((y4^2 + y5^2) + (y6^2 + y7^2)), then (g0 + g1) + (g2 + g3);    */
/* RMS = RN(sqrt(RN(sum / 32))).                                            */
/* ------------------------------------------------------------------------ */
#define QUEST_ALPHA 2.9224751f

float orc_quest_threshold(const float* y) {
  float g[4];
  for (int k = 0; k < 4; ++k) {
    const float* v = y + 8 * k;
    float a = v[0] * v[0] + v[1] * v[1];
    float b = v[2] * v[2] + v[3] * v[3];
    float c = v[4] * v[4] + v[5] * v[5];
    float d = v[6] * v[6] + v[7] * v[7];
    g[k] = (a + b) + (c + d);
  }
  float sum = (g[0] + g[1]) + (g[2] + g[3]);
  float rms = sqrtf(sum / 32.0f);
  return QUEST_ALPHA * rms;
}

float orc_quest_alpha(void) { return QUEST_ALPHA; }

static void mxfp4_rows_worker(void* p, int64_t r0, int64_t r1) {
  q1d_ctx* q = (q1d_ctx*)p;
  const int64_t C = q->C, nb = C / 32;
  for (int64_t r = r0; r < r1; ++r) {
    const float* row = q->y + r * C;
    for (int64_t b = 0; b < nb; ++b) {
      float bmax = 0.0f;
      for (int j = 0; j < 32; ++j) {
        float a = fabsf(row[b * 32 + j]);
        if (a > bmax) bmax = a;
      }
      /* round_mode 2 (QuEST): the clipping threshold replaces the block max */
      float top = (q->round_mode == 2) ? orc_quest_threshold(row + b * 32) : bmax;
      int e = (top == 0.0f) ? -127 : orc_floor_log2(top) - 2;
      if (e < -127) e = -127;
      if (e > 127) e = 127;
      q->scales[r * nb + b] = (uint8_t)(e + 127);
      float mul = (float)ldexp(1.0, -e);          /* exact power of two */
      for (int j = 0; j < 32; ++j) {
        int64_t c = b * 32 + j;
        float v = row[c] * mul;
        uint8_t code;
        if (q->round_mode != 1) {
          code = orc_e2m1_rtn(v);
        } else {
          uint64_t idx = (uint64_t)(q->row_offset + r) * (uint64_t)C + (uint64_t)c;
          code = orc_e2m1_sr(v, orc_draw16(q->sr_seed, q->sr_stream, idx));
        }
        uint8_t* byte = &q->codes[r * (C / 2) + c / 2];
        if ((c & 1) == 0) *byte = (uint8_t)((*byte & 0xF0) | code);
        else *byte = (uint8_t)((*byte & 0x0F) | (code << 4));
      }
    }
  }
}

int orc_mxfp4_quantize(const float* x, int64_t R, int64_t C, int64_t row_offset,
                       int round_mode, int rht_n, uint64_t rht_seed, uint64_t sr_seed,
                       uint32_t sr_stream, uint8_t* codes, uint8_t* scales) {
  if (R < 0 || C < 0 || C % 32) return -1;
  if (!(rht_n == 0 || rht_n == 16 || rht_n == 32) || (rht_n && C % rht_n)) return -1;
  float* y = (float*)malloc(sizeof(float) * (size_t)(R * C > 0 ? R * C : 1));
  if (!y) return -2;
  memcpy(y, x, sizeof(float) * (size_t)(R * C));
  if (rht_n) orc_rht_rows(y, R, C, rht_n, rht_seed);
  memset(codes, 0, (size_t)(R * C / 2));
  q1d_ctx q = {y, R, C, row_offset, 32, round_mode, sr_seed, sr_stream, 1.0f,
               codes, scales};
  parallel_rows(mxfp4_rows_worker, &q, R);
  free(y);
  return 0;
}

/* ------------------------------------------------------------------------ */
/* Dequantization (exact in double).  The NVFP4 tensor scale s_dec is NOT   */
/* applied here: x_hat = e2m1(code) * value(scale), so that GEMM products   */
/* of two such values stay exact; callers multiply by s_dec afterwards.     */
/* block_rows x block_cols is the area one scale covers: 1x16 (NVFP4 1-D),  */
/* 16x16 (NVFP4 2-D), 1x32 (MXFP4, E8M0 scales when is_e8m0).               */
/* ------------------------------------------------------------------------ */
void orc_dequantize(const uint8_t* codes, const uint8_t* scales, int64_t R, int64_t C,
                    int block_rows, int block_cols, int is_e8m0, double* out) {
  const int64_t sc = C / block_cols;
  for (int64_t r = 0; r < R; ++r) {
    for (int64_t c = 0; c < C; ++c) {
      uint8_t byte = codes[r * (C / 2) + c / 2];
      uint8_t code = (c & 1) ? (uint8_t)(byte >> 4) : (uint8_t)(byte & 0xF);
      uint8_t s = scales[(r / block_rows) * sc + c / block_cols];
      double sv = is_e8m0 ? orc_e8m0_value(s) : orc_e4m3_value(s);
      out[r * C + c] = orc_e2m1_value(code) * sv;
    }
  }
}

/* ------------------------------------------------------------------------ */
/* Array forms of the scalar definitions above (loops only), for tests.     */
/* ------------------------------------------------------------------------ */
void orc_e2m1_rtn_n(const float* v, int64_t n, uint8_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = orc_e2m1_rtn(v[i]);
}
void orc_e2m1_sr_n(const float* v, const uint16_t* u, int64_t n, uint8_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = orc_e2m1_sr(v[i], u[i]);
}
void orc_e4m3_rne_sat_n(const float* t, int64_t n, uint8_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = orc_e4m3_rne_sat(t[i]);
}
void orc_draw_n(uint64_t seed, uint32_t stream, uint64_t i0, int64_t n, uint32_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = orc_draw(seed, stream, i0 + (uint64_t)i);
}
void orc_draw16_n(uint64_t seed, uint32_t stream, uint64_t i0, int64_t n, uint16_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = orc_draw16(seed, stream, i0 + (uint64_t)i);
}
