// fp4_device.cuh -- device building blocks of the FP4 quantizers (sm_100a).
//
// Formats ("FP4", Robots Atlas, Components / Hyperparameters): E2M1 elements
// (levels 0, 0.5, 1, 1.5, 2, 3, 4, 6), NVFP4 = 16-value blocks with an E4M3
// scale and an FP32 tensor scale, MXFP4 = 32-value blocks with an E8M0 scale.
//
// Every floating-point step that decides a code is written with explicit
// round-to-nearest intrinsics (__fmul_rn, __fadd_rn, __fdiv_rn) so that the
// compiler cannot contract or reorder it; E2M1 and E4M3 round-to-nearest-even
// use the hardware cvt instructions.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>

namespace fp4dev {

// ---------------------------------------------------------------------------
// Philox4x32-10 (Salmon et al., SC'11), counter-based: draw i of a stream is
// word (i mod 4) of philox(counter = (i/4 lo, i/4 hi, stream, 0),
// key = (seed lo, seed hi)).
// ---------------------------------------------------------------------------
constexpr uint32_t kPhiloxM0 = 0xD2511F53u;
constexpr uint32_t kPhiloxM1 = 0xCD9E8D57u;
constexpr uint32_t kPhiloxW0 = 0x9E3779B9u;
constexpr uint32_t kPhiloxW1 = 0xBB67AE85u;
constexpr uint32_t kRhtStream = 0x48414441u;

struct U4 { uint32_t x, y, z, w; };

__host__ __device__ __forceinline__ U4 philox4x32_10(uint64_t ctr_lo64, uint32_t stream,
                                                     uint64_t seed) {
  uint32_t c0 = (uint32_t)ctr_lo64, c1 = (uint32_t)(ctr_lo64 >> 32), c2 = stream, c3 = 0;
  uint32_t k0 = (uint32_t)seed, k1 = (uint32_t)(seed >> 32);
#ifdef __CUDA_ARCH__
#pragma unroll
#endif
  for (int r = 0; r < 10; ++r) {
#ifdef __CUDA_ARCH__
    uint32_t hi0 = __umulhi(kPhiloxM0, c0), lo0 = kPhiloxM0 * c0;
    uint32_t hi1 = __umulhi(kPhiloxM1, c2), lo1 = kPhiloxM1 * c2;
#else
    uint64_t p0 = (uint64_t)kPhiloxM0 * c0, p1 = (uint64_t)kPhiloxM1 * c2;
    uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
    uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
#endif
    uint32_t n0 = hi1 ^ c1 ^ k0, n2 = hi0 ^ c3 ^ k1;
    c0 = n0; c1 = lo1; c2 = n2; c3 = lo0;
    k0 += kPhiloxW0; k1 += kPhiloxW1;
  }
  return U4{c0, c1, c2, c3};
}

// The same generator with its ten round keys precomputed (on the host, passed
// as a kernel parameter so they live in the constant bank, not in registers)
// and each 32x32 product done as one widening multiply (hi and lo together).
struct PhiloxKeys {
  uint32_t k0[10], k1[10];
};

__host__ __device__ __forceinline__ PhiloxKeys philox_keys(uint64_t seed) {
  PhiloxKeys K;
  uint32_t a = (uint32_t)seed, b = (uint32_t)(seed >> 32);
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    K.k0[r] = a; K.k1[r] = b;
    a += kPhiloxW0; b += kPhiloxW1;
  }
  return K;
}

__device__ __forceinline__ U4 philox_keyed(uint64_t ctr, uint32_t stream, const PhiloxKeys& K) {
  uint32_t c0 = (uint32_t)ctr, c1 = (uint32_t)(ctr >> 32), c2 = stream, c3 = 0;
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    const unsigned long long p0 = (unsigned long long)kPhiloxM0 * c0;
    const unsigned long long p1 = (unsigned long long)kPhiloxM1 * c2;
    const uint32_t n0 = (uint32_t)(p1 >> 32) ^ c1 ^ K.k0[r];
    const uint32_t n2 = (uint32_t)(p0 >> 32) ^ c3 ^ K.k1[r];
    c0 = n0; c1 = (uint32_t)p1; c2 = n2; c3 = (uint32_t)p0;
  }
  return U4{c0, c1, c2, c3};
}

// Bit mask of the Hadamard signs: bit j set <=> d_j = -1 (bit 31 of draw j).
__host__ inline uint32_t rht_sign_mask(uint64_t seed, int n) {
  uint32_t m = 0;
  for (int j = 0; j < n; j += 4) {
    U4 w = philox4x32_10((uint64_t)(j >> 2), kRhtStream, seed);
    uint32_t ws[4] = {w.x, w.y, w.z, w.w};
    for (int q = 0; q < 4 && j + q < n; ++q) m |= (ws[q] >> 31) << (j + q);
  }
  return m;
}

// ---------------------------------------------------------------------------
// BF16 unpacking (exact widening).
// ---------------------------------------------------------------------------
__device__ __forceinline__ void bf16x8_to_f32(const uint4& u, float* v) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    v[2 * i] = __uint_as_float(w[i] << 16);
    v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

__device__ __forceinline__ uint4 ld_nc_v4(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
  return r;
}

// ---------------------------------------------------------------------------
// E2M1 round-to-nearest-even, saturating: 8 floats -> 8 packed codes (32
// bits), element 2j in the low nibble of byte j.  cvt packs its first source
// operand into the high nibble.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t e2m1x8_rn(const float* v) {
  uint32_t out;
  asm("{\n\t.reg .b8 q0, q1, q2, q3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 q0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 q1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 q2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 q3, %8, %7;\n\t"
      "mov.b32 %0, {q0, q1, q2, q3};\n\t}"
      : "=r"(out)
      : "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]),
        "f"(v[7]));
  return out;
}

// Byte permute: result byte k is byte sel_k of the 8 bytes {b, a} (a = 0..3,
// b = 4..7); a selector nibble with bit 3 set replicates that byte's sign bit.
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t r;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
  return r;
}

__device__ __forceinline__ float fmin3(float a, float b, float c) {
  float r;
  asm("min.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// E2M1 stochastic rounding with 16-bit draws: with lo <= |v| <= hi the
// neighbouring levels (|v| clamped to 6) and p = (|v| - lo) / (hi - lo),
// round up iff floor(p * 2^16) + u >= 2^16.
//
// Branch-free.  code(lo) * 2^16 + p * 2^16 is a concave piecewise-linear map
// of a = |v|: slope 2^16 / gap for the gaps 0.5 (a < 2), 1 (2 <= a < 4) and
// 2 (4 <= a <= 6), equal to k * 2^16 at the k-th level, flat from 6 on:
//   f(a) = min(a * 2^17, (a + 2) * 2^16, (a + 8) * 2^15, 7 * 2^16).
// The floor of each line is one FMA rounded toward -inf with 2^23 added (in
// [2^23, 2^24) every float is an integer), and the floor of the min is the
// min of the floors.  So min(...) as an integer is 2^23 + code(lo) * 2^16 +
// floor(p * 2^16), below 2^23 + 2^19; adding the draw carries into bit 16
// exactly when the value rounds up, and byte 2 of the sum is the code (its
// bits 3..7 stay 0).  NaN inputs give 6 (min drops NaN); they are flagged by
// the amax check.
__device__ __forceinline__ uint32_t sr16_byte2(float a, uint32_t u16) {
  const float g1 = __fmaf_rd(a, 131072.0f, 8388608.0f);               // a*2^17 + 2^23
  const float g2 = __fmaf_rd(a, 65536.0f, 8519680.0f);                // (a+2)*2^16 + 2^23
  const float g3 = __fmaf_rd(a, 32768.0f, 8650752.0f);                // (a+8)*2^15 + 2^23
  const float m = fminf(fmin3(g1, g2, g3), 8847360.0f);              // 7*2^16 + 2^23
  return __float_as_uint(m) + u16;
}

// Codes of 4 elements, one per byte (byte k = element k), from their sr16_byte2
// results.
__device__ __forceinline__ uint32_t gather_byte2(uint32_t t0, uint32_t t1, uint32_t t2, uint32_t t3) {
  return prmt(prmt(t0, t1, 0x0062u), prmt(t2, t3, 0x0062u), 0x5410u);
}

// Eight 4-bit codes (element k in byte k of lo / hi, magnitude in bits 0..2,
// sign in bit 3) packed into one word, element k in bits 4k..4k+3.
__device__ __forceinline__ uint32_t pack_nibbles(uint32_t lo, uint32_t hi) {
  lo |= lo >> 4;                                  // bytes 0 and 2 now hold two codes each
  hi |= hi >> 4;
  return prmt(lo, hi, 0x6420u);
}

// Magnitudes a[8] = |RN(x * inv)| of eight elements with sign bytes `sgn_lo`
// (elements 0..3) and `sgn_hi` (4..7), byte k 0xFF for a negative element and
// 0 otherwise: stochastically rounded E2M1 codes, element k in bits 4k..4k+3,
// with the 16-bit draws of one Philox block (element k: the low (k even) or
// high (k odd) half of word k / 2).
__device__ __forceinline__ uint32_t e2m1x8_sr_mag(const float* a, uint32_t sgn_lo, uint32_t sgn_hi,
                                                  const U4& w) {
  const uint32_t t0 = sr16_byte2(a[0], w.x & 0xFFFFu), t1 = sr16_byte2(a[1], w.x >> 16);
  const uint32_t t2 = sr16_byte2(a[2], w.y & 0xFFFFu), t3 = sr16_byte2(a[3], w.y >> 16);
  const uint32_t t4 = sr16_byte2(a[4], w.z & 0xFFFFu), t5 = sr16_byte2(a[5], w.z >> 16);
  const uint32_t t6 = sr16_byte2(a[6], w.w & 0xFFFFu), t7 = sr16_byte2(a[7], w.w >> 16);
  const uint32_t lo = gather_byte2(t0, t1, t2, t3) | (sgn_lo & 0x08080808u);
  const uint32_t hi = gather_byte2(t4, t5, t6, t7) | (sgn_hi & 0x08080808u);
  return pack_nibbles(lo, hi);
}

// Sign bytes of four BF16 values held as two pairs (element 2j in the low
// half of word j): byte k is 0xFF when element k is negative.
__device__ __forceinline__ uint32_t bf16_sign_bytes(uint32_t w0, uint32_t w1) {
  return prmt(w0, w1, 0xFDB9u);
}

// Sign bytes of four floats.
__device__ __forceinline__ uint32_t f32_sign_bytes(float v0, float v1, float v2, float v3) {
  return prmt(prmt(__float_as_uint(v0), __float_as_uint(v1), 0x00FBu),
              prmt(__float_as_uint(v2), __float_as_uint(v3), 0x00FBu), 0x5410u);
}

// Eight signed values v[8] (already multiplied by the block's inverse scale):
// stochastically rounded codes as e2m1x8_sr_mag.
__device__ __forceinline__ uint32_t e2m1x8_sr(const float* v, const U4& w) {
  float a[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) a[j] = fabsf(v[j]);
  return e2m1x8_sr_mag(a, f32_sign_bytes(v[0], v[1], v[2], v[3]),
                       f32_sign_bytes(v[4], v[5], v[6], v[7]), w);
}

// RN(y / 6) for the block-scale step, as Markstein's correction of a product
// by the rounded reciprocal (P. Markstein, IBM J. Res. Dev. 34(1), 1990):
// q0 = RN(y * RN(1/6)), e = y - 6 q0 (exact by FMA), q1 = RN(q0 + e * RN(1/6)).
// Checked on the CPU for every non-negative binary32 y against the exactly
// rounded quotient: equal for all y >= 2^-125; below that both quotients are
// under 2^-127, far under half of E4M3's smallest step (2^-10), so the E4M3
// scale chosen from them is the same for every y.
__device__ __forceinline__ float div6_for_scale(float y) {
  const float r = 0.16666667163372040f;              // RN(1/6) = 0x3E2AAAAB
  const float q0 = __fmul_rn(y, r);
  const float e = __fmaf_rn(-6.0f, q0, y);
  return __fmaf_rn(e, r, q0);
}

// ---------------------------------------------------------------------------
// E4M3 (bias 7, max 448, subnormals down to 2^-9) round-to-nearest-even with
// saturation for a non-negative scale, and its exact decode.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t e4m3_rn_sat(float t) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(t));
  return (uint32_t)(r & 0xFFu);
}

__device__ __forceinline__ float e4m3_value(uint32_t c) {
  const uint32_t e = (c >> 3) & 15u, m = c & 7u;
  if (e == 0) return __fmul_rn((float)m, 0.001953125f);          // m * 2^-9
  return __uint_as_float(((e + 120u) << 23) | (m << 20));        // 2^(e-7) (1 + m/8)
}

// E8M0 scale 2^-e as an exact float for e in [-127, 127].
__device__ __forceinline__ float exp2_neg_exact(int e) {
  const int x = -e;                          // result 2^x, x in [-127, 127]
  if (x >= -126) return __uint_as_float((uint32_t)(x + 127) << 23);
  return __uint_as_float(1u << 22);          // 2^-127 (subnormal)
}

// floor(log2 b) from the binary32 encoding, b finite and > 0.
__device__ __forceinline__ int floor_log2_f32(float b) {
  const uint32_t bits = __float_as_uint(b);
  const int E = (int)((bits >> 23) & 0xFF);
  if (E > 0) return E - 127;
  return (31 - __clz(bits & 0x7FFFFF)) - 149;
}

// NVFP4 tensor scales from the amax: s_enc = RN(2688 / A) (largest finite
// float on overflow), s_dec = RN(A / 2688); A = 0 gives 1 and 1.
__device__ __forceinline__ void nvfp4_global_scales(float A, float& s_enc, float& s_dec) {
  if (A == 0.0f) { s_enc = 1.0f; s_dec = 1.0f; return; }
  float e = __fdiv_rn(2688.0f, A);
  if (isinf(e)) e = 3.402823466e38f;
  s_enc = e;
  s_dec = __fdiv_rn(A, 2688.0f);
}

// Byte offset of scale (r, s) in the tensor-core scale layout: 512-byte atoms
// of 128 rows x 4 blocks, atoms ordered row-block major; within an atom, row
// r%32 owns 16 bytes holding rows r, r+32, r+64, r+96 (4 blocks each).
__host__ __device__ __forceinline__ int64_t mma_sf_offset(int64_t r, int64_t s, int64_t S) {
  return ((r >> 7) * (S >> 2) + (s >> 2)) * 512 + (r & 31) * 16 + ((r & 127) >> 5) * 4 + (s & 3);
}

// ---------------------------------------------------------------------------
// In-register Walsh-Hadamard butterflies on 8 values: strides 1, 2, 4,
// (a, b) -> (a + b, a - b).
// ---------------------------------------------------------------------------
__device__ __forceinline__ void wht8(float* v) {
#pragma unroll
  for (int h = 1; h < 8; h <<= 1) {
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      if (j & h) continue;
      const float a = v[j], b = v[j + h];
      v[j] = __fadd_rn(a, b);
      v[j + h] = __fsub_rn(a, b);
    }
  }
}

// Stride-h stage across threads: this thread holds chunk `mine` of 8 values
// and the partner (lane ^ lane_xor) holds the chunk h = 8 * lane_xor away.
// The lower chunk becomes a + b, the upper one a - b (a = lower, b = upper).
__device__ __forceinline__ void wht_cross(float* v, int lane_xor, bool upper) {
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const float p = __shfl_xor_sync(0xFFFFFFFFu, v[j], lane_xor);
    v[j] = upper ? __fsub_rn(p, v[j]) : __fadd_rn(v[j], p);
  }
}

}  // namespace fp4dev
