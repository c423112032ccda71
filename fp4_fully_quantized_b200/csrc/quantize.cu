// quantize.cu -- HBM-bound FP4 quantizers for sm_100a.
//
// NVFP4 ("FP4", Robots Atlas, How it works / Components "NVFP4"): 16-value
// blocks, E4M3 block scale, FP32 tensor scale from the tensor amax.
// MXFP4 (Components "MXFP4"): 32-value blocks, E8M0 power-of-two scale.
// Rounding ("FP4 All the Way", Key points): round-to-nearest in the forward
// pass, stochastic rounding (Philox draws) in the backward and update passes.
// Optional block-wise random Hadamard transform before quantizing ("FP4",
// How it works; "Quartet", Approach).
//
// Row-wise kernels: each thread owns one 16-byte load (8 BF16 values); the
// 2 (NVFP4) or 4 (MXFP4) threads of a block are adjacent lanes and combine
// their block max and cross-thread Hadamard stages with warp shuffles, so a
// warp reads 512 contiguous bytes per load instruction.
// Transposed kernels: a 64 x 64 tile is staged through shared memory; each
// thread then owns 32 consecutive rows of one column (blocks run down x's
// columns) and writes 16 bytes of codes of the transposed operand.
#include <cfloat>
#include <cstdint>

#include "fp4_device.cuh"
#include "internal.h"

namespace fp4impl {
using namespace fp4dev;

namespace {

constexpr int kThreads = 256;
constexpr float kRht32Scale = 0.17677669227123260f;   // RN(1/sqrt(32)) = 0x3E3504F3

template <int RHT_N>
__device__ __forceinline__ float rht_scale() {
  return RHT_N == 16 ? 0.25f : kRht32Scale;
}

// Rotates the 8 values of chunk `q` (chunk index within its Hadamard block)
// held by this lane; lanes holding the other chunks of the block are the
// adjacent lanes (lane ^ 1, lane ^ 2).
template <int RHT_N>
__device__ __forceinline__ void rht_chunk(float* v, uint32_t mask, int q) {
  if constexpr (RHT_N > 0) {
#pragma unroll
    for (int i = 0; i < 8; ++i)
      if ((mask >> (8 * q + i)) & 1u) v[i] = -v[i];
    wht8(v);
#pragma unroll
    for (int lx = 1; lx < RHT_N / 8; lx <<= 1) wht_cross(v, lx, (q & lx) != 0);
    const float c = rht_scale<RHT_N>();
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = __fmul_rn(v[i], c);
  }
}

// QuEST-style clipping threshold of an MXFP4 32-block held by four adjacent
// lanes (8 consecutive values each, lane % 4 = group): T = RN(alpha * RMS)
// with the mean square summed in binary32 as ((y0^2 + y1^2) + (y2^2 + y3^2))
// + ((y4^2 + y5^2) + (y6^2 + y7^2)) per lane, then (g0 + g1) + (g2 + g3) over
// the lanes (two butterfly stages; both orders of each add give the same
// bits); alpha = 2.9224751 minimises the E2M1 rounding MSE of a unit
// Gaussian ("Quartet", Approach: QuEST-style forward quantization).
constexpr float kQuestAlpha = 2.9224751f;

__device__ __forceinline__ float quest_threshold(const float* v) {
  const float a = __fadd_rn(__fmul_rn(v[0], v[0]), __fmul_rn(v[1], v[1]));
  const float b = __fadd_rn(__fmul_rn(v[2], v[2]), __fmul_rn(v[3], v[3]));
  const float c = __fadd_rn(__fmul_rn(v[4], v[4]), __fmul_rn(v[5], v[5]));
  const float d = __fadd_rn(__fmul_rn(v[6], v[6]), __fmul_rn(v[7], v[7]));
  float g = __fadd_rn(__fadd_rn(a, b), __fadd_rn(c, d));
  g = __fadd_rn(g, __shfl_xor_sync(0xFFFFFFFFu, g, 1));
  g = __fadd_rn(g, __shfl_xor_sync(0xFFFFFFFFu, g, 2));
  return __fmul_rn(kQuestAlpha, __fsqrt_rn(__fmul_rn(g, 0.03125f)));
}

__device__ __forceinline__ void block_amax_atomic(float m, float* amax) {
  __shared__ float red[kThreads / 32];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  if (l == 0) red[w] = m;
  __syncthreads();
  if (w == 0) {
    m = (l < (int)(blockDim.x >> 5)) ? red[l] : 0.0f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
    // |x| has a clear sign bit, so integer order equals float order; NaN
    // patterns sort above +Inf and survive the max.
    if (l == 0) atomicMax(reinterpret_cast<unsigned int*>(amax), __float_as_uint(m));
  }
}

// |v| max that keeps NaN (fmaxf would drop it).
__device__ __forceinline__ float absmax_keep_nan(float m, float v) {
  const uint32_t a = __float_as_uint(v) & 0x7FFFFFFFu;
  return __uint_as_float(max(__float_as_uint(m), a));
}

// ---------------------------------------------------------------------------
// Row-wise amax (optionally of the rotated values).
// ---------------------------------------------------------------------------
template <int RHT_N>
__global__ void __launch_bounds__(kThreads)
amax_rows_kernel(const __nv_bfloat16* __restrict__ x, int64_t rows, int64_t cols, int64_t ld,
                 uint32_t rht_mask, float* amax) {
  // one warp per row segment of 32 x 4 16-byte chunks, all four loads in
  // flight before the rotation (the lanes of a Hadamard block are adjacent)
  constexpr int CH = 4, SEG = 32 * CH;
  const int64_t cpr = cols >> 3;
  const int64_t segs = (cpr + SEG - 1) / SEG, units = rows * segs;
  const int lane = threadIdx.x & 31;
  const int64_t warp0 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  float m = 0.0f;
  for (int64_t u = warp0; u < units; u += nwarps) {
    const int64_t r = u / segs, c0 = (u - r * segs) * SEG;
    const __nv_bfloat16* xr = x + r * ld;
    uint4 raw[CH];
#pragma unroll
    for (int q = 0; q < CH; ++q) {
      const int64_t c = c0 + 32 * q + lane;
      raw[q] = (c < cpr) ? ld_nc_v4(xr + c * 8) : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int q = 0; q < CH; ++q) {
      float v[8];
      bf16x8_to_f32(raw[q], v);
      if constexpr (RHT_N > 0) rht_chunk<RHT_N>(v, rht_mask, lane % (RHT_N / 8));
#pragma unroll
      for (int i = 0; i < 8; ++i) m = absmax_keep_nan(m, v[i]);
    }
  }
  block_amax_atomic(m, amax);
}

// Plain amax (no rotation): 4 independent 16-byte loads per thread in
// flight; |x| max taken on the BF16 bit patterns two at a time (sign bits
// cleared, per-halfword unsigned max), which is exact and keeps NaN
// patterns above +Inf.
__global__ void __launch_bounds__(kThreads)
amax_plain_kernel(const __nv_bfloat16* __restrict__ x, int64_t rows, int64_t cols, int64_t ld,
                  float* amax) {
  const int64_t cpr = cols >> 3;
  const int64_t total = rows * cpr;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  uint32_t m2 = 0;
  const bool dense = (ld == cols);
  int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  for (; g + 3 * stride < total; g += 4 * stride) {
    uint4 u[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int64_t gg = g + q * stride;
      const int64_t off = dense ? gg * 8 : (gg / cpr) * ld + (gg % cpr) * 8;
      u[q] = ld_nc_v4(x + off);
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      m2 = __vmaxu2(m2, u[q].x & 0x7FFF7FFFu);
      m2 = __vmaxu2(m2, u[q].y & 0x7FFF7FFFu);
      m2 = __vmaxu2(m2, u[q].z & 0x7FFF7FFFu);
      m2 = __vmaxu2(m2, u[q].w & 0x7FFF7FFFu);
    }
  }
  for (; g < total; g += stride) {
    const int64_t off = dense ? g * 8 : (g / cpr) * ld + (g % cpr) * 8;
    const uint4 u = ld_nc_v4(x + off);
    m2 = __vmaxu2(m2, u.x & 0x7FFF7FFFu);
    m2 = __vmaxu2(m2, u.y & 0x7FFF7FFFu);
    m2 = __vmaxu2(m2, u.z & 0x7FFF7FFFu);
    m2 = __vmaxu2(m2, u.w & 0x7FFF7FFFu);
  }
  const uint32_t hi = m2 >> 16, lo = m2 & 0xFFFFu;
  block_amax_atomic(__uint_as_float(max(hi, lo) << 16), amax);
}

// ---------------------------------------------------------------------------
// Amax of the column-rotated tensor (the transposed operand's Hadamard runs
// down x's columns in blocks of RHT_N rows), optionally together with the
// plain amax, from one read of x.  A warp takes RHT_N rows x 256 columns:
// lane l loads its 8 columns of every row (RHT_N 16-byte loads in flight),
// then rotates each of its 8 columns in registers.
// ---------------------------------------------------------------------------
template <int RHT_N>
__global__ void __launch_bounds__(kThreads)
amax_cols_rht_kernel(const __nv_bfloat16* __restrict__ x, int64_t rows, int64_t cols, int64_t ld,
                     uint32_t rht_mask, float* amax_col, float* amax_plain) {
  const int64_t segs = (cols + 255) / 256, units = (rows / RHT_N) * segs;
  const int lane = threadIdx.x & 31;
  const int64_t warp0 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  const float cn = rht_scale<RHT_N>();
  float mc = 0.0f, mp = 0.0f;
  for (int64_t u = warp0; u < units; u += nwarps) {
    const int64_t rb = u / segs;
    const int64_t c = (u - rb * segs) * 256 + 8 * lane;
    if (c >= cols) continue;                  // rows % RHT_N == 0, cols % 8 == 0
    const __nv_bfloat16* xp = x + rb * RHT_N * ld + c;
    uint4 raw[RHT_N];
#pragma unroll
    for (int q = 0; q < RHT_N; ++q) raw[q] = ld_nc_v4(xp + q * ld);
#pragma unroll
    for (int e = 0; e < 8; ++e) {             // column c + e
      float v[RHT_N];
#pragma unroll
      for (int q = 0; q < RHT_N; ++q) {
        const uint32_t w = (&raw[q].x)[e >> 1];
        v[q] = __uint_as_float((e & 1) ? (w & 0xFFFF0000u) : (w << 16));
        mp = absmax_keep_nan(mp, v[q]);
        if ((rht_mask >> q) & 1u) v[q] = -v[q];
      }
#pragma unroll
      for (int hh = 1; hh < RHT_N; hh <<= 1) {
#pragma unroll
        for (int q = 0; q < RHT_N; ++q) {
          if (q & hh) continue;
          const float a = v[q], b = v[q + hh];
          v[q] = __fadd_rn(a, b);
          v[q + hh] = __fsub_rn(a, b);
        }
      }
#pragma unroll
      for (int q = 0; q < RHT_N; ++q) mc = absmax_keep_nan(mc, __fmul_rn(v[q], cn));
    }
  }
  block_amax_atomic(mc, amax_col);
  if (amax_plain != nullptr) block_amax_atomic(mp, amax_plain);
}

// ---------------------------------------------------------------------------
// Row-wise quantization (NVFP4 BS = 16 or MXFP4 BS = 32).  A warp takes one
// row segment of 32 x kRowChunks 16-byte chunks (1024 elements): lane l owns
// chunks l, l + 32, ... of the segment, all of whose loads are issued before
// any is encoded; the lanes of a block (2 for NVFP4, 4 for MXFP4) are
// adjacent, so the block max and the Hadamard stages are warp shuffles.
// NVFP4 reads RN(s_enc / value(sf)) from a per-CTA table of the 128 E4M3
// codes instead of dividing per block.
// ---------------------------------------------------------------------------
constexpr int kRowChunks = 4;

template <int BS, int RHT_N, bool SR, bool QUEST = false>
__global__ void __launch_bounds__(kThreads)
quant_rows_kernel(const __nv_bfloat16* __restrict__ x, int64_t rows, int64_t cols, int64_t ld,
                  uint32_t rht_mask, const __grid_constant__ PhiloxKeys K, uint32_t sr_stream,
                  const float* __restrict__ amax_src, float* amax_out, float* s_dec_out,
                  uint8_t* __restrict__ codes, uint8_t* __restrict__ scales,
                  uint8_t* __restrict__ scales_mma, uint32_t* status) {
  constexpr bool NV = (BS == 16);
  constexpr int TPB = BS / 8;                 // lanes per block
  constexpr int SEG = 32 * kRowChunks;        // chunks per warp step
  const int64_t cpr = cols >> 3;              // 16-byte chunks per row
  const int64_t segs = (cpr + SEG - 1) / SEG; // warp steps per row
  const int64_t units = rows * segs;
  const int64_t S = cols / BS, S4 = (S + 3) & ~3LL;
  const int lane = threadIdx.x & 31;
  const int64_t warp0 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;

  float s_enc = 1.0f, s_dec = 1.0f;
  __shared__ float inv_tab[128];
  if constexpr (NV) {
    const float A = *amax_src;
    if (!(A <= FLT_MAX)) {                    // Inf or NaN: precondition violated
      if (blockIdx.x == 0 && threadIdx.x == 0) set_status(status, FP4_ERR_NONFINITE, 1);
    }
    nvfp4_global_scales(A, s_enc, s_dec);
    if (blockIdx.x == 0 && threadIdx.x == 0) {
      if (amax_out != nullptr && amax_out != amax_src) *amax_out = A;
    }
    for (int c = threadIdx.x; c < 128; c += blockDim.x)
      inv_tab[c] = (c == 0 || c == 127) ? 0.0f : fminf(__fdiv_rn(s_enc, e4m3_value((uint32_t)c)), FLT_MAX);
    __syncthreads();
  }
  if (blockIdx.x == 0 && threadIdx.x == 0 && s_dec_out != nullptr) *s_dec_out = s_dec;

  for (int64_t u = warp0; u < units; u += nwarps) {
    const int64_t r = u / segs;
    const int64_t c0 = (u - r * segs) * SEG;
    const __nv_bfloat16* xr = x + r * ld;
    uint4 raw[kRowChunks];
#pragma unroll
    for (int q = 0; q < kRowChunks; ++q) {
      const int64_t c = c0 + 32 * q + lane;
      raw[q] = (c < cpr) ? ld_nc_v4(xr + c * 8) : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int q = 0; q < kRowChunks; ++q) {
      const int64_t c = c0 + 32 * q + lane;
      if (c0 + 32 * q >= cpr) break;          // warp-uniform: the segment's tail is done
      float v[8];
      bf16x8_to_f32(raw[q], v);
      if constexpr (RHT_N > 0) rht_chunk<RHT_N>(v, rht_mask, lane % (RHT_N / 8));
      float bmax = 0.0f;
#pragma unroll
      for (int i = 0; i < 8; ++i) bmax = fmaxf(bmax, fabsf(v[i]));
#pragma unroll
      for (int lx = 1; lx < TPB; lx <<= 1) bmax = fmaxf(bmax, __shfl_xor_sync(0xFFFFFFFFu, bmax, lx));
      uint32_t sf;
      float inv;
      if constexpr (NV) {
        const float t = div6_for_scale(__fmul_rn(bmax, s_enc));
        sf = e4m3_rn_sat(t);                  // 0 .. 126
        inv = inv_tab[sf];
      } else {
        // QuEST: the clipping threshold takes the block max's place
        const float top = QUEST ? quest_threshold(v) : bmax;
        int e = (top == 0.0f) ? -127 : floor_log2_f32(top) - 2;
        e = max(-127, min(127, e));
        sf = (uint32_t)(e + 127);
        inv = exp2_neg_exact(e);
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) v[i] = __fmul_rn(v[i], inv);
      uint32_t packed;
      if constexpr (!SR) {
        packed = e2m1x8_rn(v);
      } else {
        // one Philox block: the 16-bit draws of these 8 elements
        const uint64_t i0 = (uint64_t)r * (uint64_t)cols + (uint64_t)(c * 8);
        const U4 w = philox_keyed(i0 >> 3, sr_stream, K);
        if constexpr (RHT_N > 0) {
          packed = e2m1x8_sr(v, w);
        } else {
          float a[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) a[i] = fabsf(v[i]);
          packed = e2m1x8_sr_mag(a, bf16_sign_bytes(raw[q].x, raw[q].y),
                                 bf16_sign_bytes(raw[q].z, raw[q].w), w);
        }
      }
      if (c < cpr) {
        *reinterpret_cast<uint32_t*>(codes + r * (cols >> 1) + c * 4) = packed;
        if ((lane % TPB) == 0) {
          const int64_t sb = c / TPB;
          if (scales != nullptr) scales[r * S + sb] = (uint8_t)sf;
          if (scales_mma != nullptr) scales_mma[mma_sf_offset(r, sb, S4)] = (uint8_t)sf;
        }
      }
    }
  }
}

// ---------------------------------------------------------------------------
// Transposed quantization / amax: x [rows, cols] -> operand x^T [cols, rows],
// blocks of BS run along x's rows.  64 x 64 tile per CTA (128 threads); the
// thread owning (column k, half h) handles rows 32h .. 32h + 31 of the tile.
// ---------------------------------------------------------------------------
constexpr int kTile = 64;
constexpr int kColThreads = 128;

template <int BS, int RHT_N, bool SR, bool AMAX_ONLY>
__global__ void __launch_bounds__(kColThreads)
quant_cols_kernel(const __nv_bfloat16* __restrict__ x, int64_t rows, int64_t cols, int64_t ld,
                  uint32_t rht_mask, uint64_t sr_seed, uint32_t sr_stream,
                  const float* __restrict__ amax_src, float* amax_out, float* s_dec_out,
                  uint8_t* __restrict__ codes, uint8_t* __restrict__ scales,
                  uint8_t* __restrict__ scales_mma, uint32_t* status) {
  constexpr bool NV = (BS == 16);
  __shared__ __align__(16) __nv_bfloat16 tile[kTile][kTile];
  __shared__ float red[kColThreads / 32];

  const int64_t tiles_m = (rows + kTile - 1) / kTile, tiles_k = (cols + kTile - 1) / kTile;
  const int64_t ntiles = tiles_m * tiles_k;
  const int64_t S = rows / BS;             // blocks per row of x^T
  const int t = threadIdx.x;
  const int kk = t & 63, h = t >> 6;

  float s_enc = 1.0f, s_dec = 1.0f;
  if constexpr (NV && !AMAX_ONLY) {
    const float A = *amax_src;
    if (!(A <= FLT_MAX)) {
      if (blockIdx.x == 0 && t == 0) set_status(status, FP4_ERR_NONFINITE, 2);
    }
    nvfp4_global_scales(A, s_enc, s_dec);
    if (blockIdx.x == 0 && t == 0 && amax_out != nullptr && amax_out != amax_src) *amax_out = A;
  }
  if constexpr (!AMAX_ONLY) {
    if (blockIdx.x == 0 && t == 0 && s_dec_out != nullptr) *s_dec_out = s_dec;
  }
  float m = 0.0f;

  for (int64_t tile_id = blockIdx.x; tile_id < ntiles; tile_id += gridDim.x) {
    const int64_t tm = tile_id / tiles_k, tk = tile_id - tm * tiles_k;
    const int64_t m0 = tm * kTile, k0 = tk * kTile;
    __syncthreads();                      // previous tile fully consumed
#pragma unroll
    for (int it = 0; it < 4; ++it) {
      const int rr = (t >> 3) + 16 * it, cc = (t & 7) * 8;
      uint4 u = make_uint4(0, 0, 0, 0);
      if (m0 + rr < rows && k0 + cc < cols) u = ld_nc_v4(x + (m0 + rr) * ld + k0 + cc);
      *reinterpret_cast<uint4*>(&tile[rr][cc]) = u;
    }
    __syncthreads();

    const int64_t k = k0 + kk;
    float v[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __bfloat162float(tile[32 * h + i][kk]);

    if constexpr (RHT_N > 0) {
#pragma unroll
      for (int base = 0; base < 32; base += RHT_N) {
#pragma unroll
        for (int i = 0; i < RHT_N; ++i)
          if ((rht_mask >> i) & 1u) v[base + i] = -v[base + i];
#pragma unroll
        for (int hh = 1; hh < RHT_N; hh <<= 1) {
#pragma unroll
          for (int i = 0; i < RHT_N; ++i) {
            if (i & hh) continue;
            const float a = v[base + i], b = v[base + i + hh];
            v[base + i] = __fadd_rn(a, b);
            v[base + i + hh] = __fsub_rn(a, b);
          }
        }
        const float c = rht_scale<RHT_N>();
#pragma unroll
        for (int i = 0; i < RHT_N; ++i) v[base + i] = __fmul_rn(v[base + i], c);
      }
    }

    const int64_t mrow0 = m0 + 32 * h;    // first x row of this thread's run
    if constexpr (AMAX_ONLY) {
      if (k < cols) {
#pragma unroll
        for (int i = 0; i < 32; ++i)
          if (mrow0 + i < rows) m = absmax_keep_nan(m, v[i]);
      }
      continue;
    } else {
      if (k >= cols || mrow0 >= rows) continue;
      uint32_t packed[4] = {0, 0, 0, 0};
#pragma unroll
      for (int b = 0; b < 32 / BS; ++b) {
        if (mrow0 + b * BS >= rows) break;
        float bmax = 0.0f;
#pragma unroll
        for (int i = 0; i < BS; ++i) bmax = fmaxf(bmax, fabsf(v[b * BS + i]));
        uint32_t sf;
        float inv;
        if constexpr (NV) {
          const float tt = div6_for_scale(__fmul_rn(bmax, s_enc));
          sf = e4m3_rn_sat(tt);
          inv = (sf == 0) ? 0.0f : fminf(__fdiv_rn(s_enc, e4m3_value(sf)), FLT_MAX);
        } else {
          int e = (bmax == 0.0f) ? -127 : floor_log2_f32(bmax) - 2;
          e = max(-127, min(127, e));
          sf = (uint32_t)(e + 127);
          inv = exp2_neg_exact(e);
        }
#pragma unroll
        for (int i = 0; i < BS; ++i) v[b * BS + i] = __fmul_rn(v[b * BS + i], inv);
        const int64_t s = (mrow0 + b * BS) / BS;
        if (scales != nullptr) scales[k * S + s] = (uint8_t)sf;
        if (scales_mma != nullptr) scales_mma[mma_sf_offset(k, s, (S + 3) & ~3LL)] = (uint8_t)sf;
      }
      if constexpr (!SR) {
#pragma unroll
        for (int q = 0; q < 4; ++q) packed[q] = e2m1x8_rn(&v[8 * q]);
      } else {
        const uint64_t i0 = (uint64_t)k * (uint64_t)rows + (uint64_t)mrow0;   // a multiple of 16
#pragma unroll
        for (int q = 0; q < 4; ++q)
          packed[q] = e2m1x8_sr(&v[8 * q], philox4x32_10((i0 >> 3) + q, sr_stream, sr_seed));
      }
      uint8_t* dst = codes + k * (rows >> 1) + (mrow0 >> 1);
      *reinterpret_cast<uint2*>(dst) = make_uint2(packed[0], packed[1]);
      if (mrow0 + 16 < rows) *reinterpret_cast<uint2*>(dst + 8) = make_uint2(packed[2], packed[3]);
    }
  }
  if constexpr (AMAX_ONLY) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
    if ((t & 31) == 0) red[t >> 5] = m;
    __syncthreads();
    if (t == 0) {
      float mm = red[0];
      for (int w = 1; w < kColThreads / 32; ++w) mm = fmaxf(mm, red[w]);
      atomicMax(reinterpret_cast<unsigned int*>(amax_out), __float_as_uint(mm));
    }
  }
}

// ---------------------------------------------------------------------------
// NVFP4 16x16 2-D quantization (round to nearest): one E4M3 scale per tile.
// 64 x 64 region per CTA, 256 threads.  Emits W and W^T from the same codes.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256)
quant_2d_kernel(const __nv_bfloat16* __restrict__ x, int64_t rows, int64_t cols, int64_t ld,
                const float* __restrict__ amax_src, float* s_dec_out, float* s_dec_out_t,
                float* amax_out, float* amax_out_t, uint8_t* __restrict__ codes, uint8_t* __restrict__ scales,
                uint8_t* __restrict__ scales_mma, uint8_t* __restrict__ codes_t,
                uint8_t* __restrict__ scales_t, uint8_t* __restrict__ scales_mma_t,
                uint32_t* status) {
  __shared__ float tile[kTile][kTile + 1];
  __shared__ float tinv[16];
  __shared__ uint32_t tsf[16];
  const int t = threadIdx.x;
  const int64_t tiles_r = (rows + kTile - 1) / kTile, tiles_c = (cols + kTile - 1) / kTile;
  const int64_t S = cols / 16, St = rows / 16;

  const float A = *amax_src;
  if (!(A <= FLT_MAX) && blockIdx.x == 0 && t == 0) set_status(status, FP4_ERR_NONFINITE, 3);
  float s_enc, s_dec;
  nvfp4_global_scales(A, s_enc, s_dec);
  if (blockIdx.x == 0 && t == 0) {
    if (s_dec_out) *s_dec_out = s_dec;
    if (s_dec_out_t) *s_dec_out_t = s_dec;
    if (amax_out && amax_out != amax_src) *amax_out = A;
    if (amax_out_t && amax_out_t != amax_src) *amax_out_t = A;
  }

  // The next tile's two 16-byte loads per thread are issued before the
  // current tile is encoded, so their latency overlaps the encode.
  const int64_t ntiles = tiles_r * tiles_c;
  auto load_tile = [&](int64_t tid, uint4* raw) {
    const int64_t r0 = (tid / tiles_c) * kTile, c0 = (tid % tiles_c) * kTile;
#pragma unroll
    for (int it = 0; it < 2; ++it) {
      const int rr = (t >> 3) + 32 * it, cc = (t & 7) * 8;
      raw[it] = (r0 + rr < rows && c0 + cc < cols) ? ld_nc_v4(x + (r0 + rr) * ld + c0 + cc)
                                                  : make_uint4(0u, 0u, 0u, 0u);
    }
  };
  uint4 nxt[2];
  if (blockIdx.x < ntiles) load_tile(blockIdx.x, nxt);
  for (int64_t tid = blockIdx.x; tid < ntiles; tid += gridDim.x) {
    const int64_t r0 = (tid / tiles_c) * kTile, c0 = (tid % tiles_c) * kTile;
    __syncthreads();                          // the previous tile's reads are done
#pragma unroll
    for (int it = 0; it < 2; ++it) {
      const int rr = (t >> 3) + 32 * it, cc = (t & 7) * 8;
      float v[8];
      bf16x8_to_f32(nxt[it], v);
#pragma unroll
      for (int i = 0; i < 8; ++i) tile[rr][cc + i] = v[i];
    }
    if (tid + gridDim.x < ntiles) load_tile(tid + gridDim.x, nxt);
    __syncthreads();
    {  // tile max: 16 threads per 16x16 tile, one tile row each
      const int q = t >> 4, rr = t & 15;
      const int tr = q >> 2, tc = q & 3;
      float bm = 0.0f;
#pragma unroll
      for (int i = 0; i < 16; ++i) bm = fmaxf(bm, fabsf(tile[tr * 16 + rr][tc * 16 + i]));
#pragma unroll
      for (int o = 8; o > 0; o >>= 1) bm = fmaxf(bm, __shfl_xor_sync(0xFFFFFFFFu, bm, o));
      if (rr == 0) {
        const float tt = div6_for_scale(__fmul_rn(bm, s_enc));
        const uint32_t sf = e4m3_rn_sat(tt);
        tsf[q] = sf;
        tinv[q] = (sf == 0) ? 0.0f : fminf(__fdiv_rn(s_enc, e4m3_value(sf)), FLT_MAX);
        const int64_t gr = r0 / 16 + tr, gc = c0 / 16 + tc;
        if (gr < St && gc < S) {
          if (scales) scales[gr * S + gc] = (uint8_t)sf;
          if (scales_t) scales_t[gc * St + gr] = (uint8_t)sf;
        }
      }
    }
    __syncthreads();
    {  // W: row r0 + (t >> 2), 16-block (t & 3)
      const int rr = t >> 2, kb = t & 3;
      const int64_t r = r0 + rr, c = c0 + kb * 16;
      if (r < rows && c < cols) {
        const int q = (rr >> 4) * 4 + kb;
        float v[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) v[i] = __fmul_rn(tile[rr][kb * 16 + i], tinv[q]);
        if (codes) {
          *reinterpret_cast<uint2*>(codes + r * (cols >> 1) + (c >> 1)) =
              make_uint2(e2m1x8_rn(v), e2m1x8_rn(v + 8));
        }
        if (scales_mma) scales_mma[mma_sf_offset(r, c / 16, (S + 3) & ~3LL)] = (uint8_t)tsf[q];
      }
    }
    {  // W^T: row c0 + (t >> 2) of W^T (a column of W), 16-block (t & 3) of W rows
      const int cc = t >> 2, rb = t & 3;
      const int64_t k = c0 + cc, r = r0 + rb * 16;
      if (k < cols && r < rows) {
        const int q = rb * 4 + (cc >> 4);
        float v[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) v[i] = __fmul_rn(tile[rb * 16 + i][cc], tinv[q]);
        if (codes_t) {
          *reinterpret_cast<uint2*>(codes_t + k * (rows >> 1) + (r >> 1)) =
              make_uint2(e2m1x8_rn(v), e2m1x8_rn(v + 8));
        }
        if (scales_mma_t) scales_mma_t[mma_sf_offset(k, r / 16, (St + 3) & ~3LL)] = (uint8_t)tsf[q];
      }
    }
  }
}

// ---------------------------------------------------------------------------
// Fused row-wise + transposed quantization: each 64 x 256 tile of x is read
// from HBM once (cp.async into a double-buffered shared tile, the next tile in
// flight while this one is encoded) and produces both outputs:
//   row phase   warp w takes rows w, w + 8, ...; lane l the 8 values at columns
//               8l .. 8l + 7 (blocks of 16/32 = 2/4 adjacent lanes, Hadamard
//               stages across lanes by shuffles), 4 code bytes per lane;
//   column phase thread t takes columns 2p, 2p + 1 (p = t % 128) over the
//               tile's rows 32h .. 32h + 31 (h = t / 128), block by block
//               down the columns, and writes each column's 16 code bytes and
//               2 (1) scale bytes of the transposed operand in one go.
// Stochastic rounding draws 16 bits per element: one Philox block serves
// eight consecutive elements of an output's logical layout.
// ---------------------------------------------------------------------------
constexpr int kDualTM = 64, kDualTK = 256, kDualThreads = 256;
#ifndef FP4_DUAL_CTAS_PER_SM
#define FP4_DUAL_CTAS_PER_SM 3
#endif
constexpr int kDualCtasPerSm = FP4_DUAL_CTAS_PER_SM;   // resident CTAs per SM
constexpr int kDualSmem = 2 * kDualTM * kDualTK * 2;   // two bf16 tiles: 64 KB

__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gsrc, bool valid) {
  const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(smem_dst));
  const int n = valid ? 16 : 0;                        // 0 source bytes: zero fill
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(d), "l"(gsrc), "r"(n)
               : "memory");
}

template <bool NV>
__device__ __forceinline__ void block_scale(float bmax, float s_enc, const float* inv_tab,
                                            uint32_t& sf, float& inv) {
  if constexpr (NV) {
    const float t = div6_for_scale(__fmul_rn(bmax, s_enc));
    sf = e4m3_rn_sat(t);                  // 0 .. 126 (satfinite)
    inv = inv_tab[sf];                    // RN(s_enc / value(sf)), 0 for sf = 0
  } else {
    int e = (bmax == 0.0f) ? -127 : floor_log2_f32(bmax) - 2;
    e = max(-127, min(127, e));
    sf = (uint32_t)(e + 127);
    inv = exp2_neg_exact(e);
  }
}

// Resident CTAs per SM: three for the round-to-nearest NVFP4 forms (at most
// 80 registers a thread), two where stochastic rounding or 32-value blocks
// need more registers than that without spilling.
template <int BS, bool SR_R, bool SR_C>
constexpr int dual_ctas_per_sm() { return (BS == 16 && !SR_R && !SR_C) ? kDualCtasPerSm : 2; }

template <int BS, int RHT_R, int RHT_C, bool SR_R, bool SR_C, bool QUEST_R = false>
__global__ void __launch_bounds__(kDualThreads, (dual_ctas_per_sm<BS, SR_R, SR_C>()))
quant_dual_kernel(const __nv_bfloat16* __restrict__ x, int64_t rows, int64_t cols, int64_t ld,
                  uint32_t mask_r, uint32_t mask_c, const __grid_constant__ PhiloxKeys K,
                  uint32_t stream_r,
                  uint32_t stream_c, const float* __restrict__ amax_src_r,
                  const float* __restrict__ amax_src_c, float* amax_out_r, float* amax_out_c,
                  float* s_dec_r, float* s_dec_c, uint8_t* __restrict__ codes_r,
                  uint8_t* __restrict__ scales_r, uint8_t* __restrict__ mma_r,
                  uint8_t* __restrict__ codes_c, uint8_t* __restrict__ scales_c,
                  uint8_t* __restrict__ mma_c, uint32_t* status) {
  constexpr bool NV = (BS == 16);
  constexpr int TPB = BS / 8;
  extern __shared__ __align__(16) uint8_t dual_smem[];
  __nv_bfloat16 (*tile)[kDualTM][kDualTK] =
      reinterpret_cast<__nv_bfloat16 (*)[kDualTM][kDualTK]>(dual_smem);

  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const int64_t tiles_k = (cols + kDualTK - 1) / kDualTK;
  const int64_t ntiles = ((rows + kDualTM - 1) / kDualTM) * tiles_k;
  const int64_t S_r = cols / BS, S_r4 = (S_r + 3) & ~3LL;   // blocks per row, row output
  const int64_t S_c = rows / BS, S_c4 = (S_c + 3) & ~3LL;   // blocks per row of x^T

  float se_r = 1.0f, sd_r = 1.0f, se_c = 1.0f, sd_c = 1.0f;
  if constexpr (NV) {
    const float Ar = *amax_src_r, Ac = *amax_src_c;
    if ((!(Ar <= FLT_MAX) || !(Ac <= FLT_MAX)) && blockIdx.x == 0 && t == 0)
      set_status(status, FP4_ERR_NONFINITE, 4);
    nvfp4_global_scales(Ar, se_r, sd_r);
    nvfp4_global_scales(Ac, se_c, sd_c);
    if (blockIdx.x == 0 && t == 0) {
      if (amax_out_r != amax_src_r) *amax_out_r = Ar;
      if (amax_out_c != amax_src_c) *amax_out_c = Ac;
    }
  }
  if (blockIdx.x == 0 && t == 0) { *s_dec_r = sd_r; *s_dec_c = sd_c; }
  // RN(s_enc / value(sf)) for every E4M3 code, both orientations (NVFP4);
  // the first tile's __syncthreads publishes it.
  __shared__ float inv_tab[2][128];
  if constexpr (NV) {
    const int o = t >> 7, code = t & 127;
    const float se = o ? se_c : se_r;
    inv_tab[o][code] = (code == 0 || code == 127)
                           ? 0.0f : fminf(__fdiv_rn(se, e4m3_value((uint32_t)code)), FLT_MAX);
  }

  auto issue = [&](int64_t tile_id, int buf) {
    const int64_t m0 = (tile_id / tiles_k) * kDualTM, k0 = (tile_id % tiles_k) * kDualTK;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int rr = i * 8 + warp, cc = lane * 8;
      const bool ok = (m0 + rr < rows) && (k0 + cc < cols);
      const __nv_bfloat16* src = ok ? x + (m0 + rr) * ld + k0 + cc : x;
      cp_async16(&tile[buf][rr][cc], src, ok);
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };

  int64_t tile_id = blockIdx.x;
  if (tile_id < ntiles) issue(tile_id, 0);
  for (int it = 0; tile_id < ntiles; tile_id += gridDim.x, ++it) {
    const int buf = it & 1;
    const int64_t next = tile_id + gridDim.x;
    if (next < ntiles) {
      issue(next, buf ^ 1);
      asm volatile("cp.async.wait_group 1;" ::: "memory");
    } else {
      asm volatile("cp.async.wait_group 0;" ::: "memory");
    }
    __syncthreads();
    const int64_t m0 = (tile_id / tiles_k) * kDualTM, k0 = (tile_id % tiles_k) * kDualTK;

    // ---------------- row phase (blocks along x's rows) -----------------
    {
      const int cc = lane * 8;
      const int64_t c = k0 + cc;
      const bool col_ok = c < cols;
      const int64_t sb = c / BS;
      // tensor-core scale layout, split into the tile's row-block part (r >> 7
      // is the same for the tile's 64 rows) and this lane's block part
      const int64_t mma_tile = (m0 >> 7) * (S_r4 >> 2) * 512 + (sb >> 2) * 512 + (sb & 3);
      uint8_t* cptr = codes_r + (m0 + warp) * (cols >> 1) + (c >> 1);
      const int64_t cstep = 8 * (cols >> 1);
#pragma unroll 2
      for (int i = 0; i < 8; ++i, cptr += cstep) {
        const int rr = i * 8 + warp;
        const int64_t r = m0 + rr;
        const uint4 raw = *reinterpret_cast<const uint4*>(&tile[buf][rr][cc]);
        float v[8];
        bf16x8_to_f32(raw, v);
        if constexpr (RHT_R > 0) rht_chunk<RHT_R>(v, mask_r, lane % (RHT_R / 8));
        float bmax = 0.0f;
#pragma unroll
        for (int q = 0; q < 8; ++q) bmax = fmaxf(bmax, fabsf(v[q]));
#pragma unroll
        for (int lx = 1; lx < TPB; lx <<= 1) bmax = fmaxf(bmax, __shfl_xor_sync(0xFFFFFFFFu, bmax, lx));
        uint32_t sf;
        float inv;
        if constexpr (QUEST_R) {
          // QuEST (MXFP4): the clipping threshold takes the block max's place
          block_scale<NV>(quest_threshold(v), se_r, inv_tab[0], sf, inv);
        } else {
          block_scale<NV>(bmax, se_r, inv_tab[0], sf, inv);
        }
        uint32_t packed;
        if constexpr (!SR_R) {
#pragma unroll
          for (int q = 0; q < 8; ++q) v[q] = __fmul_rn(v[q], inv);
          packed = e2m1x8_rn(v);
        } else {
          // one Philox block: the 16-bit draws of these 8 elements
          const uint64_t i0 = (uint64_t)r * (uint64_t)cols + (uint64_t)c;    // a multiple of 8
          const U4 w = philox_keyed(i0 >> 3, stream_r, K);
          if constexpr (RHT_R > 0) {
#pragma unroll
            for (int q = 0; q < 8; ++q) v[q] = __fmul_rn(v[q], inv);
            packed = e2m1x8_sr(v, w);
          } else {
            float a[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) a[q] = __fmul_rn(fabsf(v[q]), inv);
            packed = e2m1x8_sr_mag(a, bf16_sign_bytes(raw.x, raw.y), bf16_sign_bytes(raw.z, raw.w), w);
          }
        }
        if (col_ok && r < rows) {
          *reinterpret_cast<uint32_t*>(cptr) = packed;
          if ((lane % TPB) == 0) {
            if (scales_r != nullptr) scales_r[r * S_r + sb] = (uint8_t)sf;
            if (mma_r != nullptr) mma_r[mma_tile + (rr & 31) * 16 + (((int)(m0 & 127) + rr) >> 5) * 4] = (uint8_t)sf;
          }
        }
      }
    }

    // ---------------- column phase (blocks along x's columns) -----------
    // Thread t encodes the column pair k0 + 2p, k0 + 2p + 1 (p = t % 128)
    // over the tile's rows 32h .. 32h + 31 (h = t / 128): one 32-bit shared
    // load per row gives both columns (a warp reads 128 contiguous bytes); the
    // 16 code bytes and the 32 / BS block scales of each column are written
    // with as few stores as alignment allows.
    {
      const int p = t & 127, h = t >> 7;
      const int64_t kc = k0 + 2 * p;                    // cols % 8 == 0: kc + 1 < cols too
      const int64_t mh = m0 + 32 * h;                   // first x row of this half
      if (kc < cols && mh < rows) {
        constexpr int NB = 32 / BS;                     // blocks per column in a half
        uint32_t cw[2][4];                              // codes, 8 per word, per column
        uint32_t sfw[2] = {0u, 0u};                     // scale byte of block b at 8b
#pragma unroll
        for (int b = 0; b < NB; ++b) {
          const int tr0 = 32 * h + BS * b;              // first tile row of the block
          const int64_t mrow0 = m0 + tr0;
          if (mrow0 >= rows) {                          // rows % BS == 0: whole block out
#pragma unroll
            for (int e = 0; e < 2; ++e)
#pragma unroll
              for (int w = 0; w < BS / 8; ++w) cw[e][b * (BS / 8) + w] = 0u;
            continue;
          }
          uint32_t raw[BS];
#pragma unroll
          for (int q = 0; q < BS; ++q)
            raw[q] = *reinterpret_cast<const uint32_t*>(&tile[buf][tr0 + q][2 * p]);
          // sign bytes of both columns, 4 rows per word (stochastic rounding
          // without rotation takes them from the BF16 pairs directly)
          uint32_t sgn[2][BS / 4];
          if constexpr (SR_C && RHT_C == 0) {
#pragma unroll
            for (int g = 0; g < BS / 4; ++g) {
              const uint32_t P = prmt(raw[4 * g], raw[4 * g + 1], 0xFDB9u);
              const uint32_t Q = prmt(raw[4 * g + 2], raw[4 * g + 3], 0xFDB9u);
              sgn[0][g] = prmt(P, Q, 0x6420u);
              sgn[1][g] = prmt(P, Q, 0x7531u);
            }
          }
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            float v[BS];
#pragma unroll
            for (int q = 0; q < BS; ++q)
              v[q] = __uint_as_float(e ? (raw[q] & 0xFFFF0000u) : (raw[q] << 16));
            if constexpr (RHT_C > 0) {
#pragma unroll
              for (int q = 0; q < RHT_C; ++q)
                if ((mask_c >> q) & 1u) v[q] = -v[q];
#pragma unroll
              for (int hh = 1; hh < RHT_C; hh <<= 1) {
#pragma unroll
                for (int q = 0; q < RHT_C; ++q) {
                  if (q & hh) continue;
                  const float x0 = v[q], x1 = v[q + hh];
                  v[q] = __fadd_rn(x0, x1);
                  v[q + hh] = __fsub_rn(x0, x1);
                }
              }
              const float cn = rht_scale<RHT_C>();
#pragma unroll
              for (int q = 0; q < RHT_C; ++q) v[q] = __fmul_rn(v[q], cn);
            }
            float bmax = 0.0f;
#pragma unroll
            for (int q = 0; q < BS; ++q) bmax = fmaxf(bmax, fabsf(v[q]));
            uint32_t sf;
            float inv;
            block_scale<NV>(bmax, se_c, inv_tab[1], sf, inv);
            sfw[e] |= sf << (8 * b);
            if constexpr (!SR_C) {
#pragma unroll
              for (int q = 0; q < BS; ++q) v[q] = __fmul_rn(v[q], inv);
#pragma unroll
              for (int w = 0; w < BS / 8; ++w) cw[e][b * (BS / 8) + w] = e2m1x8_rn(&v[8 * w]);
            } else {
              // element (kc + e, mrow0 + q) of x^T: draw index (kc + e) * rows + mrow0 + q,
              // a multiple of 8 at q = 0
              const uint64_t i0 = (uint64_t)(kc + e) * (uint64_t)rows + (uint64_t)mrow0;
#pragma unroll
              for (int w = 0; w < BS / 8; ++w) {
                const U4 d = philox_keyed((i0 >> 3) + w, stream_c, K);
                if constexpr (RHT_C > 0) {
#pragma unroll
                  for (int q = 0; q < 8; ++q) v[8 * w + q] = __fmul_rn(v[8 * w + q], inv);
                  cw[e][b * (BS / 8) + w] = e2m1x8_sr(&v[8 * w], d);
                } else {
                  float a[8];
#pragma unroll
                  for (int q = 0; q < 8; ++q) a[q] = __fmul_rn(fabsf(v[8 * w + q]), inv);
                  cw[e][b * (BS / 8) + w] = e2m1x8_sr_mag(a, sgn[e][2 * w], sgn[e][2 * w + 1], d);
                }
              }
            }
          }
        }
        const int64_t left = rows - mh;                 // valid rows in this half (> 0)
        const int nvalid = left >= 32 ? NB : (int)(left / BS);
        const int64_t sb0 = mh / BS;                    // first block of this half
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int64_t k = kc + e;
          uint8_t* dst = codes_c + k * (rows >> 1) + (mh >> 1);
          if (nvalid == NB && ((rows >> 1) & 15) == 0) {  // 16-byte aligned row of x^T
            *reinterpret_cast<uint4*>(dst) = make_uint4(cw[e][0], cw[e][1], cw[e][2], cw[e][3]);
          } else {                                         // rows % 16 == 0: 8-byte aligned
            *reinterpret_cast<uint2*>(dst) = make_uint2(cw[e][0], cw[e][1]);
            if (left > 16) *reinterpret_cast<uint2*>(dst + 8) = make_uint2(cw[e][2], cw[e][3]);
          }
          if (scales_c != nullptr) {
            uint8_t* sd = scales_c + k * S_c + sb0;
            if (NB == 2 && nvalid == 2 && (reinterpret_cast<uintptr_t>(sd) & 1) == 0)
              *reinterpret_cast<uint16_t*>(sd) = (uint16_t)sfw[e];
            else
              for (int b = 0; b < nvalid; ++b) sd[b] = (uint8_t)(sfw[e] >> (8 * b));
          }
          if (mma_c != nullptr) {
            // NVFP4: sb0 % 4 is 0 or 2, so both bytes share one 4-byte slot group
            uint8_t* md = mma_c + mma_sf_offset(k, sb0, S_c4);
            if (NB == 2 && nvalid == 2) *reinterpret_cast<uint16_t*>(md) = (uint16_t)sfw[e];
            else for (int b = 0; b < nvalid; ++b) md[b] = (uint8_t)(sfw[e] >> (8 * b));
          }
        }
      }
    }
    __syncthreads();          // all reads of this buffer done before it is refilled
  }
}

int grid_for(int64_t work_items, int per_block, int max_blocks_per_sm) {
  int64_t need = (work_items + per_block - 1) / per_block;
  const int64_t cap = (int64_t)sm_count() * max_blocks_per_sm;
  if (need > cap) need = cap;
  if (need < 1) need = 1;
  return (int)need;
}

}  // namespace

// ---------------------------------------------------------------------------
// Launchers
// ---------------------------------------------------------------------------
cudaError_t launch_amax_rows(const void* x, int64_t rows, int64_t cols, int64_t ld, int rht_n,
                             uint32_t mask, float* amax, cudaStream_t s) {
  auto xp = static_cast<const __nv_bfloat16*>(x);
  if (rht_n == 0) {
    const int g = grid_for(rows * (cols / 8), kThreads * 4, 8);
    amax_plain_kernel<<<g, kThreads, 0, s>>>(xp, rows, cols, ld, amax);
    count_launches(1);
    return cudaGetLastError();
  }
  const int64_t segs = ((cols / 8) + 32 * kRowChunks - 1) / (32 * kRowChunks);
  const int grid = grid_for(rows * segs, kThreads / 32, 8);
  if (rht_n == 16) amax_rows_kernel<16><<<grid, kThreads, 0, s>>>(xp, rows, cols, ld, mask, amax);
  else if (rht_n == 32) amax_rows_kernel<32><<<grid, kThreads, 0, s>>>(xp, rows, cols, ld, mask, amax);
  else amax_rows_kernel<0><<<grid, kThreads, 0, s>>>(xp, rows, cols, ld, mask, amax);
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_amax_cols_rht(const void* x, int64_t rows, int64_t cols, int64_t ld,
                                 int rht_n, uint32_t mask, float* amax_col, float* amax_plain,
                                 cudaStream_t s) {
  auto xp = static_cast<const __nv_bfloat16*>(x);
  const int64_t units = (rows / rht_n) * ((cols + 255) / 256);
  const int grid = grid_for(units, kThreads / 32, 8);
  if (rht_n != 16) return cudaErrorInvalidValue;   // 16-point blocks only (NVFP4)
  amax_cols_rht_kernel<16><<<grid, kThreads, 0, s>>>(xp, rows, cols, ld, mask, amax_col, amax_plain);
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_amax_cols(const void* x, int64_t rows, int64_t cols, int64_t ld, int rht_n,
                             uint32_t mask, float* amax, cudaStream_t s) {
  const int64_t ntiles = ((rows + kTile - 1) / kTile) * ((cols + kTile - 1) / kTile);
  const int grid = grid_for(ntiles, 1, 16);
  auto xp = static_cast<const __nv_bfloat16*>(x);
#define FP4_AMAXC(N) quant_cols_kernel<16, N, false, true><<<grid, kColThreads, 0, s>>>( \
      xp, rows, cols, ld, mask, 0, 0, nullptr, amax, nullptr, nullptr, nullptr, nullptr, nullptr)
  if (rht_n == 16) FP4_AMAXC(16);
  else if (rht_n == 32) FP4_AMAXC(32);
  else FP4_AMAXC(0);
#undef FP4_AMAXC
  count_launches(1);
  return cudaGetLastError();
}

template <int BS, int RHT_N, bool SR, bool QUEST = false>
static void rows_variant(const RowQuantArgs& a, int grid, cudaStream_t s) {
  quant_rows_kernel<BS, RHT_N, SR, QUEST><<<grid, kThreads, 0, s>>>(
      static_cast<const __nv_bfloat16*>(a.x), a.rows, a.cols, a.ld, a.rht_mask, philox_keys(a.sr_seed),
      a.sr_stream, a.amax_src, a.amax_out, a.s_dec, a.codes, a.scales, a.scales_mma, a.status);
}

template <int BS, int RHT_N, bool SR>
static void cols_variant(const RowQuantArgs& a, int grid, cudaStream_t s) {
  quant_cols_kernel<BS, RHT_N, SR, false><<<grid, kColThreads, 0, s>>>(
      static_cast<const __nv_bfloat16*>(a.x), a.rows, a.cols, a.ld, a.rht_mask, a.sr_seed,
      a.sr_stream, a.amax_src, a.amax_out, a.s_dec, a.codes, a.scales, a.scales_mma, a.status);
}

#define FP4_DISPATCH(FN, a, grid, s)                                                    \
  do {                                                                                  \
    const bool sr = (a).round == FP4_SR;                                                \
    if ((a).fmt == FP4_NVFP4) {                                                         \
      if ((a).rht_n == 16) { sr ? FN<16, 16, true>(a, grid, s) : FN<16, 16, false>(a, grid, s); } \
      else if ((a).rht_n == 32) { sr ? FN<16, 32, true>(a, grid, s) : FN<16, 32, false>(a, grid, s); } \
      else { sr ? FN<16, 0, true>(a, grid, s) : FN<16, 0, false>(a, grid, s); }          \
    } else {                                                                            \
      if ((a).rht_n == 16) { sr ? FN<32, 16, true>(a, grid, s) : FN<32, 16, false>(a, grid, s); } \
      else if ((a).rht_n == 32) { sr ? FN<32, 32, true>(a, grid, s) : FN<32, 32, false>(a, grid, s); } \
      else { sr ? FN<32, 0, true>(a, grid, s) : FN<32, 0, false>(a, grid, s); }          \
    }                                                                                   \
  } while (0)

cudaError_t launch_quant_rows(const RowQuantArgs& a, cudaStream_t s) {
  const int64_t segs = ((a.cols / 8) + 32 * kRowChunks - 1) / (32 * kRowChunks);
  const int grid = grid_for(a.rows * segs, kThreads / 32, 8);
  if (a.round == FP4_QUEST) {       // MXFP4 only (checked by the caller)
    if (a.rht_n == 32) rows_variant<32, 32, false, true>(a, grid, s);
    else if (a.rht_n == 16) rows_variant<32, 16, false, true>(a, grid, s);
    else rows_variant<32, 0, false, true>(a, grid, s);
    count_launches(1);
    return cudaGetLastError();
  }
  FP4_DISPATCH(rows_variant, a, grid, s);
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_quant_cols(const RowQuantArgs& a, cudaStream_t s) {
  const int64_t ntiles = ((a.rows + kTile - 1) / kTile) * ((a.cols + kTile - 1) / kTile);
  const int grid = grid_for(ntiles, 1, 16);
  FP4_DISPATCH(cols_variant, a, grid, s);
  count_launches(1);
  return cudaGetLastError();
}

template <int BS, int RR, int RC, bool SRR, bool SRC, bool QR = false>
static cudaError_t dual_variant(const DualQuantArgs& a, cudaStream_t s) {
  auto kern = quant_dual_kernel<BS, RR, RC, SRR, SRC, QR>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kDualSmem);
  if (e != cudaSuccess) return e;
  const int64_t ntiles = ((a.rows + kDualTM - 1) / kDualTM) * ((a.cols + kDualTK - 1) / kDualTK);
  const int grid = grid_for(ntiles, 1, dual_ctas_per_sm<BS, SRR, SRC>());
  kern<<<grid, kDualThreads, kDualSmem, s>>>(
      static_cast<const __nv_bfloat16*>(a.x), a.rows, a.cols, a.ld, a.mask_r, a.mask_c,
      philox_keys(a.sr_seed), a.stream_r, a.stream_c, a.amax_src_r, a.amax_src_c, a.amax_out_r,
      a.amax_out_c, a.s_dec_r,
      a.s_dec_c, a.codes_r, a.scales_r, a.mma_r, a.codes_c, a.scales_c, a.mma_c, a.status);
  count_launches(1);
  return cudaGetLastError();
}

template <int BS, int RR, int RC>
static cudaError_t dual_rounding(const DualQuantArgs& a, cudaStream_t s) {
  if constexpr (BS == 32) {
    if (a.quest_r) return a.sr_c ? dual_variant<BS, RR, RC, false, true, true>(a, s)
                                 : dual_variant<BS, RR, RC, false, false, true>(a, s);
  }
  if (a.sr_r) return a.sr_c ? dual_variant<BS, RR, RC, true, true>(a, s)
                            : dual_variant<BS, RR, RC, true, false>(a, s);
  return a.sr_c ? dual_variant<BS, RR, RC, false, true>(a, s)
                : dual_variant<BS, RR, RC, false, false>(a, s);
}

bool dual_supported(int fmt, int rht_r, int rht_c) {
  const int n = fmt == FP4_NVFP4 ? 16 : 32;
  return (rht_r == 0 || rht_r == n) && (rht_c == 0 || rht_c == n);
}

cudaError_t launch_quant_dual(const DualQuantArgs& a, cudaStream_t s) {
  if (a.fmt == FP4_NVFP4) {
    if (a.rht_r) return a.rht_c ? dual_rounding<16, 16, 16>(a, s) : dual_rounding<16, 16, 0>(a, s);
    return a.rht_c ? dual_rounding<16, 0, 16>(a, s) : dual_rounding<16, 0, 0>(a, s);
  }
  if (a.rht_r) return a.rht_c ? dual_rounding<32, 32, 32>(a, s) : dual_rounding<32, 32, 0>(a, s);
  return a.rht_c ? dual_rounding<32, 0, 32>(a, s) : dual_rounding<32, 0, 0>(a, s);
}

cudaError_t launch_quant_2d(const Quant2DArgs& a, cudaStream_t s) {
  const int64_t ntiles = ((a.rows + kTile - 1) / kTile) * ((a.cols + kTile - 1) / kTile);
  const int grid = grid_for(ntiles, 1, 8);
  quant_2d_kernel<<<grid, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(a.x), a.rows, a.cols,
                                       a.ld, a.amax_src, a.s_dec, a.s_dec_t, a.amax_out,
                                       a.amax_out_t, a.codes,
                                       a.scales, a.scales_mma, a.codes_t, a.scales_t,
                                       a.scales_mma_t, a.status);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace fp4impl
