// noise.cu -- gradient-norm vs quantization-noise diagnostic.
//
// The "FP4 All the Way" page (Summary) states that quantized training stops
// being effective below a threshold set by the gradient norm relative to the
// quantization noise.  The page gives no formula, so the library reports the
// two quantities: sum x^2 and sum (deq(q) - x)^2 for a BF16 tensor x and its
// row-wise quantization q, accumulated in double.  deq is exact in double:
// an E2M1 level (3 significant bits) times an E4M3 (4 bits) or power-of-two
// block scale times the FP32 decode scale.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "fp4_device.cuh"
#include "internal.h"

namespace fp4impl {
using namespace fp4dev;
namespace {

__device__ __forceinline__ double e2m1_level(uint32_t code) {
  // 0, 0.5, 1, 1.5, 2, 3, 4, 6 for codes 0..7; bit 3 is the sign
  const uint32_t m = code & 7u;
  const double mag = m < 4u ? 0.5 * (double)m : (double)(1u << ((m >> 1) - 1u)) * (m & 1u ? 1.5 : 1.0);
  return (code & 8u) ? -mag : mag;
}

__device__ __forceinline__ double warp_sum(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
  return v;
}

// One thread per 8 consecutive elements of a row (one 16-byte load of x, one
// 4-byte load of codes).  BS = 16 (NVFP4, E4M3 scale) or 32 (MXFP4, E8M0).
template <int BS>
__global__ void __launch_bounds__(256)
quant_noise_kernel(const __nv_bfloat16* __restrict__ x, int64_t rows, int64_t cols, int64_t ld,
                   const uint8_t* __restrict__ codes, const uint8_t* __restrict__ scales,
                   const uint8_t* __restrict__ scales_mma, int scales_rows_per_entry,
                   const float* __restrict__ s_dec, double* sums) {
  const int64_t cpr = cols >> 3, total = rows * cpr;
  const int64_t S = cols / BS, S4 = (S + 3) & ~3LL;
  const double sd = (double)*s_dec;
  double sx = 0.0, sn = 0.0;
  for (int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; g < total;
       g += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = g / cpr, j = g - r * cpr;
    float v[8];
    bf16x8_to_f32(ld_nc_v4(x + r * ld + j * 8), v);
    const uint32_t cw = *reinterpret_cast<const uint32_t*>(codes + r * (cols >> 1) + j * 4);
    const int64_t sb = (j * 8) / BS;
    const uint32_t sf = scales_mma != nullptr
                            ? scales_mma[mma_sf_offset(r, sb, S4)]
                            : scales[(r / scales_rows_per_entry) * S + sb];
    const double scale = (BS == 16) ? (double)e4m3_value(sf) : ldexp(1.0, (int)sf - 127);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const double xv = (double)v[i];
      const double d = e2m1_level((cw >> (4 * i)) & 15u) * scale * sd - xv;
      sx += xv * xv;
      sn += d * d;
    }
  }
  sx = warp_sum(sx);
  sn = warp_sum(sn);
  if ((threadIdx.x & 31) == 0) {
    atomicAdd(sums, sx);
    atomicAdd(sums + 1, sn);
  }
}

}  // namespace
}  // namespace fp4impl

using namespace fp4impl;

extern "C" fp4_status fp4_quant_noise(const void* x_bf16, int64_t rows, int64_t cols, int64_t ld,
                                      const fp4_qtensor* q, double* sums, void* ws,
                                      size_t ws_bytes, void* stream) {
  (void)ws;
  (void)ws_bytes;
  if (q == nullptr || sums == nullptr) return FP4_ERR_NULL;
  if (rows < 0 || cols < 0 || ld < cols || (ld % 8) != 0) return FP4_ERR_SHAPE;
  const bool empty = rows == 0 || cols == 0;
  if (!empty && (x_bf16 == nullptr || q->codes == nullptr || q->s_dec == nullptr ||
                 (q->scales == nullptr && q->scales_mma == nullptr)))
    return FP4_ERR_NULL;
  if (q->rows != rows || q->cols != cols) return FP4_ERR_SHAPE;
  if (q->fmt != FP4_NVFP4 && q->fmt != FP4_MXFP4) return FP4_ERR_FORMAT;
  if (q->block == FP4_BLOCK_2D && q->fmt != FP4_NVFP4) return FP4_ERR_FORMAT;
  const int bs = q->fmt == FP4_MXFP4 ? 32 : 16;
  if (cols % bs) return FP4_ERR_SHAPE;
  if (q->block == FP4_BLOCK_2D && (rows % 16)) return FP4_ERR_SHAPE;
  if ((reinterpret_cast<uintptr_t>(x_bf16) & 15u) || (reinterpret_cast<uintptr_t>(q->codes) & 3u) ||
      (reinterpret_cast<uintptr_t>(sums) & 7u))
    return FP4_ERR_ALIGN;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(sums, 0, 2 * sizeof(double), s) != cudaSuccess) return FP4_ERR_CUDA;
  if (empty) return FP4_OK;
  const int64_t chunks = rows * (cols / 8);
  const int grid = (int)((chunks + 255) / 256 < (int64_t)sm_count() * 8 ? (chunks + 255) / 256
                                                                        : (int64_t)sm_count() * 8);
  const int rpe = q->block == FP4_BLOCK_2D ? 16 : 1;    // logical 2-D scales: one per 16 rows
  const auto* xp = static_cast<const __nv_bfloat16*>(x_bf16);
  if (bs == 16)
    quant_noise_kernel<16><<<grid, 256, 0, s>>>(xp, rows, cols, ld, q->codes, q->scales,
                                                 q->scales_mma, rpe, q->s_dec, sums);
  else
    quant_noise_kernel<32><<<grid, 256, 0, s>>>(xp, rows, cols, ld, q->codes, q->scales,
                                                 q->scales_mma, rpe, q->s_dec, sums);
  count_launches(1);
  return cudaGetLastError() == cudaSuccess ? FP4_OK : FP4_ERR_CUDA;
}
