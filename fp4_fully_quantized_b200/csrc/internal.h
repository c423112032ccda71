// internal.h -- launchers shared between the C-ABI layer and the kernels.
#pragma once
#include <cstdint>
#include <cuda_runtime.h>

#include "fp4.h"

namespace fp4impl {

// Status block at the start of every workspace.
struct DeviceStatus {
  uint32_t code;         // first device-detected fp4_status, 0 = none
  uint32_t where;        // kernel-specific detail (e.g. which wait expired)
  uint32_t pad[62];
};
static_assert(sizeof(DeviceStatus) == 256, "status block is 256 bytes");

int sm_count();

// Counts kernel launches enqueued by this library (fp4_kernel_launches).
void count_launches(uint64_t n);

// Records `code` into the status word unless one is already set.
__device__ __forceinline__ void set_status(uint32_t* status, uint32_t code, uint32_t where) {
  if (status != nullptr && atomicCAS(status, 0u, code) == 0u) status[1] = where;
}

// --- quantizer launchers (quantize.cu) ------------------------------------
struct RowQuantArgs {
  const void* x; int64_t rows, cols, ld;
  int fmt, round, rht_n; uint32_t rht_mask;
  uint64_t sr_seed; uint32_t sr_stream;
  const float* amax_src;   // NVFP4: amax to encode with
  float* amax_out;         // NVFP4: written with *amax_src when != amax_src
  float* s_dec;            // written (NVFP4: amax/2688; MXFP4: 1)
  uint8_t* codes; uint8_t* scales; uint8_t* scales_mma;
  uint32_t* status;
};

cudaError_t launch_amax_rows(const void* x, int64_t rows, int64_t cols, int64_t ld,
                             int rht_n, uint32_t rht_mask, float* amax, cudaStream_t s);
cudaError_t launch_amax_cols(const void* x, int64_t rows, int64_t cols, int64_t ld,
                             int rht_n, uint32_t rht_mask, float* amax, cudaStream_t s);
// Amax of x rotated down its columns (16-row Hadamard blocks; rows must be a
// multiple of 16; other block sizes return an error) and, when amax_plain is
// not NULL, the plain amax, from one read.  Both destinations must be zeroed
// first.
cudaError_t launch_amax_cols_rht(const void* x, int64_t rows, int64_t cols, int64_t ld,
                                 int rht_n, uint32_t rht_mask, float* amax_col,
                                 float* amax_plain, cudaStream_t s);
cudaError_t launch_quant_rows(const RowQuantArgs& a, cudaStream_t s);
// Transposed output: the quantized operand is x^T ([cols, rows]); rows of x
// are the blocked dimension.  Fields keep the meaning of RowQuantArgs with
// rows/cols those of x.
cudaError_t launch_quant_cols(const RowQuantArgs& a, cudaStream_t s);
// Row-wise and transposed outputs from one read of x (both outputs 1-D
// blocks of the same format).  Supported Hadamard sizes: 0 or the format's
// block size (16 NVFP4, 32 MXFP4) on either output.
struct DualQuantArgs {
  const void* x; int64_t rows, cols, ld;
  int fmt, rht_r, rht_c; bool sr_r, sr_c;
  bool quest_r;            // MXFP4 row-wise output: QuEST-style (RMS-based) block scale
  uint32_t mask_r, mask_c;
  uint64_t sr_seed; uint32_t stream_r, stream_c;
  const float* amax_src_r; const float* amax_src_c;   // NVFP4 (ignored for MXFP4)
  float* amax_out_r; float* amax_out_c; float* s_dec_r; float* s_dec_c;
  uint8_t* codes_r; uint8_t* scales_r; uint8_t* mma_r;
  uint8_t* codes_c; uint8_t* scales_c; uint8_t* mma_c;
  uint32_t* status;
};
bool dual_supported(int fmt, int rht_r, int rht_c);
cudaError_t launch_quant_dual(const DualQuantArgs& a, cudaStream_t s);
// NVFP4 16x16 tiles: W (codes/scales/scales_mma) and W^T (codes_t/...).
struct Quant2DArgs {
  const void* x; int64_t rows, cols, ld;
  const float* amax_src; float* s_dec; float* s_dec_t; float* amax_out; float* amax_out_t;
  uint8_t* codes; uint8_t* scales; uint8_t* scales_mma;
  uint8_t* codes_t; uint8_t* scales_t; uint8_t* scales_mma_t;
  uint32_t* status;
};
cudaError_t launch_quant_2d(const Quant2DArgs& a, cudaStream_t s);

// --- GEMM (gemm_sfst.cu) ----------------------------------------------------
struct GemmArgs {
  const uint8_t* a_codes; const uint8_t* a_sf; const float* a_sdec;
  const uint8_t* b_codes; const uint8_t* b_sf; const float* b_sdec;
  int64_t M, N, K;
  int fmt;               // FP4_NVFP4 / FP4_MXFP4
  float alpha;
  void* c; int64_t ldc; int out_mode;    // 0 BF16, 1 FP32, 2 NVFP4 1x16 RTN into q_*
  float* c_amax;
  // out_mode 2: the quantized output [M, N] and the supplied tensor amax
  uint8_t* q_codes; uint8_t* q_scales; uint8_t* q_scales_mma;
  const float* q_amax_in; float* q_amax_out; float* q_s_dec;
  int q_sr; uint64_t q_seed; uint32_t q_stream;   // out_mode 2 rounding
  uint32_t* status;
};
fp4_status gemm_launch(const GemmArgs& g, cudaStream_t s);
// Every argument check of fp4_gemm, with nothing enqueued (api.cu).
fp4_status gemm_validate(const fp4_qtensor* a, const fp4_qtensor* b, const void* c, int64_t ldc,
                         int32_t out_dtype, const void* ws, size_t ws_bytes);

}  // namespace fp4impl
