// api.cu -- the C ABI of libfp4fqt.so: argument checking and orchestration.
//
// Every entry point validates its arguments before enqueuing anything and
// returns a status; device work is enqueued on the caller's stream only.
// The linear-layer entry points compose fp4_quantize and fp4_gemm in the
// order of a fully quantized linear layer: "FP4 All the Way", Key points
// (round-to-nearest forward, stochastic rounding in backward and update)
// and "Quartet", Abstract (fprop, dgrad and wgrad all in FP4).
#include <cuda_runtime.h>

#include <atomic>
#include <climits>
#include <cstdint>
#include <cstring>

#include "fp4.h"
#include "fp4_device.cuh"
#include "internal.h"

namespace fp4impl {

int sm_count() {
  // per-device cache; threads that race here store the same value
  static std::atomic<int> cached[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  int n = cached[dev].load(std::memory_order_relaxed);
  if (n == 0) {
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    cached[dev].store(n, std::memory_order_relaxed);
  }
  return n;
}

static std::atomic<uint64_t> g_launches{0};
void count_launches(uint64_t n) { g_launches.fetch_add(n, std::memory_order_relaxed); }

}  // namespace fp4impl

using namespace fp4impl;

namespace {

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline int block_size(int32_t fmt) { return fmt == FP4_MXFP4 ? 32 : 16; }
inline uint32_t* status_ptr(void* ws) { return static_cast<uint32_t*>(ws); }
inline cudaStream_t as_stream(void* s) { return static_cast<cudaStream_t>(s); }

fp4_status check_qtensor(const fp4_qtensor* q, int64_t rows, int64_t cols, int32_t fmt,
                         int32_t block) {
  const bool empty = rows == 0 || cols == 0;   // nothing to encode: buffers may be NULL
  if (q->codes == nullptr && !empty) return FP4_ERR_NULL;
  if (q->scales == nullptr && q->scales_mma == nullptr && !empty) return FP4_ERR_NULL;
  if (q->s_dec == nullptr) return FP4_ERR_NULL;
  if (fmt == FP4_NVFP4 && q->amax == nullptr) return FP4_ERR_NULL;
  if (q->rows != rows || q->cols != cols) return FP4_ERR_SHAPE;
  if (q->fmt != fmt || q->block != block) return FP4_ERR_FORMAT;
  if (!aligned16(q->codes)) return FP4_ERR_ALIGN;
  if (((reinterpret_cast<uintptr_t>(q->amax)) & 3u) || ((reinterpret_cast<uintptr_t>(q->s_dec)) & 3u))
    return FP4_ERR_ALIGN;
  return FP4_OK;
}

fp4_status cuda_status(cudaError_t e) { return e == cudaSuccess ? FP4_OK : FP4_ERR_CUDA; }

}  // namespace

extern "C" {

int32_t fp4_abi_version(void) { return FP4_ABI_VERSION; }

uint64_t fp4_kernel_launches(void) { return g_launches.load(std::memory_order_relaxed); }

const char* fp4_status_str(int32_t s) {
  switch (s) {
    case FP4_OK: return "ok";
    case FP4_ERR_NULL: return "a required pointer is NULL";
    case FP4_ERR_SHAPE: return "sizes violate the divisibility rules";
    case FP4_ERR_ALIGN: return "a pointer or leading dimension is not aligned";
    case FP4_ERR_FORMAT: return "inconsistent format, block or rounding request";
    case FP4_ERR_WORKSPACE: return "workspace missing or too small";
    case FP4_ERR_CUDA: return "a CUDA call or kernel launch failed";
    case FP4_ERR_NONFINITE: return "a tensor amax was Inf or NaN";
    case FP4_ERR_TIMEOUT: return "a bounded wait inside a GEMM expired";
    case FP4_ERR_UNSUPPORTED: return "request not supported by this build";
    default: return "unknown status";
  }
}

void fp4_qtensor_sizes(int64_t rows, int64_t cols, int32_t fmt, int32_t block,
                       size_t* codes_bytes, size_t* scales_bytes, size_t* scales_mma_bytes) {
  const int bs = block_size(fmt);
  const int64_t S = cols / bs;
  if (codes_bytes) *codes_bytes = (size_t)(rows * (cols / 2));
  if (scales_bytes) {
    if (fmt == FP4_NVFP4 && block == FP4_BLOCK_2D) *scales_bytes = (size_t)((rows / 16) * (cols / 16));
    else *scales_bytes = (size_t)(rows * S);
  }
  if (scales_mma_bytes) {
    const int64_t r128 = (rows + 127) / 128 * 128, s4 = (S + 3) / 4 * 4;
    *scales_mma_bytes = (size_t)(r128 * s4);
  }
}

void fp4_qparams_default(fp4_qparams* p) {
  if (!p) return;
  std::memset(p, 0, sizeof(*p));
  p->fmt = FP4_NVFP4;
  p->block = FP4_BLOCK_1D;
  p->round = FP4_RTN;
  p->round_t = FP4_RTN;
}

size_t fp4_workspace_bytes(int64_t M, int64_t N, int64_t K) {
  (void)M; (void)N; (void)K;
  return sizeof(DeviceStatus);
}

// fp4_quantize; with `dry` it only validates the arguments and returns at the
// point where the first copy or kernel would be enqueued.
static fp4_status quantize_impl(const void* x, int64_t rows, int64_t cols, int64_t ld,
                                const fp4_qparams* p, fp4_qtensor* out, fp4_qtensor* out_t,
                                void* ws, size_t ws_bytes, void* stream, bool dry) {
  if (p == nullptr) return FP4_ERR_NULL;
  if (out == nullptr && out_t == nullptr) return FP4_ERR_NULL;
  if (ws != nullptr && ws_bytes < sizeof(DeviceStatus)) return FP4_ERR_WORKSPACE;
  if (rows < 0 || cols < 0 || ld < cols) return FP4_ERR_SHAPE;
  const bool empty_x = rows == 0 || cols == 0;    // x may then be NULL
  if (x == nullptr && !empty_x) return FP4_ERR_NULL;
  if ((!empty_x && !aligned16(x)) || (ld % 8) != 0) return FP4_ERR_ALIGN;
  if (p->fmt != FP4_NVFP4 && p->fmt != FP4_MXFP4) return FP4_ERR_FORMAT;
  if (p->block != FP4_BLOCK_1D && p->block != FP4_BLOCK_2D) return FP4_ERR_FORMAT;
  if (p->block == FP4_BLOCK_2D && p->fmt != FP4_NVFP4) return FP4_ERR_FORMAT;
  if ((p->round != FP4_RTN && p->round != FP4_SR && p->round != FP4_QUEST) ||
      (p->round_t != FP4_RTN && p->round_t != FP4_SR && p->round_t != FP4_QUEST))
    return FP4_ERR_FORMAT;
  // the QuEST-style scale is defined for MXFP4 row-wise (forward) outputs
  if (p->round == FP4_QUEST && (p->fmt != FP4_MXFP4 || p->block != FP4_BLOCK_1D))
    return FP4_ERR_UNSUPPORTED;
  if (out_t != nullptr && p->round_t == FP4_QUEST) return FP4_ERR_UNSUPPORTED;
  for (int n : {p->rht_n, p->rht_n_t})
    if (n != 0 && n != 16 && n != 32) return FP4_ERR_FORMAT;
  const int bs = block_size(p->fmt);
  uint32_t* status = ws ? status_ptr(ws) : nullptr;
  cudaStream_t s = as_stream(stream);

  if (p->block == FP4_BLOCK_2D) {
    if (p->round != FP4_RTN || p->rht_n != 0 || (out_t && (p->round_t != FP4_RTN || p->rht_n_t != 0)))
      return FP4_ERR_UNSUPPORTED;   // 2-D tiles: round-to-nearest weights, no rotation
    if (rows % 16 || cols % 16) return FP4_ERR_SHAPE;
    fp4_status st;
    if (out && (st = check_qtensor(out, rows, cols, FP4_NVFP4, FP4_BLOCK_2D)) != FP4_OK) return st;
    if (out_t && (st = check_qtensor(out_t, cols, rows, FP4_NVFP4, FP4_BLOCK_2D)) != FP4_OK) return st;
    if (dry) return FP4_OK;
    float* amax_dst = out ? out->amax : out_t->amax;
    const float* src = p->amax_in;
    if (src == nullptr) {
      if (cudaMemsetAsync(amax_dst, 0, sizeof(float), s) != cudaSuccess) return FP4_ERR_CUDA;
      if (launch_amax_rows(x, rows, cols, ld, 0, 0, amax_dst, s) != cudaSuccess) return FP4_ERR_CUDA;
      src = amax_dst;
    }
    Quant2DArgs a{};
    a.x = x; a.rows = rows; a.cols = cols; a.ld = ld; a.amax_src = src;
    a.s_dec = out ? out->s_dec : nullptr;
    a.s_dec_t = out_t ? out_t->s_dec : nullptr;
    a.amax_out = out ? out->amax : nullptr;
    a.amax_out_t = out_t ? out_t->amax : nullptr;
    if (out) { a.codes = out->codes; a.scales = out->scales; a.scales_mma = out->scales_mma; }
    if (out_t) { a.codes_t = out_t->codes; a.scales_t = out_t->scales; a.scales_mma_t = out_t->scales_mma; }
    a.status = status;
    return cuda_status(launch_quant_2d(a, s));
  }

  // 1-D blocks
  fp4_status st;
  if (out) {
    if (cols % bs) return FP4_ERR_SHAPE;
    if (p->rht_n && cols % p->rht_n) return FP4_ERR_SHAPE;
    if ((st = check_qtensor(out, rows, cols, p->fmt, FP4_BLOCK_1D)) != FP4_OK) return st;
  }
  if (out_t) {
    if (rows % bs || cols % 8) return FP4_ERR_SHAPE;
    if (p->rht_n_t && rows % p->rht_n_t) return FP4_ERR_SHAPE;
    if ((st = check_qtensor(out_t, cols, rows, p->fmt, FP4_BLOCK_1D)) != FP4_OK) return st;
  }
  if (dry) return FP4_OK;
  const uint32_t mask = p->rht_n ? fp4dev::rht_sign_mask(p->rht_seed, p->rht_n) : 0u;
  const uint32_t mask_t = p->rht_n_t ? fp4dev::rht_sign_mask(p->rht_seed, p->rht_n_t) : 0u;
  const bool nv = p->fmt == FP4_NVFP4;

  // Tensor amax of each requested output (NVFP4 only).
  const float* src_row = nullptr;
  const float* src_col = nullptr;
  const bool fused_amax = nv && out && out_t && p->amax_in == nullptr &&
                          p->amax_in_t == nullptr && p->rht_n == 0 && p->rht_n_t == 16;
  if (fused_amax) {
    // plain amax for the row-wise output and the amax of the column-rotated
    // tensor for the transposed one, from one read of x
    if (cudaMemsetAsync(out->amax, 0, sizeof(float), s) != cudaSuccess ||
        cudaMemsetAsync(out_t->amax, 0, sizeof(float), s) != cudaSuccess)
      return FP4_ERR_CUDA;
    if (launch_amax_cols_rht(x, rows, cols, ld, 16, mask_t, out_t->amax, out->amax, s) != cudaSuccess)
      return FP4_ERR_CUDA;
    src_row = out->amax;
    src_col = out_t->amax;
  }
  if (nv && out && !fused_amax) {
    src_row = p->amax_in;
    if (src_row == nullptr) {
      if (cudaMemsetAsync(out->amax, 0, sizeof(float), s) != cudaSuccess) return FP4_ERR_CUDA;
      if (launch_amax_rows(x, rows, cols, ld, p->rht_n, mask, out->amax, s) != cudaSuccess)
        return FP4_ERR_CUDA;
      src_row = out->amax;
    }
  }
  if (nv && out_t && !fused_amax) {
    src_col = p->amax_in_t;
    if (src_col == nullptr) {
      if (out && p->amax_in == nullptr && p->rht_n == 0 && p->rht_n_t == 0) {
        src_col = out->amax;      // same tensor, same orientation-free amax
      } else {
        if (cudaMemsetAsync(out_t->amax, 0, sizeof(float), s) != cudaSuccess) return FP4_ERR_CUDA;
        cudaError_t e = p->rht_n_t == 16
            ? launch_amax_cols_rht(x, rows, cols, ld, 16, mask_t, out_t->amax, nullptr, s)
            : p->rht_n_t ? launch_amax_cols(x, rows, cols, ld, p->rht_n_t, mask_t, out_t->amax, s)
                         : launch_amax_rows(x, rows, cols, ld, 0, 0, out_t->amax, s);
        if (e != cudaSuccess) return FP4_ERR_CUDA;
        src_col = out_t->amax;
      }
    }
  }

  // Both outputs from one read of x.
  if (out && out_t && dual_supported(p->fmt, p->rht_n, p->rht_n_t)) {
    DualQuantArgs a{};
    a.x = x; a.rows = rows; a.cols = cols; a.ld = ld;
    a.fmt = p->fmt; a.rht_r = p->rht_n; a.rht_c = p->rht_n_t;
    a.sr_r = p->round == FP4_SR; a.sr_c = p->round_t == FP4_SR;
    a.quest_r = p->round == FP4_QUEST;
    a.mask_r = mask; a.mask_c = mask_t;
    a.sr_seed = p->sr_seed; a.stream_r = p->sr_stream; a.stream_c = p->sr_stream_t;
    a.amax_src_r = src_row; a.amax_src_c = src_col;
    a.amax_out_r = out->amax; a.amax_out_c = out_t->amax;
    a.s_dec_r = out->s_dec; a.s_dec_c = out_t->s_dec;
    a.codes_r = out->codes; a.scales_r = out->scales; a.mma_r = out->scales_mma;
    a.codes_c = out_t->codes; a.scales_c = out_t->scales; a.mma_c = out_t->scales_mma;
    a.status = status;
    return cuda_status(launch_quant_dual(a, s));
  }

  if (out) {
    RowQuantArgs a{};
    a.x = x; a.rows = rows; a.cols = cols; a.ld = ld;
    a.fmt = p->fmt; a.round = p->round; a.rht_n = p->rht_n; a.rht_mask = mask;
    a.sr_seed = p->sr_seed; a.sr_stream = p->sr_stream;
    a.amax_src = src_row;
    a.amax_out = out->amax;
    a.s_dec = out->s_dec;
    a.codes = out->codes; a.scales = out->scales; a.scales_mma = out->scales_mma;
    a.status = status;
    if (launch_quant_rows(a, s) != cudaSuccess) return FP4_ERR_CUDA;
  }
  if (out_t) {
    RowQuantArgs a{};
    a.x = x; a.rows = rows; a.cols = cols; a.ld = ld;
    a.fmt = p->fmt; a.round = p->round_t; a.rht_n = p->rht_n_t; a.rht_mask = mask_t;
    a.sr_seed = p->sr_seed; a.sr_stream = p->sr_stream_t;
    a.amax_src = src_col;
    a.amax_out = out_t->amax;
    a.s_dec = out_t->s_dec;
    a.codes = out_t->codes; a.scales = out_t->scales; a.scales_mma = out_t->scales_mma;
    a.status = status;
    if (launch_quant_cols(a, s) != cudaSuccess) return FP4_ERR_CUDA;
  }
  return FP4_OK;
}

fp4_status fp4_quantize(const void* x, int64_t rows, int64_t cols, int64_t ld,
                        const fp4_qparams* p, fp4_qtensor* out, fp4_qtensor* out_t, void* ws,
                        size_t ws_bytes, void* stream) {
  return quantize_impl(x, rows, cols, ld, p, out, out_t, ws, ws_bytes, stream, false);
}

// The GEMM kernel numbers its 128 x 256 output tiles with 32-bit integers and
// steps through them by the grid size (at most a few thousand CTAs): with at
// most 2^30 tiles, tile + gridDim.x never overflows.
static bool gemm_tiles_fit(int64_t M, int64_t N) {
  return (M / 128) * ((N + 255) / 256) <= (int64_t)1 << 30;
}

// fp4_gemm; with `dry` it only validates the arguments.
static fp4_status gemm_impl(const fp4_qtensor* a, const fp4_qtensor* b, float alpha, void* c,
                            int64_t ldc, int32_t out_dtype, float* c_amax, void* ws,
                            size_t ws_bytes, void* stream, bool dry) {
  if (a == nullptr || b == nullptr || c == nullptr) return FP4_ERR_NULL;
  if (a->codes == nullptr || b->codes == nullptr || a->scales_mma == nullptr ||
      b->scales_mma == nullptr || a->s_dec == nullptr || b->s_dec == nullptr)
    return FP4_ERR_NULL;
  if (a->fmt != b->fmt || (a->fmt != FP4_NVFP4 && a->fmt != FP4_MXFP4)) return FP4_ERR_FORMAT;
  if (out_dtype != FP4_OUT_BF16 && out_dtype != FP4_OUT_F32) return FP4_ERR_FORMAT;
  const int64_t M = a->rows, N = b->rows, K = a->cols;
  if (b->cols != K) return FP4_ERR_SHAPE;
  if (M <= 0 || N <= 0 || K <= 0 || M % 128 || N % 128 || K % 64) return FP4_ERR_SHAPE;
  if (M > (1ll << 30) || N > (1ll << 30) || K > (1ll << 30)) return FP4_ERR_SHAPE;
  if (!gemm_tiles_fit(M, N)) return FP4_ERR_SHAPE;
  const int64_t esize = out_dtype == FP4_OUT_F32 ? 4 : 2;
  if (ldc < N || (ldc * esize) % 16 || !aligned16(c)) return FP4_ERR_ALIGN;
  if (!aligned16(a->codes) || !aligned16(b->codes) || !aligned16(a->scales_mma) ||
      !aligned16(b->scales_mma))
    return FP4_ERR_ALIGN;
  if (ws == nullptr || ws_bytes < fp4_workspace_bytes(M, N, K)) return FP4_ERR_WORKSPACE;
  if (dry) return FP4_OK;
  GemmArgs g{};
  g.a_codes = a->codes; g.a_sf = a->scales_mma; g.a_sdec = a->s_dec;
  g.b_codes = b->codes; g.b_sf = b->scales_mma; g.b_sdec = b->s_dec;
  g.M = M; g.N = N; g.K = K; g.fmt = a->fmt; g.alpha = alpha;
  g.c = c; g.ldc = ldc; g.out_mode = out_dtype == FP4_OUT_F32 ? 1 : 0;
  g.c_amax = c_amax; g.status = status_ptr(ws);
  return gemm_launch(g, as_stream(stream));
}

fp4_status fp4_gemm(const fp4_qtensor* a, const fp4_qtensor* b, float alpha, void* c, int64_t ldc,
                    int32_t out_dtype, float* c_amax, void* ws, size_t ws_bytes, void* stream) {
  return gemm_impl(a, b, alpha, c, ldc, out_dtype, c_amax, ws, ws_bytes, stream, false);
}


static fp4_status gemm_quant_impl(const fp4_qtensor* a, const fp4_qtensor* b, float alpha,
                                  const float* out_amax_in, int32_t round, uint64_t sr_seed,
                                  uint32_t sr_stream, fp4_qtensor* out, void* c_bf16, int64_t ldc,
                                  float* c_amax, void* ws, size_t ws_bytes, void* stream) {
  if (a == nullptr || b == nullptr || out == nullptr || out_amax_in == nullptr) return FP4_ERR_NULL;
  if (a->codes == nullptr || b->codes == nullptr || a->scales_mma == nullptr ||
      b->scales_mma == nullptr || a->s_dec == nullptr || b->s_dec == nullptr)
    return FP4_ERR_NULL;
  if (out->codes == nullptr || out->scales_mma == nullptr || out->s_dec == nullptr ||
      out->amax == nullptr)
    return FP4_ERR_NULL;
  if (a->fmt != b->fmt || (a->fmt != FP4_NVFP4 && a->fmt != FP4_MXFP4)) return FP4_ERR_FORMAT;
  if (out->fmt != FP4_NVFP4 || out->block != FP4_BLOCK_1D) return FP4_ERR_FORMAT;
  if (round != FP4_RTN && round != FP4_SR) return FP4_ERR_FORMAT;
  const int64_t M = a->rows, N = b->rows, K = a->cols;
  if (b->cols != K || out->rows != M || out->cols != N) return FP4_ERR_SHAPE;
  if (M <= 0 || N <= 0 || K <= 0 || M % 128 || N % 128 || K % 64) return FP4_ERR_SHAPE;
  if (M > (1ll << 30) || N > (1ll << 30) || K > (1ll << 30)) return FP4_ERR_SHAPE;
  if (!gemm_tiles_fit(M, N)) return FP4_ERR_SHAPE;
  if (!aligned16(a->codes) || !aligned16(b->codes) || !aligned16(a->scales_mma) ||
      !aligned16(b->scales_mma) || !aligned16(out->codes) ||
      (reinterpret_cast<uintptr_t>(out->scales_mma) & 3u) ||
      (reinterpret_cast<uintptr_t>(out->scales) & 3u))
    return FP4_ERR_ALIGN;
  if (c_bf16 != nullptr && (ldc < N || (ldc * 2) % 16 || !aligned16(c_bf16))) return FP4_ERR_ALIGN;
  if (ws == nullptr || ws_bytes < fp4_workspace_bytes(M, N, K)) return FP4_ERR_WORKSPACE;
  GemmArgs g{};
  g.a_codes = a->codes; g.a_sf = a->scales_mma; g.a_sdec = a->s_dec;
  g.b_codes = b->codes; g.b_sf = b->scales_mma; g.b_sdec = b->s_dec;
  g.M = M; g.N = N; g.K = K; g.fmt = a->fmt; g.alpha = alpha;
  g.c = c_bf16; g.ldc = c_bf16 ? ldc : N; g.out_mode = 2;
  g.q_codes = out->codes; g.q_scales = out->scales; g.q_scales_mma = out->scales_mma;
  g.q_amax_in = out_amax_in; g.q_amax_out = out->amax; g.q_s_dec = out->s_dec;
  g.q_sr = round == FP4_SR; g.q_seed = sr_seed; g.q_stream = sr_stream;
  g.c_amax = c_amax; g.status = status_ptr(ws);
  return gemm_launch(g, as_stream(stream));
}

fp4_status fp4_gemm_quant(const fp4_qtensor* a, const fp4_qtensor* b, float alpha,
                          const float* out_amax_in, fp4_qtensor* out, float* c_amax, void* ws,
                          size_t ws_bytes, void* stream) {
  return gemm_quant_impl(a, b, alpha, out_amax_in, FP4_RTN, 0, 0, out, nullptr, 0, c_amax, ws,
                         ws_bytes, stream);
}

fp4_status fp4_gemm_quant_ex(const fp4_qtensor* a, const fp4_qtensor* b, float alpha,
                             const float* out_amax_in, int32_t round, uint64_t sr_seed,
                             uint32_t sr_stream, fp4_qtensor* out, void* c_bf16, int64_t ldc,
                             float* c_amax, void* ws, size_t ws_bytes, void* stream) {
  return gemm_quant_impl(a, b, alpha, out_amax_in, round, sr_seed, sr_stream, out, c_bf16, ldc,
                         c_amax, ws, ws_bytes, stream);
}

void fqt_linear_cfg_default(fqt_linear_cfg* cfg, int32_t fmt) {
  if (!cfg) return;
  std::memset(cfg, 0, sizeof(*cfg));
  cfg->fmt = fmt;
  cfg->out_dtype = FP4_OUT_BF16;
  if (fmt == FP4_MXFP4) {
    cfg->w_block = FP4_BLOCK_1D;
    cfg->round_fwd = FP4_RTN; cfg->round_bwd = FP4_RTN; cfg->round_x_t = FP4_RTN;
    cfg->rht_mask = FQT_RHT_FPROP | FQT_RHT_DGRAD | FQT_RHT_WGRAD;
    cfg->rht_n = 32;
  } else {
    cfg->w_block = FP4_BLOCK_2D;
    cfg->round_fwd = FP4_RTN; cfg->round_bwd = FP4_SR; cfg->round_x_t = FP4_SR;
    cfg->rht_mask = 0;
    cfg->rht_n = 16;
  }
}

static fp4_status check_cfg(const fqt_linear_cfg* cfg) {
  if (cfg == nullptr) return FP4_ERR_NULL;
  if (cfg->fmt != FP4_NVFP4 && cfg->fmt != FP4_MXFP4) return FP4_ERR_FORMAT;
  if (cfg->round_bwd == FP4_QUEST || cfg->round_x_t == FP4_QUEST) return FP4_ERR_UNSUPPORTED;
  if (cfg->round_fwd == FP4_QUEST && cfg->fmt != FP4_MXFP4) return FP4_ERR_UNSUPPORTED;
  if (cfg->rht_mask & ~7) return FP4_ERR_FORMAT;
  if (cfg->rht_mask && cfg->rht_n != 16 && cfg->rht_n != 32) return FP4_ERR_FORMAT;
  if (cfg->w_block == FP4_BLOCK_2D) {
    if (cfg->fmt != FP4_NVFP4) return FP4_ERR_FORMAT;
    // 2-D weight tiles are shared by fprop and dgrad: no rotation there
    if (cfg->rht_mask & (FQT_RHT_FPROP | FQT_RHT_DGRAD)) return FP4_ERR_UNSUPPORTED;
    if (cfg->round_fwd != FP4_RTN) return FP4_ERR_UNSUPPORTED;
  }
  return FP4_OK;
}

// The layer's calls, run twice: first validating only (`dry`), so that an
// argument error of any of them returns before anything is enqueued, then
// for real.
fp4_status fqt_linear_fwd(const fqt_linear_cfg* cfg, int64_t M, int64_t N, int64_t K,
                          const void* x, const void* w, void* y, fqt_saved* sv, void* ws,
                          size_t ws_bytes, void* stream) {
  fp4_status st = check_cfg(cfg);
  if (st != FP4_OK) return st;
  if (x == nullptr || w == nullptr || y == nullptr || sv == nullptr) return FP4_ERR_NULL;
  const int rn = cfg->rht_n;
  // X: row-wise for fprop, transposed for wgrad
  fp4_qparams px;
  fp4_qparams_default(&px);
  px.fmt = cfg->fmt;
  px.round = cfg->round_fwd;
  px.round_t = cfg->round_x_t;
  px.rht_n = (cfg->rht_mask & FQT_RHT_FPROP) ? rn : 0;
  px.rht_n_t = (cfg->rht_mask & FQT_RHT_WGRAD) ? rn : 0;
  px.rht_seed = cfg->seed;
  px.sr_seed = cfg->seed;
  px.sr_stream = 0;
  px.sr_stream_t = 3;
  // W: fprop operand [N, K] and dgrad operand W^T [K, N]
  fp4_qparams pw;
  fp4_qparams_default(&pw);
  pw.fmt = cfg->fmt;
  pw.block = cfg->w_block;
  pw.round = cfg->round_fwd;
  pw.round_t = cfg->round_fwd == FP4_QUEST ? FP4_RTN : cfg->round_fwd;   // W^T feeds dgrad
  pw.rht_n = (cfg->rht_mask & FQT_RHT_FPROP) ? rn : 0;
  pw.rht_n_t = (cfg->rht_mask & FQT_RHT_DGRAD) ? rn : 0;
  pw.rht_seed = cfg->seed;
  for (const bool dry : {true, false}) {
    st = quantize_impl(x, M, K, K, &px, &sv->xq, &sv->xq_t, ws, ws_bytes, stream, dry);
    if (st != FP4_OK) return st;
    st = quantize_impl(w, N, K, K, &pw, &sv->wq, &sv->wq_t, ws, ws_bytes, stream, dry);
    if (st != FP4_OK) return st;
    st = gemm_impl(&sv->xq, &sv->wq, 1.0f, y, N, cfg->out_dtype, nullptr, ws, ws_bytes, stream,
                   dry);
    if (st != FP4_OK) return st;
  }
  return FP4_OK;
}

fp4_status fqt_linear_bwd(const fqt_linear_cfg* cfg, int64_t M, int64_t N, int64_t K,
                          const void* dy, fqt_saved* sv, void* dx, float* dw, void* ws,
                          size_t ws_bytes, void* stream) {
  fp4_status st = check_cfg(cfg);
  if (st != FP4_OK) return st;
  if (dy == nullptr || dx == nullptr || dw == nullptr || sv == nullptr) return FP4_ERR_NULL;
  const int rn = cfg->rht_n;
  fp4_qparams pd;
  fp4_qparams_default(&pd);
  pd.fmt = cfg->fmt;
  pd.round = cfg->round_bwd;
  pd.round_t = cfg->round_bwd;
  pd.rht_n = (cfg->rht_mask & FQT_RHT_DGRAD) ? rn : 0;
  pd.rht_n_t = (cfg->rht_mask & FQT_RHT_WGRAD) ? rn : 0;
  pd.rht_seed = cfg->seed;
  pd.sr_seed = cfg->seed;
  pd.sr_stream = 1;
  pd.sr_stream_t = 2;
  for (const bool dry : {true, false}) {
    st = quantize_impl(dy, M, N, N, &pd, &sv->dyq, &sv->dyq_t, ws, ws_bytes, stream, dry);
    if (st != FP4_OK) return st;
    st = gemm_impl(&sv->dyq, &sv->wq_t, 1.0f, dx, K, cfg->out_dtype, nullptr, ws, ws_bytes,
                   stream, dry);
    if (st != FP4_OK) return st;
    st = gemm_impl(&sv->dyq_t, &sv->xq_t, 1.0f, dw, K, FP4_OUT_F32, nullptr, ws, ws_bytes,
                   stream, dry);
    if (st != FP4_OK) return st;
  }
  return FP4_OK;
}

fp4_status fp4_read_device_status(const void* ws, void* stream) {
  if (ws == nullptr) return FP4_ERR_NULL;
  if (cudaStreamSynchronize(as_stream(stream)) != cudaSuccess) return FP4_ERR_CUDA;
  uint32_t code = 0;
  if (cudaMemcpy(&code, ws, sizeof(code), cudaMemcpyDeviceToHost) != cudaSuccess) return FP4_ERR_CUDA;
  return static_cast<fp4_status>(code);
}

fp4_status fp4_clear_device_status(void* ws, void* stream) {
  if (ws == nullptr) return FP4_ERR_NULL;
  return cuda_status(cudaMemsetAsync(ws, 0, sizeof(DeviceStatus), as_stream(stream)));
}

}  // extern "C"

namespace fp4impl {
fp4_status gemm_validate(const fp4_qtensor* a, const fp4_qtensor* b, const void* c, int64_t ldc,
                         int32_t out_dtype, const void* ws, size_t ws_bytes) {
  return gemm_impl(a, b, 1.0f, const_cast<void*>(c), ldc, out_dtype, nullptr,
                   const_cast<void*>(ws), ws_bytes, nullptr, true);
}
}  // namespace fp4impl
