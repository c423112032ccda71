/*
 * fp4.h -- C ABI of libfp4fqt.so, a B200 (sm_100a) library for the
 * fully-quantized FP4 linear layer: block quantization of BF16 tensors to
 * NVFP4 / MXFP4 and the three block-scaled FP4 GEMMs of a linear layer
 * (fprop, dgrad, wgrad), accumulated in FP32 on the tensor cores.
 *
 * What is computed (page title, section):
 *   - "FP4" (Robots Atlas), How it works: values are cast to 4-bit E2M1;
 *     runs of 16 (NVFP4) or 32 (MXFP4) consecutive values share one scale
 *     each (E4M3 for NVFP4, E8M0 for MXFP4);
 *     NVFP4 adds one FP32 scale for the whole tensor; matrix products run
 *     on the tensor cores in FP4 and accumulate in higher precision; random
 *     Hadamard transforms, two-dimensional quantization and stochastic
 *     rounding of gradients stabilise training.
 *   - "FP4" (Robots Atlas), Components: the eight E2M1 magnitudes 0, 0.5,
 *     1, 1.5, 2, 3, 4, 6, each with either sign; NVFP4 and MXFP4 block
 *     formats.
 *   - "FP4 All the Way: Fully Quantized Training of LLMs", Key points:
 *     NVFP4, round-to-nearest in the forward pass, stochastic rounding in
 *     the backward and update passes.
 *   - "Quartet: Native FP4 Training Can Be Optimal for Large Language
 *     Models", Approach: fprop, dgrad and wgrad each computed from FP4
 *     operands, round-to-nearest backward with block-wise Hadamard
 *     rotations (the MXFP4 mode).
 *
 * Conventions shared by every entry point:
 *   - Every tensor pointer is DEVICE memory owned by the caller.  The
 *     library allocates no device memory and keeps no global mutable state;
 *     calls on different streams do not interfere unless they share
 *     buffers.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  All work is enqueued asynchronously on it; no entry point
 *     synchronises except fp4_read_device_status.
 *   - Argument errors are returned synchronously, before anything is
 *     enqueued.  A failed launch returns FP4_ERR_CUDA.  Conditions found on
 *     the device (non-finite amax, expired bounded wait) are OR-ed into the
 *     status word at the start of the workspace `ws`, read with
 *     fp4_read_device_status; they are sticky until fp4_clear_device_status.
 *   - Matrices are row-major.  Packed FP4 codes: two per byte, element 2j in
 *     the low nibble of byte j.  A code is sign (bit 3), exponent (bits 2-1),
 *     mantissa (bit 0).  Pointers must be 16-byte aligned.
 *   - Stochastic rounding is counter-based, 16 random bits per element:
 *     element i (row-major index in the quantized operand's own logical
 *     layout) takes the low (i even) or high (i odd) half of 32-bit draw
 *     j = i/2, draw j being word j mod 4 of Philox4x32-10 with key
 *     (seed lo, seed hi) and counter (j/4 lo, j/4 hi, stream, 0); with p the
 *     value's fraction of the gap between its two neighbouring E2M1 levels,
 *     it rounds up iff floor(p * 2^16) + u >= 2^16.  Results do not depend on
 *     the launch configuration.  The Hadamard sign vector d (d_j = -1 iff
 *     bit 31 of 32-bit draw j of stream 0x48414441 under the RHT seed) is
 *     shared by every block of both operands of a GEMM.
 */
#ifndef FP4FQT_FP4_H
#define FP4FQT_FP4_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define FP4_ABI_VERSION 1

/* ---------------------------------------------------------------------- */
/* Status codes                                                            */
/* ---------------------------------------------------------------------- */
typedef enum fp4_status {
  FP4_OK = 0,
  FP4_ERR_NULL = 1,        /* a required pointer is NULL                        */
  FP4_ERR_SHAPE = 2,       /* sizes violate the divisibility rules              */
  FP4_ERR_ALIGN = 3,       /* a pointer or leading dimension is not aligned     */
  FP4_ERR_FORMAT = 4,      /* inconsistent format / block / rounding request    */
  FP4_ERR_WORKSPACE = 5,   /* workspace missing or smaller than required        */
  FP4_ERR_CUDA = 6,        /* a CUDA call or kernel launch failed               */
  FP4_ERR_NONFINITE = 7,   /* device: a tensor amax was Inf or NaN              */
  FP4_ERR_TIMEOUT = 8,     /* device: a bounded wait inside a GEMM expired      */
  FP4_ERR_UNSUPPORTED = 9  /* a valid request this build does not implement     */
} fp4_status;

/* Values of the int32_t selector fields below. */
enum { FP4_NVFP4 = 0, FP4_MXFP4 = 1 };            /* format                  */
enum { FP4_RTN = 0, FP4_SR = 1, FP4_QUEST = 2 };  /* rounding (see below)    */
enum { FP4_BLOCK_1D = 0, FP4_BLOCK_2D = 1 };      /* 1x16 / 1x32, or 16x16    */
enum { FP4_OUT_BF16 = 0, FP4_OUT_F32 = 1 };       /* GEMM output type         */
enum { FQT_RHT_FPROP = 1, FQT_RHT_DGRAD = 2, FQT_RHT_WGRAD = 4 };

/* ---------------------------------------------------------------------- */
/* A quantized operand (all buffers caller-allocated device memory).       */
/*                                                                         */
/* codes      [rows, cols/2] bytes (may be NULL for an empty operand).     */
/* scales     logical block scales, may be NULL:                           */
/*              NVFP4 1-D: [rows, cols/16] E4M3; NVFP4 2-D: [rows/16,      */
/*              cols/16] E4M3 (one per 16x16 tile); MXFP4: [rows, cols/32]  */
/*              E8M0.                                                       */
/* scales_mma the same scales in the tensor-core layout, may be NULL;      */
/*              required by fp4_gemm.  One byte per (row, block of 16 or 32 */
/*              columns), 2-D tile scales replicated to each of the tile's  */
/*              16 rows, arranged in 512-byte atoms of 128 rows x 4 blocks: */
/*              byte offset of (r, s) with S = cols/blocksize blocks a row: */
/*                ((r/128) * (S/4) + s/4) * 512                             */
/*                  + (r%32)*16 + ((r%128)/32)*4 + s%4.                     */
/*              Needs rows % 128 == 0 and S % 4 == 0; size rows*S bytes.    */
/* amax       [1] float: tensor amax (of the rotated values when a Hadamard */
/*              transform is applied); written by fp4_quantize.  NVFP4 only */
/*              (may be NULL for MXFP4).                                    */
/* s_dec      [1] float: per-tensor decode scale.  NVFP4: amax/2688 (1 when */
/*              amax = 0); MXFP4: 1.  Written by fp4_quantize.              */
/* ---------------------------------------------------------------------- */
typedef struct fp4_qtensor {
  uint8_t* codes;
  uint8_t* scales;
  uint8_t* scales_mma;
  float* amax;
  float* s_dec;
  int64_t rows;
  int64_t cols;
  int32_t fmt;      /* FP4_NVFP4 / FP4_MXFP4 */
  int32_t block;    /* FP4_BLOCK_1D / FP4_BLOCK_2D */
} fp4_qtensor;

/* Byte sizes of the buffers of a quantized operand of logical shape
 * [rows, cols]; any output pointer may be NULL. */
void fp4_qtensor_sizes(int64_t rows, int64_t cols, int32_t fmt, int32_t block,
                       size_t* codes_bytes, size_t* scales_bytes, size_t* scales_mma_bytes);

/* ---------------------------------------------------------------------- */
/* Quantization request.                                                   */
/* The row-wise output quantizes x along its columns (blocks run along a   */
/* row); the transposed output quantizes x^T, i.e. blocks run down x's      */
/* columns, and is stored as a [cols, rows] operand.                        */
/* ---------------------------------------------------------------------- */
typedef struct fp4_qparams {
  int32_t fmt;            /* FP4_NVFP4 or FP4_MXFP4                                  */
  int32_t block;          /* FP4_BLOCK_1D, or FP4_BLOCK_2D (NVFP4 weights, RTN only) */
  int32_t round;          /* rounding of the row-wise output: FP4_RTN, FP4_SR, or    */
                          /* FP4_QUEST (MXFP4 only): the QuEST-style forward scale   */
                          /* of "Quartet" (Approach): each 32-block's scale from     */
                          /* T = RN(2.9224751 * RMS) by the power-of-two rule         */
                          /* floor(log2 T) - 2 in place of the block max (values      */
                          /* beyond the top level clip), then round to nearest; the  */
                          /* mean square is summed in binary32 as ((y0^2 + y1^2) +   */
                          /* (y2^2 + y3^2)) + ((y4^2 + y5^2) + (y6^2 + y7^2)) per    */
                          /* group of 8, then (g0 + g1) + (g2 + g3)                  */
  int32_t round_t;        /* rounding of the transposed output                       */
  int32_t rht_n;          /* 0, 16 or 32: Hadamard block of the row-wise output      */
  int32_t rht_n_t;        /* 0, 16 or 32: Hadamard block of the transposed output    */
  uint64_t rht_seed;      /* seed of the Hadamard sign vector                        */
  uint64_t sr_seed;       /* seed of the stochastic-rounding draws                   */
  uint32_t sr_stream;     /* Philox stream of the row-wise output                    */
  uint32_t sr_stream_t;   /* Philox stream of the transposed output                  */
  const float* amax_in;   /* optional device float: use this amax for the row-wise  */
                          /* output instead of computing it (single-pass encode)     */
  const float* amax_in_t; /* same for the transposed output                          */
} fp4_qparams;

/* Defaults: NVFP4 1-D, RTN, no Hadamard, seed 0, streams 0. */
void fp4_qparams_default(fp4_qparams* p);

/* Workspace bytes needed by fp4_gemm for an M x N x K product (also enough
 * for every other entry point).  At least 256: the status block. */
size_t fp4_workspace_bytes(int64_t M, int64_t N, int64_t K);

/* Quantize x (BF16, [rows, cols] with leading dimension ld >= cols, in
 * elements, ld % 8 == 0; NULL allowed when rows or cols is 0, which only
 * writes amax = 0 and s_dec = 1) into `out` (row-wise, may be NULL) and/or `out_t`
 * (transposed, may be NULL).  Shape rules: NVFP4 1-D needs cols % 16 == 0
 * for `out` and rows % 16 == 0 for `out_t`; MXFP4 the same with 32; NVFP4
 * 2-D needs rows % 16 == 0 and cols % 16 == 0 and produces W (`out`) and
 * W^T (`out_t`) from one tile scale per 16x16 tile (identical codes,
 * transposed).  A Hadamard block must divide the blocked dimension.  The
 * qtensors' rows/cols/fmt/block must describe the requested outputs.
 * `ws` may be NULL (device conditions are then not recorded).
 * Two passes over x (amax, then encode) unless the amax is supplied. */
fp4_status fp4_quantize(const void* x_bf16, int64_t rows, int64_t cols, int64_t ld,
                        const fp4_qparams* params, fp4_qtensor* out, fp4_qtensor* out_t,
                        void* ws, size_t ws_bytes, void* stream);

/* Block-scaled FP4 GEMM, both operands K-major ("NT"):
 *   C[m, n] = alpha * s_dec(a) * s_dec(b) * sum_k a_hat[m, k] * b_hat[n, k]
 * with a_hat = e2m1(code) * block scale, M = a->rows, N = b->rows,
 * K = a->cols = b->cols, accumulated in FP32 on the tensor cores.
 * Requires a->fmt == b->fmt, both scales_mma set, M % 128 == 0,
 * N % 128 == 0, K % 64 == 0, K > 0.  C is [M, ldc] of `out_dtype` with
 * ldc >= N and ldc * element size a multiple of 16 bytes.
 * c_amax (nullable device float) receives max |C| over the output.
 * ws must hold fp4_workspace_bytes(M, N, K) bytes. */
fp4_status fp4_gemm(const fp4_qtensor* a, const fp4_qtensor* b, float alpha, void* c,
                    int64_t ldc, int32_t out_dtype, float* c_amax, void* ws,
                    size_t ws_bytes, void* stream);

/* The same GEMM with the result quantized in the epilogue instead of
 * written as BF16/FP32: each FP32 value C[m, n] (as fp4_gemm computes it)
 * is encoded to NVFP4 1x16 with round-to-nearest, exactly as fp4_quantize
 * encodes a row-wise output with a supplied tensor amax, into `out`
 * (rows M, cols N, FP4_NVFP4, FP4_BLOCK_1D; codes and scales_mma required,
 * logical scales optional; out->amax receives *out_amax_in and out->s_dec the
 * matching decode scale).  The tensor amax must be supplied (device float:
 * for example the previous step's c_amax of this output, "delayed
 * scaling"); c_amax (nullable) receives this call's max |C| for the next
 * one.  The output is never stored in BF16: it replaces a BF16 write and the
 * quantizer's two reads of it ("FP4 All the Way" / "Quartet" pages: quantize
 * operands in fused kernels).  Shape and alignment rules as fp4_gemm, plus
 * out->codes 16-byte and the scale pointers 4-byte aligned. */
fp4_status fp4_gemm_quant(const fp4_qtensor* a, const fp4_qtensor* b, float alpha,
                          const float* out_amax_in, fp4_qtensor* out, float* c_amax, void* ws,
                          size_t ws_bytes, void* stream);

/* fp4_gemm_quant with a choice of rounding and an optional BF16 copy:
 *   - round FP4_RTN or FP4_SR.  Stochastic rounding uses the library's
 *     16-bit draws of (sr_seed, sr_stream) with element index m * N + n of
 *     the [M, N] output, exactly as fp4_quantize rounds a row-wise output
 *     ("FP4 All the Way", Key points: stochastic rounding for gradients);
 *   - c_bf16 (nullable): the same FP32 results also stored as BF16,
 *     [M, ldc] with ldc >= N and ldc * 2 a multiple of 16 bytes, for a
 *     consumer that still needs them -- the transposed quantization of a
 *     gradient (blocks down the columns), which one thread per output row
 *     cannot form in the epilogue.
 * Everything else as fp4_gemm_quant (which is this call with FP4_RTN and no
 * BF16 copy). */
fp4_status fp4_gemm_quant_ex(const fp4_qtensor* a, const fp4_qtensor* b, float alpha,
                             const float* out_amax_in, int32_t round, uint64_t sr_seed,
                             uint32_t sr_stream, fp4_qtensor* out, void* c_bf16, int64_t ldc,
                             float* c_amax, void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------- */
/* Linear layer  Y = X W^T  with X [M, K], W [N, K], dY [M, N]:            */
/*   fprop  Y  = X . W^T      (contract K)                                 */
/*   dgrad  dX = dY . W       (contract N; uses W^T stored [K, N])          */
/*   wgrad  dW = dY^T . X     (contract M; uses dY^T [N, M] and X^T [K, M]) */
/* ---------------------------------------------------------------------- */
typedef struct fqt_linear_cfg {
  int32_t fmt;        /* FP4_NVFP4 or FP4_MXFP4                                   */
  int32_t w_block;    /* NVFP4: FP4_BLOCK_2D (16x16 weight tiles) or FP4_BLOCK_1D  */
  int32_t round_fwd;  /* rounding of X and W for fprop (FP4_QUEST: MXFP4 only;    */
                      /* W^T for dgrad then rounds to nearest)                    */
  int32_t round_bwd;  /* rounding of dY (dgrad and wgrad operands)                */
  int32_t round_x_t;  /* rounding of X^T, the wgrad ("update pass") operand       */
  int32_t rht_mask;   /* FQT_RHT_* bits: GEMMs whose operands are rotated first    */
  int32_t rht_n;      /* Hadamard block: 16 (NVFP4 default) or 32 (MXFP4 default)  */
  int32_t out_dtype;  /* FP4_OUT_BF16 / FP4_OUT_F32 for Y and dX (dW is FP32)      */
  uint64_t seed;      /* stochastic-rounding and Hadamard seed                    */
} fqt_linear_cfg;

/* Defaults. NVFP4: 2-D weights, RTN forward, SR for dY and X^T, no Hadamard.
 * MXFP4: 1-D weights, RTN everywhere, 32-point Hadamard on all three GEMMs.
 * Philox streams used by the layer: dY row-wise 1, dY^T 2, X^T 3. */
void fqt_linear_cfg_default(fqt_linear_cfg* cfg, int32_t fmt);

/* Quantized operands of one layer (caller-allocated, shapes as listed). */
typedef struct fqt_saved {
  fp4_qtensor xq;     /* X   [M, K]  fprop A   */
  fp4_qtensor xq_t;   /* X^T [K, M]  wgrad B   */
  fp4_qtensor wq;     /* W   [N, K]  fprop B   */
  fp4_qtensor wq_t;   /* W^T [K, N]  dgrad B   */
  fp4_qtensor dyq;    /* dY  [M, N]  dgrad A   */
  fp4_qtensor dyq_t;  /* dY^T [N, M] wgrad A   */
} fqt_saved;

/* Forward: quantize X (row-wise and transposed) and W (both orientations),
 * then Y = fprop.  x, w BF16; y of cfg->out_dtype, [M, N] dense.  The
 * shape, alignment and workspace rules are those of the fp4_quantize and
 * fp4_gemm calls it makes (M, N multiples of 128, K of 128 for the backward's
 * outputs); all of them are checked before the first is enqueued, so an
 * argument error leaves the stream untouched. */
fp4_status fqt_linear_fwd(const fqt_linear_cfg* cfg, int64_t M, int64_t N, int64_t K,
                          const void* x, const void* w, void* y, fqt_saved* saved,
                          void* ws, size_t ws_bytes, void* stream);

/* Backward: quantize dY (row-wise and transposed), then dX = dgrad
 * ([M, K], cfg->out_dtype) and dW = wgrad ([N, K], FP32), from the operands
 * fqt_linear_fwd left in `saved`.  Argument errors as for the forward. */
fp4_status fqt_linear_bwd(const fqt_linear_cfg* cfg, int64_t M, int64_t N, int64_t K,
                          const void* dy, fqt_saved* saved, void* dx, float* dw,
                          void* ws, size_t ws_bytes, void* stream);

/* fp4_gemm for callers that cannot allocate device memory (no counterpart
 * in the paper; an addition of this library).
 *
 * fp4_gemm needs a caller-allocated workspace, which the GEMM uses as scratch
 * for its device status block.  Callers that cannot call cudaMalloc -- code
 * running while a framework's pool or arena owns all device memory, plugins
 * in host processes that forbid device allocation, paths that must not risk
 * the synchronisation cudaMalloc can cause -- use this entry point instead.
 * Its scratch is a static device array inside the library of
 * FP4_NOALLOC_SCRATCH_BYTES bytes per device, held by every GPU that loads
 * the library until the process exits.  Same arguments and results as
 * fp4_gemm, without `ws`; inputs and outputs are still caller-provided.
 *   - Problems whose workspace need (fp4_workspace_bytes(M, N, K)) exceeds
 *     FP4_NOALLOC_SCRATCH_BYTES are rejected with FP4_ERR_WORKSPACE.
 *   - Allocates nothing: no cudaMalloc, cudaFree or allocating library call.
 *   - The first call on a device looks up the array's device address (with
 *     that device current) and keeps it for the rest of the process; make
 *     that first call before any stream capture.  A lookup that fails returns
 *     FP4_ERR_CUDA, keeps nothing, and is tried again by the next call.
 *   - Every call shares the one array: each call clears its status block on
 *     `stream` first, and calls that overlap on the GPU (other streams, other
 *     threads) race on it.  Device conditions of a call are not reported
 *     through this entry point; callers that need them use fp4_gemm. */
#define FP4_NOALLOC_SCRATCH_BYTES 4096
fp4_status fp4_gemm_noalloc(const fp4_qtensor* a, const fp4_qtensor* b, float alpha, void* c,
                            int64_t ldc, int32_t out_dtype, float* c_amax, void* stream);

/* Data-parallel weight-gradient sum: buf[0 .. count) (FP32, device memory)
 * is replaced by its sum over the ranks of `nccl_comm` (an ncclComm_t the
 * caller created, passed as void*), enqueued with NCCL on `stream` after the
 * work already queued there (typically the layer's wgrad).  The one exchange
 * of data-parallel training of the layer: every rank quantizes its own token
 * shard and computes its own dW ("FP4 All the Way", Summary: the 7B model
 * trained on 256 accelerators).  Every rank must make the same calls in the
 * same order.  The library does not link NCCL: the process's NCCL is found
 * by its soname (libnccl.so.2) on first use; FP4_ERR_UNSUPPORTED when there
 * is none, FP4_ERR_CUDA when NCCL reports an error.  count == 0 does
 * nothing. */
fp4_status fp4_allreduce_sum_f32(void* nccl_comm, float* buf, int64_t count, void* stream);

/* Gradient-norm vs quantization-noise diagnostic ("FP4 All the Way" page,
 * Summary: quantized training stops being effective below a threshold set
 * by the relation between the gradient norm and the quantization noise; the
 * page gives no formula, so this reports the two quantities themselves).
 * With x the BF16 tensor [rows, cols] (leading dimension ld, ld % 8 == 0)
 * and q its row-wise quantization (q->rows == rows, q->cols == cols, 1-D or
 * 2-D NVFP4 or MXFP4, scales_mma or scales set):
 *   sums[0] = sum x^2,  sums[1] = sum (deq(q) - x)^2,
 *   deq(q) = e2m1(code) * block scale * s_dec(q)   (exact in double),
 * accumulated in double.  `sums` is caller-owned device memory, two doubles,
 * overwritten (zeroed first on `stream`).  The order of the additions is not
 * fixed, so results agree with an exact sum to about 1e-12 relative.
 * ||x|| / ||deq(q) - x|| = sqrt(sums[0] / sums[1]) is the signal-to-noise
 * ratio of the quantized tensor. */
fp4_status fp4_quant_noise(const void* x_bf16, int64_t rows, int64_t cols, int64_t ld,
                           const fp4_qtensor* q, double* sums, void* ws, size_t ws_bytes,
                           void* stream);

/* Synchronise `stream`, then return the device status word of `ws`
 * (FP4_OK when no device condition was recorded). */
fp4_status fp4_read_device_status(const void* ws, void* stream);

/* Enqueue a reset of the device status word of `ws`. */
fp4_status fp4_clear_device_status(void* ws, void* stream);

const char* fp4_status_str(int32_t status);
int32_t fp4_abi_version(void);

/* Tensor-core rate microbenchmark (synchronises `stream`): one persistent CTA
 * (variants 0, 1, 4, 6) or CTA pair (2, 3, 5, 7) per SM issues `iters` x 4
 * back-to-back block-scaled NVFP4 MMAs (128x256x64, or 256x256x64 for a
 * pair) on operands resident in shared memory; variants 1 and 3 add, from the
 * MMA thread, the three scale-factor copies into tensor memory that one MMA
 * of a GEMM K step needs; variants 4 and 5 issue the same copies from a
 * second warp concurrently with the MMAs; variants 6 and 7 issue a K step's
 * twelve copies together before its four MMAs, into rotating slots.  Any other
 * variant, or iters <= 0, returns FP4_ERR_SHAPE.  Writes the
 * achieved TFLOP/s: what the tensor pipe sustains with and without the
 * scale-factor traffic, the context for the GEMM's rate ("FP4" page,
 * Hardware: FP4 on fifth-generation Tensor Cores). */
fp4_status fp4_mma_rate(int32_t variant, int32_t iters, float* tflops_out, void* ws,
                        size_t ws_bytes, void* stream);

/* Number of CUDA kernels this library has enqueued in the calling process
 * since it was loaded (all devices, all streams).  Host-side counter, no
 * synchronisation; used to attribute work in a timed region. */
uint64_t fp4_kernel_launches(void);

#ifdef __cplusplus
}
#endif

#endif /* FP4FQT_FP4_H */
