// gemm_sm100.cu -- block-scaled FP4 GEMM on the 5th-generation tensor cores.
//
// C[m, n] = alpha * s_dec(A) * s_dec(B) * sum_k A[m, k] B[n, k], both operands
// K-major packed E2M1 with per-block scales (E4M3 per 16 for NVFP4, E8M0 per
// 32 for MXFP4), accumulated in FP32 in tensor memory.  "FP4" (Robots Atlas),
// How it works: matrix multiplications run on Tensor Cores in FP4 while
// accumulation happens in higher precision; "Quartet", abstract line: all
// three linear-layer GEMMs in FP4.
//
// Structure (one persistent CTA per SM, 320 threads):
//   warp 8      TMA producer: A/B tiles (128B-swizzled) and the scale-factor
//               atoms (bulk copies) into a 4-stage shared-memory ring;
//   warp 9      TMEM allocator and MMA issuer: tcgen05.cp moves the scale
//               atoms into tensor memory, tcgen05.mma (kind::mxf4nvf4 /
//               kind::mxf4, block_scale) accumulates a 128 x 256 tile into
//               TMEM, tcgen05.commit releases ring slots and the accumulator;
//   warps 0..7  epilogue: warp w drains TMEM lanes 32 (w % 4) .. + 31, columns
//               128 (w / 4) .. + 127 into registers, releases the accumulator
//               (the next tile's MMAs start), then scales, converts, stores
//               and tracks |C| max.
// Every mbarrier wait is bounded (2 s of %globaltimer); on expiry the kernel
// records FP4_ERR_TIMEOUT, drains its own copies and MMAs, frees TMEM and
// returns.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>
#include <mutex>

#include "internal.h"
#include "sm100_ptx.cuh"

namespace fp4impl {
namespace {

constexpr int BM = 128;              // tile rows (M) per CTA
constexpr int BN = 256;              // tile cols (N) per CTA = UMMA N
constexpr int BK = 256;              // K elements per stage (128 bytes of FP4 per row)
constexpr int MMA_K = 64;            // K elements per tcgen05.mma
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * BK / 2;          // 16 KB
constexpr int B_BYTES = BN * BK / 2;          // 32 KB
constexpr int SFA_BYTES = 4 * 512;            // up to 4 atoms of 128 rows x 4 scales
constexpr int SFB_BYTES = 2 * 4 * 512;        // two 128-row blocks
constexpr int STAGE_BYTES = A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES;
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 /*align*/ + 256 /*barriers*/;
constexpr int NUM_THREADS = 320;
constexpr int EPI_WARPS = 8;
constexpr int PRODUCER_WARP = 8;
constexpr int MMA_WARP = 9;
constexpr int TMEM_COLS = 512;
constexpr int TMEM_SF_BASE = 256;             // accumulator uses columns [0, 256)
constexpr int TMEM_SF_STAGE = 48;             // 16 (A) + 32 (B) columns per stage

using namespace ptx;

struct Smem {
  uint8_t* base;   // 1024-aligned
  __device__ uint8_t* a(int s) const { return base + s * A_BYTES; }
  __device__ uint8_t* b(int s) const { return base + STAGES * A_BYTES + s * B_BYTES; }
  __device__ uint8_t* sfa(int s) const { return base + STAGES * (A_BYTES + B_BYTES) + s * SFA_BYTES; }
  __device__ uint8_t* sfb(int s) const {
    return base + STAGES * (A_BYTES + B_BYTES + SFA_BYTES) + s * SFB_BYTES;
  }
  __device__ uint64_t* bars() const {
    return reinterpret_cast<uint64_t*>(base + STAGES * STAGE_BYTES);
  }
};

struct KParams {
  const uint8_t* a_sf; const uint8_t* b_sf;
  const float* a_sdec; const float* b_sdec;
  int M, N, K;
  float alpha;
  void* c; int64_t ldc; int out_f32;
  float* c_amax;
  uint32_t* status;
};

template <bool NV>
__global__ void __launch_bounds__(NUM_THREADS, 1)
fp4_gemm_kernel(const __grid_constant__ CUtensorMap tmap_a,
                const __grid_constant__ CUtensorMap tmap_b, const KParams p) {
  extern __shared__ uint8_t smem_raw[];
  Smem sm{reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                     ~static_cast<uintptr_t>(1023))};
  uint64_t* bars = sm.bars();
  // barrier slots: full[0..S), empty[S..2S), acc_full, acc_empty, drain
  const uint32_t bar0 = smem_u32(bars);
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (STAGES + s); };
  const uint32_t acc_full = bar0 + 8u * (2 * STAGES);
  const uint32_t acc_empty = bar0 + 8u * (2 * STAGES + 1);
  const uint32_t drain_bar = bar0 + 8u * (2 * STAGES + 2);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + 2 * STAGES + 3);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tiles_m = p.M / BM, tiles_n = (p.N + BN - 1) / BN;
  const int num_tiles = tiles_m * tiles_n;
  const int k_blocks = (p.K + BK - 1) / BK;
  const int atoms_per_rowblk_nv = p.K / 64;          // NVFP4: 4 scales per atom = 64 K
  const int S_mx = ((p.K / 32) + 3) & ~3;             // MXFP4 scales per row, padded
  const int atoms_per_rowblk = NV ? atoms_per_rowblk_nv : S_mx / 4;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, EPI_WARPS);
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == MMA_WARP) tmem_alloc(smem_u32(tmem_holder), TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;

  if (warp == PRODUCER_WARP) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_a)) : "memory");
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_b)) : "memory");
      uint32_t it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        const int mb = tile / tiles_n, nb = tile % tiles_n;
        const bool b_hi = (nb * 2 + 1) * 128 < p.N;   // second 128-row block of B exists
        for (int kb = 0; kb < k_blocks; ++kb, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1u;
          if (!mbar_wait(empty_bar(s), ph ^ 1u, abort_flag, p.status, 0x100 + s)) { ok = false; break; }
          // scale atoms covered by this K block
          int n_atoms;
          if (NV) n_atoms = min(4, atoms_per_rowblk - kb * 4);
          else n_atoms = min(2, atoms_per_rowblk - kb * 2);
          const uint32_t atom_bytes = (uint32_t)n_atoms * 512u;
          const uint32_t tx = A_BYTES + B_BYTES + atom_bytes * (b_hi ? 3u : 2u);
          mbar_arrive_expect_tx(full_bar(s), tx);
          tma_load_2d(smem_u32(sm.a(s)), &tmap_a, full_bar(s), kb * (BK / 2), mb * BM);
          tma_load_2d(smem_u32(sm.b(s)), &tmap_b, full_bar(s), kb * (BK / 2), nb * BN);
          const int atom0 = kb * (NV ? 4 : 2);
          bulk_load(smem_u32(sm.sfa(s)),
                    p.a_sf + ((size_t)mb * atoms_per_rowblk + atom0) * 512, atom_bytes, full_bar(s));
          bulk_load(smem_u32(sm.sfb(s)),
                    p.b_sf + ((size_t)(2 * nb) * atoms_per_rowblk + atom0) * 512, atom_bytes,
                    full_bar(s));
          if (b_hi)
            bulk_load(smem_u32(sm.sfb(s) + 4 * 512),
                      p.b_sf + ((size_t)(2 * nb + 1) * atoms_per_rowblk + atom0) * 512, atom_bytes,
                      full_bar(s));
        }
      }
      // Drain: every armed stage's copies must land before the CTA exits.
      if (it > 0) {
        const uint32_t first = it > (uint32_t)STAGES ? it - STAGES : 0;
        for (uint32_t j = first; j < it; ++j) {
          const int s = j % STAGES;
          const uint32_t ph = (j / STAGES) & 1u;
          volatile int no_abort = 0;
          mbar_wait(full_bar(s), ph, &no_abort, p.status, 0x200 + s);
        }
      }
    }
  } else if (warp == MMA_WARP) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      uint32_t it = 0, tile_iter = 0;
      bool ok = true;
      bool issued = false;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x, ++tile_iter) {
        if (!mbar_wait(acc_empty, (tile_iter & 1u) ^ 1u, abort_flag, p.status, 0x300)) { ok = false; break; }
        tc_fence_after();
        for (int kb = 0; kb < k_blocks; ++kb, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1u;
          if (!mbar_wait(full_bar(s), ph, abort_flag, p.status, 0x400 + s)) { ok = false; break; }
          const int n_mma = min(BK / MMA_K, (p.K - kb * BK) / MMA_K);
          const uint32_t t_sfa = tmem_base + TMEM_SF_BASE + s * TMEM_SF_STAGE;
          const uint32_t t_sfb = t_sfa + 16;
          const uint32_t a_base = smem_u32(sm.a(s)), b_base = smem_u32(sm.b(s));
          const uint32_t sfa_s = smem_u32(sm.sfa(s)), sfb_s = smem_u32(sm.sfb(s));
          // Each MMA's scale atoms are copied into TMEM right before it (the
          // copies and MMAs of one thread execute in issue order).
          auto step = [&](int kk) {
            uint32_t sfa_addr, sfb_addr, idesc;
            const int atom = NV ? kk : (kk >> 1);
            if (NV || (kk & 1) == 0) {
              tc_cp_32x128b(t_sfa + 4 * atom, smem_desc(sfa_s + atom * 512, 0, 128, 0));
              tc_cp_32x128b(t_sfb + 8 * atom, smem_desc(sfb_s + atom * 512, 0, 128, 0));
              tc_cp_32x128b(t_sfb + 8 * atom + 4, smem_desc(sfb_s + 2048 + atom * 512, 0, 128, 0));
            }
            if (NV) {
              sfa_addr = t_sfa + 4 * kk;
              sfb_addr = t_sfb + 8 * kk;
              idesc = make_idesc(BN, BM, 0u, 0u, 0u);
            } else {
              const uint32_t byte = (uint32_t)(kk & 1) * 2u;
              sfa_addr = (t_sfa + 4 * atom) | (byte << 30);
              sfb_addr = (t_sfb + 8 * atom) | (byte << 30);
              idesc = make_idesc(BN, BM, 1u, byte, byte);
            }
            tc_mma<NV>(tmem_base, smem_desc(a_base + kk * (MMA_K / 2), 16, 1024, 2),
                       smem_desc(b_base + kk * (MMA_K / 2), 16, 1024, 2), idesc, sfa_addr,
                       sfb_addr, (kb > 0 || kk > 0) ? 1u : 0u);
          };
          if (n_mma == BK / MMA_K) {
#pragma unroll
            for (int kk = 0; kk < BK / MMA_K; ++kk) step(kk);
          } else {
            for (int kk = 0; kk < n_mma; ++kk) step(kk);
          }
          issued = true;
          tc_commit(empty_bar(s));     // ring slot free once these MMAs finish
        }
        if (!ok) break;
        tc_commit(acc_full);           // accumulator ready for the epilogue
      }
      if (issued) {
        // Wait for every MMA this thread issued before TMEM is released.
        tc_commit(drain_bar);
        volatile int no_abort = 0;
        mbar_wait(drain_bar, 0, &no_abort, p.status, 0x500);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const float scale = p.alpha * (*p.a_sdec) * (*p.b_sdec);
    float amax = 0.0f;
    uint32_t tile_iter = 0;
    const int quad = warp & 3, half = warp >> 2;
    const int row_in_tile = quad * 32 + lane;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++tile_iter) {
      // one lane per warp polls the barrier; the warp then proceeds together
      int ok = 1;
      if (lane == 0) ok = mbar_wait(acc_full, tile_iter & 1u, abort_flag, p.status, 0x600 + warp);
      ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
      if (!ok) break;
      tc_fence_after();
      const int mb = tile / tiles_n, nb = tile % tiles_n;
      const int64_t row = (int64_t)mb * BM + row_in_tile;
      const int c_begin = half * (BN / 2);
      const int ncols = min(BN / 2, p.N - nb * BN - c_begin);   // 128, 0 (ragged N)
      uint32_t r[BN / 2];
      const uint32_t taddr = tmem_base + ((uint32_t)(quad * 32) << 16) + (uint32_t)c_begin;
#pragma unroll
      for (int q = 0; q < BN / 2 / 32; ++q) tmem_ld32_nowait(taddr + 32 * q, &r[32 * q]);
      asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acc_empty);        // TMEM free: next tile may start
      if (ncols > 0) {
        const int64_t col = (int64_t)nb * BN + c_begin;
        if (p.out_f32) {
          float4* dst = reinterpret_cast<float4*>(static_cast<float*>(p.c) + row * p.ldc + col);
#pragma unroll
          for (int q = 0; q < BN / 2 / 4; ++q) {
            float4 o;
            o.x = __uint_as_float(r[4 * q]) * scale;
            o.y = __uint_as_float(r[4 * q + 1]) * scale;
            o.z = __uint_as_float(r[4 * q + 2]) * scale;
            o.w = __uint_as_float(r[4 * q + 3]) * scale;
            amax = fmaxf(amax, fmaxf(fmaxf(fabsf(o.x), fabsf(o.y)), fmaxf(fabsf(o.z), fabsf(o.w))));
            dst[q] = o;
          }
        } else {
          uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.c) + row * p.ldc + col);
#pragma unroll
          for (int q = 0; q < BN / 2 / 8; ++q) {
            uint32_t w[4];
#pragma unroll
            for (int h = 0; h < 4; ++h) {
              const float a0 = __uint_as_float(r[8 * q + 2 * h]) * scale;
              const float a1 = __uint_as_float(r[8 * q + 2 * h + 1]) * scale;
              amax = fmaxf(amax, fmaxf(fabsf(a0), fabsf(a1)));
              __nv_bfloat162 b2 = __floats2bfloat162_rn(a0, a1);
              memcpy(&w[h], &b2, 4);
            }
            dst[q] = make_uint4(w[0], w[1], w[2], w[3]);
          }
        }
      }
    }
    if (p.c_amax != nullptr) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
      if (lane == 0) atomicMax(reinterpret_cast<unsigned int*>(p.c_amax), __float_as_uint(amax));
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

// ---------------------------------------------------------------------------
// Host side: tensor maps through the driver entry point (no libcuda link).
// ---------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

bool make_kmajor_map(CUtensorMap* map, const uint8_t* codes, int64_t rows, int64_t K,
                     uint32_t box_rows) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)(K / 2), (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)(K / 2)};
  cuuint32_t box[2] = {128u, box_rows};
  cuuint32_t estr[2] = {1u, 1u};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(codes), dims,
                   strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace

fp4_status gemm_launch(const GemmArgs& g, cudaStream_t s) {
  // Two or more 128-row blocks: the CTA-pair kernel (256 x 256 tiles, half
  // the B traffic per SM).  A single row block keeps the one-SM kernel.
  return gemm_launch_sfst(g, s);
  CUtensorMap ta, tb;
  if (!make_kmajor_map(&ta, g.a_codes, g.M, g.K, BM)) return FP4_ERR_CUDA;
  if (!make_kmajor_map(&tb, g.b_codes, g.N, g.K, BN)) return FP4_ERR_CUDA;
  KParams p;
  p.a_sf = g.a_sf; p.b_sf = g.b_sf; p.a_sdec = g.a_sdec; p.b_sdec = g.b_sdec;
  p.M = (int)g.M; p.N = (int)g.N; p.K = (int)g.K;
  p.alpha = g.alpha; p.c = g.c; p.ldc = g.ldc; p.out_f32 = g.out_f32;
  p.c_amax = g.c_amax; p.status = g.status;
  const int tiles = (int)(g.M / BM) * (int)((g.N + BN - 1) / BN);
  const int grid = tiles < sm_count() ? tiles : sm_count();
  if (g.c_amax != nullptr && cudaMemsetAsync(g.c_amax, 0, sizeof(float), s) != cudaSuccess)
    return FP4_ERR_CUDA;
  const int which = g.fmt == FP4_NVFP4 ? 0 : 1;
  cudaError_t e = which == 0
      ? cudaFuncSetAttribute(fp4_gemm_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES)
      : cudaFuncSetAttribute(fp4_gemm_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
  if (e != cudaSuccess) return FP4_ERR_CUDA;
  if (which == 0) fp4_gemm_kernel<true><<<grid, NUM_THREADS, SMEM_BYTES, s>>>(ta, tb, p);
  else fp4_gemm_kernel<false><<<grid, NUM_THREADS, SMEM_BYTES, s>>>(ta, tb, p);
  count_launches(1);
  return cudaGetLastError() == cudaSuccess ? FP4_OK : FP4_ERR_CUDA;
}

}  // namespace fp4impl
