// gemm_pair.cu -- block-scaled FP4 GEMM with the CTA-pair (cta_group::2) MMA.
//
// Same product as gemm_sm100.cu ("FP4" page, How it works: FP4 tensor-core
// matrix products with higher-precision accumulation), but a cluster of two
// CTAs on two SMs computes one 256 x 256 output tile: each CTA loads its 128
// rows of A and its 128-row half of B, so the operand traffic per SM per
// 256-element K step drops from 48 KB to 32 KB, and the leader CTA issues
// tcgen05.mma.cta_group::2 (256 x 256 x 64), which reads A and B from both
// CTAs' shared memory and accumulates each CTA's 128 rows in its own TMEM.
//
// Per CTA (320 threads): warp 8 = TMA producer (A, half of B, this CTA's
// scale atoms and the pair's B scale atoms; every copy completes on the
// leader's stage barrier), warp 9 = TMEM allocation (both CTAs) and, in the
// leader only, scale-factor copies into TMEM plus the MMAs, whose completion is
// multicast to both CTAs' barriers; warps 0..7 = epilogue of the CTA's own
// 128 rows (drain to registers, release to the leader, scale, store).
// No TMA load uses cluster multicast.  All mbarrier waits are bounded.
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
using namespace ptx;

constexpr int PM = 256;              // pair tile rows (M); 128 per CTA
constexpr int PN = 256;              // pair tile cols (N) = UMMA N
constexpr int CM = 128;              // rows per CTA
constexpr int BK = 256;              // K elements per stage
constexpr int MMA_K = 64;
constexpr int STAGES = 5;
constexpr int A_BYTES = CM * BK / 2;            // 16 KB
constexpr int B_BYTES = (PN / 2) * BK / 2;      // 16 KB (this CTA's half of B)
constexpr int SFA_BYTES = 4 * 512;              // scale atoms of this CTA's 128 rows
constexpr int SFB_BYTES = 2 * 4 * 512;          // scale atoms of the pair's 256 B rows
constexpr int STAGE_BYTES = A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES;
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 + 256;
constexpr int NUM_THREADS = 320;
constexpr int EPI_WARPS = 8;
constexpr int PRODUCER_WARP = 8;
constexpr int MMA_WARP = 9;
constexpr int TMEM_COLS = 512;
constexpr int TMEM_SF_BASE = 256;
constexpr int TMEM_SF_STAGE = 48;               // 16 (A) + 32 (B) columns per stage
static_assert(TMEM_SF_BASE + STAGES * TMEM_SF_STAGE <= TMEM_COLS, "TMEM budget");
static_assert(SMEM_BYTES <= 232448, "shared-memory budget");

struct PairParams {
  const float* a_sdec; const float* b_sdec;
  int M, N, K;
  int atoms_per_rowblk;     // scale atoms (128 rows x 4 scales) per 128-row block
  int atoms_per_stage;      // NVFP4: 4 (64 K each), MXFP4: 2 (128 K each)
  float alpha;
  void* c; int64_t ldc; int out_f32;
  float* c_amax;
  uint32_t* status;
};

template <bool NV>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(NUM_THREADS, 1)
fp4_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmap_a,
                     const __grid_constant__ CUtensorMap tmap_b,
                     const __grid_constant__ CUtensorMap tmap_sfa,
                     const __grid_constant__ CUtensorMap tmap_sfb, const PairParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  auto sA = [&](int s) { return base + s * A_BYTES; };
  auto sB = [&](int s) { return base + STAGES * A_BYTES + s * B_BYTES; };
  auto sSFA = [&](int s) { return base + STAGES * (A_BYTES + B_BYTES) + s * SFA_BYTES; };
  auto sSFB = [&](int s) {
    return base + STAGES * (A_BYTES + B_BYTES + SFA_BYTES) + s * SFB_BYTES;
  };
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + STAGES * STAGE_BYTES);
  const uint32_t bar0 = smem_u32(bars);
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (STAGES + s); };
  const uint32_t acc_full = bar0 + 8u * (2 * STAGES);
  const uint32_t acc_empty = bar0 + 8u * (2 * STAGES + 1);
  const uint32_t drain_bar = bar0 + 8u * (2 * STAGES + 2);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + 2 * STAGES + 3);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int pair_id = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  const int tiles_m = (p.M + PM - 1) / PM, tiles_n = (p.N + PN - 1) / PN;
  const int num_tiles = tiles_m * tiles_n;
  const int k_blocks = (p.K + BK - 1) / BK;
  const int APS = p.atoms_per_stage;
  const uint32_t stage_tx = (uint32_t)(A_BYTES + B_BYTES + 3 * APS * 512);   // per CTA

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, 2 * EPI_WARPS);
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == MMA_WARP) tmem_alloc_pair(smem_u32(tmem_holder), TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  cluster_sync();                 // peer barriers initialised before any remote arrive
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;

  if (warp == PRODUCER_WARP) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_a)) : "memory");
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_b)) : "memory");
      uint32_t it = 0;
      bool ok = true;
      for (int tile = pair_id; tile < num_tiles && ok; tile += npairs) {
        const int pm = tile / tiles_n, nb = tile % tiles_n;
        const int arow = pm * PM + (int)rank * CM;
        const int brow = nb * PN + (int)rank * (PN / 2);
        const int sfa_row = (pm * 2 + (int)rank) * p.atoms_per_rowblk;
        const int sfb_row0 = (nb * 2) * p.atoms_per_rowblk;
        const int sfb_row1 = (nb * 2 + 1) * p.atoms_per_rowblk;
        for (int kb = 0; kb < k_blocks; ++kb, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1u;
          if (!mbar_wait(empty_bar(s), ph ^ 1u, abort_flag, p.status, 0x1100 + s)) { ok = false; break; }
          const uint32_t fb = mapa_shared(full_bar(s), 0);     // the leader's barrier
          if (leader) mbar_arrive_expect_tx(full_bar(s), 2u * stage_tx);
          tma_load_2d_pair(smem_u32(sA(s)), &tmap_a, fb, kb * (BK / 2), arow);
          tma_load_2d_pair(smem_u32(sB(s)), &tmap_b, fb, kb * (BK / 2), brow);
          const int a0 = kb * APS;
          tma_load_2d_pair(smem_u32(sSFA(s)), &tmap_sfa, fb, 0, sfa_row + a0);
          tma_load_2d_pair(smem_u32(sSFB(s)), &tmap_sfb, fb, 0, sfb_row0 + a0);
          tma_load_2d_pair(smem_u32(sSFB(s) + 4 * 512), &tmap_sfb, fb, 0, sfb_row1 + a0);
        }
      }
      // Drain (leader): its stage barriers count both CTAs' copies, so once
      // the last armed phases complete no copy into either CTA is in flight.
      if (leader && it > 0) {
        const uint32_t first = it > (uint32_t)STAGES ? it - STAGES : 0;
        for (uint32_t j = first; j < it; ++j) {
          volatile int no_abort = 0;
          mbar_wait(full_bar(j % STAGES), (j / STAGES) & 1u, &no_abort, p.status, 0x1200 + j % STAGES);
        }
      }
    }
  } else if (warp == MMA_WARP) {
    // ------------------------------------------------------------ MMA (leader)
    if (leader && lane == 0) {
      uint32_t it = 0, tile_iter = 0;
      bool ok = true, issued = false;
      const uint32_t idesc_nv = make_idesc(PN, PM, 0u, 0u, 0u);
      for (int tile = pair_id; tile < num_tiles && ok; tile += npairs, ++tile_iter) {
        if (!mbar_wait(acc_empty, (tile_iter & 1u) ^ 1u, abort_flag, p.status, 0x1300)) { ok = false; break; }
        tc_fence_after();
        for (int kb = 0; kb < k_blocks; ++kb, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1u;
          if (!mbar_wait(full_bar(s), ph, abort_flag, p.status, 0x1400 + s)) { ok = false; break; }
          const int n_mma = min(BK / MMA_K, (p.K - kb * BK) / MMA_K);
          const uint32_t t_sfa = tmem_base + TMEM_SF_BASE + s * TMEM_SF_STAGE;
          const uint32_t t_sfb = t_sfa + 16;
          const uint32_t a_base = smem_u32(sA(s)), b_base = smem_u32(sB(s));
          const uint32_t sfa_s = smem_u32(sSFA(s)), sfb_s = smem_u32(sSFB(s));
          auto step = [&](int kk) {
            uint32_t sfa_addr, sfb_addr, idesc;
            const int atom = NV ? kk : (kk >> 1);
            if (NV || (kk & 1) == 0) {
              tc_cp_pair_32x128b(t_sfa + 4 * atom, smem_desc(sfa_s + atom * 512, 0, 128, 0));
              tc_cp_pair_32x128b(t_sfb + 8 * atom, smem_desc(sfb_s + atom * 512, 0, 128, 0));
              tc_cp_pair_32x128b(t_sfb + 8 * atom + 4, smem_desc(sfb_s + 2048 + atom * 512, 0, 128, 0));
            }
            if (NV) {
              sfa_addr = t_sfa + 4 * kk;
              sfb_addr = t_sfb + 8 * kk;
              idesc = idesc_nv;
            } else {
              const uint32_t byte = (uint32_t)(kk & 1) * 2u;
              sfa_addr = (t_sfa + 4 * atom) | (byte << 30);
              sfb_addr = (t_sfb + 8 * atom) | (byte << 30);
              idesc = make_idesc(PN, PM, 1u, byte, byte);
            }
            tc_mma_pair<NV>(tmem_base, smem_desc(a_base + kk * (MMA_K / 2), 16, 1024, 2),
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
          tc_commit_pair(empty_bar(s), 0x3);      // both CTAs may refill stage s
        }
        if (!ok) break;
        tc_commit_pair(acc_full, 0x3);            // both CTAs' accumulators ready
      }
      if (issued) {
        tc_commit_pair(drain_bar, 0x1);
        volatile int no_abort = 0;
        mbar_wait(drain_bar, 0, &no_abort, p.status, 0x1500);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const float scale = p.alpha * (*p.a_sdec) * (*p.b_sdec);
    const uint32_t leader_acc_empty = mapa_shared(acc_empty, 0);
    float amax = 0.0f;
    uint32_t tile_iter = 0;
    const int quad = warp & 3, half = warp >> 2;
    for (int tile = pair_id; tile < num_tiles; tile += npairs, ++tile_iter) {
      int ok = 1;
      if (lane == 0) ok = mbar_wait(acc_full, tile_iter & 1u, abort_flag, p.status, 0x1600 + warp);
      ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
      if (!ok) break;
      tc_fence_after();
      const int pm = tile / tiles_n, nb = tile % tiles_n;
      const int64_t row = (int64_t)pm * PM + (int64_t)rank * CM + quad * 32 + lane;
      const int c_begin = half * (PN / 2);
      const int ncols = min(PN / 2, p.N - nb * PN - c_begin);
      uint32_t r[PN / 2];
      const uint32_t taddr = tmem_base + ((uint32_t)(quad * 32) << 16) + (uint32_t)c_begin;
#pragma unroll
      for (int q = 0; q < PN / 2 / 32; ++q) tmem_ld32_nowait(taddr + 32 * q, &r[32 * q]);
      asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(leader_acc_empty);
      if (ncols > 0 && row < p.M) {
        const int64_t col = (int64_t)nb * PN + c_begin;
        if (p.out_f32) {
          float4* dst = reinterpret_cast<float4*>(static_cast<float*>(p.c) + row * p.ldc + col);
#pragma unroll
          for (int q = 0; q < PN / 2 / 4; ++q) {
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
          for (int q = 0; q < PN / 2 / 8; ++q) {
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
  cluster_sync();                 // no remote arrive or copy targets an exited CTA
  if (warp == MMA_WARP) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, TMEM_COLS);
  }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* q = nullptr;
    cudaDriverEntryPointQueryResult r;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &q, 12000, cudaEnableDefault,
                                         &r) == cudaSuccess &&
        r == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(q);
  });
  return fn;
}

// K-major FP4 codes [rows, K/2] bytes, 128-byte x box_rows tiles, 128B swizzle.
bool codes_map(CUtensorMap* m, const uint8_t* codes, int64_t rows, int64_t K, uint32_t box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)(K / 2), (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)(K / 2)};
  cuuint32_t box[2] = {128u, box_rows};
  cuuint32_t es[2] = {1u, 1u};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(codes), dims, strides, box,
             es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Tensor-core scale layout viewed as [atoms, 128 x u32] (one 512-byte atom a
// row); a box is `atoms_per_stage` consecutive atoms.
bool scales_map(CUtensorMap* m, const uint8_t* sf, int64_t total_atoms, uint32_t box_atoms) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {128u, (cuuint64_t)total_atoms};
  cuuint64_t strides[1] = {512u};
  cuuint32_t box[2] = {128u, box_atoms};
  cuuint32_t es[2] = {1u, 1u};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<uint8_t*>(sf), dims, strides, box,
             es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

fp4_status gemm_launch_pair(const GemmArgs& g, cudaStream_t s) {
  const bool nv = g.fmt == FP4_NVFP4;
  const int64_t S4 = nv ? g.K / 16 : ((g.K / 32) + 3) / 4 * 4;       // scales per row, padded
  const int apr = (int)(S4 / 4);
  const int aps = nv ? 4 : 2;
  const int64_t m_blocks = (g.M + 127) / 128, n_blocks = (g.N + 127) / 128;
  CUtensorMap ta, tb, tsa, tsb;
  if (!codes_map(&ta, g.a_codes, g.M, g.K, CM)) return FP4_ERR_CUDA;
  if (!codes_map(&tb, g.b_codes, g.N, g.K, PN / 2)) return FP4_ERR_CUDA;
  if (!scales_map(&tsa, g.a_sf, m_blocks * apr, aps)) return FP4_ERR_CUDA;
  if (!scales_map(&tsb, g.b_sf, n_blocks * apr, aps)) return FP4_ERR_CUDA;
  PairParams p;
  p.a_sdec = g.a_sdec; p.b_sdec = g.b_sdec;
  p.M = (int)g.M; p.N = (int)g.N; p.K = (int)g.K;
  p.atoms_per_rowblk = apr; p.atoms_per_stage = aps;
  p.alpha = g.alpha; p.c = g.c; p.ldc = g.ldc; p.out_f32 = g.out_f32;
  p.c_amax = g.c_amax; p.status = g.status;
  const int tiles = (int)(((g.M + PM - 1) / PM) * ((g.N + PN - 1) / PN));
  int grid = (sm_count() / 2) * 2;
  if (2 * tiles < grid) grid = 2 * tiles;
  if (g.c_amax != nullptr && cudaMemsetAsync(g.c_amax, 0, sizeof(float), s) != cudaSuccess)
    return FP4_ERR_CUDA;
  cudaError_t e;
  if (nv) {
    e = cudaFuncSetAttribute(fp4_gemm_pair_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             SMEM_BYTES);
    if (e != cudaSuccess) return FP4_ERR_CUDA;
    fp4_gemm_pair_kernel<true><<<grid, NUM_THREADS, SMEM_BYTES, s>>>(ta, tb, tsa, tsb, p);
  } else {
    e = cudaFuncSetAttribute(fp4_gemm_pair_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             SMEM_BYTES);
    if (e != cudaSuccess) return FP4_ERR_CUDA;
    fp4_gemm_pair_kernel<false><<<grid, NUM_THREADS, SMEM_BYTES, s>>>(ta, tb, tsa, tsb, p);
  }
  count_launches(1);
  return cudaGetLastError() == cudaSuccess ? FP4_OK : FP4_ERR_CUDA;
}

}  // namespace fp4impl
