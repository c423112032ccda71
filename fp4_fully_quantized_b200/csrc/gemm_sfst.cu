// gemm_sfst.cu -- block-scaled FP4 GEMM with scale factors staged by
// tcgen05.st (one SM per 128 x 256 output tile).
//
// The product is the one of the "FP4" page (How it works: FP4 tensor-core
// products with higher-precision accumulation).  The design point is how the
// per-block scales reach tensor memory.  Copying them with tcgen05.cp from the
// MMA-issuing thread puts 12 copies per 256-element K step into the same
// in-order tensor pipe as the 4 MMAs, and measured on B200 the MMAs then run at
// about half their rate.  Here four "scale" warps, one per TMEM lane quadrant,
// read each stage's scale atoms from shared memory and write them into the
// stage's TMEM slot with tcgen05.st, which proceeds alongside the MMAs; the
// MMA thread only issues MMAs.
//
// 512 threads:
//   warps 0..3   scale stagers (TMEM lane quadrant = warp), one K step at a time
//   warps 4..11  epilogue: quadrant warp % 4, column half (warp - 4) / 4
//   warp 12      TMA producer (A, B and the scale atoms into a 4-stage ring)
//   warp 13      TMEM allocation and MMA issue
// Barriers per stage: atoms (the scale atoms landed) -> scales (4 stagers
// wrote TMEM); full (the A and B tiles landed); the MMAs wait for both, and
// empty (the MMAs that read the stage finished; tcgen05.commit) frees the stage
// and its TMEM slot.  All waits are bounded.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cfloat>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "fp4_device.cuh"
#include "internal.h"
#include "sm100_ptx.cuh"

namespace fp4impl {
namespace {
using namespace ptx;

constexpr int BM = 128, BN = 256, BK = 256, MMA_K = 64;
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * BK / 2;          // 16 KB
constexpr int B_BYTES = BN * BK / 2;          // 32 KB
constexpr int SFA_BYTES = 4 * 512;
constexpr int SFB_BYTES = 2 * 4 * 512;
constexpr int STAGE_BYTES = A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES;
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 + 256;
constexpr int NUM_THREADS = 512;
constexpr int SF_WARP0 = 0, EPI_WARP0 = 4, EPI_WARPS = 8, PRODUCER_WARP = 12, MMA_WARP = 13;
constexpr int TMEM_COLS = 512;
constexpr int TMEM_SF_BASE = 256;
constexpr int TMEM_SF_STAGE = 48;             // 16 (A) + 32 (B) columns per stage
static_assert(TMEM_SF_BASE + STAGES * TMEM_SF_STAGE <= TMEM_COLS, "TMEM budget");
static_assert(SMEM_BYTES <= 232448, "shared-memory budget");

struct StParams {
  const uint8_t* a_sf; const uint8_t* b_sf;
  const float* a_sdec; const float* b_sdec;
  int M, N, K;
  int atoms_per_rowblk;
  float alpha;
  void* c; int64_t ldc; int out_mode;     // 0 BF16, 1 FP32, 2 NVFP4 1x16 RTN (q_*)
  float* c_amax;
  uint8_t* q_codes; uint8_t* q_scales; uint8_t* q_scales_mma;
  const float* q_amax_in; float* q_amax_out; float* q_s_dec;
  int q_sr;                   // out_mode 2: stochastic rounding (else to nearest)
  uint32_t q_stream;          // its Philox stream; keys below
  fp4dev::PhiloxKeys q_keys;
  uint32_t* status;
};

// Tile order: groups of kGroupM row blocks are walked column block by column
// block (row block fastest), so the tiles the persistent CTAs work on at one
// time share few A row blocks and few B column blocks, and both stay in L2
// while every CTA that needs them streams them (a row-major walk over all
// column blocks streams the whole of B once per wave of tiles).
constexpr int kGroupM = 16;

__device__ __forceinline__ void tile_coords(int tile, int tiles_m, int tiles_n, int& mb, int& nb) {
  const int per_group = kGroupM * tiles_n;
  const int g = tile / per_group, r = tile - g * per_group;
  const int m0 = g * kGroupM;
  const int gm = min(kGroupM, tiles_m - m0);
  nb = r / gm;
  mb = m0 + (r - nb * gm);
}

// Waits with one lane and broadcasts the result to the warp.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                          uint32_t* status, uint32_t where, int lane) {
  int ok = 1;
  if (lane == 0) ok = mbar_wait(bar, parity, abort_flag, status, where);
  return __shfl_sync(0xFFFFFFFFu, ok, 0) != 0;
}

template <bool NV>
__global__ void __launch_bounds__(NUM_THREADS, 1)
fp4_gemm_sfst_kernel(const __grid_constant__ CUtensorMap tmap_a,
                     const __grid_constant__ CUtensorMap tmap_b, const StParams p) {
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
  auto sf_bar = [&](int s) { return bar0 + 8u * (2 * STAGES + s); };
  auto atoms_bar = [&](int s) { return bar0 + 8u * (3 * STAGES + s); };
  const uint32_t acc_full = bar0 + 8u * (4 * STAGES);
  const uint32_t acc_empty = bar0 + 8u * (4 * STAGES + 1);
  const uint32_t drain_bar = bar0 + 8u * (4 * STAGES + 2);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + 4 * STAGES + 3);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tiles_m = p.M / BM, tiles_n = (p.N + BN - 1) / BN;
  const int num_tiles = tiles_m * tiles_n;
  const int k_blocks = (p.K + BK - 1) / BK;
  const int apr = p.atoms_per_rowblk;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
      mbar_init(sf_bar(s), 4);
      mbar_init(atoms_bar(s), 1);
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
        int mb, nb;
        tile_coords(tile, tiles_m, tiles_n, mb, nb);
        const bool b_hi = (nb * 2 + 1) * 128 < p.N;
        for (int kb = 0; kb < k_blocks; ++kb, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1u;
          if (!mbar_wait(empty_bar(s), ph ^ 1u, abort_flag, p.status, 0x3100 + s)) { ok = false; break; }
          const int n_atoms = NV ? min(4, apr - kb * 4) : min(2, apr - kb * 2);
          const uint32_t atom_bytes = (uint32_t)n_atoms * 512u;
          // scale atoms first, on their own barrier: the stagers move them into
          // tensor memory while the operand tiles are still in flight
          mbar_arrive_expect_tx(atoms_bar(s), atom_bytes * (b_hi ? 3u : 2u));
          const int atom0 = kb * (NV ? 4 : 2);
          bulk_load(smem_u32(sSFA(s)), p.a_sf + ((size_t)mb * apr + atom0) * 512, atom_bytes,
                    atoms_bar(s));
          bulk_load(smem_u32(sSFB(s)), p.b_sf + ((size_t)(2 * nb) * apr + atom0) * 512, atom_bytes,
                    atoms_bar(s));
          if (b_hi)
            bulk_load(smem_u32(sSFB(s) + 4 * 512), p.b_sf + ((size_t)(2 * nb + 1) * apr + atom0) * 512,
                      atom_bytes, atoms_bar(s));
          mbar_arrive_expect_tx(full_bar(s), A_BYTES + B_BYTES);
          tma_load_2d(smem_u32(sA(s)), &tmap_a, full_bar(s), kb * (BK / 2), mb * BM);
          tma_load_2d(smem_u32(sB(s)), &tmap_b, full_bar(s), kb * (BK / 2), nb * BN);
        }
      }
      if (it > 0) {
        const uint32_t first = it > (uint32_t)STAGES ? it - STAGES : 0;
        for (uint32_t j = first; j < it; ++j) {
          volatile int no_abort = 0;
          mbar_wait(atoms_bar(j % STAGES), (j / STAGES) & 1u, &no_abort, p.status, 0x3200 + j % STAGES);
          mbar_wait(full_bar(j % STAGES), (j / STAGES) & 1u, &no_abort, p.status, 0x3200 + j % STAGES);
        }
      }
    }
  } else if (warp < SF_WARP0 + 4) {
    // ------------------------------------------------------------ scale stagers
    // Tensor-memory scale layout the MMA reads (what a 32x128b.warpx4 copy of
    // a 512-byte atom produces): every lane quadrant holds the whole atom,
    // lane 32q + r holds the atom's 16-byte row r in 4 consecutive columns.
    const int q = warp - SF_WARP0;
    const uint32_t lane_base = (uint32_t)(q * 32) << 16;
    uint32_t it = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
      for (int kb = 0; kb < k_blocks; ++kb, ++it) {
        const int s = it % STAGES;
        const uint32_t ph = (it / STAGES) & 1u;
        if (!warp_wait(atoms_bar(s), ph, abort_flag, p.status, 0x3300 + s, lane)) { ok = false; break; }
        uint32_t va[16], vb[32];
        const uint8_t* fa = sSFA(s) + lane * 16;
        const uint8_t* fb = sSFB(s) + lane * 16;
#pragma unroll
        for (int a = 0; a < 4; ++a) {
          const uint4 x = *reinterpret_cast<const uint4*>(fa + a * 512);
          va[4 * a] = x.x; va[4 * a + 1] = x.y; va[4 * a + 2] = x.z; va[4 * a + 3] = x.w;
          const uint4 y0 = *reinterpret_cast<const uint4*>(fb + a * 512);
          const uint4 y1 = *reinterpret_cast<const uint4*>(fb + 2048 + a * 512);
          vb[8 * a] = y0.x; vb[8 * a + 1] = y0.y; vb[8 * a + 2] = y0.z; vb[8 * a + 3] = y0.w;
          vb[8 * a + 4] = y1.x; vb[8 * a + 5] = y1.y; vb[8 * a + 6] = y1.z; vb[8 * a + 7] = y1.w;
        }
        const uint32_t t_sfa = tmem_base + TMEM_SF_BASE + s * TMEM_SF_STAGE;
        tmem_st_x16(lane_base + t_sfa, va);
        tmem_st_x32(lane_base + t_sfa + 16, vb);
        asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(sf_bar(s));
      }
    }
  } else if (warp == MMA_WARP) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      uint32_t it = 0, tile_iter = 0;
      bool ok = true, issued = false;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x, ++tile_iter) {
        if (!mbar_wait(acc_empty, (tile_iter & 1u) ^ 1u, abort_flag, p.status, 0x3400)) { ok = false; break; }
        tc_fence_after();
        for (int kb = 0; kb < k_blocks; ++kb, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1u;
          if (!mbar_wait(sf_bar(s), ph, abort_flag, p.status, 0x3500 + s)) { ok = false; break; }
          if (!mbar_wait(full_bar(s), ph, abort_flag, p.status, 0x3580 + s)) { ok = false; break; }
          tc_fence_after();
          const int n_mma = min(BK / MMA_K, (p.K - kb * BK) / MMA_K);
          const uint32_t t_sfa = tmem_base + TMEM_SF_BASE + s * TMEM_SF_STAGE;
          const uint32_t t_sfb = t_sfa + 16;
          const uint32_t a_base = smem_u32(sA(s)), b_base = smem_u32(sB(s));
          auto step = [&](int kk) {
            uint32_t sfa_addr, sfb_addr, idesc;
            if (NV) {
              sfa_addr = t_sfa + 4 * kk;
              sfb_addr = t_sfb + 8 * kk;
              idesc = make_idesc(BN, BM, 0u, 0u, 0u);
            } else {
              const uint32_t byte = (uint32_t)(kk & 1) * 2u;
              sfa_addr = (t_sfa + 4 * (kk >> 1)) | (byte << 30);
              sfb_addr = (t_sfb + 8 * (kk >> 1)) | (byte << 30);
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
          tc_commit(empty_bar(s));
        }
        if (!ok) break;
        tc_commit(acc_full);
      }
      if (issued) {
        tc_commit(drain_bar);
        volatile int no_abort = 0;
        mbar_wait(drain_bar, 0, &no_abort, p.status, 0x3600);
      }
    }
  } else if (warp >= EPI_WARP0 && warp < EPI_WARP0 + EPI_WARPS) {
    // ------------------------------------------------------------ epilogue
    const float scale = p.alpha * (*p.a_sdec) * (*p.b_sdec);
    const int esize = p.out_mode == 1 ? 4 : 2;
    const bool wide_st = (reinterpret_cast<uintptr_t>(p.c) % 32) == 0 && (p.ldc * esize) % 32 == 0;
    float q_senc = 1.0f;
    if (p.out_mode == 2) {
      // encode with the supplied tensor amax (the two-level NVFP4 scale of the
      // quantizers); record it and the decode scale with the codes
      const float A = *p.q_amax_in;
      float q_sdec;
      fp4dev::nvfp4_global_scales(A, q_senc, q_sdec);
      if (blockIdx.x == 0 && threadIdx.x == EPI_WARP0 * 32) {
        if (!(A <= FLT_MAX)) set_status(p.status, FP4_ERR_NONFINITE, 5);
        *p.q_s_dec = q_sdec;
        if (p.q_amax_out != p.q_amax_in) *p.q_amax_out = A;
      }
    }
    float amax = 0.0f;
    uint32_t tile_iter = 0;
    const int quad = warp & 3, half = (warp - EPI_WARP0) >> 2;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++tile_iter) {
      if (!warp_wait(acc_full, tile_iter & 1u, abort_flag, p.status, 0x3700 + warp, lane)) break;
      tc_fence_after();
      int mb, nb;
      tile_coords(tile, tiles_m, tiles_n, mb, nb);
      const int64_t row = (int64_t)mb * BM + quad * 32 + lane;
      const int c_begin = half * (BN / 2);
      const int ncols = min(BN / 2, p.N - nb * BN - c_begin);
      const int64_t col = (int64_t)nb * BN + c_begin;
      const uint32_t taddr = tmem_base + ((uint32_t)(quad * 32) << 16) + (uint32_t)c_begin;
      if (p.out_mode == 0) {
        // drain 128 columns in two 64-column loads, packing to BF16 as they
        // arrive (64 registers); the accumulator is released as soon as the
        // second load has landed, before that half is packed, so the next
        // tile's MMAs wait for two TMEM round trips and one packing only
        uint32_t pk[64];
        {
          uint32_t r2[64];
          tmem_ld32_nowait(taddr, r2);
          tmem_ld32_nowait(taddr + 32, r2 + 32);
          asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
          for (int h = 0; h < 32; ++h) {
            const float a0 = __uint_as_float(r2[2 * h]) * scale;
            const float a1 = __uint_as_float(r2[2 * h + 1]) * scale;
            amax = fmaxf(amax, fmaxf(fabsf(a0), fabsf(a1)));
            __nv_bfloat162 b2 = __floats2bfloat162_rn(a0, a1);
            memcpy(&pk[h], &b2, 4);
          }
        }
        {
          uint32_t r2[64];
          tmem_ld32_nowait(taddr + 64, r2);
          tmem_ld32_nowait(taddr + 96, r2 + 32);
          asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(acc_empty);
#pragma unroll
          for (int h = 0; h < 32; ++h) {
            const float a0 = __uint_as_float(r2[2 * h]) * scale;
            const float a1 = __uint_as_float(r2[2 * h + 1]) * scale;
            amax = fmaxf(amax, fmaxf(fabsf(a0), fabsf(a1)));
            __nv_bfloat162 b2 = __floats2bfloat162_rn(a0, a1);
            memcpy(&pk[32 + h], &b2, 4);
          }
        }
        if (ncols > 0) {
          __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(p.c) + row * p.ldc + col;
          if (wide_st) {          // full 32-byte sectors
#pragma unroll
            for (int q = 0; q < 8; ++q)
              st_global_v8(dst + 16 * q, pk[8 * q], pk[8 * q + 1], pk[8 * q + 2], pk[8 * q + 3],
                           pk[8 * q + 4], pk[8 * q + 5], pk[8 * q + 6], pk[8 * q + 7]);
          } else {
            uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
            for (int q = 0; q < 16; ++q) d4[q] = make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
          }
        }
      } else if (p.out_mode == 2) {
        // NVFP4 1x16, round to nearest: each 16-column block of the FP32
        // result gets its E4M3 scale from its own max, then 16 E2M1 codes;
        // two halves of 64 columns, the accumulator released after the second
        const int64_t S = p.N >> 4, S4 = (S + 3) & ~3LL;
#pragma unroll 1
        for (int h2 = 0; h2 < 2; ++h2) {
          uint32_t v[64];
          tmem_ld32_nowait(taddr + 64 * h2, v);
          tmem_ld32_nowait(taddr + 64 * h2 + 32, v + 32);
          asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
          if (h2 == 1) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(acc_empty);
          }
          if (ncols > 0) {
            uint32_t cw[8];
            uint32_t sfw = 0;
#pragma unroll
            for (int b = 0; b < 4; ++b) {
              float o[16];
              float bmax = 0.0f;
#pragma unroll
              for (int e = 0; e < 16; ++e) {
                o[e] = __uint_as_float(v[16 * b + e]) * scale;
                bmax = fmaxf(bmax, fabsf(o[e]));
              }
              amax = fmaxf(amax, bmax);
              const int64_t cb = col + 64 * h2 + 16 * b;   // first column of the block
              if (p.c != nullptr) {
                // the FP32 result also leaves as BF16 (for a consumer that
                // still needs it, e.g. the transposed quantization)
                uint32_t pk[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                  __nv_bfloat162 b2 = __floats2bfloat162_rn(o[2 * e], o[2 * e + 1]);
                  memcpy(&pk[e], &b2, 4);
                }
                __nv_bfloat16* bd = static_cast<__nv_bfloat16*>(p.c) + row * p.ldc + cb;
                if (wide_st) {
                  st_global_v8(bd, pk[0], pk[1], pk[2], pk[3], pk[4], pk[5], pk[6], pk[7]);
                } else {
                  reinterpret_cast<uint4*>(bd)[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                  reinterpret_cast<uint4*>(bd)[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
                }
              }
              const uint32_t sf = fp4dev::e4m3_rn_sat(fp4dev::div6_for_scale(__fmul_rn(bmax, q_senc)));
              const float inv = (sf == 0u || sf == 127u)
                                    ? 0.0f : fminf(__fdiv_rn(q_senc, fp4dev::e4m3_value(sf)), FLT_MAX);
#pragma unroll
              for (int e = 0; e < 16; ++e) o[e] = __fmul_rn(o[e], inv);
              if (p.q_sr) {
                // draws of elements row * N + cb .. + 15: two Philox blocks
                const uint64_t i0 = (uint64_t)row * (uint64_t)p.N + (uint64_t)cb;
                cw[2 * b] = fp4dev::e2m1x8_sr(o, fp4dev::philox_keyed(i0 >> 3, p.q_stream, p.q_keys));
                cw[2 * b + 1] = fp4dev::e2m1x8_sr(o + 8, fp4dev::philox_keyed((i0 >> 3) + 1, p.q_stream, p.q_keys));
              } else {
                cw[2 * b] = fp4dev::e2m1x8_rn(o);
                cw[2 * b + 1] = fp4dev::e2m1x8_rn(o + 8);
              }
              sfw |= sf << (8 * b);
            }
            const int64_t c0 = col + 64 * h2;              // first column of these 4 blocks
            uint4* cd = reinterpret_cast<uint4*>(p.q_codes + row * (p.N >> 1) + (c0 >> 1));
            cd[0] = make_uint4(cw[0], cw[1], cw[2], cw[3]);
            cd[1] = make_uint4(cw[4], cw[5], cw[6], cw[7]);
            const int64_t sb0 = c0 >> 4;                   // a multiple of 4
            if (p.q_scales != nullptr) *reinterpret_cast<uint32_t*>(p.q_scales + row * S + sb0) = sfw;
            if (p.q_scales_mma != nullptr)
              *reinterpret_cast<uint32_t*>(p.q_scales_mma + fp4dev::mma_sf_offset(row, sb0, S4)) = sfw;
          }
        }
      } else {
        // FP32: two halves of 64 columns; the accumulator is released after
        // the second half is in registers
        float* dst = static_cast<float*>(p.c) + row * p.ldc + col;
#pragma unroll 1
        for (int h2 = 0; h2 < 2; ++h2) {
          uint32_t v[64];
          tmem_ld32_nowait(taddr + 64 * h2, v);
          tmem_ld32_nowait(taddr + 64 * h2 + 32, v + 32);
          asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
          if (h2 == 1) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(acc_empty);
          }
          if (ncols > 0) {
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              float o[8];
#pragma unroll
              for (int e = 0; e < 8; ++e) {
                o[e] = __uint_as_float(v[8 * q + e]) * scale;
                amax = fmaxf(amax, fabsf(o[e]));
              }
              float* d = dst + 64 * h2 + 8 * q;
              if (wide_st) {
                st_global_v8(d, __float_as_uint(o[0]), __float_as_uint(o[1]), __float_as_uint(o[2]),
                             __float_as_uint(o[3]), __float_as_uint(o[4]), __float_as_uint(o[5]),
                             __float_as_uint(o[6]), __float_as_uint(o[7]));
              } else {
                reinterpret_cast<float4*>(d)[0] = make_float4(o[0], o[1], o[2], o[3]);
                reinterpret_cast<float4*>(d)[1] = make_float4(o[4], o[5], o[6], o[7]);
              }
            }
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

}  // namespace

fp4_status gemm_launch(const GemmArgs& g, cudaStream_t s) {
  const bool nv = g.fmt == FP4_NVFP4;
  CUtensorMap ta, tb;
  if (!codes_map(&ta, g.a_codes, g.M, g.K, BM)) return FP4_ERR_CUDA;
  if (!codes_map(&tb, g.b_codes, g.N, g.K, BN)) return FP4_ERR_CUDA;
  StParams p;
  p.a_sf = g.a_sf; p.b_sf = g.b_sf; p.a_sdec = g.a_sdec; p.b_sdec = g.b_sdec;
  p.M = (int)g.M; p.N = (int)g.N; p.K = (int)g.K;
  p.atoms_per_rowblk = nv ? (int)(g.K / 64) : (int)((((g.K / 32) + 3) / 4 * 4) / 4);
  p.alpha = g.alpha; p.c = g.c; p.ldc = g.ldc; p.out_mode = g.out_mode;
  p.q_codes = g.q_codes; p.q_scales = g.q_scales; p.q_scales_mma = g.q_scales_mma;
  p.q_amax_in = g.q_amax_in; p.q_amax_out = g.q_amax_out; p.q_s_dec = g.q_s_dec;
  p.q_sr = g.q_sr; p.q_stream = g.q_stream; p.q_keys = fp4dev::philox_keys(g.q_seed);
  p.c_amax = g.c_amax; p.status = g.status;
  const int tiles = (int)(g.M / BM) * (int)((g.N + BN - 1) / BN);
  const int grid = tiles < sm_count() ? tiles : sm_count();
  if (g.c_amax != nullptr && cudaMemsetAsync(g.c_amax, 0, sizeof(float), s) != cudaSuccess)
    return FP4_ERR_CUDA;
  cudaError_t e;
  if (nv) {
    e = cudaFuncSetAttribute(fp4_gemm_sfst_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             SMEM_BYTES);
    if (e != cudaSuccess) return FP4_ERR_CUDA;
    fp4_gemm_sfst_kernel<true><<<grid, NUM_THREADS, SMEM_BYTES, s>>>(ta, tb, p);
  } else {
    e = cudaFuncSetAttribute(fp4_gemm_sfst_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             SMEM_BYTES);
    if (e != cudaSuccess) return FP4_ERR_CUDA;
    fp4_gemm_sfst_kernel<false><<<grid, NUM_THREADS, SMEM_BYTES, s>>>(ta, tb, p);
  }
  count_launches(1);
  return cudaGetLastError() == cudaSuccess ? FP4_OK : FP4_ERR_CUDA;
}

}  // namespace fp4impl
