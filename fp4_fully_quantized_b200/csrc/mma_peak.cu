// mma_peak.cu -- tensor-core rate microbenchmark for the FP4 GEMM roofline.
//
// One persistent CTA (or CTA pair) per SM issues back-to-back block-scaled
// FP4 MMAs on operands resident in shared memory, with nothing else in the
// loop, so the elapsed time measures the instruction rate the tensor cores
// sustain on this part (the denominator the GEMM's tensor-pipe fraction is
// reported against, next to the nominal figure).  Variants:
//   0  cta_group::1, kind::mxf4nvf4 (NVFP4 scales), 128 x 256 x 64 per MMA
//   1  as 0, plus the 3 scale-factor copies (tcgen05.cp) per MMA that a GEMM
//      K step needs
//   2  cta_group::2, 256 x 256 x 64 per MMA (CTA pair)
//   3  as 2, plus the scale-factor copies
//   4  as 0, with the copies issued concurrently by a second warp (into a
//      separate TMEM region) instead of by the MMA thread
//   5  as 2, the same for the CTA pair
//   6  as 0, with one K step's twelve copies (4 A atoms, 8 B atoms) issued
//      together before its 4 MMAs, into five rotating 48-column slots: the
//      order and tensor-memory layout a copy-fed GEMM would use
//   7  as 6, for the CTA pair (tcgen05.cp.cta_group::2)
// Operands are filled with pseudo-random codes and unit scales.  Waits are
// bounded like the GEMM's.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "internal.h"
#include "sm100_ptx.cuh"

namespace fp4impl {
namespace {
using namespace ptx;

// ---------------------------------------------------------------------------
// CTA-pair (cta_group::2) forms: a cluster of two CTAs on two SMs shares one
// MMA.  Only this microbenchmark uses them; the library's GEMM is one SM per
// tile.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" :::
                   "memory");
}
__device__ __forceinline__ void tmem_alloc_pair(uint32_t holder_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   holder_smem),
               "r"(ncols));
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols));
}
// Arrive (once) on the mbarrier at this offset in every CTA of `mask` when
// all tcgen05 operations issued so far by this thread have completed.
__device__ __forceinline__ void tc_commit_pair(uint32_t bar, uint16_t mask) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
      " [%0], %1;" ::"r"(bar), "h"(mask)
      : "memory");
}
__device__ __forceinline__ void tc_cp_pair_32x128b(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::2.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc));
}
template <bool NV>
__device__ __forceinline__ void tc_mma_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                            uint32_t idesc, uint32_t sfa, uint32_t sfb,
                                            uint32_t accumulate) {
  if constexpr (NV) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.scale_vec::4X"
        " [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb));
  } else {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::mxf4.block_scale.scale_vec::2X"
        " [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb));
  }
}


constexpr int A_BYTES = 128 * 128;      // 128 rows x 256 FP4
constexpr int B_BYTES = 256 * 128;      // 256 rows (1 SM) / 128 rows per CTA (pair)
constexpr int SF_BYTES = 3 * 512;
constexpr int PEAK_SMEM = A_BYTES + B_BYTES + SF_BYTES + 1024 + 64 + 16;

__device__ __forceinline__ uint32_t hash32(uint32_t x) {
  x ^= x >> 16; x *= 0x7FEB352Du; x ^= x >> 15; x *= 0x846CA68Bu; x ^= x >> 16;
  return x;
}

template <bool PAIR, bool WITH_CP, bool CP_WARP = false, bool BATCH = false>
__device__ void peak_body(int iters, uint32_t* status, uint8_t* base) {
  uint8_t* sA = base;
  uint8_t* sB = base + A_BYTES;
  uint8_t* sSF = base + A_BYTES + B_BYTES;
  uint64_t* bar = reinterpret_cast<uint64_t*>(sSF + SF_BYTES);   // [0] MMAs, [1] copier
  uint32_t* holder = reinterpret_cast<uint32_t*>(bar + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(holder + 1);
  const int t = threadIdx.x;
  // random E2M1 codes (no NaN in FP4), unit E4M3 scales (0x38 = 1.0)
  for (int i = t; i < (A_BYTES + B_BYTES) / 4; i += blockDim.x)
    reinterpret_cast<uint32_t*>(sA)[i] = hash32(i * 2654435761u + blockIdx.x);
  for (int i = t; i < SF_BYTES; i += blockDim.x) sSF[i] = 0x38;
  if (t == 0) {
    mbar_init(smem_u32(bar), 1);
    mbar_init(smem_u32(bar + 1), 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  if (t < 32) {
    if (PAIR) tmem_alloc_pair(smem_u32(holder), 512);
    else tmem_alloc(smem_u32(holder), 512);
  }
  tc_fence_before();
  __syncthreads();
  if (PAIR) cluster_sync();
  tc_fence_after();
  const uint32_t tmem = *holder;
  const bool issuer = PAIR ? (cluster_ctarank() == 0 && t == 0) : (t == 0);
  const bool copier = CP_WARP && (PAIR ? (cluster_ctarank() == 0 && t == 32) : (t == 32));
  if (copier) {
    // the copies of variant 1 / 3, from another warp, into columns 448+
    const uint64_t sf0 = smem_desc(smem_u32(sSF), 0, 128, 0);
    const uint64_t sf1 = smem_desc(smem_u32(sSF + 512), 0, 128, 0);
    const uint64_t sf2 = smem_desc(smem_u32(sSF + 1024), 0, 128, 0);
    const uint32_t t_cp = tmem + 448;
    for (int i = 0; i < iters; ++i) {
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        if (PAIR) {
          tc_cp_pair_32x128b(t_cp, sf0); tc_cp_pair_32x128b(t_cp + 4, sf1); tc_cp_pair_32x128b(t_cp + 8, sf2);
        } else {
          tc_cp_32x128b(t_cp, sf0); tc_cp_32x128b(t_cp + 4, sf1); tc_cp_32x128b(t_cp + 8, sf2);
        }
      }
    }
    if (PAIR) tc_commit_pair(smem_u32(bar + 1), 0x1);
    else tc_commit(smem_u32(bar + 1));
    mbar_wait(smem_u32(bar + 1), 0, abort_flag, status, 0x2001);
  }
  if (issuer) {
    const uint32_t t_sfa = tmem + 256, t_sfb = tmem + 260;
    const uint64_t sf0 = smem_desc(smem_u32(sSF), 0, 128, 0);
    const uint64_t sf1 = smem_desc(smem_u32(sSF + 512), 0, 128, 0);
    const uint64_t sf2 = smem_desc(smem_u32(sSF + 1024), 0, 128, 0);
    auto cp_all = [&]() {
      if (PAIR) {
        tc_cp_pair_32x128b(t_sfa, sf0); tc_cp_pair_32x128b(t_sfb, sf1); tc_cp_pair_32x128b(t_sfb + 4, sf2);
      } else {
        tc_cp_32x128b(t_sfa, sf0); tc_cp_32x128b(t_sfb, sf1); tc_cp_32x128b(t_sfb + 4, sf2);
      }
    };
    cp_all();
    const uint32_t idesc = make_idesc(256, PAIR ? 256 : 128, 0u, 0u, 0u);
    const uint32_t a_base = smem_u32(sA), b_base = smem_u32(sB);
    for (int i = 0; i < iters; ++i) {
      // BATCH: this K step's slot (columns 256..495)
      const uint32_t ks = tmem + 256 + 48 * (uint32_t)(i % 5);
      if (BATCH) {
#pragma unroll
        for (int a = 0; a < 4; ++a) {
          if (PAIR) tc_cp_pair_32x128b(ks + 4 * a, sf0);
          else tc_cp_32x128b(ks + 4 * a, sf0);
        }
#pragma unroll
        for (int a = 0; a < 8; ++a) {
          if (PAIR) tc_cp_pair_32x128b(ks + 16 + 4 * a, sf1);
          else tc_cp_32x128b(ks + 16 + 4 * a, sf1);
        }
      }
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        if (WITH_CP) cp_all();
        const uint64_t ad = smem_desc(a_base + kk * 32, 16, 1024, 2);
        const uint64_t bd = smem_desc(b_base + kk * 32, 16, 1024, 2);
        const uint32_t sfa = BATCH ? ks + 4 * kk : t_sfa;
        const uint32_t sfb = BATCH ? ks + 16 + 8 * kk : t_sfb;
        if (PAIR) tc_mma_pair<true>(tmem, ad, bd, idesc, sfa, sfb, 1u);
        else tc_mma<true>(tmem, ad, bd, idesc, sfa, sfb, 1u);
      }
    }
    if (PAIR) tc_commit_pair(smem_u32(bar), 0x1);
    else tc_commit(smem_u32(bar));
    mbar_wait(smem_u32(bar), 0, abort_flag, status, 0x2000);
  }
  tc_fence_before();
  __syncthreads();
  if (PAIR) cluster_sync();
  if (t < 32) {
    tc_fence_after();
    if (PAIR) tmem_dealloc_pair(tmem, 512);
    else tmem_dealloc(tmem, 512);
  }
}

template <bool WITH_CP, bool CP_WARP, bool BATCH = false>
__global__ void __launch_bounds__(128, 1) mma_peak_single(int iters, uint32_t* status) {
  extern __shared__ uint8_t sm[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(sm) + 1023) & ~uintptr_t(1023));
  peak_body<false, WITH_CP, CP_WARP, BATCH>(iters, status, base);
}

template <bool WITH_CP, bool CP_WARP, bool BATCH = false>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(128, 1)
mma_peak_pair(int iters, uint32_t* status) {
  extern __shared__ uint8_t sm[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(sm) + 1023) & ~uintptr_t(1023));
  peak_body<true, WITH_CP, CP_WARP, BATCH>(iters, status, base);
}

}  // namespace
}  // namespace fp4impl

using namespace fp4impl;

extern "C" fp4_status fp4_mma_rate(int32_t variant, int32_t iters, float* tflops_out,
                                   void* ws, size_t ws_bytes, void* stream) {
  if (tflops_out == nullptr || ws == nullptr) return FP4_ERR_NULL;
  if (ws_bytes < sizeof(DeviceStatus)) return FP4_ERR_WORKSPACE;
  if (variant < 0 || variant > 7 || iters <= 0) return FP4_ERR_SHAPE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int grid = (sm_count() / 2) * 2;
  uint32_t* status = static_cast<uint32_t*>(ws);
  cudaEvent_t e0, e1;
  if (cudaEventCreate(&e0) != cudaSuccess || cudaEventCreate(&e1) != cudaSuccess) return FP4_ERR_CUDA;
  auto launch = [&]() {
    switch (variant) {
#define FP4_PEAK_LAUNCH(KERN)                                                              \
  cudaFuncSetAttribute(KERN, cudaFuncAttributeMaxDynamicSharedMemorySize, PEAK_SMEM);     \
  KERN<<<grid, 128, PEAK_SMEM, s>>>(iters, status);
      case 0: FP4_PEAK_LAUNCH((mma_peak_single<false, false>)); break;
      case 1: FP4_PEAK_LAUNCH((mma_peak_single<true, false>)); break;
      case 2: FP4_PEAK_LAUNCH((mma_peak_pair<false, false>)); break;
      case 3: FP4_PEAK_LAUNCH((mma_peak_pair<true, false>)); break;
      case 4: FP4_PEAK_LAUNCH((mma_peak_single<false, true>)); break;
      case 5: FP4_PEAK_LAUNCH((mma_peak_pair<false, true>)); break;
      case 6: FP4_PEAK_LAUNCH((mma_peak_single<false, false, true>)); break;
      default: FP4_PEAK_LAUNCH((mma_peak_pair<false, false, true>)); break;
#undef FP4_PEAK_LAUNCH
    }
    count_launches(1);
  };
  launch();                                   // warm-up
  cudaEventRecord(e0, s);
  launch();
  cudaEventRecord(e1, s);
  fp4_status st = FP4_OK;
  if (cudaEventSynchronize(e1) != cudaSuccess || cudaGetLastError() != cudaSuccess) st = FP4_ERR_CUDA;
  float ms = 0.0f;
  cudaEventElapsedTime(&ms, e0, e1);
  cudaEventDestroy(e0);
  cudaEventDestroy(e1);
  // flops: each CTA (single) or CTA pair issues iters * 4 MMAs of
  // 128x256x64 (single) or 256x256x64 (pair)
  const bool pair = variant == 2 || variant == 3 || variant == 5 || variant == 7;
  const double per_mma = pair ? 2.0 * 256 * 256 * 64 : 2.0 * 128 * 256 * 64;
  const double issuers = pair ? grid / 2 : grid;
  *tflops_out = (float)(issuers * 4.0 * iters * per_mma / (ms * 1e-3) / 1e12);
  return st;
}
