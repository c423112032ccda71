// noalloc.cu -- fp4_gemm for callers that cannot allocate device memory.
//
// fp4_gemm needs a caller-allocated workspace: the kernels use it as scratch
// for the device status block (bounded-wait timeouts and similar conditions
// found on the GPU are recorded there).  Some callers cannot call cudaMalloc
// at all -- code that runs while another component owns every allocation
// (a memory pool or arena handed out by a framework), a plugin loaded into a
// host process that forbids device allocation, or code on a path that must
// not synchronise, which cudaMalloc may do.  fp4_gemm_noalloc serves them: the
// scratch lives in a file-scope static device array that every GPU which loads
// this library holds until the process exits.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "fp4.h"
#include "internal.h"

namespace {

// Stated maximum of the library-held scratch: 4 KiB per device.
constexpr size_t kNoAllocScratchBytes = 4096;
static_assert(kNoAllocScratchBytes >= sizeof(fp4impl::DeviceStatus), "status block must fit");
static_assert(FP4_NOALLOC_SCRATCH_BYTES == kNoAllocScratchBytes, "header and library agree");

static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

struct DeviceScratch {
  std::once_flag once;
  void* ptr = nullptr;
  cudaError_t err = cudaSuccess;
};
constexpr int kMaxDevices = 64;
DeviceScratch g_scratch[kMaxDevices];

// Device address of the scratch array on the current device.  In host code
// the array's name is only a host-side stand-in, so the address comes from
// cudaGetSymbolAddress, once per device, with that device current.
fp4_status scratch_for_current_device(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return FP4_ERR_CUDA;
  DeviceScratch& d = g_scratch[dev];
  std::call_once(d.once, [&d] {
    d.err = cudaGetSymbolAddress(&d.ptr, g_noalloc_scratch);
  });
  if (d.err != cudaSuccess || d.ptr == nullptr) return FP4_ERR_CUDA;
  *out = d.ptr;
  return FP4_OK;
}

}  // namespace

extern "C" fp4_status fp4_gemm_noalloc(const fp4_qtensor* a, const fp4_qtensor* b, float alpha,
                                       void* c, int64_t ldc, int32_t out_dtype, float* c_amax,
                                       void* stream) {
  if (a == nullptr || b == nullptr) return FP4_ERR_NULL;
  // Reject problems whose scratch need exceeds the library-held array.
  if (fp4_workspace_bytes(a->rows, b->rows, a->cols) > kNoAllocScratchBytes)
    return FP4_ERR_WORKSPACE;
  void* scratch = nullptr;
  fp4_status st = scratch_for_current_device(&scratch);
  if (st != FP4_OK) return st;
  // Every argument error returns before the clear below is enqueued.
  st = fp4impl::gemm_validate(a, b, c, ldc, out_dtype, scratch, kNoAllocScratchBytes);
  if (st != FP4_OK) return st;
  // The array keeps the previous call's contents: the status block must start
  // at zero for this call's device conditions to be recorded.
  if (cudaMemsetAsync(scratch, 0, sizeof(fp4impl::DeviceStatus),
                      static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return FP4_ERR_CUDA;
  return fp4_gemm(a, b, alpha, c, ldc, out_dtype, c_amax, scratch, kNoAllocScratchBytes, stream);
}
