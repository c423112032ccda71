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
#include <cstdlib>
#include <mutex>

#include "fp4.h"
#include "internal.h"

namespace {

// Stated maximum of the library-held scratch: 4 KiB per device.
constexpr size_t kNoAllocScratchBytes = 4096;
static_assert(kNoAllocScratchBytes >= sizeof(fp4impl::DeviceStatus), "status block must fit");
static_assert(FP4_NOALLOC_SCRATCH_BYTES == kNoAllocScratchBytes, "header and library agree");

static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_lookup_mutex;
void* g_scratch_ptr[kMaxDevices] = {};   // device address once a lookup succeeded

// Host-side fault injection for the failure path of the lookup: the first
// FP4_NOALLOC_FAIL_LOOKUPS lookups of the process report cudaErrorNotReady
// instead of calling cudaGetSymbolAddress (read once; unset means 0).
int injected_failures_left() {
  static int left = [] {
    const char* s = std::getenv("FP4_NOALLOC_FAIL_LOOKUPS");
    return s ? std::atoi(s) : 0;
  }();
  return left > 0 ? left-- : 0;
}

// Device address of the scratch array on the current device.  In host code
// the array's name is only a host-side stand-in, so the address comes from
// cudaGetSymbolAddress, with that device current.  Only a successful lookup
// is kept: a failed one (a call made during stream capture, a context not yet
// usable, an error left pending by unrelated work) is retried by the next call
// and its CUDA error is returned to this one as FP4_ERR_CUDA.
fp4_status scratch_for_current_device(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return FP4_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_lookup_mutex);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    const cudaError_t e = injected_failures_left() > 0
                              ? cudaErrorNotReady
                              : cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr) return FP4_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
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
