// dp.cu -- the data-parallel exchange of the linear layer's weight gradient.
//
// In data-parallel training every GPU quantizes its own token shard and runs
// fprop, dgrad and wgrad on it; the one exchange is the sum of the FP32 dW
// over the ranks ("FP4 All the Way", Summary: the 7B model was trained with
// FP4 on 256 accelerators, i.e. data-parallel; the pages give no scheme
// beyond that).  fp4_allreduce_sum_f32 enqueues that sum, in place, with
// NCCL on the caller's stream, so it runs after the wgrad GEMM queued before
// it and overlaps whatever the caller queues on other streams.
//
// The library does not link NCCL: the process's NCCL (the one the framework
// already loaded, found by its soname) is resolved on first use, so the
// library never brings a second copy into a process that has one.
#include <cuda_runtime.h>
#include <dlfcn.h>

#include <cstdint>
#include <mutex>

#include "fp4.h"

namespace {

// The few NCCL declarations used here (public ABI of nccl.h): result codes,
// the FP32 data type and the sum reduction.
typedef int nccl_result_t;                  // ncclResult_t, 0 = ncclSuccess
constexpr int kNcclFloat32 = 7;             // ncclFloat32
constexpr int kNcclSum = 0;                 // ncclSum
typedef nccl_result_t (*AllReduceFn)(const void*, void*, size_t, int, int, void*, cudaStream_t);

AllReduceFn resolve_allreduce() {
  static AllReduceFn fn = nullptr;
  static std::mutex mu;
  std::lock_guard<std::mutex> lock(mu);
  if (fn == nullptr) {
    void* h = dlopen("libnccl.so.2", RTLD_LAZY | RTLD_NOLOAD);   // already in the process?
    if (h == nullptr) h = dlopen("libnccl.so.2", RTLD_LAZY);
    if (h != nullptr) fn = reinterpret_cast<AllReduceFn>(dlsym(h, "ncclAllReduce"));
  }
  return fn;
}

}  // namespace

extern "C" fp4_status fp4_allreduce_sum_f32(void* nccl_comm, float* buf, int64_t count,
                                            void* stream) {
  if (nccl_comm == nullptr) return FP4_ERR_NULL;
  if (count < 0) return FP4_ERR_SHAPE;
  if (count == 0) return FP4_OK;
  if (buf == nullptr) return FP4_ERR_NULL;
  if ((reinterpret_cast<uintptr_t>(buf) & 3u) != 0) return FP4_ERR_ALIGN;
  AllReduceFn f = resolve_allreduce();
  if (f == nullptr) return FP4_ERR_UNSUPPORTED;
  return f(buf, buf, (size_t)count, kNcclFloat32, kNcclSum, nccl_comm,
           static_cast<cudaStream_t>(stream)) == 0
             ? FP4_OK
             : FP4_ERR_CUDA;
}
