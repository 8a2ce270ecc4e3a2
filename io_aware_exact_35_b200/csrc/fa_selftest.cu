// fa_selftest.cu - fa_check_bounded_wait: exercises the library's failure
// detection without a GPU fault.  One CTA waits, with the same bounded waits
// the attention kernels use, on an mbarrier that nothing ever arrives on: the
// wait must give up after its limit (FA_WAIT_TIMEOUT_NS), record
// FA_ERR_TIMEOUT in the device error word, raise the CTA's abort flag and
// return, leaving the context usable.  No trap, no fault, no unbounded loop.
#include "fa_internal.h"
#include "sm100.cuh"

namespace fa {

namespace {

__global__ void __launch_bounds__(64) fa_bounded_wait_kernel(int* gave_up) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);  // one arrival expected; none will come
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  volatile int* flag = &abort_flag;
  if (threadIdx.x < 32) {
    // a single-thread wait (as the producer and MMA warps use) ...
    if (threadIdx.x == 0 && !mbar_wait(&bar, 0, flag)) atomicAdd(gave_up, 1);
  } else {
    // ... and a warp-collective one (as the softmax warpgroups use), which
    // also gives up once the abort flag is raised
    if (!mbar_wait_warp(&bar, 0, flag) && threadIdx.x == 32) atomicAdd(gave_up, 1);
  }
}

}  // namespace

}  // namespace fa

extern "C" fa_status fa_check_bounded_wait(int* gave_up, fa_stream_t stream) {
  using namespace fa;
  if (gave_up == nullptr || (reinterpret_cast<uintptr_t>(gave_up) & 3u)) return FA_ERR_INVALID_ARG;
  int major = 0, dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
    return FA_ERR_CUDA;
  if (major != 10) return FA_ERR_UNSUPPORTED;
  fa_bounded_wait_kernel<<<1, 64, 0, reinterpret_cast<cudaStream_t>(stream)>>>(gave_up);
  return cuda_status(cudaGetLastError());
}
