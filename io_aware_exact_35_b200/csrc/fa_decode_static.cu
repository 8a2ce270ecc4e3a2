// fa_decode_static.cu - fa_decode_static: split-KV decode whose partial
// results live in a fixed, library-owned device array instead of a
// caller-provided workspace.
//
// Who needs it: callers that cannot call cudaMalloc.  Examples are plug-ins
// inside a host program that has already reserved (almost) all device memory
// for its own pool, so any allocation of theirs would fail or break the host's
// accounting, and latency-critical loops that must not run cudaMalloc because
// it can synchronise the whole device.  Such callers still pass their inputs
// and outputs; only the scratch for the per-chunk softmax partials comes from
// here.
//
// The scratch is one file-scope __device__ array of FA_DECODE_STATIC_SCRATCH_BYTES
// bytes.  Every device that loads this library holds it until the process
// exits.  In host code the array's name is only a host-side stand-in, so its
// device address is looked up with cudaGetSymbolAddress, once per device, with
// that device current, on the first call made on that device; make that first
// call before starting any stream capture.
//
// All calls share the one array and it keeps whatever the last call wrote.
// Nothing in it has to start at zero: a call reads only the partials that its
// own split kernel has just written.  Calls whose execution overlaps on the GPU
// (different streams, no ordering between them) race on the array and give
// undefined results; serialise them.
#include <mutex>

#include "fa_internal.h"

namespace fa {

namespace {

static __device__ __align__(256) float g_decode_static_scratch[FA_DECODE_STATIC_SCRATCH_BYTES /
                                                                sizeof(float)];

constexpr int kMaxStaticDevices = 64;
std::mutex g_static_mu;
float* g_static_ptr[kMaxStaticDevices] = {};

// Device address of the scratch array on the current device (set-up on first use).
fa_status static_scratch(float** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return FA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxStaticDevices) return FA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_static_mu);
  if (g_static_ptr[dev] == nullptr) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_decode_static_scratch);
    if (e != cudaSuccess || p == nullptr) return FA_ERR_CUDA;
    g_static_ptr[dev] = static_cast<float*>(p);
  }
  *out = g_static_ptr[dev];
  return FA_OK;
}

}  // namespace

}  // namespace fa

extern "C" fa_status fa_decode_static(const void* q, const void* kcache, const void* vcache,
                                      const int* seqlens, void* o, float* lse, int B, int H,
                                      int Lmax, int d, float scale, fa_stream_t stream) {
  using namespace fa;
  if (B < 1 || H < 1 || Lmax < 0) return FA_ERR_INVALID_ARG;
  if (static_cast<long long>(B) * H > 0x7fffffffLL) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  if (!q || !kcache || !vcache || !seqlens || !o) return FA_ERR_INVALID_ARG;
  const uintptr_t mis = reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(kcache) |
                        reinterpret_cast<uintptr_t>(vcache) | reinterpret_cast<uintptr_t>(o);
  if ((mis & 15u) || (reinterpret_cast<uintptr_t>(seqlens) & 3u) ||
      (lse != nullptr && (reinterpret_cast<uintptr_t>(lse) & 3u)))
    return FA_ERR_INVALID_ARG;
  if (!(scale == scale)) return FA_ERR_INVALID_ARG;
  // The partials must fit the fixed array.
  if (fa_decode_workspace_size(B, H, Lmax, d) > FA_DECODE_STATIC_SCRATCH_BYTES)
    return FA_ERR_WORKSPACE;
  int major = 0, dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
    return FA_ERR_CUDA;
  if (major != 10) return FA_ERR_UNSUPPORTED;
  float* scratch = nullptr;
  const fa_status st = static_scratch(&scratch);
  if (st != FA_OK) return st;
  return launch_decode(q, kcache, vcache, seqlens, o, lse, B, H, H, Lmax, d, scale, scratch,
                       reinterpret_cast<cudaStream_t>(stream));
}
