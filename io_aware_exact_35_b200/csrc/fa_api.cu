// fa_api.cu - the C ABI declared in include/fa_b200.h: argument validation,
// tensor-map encoding, workspace sizing and the device error word.
#include <climits>
#include <cstring>
#include <mutex>

#include <nvtx3/nvToolsExt.h>

#include "fa_internal.h"
#include "sm100.cuh"

namespace fa {

MainKernelEvents g_main_events = {nullptr, nullptr};
std::atomic<int> g_fwd_schedule{FA_SCHEDULE_AUTO};
std::atomic<int> g_bwd_order{FA_SCHEDULE_AUTO};

namespace {

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

constexpr int kMaxDevices = 64;

// NVTX range around one ABI call, so that a timeline (nsys, ncu's NVTX
// filter) shows which entry point launched which kernels.  Without a tool
// attached a push / pop is a call to an empty function.
struct Range {
  explicit Range(const char* name) { nvtxRangePushA(name); }
  ~Range() { nvtxRangePop(); }
  Range(const Range&) = delete;
  Range& operator=(const Range&) = delete;
};

// 1 = sm_100 family, 0 = other, -1 = unknown (query failed).
fa_status check_device() {
  static int cache[kMaxDevices];
  static std::once_flag once;
  std::call_once(once, [] {
    for (int i = 0; i < kMaxDevices; ++i) cache[i] = -2;
  });
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return FA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return FA_ERR_UNSUPPORTED;
  if (cache[dev] == -2) {
    int major = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
      return FA_ERR_CUDA;
    cache[dev] = (major == 10) ? 1 : 0;
  }
  return cache[dev] == 1 ? FA_OK : FA_ERR_UNSUPPORTED;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned256(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 255u) == 0; }

fa_status check_shape(int B, int H, int N, int d) {
  if (B < 1 || H < 1 || N < 0) return FA_ERR_INVALID_ARG;
  if (static_cast<long long>(B) * H > INT_MAX) return FA_ERR_INVALID_ARG;
  if ((static_cast<long long>(N) + 127) / 128 * B * H > 0x7fffffffLL) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  return FA_OK;
}

}  // namespace

fa_status make_tmap_bf16_3d(CUtensorMap* map, const void* base, uint64_t d, uint64_t rows,
                            uint64_t outer, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return FA_ERR_CUDA;
  const cuuint64_t dims[3] = {d, rows, outer};
  const cuuint64_t strides[2] = {d * 2, rows * d * 2};  // bytes, dims 1 and 2
  const cuuint32_t box[3] = {64u, box_rows, 1u};
  const cuuint32_t estr[3] = {1u, 1u, 1u};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims,
                  strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? FA_OK : FA_ERR_CUDA;
}

fa_status make_tmap_bf16_rows_heads(CUtensorMap* map, const void* base, uint64_t d,
                                    uint64_t heads, uint64_t rows, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return FA_ERR_CUDA;
  const cuuint64_t dims[3] = {d, heads, rows};
  const cuuint64_t strides[2] = {d * 2, heads * d * 2};  // bytes, dims 1 and 2
  const cuuint32_t box[3] = {64u, 1u, box_rows};
  const cuuint32_t estr[3] = {1u, 1u, 1u};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims,
                  strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? FA_OK : FA_ERR_CUDA;
}

fa_status make_tmap_f32_rows_heads_sw128(CUtensorMap* map, const void* base, uint64_t d,
                                         uint64_t heads, uint64_t rows) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return FA_ERR_CUDA;
  const cuuint64_t dims[3] = {d, heads, rows};
  const cuuint64_t strides[2] = {d * 4, heads * d * 4};
  const cuuint32_t box[3] = {32u, 1u, 128u};
  const cuuint32_t estr[3] = {1u, 1u, 1u};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? FA_OK : FA_ERR_CUDA;
}

fa_status make_tmap_u8_3d(CUtensorMap* map, const void* base, uint64_t inner, uint64_t rows,
                          uint64_t outer, uint32_t box_inner, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return FA_ERR_CUDA;
  const cuuint64_t dims[3] = {inner, rows, outer};
  const cuuint64_t strides[2] = {inner, rows * inner};  // bytes, dims 1 and 2
  const cuuint32_t box[3] = {box_inner, box_rows, 1u};
  const cuuint32_t estr[3] = {1u, 1u, 1u};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? FA_OK : FA_ERR_CUDA;
}

fa_status make_tmap_f32_2d(CUtensorMap* map, const void* base, uint64_t n, uint64_t outer) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return FA_ERR_CUDA;
  const cuuint64_t dims[2] = {n, outer};
  const cuuint64_t strides[1] = {n * 4};
  const cuuint32_t box[2] = {128u, 1u};
  const cuuint32_t estr[2] = {1u, 1u};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? FA_OK : FA_ERR_CUDA;
}

fa_status make_tmap_f32_3d_sw128(CUtensorMap* map, const void* base, uint64_t d, uint64_t rows,
                                 uint64_t outer) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return FA_ERR_CUDA;
  const cuuint64_t dims[3] = {d, rows, outer};
  const cuuint64_t strides[2] = {d * 4, rows * d * 4};
  const cuuint32_t box[3] = {32u, 128u, 1u};
  const cuuint32_t estr[3] = {1u, 1u, 1u};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? FA_OK : FA_ERR_CUDA;
}

}  // namespace fa

using namespace fa;

extern "C" {

const char* fa_status_string(fa_status s) {
  switch (s) {
    case FA_OK: return "ok";
    case FA_ERR_INVALID_ARG: return "invalid argument";
    case FA_ERR_UNSUPPORTED: return "unsupported head dimension or device";
    case FA_ERR_WORKSPACE: return "workspace missing or too small";
    case FA_ERR_CUDA: return "CUDA error";
    case FA_ERR_TIMEOUT: return "a kernel's bounded wait expired";
    case FA_ERR_BOUNDS: return "a bounds check of the debug build failed";
  }
  return "unknown status";
}

int fa_version(void) { return 100; }

fa_status fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
                 int N, int d, int causal, float scale, fa_stream_t stream) {
  return fa_fwd_gqa(q, k, v, o, lse, B, H, H, N, d, causal, scale, stream);
}

fa_status fa_fwd_gqa(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                     int H, int Hkv, int N, int d, int causal, float scale, fa_stream_t stream) {
  return fa_fwd_ext(q, k, v, o, lse, B, H, Hkv, N, N, d, causal, scale, stream);
}

fa_status fa_fwd_ext(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                     int H, int Hkv, int Nq, int Nk, int d, int causal, float scale,
                     fa_stream_t stream) {
  Range nvtx_range("fa_fwd_ext");
  fa_status st = check_shape(B, H, Nq, d);
  if (st != FA_OK) return st;
  if ((st = check_shape(B, Hkv, Nk, d)) != FA_OK) return st;
  if (static_cast<long long>(Nq) + Nk > INT_MAX) return FA_ERR_INVALID_ARG;
  if (Hkv < 1 || H % Hkv != 0) return FA_ERR_INVALID_ARG;
  // arrays of zero size may be null
  if (Nq > 0 && (!q || !o || (Nk > 0 && (!k || !v)))) return FA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return FA_ERR_INVALID_ARG;
  if (lse != nullptr && (reinterpret_cast<uintptr_t>(lse) & 3u)) return FA_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return FA_ERR_INVALID_ARG;
  if (!(scale == scale)) return FA_ERR_INVALID_ARG;  // NaN
  if ((st = check_device()) != FA_OK) return st;
  if (Nq == 0) return FA_OK;
  return launch_fwd(q, k, v, o, lse, B, H, Hkv, Nq, Nk, d, causal, scale,
                    reinterpret_cast<cudaStream_t>(stream));
}

fa_status fa_fwd_varlen(const void* q, const void* k, const void* v, void* o, float* lse,
                        const int* cu_seqlens_q, const int* cu_seqlens_k, int B, int H, int Hkv,
                        int total_q, int total_k, int max_seqlen_q, int d, int causal,
                        float scale, fa_stream_t stream) {
  Range nvtx_range("fa_fwd_varlen");
  if (B < 1 || H < 1 || Hkv < 1 || H % Hkv != 0) return FA_ERR_INVALID_ARG;
  if (total_q < 0 || total_k < 0 || max_seqlen_q < 0) return FA_ERR_INVALID_ARG;
  if (static_cast<long long>(B) * H > INT_MAX) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  if (!cu_seqlens_q || !cu_seqlens_k) return FA_ERR_INVALID_ARG;
  if (total_q > 0 && (!q || !o)) return FA_ERR_INVALID_ARG;
  if (total_k > 0 && (!k || !v)) return FA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) ||
      (reinterpret_cast<uintptr_t>(cu_seqlens_q) & 3u) ||
      (reinterpret_cast<uintptr_t>(cu_seqlens_k) & 3u) ||
      (lse != nullptr && (reinterpret_cast<uintptr_t>(lse) & 3u)))
    return FA_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return FA_ERR_INVALID_ARG;
  if (!(scale == scale)) return FA_ERR_INVALID_ARG;
  fa_status st = check_device();
  if (st != FA_OK) return st;
  return launch_fwd_varlen(q, k, v, o, lse, cu_seqlens_q, cu_seqlens_k, B, H, Hkv, total_q,
                           total_k, max_seqlen_q, d, causal, scale,
                           reinterpret_cast<cudaStream_t>(stream));
}

fa_status fa_fwd_fp8(const void* q, const void* k, const void* vt, void* o, float* lse,
                     float q_scale, float k_scale, float v_scale, int B, int H, int Hkv, int Nq,
                     int Nk, int d, int causal, float scale, fa_stream_t stream) {
  Range nvtx_range("fa_fwd_fp8");
  fa_status st = check_shape(B, H, Nq, d);
  if (st != FA_OK) return st;
  if ((st = check_shape(B, Hkv, Nk, d)) != FA_OK) return st;
  if (d != 128) return FA_ERR_UNSUPPORTED;
  if (Nk % 16 != 0) return FA_ERR_UNSUPPORTED;  // rows of vt must be 16-byte multiples
  if (static_cast<long long>(Nq) + Nk > INT_MAX) return FA_ERR_INVALID_ARG;
  if (Hkv < 1 || H % Hkv != 0) return FA_ERR_INVALID_ARG;
  if (Nq > 0 && (!q || !o || (Nk > 0 && (!k || !vt)))) return FA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(vt) || !aligned16(o)) return FA_ERR_INVALID_ARG;
  if (lse != nullptr && (reinterpret_cast<uintptr_t>(lse) & 3u)) return FA_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return FA_ERR_INVALID_ARG;
  if (!(scale == scale) || !(q_scale == q_scale) || !(k_scale == k_scale) ||
      !(v_scale == v_scale))
    return FA_ERR_INVALID_ARG;
  if ((st = check_device()) != FA_OK) return st;
  if (Nq == 0) return FA_OK;
  return launch_fwd_fp8(q, k, vt, o, lse, q_scale, k_scale, v_scale, B, H, Hkv, Nq, Nk, causal,
                        scale, reinterpret_cast<cudaStream_t>(stream));
}

size_t fa_bwd_workspace_size(int B, int H, int N, int d) {
  if (check_shape(B, H, N, d) != FA_OK) return 0;
  const size_t bh = static_cast<size_t>(B) * H;
  const size_t padded = bh * bwd_row_pad(N);
  // D and log2(e) * LSE on 128-padded rows, the fp32 dQ accumulator, then
  // one completion counter per (batch, head)
  return 2 * align_up(padded * sizeof(float), 256) +
         align_up(bh * static_cast<size_t>(N) * d * sizeof(float), 256) +
         align_up(bh * sizeof(unsigned), 256);
}

fa_status fa_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout,
                 const float* lse, void* dq, void* dk, void* dv, void* workspace,
                 size_t ws_bytes, int B, int H, int N, int d, int causal, float scale,
                 fa_stream_t stream) {
  return fa_bwd_gqa(q, k, v, o, dout, lse, dq, dk, dv, workspace, ws_bytes, B, H, H, N, d, causal,
                    scale, stream);
}

fa_status fa_bwd_gqa(const void* q, const void* k, const void* v, const void* o,
                     const void* dout, const float* lse, void* dq, void* dk, void* dv,
                     void* workspace, size_t ws_bytes, int B, int H, int Hkv, int N, int d,
                     int causal, float scale, fa_stream_t stream) {
  return fa_bwd_ext(q, k, v, o, dout, lse, dq, dk, dv, workspace, ws_bytes, B, H, Hkv, N, N, d,
                    causal, scale, stream);
}

fa_status fa_bwd_ext(const void* q, const void* k, const void* v, const void* o,
                     const void* dout, const float* lse, void* dq, void* dk, void* dv,
                     void* workspace, size_t ws_bytes, int B, int H, int Hkv, int Nq, int Nk,
                     int d, int causal, float scale, fa_stream_t stream) {
  Range nvtx_range("fa_bwd_ext");
  fa_status st = check_shape(B, H, Nq, d);
  if (st != FA_OK) return st;
  if ((st = check_shape(B, Hkv, Nk, d)) != FA_OK) return st;
  if (static_cast<long long>(Nq) + Nk > INT_MAX) return FA_ERR_INVALID_ARG;
  if (Hkv < 1 || H % Hkv != 0) return FA_ERR_INVALID_ARG;
  // arrays of zero size may be null
  if (Nq > 0 && (!q || !o || !dout || !lse || !dq)) return FA_ERR_INVALID_ARG;
  if (Nk > 0 && (!dk || !dv || (Nq > 0 && (!k || !v)))) return FA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(dout) ||
      !aligned16(dq) || !aligned16(dk) || !aligned16(dv) ||
      (reinterpret_cast<uintptr_t>(lse) & 3u))
    return FA_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return FA_ERR_INVALID_ARG;
  if (!(scale == scale)) return FA_ERR_INVALID_ARG;
  const size_t need = fa_bwd_workspace_size(B, H, Nq, d);
  if (Nq > 0 && Nk > 0 && (workspace == nullptr || ws_bytes < need || !aligned256(workspace)))
    return FA_ERR_WORKSPACE;
  if ((st = check_device()) != FA_OK) return st;
  if (Nq == 0 && Nk == 0) return FA_OK;
  return launch_bwd(q, k, v, o, dout, lse, dq, dk, dv, workspace, B, H, Hkv, Nq, Nk, d, causal,
                    scale, reinterpret_cast<cudaStream_t>(stream));
}

size_t fa_bwd_varlen_workspace_size(int B, int H, int total_q, int d) {
  if (B < 1 || H < 1 || total_q < 0 || (d != 64 && d != 128)) return 0;
  if (static_cast<long long>(B) * H > INT_MAX) return 0;
  const size_t P = bwd_varlen_table_rows(B, total_q);
  return 2 * align_up(static_cast<size_t>(H) * P * sizeof(float), 256) +
         align_up(static_cast<size_t>(total_q) * H * d * sizeof(float), 256);
}

fa_status fa_bwd_varlen(const void* q, const void* k, const void* v, const void* o,
                        const void* dout, const float* lse, void* dq, void* dk, void* dv,
                        const int* cu_seqlens_q, const int* cu_seqlens_k, void* workspace,
                        size_t ws_bytes, int B, int H, int Hkv, int total_q, int total_k,
                        int max_seqlen_k, int d, int causal, float scale, fa_stream_t stream) {
  Range nvtx_range("fa_bwd_varlen");
  if (B < 1 || H < 1 || Hkv < 1 || H % Hkv != 0) return FA_ERR_INVALID_ARG;
  if (total_q < 0 || total_k < 0 || max_seqlen_k < 0) return FA_ERR_INVALID_ARG;
  if (static_cast<long long>(B) * H > INT_MAX) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  if (!cu_seqlens_q || !cu_seqlens_k) return FA_ERR_INVALID_ARG;
  if (total_q > 0 && (!q || !o || !dout || !lse || !dq)) return FA_ERR_INVALID_ARG;
  if (total_k > 0 && (!k || !v || !dk || !dv)) return FA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(dout) ||
      !aligned16(dq) || !aligned16(dk) || !aligned16(dv) ||
      (reinterpret_cast<uintptr_t>(lse) & 3u) ||
      (reinterpret_cast<uintptr_t>(cu_seqlens_q) & 3u) ||
      (reinterpret_cast<uintptr_t>(cu_seqlens_k) & 3u))
    return FA_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return FA_ERR_INVALID_ARG;
  if (!(scale == scale)) return FA_ERR_INVALID_ARG;
  const size_t need = fa_bwd_varlen_workspace_size(B, H, total_q, d);
  if (total_q > 0 && total_k > 0 &&
      (workspace == nullptr || ws_bytes < need || !aligned256(workspace)))
    return FA_ERR_WORKSPACE;
  fa_status st = check_device();
  if (st != FA_OK) return st;
  return launch_bwd_varlen(q, k, v, o, dout, lse, dq, dk, dv, cu_seqlens_q, cu_seqlens_k,
                           workspace, B, H, Hkv, total_q, total_k, max_seqlen_k, d, causal, scale,
                           reinterpret_cast<cudaStream_t>(stream));
}

size_t fa_decode_workspace_size(int B, int H, int Lmax, int d) {
  if (B < 1 || H < 1 || Lmax < 0 || (d != 64 && d != 128)) return 0;
  if (static_cast<long long>(B) * H > INT_MAX) return 0;
  const size_t splits = static_cast<size_t>(decode_num_splits(Lmax));
  return align_up(static_cast<size_t>(B) * H * splits * (d + 2) * sizeof(float), 256);
}

fa_status fa_decode(const void* q, const void* kcache, const void* vcache, const int* seqlens,
                    void* o, float* lse, int B, int H, int Lmax, int d, float scale,
                    void* workspace, size_t ws_bytes, fa_stream_t stream) {
  return fa_decode_gqa(q, kcache, vcache, seqlens, o, lse, B, H, H, Lmax, d, scale, workspace,
                       ws_bytes, stream);
}

fa_status fa_decode_gqa(const void* q, const void* kcache, const void* vcache, const int* seqlens,
                        void* o, float* lse, int B, int H, int Hkv, int Lmax, int d, float scale,
                        void* workspace, size_t ws_bytes, fa_stream_t stream) {
  Range nvtx_range("fa_decode_gqa");
  if (B < 1 || H < 1 || Lmax < 0) return FA_ERR_INVALID_ARG;
  if (Hkv < 1 || H % Hkv != 0) return FA_ERR_INVALID_ARG;
  if (static_cast<long long>(B) * H > INT_MAX) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  if (!q || !kcache || !vcache || !seqlens || !o) return FA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(kcache) || !aligned16(vcache) || !aligned16(o) ||
      (reinterpret_cast<uintptr_t>(seqlens) & 3u) ||
      (lse != nullptr && (reinterpret_cast<uintptr_t>(lse) & 3u)))
    return FA_ERR_INVALID_ARG;
  if (!(scale == scale)) return FA_ERR_INVALID_ARG;
  const size_t need = fa_decode_workspace_size(B, H, Lmax, d);
  if (need > 0 && (workspace == nullptr || ws_bytes < need || !aligned256(workspace)))
    return FA_ERR_WORKSPACE;
  fa_status st = check_device();
  if (st != FA_OK) return st;
  return launch_decode(q, kcache, vcache, seqlens, o, lse, B, H, Hkv, Lmax, d, scale,
                       static_cast<float*>(workspace), reinterpret_cast<cudaStream_t>(stream));
}

fa_status fa_decode_paged(const void* q, const void* kpages, const void* vpages,
                          const int* block_table, const int* seqlens, void* o, float* lse, int B,
                          int H, int Hkv, int page_size, int pages_per_seq, int num_pages, int d,
                          float scale, void* workspace, size_t ws_bytes, fa_stream_t stream) {
  Range nvtx_range("fa_decode_paged");
  if (B < 1 || H < 1 || pages_per_seq < 0 || num_pages < 0) return FA_ERR_INVALID_ARG;
  if (Hkv < 1 || H % Hkv != 0) return FA_ERR_INVALID_ARG;
  if (static_cast<long long>(B) * H > INT_MAX) return FA_ERR_INVALID_ARG;
  // rows per page: a power of two from 1 to 65536
  if (page_size < 1 || page_size > 65536 || (page_size & (page_size - 1)) != 0)
    return FA_ERR_INVALID_ARG;
  const long long lmax = static_cast<long long>(page_size) * pages_per_seq;
  if (lmax > INT_MAX) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  if (!q || !seqlens || !o || (pages_per_seq > 0 && !block_table) ||
      (num_pages > 0 && (!kpages || !vpages)))
    return FA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(kpages) || !aligned16(vpages) || !aligned16(o) ||
      (reinterpret_cast<uintptr_t>(seqlens) & 3u) ||
      (reinterpret_cast<uintptr_t>(block_table) & 3u) ||
      (lse != nullptr && (reinterpret_cast<uintptr_t>(lse) & 3u)))
    return FA_ERR_INVALID_ARG;
  if (!(scale == scale)) return FA_ERR_INVALID_ARG;
  const int Lmax = static_cast<int>(lmax);
  const size_t need = fa_decode_workspace_size(B, H, Lmax, d);
  if (need > 0 && (workspace == nullptr || ws_bytes < need || !aligned256(workspace)))
    return FA_ERR_WORKSPACE;
  fa_status st = check_device();
  if (st != FA_OK) return st;
  int log2_page = 0;
  while ((1 << log2_page) < page_size) ++log2_page;
  // a table of no pages (or a pool of none) leaves every sequence empty
  const int* table = (pages_per_seq > 0 && num_pages > 0) ? block_table : nullptr;
  if (table == nullptr) {
    // O = 0, LSE = -inf for every (b, h): the combine kernel alone with
    // zero splits does exactly that (no partial is read)
    return launch_decode(q, kpages, vpages, seqlens, o, lse, B, H, Hkv, 0, d, scale,
                         static_cast<float*>(workspace), reinterpret_cast<cudaStream_t>(stream));
  }
  return launch_decode(q, kpages, vpages, seqlens, o, lse, B, H, Hkv, Lmax, d, scale,
                       static_cast<float*>(workspace), reinterpret_cast<cudaStream_t>(stream),
                       table, pages_per_seq, log2_page, num_pages);
}

fa_status fa_set_timing_events(fa_event_t start, fa_event_t stop) {
  fa::g_main_events.start = reinterpret_cast<cudaEvent_t>(start);
  fa::g_main_events.stop = reinterpret_cast<cudaEvent_t>(stop);
  return FA_OK;
}

fa_status fa_set_schedule(int fwd_schedule, int bwd_order) {
  auto valid = [](int v) {
    return v == FA_SCHEDULE_AUTO || v == FA_SCHEDULE_GRID || v == FA_SCHEDULE_PERSISTENT;
  };
  if (!valid(fwd_schedule) || !valid(bwd_order)) return FA_ERR_INVALID_ARG;
  fa::g_fwd_schedule.store(fwd_schedule, std::memory_order_relaxed);
  fa::g_bwd_order.store(bwd_order, std::memory_order_relaxed);
  return FA_OK;
}

fa_status fa_get_device_error(fa_stream_t stream) {
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return FA_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, fa::g_device_error, sizeof(int)) != cudaSuccess)
    return FA_ERR_CUDA;
  if (v != 0) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(fa::g_device_error, &zero, sizeof(int)) != cudaSuccess)
      return FA_ERR_CUDA;
  }
  return v == 0 ? FA_OK : static_cast<fa_status>(v);
}

}  // extern "C"
