// fa_internal.h - host-side declarations shared by the C-ABI front end and the
// kernel launchers.  Not part of the public interface.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstddef>
#include <cstdint>

#include "../../include/fa_b200.h"

namespace fa {

// Encodes a 3-D bf16 tensor map over a [outer, rows, d] array (d innermost)
// with a box of 64 x box_rows x 1 elements and 128-byte swizzle.  Rows beyond
// `rows` read as zero, so a tile never spills into the next (batch, head).
fa_status make_tmap_bf16_3d(CUtensorMap* map, const void* base, uint64_t d, uint64_t rows,
                            uint64_t outer, uint32_t box_rows);

// 3-D bf16 tensor map over a token-major [rows, heads, d] array (d
// innermost) with a box of 64 x 1 x box_rows and 128-byte swizzle; the
// coordinates are (column, head, row).  Rows beyond `rows` read as zero.
fa_status make_tmap_bf16_rows_heads(CUtensorMap* map, const void* base, uint64_t d,
                                    uint64_t heads, uint64_t rows, uint32_t box_rows);

// 3-D byte tensor map over an [outer, rows, inner] array (inner contiguous,
// inner a multiple of 16) with a box_inner x box_rows x 1 box, box_inner = 128
// (one 128-byte swizzle row); coordinates (column, row, outer).
fa_status make_tmap_u8_3d(CUtensorMap* map, const void* base, uint64_t inner, uint64_t rows,
                          uint64_t outer, uint32_t box_inner, uint32_t box_rows);

// 2-D float32 tensor map over a [outer, n] array with a 128 x 1 box and no
// swizzle; n * 4 must be a multiple of 16 bytes.
fa_status make_tmap_f32_2d(CUtensorMap* map, const void* base, uint64_t n, uint64_t outer);

// 3-D float32 tensor map over a [outer, rows, d] array with a 32 x 128 x 1 box
// (128 bytes wide) and 128-byte swizzle, for bulk reductions of 128-row tiles.
fa_status make_tmap_f32_3d_sw128(CUtensorMap* map, const void* base, uint64_t d, uint64_t rows,
                                 uint64_t outer);

// 3-D float32 tensor map over a token-major [rows, heads, d] array with a
// 32 x 1 x 128 box (128 bytes wide) and 128-byte swizzle, for bulk
// reductions of 128-row tiles; coordinates (column, head, row).
fa_status make_tmap_f32_rows_heads_sw128(CUtensorMap* map, const void* base, uint64_t d,
                                         uint64_t heads, uint64_t rows);

// Row stride (elements) of the per-row float32 tables of the backward
// workspace: N rounded up to whole 128-row tiles.
inline size_t bwd_row_pad(int N) { return (static_cast<size_t>(N) + 127) / 128 * 128; }

// Hkv = number of key/value heads; H (query heads) is a multiple of it.
// Nq query rows, Nk key rows per head; causal masking keeps j <= i + Nk - Nq.
fa_status launch_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                     int H, int Hkv, int Nq, int Nk, int d, int causal, float scale,
                     cudaStream_t stream);

// Ragged batch, token-major packing: q / o [total_q, H, d], k / v
// [total_k, Hkv, d], lse [H, total_q]; cu_q / cu_k int32 [B + 1] on the device.
fa_status launch_fwd_varlen(const void* q, const void* k, const void* v, void* o, float* lse,
                            const int* cu_q, const int* cu_k, int B, int H, int Hkv,
                            int total_q, int total_k, int max_seqlen_q, int d, int causal,
                            float scale, cudaStream_t stream);

// Ragged batch backward (layouts as launch_fwd_varlen; dq like q, dk / dv like
// k).  The workspace holds D and log2(e) * LSE as float32 [H, P] with
// P = bwd_varlen_table_rows(B, total_q), then the float32 dQ accumulator
// [total_q, H, d], each region 256-byte aligned.
size_t bwd_varlen_table_rows(int B, int total_q);
fa_status launch_bwd_varlen(const void* q, const void* k, const void* v, const void* o,
                            const void* dout, const float* lse, void* dq, void* dk, void* dv,
                            const int* cu_q, const int* cu_k, void* workspace, int B, int H,
                            int Hkv, int total_q, int total_k, int max_seqlen_k, int d,
                            int causal, float scale, cudaStream_t stream);

// e4m3 forward: q [B*H, Nq, 128], k [B*Hkv, Nk, 128], vt [B*Hkv, 128, Nk]
// (V transposed), real values = stored values x the per-tensor descales.
fa_status launch_fwd_fp8(const void* q, const void* k, const void* vt, void* o, float* lse,
                         float q_scale, float k_scale, float v_scale, int B, int H, int Hkv,
                         int Nq, int Nk, int causal, float scale, cudaStream_t stream);

fa_status launch_bwd(const void* q, const void* k, const void* v, const void* o,
                     const void* dout, const float* lse, void* dq, void* dk, void* dv,
                     void* workspace, int B, int H, int Hkv, int Nq, int Nk, int d, int causal,
                     float scale, cudaStream_t stream);

int decode_num_splits(int Lmax);
// page_table == nullptr: contiguous caches [B, Hkv, Lmax, d].  Otherwise paged
// pools [num_pages, Hkv, 1 << log2_page, d] addressed through
// page_table[B, pages_per_seq], with Lmax = pages_per_seq << log2_page.
fa_status launch_decode(const void* q, const void* kc, const void* vc, const int* seqlens,
                        void* o, float* lse, int B, int H, int Hkv, int Lmax, int d,
                        float scale, float* partials, cudaStream_t stream,
                        const int* page_table = nullptr, int pages_per_seq = 0,
                        int log2_page = 0, int num_pages = 0);

inline fa_status cuda_status(cudaError_t e) { return e == cudaSuccess ? FA_OK : FA_ERR_CUDA; }

// Caller-owned events recorded on the launch stream just before and just
// after the dominant kernel of every call (fa_set_timing_events); null when
// unset.
struct MainKernelEvents {
  cudaEvent_t start;
  cudaEvent_t stop;
};
extern MainKernelEvents g_main_events;
inline void main_kernel_begin(cudaStream_t s) {
  if (g_main_events.start != nullptr) cudaEventRecord(g_main_events.start, s);
}
inline void main_kernel_end(cudaStream_t s) {
  if (g_main_events.stop != nullptr) cudaEventRecord(g_main_events.stop, s);
}

// Work-distribution overrides set by fa_set_schedule (FA_SCHEDULE_*).
extern std::atomic<int> g_fwd_schedule;
extern std::atomic<int> g_bwd_order;

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Dynamic shared memory above 48 KB must be enabled per kernel function and
// per device (the attribute belongs to the function as loaded on each
// device).  One flag per device records that the current device has been
// configured; two threads racing here both set the same value, which is
// harmless.  Devices beyond the table are configured on every call.
struct SmemOptIn {
  static constexpr int kMaxDevices = 64;
  std::atomic<bool> done[kMaxDevices] = {};
  template <typename Kern>
  fa_status ensure(Kern kern, int bytes) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return FA_ERR_CUDA;
    const bool cached = dev >= 0 && dev < kMaxDevices;
    if (cached && done[dev].load(std::memory_order_acquire)) return FA_OK;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) !=
        cudaSuccess)
      return FA_ERR_CUDA;
    if (cached) done[dev].store(true, std::memory_order_release);
    return FA_OK;
  }
};

}  // namespace fa
