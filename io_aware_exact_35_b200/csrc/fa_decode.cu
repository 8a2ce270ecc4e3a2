// fa_decode.cu - KV-cache decode: one query per (batch, head) against the
// cached prefix 0 .. L_b-1 ("DL101 chapter 9" (handsonai.io), section 1.1
// Key/Value Caching: the newest token attends K_{<=t}, V_{<=t}).
//
// Decode reads every cached key and value exactly once and does two FMAs per
// element, so it is bound by HBM bandwidth.  The cache is cut into chunks of
// CHUNK keys; one CTA streams one chunk of one (batch, head) with 16-byte
// loads and keeps the online-softmax state of "Flash Attention: principle &
// practice" (holysheep.ai), section 2.1 (running max m, running sum l, here
// with an unnormalised output vector).  A second kernel merges the per-chunk
// states with the same rescale-and-add rule:
//   M = max_s m_s,  w_s = 2^(m_s - M),  o = sum w_s acc_s / sum w_s l_s,
//   lse = (M + log2 sum w_s l_s) * ln 2      (m in log2 units).
//
// Layout inside a CTA (4 warps): D/8 lanes share one key (8 bf16 = 16 bytes
// each), so a warp covers 32/(D/8) consecutive keys per step and issues
// UNROLL steps of K and V loads before using any of them.
//
// The cache is either contiguous, [B, Hkv, Lmax, d], or paged: pools of
// [num_pages, Hkv, page, d] with page a power of two and a per-sequence page
// table (logical page p of sequence b lives in pool page table[b][p]).  A
// paged CTA first copies the table entries of its chunk to shared memory;
// rows inside a page are contiguous, so the loads stay 16-byte vectors.  An
// entry outside [0, num_pages) is never dereferenced: its keys count as
// masked and FA_ERR_INVALID_ARG is recorded in the device error word.
#include "fa_internal.h"
#include "sm100.cuh"

namespace fa {

namespace dec {

constexpr int CHUNK = 512;   // keys per split
constexpr int WARPS = 4;
constexpr int THREADS = WARPS * 32;
constexpr int UNROLL = 8;

__device__ __forceinline__ uint4 ld_stream(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

// Page table of a paged cache; table == nullptr means a contiguous cache.
struct Pages {
  const int* table;   // [B, pages_per_seq] int32, device
  int pages_per_seq;
  int log2_page;      // rows per page = 1 << log2_page
  int num_pages;      // pool size, for bounds checks
};

// Row addressing of one (batch, key/value head) in either layout.
template <int D, bool PAGED>
struct KvRows {
  const __nv_bfloat16* k;  // contiguous: first row of this head; paged: pool + head offset
  const __nv_bfloat16* v;
  const int* pages;        // paged: shared-memory page entries of the chunk
  int p0;                  // paged: logical page of the chunk's first key
  int log2_page;
  size_t page_stride;      // paged: elements between consecutive pool pages
  // element offset of key `key`; -1 when its page entry is invalid
  __device__ __forceinline__ long long off(int key) const {
    if constexpr (!PAGED) {
      return static_cast<long long>(key) * D;
    } else {
      const int page = pages[(key >> log2_page) - p0];
      if (page < 0) return -1;
      return static_cast<long long>(page) * static_cast<long long>(page_stride) +
             static_cast<long long>(key & ((1 << log2_page) - 1)) * D;
    }
  }
};

// Sets up KvRows for keys c0 .. c1-1 of (b, hk); paged: fills `spages`
// (one entry per page of the chunk) and synchronises the CTA.
template <int D, bool PAGED>
__device__ __forceinline__ KvRows<D, PAGED> kv_rows(const __nv_bfloat16* kc,
                                                    const __nv_bfloat16* vc, const Pages& pg,
                                                    int* spages, int b, int hk, int Hkv, int Lmax,
                                                    int c0, int c1, int sub) {
  KvRows<D, PAGED> r;
  if constexpr (!PAGED) {
    const size_t head = (static_cast<size_t>(b) * Hkv + hk) * static_cast<size_t>(Lmax) * D;
    r.k = kc + head + sub * 8;
    r.v = vc + head + sub * 8;
    r.pages = nullptr;
    r.p0 = 0;
    r.log2_page = 0;
    r.page_stride = 0;
  } else {
    const size_t rows = static_cast<size_t>(1) << pg.log2_page;
    r.k = kc + static_cast<size_t>(hk) * rows * D + sub * 8;
    r.v = vc + static_cast<size_t>(hk) * rows * D + sub * 8;
    r.pages = spages;
    r.p0 = c0 >> pg.log2_page;
    r.log2_page = pg.log2_page;
    r.page_stride = static_cast<size_t>(Hkv) * rows * D;
    const int n = ((c1 - 1) >> pg.log2_page) - r.p0 + 1;
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
      int page = pg.table[static_cast<size_t>(b) * pg.pages_per_seq + r.p0 + i];
      if (page < 0 || page >= pg.num_pages) {
        record_error(1 /* FA_ERR_INVALID_ARG */);
        page = -1;
      }
      spages[i] = page;
    }
    __syncthreads();
  }
  return r;
}

__device__ __forceinline__ void bf16x8_to_f32(const uint4& u, float (&f)[8]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

template <int D, bool PAGED>
__global__ void __launch_bounds__(THREADS)
    fa_decode_split_kernel(const __nv_bfloat16* __restrict__ q,
                           const __nv_bfloat16* __restrict__ kc,
                           const __nv_bfloat16* __restrict__ vc, const int* __restrict__ seqlens,
                           float* __restrict__ part, int H, int group, int Lmax, int S,
                           float scale_log2, const Pages pg) {
  constexpr int LPK = D / 8;         // lanes per key
  constexpr int KPW = 32 / LPK;      // keys per warp step
  constexpr int HW = WARPS * KPW;    // key groups per CTA
  const int split = blockIdx.x;
  const int h = blockIdx.y;
  const int b = blockIdx.z;
  const int L = min(max(seqlens[b], 0), Lmax);
  const int c0 = split * CHUNK;
  if (c0 >= L) return;  // beyond this sequence's prefix
  const int c1 = min(c0 + CHUNK, L);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int sub = lane % LPK;        // which 8-element slice of d
  const int kin = lane / LPK;        // which key of the warp step
  const int grp = warp * KPW + kin;  // key group index within the CTA
  const size_t bh = static_cast<size_t>(b) * H + h;

  float qf[8];
  {
    const uint4 qu = *reinterpret_cast<const uint4*>(q + bh * D + sub * 8);
    bf16x8_to_f32(qu, qf);
#pragma unroll
    for (int e = 0; e < 8; ++e) qf[e] *= scale_log2;
  }
  // query head bh reads key/value head bh / group (grouped-query attention)
  const size_t bkv = bh / static_cast<size_t>(group);
  const __nv_bfloat16* kbase = kc + bkv * static_cast<size_t>(Lmax) * D + sub * 8;
  const __nv_bfloat16* vbase = vc + bkv * static_cast<size_t>(Lmax) * D + sub * 8;
  __shared__ int spages[PAGED ? CHUNK : 1];
  const auto rows = kv_rows<D, PAGED>(kc, vc, pg, spages, b, h / group, H / group, Lmax, c0,
                                      c1, sub);

  float m = -INFINITY, l = 0.f, acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.f;

  constexpr int KEYS_PER_ROUND = WARPS * UNROLL * KPW;
  for (int r0 = c0; r0 < c1; r0 += KEYS_PER_ROUND) {
    uint4 ku[UNROLL], vu[UNROLL];
    int key[UNROLL];
    bool live[UNROLL];  // paged: the key exists and its page entry is valid
#pragma unroll
    for (int u = 0; u < UNROLL; ++u) {
      key[u] = r0 + (warp * UNROLL + u) * KPW + kin;
      if constexpr (PAGED) {
        const long long off = key[u] < c1 ? rows.off(key[u]) : 0;
        live[u] = key[u] < c1 && off >= 0;
        if (live[u]) {
          ku[u] = ld_stream(rows.k + off);
          vu[u] = ld_stream(rows.v + off);
        } else {
          ku[u] = make_uint4(0, 0, 0, 0);
          vu[u] = make_uint4(0, 0, 0, 0);
        }
      } else {
        if (key[u] < c1) {
          ku[u] = ld_stream(kbase + static_cast<size_t>(key[u]) * D);
          vu[u] = ld_stream(vbase + static_cast<size_t>(key[u]) * D);
        } else {
          ku[u] = make_uint4(0, 0, 0, 0);
          vu[u] = make_uint4(0, 0, 0, 0);
        }
      }
    }
    float s[UNROLL];
#pragma unroll
    for (int u = 0; u < UNROLL; ++u) {
      float kf[8];
      bf16x8_to_f32(ku[u], kf);
      float t = 0.f;
#pragma unroll
      for (int e = 0; e < 8; ++e) t = fmaf(qf[e], kf[e], t);
#pragma unroll
      for (int off = LPK / 2; off > 0; off >>= 1) t += __shfl_xor_sync(0xffffffffu, t, off);
      bool keep;
      if constexpr (PAGED) keep = live[u];
      else keep = key[u] < c1;
      s[u] = keep ? t : -INFINITY;
    }
    float mg = m;
#pragma unroll
    for (int u = 0; u < UNROLL; ++u) mg = fmaxf(mg, s[u]);
    const float mref = (mg == -INFINITY) ? 0.f : mg;
    const float alpha = ex2_approx(m - mref);
    l *= alpha;
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] *= alpha;
#pragma unroll
    for (int u = 0; u < UNROLL; ++u) {
      const float pu = ex2_approx(s[u] - mref);
      l += pu;
      float vf[8];
      bf16x8_to_f32(vu[u], vf);
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[e] = fmaf(pu, vf[e], acc[e]);
    }
    m = mg;
  }

  // Merge the HW key groups of this CTA.
  __shared__ float red_m[HW], red_l[HW];
  __shared__ float red_o[HW][D];
#pragma unroll
  for (int e = 0; e < 8; ++e) red_o[grp][sub * 8 + e] = acc[e];
  if (sub == 0) {
    red_m[grp] = m;
    red_l[grp] = l;
  }
  __syncthreads();
  float* out = part + (bh * S + split) * (D + 2);
  for (int t = threadIdx.x; t < D; t += THREADS) {
    float M = -INFINITY;
#pragma unroll
    for (int g = 0; g < HW; ++g) M = fmaxf(M, red_m[g]);
    float o = 0.f, lt = 0.f;
#pragma unroll
    for (int g = 0; g < HW; ++g) {
      const float w = (red_m[g] == -INFINITY) ? 0.f : ex2_approx(red_m[g] - M);
      o = fmaf(w, red_o[g][t], o);
      lt = fmaf(w, red_l[g], lt);
    }
    out[t] = o;
    if (t == 0) {
      out[D] = M;
      out[D + 1] = lt;
    }
  }
}

// Grouped-query decode: one CTA streams one chunk of one key/value head and
// serves all G query heads that share it, so every cached row is read once.
// Each lane keeps the G query slices, and per head a running (m, l, acc).
template <int D, int G, bool PAGED>
__global__ void __launch_bounds__(THREADS)
    fa_decode_group_split_kernel(const __nv_bfloat16* __restrict__ q,
                                 const __nv_bfloat16* __restrict__ kc,
                                 const __nv_bfloat16* __restrict__ vc,
                                 const int* __restrict__ seqlens, float* __restrict__ part, int H,
                                 int Hkv, int Lmax, int S, float scale_log2, const Pages pg) {
  constexpr int LPK = D / 8;
  constexpr int KPW = 32 / LPK;
  constexpr int HW = WARPS * KPW;
  constexpr int UN = G <= 2 ? 8 : (G == 4 ? 4 : 2);  // keys in flight per lane (registers)
  const int split = blockIdx.x;
  const int hk = blockIdx.y;
  const int b = blockIdx.z;
  const int L = min(max(seqlens[b], 0), Lmax);
  const int c0 = split * CHUNK;
  if (c0 >= L) return;
  const int c1 = min(c0 + CHUNK, L);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int sub = lane % LPK;
  const int kin = lane / LPK;
  const int grp = warp * KPW + kin;
  const size_t bh0 = static_cast<size_t>(b) * H + static_cast<size_t>(hk) * G;  // first query head

  float qf[G][8];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    const uint4 qu = *reinterpret_cast<const uint4*>(q + (bh0 + g) * D + sub * 8);
    bf16x8_to_f32(qu, qf[g]);
#pragma unroll
    for (int e = 0; e < 8; ++e) qf[g][e] *= scale_log2;
  }
  const size_t bkv = static_cast<size_t>(b) * Hkv + hk;
  const __nv_bfloat16* kbase = kc + bkv * static_cast<size_t>(Lmax) * D + sub * 8;
  const __nv_bfloat16* vbase = vc + bkv * static_cast<size_t>(Lmax) * D + sub * 8;
  __shared__ int spages[PAGED ? CHUNK : 1];
  const auto rows = kv_rows<D, PAGED>(kc, vc, pg, spages, b, hk, Hkv, Lmax, c0, c1, sub);
  float m[G], l[G], acc[G][8];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    m[g] = -INFINITY;
    l[g] = 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[g][e] = 0.f;
  }
  constexpr int KEYS_PER_ROUND = WARPS * UN * KPW;
  for (int r0 = c0; r0 < c1; r0 += KEYS_PER_ROUND) {
    uint4 ku[UN], vu[UN];
    int key[UN];
    bool live[UN];  // paged: the key exists and its page entry is valid
#pragma unroll
    for (int u = 0; u < UN; ++u) {
      key[u] = r0 + (warp * UN + u) * KPW + kin;
      if constexpr (PAGED) {
        const long long off = key[u] < c1 ? rows.off(key[u]) : 0;
        live[u] = key[u] < c1 && off >= 0;
        if (live[u]) {
          ku[u] = ld_stream(rows.k + off);
          vu[u] = ld_stream(rows.v + off);
        } else {
          ku[u] = make_uint4(0, 0, 0, 0);
          vu[u] = make_uint4(0, 0, 0, 0);
        }
      } else {
        if (key[u] < c1) {
          ku[u] = ld_stream(kbase + static_cast<size_t>(key[u]) * D);
          vu[u] = ld_stream(vbase + static_cast<size_t>(key[u]) * D);
        } else {
          ku[u] = make_uint4(0, 0, 0, 0);
          vu[u] = make_uint4(0, 0, 0, 0);
        }
      }
    }
    float s[UN][G];
#pragma unroll
    for (int u = 0; u < UN; ++u) {
      float kf[8];
      bf16x8_to_f32(ku[u], kf);
#pragma unroll
      for (int g = 0; g < G; ++g) {
        float t = 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) t = fmaf(qf[g][e], kf[e], t);
#pragma unroll
        for (int off = LPK / 2; off > 0; off >>= 1) t += __shfl_xor_sync(0xffffffffu, t, off);
        bool keep;
        if constexpr (PAGED) keep = live[u];
        else keep = key[u] < c1;
        s[u][g] = keep ? t : -INFINITY;
      }
    }
#pragma unroll
    for (int g = 0; g < G; ++g) {
      float mg = m[g];
#pragma unroll
      for (int u = 0; u < UN; ++u) mg = fmaxf(mg, s[u][g]);
      const float mref = (mg == -INFINITY) ? 0.f : mg;
      const float alpha = ex2_approx(m[g] - mref);
      l[g] *= alpha;
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[g][e] *= alpha;
#pragma unroll
      for (int u = 0; u < UN; ++u) {
        const float pu = ex2_approx(s[u][g] - mref);
        l[g] += pu;
        float vf[8];
        bf16x8_to_f32(vu[u], vf);
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[g][e] = fmaf(pu, vf[e], acc[g][e]);
      }
      m[g] = mg;
    }
  }
  __shared__ float red_m[G][HW], red_l[G][HW];
  __shared__ float red_o[G][HW][D];
#pragma unroll
  for (int g = 0; g < G; ++g) {
#pragma unroll
    for (int e = 0; e < 8; ++e) red_o[g][grp][sub * 8 + e] = acc[g][e];
    if (sub == 0) {
      red_m[g][grp] = m[g];
      red_l[g][grp] = l[g];
    }
  }
  __syncthreads();
  for (int t = threadIdx.x; t < D; t += THREADS) {
#pragma unroll 1
    for (int g = 0; g < G; ++g) {
      float M = -INFINITY;
#pragma unroll
      for (int k2 = 0; k2 < HW; ++k2) M = fmaxf(M, red_m[g][k2]);
      float o = 0.f, lt = 0.f;
#pragma unroll
      for (int k2 = 0; k2 < HW; ++k2) {
        const float w = (red_m[g][k2] == -INFINITY) ? 0.f : ex2_approx(red_m[g][k2] - M);
        o = fmaf(w, red_o[g][k2][t], o);
        lt = fmaf(w, red_l[g][k2], lt);
      }
      float* out = part + ((bh0 + g) * S + split) * (D + 2);
      out[t] = o;
      if (t == 0) {
        out[D] = M;
        out[D + 1] = lt;
      }
    }
  }
}

template <int D>
__global__ void __launch_bounds__(D)
    fa_decode_combine_kernel(const float* __restrict__ part, const int* __restrict__ seqlens,
                             __nv_bfloat16* __restrict__ o, float* __restrict__ lse, int H,
                             int Lmax, int S) {
  const int bh = blockIdx.x;
  const int b = bh / H;
  const int t = threadIdx.x;
  const int L = min(max(seqlens[b], 0), Lmax);
  const int n = (L + CHUNK - 1) / CHUNK;
  const float* base = part + static_cast<size_t>(bh) * S * (D + 2);
  float M = -INFINITY;
  for (int s = 0; s < n; ++s) M = fmaxf(M, base[s * (D + 2) + D]);
  float acc = 0.f, lt = 0.f;
  for (int s = 0; s < n; ++s) {
    const float ms = base[s * (D + 2) + D];
    const float w = (ms == -INFINITY) ? 0.f : ex2_approx(ms - M);
    acc = fmaf(w, base[s * (D + 2) + t], acc);
    lt = fmaf(w, base[s * (D + 2) + D + 1], lt);
  }
  const float val = (lt > 0.f) ? acc / lt : 0.f;
  o[static_cast<size_t>(bh) * D + t] = __float2bfloat16_rn(val);
  if (t == 0 && lse != nullptr)
    lse[bh] = (lt > 0.f) ? (M + lg2_approx(lt)) * 0.6931471805599453f : -INFINITY;
}

template <int D, bool PAGED>
void launch_split(const __nv_bfloat16* qq, const __nv_bfloat16* kk, const __nv_bfloat16* vv,
                  const int* seqlens, float* part, int B, int H, int group, int Lmax, int S,
                  float sl2, const Pages& pg, cudaStream_t stream) {
  const int Hkv = H / group;
  // groups of 2, 4 or 8 query heads share one pass over their cache head;
  // other group sizes (and plain multi-head attention) use one CTA per head
  if (group == 2)
    fa_decode_group_split_kernel<D, 2, PAGED><<<dim3(S, Hkv, B), THREADS, 0, stream>>>(
        qq, kk, vv, seqlens, part, H, Hkv, Lmax, S, sl2, pg);
  else if (group == 4)
    fa_decode_group_split_kernel<D, 4, PAGED><<<dim3(S, Hkv, B), THREADS, 0, stream>>>(
        qq, kk, vv, seqlens, part, H, Hkv, Lmax, S, sl2, pg);
  else if (group == 8)
    fa_decode_group_split_kernel<D, 8, PAGED><<<dim3(S, Hkv, B), THREADS, 0, stream>>>(
        qq, kk, vv, seqlens, part, H, Hkv, Lmax, S, sl2, pg);
  else
    fa_decode_split_kernel<D, PAGED><<<dim3(S, H, B), THREADS, 0, stream>>>(
        qq, kk, vv, seqlens, part, H, group, Lmax, S, sl2, pg);
}

template <int D>
fa_status launch(const void* q, const void* kc, const void* vc, const int* seqlens, void* o,
                 float* lse, int B, int H, int group, int Lmax, float scale, float* part,
                 const Pages& pg, cudaStream_t stream) {
  const int S = decode_num_splits(Lmax);
  if (S > 0) {
    const auto* qq = static_cast<const __nv_bfloat16*>(q);
    const auto* kk = static_cast<const __nv_bfloat16*>(kc);
    const auto* vv = static_cast<const __nv_bfloat16*>(vc);
    const float sl2 = scale * 1.4426950408889634f;
    if (pg.table != nullptr)
      launch_split<D, true>(qq, kk, vv, seqlens, part, B, H, group, Lmax, S, sl2, pg, stream);
    else
      launch_split<D, false>(qq, kk, vv, seqlens, part, B, H, group, Lmax, S, sl2, pg, stream);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return FA_ERR_CUDA;
  }
  fa_decode_combine_kernel<D><<<B * H, D, 0, stream>>>(part, seqlens,
                                                       static_cast<__nv_bfloat16*>(o), lse, H,
                                                       Lmax, S > 0 ? S : 1);
  return cuda_status(cudaGetLastError());
}

}  // namespace dec

int decode_num_splits(int Lmax) { return (Lmax + dec::CHUNK - 1) / dec::CHUNK; }

fa_status launch_decode(const void* q, const void* kc, const void* vc, const int* seqlens,
                        void* o, float* lse, int B, int H, int Hkv, int Lmax, int d,
                        float scale, float* partials, cudaStream_t stream,
                        const int* page_table, int pages_per_seq, int log2_page,
                        int num_pages) {
  if (H > 65535 || B > 65535) return FA_ERR_INVALID_ARG;
  const int group = H / Hkv;
  const dec::Pages pg{page_table, pages_per_seq, log2_page, num_pages};
  if (d == 128)
    return dec::launch<128>(q, kc, vc, seqlens, o, lse, B, H, group, Lmax, scale, partials, pg,
                            stream);
  return dec::launch<64>(q, kc, vc, seqlens, o, lse, B, H, group, Lmax, scale, partials, pg,
                         stream);
}

}  // namespace fa
