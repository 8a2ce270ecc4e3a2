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

__device__ __forceinline__ void bf16x8_to_f32(const uint4& u, float (&f)[8]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

template <int D>
__global__ void __launch_bounds__(THREADS)
    fa_decode_split_kernel(const __nv_bfloat16* __restrict__ q,
                           const __nv_bfloat16* __restrict__ kc,
                           const __nv_bfloat16* __restrict__ vc, const int* __restrict__ seqlens,
                           float* __restrict__ part, int H, int group, int Lmax, int S,
                           float scale_log2) {
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

  float m = -INFINITY, l = 0.f, acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.f;

  constexpr int KEYS_PER_ROUND = WARPS * UNROLL * KPW;
  for (int r0 = c0; r0 < c1; r0 += KEYS_PER_ROUND) {
    uint4 ku[UNROLL], vu[UNROLL];
    int key[UNROLL];
#pragma unroll
    for (int u = 0; u < UNROLL; ++u) {
      key[u] = r0 + (warp * UNROLL + u) * KPW + kin;
      if (key[u] < c1) {
        ku[u] = ld_stream(kbase + static_cast<size_t>(key[u]) * D);
        vu[u] = ld_stream(vbase + static_cast<size_t>(key[u]) * D);
      } else {
        ku[u] = make_uint4(0, 0, 0, 0);
        vu[u] = make_uint4(0, 0, 0, 0);
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
      s[u] = (key[u] < c1) ? t : -INFINITY;
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

template <int D>
fa_status launch(const void* q, const void* kc, const void* vc, const int* seqlens, void* o,
                 float* lse, int B, int H, int group, int Lmax, float scale, float* part,
                 cudaStream_t stream) {
  const int S = decode_num_splits(Lmax);
  if (S > 0) {
    dim3 grid(S, H, B);
    fa_decode_split_kernel<D><<<grid, THREADS, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(kc),
        static_cast<const __nv_bfloat16*>(vc), seqlens, part, H, group, Lmax, S,
        scale * 1.4426950408889634f);
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
                        float scale, float* partials, cudaStream_t stream) {
  if (H > 65535 || B > 65535) return FA_ERR_INVALID_ARG;
  const int group = H / Hkv;
  if (d == 128)
    return dec::launch<128>(q, kc, vc, seqlens, o, lse, B, H, group, Lmax, scale, partials, stream);
  return dec::launch<64>(q, kc, vc, seqlens, o, lse, B, H, group, Lmax, scale, partials, stream);
}

}  // namespace fa
