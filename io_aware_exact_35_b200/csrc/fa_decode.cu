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
// Layout inside a CTA (4 warps), one query head per CTA: D/8 lanes share one
// key (8 bf16 = 16 bytes each), so a warp covers 32/(D/8) consecutive keys
// per step and issues UNROLL steps of K and V loads before using any of them.
// Grouped query heads (several heads per key/value head) are served together
// by a tensor-core kernel that reads each cached row once for the group.
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

// Keys per split: CHUNK, or for the grouped kernel CHUNK_MAX when the
// problem has enough splits of that length to fill the GPU several times
// over (longer splits amortise each CTA's start and its merge, which pays
// off with its two steps in flight per warp).  Workspaces are sized for
// CHUNK.
constexpr int CHUNK = 512;
constexpr int CHUNK_MAX = 1024;
constexpr int WARPS = 4;
constexpr int THREADS = WARPS * 32;
constexpr int UNROLL = 8;

// The split kernels let the combine kernel (launched after them with
// programmatic stream serialisation) be scheduled once all their CTAs have
// started; the combine kernel waits for their completion before it reads a
// partial, so only its launch overlaps their tail.
__device__ __forceinline__ void allow_combine_launch() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void wait_for_splits() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}

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

// D += A B for one m16n8k16 tile: A 16 x 16 bf16 (row-major fragment a0..a3),
// B 16 x 8 bf16 (column-major fragment b0, b1), D 16 x 8 f32 (PTX ISA,
// "Matrix fragments for mma.m16n8k16").
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1,
                                               uint32_t a2, uint32_t a3, uint32_t b0,
                                               uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
      "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// A row's maximum is only moved (and O, l rescaled) once it has grown by
// more than 2^8 (log2 units).
constexpr float STALE_MAX = 8.0f;

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
  allow_combine_launch();
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
        if (key[u] < c1 && dbg_ok(key[u] < Lmax)) {
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
  if (!dbg_ok(split < S)) return;
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

// Grouped-query decode on the tensor cores.  The G query heads that share a
// key/value head form a small dense contraction, S = Q_g K^T and
// O_g += P V with Q_g of G rows, so one warp runs it with mma.sync
// m16n8k16 (bf16 operands, f32 accumulation) straight from registers, 16
// keys per step: S with the heads as the 16 rows (padded when G < 16), then
// O^T += V^T P^T with the heads as the 8 columns of each n-tile, which takes
// the S accumulator re-packed to bf16 as its B operand unchanged.  The
// per-key work drops from ~60 warp instructions of FMAs and shuffles to
// ~7, and the kernel is left bound by the cache reads.  (tcgen05 needs at
// least 64 rows and shared-memory operands; with 2-16 heads the
// register-only mma.sync form avoids staging.)
//
// Operand placement.  The dot product over d and the sum over keys do not
// depend on the order of their terms, so every lane loads whole 16-byte
// vectors and the fragment slots are assigned to match them; lane
// (g, c) = (lane / 4, lane % 4):
//   S, k-step s (16 of the d values): B = K[key g][dk .. dk+3] and
//     A = Q[head g (and g + 8)][the same d], dk = 32 (s/2) + 8c + 4 (s%2):
//     four lanes' 16-byte loads cover 64 consecutive bytes of a key row.
//   O^T, m-tile t: A = V^T, rows g and g + 8 being d values e = t and
//     e = t + D/16 of the lane's own list d(e) = 64 (e/8) + 8g + e%8, columns
//     keys 2c, 2c+1, 2c+8, 2c+9: each lane loads those four rows at d 8g ..
//     8g+7 (and 64 + 8g ..), eight lanes covering 128 consecutive bytes of a
//     row per load, and pairs two keys' bf16 with one byte permute.  B = P^T:
//     column g, keys 2c, 2c+1 (and 2c+8, 2c+9), exactly the S accumulator
//     entries of lane (g, c).
// The online softmax is the one of the other decode kernels (log2 units,
// running max m and sum l per head), with the maximum kept stale until it
// grows by more than 2^8, as in the forward kernel.
template <int D, bool HI, bool PAGED>
__global__ void __launch_bounds__(THREADS)
    fa_decode_group_mma_kernel(const __nv_bfloat16* __restrict__ q,
                               const __nv_bfloat16* __restrict__ kc,
                               const __nv_bfloat16* __restrict__ vc,
                               const int* __restrict__ seqlens, float* __restrict__ part, int H,
                               int Hkv, int group, int qh, int Lmax, int S, int chunk,
                               float scale_log2, const Pages pg) {
  constexpr int ROWS = HI ? 16 : 8;  // head rows that can be real
  constexpr int NH = HI ? 2 : 1;     // 8-head column tiles of O^T
  constexpr int KS = D / 16;         // k-steps of S = Q K^T
  constexpr int MT = D / 16;         // m-tiles of O^T
  constexpr int NKL = D / 32;        // 16-byte loads per K row per lane
  constexpr int NVL = D / 64;        // 16-byte loads per V row per lane
  allow_combine_launch();
  const int split = blockIdx.x;
  const int h0 = blockIdx.y * qh;    // first query head of this CTA
  const int b = blockIdx.z;
  const int hk = h0 / group;
  const int L = min(max(seqlens[b], 0), Lmax);
  const int c0 = split * chunk;
  if (c0 >= L) return;
  const int c1 = min(c0 + chunk, L);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int g = lane >> 2;
  const int c = lane & 3;

  // Q as the A operand of S: rows g and g + 8, 4 d values per k-step
  uint32_t qa[KS][2], qb[KS][2];
  {
    const uint32_t* q0 = reinterpret_cast<const uint32_t*>(
        q + (static_cast<size_t>(b) * H + h0 + g) * D);
    const uint32_t* q1 = reinterpret_cast<const uint32_t*>(
        q + (static_cast<size_t>(b) * H + h0 + g + 8) * D);
#pragma unroll
    for (int s = 0; s < KS; ++s) {
      const int d0 = 32 * (s >> 1) + 8 * c + 4 * (s & 1);
      qa[s][0] = g < qh ? q0[d0 >> 1] : 0u;
      qa[s][1] = g < qh ? q0[(d0 >> 1) + 1] : 0u;
      qb[s][0] = (HI && g + 8 < qh) ? q1[d0 >> 1] : 0u;
      qb[s][1] = (HI && g + 8 < qh) ? q1[(d0 >> 1) + 1] : 0u;
    }
  }
  const size_t bkv = static_cast<size_t>(b) * Hkv + hk;
  const __nv_bfloat16* kbase = kc + bkv * static_cast<size_t>(Lmax) * D;
  const __nv_bfloat16* vbase = vc + bkv * static_cast<size_t>(Lmax) * D;
  __shared__ int spages[PAGED ? CHUNK_MAX : 1];
  const auto rows = kv_rows<D, PAGED>(kc, vc, pg, spages, b, hk, Hkv, Lmax, c0, c1, 0);
  // element offset of a key's row; -1 when the key is masked (past the
  // prefix, or an invalid page entry)
  auto row_off = [&](int key) -> long long {
    if (key >= c1) return -1;
    if constexpr (PAGED) return rows.off(key);
    else return static_cast<long long>(key) * D;
  };

  // DEPTH 16-key steps in flight per warp (two with 8 head rows; one with 16,
  // whose accumulators leave no registers for a second): buffer bs holds the
  // step being computed or a later one, and is refilled DEPTH steps ahead as
  // soon as its K (after S) or V (after P V) has been used.
  constexpr int DEPTH = HI ? 1 : 2;
  uint4 kr[DEPTH][2][NKL];  // K rows kb + g and kb + 8 + g
  uint4 vr[DEPTH][4][NVL];  // V rows kb + 2c, kb + 2c + 1, kb + 8 + 2c, kb + 9 + 2c
  bool klive[DEPTH][2];
  auto load_k = [&](const int bs, int kb) {
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      const long long off = row_off(kb + 8 * t + g);
      klive[bs][t] = off >= 0;
#pragma unroll
      for (int i = 0; i < NKL; ++i)
        kr[bs][t][i] = off >= 0 ? ld_stream((PAGED ? rows.k : kbase) + off + 32 * i + 8 * c)
                            : make_uint4(0, 0, 0, 0);
    }
  };
  auto load_v = [&](const int bs, int kb) {
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const long long off = row_off(kb + 8 * (r >> 1) + 2 * c + (r & 1));
#pragma unroll
      for (int i = 0; i < NVL; ++i)
        vr[bs][r][i] = off >= 0 ? ld_stream((PAGED ? rows.v : vbase) + off + 64 * i + 8 * g)
                            : make_uint4(0, 0, 0, 0);
    }
  };
  // bf16 pair (key a, key b) at entry e of the lane's V list
  auto vpair = [&](const int bs, int ra, int rb, int e) -> uint32_t {
    const uint4& ua = vr[bs][ra][e >> 3];
    const uint4& ub = vr[bs][rb][e >> 3];
    const int w = (e & 7) >> 1;
    const uint32_t wa = w == 0 ? ua.x : w == 1 ? ua.y : w == 2 ? ua.z : ua.w;
    const uint32_t wb = w == 0 ? ub.x : w == 1 ? ub.y : w == 2 ? ub.z : ub.w;
    return __byte_perm(wa, wb, (e & 1) ? 0x7632u : 0x5410u);
  };

  float o[NH][MT][4];  // O^T: [head tile][d tile]
#pragma unroll
  for (int n = 0; n < NH; ++n)
#pragma unroll
    for (int t = 0; t < MT; ++t) o[n][t][0] = o[n][t][1] = o[n][t][2] = o[n][t][3] = 0.f;
  float m[2] = {-INFINITY, -INFINITY};  // heads g, g + 8 (log2 units, stale)
  float l[2] = {0.f, 0.f};              // this lane's share of their sums

  const int kb0 = c0 + 16 * warp;  // this warp's steps: kb0, kb0 + 64, ...
  if (kb0 < c1) {
    load_k(0, kb0);
    load_v(0, kb0);
  }
  if (DEPTH > 1 && kb0 + 16 * WARPS < c1) {
    load_k(DEPTH - 1, kb0 + 16 * WARPS);
    load_v(DEPTH - 1, kb0 + 16 * WARPS);
  }
  auto step = [&](const int bs, const int kb) {
    const int nb = kb + DEPTH * 16 * WARPS;  // the next step held by buffer bs
    // S = Q K^T for keys kb .. kb+7 (half 0) and kb+8 .. kb+15 (half 1)
    float sc[2][4];
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      sc[t][0] = sc[t][1] = sc[t][2] = sc[t][3] = 0.f;
#pragma unroll
      for (int s = 0; s < KS; ++s) {
        const uint4& u = kr[bs][t][s >> 1];
        mma_bf16_16816(sc[t], qa[s][0], qb[s][0], qa[s][1], qb[s][1], (s & 1) ? u.z : u.x,
                       (s & 1) ? u.w : u.y);
      }
    }
    // column 2c + j of half t is key kb + 8t + 2c + j, loaded (or found
    // masked) by lanes 4 (2c + j) .. 4 (2c + j) + 3
    bool live[2][2];
#pragma unroll
    for (int t = 0; t < 2; ++t)
#pragma unroll
      for (int j = 0; j < 2; ++j)
        live[t][j] = __shfl_sync(0xffffffffu, static_cast<int>(klive[bs][t]), 4 * (2 * c + j)) != 0;
    if (nb < c1) load_k(bs, nb);

    uint32_t pb[2][2] = {{0u, 0u}, {0u, 0u}};  // P^T as the B operand: [head half][key half]
    float alpha[2] = {1.f, 1.f};
    bool grew = false;
#pragma unroll
    for (int r = 0; r < NH; ++r) {
      float x[2][2];
      float mx = -INFINITY;
#pragma unroll
      for (int t = 0; t < 2; ++t)
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          x[t][j] = live[t][j] ? sc[t][2 * r + j] * scale_log2 : -INFINITY;
          mx = fmaxf(mx, x[t][j]);
        }
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
      const float m_new = fmaxf(m[r], mx);
      if (m_new - m[r] > STALE_MAX) {  // also when m = -inf < m_new
        alpha[r] = ex2_approx(m[r] - m_new);
        l[r] *= alpha[r];
        m[r] = m_new;
        grew = true;
      }
      const float mref = (m[r] == -INFINITY) ? 0.f : m[r];
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        const float p0 = ex2_approx(x[t][0] - mref);
        const float p1 = ex2_approx(x[t][1] - mref);
        l[r] += p0 + p1;
        pb[r][t] = pack_bf16x2(p0, p1);
      }
    }
    if (__any_sync(0xffffffffu, grew)) {
      // column j of head tile n is head 8n + 2c + j, whose factor lane
      // 4 (2c + j) computed
#pragma unroll
      for (int n = 0; n < NH; ++n) {
        const float a0 = __shfl_sync(0xffffffffu, alpha[n], 8 * c);
        const float a1 = __shfl_sync(0xffffffffu, alpha[n], 8 * c + 4);
#pragma unroll
        for (int t = 0; t < MT; ++t) {
          o[n][t][0] *= a0;
          o[n][t][1] *= a1;
          o[n][t][2] *= a0;
          o[n][t][3] *= a1;
        }
      }
    }

    // O^T += V^T P^T
#pragma unroll
    for (int t = 0; t < MT; ++t) {
      const uint32_t a0 = vpair(bs, 0, 1, t);
      const uint32_t a1 = vpair(bs, 0, 1, t + MT);
      const uint32_t a2 = vpair(bs, 2, 3, t);
      const uint32_t a3 = vpair(bs, 2, 3, t + MT);
#pragma unroll
      for (int n = 0; n < NH; ++n) mma_bf16_16816(o[n][t], a0, a1, a2, a3, pb[n][0], pb[n][1]);
    }
    if (nb < c1) load_v(bs, nb);
  };
  for (int kb = kb0; kb < c1; kb += DEPTH * 16 * WARPS) {
    step(0, kb);
    if (DEPTH > 1 && kb + 16 * WARPS < c1) step(DEPTH - 1, kb + 16 * WARPS);
  }

  // Merge the four warps of the CTA: per head, M = max m_w, then
  // sum_w 2^(m_w - M) (O_w, l_w).
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    l[r] += __shfl_xor_sync(0xffffffffu, l[r], 1);
    l[r] += __shfl_xor_sync(0xffffffffu, l[r], 2);
  }
  __shared__ float red_m[ROWS][WARPS], red_l[ROWS][WARPS];
  __shared__ float red_o[ROWS][WARPS][D];
#pragma unroll
  for (int n = 0; n < NH; ++n) {
#pragma unroll
    for (int t = 0; t < MT; ++t) {
      const int dlo = 64 * (t >> 3) + 8 * g + (t & 7);                  // entry t
      const int dhi = 64 * ((t + MT) >> 3) + 8 * g + ((t + MT) & 7);    // entry t + D/16
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        red_o[8 * n + 2 * c + j][warp][dlo] = o[n][t][j];
        red_o[8 * n + 2 * c + j][warp][dhi] = o[n][t][2 + j];
      }
    }
    if (c == 0) {
      red_m[8 * n + g][warp] = m[n];
      red_l[8 * n + g][warp] = l[n];
    }
  }
  __syncthreads();
  for (int idx = threadIdx.x; idx < qh * D; idx += THREADS) {
    const int row = idx / D;
    const int t = idx - row * D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < WARPS; ++w) M = fmaxf(M, red_m[row][w]);
    float acc = 0.f, lt = 0.f;
#pragma unroll
    for (int w = 0; w < WARPS; ++w) {
      const float wt = (red_m[row][w] == -INFINITY) ? 0.f : ex2_approx(red_m[row][w] - M);
      acc = fmaf(wt, red_o[row][w][t], acc);
      lt = fmaf(wt, red_l[row][w], lt);
    }
    float* out = part + ((static_cast<size_t>(b) * H + h0 + row) * S + split) * (D + 2);
    if (!dbg_ok(split < S && h0 + row < H)) continue;
    out[t] = acc;
    if (t == 0) {
      out[D] = M;
      out[D + 1] = lt;
    }
  }
}

// Block-wide max / sum over the D threads of a combine CTA (`red` holds one
// value per warp; every thread gets the result).
template <int D, bool MAX>
__device__ __forceinline__ float block_reduce(float v, float* red) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    const float u = __shfl_xor_sync(0xffffffffu, v, off);
    v = MAX ? fmaxf(v, u) : v + u;
  }
  __syncthreads();  // `red` may still be read from a previous reduction
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  v = red[0];
#pragma unroll
  for (int w = 1; w < D / 32; ++w) v = MAX ? fmaxf(v, red[w]) : v + red[w];
  return v;
}

// One CTA per (b, h), thread t owns output column t.  The split weights
// w_s = 2^(m_s - M) are computed once per split (one thread each) and shared
// through shared memory; the column sums then read the partials of up to D
// splits with independent, coalesced loads.
template <int D>
__global__ void __launch_bounds__(D)
    fa_decode_combine_kernel(const float* __restrict__ part, const int* __restrict__ seqlens,
                             __nv_bfloat16* __restrict__ o, float* __restrict__ lse, int H,
                             int Lmax, int S, int chunk) {
  wait_for_splits();
  const int bh = blockIdx.x;
  const int b = bh / H;
  const int t = threadIdx.x;
  const int L = min(max(seqlens[b], 0), Lmax);
  const int n = (L + chunk - 1) / chunk;
  const float* base = part + static_cast<size_t>(bh) * S * (D + 2);
  __shared__ float red[D / 32];
  __shared__ float wts[D];
  float M = -INFINITY;
  for (int s = t; s < n; s += D) M = fmaxf(M, base[static_cast<size_t>(s) * (D + 2) + D]);
  M = block_reduce<D, true>(M, red);
  float acc = 0.f, lpart = 0.f;
  for (int s0 = 0; s0 < n; s0 += D) {
    float w = 0.f;
    if (s0 + t < n) {
      const float* ps = base + static_cast<size_t>(s0 + t) * (D + 2);
      const float ms = ps[D];
      w = (ms == -INFINITY) ? 0.f : ex2_approx(ms - M);
      lpart = fmaf(w, ps[D + 1], lpart);
    }
    __syncthreads();  // the previous chunk's weights have been used
    wts[t] = w;
    __syncthreads();
    const int cnt = min(D, n - s0);
    const float* ob = base + static_cast<size_t>(s0) * (D + 2) + t;
    int k = 0;
    for (; k + 8 <= cnt; k += 8) {
      float v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) v[u] = ob[static_cast<size_t>(k + u) * (D + 2)];
#pragma unroll
      for (int u = 0; u < 8; ++u) acc = fmaf(wts[k + u], v[u], acc);
    }
    for (; k < cnt; ++k) acc = fmaf(wts[k], ob[static_cast<size_t>(k) * (D + 2)], acc);
  }
  const float lt = block_reduce<D, false>(lpart, red);
  const float val = (lt > 0.f) ? acc / lt : 0.f;
  o[static_cast<size_t>(bh) * D + t] = __float2bfloat16_rn(val);
  if (t == 0 && lse != nullptr)
    lse[bh] = (lt > 0.f) ? (M + lg2_approx(lt)) * 0.6931471805599453f : -INFINITY;
}

// Query heads per CTA of the grouped (tensor-core) kernel, 0 for the
// per-head kernel: the whole group when it has at most 16 heads, else 16 or
// 8 of them (the cache head is then read by several CTAs).  Plain multi-head
// attention and other group sizes use one CTA per query head.
inline int group_heads_per_cta(int group) {
  if (group <= 1) return 0;
  return group <= 16 ? group : (group % 16 == 0 ? 16 : (group % 8 == 0 ? 8 : 0));
}

template <int D, bool PAGED>
void launch_split(const __nv_bfloat16* qq, const __nv_bfloat16* kk, const __nv_bfloat16* vv,
                  const int* seqlens, float* part, int B, int H, int group, int Lmax, int S,
                  int chunk, float sl2, const Pages& pg, cudaStream_t stream) {
  const int Hkv = H / group;
  const int qh = group_heads_per_cta(group);
  if (qh > 0) {
    const dim3 grid(S, H / qh, B);
    if (qh > 8)
      fa_decode_group_mma_kernel<D, true, PAGED><<<grid, THREADS, 0, stream>>>(
          qq, kk, vv, seqlens, part, H, Hkv, group, qh, Lmax, S, chunk, sl2, pg);
    else
      fa_decode_group_mma_kernel<D, false, PAGED><<<grid, THREADS, 0, stream>>>(
          qq, kk, vv, seqlens, part, H, Hkv, group, qh, Lmax, S, chunk, sl2, pg);
  } else {
    fa_decode_split_kernel<D, PAGED><<<dim3(S, H, B), THREADS, 0, stream>>>(
        qq, kk, vv, seqlens, part, H, group, Lmax, S, sl2, pg);
  }
}

template <int D>
fa_status launch(const void* q, const void* kc, const void* vc, const int* seqlens, void* o,
                 float* lse, int B, int H, int group, int Lmax, float scale, float* part,
                 const Pages& pg, cudaStream_t stream) {
  // Split length: CHUNK for the per-head kernel; for the grouped kernel
  // CHUNK_MAX once its splits alone give at least 8 CTAs per SM (by the
  // cache capacity Lmax), else CHUNK.  The partials then take
  // ceil(Lmax / chunk) <= ceil(Lmax / CHUNK) slots per head.
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return FA_ERR_CUDA;
  const int qh = group_heads_per_cta(group);
  const long long rows = static_cast<long long>(B) * (qh > 0 ? H / qh : H);
  const long long long_splits = (static_cast<long long>(Lmax) + CHUNK_MAX - 1) / CHUNK_MAX;
  const int chunk = (qh > 0 && rows * long_splits >= 8LL * sms) ? CHUNK_MAX : CHUNK;
  const int S = (Lmax + chunk - 1) / chunk;
  if (S > 0) {
    const auto* qq = static_cast<const __nv_bfloat16*>(q);
    const auto* kk = static_cast<const __nv_bfloat16*>(kc);
    const auto* vv = static_cast<const __nv_bfloat16*>(vc);
    const float sl2 = scale * 1.4426950408889634f;
    main_kernel_begin(stream);
    if (pg.table != nullptr)
      launch_split<D, true>(qq, kk, vv, seqlens, part, B, H, group, Lmax, S, chunk, sl2, pg,
                            stream);
    else
      launch_split<D, false>(qq, kk, vv, seqlens, part, B, H, group, Lmax, S, chunk, sl2, pg,
                             stream);
    main_kernel_end(stream);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return FA_ERR_CUDA;
  }
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(B * H);
  cfg.blockDim = dim3(D);
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const float* cpart = part;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, fa_decode_combine_kernel<D>, cpart, seqlens,
                                           static_cast<__nv_bfloat16*>(o), lse, H, Lmax,
                                           S > 0 ? S : 1, chunk);
  if (e != cudaSuccess) {
    (void)cudaGetLastError();
    return FA_ERR_CUDA;
  }
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
