// fa_bwd.cu - backward pass of exact attention on sm_100a, with recomputation.
//
// "Flash Attention La Gi?" (thienlv.com glossary), Recomputation: the
// attention matrix is not stored by the forward pass; the backward pass
// recomputes it tile by tile from Q, K and the saved log-sum-exp.  With
// L = sum(O * dO) and S = scale Q K^T:
//   P = exp(S - LSE),  dV = P^T dO,  dP = dO V^T,  D = rowsum(dO * O),
//   dS = P * (dP - D),  dQ = scale dS K,  dK = scale dS^T Q.
//
// Three kernels; the second and third are launched with programmatic stream
// serialisation (each may start before the kernel before it has ended):
//   fa_bwd_preprocess  D = rowsum(dO * O) (fp32), a zeroed fp32 dQ accumulator
//                      and zeroed completion counters, one per key/value head.
//   fa_bwd_kernel      one CTA per 128-key tile j of one (batch, head); it keeps
//                      dK_j and dV_j in tensor memory and loops over the query
//                      tiles i that can see key tile j (causal: those holding a
//                      query at or after key j's position):
//                        S^T = K_j Q_i^T, dP^T = V_j dO_i^T        (tcgen05, TMEM)
//                        P^T, dS^T on the CUDA cores (one key row per thread)
//                        dV += P^T dO_i, dK += dS^T Q_i            (A from TMEM)
//                        dQ_i = dS K_j  (A = dS from shared memory), added to
//                        an fp32 accumulator with bulk tensor reductions.
//                      Its set-up and K_j / V_j loads overlap the end of the
//                      preprocess; every thread waits for the preprocess
//                      (griddepcontrol.wait) before the first table load.
//                      When its last reduction has completed, a CTA adds one
//                      to its key/value head's completion counter.
//   fa_bwd_dq_convert  dQ = scale * accumulator, rounded to bf16.  A CTA of
//                      it converts rows of one query head once the counter of
//                      that head's key/value head reaches the number of key
//                      tiles, so the heads finished first (the grid of the
//                      main kernel runs head by head) are converted on SMs
//                      that the main kernel's last CTAs leave idle.
//
// Warp roles of fa_bwd_kernel (448 threads):
//   warps 0-7  two P^T / dS^T warpgroups: thread t of warpgroup g owns key row t
//              (TMEM lane t) for queries 64g .. 64g+63 of the tile, in two
//              phases: P^T as soon as S^T is ready (dV can start), then dS^T
//              once dP^T is ready.  In the epilogue warpgroup 0 writes dV and
//              warpgroup 1 writes dK.
//   warps 8-11 dQ warpgroup: thread t owns query row t of the dQ tile.
//   warp 12    TMA producer: K_j, V_j once; Q_i with LSE_i and dO_i with D_i
//              through a two-stage ring whose Q and dO halves are filled and
//              released separately.
//   warp 13    tensor-memory allocator and MMA issuer, in the order
//                S^T(i) dP^T(i) | dV(i) | dK(i) dQ(i) | S^T(i+1) ...
//              where "|" waits for the P^T phase, the dS^T phase, and (before
//              the next dP^T) for dQ(i) to have left tensor memory.
// Tensor memory (512 columns): S^T [0,128), dP^T [128,256), dV [256, 256+d),
// dK [256+d, 256+2d).  Warpgroup g overwrites columns [64g, 64g+32) of S^T
// with P^T (bf16 pairs) and the same columns of dP^T with dS^T, i.e. only
// scores it has already read; dQ_i lands in [128, 128+d) afterwards.
// dQ_i leaves tensor memory into the Q_i / dO_i stage it was computed from
// (free once dQ_i is complete), so the dS buffer is never shared with it.
// The reduction of the half staged over Q_i is committed first: Q_{i+2} is
// needed by the next S^T before dO_{i+2} is needed by the next dP^T.
#include <cstdlib>
#include <cstring>

#include "fa_internal.h"
#include "sm100.cuh"

namespace fa {

namespace bwd {

// Orders this thread's completed bulk (async-proxy) writes to global memory
// before its later generic accesses, e.g. a release that publishes them.
__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}
// In a kernel launched with programmatic stream serialisation: wait until the
// preceding grid has completed and its writes are visible (a no-op when the
// launch had no such dependency).
__device__ __forceinline__ void griddep_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}
// Allow the next grid in the stream, if launched with programmatic stream
// serialisation, to start before this one has finished.
__device__ __forceinline__ void griddep_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

constexpr int BLOCK = 128;
constexpr int NUM_THREADS = 448;
constexpr int PANEL_BYTES = 128 * 128;
constexpr uint32_t TMEM_COLS = 512;
constexpr float LOG2E = 1.4426950408889634f;

template <int D>
struct Smem {
  static constexpr int NPANEL = D / 64;
  static constexpr int TILE = NPANEL * PANEL_BYTES;  // 128 rows x D bf16
  static constexpr int K_OFF = 0;
  static constexpr int V_OFF = TILE;
  static constexpr int Q_OFF = 2 * TILE;               // 2 stages
  static constexpr int DO_OFF = Q_OFF + 2 * TILE;      // 2 stages
  static constexpr int DS_OFF = DO_OFF + 2 * TILE;     // 128 keys x 128 queries bf16
  static constexpr int DS_BYTES = 2 * PANEL_BYTES;
  static constexpr int LSE_OFF = DS_OFF + DS_BYTES;    // 2 stages x 128 fp32
  static constexpr int DD_OFF = LSE_OFF + 2 * 512;     // 2 stages x 128 fp32
  static constexpr int BAR_OFF = DD_OFF + 2 * 512;
  // kv_full, q_full[2], q_empty[2], st_full, dpt_full, ds_full, dq_full,
  // dq_free, dkv_final, mma_final, stg_full, p_full, do_full[2], do_empty[2]
  static constexpr int NBAR = 18;
  static constexpr int MISC_OFF = BAR_OFF + NBAR * 8;
  static constexpr int BYTES = MISC_OFF + 16;
  static constexpr int ALLOC = BYTES > 118784 ? BYTES : 118784;
};

struct Params {
  __nv_bfloat16* dk;
  __nv_bfloat16* dv;
  float* dqacc;
  int Nq;            // query rows per head (padded layout)
  int Nk;            // key / value rows per head (padded layout)
  int causal_off;    // Nk - Nq: query i sits at key position i + causal_off
  int n_qt;          // query tiles per head, ceil(Nq / 128) (padded layout)
  int n_kt;          // key tiles per head, ceil(Nk / 128), or of the longest
                     // sequence (ragged batch)
  int group;         // query heads per key/value head (1 without grouping)
  int BHkv;          // batch x key/value heads
  int lpt_order;     // 1: key tile 0 of every head first; 0: head-major
  float scale_log2;  // scale * log2(e)
  float scale;
  // ragged batch (token-major packing): sequence b owns rows cu_q[b] ..
  // cu_q[b+1]-1 of q / o / dO / dQ and cu_k[b] .. of k / v / dK / dV; its
  // rows of the LSE / D tables start at table_row0(cu_q[b], b)
  const int* cu_q;
  const int* cu_k;
  int Hkv;           // key/value heads
  int total_q, total_k;
  // element strides of dK / dV: [head][row] at head * kv_head + row * kv_row
  size_t kv_head, kv_row;
  size_t kv_elems;   // elements of dK (= of dV), for the debug build's checks
  // completion counter per key/value head (padded layout), zeroed by the
  // preprocess; nullptr: the conversion waits for the whole kernel instead
  unsigned* done_cnt;
};

// First row of sequence b in the ragged LSE / D tables: a multiple of 4 (a
// bulk tensor copy must start 16-byte aligned) followed by at least 127
// padding rows before the next sequence, so a 128-row tile read from the
// sequence's last tile stays inside its padding (+inf / 0).
__host__ __device__ __forceinline__ long long table_row0(int cu_q_b, int b) {
  return 4LL * ((static_cast<long long>(cu_q_b) + 3) / 4) + 132LL * b;
}

// Where a CTA's key tile lives.  Rows are counted within the sequence; q0 /
// k0 are the sequence's first rows in the tensor maps and t0 its first row
// of the LSE / D tables (all 0 for the padded layout).
struct CtaGeo {
  int kv_tile;
  int kv_head;      // head coordinate of K / V / dK / dV
  int q_head0;      // head coordinate of the group's first query head
  int q0, k0, t0;
  int Nq, Nk, off;  // lengths of the sequence and Nk - Nq
  int n_qt;         // query tiles of the sequence
};

template <bool VARLEN>
__device__ __forceinline__ CtaGeo cta_geo(const Params& p, int bx) {
  CtaGeo g;
  int bkv;
  if (p.lpt_order) {
    g.kv_tile = bx / p.BHkv;
    bkv = bx - g.kv_tile * p.BHkv;
  } else {
    g.kv_tile = bx % p.n_kt;
    bkv = bx / p.n_kt;
  }
  if constexpr (!VARLEN) {
    g.kv_head = bkv;
    g.q_head0 = bkv * p.group;
    g.q0 = g.k0 = g.t0 = 0;
    g.Nq = p.Nq;
    g.Nk = p.Nk;
  } else {
    const int b = bkv / p.Hkv;
    g.kv_head = bkv - b * p.Hkv;
    g.q_head0 = g.kv_head * p.group;
    g.q0 = p.cu_q[b];
    g.k0 = p.cu_k[b];
    g.Nq = p.cu_q[b + 1] - g.q0;
    g.Nk = p.cu_k[b + 1] - g.k0;
    // offsets outside the packed arrays are never used: the sequence is empty
    if (g.q0 < 0 || g.Nq < 0 || g.q0 + g.Nq > p.total_q) g.Nq = 0;
    if (g.k0 < 0 || g.Nk < 0 || g.k0 + g.Nk > p.total_k) g.Nk = 0;
    g.t0 = static_cast<int>(table_row0(g.q0, b));
  }
  g.off = g.Nk - g.Nq;
  g.n_qt = (g.Nq + BLOCK - 1) / BLOCK;
  return g;
}

// Bulk tensor loads / reductions of 128 rows starting at `row` of head
// `head`: the padded maps are [heads, rows, columns], the ragged ones
// [rows, heads, columns].
template <bool VARLEN>
__device__ __forceinline__ void load_rows(void* dst, const CUtensorMap* map, uint64_t* bar, int x,
                                          int row, int head) {
  if constexpr (VARLEN)
    tma_load_3d(dst, map, bar, x, head, row);
  else
    tma_load_3d(dst, map, bar, x, row, head);
}
template <bool VARLEN>
__device__ __forceinline__ void reduce_rows(const CUtensorMap* map, const void* src, int x, int row,
                                            int head) {
  if constexpr (VARLEN)
    tma_reduce_add_3d(map, src, x, head, row);
  else
    tma_reduce_add_3d(map, src, x, row, head);
}

__device__ __forceinline__ void tma_load_2d(void* smem_dst, const void* desc, uint64_t* bar,
                                            int c0, int c1) {
  if (!dbg_ok(c0 >= 0 && (c0 & 3) == 0 && c1 >= 0)) return;  // fp32 rows, 16-byte aligned
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(smem_dst)),
      "l"(desc), "r"(c0), "r"(c1), "r"(smem_u32(bar))
      : "memory");
}

template <int D, bool CAUSAL, bool VARLEN>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    fa_bwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                  const __grid_constant__ CUtensorMap tm_lse,
                  const __grid_constant__ CUtensorMap tm_dd,
                  const __grid_constant__ CUtensorMap tm_dq, const Params p) {
  using L = Smem<D>;
  extern __shared__ __align__(1024) uint8_t smem[];
  // The swizzled operand tiles need 1024-byte alignment; the kernel declares
  // no static shared memory, so the dynamic window starts aligned.
  if ((smem_u32(smem) & 1023u) != 0) {
    if (threadIdx.x == 0) record_error(2 /* FA_ERR_UNSUPPORTED */);
    return;
  }
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::BAR_OFF);
  uint64_t* kv_full = bars + 0;
  uint64_t* q_full = bars + 1;    // [2] Q_i and LSE_i loaded
  uint64_t* q_empty = bars + 3;   // [2] Q_i stage released
  uint64_t* do_full = bars + 14;  // [2] dO_i and D_i loaded
  uint64_t* do_empty = bars + 16; // [2] dO_i stage released
  uint64_t* st_full = bars + 5;
  uint64_t* dpt_full = bars + 6;
  uint64_t* ds_full = bars + 7;    // dS^T (TMEM) and dS (shared) written
  uint64_t* dq_full = bars + 8;
  uint64_t* dq_free = bars + 9;    // dQ read out of tensor memory
  uint64_t* dkv_final = bars + 10;
  uint64_t* mma_final = bars + 11;
  uint64_t* stg_full = bars + 12;  // dQ staging written (128 arrivals)
  uint64_t* p_full = bars + 13;    // P^T written (both warpgroups)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::MISC_OFF + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // One-dimensional grid, head-major: the key tiles of one (batch, head) are
  // adjacent in launch order (so resident CTAs share that head's Q and dO
  // tiles in L2); tile 0, which sees the most query tiles, comes first.
  // bkv indexes key/value heads; the CTA accumulates dK, dV of key tile
  // kv_tile over the query tiles of all `group` query heads sharing it.
  // Head-major order keeps one head's Q / dO tiles shared in L2 by its
  // resident CTAs; longest-first order (key tile 0, which sees every query
  // tile, of all heads first) balances few long CTAs.
  const CtaGeo geo = cta_geo<VARLEN>(p, static_cast<int>(blockIdx.x));
  // ragged batch: key tiles past the end of their sequence have no work
  if (VARLEN && geo.kv_tile * BLOCK >= geo.Nk) return;
  const int key0 = geo.kv_tile * BLOCK;
  // causal: the first query that sees key key0 is row key0 - off
  const int i_begin = CAUSAL ? max(0, key0 - geo.off) / BLOCK : 0;
  const int n_per = max(0, geo.n_qt - i_begin);  // query tiles per query head
  const int n_it = n_per * p.group;              // 0: dK = dV = 0
  // iteration it -> (query head, first row of its query tile in the sequence)
  auto it_head = [&](int it) { return geo.q_head0 + it / n_per; };
  auto it_q0 = [&](int it) { return (i_begin + it % n_per) * BLOCK; };

  if (threadIdx.x == 0) {
    for (int b = 0; b < L::NBAR; ++b) mbar_init(&bars[b], 1);
    mbar_init(p_full, 2 * BLOCK);   // both P^T / dS^T warpgroups
    mbar_init(ds_full, 2 * BLOCK);
    mbar_init(dq_free, BLOCK);
    mbar_init(stg_full, BLOCK);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 13) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // The next grid (the dQ conversion) may be scheduled once every thread of
  // every CTA has got here, i.e. after the preprocess has completed: its
  // counters are zero by then.
  if (warp != 12) {
    griddep_wait();
    griddep_launch_dependents();
  }
  const uint32_t tmem_base = *tmem_slot;
  const uint32_t tSt = tmem_base;
  const uint32_t tdPt = tmem_base + 128;
  const uint32_t tdV = tmem_base + 256;
  const uint32_t tdK = tmem_base + 256 + D;

  if (warp == 12) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_do);
      mbar_arrive_expect_tx(kv_full, 2 * L::TILE);
      for (int pn = 0; pn < L::NPANEL; ++pn) {
        load_rows<VARLEN>(smem + L::K_OFF + pn * PANEL_BYTES, &tm_k, kv_full, pn * 64,
                          geo.k0 + key0, geo.kv_head);
        load_rows<VARLEN>(smem + L::V_OFF + pn * PANEL_BYTES, &tm_v, kv_full, pn * 64,
                          geo.k0 + key0, geo.kv_head);
      }
    }
    // the LSE / D tables come from the preprocess
    griddep_wait();
    griddep_launch_dependents();
    if (lane == 0) {
      int last_q[2] = {-1, -1}, last_do[2] = {-1, -1};
      for (int it = 0; it < n_it; ++it) {
        const int st = it & 1;
        const int r = it >> 1;
        const int q0 = it_q0(it);
        const int bh = it_head(it);
        if (it >= 2 && !mbar_wait(&q_empty[st], (r - 1) & 1, abort_flag)) break;
        mbar_arrive_expect_tx(&q_full[st], L::TILE + 512);
        for (int pn = 0; pn < L::NPANEL; ++pn)
          load_rows<VARLEN>(smem + L::Q_OFF + st * L::TILE + pn * PANEL_BYTES, &tm_q,
                            &q_full[st], pn * 64, geo.q0 + q0, bh);
        tma_load_2d(smem + L::LSE_OFF + st * 512, &tm_lse, &q_full[st], geo.t0 + q0, bh);
        last_q[st] = r;
        if (it >= 2 && !mbar_wait(&do_empty[st], (r - 1) & 1, abort_flag)) break;
        mbar_arrive_expect_tx(&do_full[st], L::TILE + 512);
        for (int pn = 0; pn < L::NPANEL; ++pn)
          load_rows<VARLEN>(smem + L::DO_OFF + st * L::TILE + pn * PANEL_BYTES, &tm_do,
                            &do_full[st], pn * 64, geo.q0 + q0, bh);
        tma_load_2d(smem + L::DD_OFF + st * 512, &tm_dd, &do_full[st], geo.t0 + q0, bh);
        last_do[st] = r;
      }
      mbar_wait_drain(kv_full, 0);
      for (int s = 0; s < 2; ++s) {
        if (last_q[s] >= 0) mbar_wait_drain(&q_full[s], last_q[s] & 1);
        if (last_do[s] >= 0) mbar_wait_drain(&do_full[s], last_do[s] & 1);
      }
    }
  } else if (warp == 13) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t IDESC_SS = idesc_bf16_f32(BLOCK, BLOCK, false, false);
      constexpr uint32_t IDESC_ACC = idesc_bf16_f32(BLOCK, D, false, true);
      constexpr uint32_t IDESC_DQ = idesc_bf16_f32(BLOCK, D, true, true);
      // Descriptors are built once; a k-step adds a compile-time byte offset
      // (>> 4) to the start-address field (no carry below 256 KB), so each MMA
      // costs a few instructions on a scheduler shared with busy warps.
      const uint64_t kdK = sdesc_kmajor_sw128(smem_u32(smem + L::K_OFF));
      const uint64_t vdK = sdesc_kmajor_sw128(smem_u32(smem + L::V_OFF));
      const uint64_t kdM = sdesc_mnmajor_sw128(smem_u32(smem + L::K_OFF), PANEL_BYTES);
      const uint64_t dsdM = sdesc_mnmajor_sw128(smem_u32(smem + L::DS_OFF), PANEL_BYTES);
      const uint64_t qdK0 = sdesc_kmajor_sw128(smem_u32(smem + L::Q_OFF));
      const uint64_t dodK0 = sdesc_kmajor_sw128(smem_u32(smem + L::DO_OFF));
      const uint64_t qdM0 = sdesc_mnmajor_sw128(smem_u32(smem + L::Q_OFF), PANEL_BYTES);
      const uint64_t dodM0 = sdesc_mnmajor_sw128(smem_u32(smem + L::DO_OFF), PANEL_BYTES);
      auto koff = [](int kk) {  // K-major: 16-element K slice kk of a 128-row tile
        return static_cast<uint64_t>(((kk >> 2) * PANEL_BYTES + (kk & 3) * 32) >> 4);
      };
      auto moff = [](int kk) {  // MN-major: rows 16kk .. 16kk+15
        return static_cast<uint64_t>((kk * 2048) >> 4);
      };
      bool ok = mbar_wait(kv_full, 0, abort_flag);
      for (int it = 0; ok && it < n_it; ++it) {
        const int st = it & 1;
        const uint64_t soff = static_cast<uint64_t>((st * L::TILE) >> 4);
        if (!mbar_wait(&q_full[st], (it >> 1) & 1, abort_flag)) { ok = false; break; }
        tc_fence_after();
        // S^T = K_j Q_i^T  (M = keys, N = queries, K = d)
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          mma_bf16_ss(tSt, kdK + koff(kk), qdK0 + soff + koff(kk), IDESC_SS, kk > 0 ? 1u : 0u);
        mma_commit(st_full);
        // dP^T = V_j dO_i^T, into columns the dQ warps must have emptied.
        if (!mbar_wait(&do_full[st], (it >> 1) & 1, abort_flag)) { ok = false; break; }
        if (it >= 1 && !mbar_wait(dq_free, (it - 1) & 1, abort_flag)) { ok = false; break; }
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          mma_bf16_ss(tdPt, vdK + koff(kk), dodK0 + soff + koff(kk), IDESC_SS, kk > 0 ? 1u : 0u);
        mma_commit(dpt_full);
        const uint32_t acc = it > 0 ? 1u : 0u;
        // P^T / dS^T of queries 64g .. 64g+63 sit in columns 64g .. 64g+31 of
        // their buffer (warpgroup g wrote them over scores it had read).
        if (!mbar_wait(p_full, it & 1, abort_flag)) { ok = false; break; }
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < BLOCK / 16; ++kk)  // dV += P^T dO_i
          mma_bf16_ts(tdV, tSt + (kk >> 2) * 64 + (kk & 3) * 8, dodM0 + soff + moff(kk),
                      IDESC_ACC, (acc | kk) ? 1u : 0u);
        // dS^T (tensor memory) and dS (shared memory) are ready.
        if (!mbar_wait(ds_full, it & 1, abort_flag)) { ok = false; break; }
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < BLOCK / 16; ++kk)  // dK += dS^T Q_i
          mma_bf16_ts(tdK, tdPt + (kk >> 2) * 64 + (kk & 3) * 8, qdM0 + soff + moff(kk),
                      IDESC_ACC, (acc | kk) ? 1u : 0u);
#pragma unroll
        for (int kk = 0; kk < BLOCK / 16; ++kk)  // dQ_i = dS K_j (M = queries, K = keys)
          mma_bf16_ss(tdPt, dsdM + moff(kk), kdM + moff(kk), IDESC_DQ, kk > 0 ? 1u : 0u);
        // Q_i and dO_i (stage st) are released by the dQ warps, which
        // stage dQ_i there once it is complete.
        mma_commit(dq_full);
      }
      if (ok) mma_commit(dkv_final);
      mma_commit(mma_final);
      mbar_wait_drain(mma_final, 0);
    }
  } else if (warp < 8) {
    // ------------------------------------------------------------ P^T / dS^T
    // Warpgroup g handles queries 64g .. 64g+63 of every key row.
    const int g = warp >> 2;
    const int t = threadIdx.x - g * BLOCK;  // key row, TMEM lane
    const int key_g = key0 + t;
    const bool key_ok = key_g < geo.Nk;
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const float sl2 = p.scale_log2;
    uint8_t* ds_row = smem + L::DS_OFF + g * PANEL_BYTES + t * 128;  // row t of panel g
    const uint32_t sw = static_cast<uint32_t>(t & 7);
    bool ok = true;
    for (int it = 0; it < n_it; ++it) {
      const int st = it & 1;
      const int q0 = it_q0(it);
      const float* lse_s = reinterpret_cast<const float*>(smem + L::LSE_OFF + st * 512);
      const float* dd_s = reinterpret_cast<const float*>(smem + L::DD_OFF + st * 512);
      // Queries at or beyond Nq, and queries that see no key at all, carry
      // log2(e) * LSE = +inf in the padded table, so their P is exactly 0.
      // Causal: key row t is kept for query q of the tile iff
      // key0 + t <= q0 + q + causal_off, i.e. q >= t + delta; tiles with
      // delta <= -(BLOCK - 1) keep everything.
      const int delta = key0 - q0 - geo.off;
      const bool diag = CAUSAL && (delta > -(BLOCK - 1));
      // Phase 1: P^T = exp2(scale log2(e) S^T - log2(e) LSE) as bf16 pairs,
      // over the score columns already read; kept in registers for phase 2.
      if (!mbar_wait_warp(st_full, it & 1, abort_flag)) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t pk[32];  // P^T row t, queries 64g .. 64g+63
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int c = 64 * g + 32 * h;
        uint32_t sr[32];
        tmem_ld32(tSt + lane_off + c, sr);
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          float pv[2];
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const int q = c + e + u;
            const float pp = ex2_approx(fmaf(__uint_as_float(sr[e + u]), sl2, -lse_s[q]));
            const bool keep = key_ok && (!diag || q >= t + delta);
            pv[u] = keep ? pp : 0.f;
          }
          pk[16 * h + (e >> 1)] = pack_bf16x2(pv[0], pv[1]);
        }
        // columns 64g + 16h ..: inside the range this warpgroup has read
        tmem_st16(tSt + lane_off + 64 * g + 16 * h, &pk[16 * h]);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(p_full);
      // Phase 2: dS^T = P^T * (dP^T - D), into tensor memory over the dP^T
      // columns already read and, transposed back, into the swizzled dS
      // buffer for the dQ product.
      if (!mbar_wait_warp(dpt_full, it & 1, abort_flag)) {
        ok = false;
        break;
      }
      tc_fence_after();
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int c = 64 * g + 32 * h;
        uint32_t dr[32];
        tmem_ld32(tdPt + lane_off + c, dr);
        tmem_ld_wait();
        uint32_t dk[16];
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          const uint32_t w = pk[16 * h + (e >> 1)];
          const float d0 = __uint_as_float(w << 16) * (__uint_as_float(dr[e]) - dd_s[c + e]);
          const float d1 =
              __uint_as_float(w & 0xFFFF0000u) * (__uint_as_float(dr[e + 1]) - dd_s[c + e + 1]);
          dk[e >> 1] = pack_bf16x2(d0, d1);
        }
        tmem_st16(tdPt + lane_off + 64 * g + 16 * h, dk);
        // dS row t, queries c..c+31: panel g, 16-byte chunks (c%64)/8 .. +3,
        // 128-byte swizzle (chunk index xor row % 8).
        const uint32_t ch0 = static_cast<uint32_t>((c & 63) >> 3);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const uint32_t ch = (ch0 + u) ^ sw;
          *reinterpret_cast<uint4*>(ds_row + ch * 16) =
              make_uint4(dk[4 * u], dk[4 * u + 1], dk[4 * u + 2], dk[4 * u + 3]);
        }
      }
      fence_proxy_async_smem();
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(ds_full);
    }
    // epilogue: warpgroup 0 writes dV, warpgroup 1 scale * dK, one key row per
    // thread.  A key tile that no query sees (n_it = 0) never wrote its
    // accumulators: it stores zeros.
    if (ok && mbar_wait_warp(dkv_final, 0, abort_flag)) {
      tc_fence_after();
      const size_t rowoff = static_cast<size_t>(geo.kv_head) * p.kv_head +
                            static_cast<size_t>(geo.k0 + key_g) * p.kv_row;
      {
        const int which = g;
        const uint32_t tacc = which == 0 ? tdV : tdK;
        const bool seen = n_it > 0;
        const float mul = which == 0 ? 1.f : p.scale;
        __nv_bfloat16* dst_row = (which == 0 ? p.dv : p.dk) + rowoff;
#pragma unroll
        for (int c = 0; c < D; c += 32) {
          uint32_t r[32];
          tmem_ld32(tacc + lane_off + c, r);
          tmem_ld_wait();
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 32; e += 2)
            pk[e >> 1] = seen ? pack_bf16x2(__uint_as_float(r[e]) * mul,
                                            __uint_as_float(r[e + 1]) * mul)
                              : 0u;
          if (key_ok && dbg_ok(rowoff + c + 32 <= p.kv_elems)) {
            uint4* dst = reinterpret_cast<uint4*>(dst_row + c);
#pragma unroll
            for (int v4 = 0; v4 < 4; ++v4)
              dst[v4] = make_uint4(pk[4 * v4], pk[4 * v4 + 1], pk[4 * v4 + 2], pk[4 * v4 + 3]);
          }
        }
      }
    }
    tmem_ld_wait();
    tmem_st_wait();
  } else {
    // ------------------------------------------------------------ dQ reduction
    // dQ_i (fp32, 128 query rows x d) leaves tensor memory into the shared
    // memory of the Q_i / dO_i stage it was computed from: every MMA that
    // reads Q_i or dO_i precedes dQ_i, so the stage is free once dQ_i is
    // complete.  It is written as d/32 boxes of 128 rows x 128 bytes with the
    // 128-byte swizzle (boxes 0 .. d/64-1 over Q_i's panels, the rest over
    // dO_i's), and one thread adds them to the fp32 accumulator with bulk
    // tensor reductions (performed in L2).  dq_free is signalled as soon as
    // the tensor-memory reads are done; each half of the stage goes back to
    // the producer (q_empty, do_empty) once its reduction has read it.
    const int t = threadIdx.x - 2 * BLOCK;  // query row of the dQ tile, TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t sw = static_cast<uint32_t>(t & 7);
    constexpr int NBOX = D / 32;
    auto box_addr = [&](int st, int b) {
      return b < L::NPANEL ? smem + L::Q_OFF + st * L::TILE + b * PANEL_BYTES
                           : smem + L::DO_OFF + st * L::TILE + (b - L::NPANEL) * PANEL_BYTES;
    };
    for (int it = 0; it < n_it; ++it) {
      const int st = it & 1;
      const int q0 = it_q0(it);
      const int bh = it_head(it);
      if (!mbar_wait_warp(dq_full, it & 1, abort_flag)) break;
      tc_fence_after();
#pragma unroll
      for (int b2 = 0; b2 < NBOX; b2 += 2) {
        uint32_t r[2][32];
        tmem_ld32(tdPt + lane_off + 32 * b2, r[0]);
        tmem_ld32(tdPt + lane_off + 32 * b2 + 32, r[1]);
        tmem_ld_wait();
        if (b2 + 2 == NBOX) {
          // all of dQ_i is in registers or shared memory: the next dP^T may
          // overwrite these columns
          tc_fence_before();
          mbar_arrive(dq_free);
        }
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          uint8_t* row = box_addr(st, b2 + u) + t * 128;
#pragma unroll
          for (int c = 0; c < 8; ++c)
            *reinterpret_cast<uint4*>(row + ((c ^ sw) << 4)) =
                make_uint4(r[u][4 * c], r[u][4 * c + 1], r[u][4 * c + 2], r[u][4 * c + 3]);
        }
      }
      fence_proxy_async_smem();
      mbar_arrive(stg_full);
      if (t == 0) {
        if (!mbar_wait(stg_full, it & 1, abort_flag)) break;
        // the half over Q_i first, as its own group: Q_{i+2} is needed first
#pragma unroll
        for (int b = 0; b < L::NPANEL; ++b)
          reduce_rows<VARLEN>(&tm_dq, box_addr(st, b), 32 * b, geo.q0 + q0, bh);
        bulk_commit_group();
#pragma unroll
        for (int b = L::NPANEL; b < NBOX; ++b)
          reduce_rows<VARLEN>(&tm_dq, box_addr(st, b), 32 * b, geo.q0 + q0, bh);
        bulk_commit_group();
        bulk_wait_group_read1();
        mbar_arrive(&q_empty[st]);   // Q_i's stage may be reloaded
        bulk_wait_group_read0();
        mbar_arrive(&do_empty[st]);  // dO_i's stage may be reloaded
      }
    }
    if (t == 0) {
      bulk_wait_group0();
      if (!VARLEN && p.done_cnt != nullptr) {
        // this CTA's reductions have completed: publish them
        fence_proxy_async_global();
        __threadfence();
        atomicAdd(p.done_cnt + geo.kv_head, 1u);
      }
    }
    tmem_ld_wait();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 13) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

// For every padded row (bh, n), n < Np: D = sum_k dO_k O_k and
// lse2 = log2(e) * LSE when n < N, else D = 0 and lse2 = +inf; dQacc = 0;
// and the n_cnt completion counters = 0.  A row whose LSE is -inf saw no
// key; its lse2 is +inf as well, so that every P of it is exactly 0.
template <int D>
__global__ void __launch_bounds__(256)
    fa_bwd_preprocess_kernel(const __nv_bfloat16* __restrict__ o,
                             const __nv_bfloat16* __restrict__ dout,
                             const float* __restrict__ lse, float* __restrict__ dd,
                             float* __restrict__ lse2, float* __restrict__ dqacc,
                             unsigned* __restrict__ cnt, int n_cnt, int N, int Np,
                             long long padded_rows) {
  // the main kernel may start its set-up now; it waits for this grid's
  // completion before it reads anything written here
  griddep_launch_dependents();
  {
    const long long gi = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (gi < n_cnt) cnt[gi] = 0u;
  }
  constexpr int LPR = D / 8;     // lanes per row, 16 bytes each
  constexpr int RPW = 32 / LPR;  // rows per warp
  const int lane = threadIdx.x & 31;
  const long long warp_g = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const long long prow = warp_g * RPW + lane / LPR;
  const int sub = lane % LPR;
  const long long bh = prow / Np;
  const int n = static_cast<int>(prow - bh * Np);
  const bool real = prow < padded_rows && n < N;
  const long long row = bh * N + n;
  float acc = 0.f;
  if (real) {
    const uint4 a = *reinterpret_cast<const uint4*>(o + row * D + sub * 8);
    const uint4 b = *reinterpret_cast<const uint4*>(dout + row * D + sub * 8);
    const uint32_t wa[4] = {a.x, a.y, a.z, a.w}, wb[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      acc = fmaf(__uint_as_float(wa[i] << 16), __uint_as_float(wb[i] << 16), acc);
      acc = fmaf(__uint_as_float(wa[i] & 0xFFFF0000u), __uint_as_float(wb[i] & 0xFFFF0000u), acc);
    }
    float4* z = reinterpret_cast<float4*>(dqacc + row * D + sub * 8);
    z[0] = make_float4(0.f, 0.f, 0.f, 0.f);
    z[1] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
#pragma unroll
  for (int off = LPR / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if (prow < padded_rows && sub == 0) {
    dd[prow] = real ? acc : 0.f;
    const float l = real ? lse[row] : INFINITY;
    lse2[prow] = (l == -INFINITY) ? INFINITY : l * LOG2E;
  }
}

// Ragged batch: the same tables over [H, P] with the rows of sequence b
// starting at table_row0(cu_q[b], b); rows outside every sequence hold D = 0
// and lse2 = +inf.  (dQacc is zeroed separately.)
template <int D>
__global__ void __launch_bounds__(256)
    fa_bwd_preprocess_varlen_kernel(const __nv_bfloat16* __restrict__ o,
                                    const __nv_bfloat16* __restrict__ dout,
                                    const float* __restrict__ lse, float* __restrict__ dd,
                                    float* __restrict__ lse2, const int* __restrict__ cu_q, int B,
                                    int H, int total_q, long long P) {
  griddep_launch_dependents();
  constexpr int LPR = D / 8;     // lanes per row, 16 bytes each
  constexpr int RPW = 32 / LPR;  // rows per warp
  const int lane = threadIdx.x & 31;
  const long long warp_g = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const long long prow_g = warp_g * RPW + lane / LPR;  // over H * P
  const int sub = lane % LPR;
  const bool in = prow_g < static_cast<long long>(H) * P;
  const int h = in ? static_cast<int>(prow_g / P) : 0;
  const long long prow = in ? prow_g - static_cast<long long>(h) * P : 0;
  // the sequence whose segment holds prow: the last b with table_row0(b) <= prow
  int lo = 0, hi = B - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (table_row0(cu_q[mid], mid) <= prow) lo = mid;
    else hi = mid - 1;
  }
  const int b = lo;
  const long long n = prow - table_row0(cu_q[b], b);
  const int q0 = cu_q[b], q1 = cu_q[b + 1];
  const bool real = in && q0 >= 0 && q1 >= q0 && q1 <= total_q && n >= 0 && n < q1 - q0;
  const long long tok = q0 + n;
  float acc = 0.f;
  if (real) {
    const size_t off = (static_cast<size_t>(tok) * H + h) * D + sub * 8;
    const uint4 a = *reinterpret_cast<const uint4*>(o + off);
    const uint4 c = *reinterpret_cast<const uint4*>(dout + off);
    const uint32_t wa[4] = {a.x, a.y, a.z, a.w}, wc[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      acc = fmaf(__uint_as_float(wa[i] << 16), __uint_as_float(wc[i] << 16), acc);
      acc = fmaf(__uint_as_float(wa[i] & 0xFFFF0000u), __uint_as_float(wc[i] & 0xFFFF0000u), acc);
    }
  }
#pragma unroll
  for (int off = LPR / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if (in && sub == 0) {
    const float l = real ? lse[static_cast<size_t>(h) * total_q + tok] : INFINITY;
    dd[prow_g] = real ? acc : 0.f;
    lse2[prow_g] = (l == -INFINITY) ? INFINITY : l * LOG2E;
  }
}

// Bounded wait until *c >= need (acquire); false at once if the device error
// word is set (a CTA of the main kernel gave up, so the count may never be
// reached), and after the time limit, with FA_ERR_TIMEOUT recorded.
__device__ __forceinline__ bool wait_counter(const unsigned* c, unsigned need) {
  const uint64_t t0 = globaltimer_ns();
  for (;;) {
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(c) : "memory");
    if (v >= need) return true;
    if (*static_cast<volatile int*>(&g_device_error) != 0) return false;
    if (globaltimer_ns() - t0 > FA_WAIT_TIMEOUT_NS) {
      record_error(5 /* FA_ERR_TIMEOUT */);
      return false;
    }
    __nanosleep(256);
  }
}

// dQ = scale * dQacc in bf16, 8 elements per thread.  Without counters the
// grid covers all n8 groups of 8 elements.  With counters (done_cnt set) the
// grid is (groups of one head / 256, B * H): a CTA converts part of query
// head blockIdx.y once the counter of its key/value head, blockIdx.y /
// group, has reached `need` (every CTA of the main kernel for that head has
// finished adding into the accumulator).
__global__ void __launch_bounds__(256)
    fa_bwd_dq_convert_kernel(const float* __restrict__ dqacc, __nv_bfloat16* __restrict__ dq,
                             long long n8, float scale, const unsigned* __restrict__ done_cnt,
                             unsigned need, int group, long long head8) {
  long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (done_cnt != nullptr) {
    __shared__ int ready;
    if (threadIdx.x == 0) ready = wait_counter(done_cnt + blockIdx.y / group, need) ? 1 : 0;
    __syncthreads();
    if (!ready || i >= head8) return;
    i += static_cast<long long>(blockIdx.y) * head8;
  }
  if (i >= n8) return;
  const float4 a = __ldcg(reinterpret_cast<const float4*>(dqacc) + 2 * i);
  const float4 b = __ldcg(reinterpret_cast<const float4*>(dqacc) + 2 * i + 1);
  reinterpret_cast<uint4*>(dq)[i] =
      make_uint4(pack_bf16x2(a.x * scale, a.y * scale), pack_bf16x2(a.z * scale, a.w * scale),
                 pack_bf16x2(b.x * scale, b.y * scale), pack_bf16x2(b.z * scale, b.w * scale));
}

template <int D, bool CAUSAL, bool VARLEN>
fa_status launch_main(const CUtensorMap* maps, const Params& prm, int BH, cudaStream_t stream) {
  auto kern = fa_bwd_kernel<D, CAUSAL, VARLEN>;
  static SmemOptIn opt_in;  // one per instantiation of this kernel
  if (const fa_status st = opt_in.ensure(kern, Smem<D>::ALLOC); st != FA_OK) return st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(prm.n_kt * BH);
  cfg.blockDim = dim3(NUM_THREADS);
  cfg.dynamicSmemBytes = Smem<D>::ALLOC;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  main_kernel_begin(stream);
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, maps[0], maps[1], maps[2], maps[3], maps[4],
                                           maps[5], maps[6], prm);
  main_kernel_end(stream);
  if (e != cudaSuccess) {
    (void)cudaGetLastError();
    return FA_ERR_CUDA;
  }
  return cuda_status(cudaGetLastError());
}

}  // namespace bwd

fa_status launch_bwd(const void* q, const void* k, const void* v, const void* o,
                     const void* dout, const float* lse, void* dq, void* dk, void* dv,
                     void* workspace, int B, int H, int Hkv, int Nq, int Nk, int d, int causal,
                     float scale, cudaStream_t stream) {
  const int BH = B * H;
  const int BHkv = B * Hkv;
  // No queries: no gradient reaches K or V.  No keys: O was 0 whatever Q was.
  if (Nq == 0 || Nk == 0) {
    if (Nq == 0 && Nk > 0) {
      const size_t kv = static_cast<size_t>(BHkv) * Nk * d * 2;
      if (cudaMemsetAsync(dk, 0, kv, stream) != cudaSuccess ||
          cudaMemsetAsync(dv, 0, kv, stream) != cudaSuccess)
        return FA_ERR_CUDA;
    }
    if (Nk == 0 && Nq > 0 &&
        cudaMemsetAsync(dq, 0, static_cast<size_t>(BH) * Nq * d * 2, stream) != cudaSuccess)
      return FA_ERR_CUDA;
    return FA_OK;
  }
  const long long rows = static_cast<long long>(BH) * Nq;
  const int Np = static_cast<int>(bwd_row_pad(Nq));
  const long long prows = static_cast<long long>(BH) * Np;
  const size_t table = align_up(static_cast<size_t>(prows) * 4, 256);
  float* dd = static_cast<float*>(workspace);
  float* lse2 = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + table);
  float* dqacc = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + 2 * table);
  unsigned* done_cnt = reinterpret_cast<unsigned*>(
      static_cast<uint8_t*>(workspace) + 2 * table +
      align_up(static_cast<size_t>(rows) * d * sizeof(float), 256));
  // the conversion's grid has one row of CTAs per query head
  const bool counted = BH <= 65535;
  // 1. D, log2(e) * LSE (padded tables), the zeroed accumulator and counters
  {
    const int rows_per_block = (256 / 32) * (32 / (d / 8));
    const long long blocks = (prows + rows_per_block - 1) / rows_per_block;
    if (d == 128)
      bwd::fa_bwd_preprocess_kernel<128><<<static_cast<unsigned>(blocks), 256, 0, stream>>>(
          static_cast<const __nv_bfloat16*>(o), static_cast<const __nv_bfloat16*>(dout), lse, dd,
          lse2, dqacc, done_cnt, counted ? BHkv : 0, Nq, Np, prows);
    else
      bwd::fa_bwd_preprocess_kernel<64><<<static_cast<unsigned>(blocks), 256, 0, stream>>>(
          static_cast<const __nv_bfloat16*>(o), static_cast<const __nv_bfloat16*>(dout), lse, dd,
          lse2, dqacc, done_cnt, counted ? BHkv : 0, Nq, Np, prows);
    if (cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;
  }
  // 2. dK, dV and the dQ accumulation
  CUtensorMap maps[7];
  fa_status st;
  if ((st = make_tmap_bf16_3d(&maps[0], q, d, Nq, BH, bwd::BLOCK)) != FA_OK) return st;
  if ((st = make_tmap_bf16_3d(&maps[1], k, d, Nk, BHkv, bwd::BLOCK)) != FA_OK) return st;
  if ((st = make_tmap_bf16_3d(&maps[2], v, d, Nk, BHkv, bwd::BLOCK)) != FA_OK) return st;
  if ((st = make_tmap_bf16_3d(&maps[3], dout, d, Nq, BH, bwd::BLOCK)) != FA_OK) return st;
  if ((st = make_tmap_f32_2d(&maps[4], lse2, Np, BH)) != FA_OK) return st;
  if ((st = make_tmap_f32_2d(&maps[5], dd, Np, BH)) != FA_OK) return st;
  if ((st = make_tmap_f32_3d_sw128(&maps[6], dqacc, d, Nq, BH)) != FA_OK) return st;
  bwd::Params prm;
  prm.dk = static_cast<__nv_bfloat16*>(dk);
  prm.dv = static_cast<__nv_bfloat16*>(dv);
  prm.dqacc = dqacc;
  prm.Nq = Nq;
  prm.Nk = Nk;
  prm.causal_off = Nk - Nq;
  prm.n_qt = (Nq + bwd::BLOCK - 1) / bwd::BLOCK;
  prm.n_kt = (Nk + bwd::BLOCK - 1) / bwd::BLOCK;
  prm.group = H / Hkv;
  prm.BHkv = BHkv;
  {
    // Causal CTAs differ in length (later key tiles see fewer query tiles);
    // when there are only a few waves of them, launching the longest first
    // shortens the tail.  fa_set_schedule can force either order.
    const int mode = g_bwd_order.load(std::memory_order_relaxed);
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return FA_ERR_CUDA;
    const long long ctas = static_cast<long long>(prm.n_kt) * BHkv;
    prm.lpt_order = (mode == FA_SCHEDULE_PERSISTENT || (mode == FA_SCHEDULE_AUTO && causal && ctas < 8LL * sms)) ? 1 : 0;
  }
  prm.scale_log2 = scale * bwd::LOG2E;
  prm.scale = scale;
  prm.cu_q = nullptr;
  prm.cu_k = nullptr;
  prm.Hkv = Hkv;
  prm.total_q = 0;
  prm.total_k = 0;
  prm.kv_head = static_cast<size_t>(Nk) * d;
  prm.kv_row = static_cast<size_t>(d);
  prm.kv_elems = static_cast<size_t>(BHkv) * Nk * d;
  prm.done_cnt = counted ? done_cnt : nullptr;
  if (d == 128)
    st = causal ? bwd::launch_main<128, true, false>(maps, prm, BHkv, stream)
                : bwd::launch_main<128, false, false>(maps, prm, BHkv, stream);
  else
    st = causal ? bwd::launch_main<64, true, false>(maps, prm, BHkv, stream)
                : bwd::launch_main<64, false, false>(maps, prm, BHkv, stream);
  if (st != FA_OK) return st;
  // 3. dQ = scale * accumulator, head by head as the main kernel finishes
  // them (programmatic launch: the grid may start before the main kernel
  // ends; each CTA waits on its head's counter)
  {
    const long long n8 = rows * d / 8;
    const long long head8 = static_cast<long long>(Nq) * d / 8;
    const float* acc = dqacc;
    __nv_bfloat16* out = static_cast<__nv_bfloat16*>(dq);
    cudaError_t e;
    if (counted) {
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
      attr[0].val.programmaticStreamSerializationAllowed = 1;
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(static_cast<unsigned>((head8 + 255) / 256), static_cast<unsigned>(BH));
      cfg.blockDim = dim3(256);
      cfg.stream = stream;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      e = cudaLaunchKernelEx(&cfg, bwd::fa_bwd_dq_convert_kernel, acc, out, n8, scale,
                             static_cast<const unsigned*>(done_cnt),
                             static_cast<unsigned>(prm.n_kt), H / Hkv, head8);
    } else {
      const long long blocks = (n8 + 255) / 256;
      bwd::fa_bwd_dq_convert_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(
          acc, out, n8, scale, nullptr, 0u, 1, 0LL);
      e = cudaGetLastError();
    }
    if (e != cudaSuccess) {
      (void)cudaGetLastError();
      return FA_ERR_CUDA;
    }
  }
  return FA_OK;
}

size_t bwd_varlen_table_rows(int B, int total_q) {
  return static_cast<size_t>(bwd::table_row0(total_q, B));  // a multiple of 4
}

fa_status launch_bwd_varlen(const void* q, const void* k, const void* v, const void* o,
                            const void* dout, const float* lse, void* dq, void* dk, void* dv,
                            const int* cu_q, const int* cu_k, void* workspace, int B, int H,
                            int Hkv, int total_q, int total_k, int max_seqlen_k, int d,
                            int causal, float scale, cudaStream_t stream) {
  // No queries anywhere: no gradient reaches K or V.  No keys: dQ = 0.
  if (total_q == 0 || total_k == 0 || max_seqlen_k == 0) {
    if (total_k > 0) {
      const size_t kv = static_cast<size_t>(total_k) * Hkv * d * 2;
      if (cudaMemsetAsync(dk, 0, kv, stream) != cudaSuccess ||
          cudaMemsetAsync(dv, 0, kv, stream) != cudaSuccess)
        return FA_ERR_CUDA;
    }
    if (total_q > 0 &&
        cudaMemsetAsync(dq, 0, static_cast<size_t>(total_q) * H * d * 2, stream) != cudaSuccess)
      return FA_ERR_CUDA;
    return FA_OK;
  }
  const long long P = static_cast<long long>(bwd_varlen_table_rows(B, total_q));
  const size_t table = align_up(static_cast<size_t>(H) * P * 4, 256);
  float* dd = static_cast<float*>(workspace);
  float* lse2 = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + table);
  float* dqacc = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + 2 * table);
  const size_t dq_elems = static_cast<size_t>(total_q) * H * d;
  // Key rows of a sequence that no query sees get dK = dV = 0 from the main
  // kernel; key rows outside every sequence are never written: clear all.
  if (cudaMemsetAsync(dqacc, 0, dq_elems * 4, stream) != cudaSuccess ||
      cudaMemsetAsync(dk, 0, static_cast<size_t>(total_k) * Hkv * d * 2, stream) != cudaSuccess ||
      cudaMemsetAsync(dv, 0, static_cast<size_t>(total_k) * Hkv * d * 2, stream) != cudaSuccess)
    return FA_ERR_CUDA;
  // 1. D and log2(e) * LSE in per-sequence padded segments
  {
    const int rows_per_block = (256 / 32) * (32 / (d / 8));
    const long long prows = static_cast<long long>(H) * P;
    const long long blocks = (prows + rows_per_block - 1) / rows_per_block;
    if (d == 128)
      bwd::fa_bwd_preprocess_varlen_kernel<128><<<static_cast<unsigned>(blocks), 256, 0, stream>>>(
          static_cast<const __nv_bfloat16*>(o), static_cast<const __nv_bfloat16*>(dout), lse, dd,
          lse2, cu_q, B, H, total_q, P);
    else
      bwd::fa_bwd_preprocess_varlen_kernel<64><<<static_cast<unsigned>(blocks), 256, 0, stream>>>(
          static_cast<const __nv_bfloat16*>(o), static_cast<const __nv_bfloat16*>(dout), lse, dd,
          lse2, cu_q, B, H, total_q, P);
    if (cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;
  }
  // 2. dK, dV and the dQ accumulation, token-major maps
  CUtensorMap maps[7];
  fa_status st;
  if ((st = make_tmap_bf16_rows_heads(&maps[0], q, d, H, total_q, bwd::BLOCK)) != FA_OK) return st;
  if ((st = make_tmap_bf16_rows_heads(&maps[1], k, d, Hkv, total_k, bwd::BLOCK)) != FA_OK) return st;
  if ((st = make_tmap_bf16_rows_heads(&maps[2], v, d, Hkv, total_k, bwd::BLOCK)) != FA_OK) return st;
  if ((st = make_tmap_bf16_rows_heads(&maps[3], dout, d, H, total_q, bwd::BLOCK)) != FA_OK)
    return st;
  if ((st = make_tmap_f32_2d(&maps[4], lse2, P, H)) != FA_OK) return st;
  if ((st = make_tmap_f32_2d(&maps[5], dd, P, H)) != FA_OK) return st;
  if ((st = make_tmap_f32_rows_heads_sw128(&maps[6], dqacc, d, H, total_q)) != FA_OK) return st;
  bwd::Params prm;
  prm.dk = static_cast<__nv_bfloat16*>(dk);
  prm.dv = static_cast<__nv_bfloat16*>(dv);
  prm.dqacc = dqacc;
  prm.Nq = prm.Nk = prm.causal_off = prm.n_qt = 0;
  prm.n_kt = (max_seqlen_k + bwd::BLOCK - 1) / bwd::BLOCK;
  prm.group = H / Hkv;
  prm.BHkv = B * Hkv;
  prm.lpt_order = 0;  // head-major: a sequence's key tiles adjacent
  prm.scale_log2 = scale * bwd::LOG2E;
  prm.scale = scale;
  prm.cu_q = cu_q;
  prm.cu_k = cu_k;
  prm.Hkv = Hkv;
  prm.total_q = total_q;
  prm.total_k = total_k;
  prm.kv_head = static_cast<size_t>(d);
  prm.kv_row = static_cast<size_t>(Hkv) * d;
  prm.kv_elems = static_cast<size_t>(total_k) * Hkv * d;
  prm.done_cnt = nullptr;
  if (static_cast<long long>(prm.n_kt) * prm.BHkv > 0x7fffffffLL) return FA_ERR_INVALID_ARG;
  if (d == 128)
    st = causal ? bwd::launch_main<128, true, true>(maps, prm, prm.BHkv, stream)
                : bwd::launch_main<128, false, true>(maps, prm, prm.BHkv, stream);
  else
    st = causal ? bwd::launch_main<64, true, true>(maps, prm, prm.BHkv, stream)
                : bwd::launch_main<64, false, true>(maps, prm, prm.BHkv, stream);
  if (st != FA_OK) return st;
  // 3. dQ = scale * accumulator (same element order as dq)
  {
    const long long n8 = static_cast<long long>(dq_elems / 8);
    const long long blocks = (n8 + 255) / 256;
    bwd::fa_bwd_dq_convert_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(
        dqacc, static_cast<__nv_bfloat16*>(dq), n8, scale, nullptr, 0u, 1, 0LL);
    if (cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;
  }
  return FA_OK;
}

}  // namespace fa
