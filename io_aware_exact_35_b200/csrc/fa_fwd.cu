// fa_fwd.cu - forward pass of exact attention on sm_100a.
//
// One CTA computes two 128-row query tiles (256 consecutive rows) of one
// (batch, head):
//   O_i = softmax(scale * Q_i K^T [+ causal mask]) V,   LSE_i = ln sum_j exp(...)
// following the tile recurrence of "DL101 chapter 9" (handsonai.io), section
// 3.3: over key tiles j, S = Q_i K_j^T; m' = max(m, rowmax S); P = exp(S - m');
// c = exp(m - m'); l' = l c + rowsum P; O' = O c + P V_j; finally O / l.
// The five stages of "What is FlashAttention" (unite.ai, five-stage
// operational map) map onto the warp roles below: partition into tiles and
// load them on chip (TMA producer warp), local scores and running
// normalisation (MMA warp + softmax warpgroups), accumulate without the full
// matrix (MMA warp, O in tensor memory), and the kernel schedule (grid order).
//
// Warp roles (512 threads, four warpgroups; registers are moved between the
// warpgroups with setmaxnreg so that the softmax gets most of them):
//   warps 0-3  softmax warpgroup 0: thread t owns row t of query tile 0.
//   warps 4-7  softmax warpgroup 1: the same for query tile 1.
//              Each reads its S from tensor memory, masks, keeps the running
//              max m and sum l (log2 domain), writes P as bf16 into the same
//              tensor-memory columns, rescales its O when m grows, and at the
//              end of a work item writes LSE and hands 1 / l to the epilogue.
//   warps 8-11 epilogue warpgroup: once a tile's last O += P V has completed
//              it reads O out of tensor memory (thread t: row t), multiplies
//              by 1 / l and stores bf16 rows, while the softmax warpgroups
//              already work on the next item.
//   warp 12    TMA producer: the query pair of each work item, then K_j and
//              V_j through one ring of NSLOT tile-sized slots that holds K and
//              V tiles in the order they are consumed (K_0 V_0 K_1 V_1 ...), so
//              loads run about two key tiles ahead of the tensor core.
//   warp 13    tensor-memory allocator and MMA issuer (the whole warp runs
//              converged; elect.sync picks the lane that issues).  The two
//              query tiles ping-pong: while warpgroup 0 exponentiates S_0,j the
//              tensor core runs O_1 += P_1 V_{j-1} and S_1,j, and vice versa:
//                S0(0) S1(0) | PV0(0) S0(1) PV1(0) S1(1) | PV0(1) S0(2) ...
//              Since S_w(j+1) is written over the columns that hold P_w(j), it
//              follows O_w += P_w(j) V_j: per tile, softmax, P V and the next
//              S run in series, and the two tiles overlap their chains.
//   warps 14-15 idle (they complete the fourth warpgroup).
//
// Tensor memory (512 columns x 128 lanes, fp32): S_0 [0,128), S_1 [128,256),
// O_0 [256,384), O_1 [384,512).  P_w overwrites the first 64 columns of S_w
// (two bf16 per column) and is read from there by the P V MMA.
//
// The softmax keeps a stale maximum until a row's maximum grows by more than
// 2^8: P may then exceed 1 by up to 256x, which bf16 / fp32 hold just as well,
// and O and l are only rescaled (a tensor-memory round trip) when the maximum
// really moves.  Both l and O always refer to the same maximum, so the final
// O / l is unchanged.
#include <algorithm>
#include <cstdlib>
#include <cstring>

#include "fa_internal.h"
#include "sm100.cuh"

namespace fa {

// ---- 8-bit float (e4m3) helpers of the FP8 forward
// D (f32, tensor memory) (+)= A B^T with 8-bit float operands, both from
// shared memory (kind::f8f6f4: K = 32 per instruction, 32 bytes per row).
__device__ __forceinline__ void mma_f8_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Instruction descriptor for kind::f8f6f4: f32 accumulator, A and B e4m3
// (format code 0), both K-major, M x N.
__host__ __device__ constexpr uint32_t idesc_e4m3_f32(int M, int N) {
  return (1u << 4)                                   // D: f32
         | (static_cast<uint32_t>(N >> 3) << 17)      // N / 8
         | (static_cast<uint32_t>(M >> 4) << 24);     // M / 16
}

// Four float32 values rounded to e4m3 (round to nearest even, saturating to
// +-448), packed little-endian: x0 in the lowest byte.
__device__ __forceinline__ uint32_t pack_e4m3x4(float x0, float x1, float x2, float x3) {
  uint32_t r;
  asm("{\n\t.reg .b16 lo, hi;\n\t"
      "cvt.rn.satfinite.e4m3x2.f32 lo, %2, %1;\n\t"
      "cvt.rn.satfinite.e4m3x2.f32 hi, %4, %3;\n\t"
      "mov.b32 %0, {lo, hi};\n\t}"
      : "=r"(r)
      : "f"(x0), "f"(x1), "f"(x2), "f"(x3));
  return r;
}

// The same three tensor-core operations issued by a converged warp: every
// lane holds the same (warp-uniform) operands and elect.sync picks the one
// lane that issues, so the operands can stay in uniform registers.
__device__ __forceinline__ void mma_bf16_ss_w(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                              uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void mma_bf16_ts_w(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                              uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void mma_f8_ss_w(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                            uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void mma_commit_w(uint64_t* bar) {
  asm volatile(
      "{\n\t.reg .pred e;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}" ::"r"(
          smem_u32(bar))
      : "memory");
}

namespace fwd {

constexpr int TILE_M = 128;   // rows per softmax warpgroup
constexpr int NQ = 2;         // query tiles per CTA
constexpr int BLOCK_M = TILE_M * NQ;
constexpr int BLOCK_N = 128;
constexpr int NUM_THREADS = 512;
constexpr int WARP_PRODUCER = 12;
constexpr int WARP_MMA = 13;
// Registers per thread after setmaxnreg (launch: 65536 / 512 = 128 each):
// 2 x 128 x 184 + 128 x 48 + 128 x 96 = 65536.  The producer / MMA warpgroup
// needs 96: its issue loops are fully unrolled with precomputed descriptors,
// because the issue of a tensor-core instruction waits until the tensor pipe
// accepts it, so any instruction between two of them lengthens every step
// (measured: rolled loops made the forward 12% slower).
constexpr int REGS_SOFTMAX = 184;
constexpr int REGS_EPILOGUE = 48;
constexpr int REGS_OTHER = 96;
static_assert(2 * 128 * REGS_SOFTMAX + 128 * REGS_EPILOGUE + 128 * REGS_OTHER <= 65536,
              "setmaxnreg.inc would wait forever: the split exceeds the launch's registers");
constexpr int PANEL_BYTES = 128 * 128;   // 128 rows x 64 bf16 (one swizzle panel)
constexpr uint32_t TMEM_COLS = 512;
constexpr float RESCALE_THRESHOLD = 8.0f;  // log2 units

// Two f32 values as one 64-bit operand of the packed f32x2 instructions
// (sm_100), and (x0, x1) = (a0, a1) * b + c lane by lane.  ftz, as the
// scalar FFMA it replaces under fast-math.
__device__ __forceinline__ uint64_t pack_f32x2(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void fma_f32x2(float& x0, float& x1, float a0, float a1, uint64_t b,
                                          uint64_t c) {
  uint64_t d;
  asm("fma.rn.ftz.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(pack_f32x2(a0, a1)), "l"(b), "l"(c));
  asm("mov.b64 {%0, %1}, %2;" : "=f"(x0), "=f"(x1) : "l"(d));
}
// 32 lanes x 8 consecutive 32-bit columns of tensor memory (load / store).
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, uint32_t (&r)[8]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
                 "=r"(r[6]), "=r"(r[7])
               : "r"(taddr));
}
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t (&r)[8]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};"
               ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]),
                 "r"(r[6]), "r"(r[7])
               : "memory");
}

// The softmax signals "P ready" with one arrival per warp (after the warp's
// lanes have synchronised), not one per thread: 4 arrivals per step instead
// of 128 on the same barrier.
constexpr int P_ARRIVALS = TILE_M / 32;
constexpr int MAX_CHAINS = 4;  // independent chains of the row maximum

// acc += (a0, a1) lane by lane, one packed f32x2 addition.
__device__ __forceinline__ void add_f32x2(uint64_t& acc, float a0, float a1) {
  asm("add.rn.ftz.f32x2 %0, %0, %1;" : "+l"(acc) : "l"(pack_f32x2(a0, a1)));
}
__device__ __forceinline__ float sum_f32x2(uint64_t v) {
  float a, b;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(v));
  return a + b;
}

// max(a, b, c) in one instruction (three-input max.f32, sm_100).  Inputs
// here are finite or -inf, never NaN.
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}
// 2^x0, 2^x1 on the FMA pipe, two lanes per packed f32x2 instruction: the
// cubic of ex2_poly3 (sm100.cuh; Remez fit of
// io_aware_exact_35_b200/exp2_poly.py) evaluated on the pair.  Inputs are
// clamped at -125 (so masked scores must not come here).
__device__ __forceinline__ void ex2_poly3_x2(float x0, float x1, float& y0, float& y1) {
  const uint64_t x = pack_f32x2(fmaxf(x0, -125.f), fmaxf(x1, -125.f));
  const uint64_t magic = pack_f32x2(12582912.f, 12582912.f);  // 1.5 * 2^23
  uint64_t t, n, f, q;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(t) : "l"(x), "l"(magic));  // x rounded into t's mantissa
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(n) : "l"(t), "l"(magic));  // n = round(x)
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(f) : "l"(x), "l"(n));      // f in [-1/2, 1/2]
  asm("fma.rn.f32x2 %0, %1, %2, %3;"
      : "=l"(q) : "l"(pack_f32x2(kEx2C3, kEx2C3)), "l"(f), "l"(pack_f32x2(kEx2C2, kEx2C2)));
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(q) : "l"(q), "l"(f), "l"(pack_f32x2(kEx2C1, kEx2C1)));
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(q) : "l"(q), "l"(f), "l"(pack_f32x2(kEx2C0, kEx2C0)));
  float q0, q1, t0, t1;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(q0), "=f"(q1) : "l"(q));
  asm("mov.b64 {%0, %1}, %2;" : "=f"(t0), "=f"(t1) : "l"(t));
  // n sits in the low mantissa bits of t: shifting it into the exponent
  // field multiplies 2^f by 2^n
  y0 = __int_as_float(__float_as_int(q0) + (__float_as_int(t0) << 23));
  y1 = __int_as_float(__float_as_int(q1) + (__float_as_int(t1) << 23));
}

#ifndef FA_FWD_EMU_PAIRS
#define FA_FWD_EMU_PAIRS 0
#endif
constexpr int EMU_PAIRS = FA_FWD_EMU_PAIRS;  // of every 4 exp pairs, on the FMA pipe

// Shared-memory plan.  A panel is 128 rows x 128 bytes (64 bf16 or 128 e4m3
// values per row).  With 8-bit inputs (F8) the ring carries K_j and V_j^T
// tiles, and P_w goes through shared memory (the 8-bit product reads both
// operands from there).
template <int D, bool F8 = false>
struct Smem {
  static constexpr int NPANEL = F8 ? D / 128 : D / 64;
  static constexpr int TILE = NPANEL * PANEL_BYTES;  // 128 rows x D elements
  static constexpr int NSLOT = 5;                    // K/V ring slots
  static constexpr int Q_OFF = 0;                    // NQ tiles
  static constexpr int RING_OFF = NQ * TILE;
  static constexpr int P_OFF = RING_OFF + NSLOT * TILE;  // F8: NQ tiles of 128 x 128 e4m3
  static constexpr int BAR_OFF = P_OFF + (F8 ? NQ * PANEL_BYTES : 0);
  // barriers: q_full, q_empty, full[NSLOT], empty[NSLOT],
  //           s_full[NQ], p_full[NQ], o_final[NQ], o_free[NQ], mma_final,
  //           l_ready[NQ][2]
  static constexpr int NBAR = 2 + 2 * NSLOT + 4 * NQ + 1 + 2 * NQ;
  // 1 / l of every row, per query tile, for work items of even / odd index
  static constexpr int STAT_OFF = BAR_OFF + NBAR * 8;
  static constexpr int MISC_OFF = STAT_OFF + 2 * NQ * TILE_M * 4;
  static constexpr int BYTES = MISC_OFF + 16;
  // at least 116 KB so that a single CTA (and its 512 tensor-memory columns)
  // occupies an SM.
  static constexpr int ALLOC = BYTES > 118784 ? BYTES : 118784;
};

struct Params {
  __nv_bfloat16* o;
  float* lse;
  int Nq;            // query rows per head (padded layout)
  int Nk;            // key / value rows per head (padded layout)
  int causal_off;    // Nk - Nq: query i sits at key position i + causal_off
  int BH;            // batch x query heads
  int group;         // query heads per key/value head (1 without grouping)
  int n_cta_tiles;   // 256-row tiles per (batch, head): ceil(Nq / 256), or of
                     // the longest sequence (ragged batch)
  int total_items;   // BH * n_cta_tiles
  int lpt_order;     // 1: all heads' longest tiles first; 0: head-major
  int head_band;     // head-major order: heads per band (>= 1)
  // 1: a work item is one 128-row tile of two query heads that share a
  // key/value head (grouped heads, an even group); item coordinates then count
  // head pairs and 128-row tiles.  0: two consecutive 128-row tiles of one head.
  int pair_heads;
  // with paired heads and no grouping: the two heads have their own K / V, and
  // the ring carries each tile's keys and values separately
  int kv_split;
  float scale_log2;  // scale * log2(e) (times the q and k descales for e4m3)
  float o_scale;     // multiplies O / l: 1, or the v descale for e4m3
  // ragged batch (token-major packing): sequence b owns rows cu_q[b] ..
  // cu_q[b+1]-1 of q / o and cu_k[b] .. cu_k[b+1]-1 of k / v
  const int* cu_q;
  const int* cu_k;
  int H;             // query heads
  int total_q;       // packed query rows
  int total_k;       // packed key rows
  // element strides of O and LSE: O[head][row] at head * o_head + row * o_row,
  // LSE at head * lse_head + row, with head = b*H + h (padded) or h (ragged)
  size_t o_head, o_row, lse_head;
  size_t o_elems, lse_elems;  // sizes of O and LSE, for the debug build's checks
};

// Work item -> (batch*head (or head pair), query tile).  In LPT order the longest tiles of
// every head come first (good balance; used when all K/V fit in L2).  In
// head-major order the heads go in bands of head_band adjacent heads, a
// band's tiles longest first across its heads: the resident CTAs share a
// band's K/V in L2 for long sequences, and the last CTAs to start are short
// ones (with one head per band the last head's longest tile would start
// near the end and run alone).
__device__ __forceinline__ void item_coords(const Params& p, int item, int& bh, int& tile) {
  if (p.lpt_order) {
    const int r = item / p.BH;
    bh = item - r * p.BH;
    tile = p.n_cta_tiles - 1 - r;
  } else {
    const int per = p.head_band * p.n_cta_tiles;
    const int band = item / per;
    const int in_band = item - band * per;
    const int h0 = band * p.head_band;
    const int nb = min(p.head_band, p.BH - h0);
    const int r = in_band / nb;
    bh = h0 + (in_band - r * nb);
    tile = p.n_cta_tiles - 1 - r;
  }
}

// Where a work item lives.  Rows are counted within the sequence; q0 / k0 are
// the sequence's first rows in the tensor maps (0 for the padded layout).
struct ItemGeo {
  int tile;        // query tile of the sequence (256 rows, or 128 with paired heads)
  // query tile w starts at row qrow0 + w * qstep of the sequence and has the
  // head coordinate (of Q / O / LSE) hd0 + w * hstep
  int qrow0, qstep, hd0, hstep;
  __device__ __forceinline__ int qrow(int w) const { return qrow0 + w * qstep; }
  __device__ __forceinline__ int hd(int w) const { return hd0 + w * hstep; }
  int kv_head;     // head coordinate of K / V of query tile 0
  int kv_hstep;    // ... of query tile w: kv_head + w * kv_hstep
  int q0, k0;
  int Nq, Nk, off; // lengths of the sequence and Nk - Nq
  int n_kv_total;  // key tiles of the sequence, at least 1
};

template <bool VARLEN>
__device__ __forceinline__ ItemGeo item_geo(const Params& p, int item) {
  ItemGeo g;
  int bh;
  item_coords(p, item, bh, g.tile);
  if constexpr (!VARLEN) {
    if (p.pair_heads) {
      // bh counts head pairs: heads 2i and 2i+1 of one batch row, the same
      // rows of both, one key/value head (the group is even)
      const int half = p.H >> 1;
      const int b = bh / half;
      const int h0 = b * p.H + 2 * (bh - b * half);
      g.hd0 = h0;
      g.hstep = 1;
      g.qrow0 = g.tile * TILE_M;
      g.qstep = 0;
      g.kv_head = h0 / p.group;
      g.kv_hstep = p.kv_split;  // own K / V (no grouping), or the shared head
    } else {
      g.hd0 = bh;
      g.hstep = 0;
      g.qrow0 = g.tile * BLOCK_M;
      g.qstep = TILE_M;
      g.kv_head = bh / p.group;
      g.kv_hstep = 0;
    }
    g.q0 = 0;
    g.k0 = 0;
    g.Nq = p.Nq;
    g.Nk = p.Nk;
  } else {
    const int b = bh / p.H;
    const int h = bh - b * p.H;
    g.hd0 = h;
    g.hstep = 0;
    g.qrow0 = g.tile * BLOCK_M;
    g.qstep = TILE_M;
    g.kv_head = h / p.group;
    g.kv_hstep = 0;
    g.q0 = p.cu_q[b];
    g.k0 = p.cu_k[b];
    g.Nq = p.cu_q[b + 1] - g.q0;
    g.Nk = p.cu_k[b + 1] - g.k0;
    // offsets outside the packed arrays are never used: the sequence is empty
    if (g.q0 < 0 || g.Nq < 0 || g.q0 + g.Nq > p.total_q) g.Nq = 0;
    if (g.k0 < 0 || g.Nk < 0 || g.k0 + g.Nk > p.total_k) g.Nk = 0;
  }
  g.off = g.Nk - g.Nq;
  g.n_kv_total = max(1, (g.Nk + BLOCK_N - 1) / BLOCK_N);
  return g;
}

// TMA load of 128 rows x 64 columns starting at `row` of head `head`: the
// padded maps are [heads, rows, d], the ragged ones [rows, heads, d].
template <bool VARLEN>
__device__ __forceinline__ void load_rows(void* dst, const CUtensorMap* map, uint64_t* bar, int x,
                                          int row, int head) {
  if constexpr (VARLEN)
    tma_load_3d(dst, map, bar, x, head, row);
  else
    tma_load_3d(dst, map, bar, x, row, head);
}

// The k-th work item of CTA c out of G: rounds alternate direction so that a
// CTA that drew a long item in one round draws a short one in the next.
__device__ __forceinline__ int cta_item(int c, int k, int G) {
  return k * G + ((k & 1) ? (G - 1 - c) : c);
}

// F8: q, k are e4m3 [heads, rows, d], v is given transposed, e4m3
// [heads, d, rows], so that both products read K-major tiles; P_w is rounded
// to e4m3 (P <= 2^8 < 448 under the stale-maximum rule) and the accumulators
// stay f32.
template <int D, bool CAUSAL, bool VARLEN, bool F8 = false>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    fa_fwd_kernel(const __grid_constant__ CUtensorMap tm_q,
                  const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const Params p) {
  static_assert(!F8 || (D == 128 && !VARLEN), "e4m3 inputs: d = 128, padded layout");
  using L = Smem<D, F8>;
  constexpr int XSTEP = F8 ? 128 : 64;  // columns per panel
  constexpr int NSLOT = L::NSLOT;
  extern __shared__ __align__(1024) uint8_t smem[];
  // The swizzled operand tiles need 1024-byte alignment; the kernel declares
  // no static shared memory, so the dynamic window starts aligned.
  if ((smem_u32(smem) & 1023u) != 0) {
    if (threadIdx.x == 0) record_error(2 /* FA_ERR_UNSUPPORTED */);
    return;
  }

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::BAR_OFF);
  uint64_t* q_full = bars;
  uint64_t* q_empty = bars + 1;
  uint64_t* full = bars + 2;        // [NSLOT] ring slot loaded
  uint64_t* empty = full + NSLOT;   // [NSLOT] ring slot consumed
  uint64_t* s_full = empty + NSLOT; // [NQ]
  uint64_t* p_full = s_full + NQ;   // [NQ]
  uint64_t* o_final = p_full + NQ;  // [NQ] one phase per work item: its last O += P V
  uint64_t* o_free = o_final + NQ;  // [NQ] one phase per work item: O read out
  uint64_t* mma_final = o_free + NQ;
  uint64_t* l_ready = mma_final + 1;  // [NQ][2]: 1 / l written, per item parity
  float* inv_l_buf = reinterpret_cast<float*>(smem + L::STAT_OFF);  // [2][NQ][TILE_M]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::MISC_OFF + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int G = static_cast<int>(gridDim.x);
  const int cta = static_cast<int>(blockIdx.x);
  // Key tiles seen by query tile w (128 rows) of an item; causal: up to the
  // tile holding the last admissible key of its last row.  At least one, so
  // that rows that see no key at all (Nq > Nk, or no keys) still run the
  // pipeline once and come out fully masked: O = 0, LSE = -inf.
  auto n_kv_of = [&](const ItemGeo& g, int w) {
    if (!CAUSAL) return g.n_kv_total;
    const int last_key = g.qrow(w) + TILE_M - 1 + g.off;
    return last_key < 0 ? 1 : min(last_key / BLOCK_N + 1, g.n_kv_total);
  };
  if constexpr (VARLEN) {
    // one item per CTA; tiles past the end of their sequence have no work
    const ItemGeo g = item_geo<true>(p, cta);
    if (g.tile == 0 && g.Nq > p.n_cta_tiles * BLOCK_M) {
      if (threadIdx.x == 0) record_error(1 /* FA_ERR_INVALID_ARG: max_seqlen_q too small */);
    }
    if (g.tile * BLOCK_M >= g.Nq) return;
  }

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int s = 0; s < NSLOT; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int w = 0; w < NQ; ++w) {
      mbar_init(&s_full[w], 1);
      mbar_init(&p_full[w], P_ARRIVALS);
      mbar_init(&o_final[w], 1);
      mbar_init(&o_free[w], TILE_M);
      mbar_init(&l_ready[2 * w], TILE_M);
      mbar_init(&l_ready[2 * w + 1], TILE_M);
    }
    mbar_init(mma_final, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == WARP_MMA) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == WARP_PRODUCER && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp >= 12) {
   asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(REGS_OTHER));
   if (warp == WARP_PRODUCER) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int kv = 0;        // key tiles loaded so far (all work items)
      int loaded = 0;    // ring tiles (K or V) loaded so far
      int n_items = 0;   // query pairs loaded so far
      bool ok = true;
      for (int k = 0; ok; ++k) {
        const int item = cta_item(cta, k, G);
        if (item >= p.total_items) break;
        const ItemGeo g = item_geo<VARLEN>(p, item);
        const int n_kv1 = n_kv_of(g, 1);
        // the Q pair of the previous item must have been consumed by its S MMAs
        if (k > 0 && !mbar_wait(q_empty, (k - 1) & 1, abort_flag)) break;
        mbar_arrive_expect_tx(q_full, NQ * L::TILE);
        for (int w = 0; w < NQ; ++w)
          for (int pn = 0; pn < L::NPANEL; ++pn)
            load_rows<VARLEN>(smem + L::Q_OFF + w * L::TILE + pn * PANEL_BYTES, &tm_q, q_full,
                              pn * XSTEP, g.q0 + g.qrow(w), g.hd(w));
        ++n_items;
        // one ring tile: K or V, key tile j, of key/value head kvh
        auto ring = [&](bool is_v, int j, int kvh) -> bool {
          const int u = loaded;
          const int slot = u % NSLOT;
          if (u >= NSLOT && !mbar_wait(&empty[slot], (u / NSLOT - 1) & 1, abort_flag))
            return false;
          mbar_arrive_expect_tx(&full[slot], L::TILE);
          if (F8 && is_v) {
            // V_j^T: rows d, columns keys j*128 ..
            tma_load_3d(smem + L::RING_OFF + slot * L::TILE, &tm_v, &full[slot], j * BLOCK_N, 0,
                        kvh);
          } else {
            for (int pn = 0; pn < L::NPANEL; ++pn)
              load_rows<VARLEN>(smem + L::RING_OFF + slot * L::TILE + pn * PANEL_BYTES,
                                is_v ? &tm_v : &tm_k, &full[slot], pn * XSTEP,
                                g.k0 + j * BLOCK_N, kvh);
          }
          ++loaded;
          return true;
        };
        if (!p.kv_split) {
          // both tiles read K_j and V_j: ring tiles K_0 V_0 K_1 V_1 ...
          for (int j = 0; j < n_kv1 && ok; ++j, ++kv)
            ok = ring(false, j, g.kv_head) && ring(true, j, g.kv_head);
        } else {
          // each tile has its own K / V, in the order the MMA warp takes them:
          // K0_0 K1_0 | V0_j K0_{j+1} V1_j K1_{j+1} | ...  (n0 = n1)
          const int kv0 = g.kv_head, kv1 = g.kv_head + g.kv_hstep;
          ok = ring(false, 0, kv0) && ring(false, 0, kv1);
          for (int j = 0; j < n_kv1 && ok; ++j) {
            const bool more = j + 1 < n_kv1;
            ok = ring(true, j, kv0) && (!more || ring(false, j + 1, kv0)) && ring(true, j, kv1) &&
                 (!more || ring(false, j + 1, kv1));
          }
        }
      }
      // Every copy issued must land before this CTA's shared memory is freed:
      // the last phase of each barrier that received copies.
      if (n_items > 0) mbar_wait_drain(q_full, (n_items - 1) & 1);
      for (int u = max(0, loaded - NSLOT); u < loaded; ++u)
        mbar_wait_drain(&full[u % NSLOT], (u / NSLOT) & 1);
    }
   } else if (warp == WARP_MMA) {
    // ------------------------------------------------------------ MMA issuer
    {
      // The whole warp runs the issue loop converged, and elect.sync picks
      // the lane that issues each tensor-core instruction: lane 0 alone
      // (a divergent branch) issued measurably slower.
      auto mwait = [&](uint64_t* bar, uint32_t parity) {
        return mbar_wait_warp(bar, parity, abort_flag);
      };
      auto commit = [&](uint64_t* bar) { mma_commit_w(bar); };
      constexpr uint32_t IDESC_S =
          F8 ? idesc_e4m3_f32(TILE_M, BLOCK_N) : idesc_bf16_f32(TILE_M, BLOCK_N, false, false);
      constexpr uint32_t IDESC_O =
          F8 ? idesc_e4m3_f32(TILE_M, D) : idesc_bf16_f32(TILE_M, D, false, true);
      const uint64_t p_desc0 = sdesc_kmajor_sw128(smem_u32(smem + L::P_OFF));  // F8 only
      const uint32_t q_addr = smem_u32(smem + L::Q_OFF);
      const uint32_t ring_addr = smem_u32(smem + L::RING_OFF);
      int pcount[NQ] = {0, 0};  // P tiles consumed per warpgroup (all items)

      // S_w = Q_w K^T with K in ring slot `slot`
      // Shared-memory descriptors are built once; a k-step only adds a
      // compile-time byte offset (>> 4) to the start-address field, which
      // never carries out of its 14 bits for addresses below 256 KB.  This
      // keeps the issue loop at a few instructions per MMA: the MMA warp
      // shares its scheduler with two busy softmax warps.
      const uint64_t q_desc0 = sdesc_kmajor_sw128(q_addr);
      const uint64_t ring_kdesc0 = sdesc_kmajor_sw128(ring_addr);
      const uint64_t ring_vdesc0 = sdesc_mnmajor_sw128(ring_addr, PANEL_BYTES);
      auto issue_s = [&](int w, int slot) {
        const uint64_t qd = q_desc0 + static_cast<uint64_t>((w * L::TILE) >> 4);
        const uint64_t kd = ring_kdesc0 + static_cast<uint64_t>((slot * L::TILE) >> 4);
        const uint32_t dS = tmem_base + w * 128;
        if constexpr (F8) {
#pragma unroll
          for (int kk = 0; kk < D / 32; ++kk) {  // 32 e4m3 = 32 bytes per step
            const uint64_t off = static_cast<uint64_t>(((kk >> 2) * PANEL_BYTES + (kk & 3) * 32) >> 4);
            mma_f8_ss_w(dS, qd + off, kd + off, IDESC_S, kk > 0 ? 1u : 0u);
          }
        } else {
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint64_t off = static_cast<uint64_t>(((kk >> 2) * PANEL_BYTES + (kk & 3) * 32) >> 4);
            mma_bf16_ss_w(dS, qd + off, kd + off, IDESC_S, kk > 0 ? 1u : 0u);
          }
        }
        commit(&s_full[w]);
      };
      // O_w (+)= P_w V with V in ring slot `slot`, once warpgroup w wrote P_w
      auto issue_pv = [&](int w, int slot, bool first, bool last) -> bool {
        const uint32_t tO = tmem_base + 256 + w * 128;
        // keys [16 kk0, 16 kk1) (bf16) or [32 kk0, 32 kk1) (e4m3)
        auto pv_range = [&](int kk0, int kk1) {
          if constexpr (F8) {
            // A = P_w (queries x keys) and B = V_j^T (d x keys), both K-major
            const uint64_t pd = p_desc0 + static_cast<uint64_t>((w * PANEL_BYTES) >> 4);
            const uint64_t vd = ring_kdesc0 + static_cast<uint64_t>((slot * L::TILE) >> 4);
#pragma unroll
            for (int kk = kk0; kk < kk1; ++kk) {
              const uint64_t off = static_cast<uint64_t>((kk * 32) >> 4);
              mma_f8_ss_w(tO, pd + off, vd + off, IDESC_O, (!first || kk > 0) ? 1u : 0u);
            }
          } else {
            const uint64_t vd = ring_vdesc0 + static_cast<uint64_t>((slot * L::TILE) >> 4);
            const uint32_t tP = tmem_base + w * 128;
#pragma unroll
            for (int kk = kk0; kk < kk1; ++kk) {
              // keys 16kk .. 16kk+15: P columns 8kk.., V rows 16kk.. (2048 bytes per step)
              const uint64_t vdk = vd + static_cast<uint64_t>((kk * 2048) >> 4);
              mma_bf16_ts_w(tO, tP + kk * 8, vdk, IDESC_O, (!first || kk > 0) ? 1u : 0u);
            }
          }
        };
        constexpr int KK = F8 ? BLOCK_N / 32 : BLOCK_N / 16;
        if (!mwait(&p_full[w], pcount[w] & 1)) return false;
        ++pcount[w];
        tc_fence_after();
        pv_range(0, KK);
        if (last) commit(&o_final[w]);
        return true;
      };

      int kv = 0;  // key tiles consumed so far (all work items)
      auto kslot = [&](int g) { return (2 * g) % NSLOT; };
      auto vslot = [&](int g) { return (2 * g + 1) % NSLOT; };
      auto kwait = [&](int g) { return mwait(&full[kslot(g)], ((2 * g) / NSLOT) & 1); };
      auto vwait = [&](int g) { return mwait(&full[vslot(g)], ((2 * g + 1) / NSLOT) & 1); };
      bool ok = true;
      if (p.kv_split) {
        // Paired heads with their own K / V: every ring tile is used by one
        // product and released right after it, in the order they are taken.
        int racq = 0;
        auto acq = [&](int& slot) {
          slot = racq % NSLOT;
          const bool r = mwait(&full[slot], (racq / NSLOT) & 1);
          ++racq;
          return r;
        };
        for (int k = 0; ok; ++k) {
          const int item = cta_item(cta, k, G);
          if (item >= p.total_items) break;
          const ItemGeo g = item_geo<VARLEN>(p, item);
          const int n = n_kv_of(g, 1);  // both tiles: the same rows
          int sl = 0;
          if (!mwait(q_full, k & 1)) { ok = false; break; }
          for (int w = 0; w < NQ && ok; ++w) {
            if (!acq(sl)) { ok = false; break; }
            tc_fence_after();
            issue_s(w, sl);
            commit(&empty[sl]);
          }
          if (!ok) break;
          if (n == 1) commit(q_empty);
          for (int j = 0; j < n && ok; ++j) {
            const bool more = j + 1 < n;
            for (int w = 0; w < NQ; ++w) {
              // the first product of an item overwrites O_w: its read-out by
              // the previous item's epilogue must be complete
              if (!acq(sl) || (j == 0 && k > 0 && !mwait(&o_free[w], (k - 1) & 1)) ||
                  !issue_pv(w, sl, j == 0, j == n - 1)) {
                ok = false;
                break;
              }
              commit(&empty[sl]);
              if (more) {
                if (!acq(sl)) { ok = false; break; }
                tc_fence_after();
                issue_s(w, sl);
                commit(&empty[sl]);
              }
            }
            if (ok && j + 2 == n) commit(q_empty);  // last S of this item issued
          }
        }
      }
      for (int k = 0; ok && !p.kv_split; ++k) {
        const int item = cta_item(cta, k, G);
        if (item >= p.total_items) break;
        const ItemGeo g = item_geo<VARLEN>(p, item);
        const int n0 = n_kv_of(g, 0);
        const int n1 = n_kv_of(g, 1);
        if (!mwait(q_full, k & 1) || !kwait(kv)) { ok = false; break; }
        tc_fence_after();
        issue_s(0, kslot(kv));
        issue_s(1, kslot(kv));
        commit(&empty[kslot(kv)]);
        if (n1 == 1) commit(q_empty);
        for (int j = 0; j < n1; ++j) {
          const int g = kv + j;
          const bool more = j + 1 < n1;
          if (!vwait(g)) { ok = false; break; }
          if (j < n0) {
            // the first product of an item overwrites O_0: its read-out by the
            // previous item's epilogue must be complete
            if (j == 0 && k > 0 && !mwait(&o_free[0], (k - 1) & 1)) { ok = false; break; }
            if (!issue_pv(0, vslot(g), j == 0, j == n0 - 1)) { ok = false; break; }
          }
          if (more) {
            if (!kwait(g + 1)) { ok = false; break; }
            tc_fence_after();
            if (j + 1 < n0) issue_s(0, kslot(g + 1));
          }
          if (j == 0 && k > 0 && !mwait(&o_free[1], (k - 1) & 1)) { ok = false; break; }
          if (!issue_pv(1, vslot(g), j == 0, j == n1 - 1)) { ok = false; break; }
          commit(&empty[vslot(g)]);
          if (more) {
            issue_s(1, kslot(g + 1));
            commit(&empty[kslot(g + 1)]);
            if (j + 2 == n1) commit(q_empty);  // last S of this item issued
          }
        }
        kv += n1;
      }
      // All MMAs must retire before tensor memory is released.
      commit(mma_final);
      mbar_wait_drain(mma_final, 0);
    }
   }
  } else if (warp >= 8) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(REGS_EPILOGUE));
    // ------------------------------------------------------------ epilogue
    // Thread t of the warpgroup owns row t of each query tile: tensor-memory
    // lanes 32 (warp % 4) .. +31 are this warp's.
    const int row = threadIdx.x - 8 * 32;
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    bool ok = true;
    for (int k = 0; ok; ++k) {
      const int item = cta_item(cta, k, G);
      if (item >= p.total_items) break;
      const ItemGeo g = item_geo<VARLEN>(p, item);
      for (int w = 0; w < NQ; ++w) {
        // the tile's last O += P V has completed, and its 1 / l is written
        if (!mbar_wait_warp(&o_final[w], k & 1, abort_flag) ||
            !mbar_wait_warp(&l_ready[2 * w + (k & 1)], (k >> 1) & 1, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const float inv_l = inv_l_buf[((k & 1) * NQ + w) * TILE_M + row];
        const uint32_t tO = tmem_base + 256 + w * 128 + lane_off;
        const int row_g = g.qrow(w) + row;  // within the sequence
        const size_t orow_off = static_cast<size_t>(g.hd(w)) * p.o_head +
                                static_cast<size_t>(g.q0 + row_g) * p.o_row;
        const bool valid = row_g < g.Nq && dbg_ok(orow_off + D <= p.o_elems);
        __nv_bfloat16* orow_g = p.o + orow_off;
#pragma unroll
        for (int c = 0; c < D; c += 32) {
          uint32_t orow[32];
          tmem_ld32(tO + c, orow);
          tmem_ld_wait();
          if (c + 32 == D) {
            // O_w has been read: the next item's first O += P V may overwrite it.
            tc_fence_before();
            mbar_arrive(&o_free[w]);
          }
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 32; e += 2)
            pk[e >> 1] = pack_bf16x2(__uint_as_float(orow[e]) * inv_l,
                                     __uint_as_float(orow[e + 1]) * inv_l);
          if (valid) {
            uint4* dst = reinterpret_cast<uint4*>(orow_g + c);
#pragma unroll
            for (int v4 = 0; v4 < 4; ++v4)
              dst[v4] = make_uint4(pk[4 * v4], pk[4 * v4 + 1], pk[4 * v4 + 2], pk[4 * v4 + 3]);
          }
        }
      }
    }
    tmem_ld_wait();
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(REGS_SOFTMAX));
    // ------------------------------------------------------------ softmax
    const int w = warp >> 2;                       // query tile of this warpgroup
    const int row = threadIdx.x - w * TILE_M;      // 0..127, TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tS = tmem_base + w * 128 + lane_off;
    const uint32_t tO = tmem_base + 256 + w * 128 + lane_off;
    const float sl2 = p.scale_log2;
    int scount = 0;   // S tiles consumed (all items)
    bool ok = true;
    for (int k = 0; ok; ++k) {
      const int item = cta_item(cta, k, G);
      if (item >= p.total_items) break;
      const ItemGeo g = item_geo<VARLEN>(p, item);
      const int q_row0 = g.qrow(w);  // within the sequence
      const int row_g = q_row0 + row;
      const int n_kv = n_kv_of(g, w);
      float m = -INFINITY;  // running max of scale * log2(e) * s
      float l = 0.f;
      for (int j = 0; j < n_kv; ++j) {
        if (!mbar_wait_warp(&s_full[w], scount & 1, abort_flag)) {
          ok = false;
          break;
        }
        ++scount;
        tc_fence_after();
        uint32_t sr[128];
        tmem_ld32(tS + 0, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
        tmem_ld32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
        tmem_ld32(tS + 64, *reinterpret_cast<uint32_t(*)[32]>(&sr[64]));
        tmem_ld32(tS + 96, *reinterpret_cast<uint32_t(*)[32]>(&sr[96]));
        tmem_ld_wait();
        const int key0 = j * BLOCK_N;
        const bool need_mask = (key0 + BLOCK_N > g.Nk) ||
                               (CAUSAL && key0 + BLOCK_N - 1 > q_row0 + g.off);
        // MAX_CHAINS independent max chains (latency, not throughput, bounds
        // this loop), each taking two new values per three-input max
        float mx[MAX_CHAINS];
#pragma unroll
        for (int i = 0; i < MAX_CHAINS; ++i) mx[i] = -INFINITY;
        if (need_mask) {
          // last admissible key (below 0: none, the row stays at -inf)
          const int lim = CAUSAL ? min(g.Nk - 1, row_g + g.off) : g.Nk - 1;
#pragma unroll
          for (int c = 0; c < 128; ++c) {
            const float s = (key0 + c <= lim) ? __uint_as_float(sr[c]) : -INFINITY;
            sr[c] = __float_as_uint(s);
          }
        }
#pragma unroll
        for (int c = 0; c < 128; c += 2)
          mx[(c >> 1) % MAX_CHAINS] =
              fmax3(mx[(c >> 1) % MAX_CHAINS], __uint_as_float(sr[c]), __uint_as_float(sr[c + 1]));
#pragma unroll
        for (int h = MAX_CHAINS / 2; h >= 1; h /= 2)
#pragma unroll
          for (int i = 0; i < h; ++i) mx[i] = fmaxf(mx[i], mx[i + h]);
        // scale * log2(e) > 0, so the maximum of the scaled row is the scaled maximum
        const float m_new = fmaxf(m, mx[0] * sl2);
        // true when m = -inf < m_new; false while the whole row is masked
        const bool grow = (m_new - m) > RESCALE_THRESHOLD;
        const bool warp_grow = __any_sync(0xffffffffu, grow);
        const float m_use = warp_grow ? m_new : m;
        const float m_ref = (m_use == -INFINITY) ? 0.f : m_use;
        // 1 unless the maximum moves (then 0 when m = -inf).  Evaluated only
        // when needed: on the critical path an exponential would queue behind
        // the other warpgroup's exponentials on the shared MUFU unit.
        const float alpha = warp_grow ? ex2_approx(m - m_ref) : 1.f;
        if (warp_grow && j > 0) {
          // O holds P_0 V_0 + ... + P_{j-1} V_{j-1} relative to the old max:
          // rescale it before this step's P is handed over.  It is complete:
          // S_w,j was issued after O_w += P_{j-1} V_{j-1} by the same thread,
          // and the commit that signalled S_w,j covers every tensor-core
          // operation that thread issued before it.
          // eight columns at a time: S is still live in registers here
#pragma unroll 1
          for (int c = 0; c < D; c += 8) {
            uint32_t orow[8];
            tmem_ld8(tO + c, orow);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 8; ++e)
              orow[e] = __float_as_uint(__uint_as_float(orow[e]) * alpha);
            tmem_st8(tO + c, orow);
          }
        }
        // row sum in four packed two-lane chains (one f32x2 addition per pair)
        uint64_t rs2[4] = {0, 0, 0, 0};
        // Exponentials: MUFU ex2; in unmasked tiles EMU_PAIRS of every 4 pairs
        // may go to the FMA-pipe polynomial.  Masked tiles use ex2 only, so
        // excluded keys give exactly 0.
        // x = s * scale * log2(e) - m for two keys per packed f32x2 FMA
        const uint64_t sl2_2 = pack_f32x2(sl2, sl2);
        const uint64_t negm_2 = pack_f32x2(-m_ref, -m_ref);
        // Exponentials: MUFU ex2, except that in tiles without masked keys
        // EMU_PAIRS of every 4 key pairs go to the FMA-pipe polynomial (masked
        // keys must give exactly 0, which only ex2 of -inf does).  The two
        // cases are separate loop bodies, so that the choice per pair is a
        // compile-time one.
        auto exps = [&](auto emu_c) {
          constexpr int EMU = decltype(emu_c)::value;
#pragma unroll
          for (int c = 0; c < 128; c += 32) {
            uint32_t pk[16];  // bf16 P
            float pf[32];     // e4m3 P, before rounding
            (void)pk;
            (void)pf;
#pragma unroll
            for (int e = 0; e < 32; e += 2) {
              float x0, x1;
              fma_f32x2(x0, x1, __uint_as_float(sr[c + e]), __uint_as_float(sr[c + e + 1]), sl2_2,
                        negm_2);
              float p0, p1;
              if (((e >> 1) & 3) >= 4 - EMU) {
                ex2_poly3_x2(x0, x1, p0, p1);
              } else {
                p0 = ex2_approx(x0);
                p1 = ex2_approx(x1);
              }
              add_f32x2(rs2[(e >> 1) & 3], p0, p1);
              if constexpr (F8) {
                pf[e] = p0;
                pf[e + 1] = p1;
              } else {
                pk[e >> 1] = pack_bf16x2(p0, p1);
              }
            }
            if constexpr (F8) {
              // keys c .. c+31 of row `row`: two 16-byte chunks of the 128-byte
              // row, 128-byte swizzle (chunk index xor row % 8)
              uint8_t* prow = smem + L::P_OFF + w * PANEL_BYTES + row * 128;
#pragma unroll
              for (int h = 0; h < 2; ++h) {
                const uint32_t ch =
                    static_cast<uint32_t>((c >> 4) + h) ^ static_cast<uint32_t>(row & 7);
                const float* f = pf + 16 * h;
                *reinterpret_cast<uint4*>(prow + ch * 16) = make_uint4(
                    pack_e4m3x4(f[0], f[1], f[2], f[3]), pack_e4m3x4(f[4], f[5], f[6], f[7]),
                    pack_e4m3x4(f[8], f[9], f[10], f[11]), pack_e4m3x4(f[12], f[13], f[14], f[15]));
              }
            } else {
              tmem_st16(tS + (c >> 1), pk);
            }
          }
        };
        if (EMU_PAIRS > 0 && !need_mask) exps(std::integral_constant<int, EMU_PAIRS>{});
        else exps(std::integral_constant<int, 0>{});
        // e4m3 P is read by the async proxy (tensor core) from shared memory
        if constexpr (F8) fence_proxy_async_smem();
        l = l * alpha + ((sum_f32x2(rs2[0]) + sum_f32x2(rs2[1])) +
                         (sum_f32x2(rs2[2]) + sum_f32x2(rs2[3])));
        m = m_use;
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[w]);
      }
      if (!ok) break;
      // End of the work item for this tile: LSE, and 1 / l for the epilogue
      // warpgroup (which normalises O once the last O += P V has completed).
      // The buffer and barrier alternate with the item's parity: the next
      // item of this tile can finish its softmax before the epilogue has
      // read this one, but not the item after it (its first P V waits until
      // the epilogue has read this item's O).
      inv_l_buf[((k & 1) * NQ + w) * TILE_M + row] = (l > 0.f) ? p.o_scale / l : 0.f;
      mbar_arrive(&l_ready[2 * w + (k & 1)]);
      if (row_g < g.Nq && p.lse != nullptr &&
          dbg_ok(static_cast<size_t>(g.hd(w)) * p.lse_head + g.q0 + row_g < p.lse_elems)) {
        // LSE = ln(sum exp(scale * s)) = (m + log2 l) * ln 2, m in log2 units.
        const float lse = (l > 0.f) ? (m + lg2_approx(l)) * 0.6931471805599453f : -INFINITY;
        p.lse[static_cast<size_t>(g.hd(w)) * p.lse_head + g.q0 + row_g] = lse;
      }
    }
    tmem_ld_wait();
    tmem_st_wait();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == WARP_MMA) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

template <int D, bool CAUSAL, bool VARLEN, bool F8 = false>
fa_status launch(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                 const Params& prm, int grid_size, cudaStream_t stream) {
  auto kern = fa_fwd_kernel<D, CAUSAL, VARLEN, F8>;
  constexpr int SMEM = Smem<D, F8>::ALLOC;
  static SmemOptIn opt_in;  // one per instantiation of this kernel
  if (const fa_status st = opt_in.ensure(kern, SMEM); st != FA_OK) return st;
  main_kernel_begin(stream);
  kern<<<grid_size, NUM_THREADS, SMEM, stream>>>(tq, tk, tv, prm);
  main_kernel_end(stream);
  return cuda_status(cudaGetLastError());
}

// Work distribution.  Causal problems whose K and V all fit comfortably in L2
// run persistently (one CTA per SM, longest tiles first, alternating rounds);
// everything else runs one CTA per 256-row tile in head-major order, so the
// resident CTAs share their heads' K/V tiles in L2.  fa_set_schedule can force
// one of the two.
int schedule_mode() { return g_fwd_schedule.load(std::memory_order_relaxed); }

// Heads per band of the head-major order: as many adjacent (query) heads as
// keep their K and V within about 40 MB of L2 (a band and the next one's
// first CTAs are resident together), at most 8.  kv_bytes: K and V of one
// key/value head; share: query heads (or head pairs) reading it.
int head_band(double kv_bytes, int share) {
  const double per_head = kv_bytes / (share > 0 ? share : 1);
  const double n = 40.0 * 1024 * 1024 / (per_head > 1.0 ? per_head : 1.0);
  return n >= 8.0 ? 8 : (n < 1.0 ? 1 : static_cast<int>(n));
}

// Rows with no key at all (Nk = 0): O = 0, LSE = -inf, the same values the
// main kernel gives a fully masked row.
__global__ void fa_fwd_no_keys_kernel(__nv_bfloat16* o, float* lse, size_t rows, int d) {
  const size_t stride = static_cast<size_t>(gridDim.x) * blockDim.x;
  const size_t n_o = rows * static_cast<size_t>(d) / 8;  // uint4 = 8 bf16
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n_o; i += stride)
    reinterpret_cast<uint4*>(o)[i] = make_uint4(0u, 0u, 0u, 0u);
  if (lse != nullptr)
    for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < rows;
         i += stride)
      lse[i] = -INFINITY;
}

}  // namespace fwd

fa_status launch_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                     int H, int Hkv, int Nq, int Nk, int d, int causal, float scale,
                     cudaStream_t stream) {
  const int BH = B * H;
  if (Nq == 0) return FA_OK;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return FA_ERR_CUDA;
  if (Nk == 0) {
    fwd::fa_fwd_no_keys_kernel<<<4 * sms, 256, 0, stream>>>(
        static_cast<__nv_bfloat16*>(o), lse, static_cast<size_t>(BH) * Nq, d);
    return cuda_status(cudaGetLastError());
  }
  // Grouped heads with an even group: a work item is one 128-row tile of two
  // query heads that share a key/value head, so both of its query tiles see
  // the same keys (no step in which one tile waits while the other finishes
  // its diagonal key tile) and still share every K/V tile.  Otherwise two
  // consecutive 128-row tiles of one head.
  // Without grouping, persistent causal problems pair heads too: the two
  // heads then read their own K / V (about twice the tile loads, all from L2),
  // which pays for itself where items are short.
  const int group = H / Hkv;
  const double kv_bytes = 4.0 * B * Hkv * static_cast<double>(Nk) * d;
  const bool small_kv = kv_bytes <= 96.0 * 1024 * 1024;
  const bool pair = group % 2 == 0 || (group == 1 && H % 2 == 0 && causal && small_kv);
  const int item_rows = pair ? fwd::TILE_M : fwd::BLOCK_M;
  const long long n_cta_tiles = (Nq + item_rows - 1) / item_rows;
  const long long item_bh = pair ? BH / 2 : BH;
  const long long items = item_bh * n_cta_tiles;
  if (items > 0x7fffffffLL) return FA_ERR_INVALID_ARG;
  CUtensorMap tq, tk, tv;
  fa_status st;
  if ((st = make_tmap_bf16_3d(&tq, q, d, Nq, BH, fwd::TILE_M)) != FA_OK) return st;
  // K and V carry B * Hkv heads of Nk rows; query head bh reads key/value head
  // bh / (H / Hkv)
  const uint64_t BHkv = static_cast<uint64_t>(B) * Hkv;
  if ((st = make_tmap_bf16_3d(&tk, k, d, Nk, BHkv, fwd::BLOCK_N)) != FA_OK) return st;
  if ((st = make_tmap_bf16_3d(&tv, v, d, Nk, BHkv, fwd::BLOCK_N)) != FA_OK) return st;
  const int mode = fwd::schedule_mode();
  bool persistent = causal && items > sms && small_kv;
  int grid = persistent ? sms : static_cast<int>(items);
  if (mode == FA_SCHEDULE_GRID) {
    persistent = false;
    grid = static_cast<int>(items);
  } else if (mode == FA_SCHEDULE_PERSISTENT) {  // forced: about three items per CTA even for small problems
    persistent = true;
    grid = static_cast<int>(std::min<long long>(sms, std::max<long long>(1, items / 3)));
  }
  fwd::Params prm;
  prm.o = static_cast<__nv_bfloat16*>(o);
  prm.lse = lse;
  prm.Nq = Nq;
  prm.Nk = Nk;
  prm.causal_off = Nk - Nq;
  prm.BH = static_cast<int>(item_bh);
  prm.pair_heads = pair ? 1 : 0;
  prm.kv_split = (pair && group == 1) ? 1 : 0;
  prm.group = H / Hkv;
  prm.n_cta_tiles = static_cast<int>(n_cta_tiles);
  prm.total_items = static_cast<int>(items);
  prm.lpt_order = persistent ? 1 : 0;
  prm.head_band = fwd::head_band(4.0 * Nk * d, pair ? group / 2 : group);
  prm.scale_log2 = scale * 1.4426950408889634f;
  prm.o_scale = 1.f;
  prm.cu_q = nullptr;
  prm.cu_k = nullptr;
  prm.H = H;
  prm.total_q = 0;
  prm.total_k = 0;
  prm.o_head = static_cast<size_t>(Nq) * d;
  prm.o_row = static_cast<size_t>(d);
  prm.lse_head = static_cast<size_t>(Nq);
  prm.o_elems = static_cast<size_t>(BH) * Nq * d;
  prm.lse_elems = static_cast<size_t>(BH) * Nq;
  if (d == 128)
    return causal ? fwd::launch<128, true, false>(tq, tk, tv, prm, grid, stream)
                  : fwd::launch<128, false, false>(tq, tk, tv, prm, grid, stream);
  return causal ? fwd::launch<64, true, false>(tq, tk, tv, prm, grid, stream)
                : fwd::launch<64, false, false>(tq, tk, tv, prm, grid, stream);
}

fa_status launch_fwd_varlen(const void* q, const void* k, const void* v, void* o, float* lse,
                            const int* cu_q, const int* cu_k, int B, int H, int Hkv,
                            int total_q, int total_k, int max_seqlen_q, int d, int causal,
                            float scale, cudaStream_t stream) {
  if (total_q == 0 || max_seqlen_q == 0) return FA_OK;
  const long long n_cta_tiles = (static_cast<long long>(max_seqlen_q) + fwd::BLOCK_M - 1) /
                                fwd::BLOCK_M;
  const long long items = static_cast<long long>(B) * H * n_cta_tiles;
  if (items > 0x7fffffffLL) return FA_ERR_INVALID_ARG;
  // token-major maps: [rows, heads, d]; a key map over zero rows still needs
  // one row of extent, and its loads are all masked
  CUtensorMap tq, tk, tv;
  fa_status st;
  if ((st = make_tmap_bf16_rows_heads(&tq, q, d, H, total_q, fwd::TILE_M)) != FA_OK) return st;
  const uint64_t krows = total_k > 0 ? static_cast<uint64_t>(total_k) : 1;
  const void* kb = total_k > 0 ? k : q;  // any valid address; never read unmasked
  const void* vb = total_k > 0 ? v : q;
  if ((st = make_tmap_bf16_rows_heads(&tk, kb, d, total_k > 0 ? Hkv : H, krows, fwd::BLOCK_N)) !=
      FA_OK)
    return st;
  if ((st = make_tmap_bf16_rows_heads(&tv, vb, d, total_k > 0 ? Hkv : H, krows, fwd::BLOCK_N)) !=
      FA_OK)
    return st;
  fwd::Params prm;
  prm.o = static_cast<__nv_bfloat16*>(o);
  prm.lse = lse;
  prm.Nq = 0;
  prm.Nk = 0;
  prm.causal_off = 0;
  prm.BH = B * H;
  prm.pair_heads = 0;
  prm.kv_split = 0;
  prm.group = H / Hkv;
  prm.n_cta_tiles = static_cast<int>(n_cta_tiles);
  prm.total_items = static_cast<int>(items);
  prm.lpt_order = 0;  // one CTA per tile, a head's tiles adjacent, longest first
  prm.head_band = 1;  // a sequence's tiles adjacent
  prm.scale_log2 = scale * 1.4426950408889634f;
  prm.o_scale = 1.f;
  prm.cu_q = cu_q;
  prm.cu_k = cu_k;
  prm.H = H;
  prm.total_q = total_q;
  prm.total_k = total_k;
  prm.o_head = static_cast<size_t>(d);
  prm.o_row = static_cast<size_t>(H) * d;
  prm.lse_head = static_cast<size_t>(total_q);
  prm.o_elems = static_cast<size_t>(total_q) * H * d;
  prm.lse_elems = static_cast<size_t>(H) * total_q;
  const int grid = static_cast<int>(items);
  if (d == 128)
    return causal ? fwd::launch<128, true, true>(tq, tk, tv, prm, grid, stream)
                  : fwd::launch<128, false, true>(tq, tk, tv, prm, grid, stream);
  return causal ? fwd::launch<64, true, true>(tq, tk, tv, prm, grid, stream)
                : fwd::launch<64, false, true>(tq, tk, tv, prm, grid, stream);
}

}  // namespace fa

namespace fa {

fa_status launch_fwd_fp8(const void* q, const void* k, const void* vt, void* o, float* lse,
                         float q_scale, float k_scale, float v_scale, int B, int H, int Hkv,
                         int Nq, int Nk, int causal, float scale, cudaStream_t stream) {
  constexpr int d = 128;
  const int BH = B * H;
  if (Nq == 0) return FA_OK;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return FA_ERR_CUDA;
  if (Nk == 0) {
    fwd::fa_fwd_no_keys_kernel<<<4 * sms, 256, 0, stream>>>(
        static_cast<__nv_bfloat16*>(o), lse, static_cast<size_t>(BH) * Nq, d);
    return cuda_status(cudaGetLastError());
  }
  const long long n_cta_tiles = (Nq + fwd::BLOCK_M - 1) / fwd::BLOCK_M;
  const long long items = static_cast<long long>(BH) * n_cta_tiles;
  if (items > 0x7fffffffLL) return FA_ERR_INVALID_ARG;
  CUtensorMap tq, tk, tv;
  fa_status st;
  const uint64_t BHkv = static_cast<uint64_t>(B) * Hkv;
  // q, k: [heads, rows, 128 bytes]; vt: [heads, 128 rows (d), Nk bytes]
  if ((st = make_tmap_u8_3d(&tq, q, d, Nq, BH, 128, fwd::TILE_M)) != FA_OK) return st;
  if ((st = make_tmap_u8_3d(&tk, k, d, Nk, BHkv, 128, fwd::BLOCK_N)) != FA_OK) return st;
  if ((st = make_tmap_u8_3d(&tv, vt, Nk, d, BHkv, 128, d)) != FA_OK) return st;
  const double kv_bytes = 2.0 * B * Hkv * static_cast<double>(Nk) * d;
  const int mode = fwd::schedule_mode();
  bool persistent = causal && items > sms && kv_bytes <= 96.0 * 1024 * 1024;
  int grid = persistent ? sms : static_cast<int>(items);
  if (mode == FA_SCHEDULE_GRID) {
    persistent = false;
    grid = static_cast<int>(items);
  } else if (mode == FA_SCHEDULE_PERSISTENT) {
    persistent = true;
    grid = static_cast<int>(std::min<long long>(sms, std::max<long long>(1, items / 3)));
  }
  fwd::Params prm;
  prm.o = static_cast<__nv_bfloat16*>(o);
  prm.lse = lse;
  prm.Nq = Nq;
  prm.Nk = Nk;
  prm.causal_off = Nk - Nq;
  prm.BH = BH;
  prm.pair_heads = 0;
  prm.kv_split = 0;
  prm.group = H / Hkv;
  prm.n_cta_tiles = static_cast<int>(n_cta_tiles);
  prm.total_items = static_cast<int>(items);
  prm.lpt_order = persistent ? 1 : 0;
  prm.head_band = fwd::head_band(2.0 * Nk * d, H / Hkv);  // e4m3: 1 byte per element
  // scores of the real (descaled) values: q_scale * k_scale * (Q8 K8^T)
  prm.scale_log2 = scale * q_scale * k_scale * 1.4426950408889634f;
  prm.o_scale = v_scale;
  prm.cu_q = nullptr;
  prm.cu_k = nullptr;
  prm.H = H;
  prm.total_q = 0;
  prm.total_k = 0;
  prm.o_head = static_cast<size_t>(Nq) * d;
  prm.o_row = static_cast<size_t>(d);
  prm.lse_head = static_cast<size_t>(Nq);
  prm.o_elems = static_cast<size_t>(BH) * Nq * d;
  prm.lse_elems = static_cast<size_t>(BH) * Nq;
  return causal ? fwd::launch<128, true, false, true>(tq, tk, tv, prm, grid, stream)
                : fwd::launch<128, false, false, true>(tq, tk, tv, prm, grid, stream);
}

}  // namespace fa
