// fa_fwd.cu - forward pass of exact attention on sm_100a.
//
// One CTA computes one 128-row query tile of one (batch, head):
//   O_i = softmax(scale * Q_i K^T [+ causal mask]) V,   LSE_i = ln sum_j exp(...)
// following the tile recurrence of "DL101 chapter 9" (handsonai.io), section
// 3.3: over key tiles j, S = Q_i K_j^T; m' = max(m, rowmax S); P = exp(S - m');
// c = exp(m - m'); l' = l c + rowsum P; O' = O c + P V_j; finally O / l.
// The five stages of "What is FlashAttention" (unite.ai, five-stage
// operational map) map onto the warp roles below: partition into tiles and
// load them on chip (TMA producer warp), local scores and running
// normalisation (MMA warp + softmax warpgroup), accumulate without the full
// matrix (MMA warp, O in tensor memory), and the kernel schedule (grid order).
//
// Warp roles (192 threads):
//   warps 0-3  softmax warpgroup: thread t owns row t of the tile (TMEM lane t).
//              Reads S from tensor memory, applies scale / mask, keeps the
//              running max m and sum l (log2 domain), writes P as bf16 into
//              the same tensor-memory columns, rescales O when m grows, and
//              finally writes O / l and LSE.
//   warp 4     TMA producer: Q once, then K_j and V_j through an NS-stage ring.
//   warp 5     tensor-memory allocator and MMA issuer (one thread):
//              S_j = Q K_j^T (both operands K-major in shared memory) into one
//              of two S buffers, and O += P_j V_j (P from tensor memory, V
//              MN-major in shared memory).  S_{j+1} is issued before O += P_j V_j
//              so the tensor core works while the softmax runs.
//
// Tensor memory (512 columns x 128 lanes, fp32): S0 [0,128), S1 [128,256),
// O [256, 256+d).  P_j overwrites the first 64 columns of its S buffer (two
// bf16 per column).
//
// The softmax keeps a stale maximum until a row's maximum grows by more than
// 2^8: P may then exceed 1 by up to 256x, which bf16 / fp32 hold exactly as
// well, and O and l are only rescaled (a tensor-memory round trip) when the
// maximum really moves.  Both l and O always refer to the same maximum, so the
// final O / l is unchanged.
#include "fa_internal.h"
#include "sm100.cuh"

namespace fa {

namespace fwd {

constexpr int BLOCK_M = 128;
constexpr int BLOCK_N = 128;
constexpr int NUM_THREADS = 192;
constexpr int PANEL_BYTES = 128 * 128;   // 128 rows x 64 bf16 (one swizzle panel)
constexpr uint32_t TMEM_COLS = 512;
constexpr float RESCALE_THRESHOLD = 8.0f;  // log2 units

template <int D>
struct Smem {
  static constexpr int NPANEL = D / 64;
  static constexpr int TILE = NPANEL * PANEL_BYTES;
  static constexpr int NS = 2;  // K/V ring depth
  static constexpr int Q_OFF = 0;
  static constexpr int K_OFF = TILE;
  static constexpr int V_OFF = K_OFF + NS * TILE;
  static constexpr int BAR_OFF = V_OFF + NS * TILE;
  // barriers: q_full, k_full[NS], v_full[NS], k_empty[NS], v_empty[NS],
  //           s_full[2], p_full[2], o_done, o_final, mma_final
  static constexpr int NBAR = 1 + 4 * NS + 2 + 2 + 1 + 1 + 1;
  static constexpr int MISC_OFF = BAR_OFF + NBAR * 8;
  static constexpr int BYTES = MISC_OFF + 16;
  // + slack for 1024-byte alignment; at least 116 KB so that a single CTA
  // (and its 512 tensor-memory columns) occupies an SM.
  static constexpr int ALLOC = (BYTES + 1024) > 118784 ? (BYTES + 1024) : 118784;
};

struct Params {
  __nv_bfloat16* o;
  float* lse;
  int N;
  int n_q_tiles;
  float scale_log2;  // scale * log2(e)
};

template <int D, bool CAUSAL>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    fa_fwd_kernel(const __grid_constant__ CUtensorMap tm_q,
                  const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const Params p) {
  using L = Smem<D>;
  constexpr int NS = L::NS;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::BAR_OFF);
  uint64_t* q_full = bars;
  uint64_t* k_full = bars + 1;
  uint64_t* v_full = k_full + NS;
  uint64_t* k_empty = v_full + NS;
  uint64_t* v_empty = k_empty + NS;
  uint64_t* s_full = v_empty + NS;
  uint64_t* p_full = s_full + 2;
  uint64_t* o_done = p_full + 2;    // one phase per O += P V
  uint64_t* o_final = o_done + 1;   // the last O += P V of the tile
  uint64_t* mma_final = o_final + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::MISC_OFF + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int bh = blockIdx.x;
  // Longest tiles first: blockIdx.y = 0 (launched first) is the last q tile.
  const int q_tile = p.n_q_tiles - 1 - static_cast<int>(blockIdx.y);
  const int q_row0 = q_tile * BLOCK_M;
  const int n_kv_total = (p.N + BLOCK_N - 1) / BLOCK_N;
  const int n_kv = CAUSAL ? min(q_tile + 1, n_kv_total) : n_kv_total;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < NS; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&v_full[s], 1);
      mbar_init(&k_empty[s], 1);
      mbar_init(&v_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&s_full[s], 1);
      mbar_init(&p_full[s], BLOCK_M);
    }
    mbar_init(o_done, 1);
    mbar_init(o_final, 1);
    mbar_init(mma_final, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 5) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == 4 && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const uint32_t tS0 = tmem_base;
  const uint32_t tO = tmem_base + 256;

  if (warp == 4) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int last_k[NS], last_v[NS];
      for (int s = 0; s < NS; ++s) last_k[s] = last_v[s] = -1;
      mbar_arrive_expect_tx(q_full, L::TILE);
      for (int pn = 0; pn < L::NPANEL; ++pn)
        tma_load_3d(smem + L::Q_OFF + pn * PANEL_BYTES, &tm_q, q_full, pn * 64, q_row0, bh);
      for (int j = 0; j < n_kv; ++j) {
        const int st = j % NS;
        const int r = j / NS;
        if (j >= NS && !mbar_wait(&k_empty[st], (r - 1) & 1, abort_flag)) break;
        mbar_arrive_expect_tx(&k_full[st], L::TILE);
        for (int pn = 0; pn < L::NPANEL; ++pn)
          tma_load_3d(smem + L::K_OFF + st * L::TILE + pn * PANEL_BYTES, &tm_k, &k_full[st],
                      pn * 64, j * BLOCK_N, bh);
        last_k[st] = r;
        if (j >= NS && !mbar_wait(&v_empty[st], (r - 1) & 1, abort_flag)) break;
        mbar_arrive_expect_tx(&v_full[st], L::TILE);
        for (int pn = 0; pn < L::NPANEL; ++pn)
          tma_load_3d(smem + L::V_OFF + st * L::TILE + pn * PANEL_BYTES, &tm_v, &v_full[st],
                      pn * 64, j * BLOCK_N, bh);
        last_v[st] = r;
      }
      // Every copy issued must land before this CTA's shared memory is freed.
      mbar_wait_drain(q_full, 0);
      for (int s = 0; s < NS; ++s) {
        if (last_k[s] >= 0) mbar_wait_drain(&k_full[s], last_k[s] & 1);
        if (last_v[s] >= 0) mbar_wait_drain(&v_full[s], last_v[s] & 1);
      }
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t IDESC_S = idesc_bf16_f32(BLOCK_M, BLOCK_N, false, false);
      constexpr uint32_t IDESC_O = idesc_bf16_f32(BLOCK_M, D, false, true);
      const uint32_t q_addr = smem_u32(smem + L::Q_OFF);
      const uint32_t k_addr = smem_u32(smem + L::K_OFF);
      const uint32_t v_addr = smem_u32(smem + L::V_OFF);

      auto issue_pv = [&](int i) -> bool {
        const int st = i % NS;
        const int sb = i & 1;
        if (!mbar_wait(&v_full[st], (i / NS) & 1, abort_flag)) return false;
        if (!mbar_wait(&p_full[sb], (i >> 1) & 1, abort_flag)) return false;
        tc_fence_after();
        const uint32_t vbase = v_addr + st * L::TILE;
#pragma unroll
        for (int kk = 0; kk < BLOCK_N / 16; ++kk) {
          // keys 16kk .. 16kk+15: P columns 8kk.., V rows 16kk.. (2048 bytes per step)
          const uint64_t bdesc = sdesc_mnmajor_sw128(vbase + kk * 2048, PANEL_BYTES);
          mma_bf16_ts(tO, tS0 + sb * 128 + kk * 8, bdesc, IDESC_O, (i > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(&v_empty[st]);
        mma_commit(o_done);
        return true;
      };

      bool ok = mbar_wait(q_full, 0, abort_flag);
      int j = 0;
      for (; ok && j < n_kv; ++j) {
        const int st = j % NS;
        if (!mbar_wait(&k_full[st], (j / NS) & 1, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t kbase = k_addr + st * L::TILE;
        const uint32_t dS = tS0 + (j & 1) * 128;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const int pn = kk >> 2;
          const uint32_t off = pn * PANEL_BYTES + (kk & 3) * 32;
          mma_bf16_ss(dS, sdesc_kmajor_sw128(q_addr + off), sdesc_kmajor_sw128(kbase + off),
                      IDESC_S, kk > 0 ? 1u : 0u);
        }
        mma_commit(&s_full[j & 1]);
        mma_commit(&k_empty[st]);
        if (j > 0 && !issue_pv(j - 1)) {
          ok = false;
          break;
        }
      }
      if (ok && n_kv > 0 && issue_pv(n_kv - 1)) mma_commit(o_final);
      // All MMAs must retire before tensor memory is released.
      mma_commit(mma_final);
      mbar_wait_drain(mma_final, 0);
    }
  } else {
    // ------------------------------------------------------------ softmax
    const int row = threadIdx.x;  // 0..127, TMEM lane
    const int row_g = q_row0 + row;
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
    const float sl2 = p.scale_log2;
    float m = -INFINITY;  // running max of scale*log2e*s
    float l = 0.f;
    bool ok = true;
    for (int j = 0; j < n_kv; ++j) {
      const int sb = j & 1;
      if (!mbar_wait_warp(&s_full[sb], (j >> 1) & 1, abort_flag)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t tS = tS0 + sb * 128 + lane_off;
      uint32_t sr[128];
      tmem_ld32(tS + 0, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
      tmem_ld32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
      tmem_ld32(tS + 64, *reinterpret_cast<uint32_t(*)[32]>(&sr[64]));
      tmem_ld32(tS + 96, *reinterpret_cast<uint32_t(*)[32]>(&sr[96]));
      tmem_ld_wait();
      float x[128];
      const int key0 = j * BLOCK_N;
      const bool need_mask = (key0 + BLOCK_N > p.N) || (CAUSAL && key0 + BLOCK_N - 1 > q_row0);
      float mx = -INFINITY;
      if (need_mask) {
        const int lim = CAUSAL ? min(p.N - 1, row_g) : p.N - 1;  // last admissible key
#pragma unroll
        for (int c = 0; c < 128; ++c) {
          const float s = __uint_as_float(sr[c]) * sl2;
          x[c] = (key0 + c <= lim) ? s : -INFINITY;
          mx = fmaxf(mx, x[c]);
        }
      } else {
#pragma unroll
        for (int c = 0; c < 128; ++c) {
          x[c] = __uint_as_float(sr[c]) * sl2;
          mx = fmaxf(mx, x[c]);
        }
      }
      const float m_new = fmaxf(m, mx);
      const bool grow = (m_new - m) > RESCALE_THRESHOLD;  // true when m = -inf
      const bool warp_grow = __any_sync(0xffffffffu, grow);
      const float m_use = warp_grow ? m_new : m;
      const float m_ref = (m_use == -INFINITY) ? 0.f : m_use;
      const float alpha = ex2_approx(m - m_ref);  // 0 when m = -inf
      float rs = 0.f;
#pragma unroll
      for (int c = 0; c < 128; c += 32) {
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          const float p0 = ex2_approx(x[c + e] - m_ref);
          const float p1 = ex2_approx(x[c + e + 1] - m_ref);
          rs += p0 + p1;
          pk[e >> 1] = pack_bf16x2(p0, p1);
        }
        tmem_st16(tS + (c >> 1), pk);
      }
      l = l * alpha + rs;
      if (warp_grow && j > 0) {
        // O holds P_0 V_0 + ... + P_{j-1} V_{j-1} relative to the old max:
        // wait until the last of those products has landed, then rescale.
        // o_done has completed either j-1 times (S_j was issued after the
        // (j-1)-th product) or j times (O += P_j V_j waits for this thread), so
        // the parity of completion j identifies it without ambiguity.
        if (!mbar_wait_warp(o_done, (j - 1) & 1, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < D; c += 32) {
          uint32_t orow[32];
          tmem_ld32(tO + lane_off + c, orow);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 32; ++e) orow[e] = __float_as_uint(__uint_as_float(orow[e]) * alpha);
          tmem_st32(tO + lane_off + c, orow);
        }
      }
      m = m_use;
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&p_full[sb]);
    }
    if (ok && n_kv > 0 && mbar_wait_warp(o_final, 0, abort_flag)) {
      tc_fence_after();
      const float inv_l = (l > 0.f) ? 1.f / l : 0.f;
      const bool valid = row_g < p.N;
      __nv_bfloat16* orow_g = p.o + (static_cast<size_t>(bh) * p.N + row_g) * D;
#pragma unroll
      for (int c = 0; c < D; c += 32) {
        uint32_t orow[32];
        tmem_ld32(tO + lane_off + c, orow);
        tmem_ld_wait();
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
      if (valid && p.lse != nullptr) {
        // LSE = ln(sum exp(scale * s)) = (m + log2 l) * ln 2, m in log2 units.
        const float lse = (l > 0.f) ? (m + lg2_approx(l)) * 0.6931471805599453f : -INFINITY;
        p.lse[static_cast<size_t>(bh) * p.N + row_g] = lse;
      }
    }
    tmem_ld_wait();
    tmem_st_wait();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

template <int D, bool CAUSAL>
fa_status launch(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                 const Params& prm, int BH, cudaStream_t stream) {
  auto kern = fa_fwd_kernel<D, CAUSAL>;
  static bool configured = false;  // per process; the attribute is per function
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         Smem<D>::ALLOC);
    if (e != cudaSuccess) return FA_ERR_CUDA;
    configured = true;
  }
  dim3 grid(BH, prm.n_q_tiles);
  kern<<<grid, NUM_THREADS, Smem<D>::ALLOC, stream>>>(tq, tk, tv, prm);
  return cuda_status(cudaGetLastError());
}

}  // namespace fwd

fa_status launch_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                     int H, int N, int d, int causal, float scale, cudaStream_t stream) {
  const int BH = B * H;
  CUtensorMap tq, tk, tv;
  fa_status st;
  if ((st = make_tmap_bf16_3d(&tq, q, d, N, BH, fwd::BLOCK_M)) != FA_OK) return st;
  if ((st = make_tmap_bf16_3d(&tk, k, d, N, BH, fwd::BLOCK_N)) != FA_OK) return st;
  if ((st = make_tmap_bf16_3d(&tv, v, d, N, BH, fwd::BLOCK_N)) != FA_OK) return st;
  fwd::Params prm;
  prm.o = static_cast<__nv_bfloat16*>(o);
  prm.lse = lse;
  prm.N = N;
  prm.n_q_tiles = (N + fwd::BLOCK_M - 1) / fwd::BLOCK_M;
  prm.scale_log2 = scale * 1.4426950408889634f;
  if (d == 128)
    return causal ? fwd::launch<128, true>(tq, tk, tv, prm, BH, stream)
                  : fwd::launch<128, false>(tq, tk, tv, prm, BH, stream);
  return causal ? fwd::launch<64, true>(tq, tk, tv, prm, BH, stream)
                : fwd::launch<64, false>(tq, tk, tv, prm, BH, stream);
}

}  // namespace fa
