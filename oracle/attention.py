"""Plain, slow, fp64 CPU oracle for exact scaled-dot-product attention.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
module.  The product path (the CUDA library and its Python binding) never calls
it, and this module imports nothing from the product package: callers hand it
numpy float64 arrays holding the exact values of the bf16 inputs.

Sources (page titles and sections):

* "Flash Attention: principle & practice" (holysheep.ai), §1.2 (standard
  attention S = QK^T, P = softmax(S), O = PV) and §2.1 (numerically stable
  softmax; online softmax with a running maximum m and running denominator d).
* "DL101 chapter 9" (handsonai.io), §1.1 (attention of the newest token over
  the cached keys K_{<=t}, values V_{<=t}, scaled by 1/sqrt(d_k)) and §3.3
  (tiled FlashAttention: l <- l*c + rowsum(P), O <- O*c + P V, one final
  division O / l).
* "Flash Attention La Gi?" (thienlv.com glossary), "Recomputation": the
  backward pass recomputes the attention matrix from Q, K, V instead of
  storing it.  The pages give no backward formulas; the ones below are the
  standard calculus of softmax written out (loss L = sum(O * dO)).

What the oracle computes is the plain definition: for every query row it
materialises the full score row and the full probability row.  Row blocks of
queries are processed one after another only to bound memory; rows are
independent in the definition, and no arithmetic inside a row is reordered.

Readings taken where the pages are silent or inconsistent:

* LSE (log-sum-exp) is never defined on the pages.  It is read as the natural
  logarithm of the row's softmax denominator over the *scaled* scores:
  LSE_i = m_i + ln(sum_j exp(s_ij - m_i)).
* Causal masking keeps keys j <= i (token t attends K_{<=t}); the diagonal is
  included.  With Nq != Nk the queries are read as the last Nq positions of
  the Nk-token sequence (a chunk of new tokens over a cache): query i attends
  keys j <= i + Nk - Nq (bottom-right alignment); queries that see no key
  get O = 0 and LSE = -inf.
* A row with no admissible key (decode with seqlen 0) has O = 0, LSE = -inf.
* The tiled page-1 code divides O by l inside the loop and resets l to the
  block sum; that is only right for one key block.  The tiled routine here
  follows the page-2 recurrence (carry l*c, divide once at the end).

Parity status: every public function below is pinned by tests in
``tests/test_oracle_pins.py`` (closed forms, invariants, finite differences, an
independent library routine, and the page-2 worked example).
"""

from __future__ import annotations

import math
from typing import Iterable, Sequence

import numpy as np

__all__ = [
    "softmax_rows",
    "expand_kv_heads",
    "attention_forward",
    "attention_forward_rows",
    "attention_backward",
    "decode_forward",
    "online_softmax_stats",
    "tiled_attention_forward",
    "merge_softmax_partials",
]

_ROW_BLOCK = 512  # query rows materialised at once (memory bound only)


def _check_f64(*arrays: np.ndarray) -> None:
    for a in arrays:
        if not isinstance(a, np.ndarray) or a.dtype != np.float64:
            raise TypeError("oracle inputs must be numpy float64 arrays")


def softmax_rows(s: np.ndarray) -> np.ndarray:
    """Numerically stable softmax along the last axis.

    "Flash Attention: principle & practice", §2.1: subtract the row maximum
    before exponentiating, divide by the sum.  Entries equal to -inf (masked)
    get probability 0.  A row that is entirely -inf yields all zeros.
    """
    m = np.max(s, axis=-1, keepdims=True)
    m_safe = np.where(np.isfinite(m), m, 0.0)
    e = np.exp(s - m_safe)
    tot = np.sum(e, axis=-1, keepdims=True)
    with np.errstate(invalid="ignore", divide="ignore"):
        p = np.where(tot > 0, e / np.where(tot > 0, tot, 1.0), 0.0)
    return p


def _scores(q_rows: np.ndarray, k: np.ndarray, scale: float,
            row_index: np.ndarray | None, causal: bool, offset: int = 0) -> np.ndarray:
    """Scaled scores s_ij = scale * q_i . k_j, masked to -inf where j > i + offset
    (offset = Nk - Nq: query i sits at position i + offset of the key sequence)."""
    s = scale * (q_rows @ k.T)
    if causal:
        cols = np.arange(k.shape[0])[None, :]
        s = np.where(cols > row_index[:, None] + offset, -np.inf, s)
    return s


def _row_stats(s: np.ndarray):
    """Per-row (P, LSE) from a block of scaled, masked scores."""
    m = np.max(s, axis=-1)
    finite = np.isfinite(m)
    m_safe = np.where(finite, m, 0.0)
    e = np.exp(s - m_safe[:, None])
    l = np.sum(e, axis=-1)
    with np.errstate(divide="ignore", invalid="ignore"):
        p = np.where(l[:, None] > 0, e / np.where(l > 0, l, 1.0)[:, None], 0.0)
        lse = np.where(l > 0, m_safe + np.log(np.where(l > 0, l, 1.0)), -np.inf)
    return p, lse


def expand_kv_heads(x: np.ndarray, n_heads: int) -> np.ndarray:
    """Grouped-query attention ("DL101 chapter 9", §3.1 MQA and §3.2 GQA): the
    query heads are split into groups of H / Hkv consecutive heads and every
    group shares one key/value head.  Returns x [B, Hkv, L, d] repeated to
    [B, H, L, d] (query head h reads key/value head h // (H / Hkv))."""
    hkv = x.shape[-3]
    if n_heads % hkv:
        raise ValueError("the number of query heads must be a multiple of the K/V heads")
    return np.repeat(x, n_heads // hkv, axis=-3)


def attention_forward(q: np.ndarray, k: np.ndarray, v: np.ndarray,
                      causal: bool, scale: float):
    """O = softmax(scale * Q K^T [+ causal mask]) V and LSE, per (batch, head).

    Shapes: q [..., Nq, d], k and v [..., Nk, d] (same leading dims; with
    [B, H, N, d] queries, k and v may carry fewer heads Hkv dividing H, which
    grouped-query attention shares between groups of query heads).  Returns
    o [..., Nq, d] and lse [..., Nq], both float64.

    "Flash Attention: principle & practice", §1.2 (S = QK^T * scale,
    P = softmax(S), O = PV); "DL101 chapter 9", §1.1 (causal: K_{<=t}).
    """
    _check_f64(q, k, v)
    if q.ndim == 4 and k.ndim == 4 and k.shape[1] != q.shape[1]:
        k, v = expand_kv_heads(k, q.shape[1]), expand_kv_heads(v, q.shape[1])
    offset = k.shape[-2] - q.shape[-2]
    lead = q.shape[:-2]
    nq, d = q.shape[-2:]
    qf = q.reshape((-1, nq, d))
    kf = k.reshape((-1,) + k.shape[-2:])
    vf = v.reshape((-1,) + v.shape[-2:])
    o = np.zeros((qf.shape[0], nq, v.shape[-1]))
    lse = np.zeros((qf.shape[0], nq))
    for bh in range(qf.shape[0]):
        for r0 in range(0, nq, _ROW_BLOCK):
            rows = np.arange(r0, min(nq, r0 + _ROW_BLOCK))
            s = _scores(qf[bh, rows], kf[bh], scale, rows, causal, offset)
            p, lse_blk = _row_stats(s)
            o[bh, rows] = p @ vf[bh]
            lse[bh, rows] = lse_blk
    return o.reshape(lead + (nq, v.shape[-1])), lse.reshape(lead + (nq,))


def attention_forward_rows(q: np.ndarray, k: np.ndarray, v: np.ndarray,
                           causal: bool, scale: float, rows: Sequence[int]):
    """The same definition evaluated for a chosen set of query rows only.

    q, k, v are one (batch, head): [N, d].  Returns (o [len(rows), d],
    lse [len(rows)]).  Used to check full-size outputs row by row.
    """
    _check_f64(q, k, v)
    rows = np.asarray(rows, dtype=np.int64)
    s = _scores(q[rows], k, scale, rows, causal, k.shape[0] - q.shape[0])
    p, lse = _row_stats(s)
    return p @ v, lse


def attention_backward(q: np.ndarray, k: np.ndarray, v: np.ndarray,
                       do: np.ndarray, causal: bool, scale: float):
    """Gradients of L = sum(O * dO) with respect to Q, K, V.

    Recomputes the attention matrix from Q, K, V ("Flash Attention La Gi?",
    Recomputation).  With P = softmax(S), S = scale * Q K^T (masked):
        dV = P^T dO
        dP = dO V^T
        D_i = sum_j P_ij dP_ij
        dS = P * (dP - D)          (zero where masked, since P is zero there)
        dQ = scale * dS K
        dK = scale * dS^T Q
    Shapes as in ``attention_forward`` (causal with Nq != Nk: bottom-right
    aligned, rows that see no key get zero gradient).  With grouped
    K/V heads the gradient of a shared head is the sum over its group of
    query heads.  Returns (dq, dk, dv, D) with D = the row term above,
    float64.
    """
    _check_f64(q, k, v, do)
    if q.ndim == 4 and k.ndim == 4 and k.shape[1] != q.shape[1]:
        H, hkv = q.shape[1], k.shape[1]
        dq, dk, dv, D = attention_backward(q, expand_kv_heads(k, H), expand_kv_heads(v, H),
                                           do, causal, scale)
        g = H // hkv
        dk = dk.reshape(dk.shape[0], hkv, g, *dk.shape[2:]).sum(axis=2)
        dv = dv.reshape(dv.shape[0], hkv, g, *dv.shape[2:]).sum(axis=2)
        return dq, dk, dv, D
    lead = q.shape[:-2]
    nq, d = q.shape[-2:]
    nk = k.shape[-2]
    qf, kf, vf = (x.reshape((-1,) + x.shape[-2:]) for x in (q, k, v))
    dof = do.reshape((-1,) + do.shape[-2:])
    dq = np.zeros_like(qf)
    dk = np.zeros_like(kf)
    dv = np.zeros_like(vf)
    dD = np.zeros((qf.shape[0], nq))
    rows = np.arange(nq)
    for bh in range(qf.shape[0]):
        s = _scores(qf[bh], kf[bh], scale, rows, causal, nk - nq)
        p, _ = _row_stats(s)
        dv[bh] = p.T @ dof[bh]
        dp = dof[bh] @ vf[bh].T
        D = np.sum(p * dp, axis=-1)
        ds = p * (dp - D[:, None])
        dq[bh] = scale * (ds @ kf[bh])
        dk[bh] = scale * (ds.T @ qf[bh])
        dD[bh] = D
    shape_k = lead + (nk, d)
    return (dq.reshape(q.shape), dk.reshape(shape_k),
            dv.reshape(lead + (nk, v.shape[-1])), dD.reshape(lead + (nq,)))


def decode_forward(q: np.ndarray, kcache: np.ndarray, vcache: np.ndarray,
                   seqlens: Sequence[int], scale: float):
    """Single-query attention over a KV cache prefix.

    "DL101 chapter 9", §1.1: the newest query attends the cached keys and
    values of positions 0 .. L_b - 1 (non-causal within the prefix).
    q [B, H, d]; kcache, vcache [B, H, Lmax, d] (or [B, Hkv, Lmax, d], key/
    value heads shared by groups of H / Hkv query heads); seqlens [B] with
    0 <= L_b <= Lmax.  Cache rows at or beyond L_b are never read (they may
    hold anything, NaN included).  Returns o [B, H, d], lse [B, H]; a
    sequence with L_b == 0 gives o = 0, lse = -inf.
    """
    _check_f64(q, kcache, vcache)
    if kcache.shape[1] != q.shape[1]:
        kcache = expand_kv_heads(kcache, q.shape[1])
        vcache = expand_kv_heads(vcache, q.shape[1])
    B, H, d = q.shape
    o = np.zeros((B, H, vcache.shape[-1]))
    lse = np.full((B, H), -np.inf)
    for b in range(B):
        L = int(seqlens[b])
        if L == 0:
            continue
        for h in range(H):
            kk = kcache[b, h, :L]
            vv = vcache[b, h, :L]
            s = scale * (kk @ q[b, h])
            p, l = _row_stats(s[None, :])
            o[b, h] = (p @ vv)[0]
            lse[b, h] = l[0]
    return o, lse


def online_softmax_stats(chunks: Iterable[np.ndarray]):
    """Running (m, d) over a row delivered chunk by chunk.

    "Flash Attention: principle & practice", §2.1:
        m_i = max(m_{i-1}, max(chunk_i))
        d_i = d_{i-1} * exp(m_{i-1} - m_i) + sum(exp(chunk_i - m_i))
    so that softmax(x)_j = exp(x_j - m_n) / d_n.  Returns (m_n, d_n).
    """
    m_prev, d_prev = -math.inf, 0.0
    for c in chunks:
        c = np.asarray(c, dtype=np.float64)
        if c.size == 0:
            continue
        m_cur = max(m_prev, float(np.max(c)))
        if m_cur == -math.inf:
            continue
        corr = 0.0 if m_prev == -math.inf else math.exp(m_prev - m_cur)
        d_prev = d_prev * corr + float(np.sum(np.exp(c - m_cur)))
        m_prev = m_cur
    return m_prev, d_prev


def tiled_attention_forward(q: np.ndarray, k: np.ndarray, v: np.ndarray,
                            scale: float, block_q: int, block_k: int,
                            causal: bool = False):
    """Tile-by-tile forward with the running max / sum recurrence.

    "DL101 chapter 9", §3.3, for one (batch, head): q [Nq, d], k, v [Nk, d].
    For each query block, over key blocks j:
        S = scale * Q_blk K_j^T (masked)
        m' = max(m, rowmax S);  P = exp(S - m');  c = exp(m - m')
        l' = l * c + rowsum P;   O' = O * c + P V_j
    and after the last key block O / l.  Returns (o, lse) with
    lse = m + ln l.  The N x N matrix is never formed.
    """
    _check_f64(q, k, v)
    nq, d = q.shape
    nk = k.shape[0]
    o = np.zeros((nq, v.shape[1]))
    lse = np.full(nq, -np.inf)
    for i0 in range(0, nq, block_q):
        i1 = min(nq, i0 + block_q)
        rows = np.arange(i0, i1)
        m = np.full(i1 - i0, -np.inf)
        l = np.zeros(i1 - i0)
        acc = np.zeros((i1 - i0, v.shape[1]))
        for j0 in range(0, nk, block_k):
            j1 = min(nk, j0 + block_k)
            s = scale * (q[i0:i1] @ k[j0:j1].T)
            if causal:
                cols = np.arange(j0, j1)[None, :]
                s = np.where(cols > rows[:, None], -np.inf, s)
            m_new = np.maximum(m, np.max(s, axis=1))
            m_ref = np.where(np.isfinite(m_new), m_new, 0.0)
            p = np.exp(s - m_ref[:, None])
            c = np.where(np.isfinite(m), np.exp(m - m_ref), 0.0)
            l = l * c + np.sum(p, axis=1)
            acc = acc * c[:, None] + p @ v[j0:j1]
            m = m_new
        with np.errstate(divide="ignore", invalid="ignore"):
            o[i0:i1] = np.where(l[:, None] > 0, acc / np.where(l > 0, l, 1.0)[:, None], 0.0)
            lse[i0:i1] = np.where(l > 0, m + np.log(np.where(l > 0, l, 1.0)), -np.inf)
    return o, lse


def merge_softmax_partials(m: np.ndarray, l: np.ndarray, acc: np.ndarray):
    """Merge per-chunk softmax partials into the final output and LSE.

    Each chunk s contributes its own maximum m_s, denominator
    l_s = sum exp(x - m_s) and unnormalised output acc_s = sum exp(x - m_s) v.
    This is the §2.1 recurrence of "Flash Attention: principle & practice"
    applied to whole chunks at once:
        M = max_s m_s;  w_s = exp(m_s - M)
        o = sum_s w_s acc_s / sum_s w_s l_s;  lse = M + ln(sum_s w_s l_s)
    m, l: [S]; acc: [S, d].  Chunks with m_s = -inf (empty) weigh 0.
    """
    m = np.asarray(m, dtype=np.float64)
    l = np.asarray(l, dtype=np.float64)
    acc = np.asarray(acc, dtype=np.float64)
    M = np.max(m) if m.size else -np.inf
    if not np.isfinite(M):
        return np.zeros(acc.shape[-1]), -np.inf
    w = np.where(np.isfinite(m), np.exp(m - M), 0.0)
    L = float(np.sum(w * l))
    o = np.sum(w[:, None] * acc, axis=0) / L
    return o, M + math.log(L)
