"""Pins for the fp64 oracle: facts fixed by the pages and by mathematics.

None of these re-types the oracle's formulas.  Each check compares the oracle
with a closed form, an invariant, finite differences, an independent library
routine (torch CPU scaled_dot_product_attention / logsumexp in float64) or the
worked example printed on "DL101 chapter 9", §3.3.  The mutation tests at the
end plant plausible mistakes in copies of the oracle and require at least one
pin to reject each.
"""

import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import attention as A

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
RNG = np.random.default_rng(1234)


def bf16_grid(shape, rng=RNG, std=1.0):
    """Random values that are exactly representable in bf16, as float64."""
    x = torch.from_numpy(rng.standard_normal(shape) * std).to(torch.bfloat16)
    return x.to(torch.float64).numpy()


# --------------------------------------------------------------------------
# pin checks, written against a forward function fwd(q, k, v, causal, scale)
# and a backward function bwd(q, k, v, do, causal, scale)
# --------------------------------------------------------------------------

def pin_constant_v(fwd):
    for causal in (False, True):
        q, k = bf16_grid((2, 9, 8)), bf16_grid((2, 9, 8))
        c = bf16_grid((1, 1, 8))
        v = np.broadcast_to(c, (2, 9, 8)).copy()
        o, _ = fwd(q, k, v, causal, 0.37)
        assert np.allclose(o, v, rtol=0, atol=1e-13), "constant V must give O = V"


def pin_zero_query(fwd):
    # q = 0: every admissible score is 0, so P is uniform over A(i).
    N, d = 7, 4
    q = np.zeros((N, d))
    k, v = bf16_grid((N, d)), bf16_grid((N, d))
    o, lse = fwd(q, k, v, False, 0.5)
    assert np.allclose(o, np.broadcast_to(v.mean(0), (N, d)), atol=1e-14)
    assert np.allclose(lse, math.log(N), atol=1e-14)
    o, lse = fwd(q, k, v, True, 0.5)
    counts = np.arange(1, N + 1)
    assert np.allclose(o, np.cumsum(v, 0) / counts[:, None], atol=1e-14), \
        "causal row i must average v_0..v_i"
    assert np.allclose(lse, np.log(counts), atol=1e-14)


def pin_causal_row0(fwd):
    q, k, v = bf16_grid((6, 8)), bf16_grid((6, 8)), bf16_grid((6, 8))
    s = 0.25
    o, lse = fwd(q, k, v, True, s)
    assert np.array_equal(o[0], v[0]), "causal row 0 attends only key 0"
    assert abs(lse[0] - s * float(np.dot(q[0], k[0]))) < 1e-14


def pin_two_keys(fwd):
    # One query, two keys with scores scale*a and 0: p_1 = logistic(scale*a).
    a, scale = 3.0, 0.5
    q = np.array([[1.0, 0.0]])
    k = np.array([[a, 0.0], [0.0, 0.0]])
    v = np.array([[1.0, 0.0], [0.0, 1.0]])
    o, lse = fwd(q, k, v, False, scale)
    p1 = 1.0 / (1.0 + math.exp(-scale * a))
    assert np.allclose(o[0], [p1, 1.0 - p1], atol=1e-15)
    assert abs(lse[0] - math.log(math.exp(scale * a) + 1.0)) < 1e-14


def pin_rows_sum_to_one(fwd):
    # V = identity makes O equal to P itself.
    for causal in (False, True):
        N = 10
        q, k = bf16_grid((N, 6)), bf16_grid((N, 6))
        p, _ = fwd(q, k, np.eye(N), causal, 0.8)
        assert np.allclose(p.sum(1), 1.0, atol=1e-14)
        assert (p >= 0).all()
        if causal:
            assert np.all(np.triu(p, 1) == 0.0), "causal P must vanish above the diagonal"
        else:
            assert (p > 0).all()


def pin_permutation(fwd):
    q, k, v = bf16_grid((5, 8)), bf16_grid((11, 8)), bf16_grid((11, 8))
    perm = RNG.permutation(11)
    o1, l1 = fwd(q, k, v, False, 0.3)
    o2, l2 = fwd(q, k[perm], v[perm], False, 0.3)
    assert np.allclose(o1, o2, atol=1e-14) and np.allclose(l1, l2, atol=1e-14)
    o3, _ = fwd(q, k, v[perm], False, 0.3)
    assert not np.allclose(o1, o3, atol=1e-6), "permuting V alone must change O"


def pin_sdpa(fwd):
    # Independent library routine: torch CPU SDPA in float64.
    for causal in (False, True):
        for (B, H, N, d) in ((1, 2, 33, 16), (2, 1, 64, 8)):
            q, k, v = (bf16_grid((B, H, N, d)) for _ in range(3))
            scale = 1.0 / math.sqrt(d) * 1.3
            o, lse = fwd(q, k, v, causal, scale)
            tq, tk, tv = (torch.from_numpy(x) for x in (q, k, v))
            ref = torch.nn.functional.scaled_dot_product_attention(
                tq, tk, tv, is_causal=causal, scale=scale).numpy()
            s = scale * (tq @ tk.transpose(-1, -2))
            if causal:
                s = s.masked_fill(torch.ones(N, N, dtype=torch.bool).triu(1), -math.inf)
            ref_lse = torch.logsumexp(s, dim=-1).numpy()
            assert np.allclose(o, ref, atol=1e-12), "O differs from torch SDPA"
            assert np.allclose(lse, ref_lse, atol=1e-12), "LSE differs from logsumexp"


FWD_PINS = [pin_constant_v, pin_zero_query, pin_causal_row0, pin_two_keys,
            pin_rows_sum_to_one, pin_permutation, pin_sdpa]


def _loss(fwd, q, k, v, do, causal, scale):
    o, _ = fwd(q, k, v, causal, scale)
    return float(np.sum(o * do))


def pin_finite_differences(bwd, fwd=A.attention_forward):
    rng = np.random.default_rng(7)
    for causal in (False, True):
        N, d = 6, 5
        q, k, v, do = (rng.standard_normal((N, d)) for _ in range(4))
        scale = 0.7
        dq, dk, dv = bwd(q, k, v, do, causal, scale)[:3]
        h = 1e-6
        for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
            num = np.zeros_like(x)
            for idx in np.ndindex(x.shape):
                xp, xm = x.copy(), x.copy()
                xp[idx] += h
                xm[idx] -= h
                args_p = {"q": q, "k": k, "v": v}
                args_m = dict(args_p)
                args_p[name], args_m[name] = xp, xm
                num[idx] = (_loss(fwd, args_p["q"], args_p["k"], args_p["v"], do, causal, scale)
                            - _loss(fwd, args_m["q"], args_m["k"], args_m["v"], do, causal, scale)) / (2 * h)
            assert np.allclose(g, num, atol=1e-7, rtol=1e-6), f"d{name} disagrees with finite differences"


def pin_autograd(bwd):
    # Independent library routine: torch autograd through SDPA in float64.
    for causal in (False, True):
        q, k, v, do = (bf16_grid((1, 2, 40, 16)) for _ in range(4))
        scale = 0.2
        tq, tk, tv = (torch.from_numpy(x).requires_grad_() for x in (q, k, v))
        o = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=causal, scale=scale)
        o.backward(torch.from_numpy(do))
        dq, dk, dv, D = bwd(q, k, v, do, causal, scale)
        for a, b in ((dq, tq.grad), (dk, tk.grad), (dv, tv.grad)):
            assert np.allclose(a, b.numpy(), atol=1e-11)
        assert np.allclose(D, np.sum(o.detach().numpy() * do, -1), atol=1e-11), \
            "D must equal rowsum(dO * O)"


# --------------------------------------------------------------------------
# the oracle passes every pin
# --------------------------------------------------------------------------

@pytest.mark.parametrize("pin", FWD_PINS, ids=lambda f: f.__name__)
def test_forward_pins(pin):
    pin(A.attention_forward)


def test_forward_rows_matches_full():
    q, k, v = (bf16_grid((300, 16)) for _ in range(3))
    rows = [0, 1, 127, 128, 299]
    for causal in (False, True):
        o, lse = A.attention_forward(q, k, v, causal, 0.25)
        orow, lrow = A.attention_forward_rows(q, k, v, causal, 0.25, rows)
        assert np.array_equal(orow, o[rows]) and np.array_equal(lrow, lse[rows])


def test_backward_finite_differences():
    pin_finite_differences(A.attention_backward)


def test_backward_autograd():
    pin_autograd(A.attention_backward)


def test_online_softmax_any_chunking():
    """Online softmax over any chunking equals the whole-row softmax."""
    for trial in range(20):
        x = RNG.standard_normal(int(RNG.integers(1, 200))) * 5
        cuts = np.sort(RNG.integers(0, x.size + 1, size=int(RNG.integers(0, 6))))
        chunks = np.split(x, cuts)
        m, dn = A.online_softmax_stats(chunks)
        assert m == x.max()
        assert abs(dn - np.exp(x - x.max()).sum()) < 1e-12 * x.size
        ref = torch.softmax(torch.from_numpy(x), 0).numpy()
        assert np.allclose(np.exp(x - m) / dn, ref, atol=1e-15)


def test_merge_partials_random_splits():
    """Merging per-chunk (m, l, acc) reproduces the single-query result."""
    for trial in range(10):
        L, d = int(RNG.integers(1, 300)), 8
        q, k, v = bf16_grid((d,)), bf16_grid((L, d)), bf16_grid((L, d))
        scale = 0.35
        cuts = np.unique(RNG.integers(0, L + 1, size=int(RNG.integers(0, 7))))
        ms, ls, accs = [], [], []
        for ks, vs in zip(np.split(k, cuts), np.split(v, cuts)):
            if ks.shape[0] == 0:
                ms.append(-np.inf); ls.append(0.0); accs.append(np.zeros(d))
                continue
            s = scale * ks @ q
            mm = s.max()
            e = np.exp(s - mm)
            ms.append(mm); ls.append(e.sum()); accs.append(e @ vs)
        o, lse = A.merge_softmax_partials(np.array(ms), np.array(ls), np.array(accs))
        ref_o, ref_l = A.attention_forward(q[None], k, v, False, scale)
        assert np.allclose(o, ref_o[0], atol=1e-13) and abs(lse - ref_l[0]) < 1e-12


def test_tiled_equals_plain_ragged():
    for causal in (False, True):
        N = 77
        q, k, v = (bf16_grid((N, 16)) for _ in range(3))
        o_t, l_t = A.tiled_attention_forward(q, k, v, 0.25, 16, 24, causal)
        o_p, l_p = A.attention_forward(q, k, v, causal, 0.25)
        assert np.allclose(o_t, o_p, atol=1e-13) and np.allclose(l_t, l_p, atol=1e-13)


def test_page_worked_example_tiled_vs_sdpa():
    """DL101 chapter 9, §3.3: tiled loop vs SDPA prints MSE 0.0000000000."""
    with open(os.path.join(GOLDEN, "dl101_ch9_tiled_vs_sdpa.json")) as f:
        g = json.load(f)
    gen = torch.Generator().manual_seed(g["seed"])
    Q = torch.randn(g["Lq"], g["d"], generator=gen)
    K = torch.randn(g["Lk"], g["d"], generator=gen)
    V = torch.randn(g["Lk"], g["d"], generator=gen)
    o_t, _ = A.tiled_attention_forward(Q.double().numpy(), K.double().numpy(), V.double().numpy(),
                                       g["d"] ** -0.5, g["block_q"], g["block_k"])
    ref = torch.nn.functional.scaled_dot_product_attention(Q, K, V).double().numpy()
    mse = float(np.mean((o_t - ref) ** 2))
    bound = 0.5 * 10.0 ** (-g["printed_digits"])
    assert f"{mse:.10f}" == g["printed_mse"] and mse < bound


def test_decode_matches_sdpa_and_ignores_poison():
    B, H, d, Lcap = 3, 2, 16, 40
    seqlens = [0, 1, 37]
    q = bf16_grid((B, H, d))
    kc = np.full((B, H, Lcap, d), np.nan)
    vc = np.full((B, H, Lcap, d), np.nan)
    for b, L in enumerate(seqlens):
        kc[b, :, :L] = bf16_grid((H, L, d))
        vc[b, :, :L] = bf16_grid((H, L, d))
    o, lse = A.decode_forward(q, kc, vc, seqlens, 0.25)
    assert np.all(o[0] == 0) and np.all(np.isneginf(lse[0])), "empty prefix: O = 0, LSE = -inf"
    assert np.array_equal(o[1], vc[1, :, 0]), "one cached key: O = v_0"
    for b in (1, 2):
        L = seqlens[b]
        tq = torch.from_numpy(q[b][:, None, :])
        ref = torch.nn.functional.scaled_dot_product_attention(
            tq, torch.from_numpy(kc[b, :, :L]), torch.from_numpy(vc[b, :, :L]), scale=0.25)
        assert np.allclose(o[b], ref[:, 0].numpy(), atol=1e-13)
        s = 0.25 * torch.einsum("hd,hld->hl", torch.from_numpy(q[b]), torch.from_numpy(kc[b, :, :L]))
        assert np.allclose(lse[b], torch.logsumexp(s, -1).numpy(), atol=1e-13)
    assert np.isfinite(o[1:]).all()


# --------------------------------------------------------------------------
# planted mistakes: each mutant of the oracle must fail at least one pin
# --------------------------------------------------------------------------

def _mutant_fwd(kind):
    def fwd(q, k, v, causal, scale):
        q, k, v = (np.asarray(x, np.float64) for x in (q, k, v))
        N, M = q.shape[-2], k.shape[-2]
        sc = 1.0 if kind == "no_scale" else scale
        s = sc * (q @ np.swapaxes(k, -1, -2))
        if causal:
            i = np.arange(N)[:, None]
            j = np.arange(M)[None, :]
            bad = {"mask_flipped": j < i, "mask_no_diag": j >= i}.get(kind, j > i)
            s = np.where(bad, -np.inf, s)
        m = s.max(-1, keepdims=True)
        e = np.exp(s - m)
        l = e.sum(-1, keepdims=True)
        p = e / l
        if kind == "transposed_p":
            p = np.swapaxes(p, -1, -2)
        o = p @ v
        lse = (m + np.log(l))[..., 0]
        if kind == "lse_no_max":
            lse = np.log(l)[..., 0]
        return o, lse
    return fwd


def _page1_tiled_fwd(q, k, v, causal, scale):
    """The page-1 recurrence (l reset to the block sum, O divided in the loop)."""
    if q.ndim > 2:
        outs = [_page1_tiled_fwd(q[i], k[i], v[i], causal, scale) for i in range(q.shape[0])]
        return np.stack([o for o, _ in outs]), np.stack([l for _, l in outs])
    N, bq, bk = q.shape[0], 4, 4
    o = np.zeros((N, v.shape[1]))
    lse = np.zeros(N)
    for i0 in range(0, N, bq):
        oi = np.zeros((min(bq, N - i0), v.shape[1]))
        mi = np.full(oi.shape[0], -np.inf)
        li = np.zeros(oi.shape[0])
        rows = np.arange(i0, i0 + oi.shape[0])
        for j0 in range(0, k.shape[0], bk):
            s = scale * q[i0:i0 + bq] @ k[j0:j0 + bk].T
            if causal:
                s = np.where(np.arange(j0, j0 + s.shape[1])[None] > rows[:, None], -np.inf, s)
            mn = np.maximum(mi, s.max(1))
            p = np.exp(s - mn[:, None])
            ln = p.sum(1)
            with np.errstate(invalid="ignore"):
                c = np.nan_to_num(np.exp(mi - mn))
            oi = (c[:, None] * oi + p @ v[j0:j0 + bk]) / ln[:, None]
            mi, li = mn, ln
        o[i0:i0 + bq] = oi
        lse[i0:i0 + bq] = mi + np.log(li)
    return o, lse


@pytest.mark.parametrize("kind", ["no_scale", "mask_flipped", "mask_no_diag",
                                  "transposed_p", "lse_no_max", "page1_recurrence"])
def test_pins_reject_planted_forward_mistakes(kind):
    fwd = _page1_tiled_fwd if kind == "page1_recurrence" else _mutant_fwd(kind)
    failures = 0
    for pin in FWD_PINS:
        try:
            with np.errstate(all="ignore"):
                pin(fwd)
        except (AssertionError, ValueError):
            failures += 1
    assert failures >= 1, f"no pin caught the planted mistake {kind!r}"


def _mutant_bwd(kind):
    def bwd(q, k, v, do, causal, scale):
        dq, dk, dv, D = A.attention_backward(q, k, v, do, causal, scale)
        N = q.shape[-2]
        s = scale * q @ k.T
        if causal:
            s = np.where(np.triu(np.ones((N, N), bool), 1), -np.inf, s)
        p = oracle.softmax_rows(s)
        dp = do @ v.T
        if kind == "drop_D":
            ds = p * dp
            dq, dk = scale * ds @ k, scale * ds.T @ q
        elif kind == "dq_no_scale":
            dq = dq / scale
        elif kind == "dk_untransposed":
            ds = p * (dp - np.sum(p * dp, -1, keepdims=True))
            dk = scale * ds @ q
        elif kind == "dv_untransposed":
            dv = p @ do
        return dq, dk, dv, D
    return bwd


@pytest.mark.parametrize("kind", ["drop_D", "dq_no_scale", "dk_untransposed", "dv_untransposed"])
def test_pins_reject_planted_backward_mistakes(kind):
    with pytest.raises(AssertionError):
        pin_finite_differences(_mutant_bwd(kind))


def test_grouped_query_attention_matches_sdpa_enable_gqa():
    """"DL101 chapter 9", §3.1-3.2 compute MQA / GQA with torch SDPA's
    enable_gqa; the oracle's grouped heads must agree with that routine."""
    for hkv in (1, 2, 4):
        for causal in (False, True):
            q = bf16_grid((2, 8, 40, 16))
            k, v = bf16_grid((2, hkv, 40, 16)), bf16_grid((2, hkv, 40, 16))
            o, lse = A.attention_forward(q, k, v, causal, 0.3)
            ref = torch.nn.functional.scaled_dot_product_attention(
                *(torch.from_numpy(x) for x in (q, k, v)), is_causal=causal, scale=0.3,
                enable_gqa=True).numpy()
            assert np.allclose(o, ref, atol=1e-12)


def test_grouped_query_backward_matches_autograd():
    for hkv in (1, 2):
        q, do = bf16_grid((1, 4, 24, 8)), bf16_grid((1, 4, 24, 8))
        k, v = bf16_grid((1, hkv, 24, 8)), bf16_grid((1, hkv, 24, 8))
        tq, tk, tv = (torch.from_numpy(x).requires_grad_() for x in (q, k, v))
        o = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=True, scale=0.4,
                                                             enable_gqa=True)
        o.backward(torch.from_numpy(do))
        dq, dk, dv, _ = A.attention_backward(q, k, v, do, True, 0.4)
        for a, b in ((dq, tq.grad), (dk, tk.grad), (dv, tv.grad)):
            assert a.shape == b.shape and np.allclose(a, b.numpy(), atol=1e-11)


def test_grouped_decode_matches_expanded_cache():
    q = bf16_grid((2, 6, 8))
    kc, vc = bf16_grid((2, 3, 30, 8)), bf16_grid((2, 3, 30, 8))
    o, lse = A.decode_forward(q, kc, vc, [30, 11], 0.5)
    for b, L in enumerate([30, 11]):
        for h in range(6):
            ref = torch.nn.functional.scaled_dot_product_attention(
                torch.from_numpy(q[b, h][None, None]), torch.from_numpy(kc[b, h // 2, :L][None]),
                torch.from_numpy(vc[b, h // 2, :L][None]), scale=0.5)
            assert np.allclose(o[b, h], ref[0, 0].numpy(), atol=1e-13)


def test_unequal_lengths_match_sdpa_with_bottom_right_mask():
    """Nq != Nk: non-causal against plain SDPA (the DL101 chapter 9 section 3.3
    example uses Lq = 1280, Lk = 1152); causal against SDPA with an explicit
    bottom-right mask tril(Nk - Nq)."""
    for (nq, nk) in ((40, 29), (17, 50), (1, 33)):
        q = bf16_grid((1, 2, nq, 16))
        k, v = bf16_grid((1, 2, nk, 16)), bf16_grid((1, 2, nk, 16))
        for causal in (False, True):
            o, lse = A.attention_forward(q, k, v, causal, 0.25)
            mask = torch.ones(nq, nk, dtype=torch.bool)
            if causal:
                mask = mask.tril(nk - nq)
            tq, tk, tv = (torch.from_numpy(x) for x in (q, k, v))
            ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, attn_mask=mask,
                                                                   scale=0.25).numpy()
            empty = ~mask.any(dim=1).numpy()  # rows with no admissible key
            assert np.allclose(o[..., ~empty, :], ref[..., ~empty, :], atol=1e-12)
            assert np.all(o[..., empty, :] == 0) and np.all(np.isneginf(lse[..., empty]))
            s = 0.25 * (tq @ tk.transpose(-1, -2))
            ref_lse = torch.logsumexp(s.masked_fill(~mask, -math.inf), -1).numpy()
            assert np.allclose(lse[..., ~empty], ref_lse[..., ~empty], atol=1e-12)


def test_unequal_lengths_backward_matches_autograd():
    for (nq, nk) in ((24, 40), (40, 24)):
        q, do = bf16_grid((1, 2, nq, 8)), bf16_grid((1, 2, nq, 8))
        k, v = bf16_grid((1, 2, nk, 8)), bf16_grid((1, 2, nk, 8))
        mask = torch.ones(nq, nk, dtype=torch.bool).tril(nk - nq)
        keep = mask.any(dim=1)
        tq, tk, tv = (torch.from_numpy(x).requires_grad_() for x in (q, k, v))
        o = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, attn_mask=mask, scale=0.4)
        # rows without keys are NaN in SDPA; the definition gives them O = 0
        (o[..., keep, :] * torch.from_numpy(do)[..., keep, :]).sum().backward()
        dq, dk, dv, _ = A.attention_backward(q, k, v, do, True, 0.4)
        assert np.allclose(dq[..., keep.numpy(), :], tq.grad.numpy()[..., keep.numpy(), :], atol=1e-11)
        assert np.allclose(dk, tk.grad.numpy(), atol=1e-11) and np.allclose(dv, tv.grad.numpy(), atol=1e-11)


# --------------------------------------------------------------------------
# softmax_rows: the stable softmax of "Flash Attention: principle & practice",
# section 2.1, pinned against torch's float64 softmax, closed forms and
# invariants; planted mistakes in copies of it must each fail a pin.
# --------------------------------------------------------------------------

def pin_softmax_library(sm):
    s = RNG.standard_normal((5, 13)) * 3.0
    ref = torch.softmax(torch.from_numpy(s), dim=-1).numpy()
    assert np.allclose(sm(s), ref, rtol=0, atol=1e-15), "must equal torch.softmax in float64"


def pin_softmax_rows_sum_to_one(sm):
    s = RNG.standard_normal((4, 3, 9)) * 5.0
    p = sm(s)
    assert p.shape == s.shape and np.all(p >= 0)
    assert np.allclose(p.sum(-1), 1.0, atol=1e-14), "each row must sum to 1"


def pin_softmax_logistic(sm):
    # two entries a, b: p_0 = 1 / (1 + e^(b - a)) (closed form)
    for a, b in ((0.3, -1.2), (2.0, 2.0), (-4.0, 1.5)):
        p = sm(np.array([[a, b]]))
        assert abs(p[0, 0] - 1.0 / (1.0 + math.exp(b - a))) < 1e-15
        assert abs(p[0, 1] - 1.0 / (1.0 + math.exp(a - b))) < 1e-15


def pin_softmax_large_scores(sm):
    # stability: the maximum is subtracted first, so scores of 1000 and 999
    # give the logistic weights instead of inf / inf
    with np.errstate(all="ignore"):
        p = sm(np.array([[1000.0, 999.0]]))
    assert np.all(np.isfinite(p)) and abs(p[0, 0] - 1.0 / (1.0 + math.exp(-1.0))) < 1e-15


def pin_softmax_masked(sm):
    # -inf entries get probability 0; the rest is the softmax of the others;
    # a row that is entirely -inf gives zeros
    s = np.array([[0.5, -np.inf, 1.5, -np.inf], [-np.inf] * 4])
    with np.errstate(all="ignore"):
        p = sm(s)
    assert np.all(np.isfinite(p))
    assert p[0, 1] == 0.0 and p[0, 3] == 0.0
    assert abs(p[0, 0] - 1.0 / (1.0 + math.exp(1.0))) < 1e-15
    assert np.all(p[1] == 0.0), "a fully masked row must be all zeros"


def pin_softmax_shift_invariant(sm):
    s = RNG.standard_normal((3, 11))
    assert np.allclose(sm(s), sm(s + 7.25), atol=1e-15), "adding a constant to a row changes nothing"
    assert not np.allclose(sm(s), sm(2.0 * s), atol=1e-6), "scaling the scores must change P"


SOFTMAX_PINS = [pin_softmax_library, pin_softmax_rows_sum_to_one, pin_softmax_logistic,
                pin_softmax_large_scores, pin_softmax_masked, pin_softmax_shift_invariant]


@pytest.mark.parametrize("pin", SOFTMAX_PINS, ids=lambda f: f.__name__)
def test_softmax_rows_pins(pin):
    pin(oracle.softmax_rows)


def _mutant_softmax(kind):
    def sm(s):
        if kind == "no_max":
            e = np.exp(s)
            return e / e.sum(-1, keepdims=True)
        if kind == "wrong_axis":
            m = np.max(s, axis=0, keepdims=True)
            e = np.exp(s - np.where(np.isfinite(m), m, 0.0))
            tot = e.sum(0, keepdims=True)
            return np.where(tot > 0, e / np.where(tot > 0, tot, 1.0), 0.0)
        if kind == "sum_with_max":  # divides by the sum plus the (unshifted) max
            m = np.max(s, axis=-1, keepdims=True)
            e = np.exp(s - np.where(np.isfinite(m), m, 0.0))
            return e / (e.sum(-1, keepdims=True) + 1.0)
        if kind == "masked_row_nan":  # no guard for a fully masked row
            m = np.max(s, axis=-1, keepdims=True)
            e = np.exp(s - m)
            return e / e.sum(-1, keepdims=True)
        if kind == "exp_not_shifted_back":  # uses exp(s) / sum exp(s - m)
            m = np.max(s, axis=-1, keepdims=True)
            m0 = np.where(np.isfinite(m), m, 0.0)
            return np.exp(s) / np.exp(s - m0).sum(-1, keepdims=True)
        raise ValueError(kind)
    return sm


@pytest.mark.parametrize("kind", ["no_max", "wrong_axis", "sum_with_max", "masked_row_nan",
                                  "exp_not_shifted_back"])
def test_softmax_pins_reject_planted_mistakes(kind):
    sm = _mutant_softmax(kind)
    failures = 0
    for pin in SOFTMAX_PINS:
        try:
            with np.errstate(all="ignore"):
                pin(sm)
        except (AssertionError, ValueError, FloatingPointError):
            failures += 1
    assert failures >= 1, f"no pin caught the planted softmax mistake {kind!r}"
