"""GPU parity of the ragged-batch forward (fa_fwd_varlen) against the fp64
oracle, sequence by sequence.

Sequences of different lengths are packed token-major without padding; each
is exactly the attention problem of its own rows ("DL101 chapter 9", section
3.3, for Lq x Lk; causal masking bottom-right aligned per sequence).  Cases
cover empty sequences on either side, single rows, ragged tails, grouped
heads, a chunk of new tokens over a longer cache, and equality with the
padded kernel on a batch of equal lengths."""
import numpy as np
import pytest
import torch

import oracle
from io_aware_exact_35_b200 import inputs
from tests._parity import check_lse, check_o

pytestmark = pytest.mark.gpu

DEV = torch.device("cuda:0")


def _run(fa_mod, q, k, v, cu_q, cu_k, max_q, causal, scale):
    o, lse = fa_mod.fwd_varlen(q.to(DEV), k.to(DEV), v.to(DEV), cu_q.to(DEV), cu_k.to(DEV),
                               max_q, causal=causal, scale=scale)
    torch.cuda.synchronize()
    assert fa_mod.get_device_error() == 0
    return o.cpu(), lse.cpu()


def _check_per_sequence(q, k, v, cu_q, cu_k, o, lse, causal, scale):
    for b in range(len(cu_q) - 1):
        q0, q1, k0, k1 = int(cu_q[b]), int(cu_q[b + 1]), int(cu_k[b]), int(cu_k[b + 1])
        qb = inputs.to_f64(q[q0:q1].transpose(0, 1)[None])   # [1, H, Lq, d]
        kb = inputs.to_f64(k[k0:k1].transpose(0, 1)[None])
        vb = inputs.to_f64(v[k0:k1].transpose(0, 1)[None])
        if q1 == q0:
            continue
        if k1 == k0:
            assert torch.all(o[q0:q1] == 0) and torch.all(torch.isneginf(lse[:, q0:q1]))
            continue
        o_ref, lse_ref = oracle.attention_forward(qb, kb, vb, causal, scale)
        check_o(o[q0:q1].transpose(0, 1)[None], o_ref, f"O seq {b}")
        check_lse(lse[:, q0:q1][None], lse_ref, f"LSE seq {b}")


CASES = [
    # (lens_q, lens_k, H, Hkv, d)
    ([1, 200, 513, 0, 1000, 128], None, 2, 2, 128),
    ([300, 77, 256, 1], None, 4, 2, 64),
    ([100, 300, 5], [1000, 300, 700], 2, 1, 128),  # chunks over longer caches
    ([700, 40], [200, 0], 2, 2, 128),              # more queries than keys; no keys
]


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("case", CASES, ids=lambda c: "B%d_H%d_Hkv%d_d%d" % (len(c[0]), c[2], c[3], c[4]))
def test_fwd_varlen_matches_oracle(fa_mod, cuda_device, case, causal):
    lens_q, lens_k, H, Hkv, d = case
    lens_k = lens_k if lens_k is not None else lens_q
    q, k, v, cu_q, cu_k = inputs.varlen_inputs(lens_q, lens_k, H, Hkv, d, seed=6000 + d + causal)
    scale = 1.0 / np.sqrt(d)
    o, lse = _run(fa_mod, q, k, v, cu_q, cu_k, max(lens_q), causal, scale)
    _check_per_sequence(q, k, v, cu_q, cu_k, o, lse, causal, scale)


def test_fwd_varlen_equal_lengths_match_padded_kernel(fa_mod, cuda_device):
    """On a batch of equal lengths the packed and the padded layouts hold the
    same problem: outputs agree bit for bit (same tiles, same arithmetic)."""
    B, H, Hkv, N, d = 3, 4, 2, 777, 128
    q, k, v, cu_q, cu_k = inputs.varlen_inputs([N] * B, [N] * B, H, Hkv, d, seed=6100)
    for causal in (False, True):
        o, lse = _run(fa_mod, q, k, v, cu_q, cu_k, N, causal, 0.1)
        qd = q.view(B, N, H, d).transpose(1, 2).contiguous().to(DEV)
        kd = k.view(B, N, Hkv, d).transpose(1, 2).contiguous().to(DEV)
        vd = v.view(B, N, Hkv, d).transpose(1, 2).contiguous().to(DEV)
        od, lsed = fa_mod.fwd(qd, kd, vd, causal=causal, scale=0.1)
        torch.cuda.synchronize()
        assert torch.equal(o.view(B, N, H, d).transpose(1, 2), od.cpu())
        assert torch.equal(lse.view(H, B, N).transpose(0, 1), lsed.cpu())


BWD_CASES = [
    ([1, 200, 513, 0, 300], None, 2, 2, 128),
    ([300, 77, 256], None, 4, 2, 64),
    ([100, 300, 5], [1000, 300, 700], 2, 1, 128),
    ([700, 40, 9], [200, 0, 9], 2, 2, 128),
]


def _fwd_bwd_varlen(fa_mod, q, k, v, do, cu_q, cu_k, causal, scale):
    q, k, v, do, cu_q, cu_k = (t.to(DEV) for t in (q, k, v, do, cu_q, cu_k))
    lq = (cu_q[1:] - cu_q[:-1]).max().item()
    lk = (cu_k[1:] - cu_k[:-1]).max().item()
    o, lse = fa_mod.fwd_varlen(q, k, v, cu_q, cu_k, lq, causal=causal, scale=scale)
    dq, dk, dv = fa_mod.bwd_varlen(q, k, v, o, do, lse, cu_q, cu_k, lk, causal=causal,
                                   scale=scale)
    torch.cuda.synchronize()
    assert fa_mod.get_device_error() == 0
    return dq.cpu(), dk.cpu(), dv.cpu()


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("case", BWD_CASES, ids=lambda c: "B%d_H%d_Hkv%d_d%d" % (len(c[0]), c[2], c[3], c[4]))
def test_bwd_varlen_matches_oracle(fa_mod, cuda_device, case, causal):
    from tests._parity import check_grad
    lens_q, lens_k, H, Hkv, d = case
    lens_k = lens_k if lens_k is not None else lens_q
    q, k, v, do, cu_q, cu_k = inputs.varlen_inputs(lens_q, lens_k, H, Hkv, d,
                                                   seed=6200 + d + causal, with_do=True)
    scale = 1.0 / np.sqrt(d)
    dq, dk, dv = _fwd_bwd_varlen(fa_mod, q, k, v, do, cu_q, cu_k, causal, scale)
    ref_q = np.zeros(tuple(q.shape))
    ref_k = np.zeros(tuple(k.shape))
    ref_v = np.zeros(tuple(v.shape))
    for b in range(len(lens_q)):
        q0, q1, k0, k1 = int(cu_q[b]), int(cu_q[b + 1]), int(cu_k[b]), int(cu_k[b + 1])
        if q1 == q0 or k1 == k0:
            continue  # no gradient flows: zeros
        f = [inputs.to_f64(t.transpose(0, 1)[None]) for t in
             (q[q0:q1], k[k0:k1], v[k0:k1], do[q0:q1])]
        rq, rk, rv, _ = oracle.attention_backward(*f, causal, scale)
        ref_q[q0:q1] = rq[0].transpose(1, 0, 2)
        ref_k[k0:k1] = rk[0].transpose(1, 0, 2)
        ref_v[k0:k1] = rv[0].transpose(1, 0, 2)
    check_grad(dq, ref_q, "dQ")
    check_grad(dk, ref_k, "dK")
    check_grad(dv, ref_v, "dV")
    # and per sequence and head, so that one wrong sequence or head cannot
    # hide under the others
    for b in range(len(lens_q)):
        q0, q1, k0, k1 = int(cu_q[b]), int(cu_q[b + 1]), int(cu_k[b]), int(cu_k[b + 1])
        for h in range(H):
            if q1 > q0:
                check_grad(dq[q0:q1, h], ref_q[q0:q1, h], f"dQ seq {b} head {h}")
        for h in range(Hkv):
            if k1 > k0:
                check_grad(dk[k0:k1, h], ref_k[k0:k1, h], f"dK seq {b} head {h}")
                check_grad(dv[k0:k1, h], ref_v[k0:k1, h], f"dV seq {b} head {h}")


def test_bwd_varlen_equal_lengths_match_padded_kernel(fa_mod, cuda_device):
    """Equal lengths: dK and dV of the packed backward equal the padded ones bit
    for bit (each is summed inside one CTA in a fixed order); dQ is summed by
    atomic bulk reductions in no fixed order, so it is compared within the
    gradient tolerance."""
    from tests._parity import check_grad
    B, H, Hkv, N, d = 3, 4, 2, 777, 128
    q, k, v, do, cu_q, cu_k = inputs.varlen_inputs([N] * B, [N] * B, H, Hkv, d, seed=6300,
                                                   with_do=True)
    for causal in (False, True):
        dq, dk, dv = _fwd_bwd_varlen(fa_mod, q, k, v, do, cu_q, cu_k, causal, 0.1)
        pad = [t.view(B, N, t.shape[1], d).transpose(1, 2).contiguous().to(DEV) for t in (q, k, v, do)]
        o, lse = fa_mod.fwd(pad[0], pad[1], pad[2], causal=causal, scale=0.1)
        rq, rk, rv = fa_mod.bwd(pad[0], pad[1], pad[2], o, pad[3], lse, causal=causal, scale=0.1)
        torch.cuda.synchronize()
        for got, ref, hh in ((dk, rk, Hkv), (dv, rv, Hkv)):
            assert torch.equal(got.view(B, N, hh, d).transpose(1, 2), ref.cpu())
        check_grad(dq.view(B, N, H, d).transpose(1, 2), rq.cpu().float(), "dQ packed vs padded")
