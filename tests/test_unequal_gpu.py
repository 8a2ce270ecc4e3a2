"""GPU parity for separate query and key lengths (Nq != Nk) through
fa_fwd_ext / fa_bwd_ext, against the fp64 oracle.

With Nq != Nk the queries are the last Nq positions of the Nk-token sequence
(a chunk of new tokens over a cache), so causal masking keeps key j for query
i iff j <= i + Nk - Nq; the non-causal Lq x Lk problem is the one of "DL101
chapter 9", section 3.3.  Cases cover a chunk shorter than the cache, more
queries than keys (the first Nq - Nk queries see nothing: O = 0,
LSE = -inf, zero gradient), single-query chunks, ragged tails on both sides,
grouped heads and the empty sides Nq = 0 and Nk = 0."""
import numpy as np
import pytest
import torch

import oracle
from io_aware_exact_35_b200 import inputs
from tests._parity import check_grad, check_lse, check_o

pytestmark = pytest.mark.gpu

DEV = torch.device("cuda:0")

# (B, H, Hkv, Nq, Nk, d)
FWD_CASES = [
    (1, 2, 2, 1280, 1152, 128),  # the section 3.3 shape (d = 128 here)
    (1, 2, 2, 200, 1000, 128),   # chunk over a longer cache
    (2, 2, 1, 384, 1024, 64),    # tile-aligned chunk, one shared K/V head
    (1, 2, 2, 1000, 200, 128),   # more queries than keys
    (1, 1, 1, 1, 777, 128),      # one new token
    (1, 3, 3, 129, 1, 64),       # one key
    (1, 4, 2, 300, 700, 128),    # grouped heads, ragged both sides
]


def _fwd(fa_mod, q, k, v, causal, scale):
    o, lse = fa_mod.fwd(q.to(DEV), k.to(DEV), v.to(DEV), causal=causal, scale=scale)
    torch.cuda.synchronize()
    assert fa_mod.get_device_error() == 0
    return o.cpu(), lse.cpu()


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("case", FWD_CASES, ids=lambda c: "B%dH%dHkv%dNq%dNk%dd%d" % c)
def test_fwd_unequal_lengths(fa_mod, cuda_device, case, causal):
    B, H, Hkv, Nq, Nk, d = case
    q, k, v = inputs.fwd_inputs(B, H, Nq, d, seed=3000 + Nq + 7 * Nk + causal, Hkv=Hkv, Nk=Nk)
    scale = 1.0 / np.sqrt(d)
    o, lse = _fwd(fa_mod, q, k, v, causal, scale)
    o_ref, lse_ref = oracle.attention_forward(inputs.to_f64(q), inputs.to_f64(k),
                                              inputs.to_f64(v), causal, scale)
    check_o(o, o_ref)
    check_lse(lse, lse_ref)
    if causal and Nq > Nk:
        # the first Nq - Nk queries see no key
        assert torch.all(o[:, :, :Nq - Nk] == 0)
        assert torch.all(torch.isneginf(lse[:, :, :Nq - Nk]))


def test_fwd_chunk_equals_rows_of_full_causal(fa_mod, cuda_device):
    """A causal chunk of the last Nq queries over all Nk keys equals the last Nq
    rows of the square causal problem (same kernel, same inputs)."""
    B, H, N, d, Nq = 1, 2, 1000, 128, 300
    q, k, v = inputs.fwd_inputs(B, H, N, d, seed=3100)
    o_full, lse_full = _fwd(fa_mod, q, k, v, True, 1.0 / np.sqrt(d))
    o_chunk, lse_chunk = _fwd(fa_mod, q[:, :, N - Nq:].contiguous(), k, v, True, 1.0 / np.sqrt(d))
    check_o(o_chunk, inputs.to_f64(o_full[:, :, N - Nq:]), "O chunk vs full")
    check_lse(lse_chunk, inputs.to_f64(lse_full[:, :, N - Nq:]), "LSE chunk vs full")


def test_fwd_no_keys_and_no_queries(fa_mod, cuda_device):
    B, H, d = 2, 2, 128
    q, k, v = inputs.fwd_inputs(B, H, 130, d, seed=3200, Nk=0)
    o, lse = _fwd(fa_mod, q, k, v, False, 0.1)
    assert torch.all(o == 0) and torch.all(torch.isneginf(lse))
    q, k, v = inputs.fwd_inputs(B, H, 0, d, seed=3201, Nk=50)
    o, lse = _fwd(fa_mod, q, k, v, True, 0.1)
    assert o.shape == (B, H, 0, d) and lse.shape == (B, H, 0)


BWD_CASES = [
    (1, 2, 2, 1280, 1152, 128),
    (1, 2, 2, 200, 1000, 128),
    (1, 2, 2, 1000, 200, 64),
    (2, 4, 2, 300, 700, 128),
    (1, 1, 1, 1, 300, 128),
]


def _fwd_bwd(fa_mod, q, k, v, do, causal, scale):
    q, k, v, do = (t.to(DEV) for t in (q, k, v, do))
    o, lse = fa_mod.fwd(q, k, v, causal=causal, scale=scale)
    dq, dk, dv = fa_mod.bwd(q, k, v, o, do, lse, causal=causal, scale=scale)
    torch.cuda.synchronize()
    assert fa_mod.get_device_error() == 0
    return dq.cpu(), dk.cpu(), dv.cpu()


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("case", BWD_CASES, ids=lambda c: "B%dH%dHkv%dNq%dNk%dd%d" % c)
def test_bwd_unequal_lengths(fa_mod, cuda_device, case, causal):
    B, H, Hkv, Nq, Nk, d = case
    q, k, v, do = inputs.bwd_inputs(B, H, Nq, d, seed=4000 + Nq + 7 * Nk + causal, Hkv=Hkv,
                                    Nk=Nk)
    scale = 1.0 / np.sqrt(d)
    dq, dk, dv = _fwd_bwd(fa_mod, q, k, v, do, causal, scale)
    rq, rk, rv, _ = oracle.attention_backward(*(inputs.to_f64(t) for t in (q, k, v, do)),
                                              causal, scale)
    check_grad(dq, rq, "dQ")
    check_grad(dk, rk, "dK")
    check_grad(dv, rv, "dV")
    if causal and Nq > Nk:
        assert torch.all(dq[:, :, :Nq - Nk] == 0)


def test_bwd_empty_sides(fa_mod, cuda_device):
    """Nq = 0: no gradient reaches K and V (dK = dV = 0); Nk = 0: dQ = 0."""
    B, H, d = 1, 2, 64
    q, k, v, do = inputs.bwd_inputs(B, H, 0, d, seed=4100, Nk=70)
    dq, dk, dv = _fwd_bwd(fa_mod, q, k, v, do, True, 0.125)
    assert dq.shape == (B, H, 0, d)
    assert torch.all(dk == 0) and torch.all(dv == 0)
    q, k, v, do = inputs.bwd_inputs(B, H, 90, d, seed=4101, Nk=0)
    dq, dk, dv = _fwd_bwd(fa_mod, q, k, v, do, False, 0.125)
    assert torch.all(dq == 0) and dk.shape == (B, H, 0, d)


@pytest.mark.parametrize("case", [(2, 4, 2, 300, 700, 128, True), (1, 2, 1, 520, 260, 64, True),
                                  (2, 2, 2, 640, 640, 128, False)],
                         ids=lambda c: "B%dH%dHkv%dNq%dNk%dd%dc%d" % c)
def test_bwd_workspace_contents_ignored(fa_mod, cuda_device, case):
    """The backward's workspace holds the dQ accumulator and one completion
    counter per key/value head, which the dQ conversion waits on; both are
    reset by every call.  A workspace filled with 0xFF (every counter already
    past its target) and then reused by a second call must give the oracle's
    gradients both times."""
    B, H, Hkv, Nq, Nk, d, causal = case
    q, k, v, do = inputs.bwd_inputs(B, H, Nq, d, seed=4200 + Nq + Nk, Hkv=Hkv, Nk=Nk)
    scale = 1.0 / np.sqrt(d)
    rq, rk, rv, _ = oracle.attention_backward(*(inputs.to_f64(t) for t in (q, k, v, do)),
                                              causal, scale)
    qd, kd, vd, dod = (t.to(DEV) for t in (q, k, v, do))
    o, lse = fa_mod.fwd(qd, kd, vd, causal=causal, scale=scale)
    ws = torch.full((fa_mod.bwd_workspace_size(B, H, Nq, d),), 0xFF, dtype=torch.uint8,
                    device=DEV)
    for call in range(2):
        dq, dk, dv = fa_mod.bwd(qd, kd, vd, o, dod, lse, causal=causal, scale=scale,
                                workspace=ws)
        torch.cuda.synchronize()
        assert fa_mod.get_device_error() == 0
        check_grad(dq.cpu(), rq, f"dQ (call {call})")
        check_grad(dk.cpu(), rk, f"dK (call {call})")
        check_grad(dv.cpu(), rv, f"dV (call {call})")
