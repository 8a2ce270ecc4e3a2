"""GPU parity of the backward kernels against the fp64 oracle (through the C ABI).

O and LSE come from the library's own forward pass, as in training; the
oracle recomputes everything from q, k, v, dO in fp64."""
import numpy as np
import pytest
import torch

import oracle
from io_aware_exact_35_b200 import inputs
from tests._parity import check_grad

pytestmark = pytest.mark.gpu


def _run(fa_mod, q, k, v, do, causal, scale):
    dev = torch.device("cuda:0")
    q, k, v, do = (t.to(dev) for t in (q, k, v, do))
    o, lse = fa_mod.fwd(q, k, v, causal=causal, scale=scale)
    dq, dk, dv = fa_mod.bwd(q, k, v, o, do, lse, causal=causal, scale=scale)
    torch.cuda.synchronize()
    assert fa_mod.get_device_error() == 0
    return dq.cpu(), dk.cpu(), dv.cpu()


SMALL = [(1, 1, 1, 64), (1, 2, 100, 128), (2, 1, 128, 64), (1, 2, 129, 128),
         (1, 1, 300, 64), (2, 2, 513, 128), (1, 1, 1000, 128)]


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("shape", SMALL, ids=lambda s: "B%dH%dN%dd%d" % s)
def test_bwd_small_shapes(fa_mod, cuda_device, shape, causal):
    B, H, N, d = shape
    q, k, v, do = inputs.bwd_inputs(B, H, N, d, seed=2000 + N + d + causal)
    scale = 1.0 / np.sqrt(d)
    dq, dk, dv = _run(fa_mod, q, k, v, do, causal, scale)
    rq, rk, rv, _ = oracle.attention_backward(*(inputs.to_f64(t) for t in (q, k, v, do)),
                                              causal, scale)
    check_grad(dq, rq, "dQ")
    check_grad(dk, rk, "dK")
    check_grad(dv, rv, "dV")


def test_bwd_workload_causal_B2_H16_N8192_d128_sampled_heads(fa_mod, cuda_device):
    """Full-size backward; complete dQ, dK, dV of sampled heads vs the oracle."""
    w = inputs.WORKLOADS["bwd_causal_B2_H16_N8192_d128"]
    q, k, v, do = inputs.workload_inputs(w)
    dq, dk, dv = _run(fa_mod, q, k, v, do, w.causal, w.scale)
    for t in (dq, dk, dv):
        assert torch.isfinite(t.float()).all()
    # eight (batch, head) pairs over both batches and the head-major launch order
    for (b, h) in ((0, 0), (0, 5), (0, 10), (0, 15), (1, 0), (1, 6), (1, 11), (1, 15)):
        rq, rk, rv, _ = oracle.attention_backward(
            *(inputs.to_f64(t[b, h]) for t in (q, k, v, do)), True, w.scale)
        check_grad(dq[b, h], rq, f"dQ[{b},{h}]")
        check_grad(dk[b, h], rk, f"dK[{b},{h}]")
        check_grad(dv[b, h], rv, f"dV[{b},{h}]")


@pytest.mark.parametrize("order", ["grid", "persistent"])
def test_bwd_both_cta_orders(fa_mod, cuda_device, order):
    """The backward launches its key-tile CTAs head-major or longest first;
    both orders must give the oracle's gradients."""
    fa_mod.set_schedule(bwd=order)
    try:
        for (B, H, N, d, causal) in ((2, 3, 700, 128, True), (1, 4, 1100, 64, True),
                                     (2, 2, 513, 128, False)):
            q, k, v, do = inputs.bwd_inputs(B, H, N, d, seed=3000 + N + d)
            scale = 1.0 / np.sqrt(d)
            dq, dk, dv = _run(fa_mod, q, k, v, do, causal, scale)
            for b in range(B):
                for h in range(H):
                    rq, rk, rv, _ = oracle.attention_backward(
                        *(inputs.to_f64(t[b, h]) for t in (q, k, v, do)), causal, scale)
                    check_grad(dq[b, h], rq, f"dQ[{b},{h}]")
                    check_grad(dk[b, h], rk, f"dK[{b},{h}]")
                    check_grad(dv[b, h], rv, f"dV[{b},{h}]")
    finally:
        fa_mod.set_schedule()


def test_bwd_more_than_65535_heads(fa_mod, cuda_device):
    """B * H above 65535: the dQ conversion's grid cannot give each query head
    a row of CTAs, so it runs as a plain pass after the main kernel.  Sampled
    heads on both sides of the 65535 boundary against the oracle."""
    B, H, N, d = 1, 65600, 5, 64
    q, k, v, do = inputs.bwd_inputs(B, H, N, d, seed=3400)
    scale = 1.0 / np.sqrt(d)
    dq, dk, dv = _run(fa_mod, q, k, v, do, True, scale)
    for h in (0, 1, 777, 65534, 65535, 65536, 65599):
        rq, rk, rv, _ = oracle.attention_backward(
            *(inputs.to_f64(t[0, h]) for t in (q, k, v, do)), True, scale)
        check_grad(dq[0, h], rq, f"dQ[{h}]")
        check_grad(dk[0, h], rk, f"dK[{h}]")
        check_grad(dv[0, h], rv, f"dV[{h}]")
