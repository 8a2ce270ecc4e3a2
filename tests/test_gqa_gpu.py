"""GPU parity of grouped-query attention (K/V heads shared by groups of query
heads, "DL101 chapter 9" sections 3.1-3.2) in the forward, backward and
decode kernels, against the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle
from io_aware_exact_35_b200 import inputs
from tests._parity import check_grad, check_lse, check_o

pytestmark = pytest.mark.gpu

SHAPES = [(1, 4, 1, 300, 128), (2, 6, 2, 257, 64), (1, 8, 2, 1024, 128), (2, 4, 4, 129, 128)]


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "B%dH%dHkv%dN%dd%d" % s)
def test_gqa_forward(fa_mod, cuda_device, shape, causal):
    B, H, Hkv, N, d = shape
    q, k, v = inputs.fwd_inputs(B, H, N, d, seed=300 + N + Hkv, Hkv=Hkv)
    o, lse = fa_mod.fwd(q.cuda(), k.cuda(), v.cuda(), causal=causal)
    torch.cuda.synchronize()
    assert fa_mod.get_device_error() == 0
    ref_o, ref_l = oracle.attention_forward(*(inputs.to_f64(t) for t in (q, k, v)), causal,
                                            1 / np.sqrt(d))
    check_o(o.cpu(), ref_o)
    check_lse(lse.cpu(), ref_l)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "B%dH%dHkv%dN%dd%d" % s)
def test_gqa_backward(fa_mod, cuda_device, shape, causal):
    B, H, Hkv, N, d = shape
    q, k, v, do = inputs.bwd_inputs(B, H, N, d, seed=400 + N + Hkv, Hkv=Hkv)
    qd, kd, vd, dod = (t.cuda() for t in (q, k, v, do))
    o, lse = fa_mod.fwd(qd, kd, vd, causal=causal)
    dq, dk, dv = fa_mod.bwd(qd, kd, vd, o, dod, lse, causal=causal)
    torch.cuda.synchronize()
    assert fa_mod.get_device_error() == 0
    assert dk.shape == k.shape and dv.shape == v.shape
    rq, rk, rv, _ = oracle.attention_backward(*(inputs.to_f64(t) for t in (q, k, v, do)), causal,
                                              1 / np.sqrt(d))
    dq, dk, dv = dq.cpu(), dk.cpu(), dv.cpu()
    check_grad(dq, rq, "dQ")
    check_grad(dk, rk, "dK")
    check_grad(dv, rv, "dV")
    # per head as well: a wrong head must not hide under the others
    for b in range(B):
        for h in range(H):
            check_grad(dq[b, h], rq[b, h], f"dQ[{b},{h}]")
        for h in range(Hkv):
            check_grad(dk[b, h], rk[b, h], f"dK[{b},{h}]")
            check_grad(dv[b, h], rv[b, h], f"dV[{b},{h}]")


@pytest.mark.parametrize("d", [128, 64])
@pytest.mark.parametrize("Hkv", [1, 2, 4, 8])
def test_gqa_decode(fa_mod, cuda_device, Hkv, d):
    """Groups of 8, 4, 2 and 1 query heads per cached head; lengths around the
    shared-memory stage (32 / 64 rows) and split (512 rows) boundaries, and 0."""
    sl = [0, 1, 31, 32, 33, 64, 511, 512, 513, 700, 2100]
    q, kc, vc, sl = inputs.decode_inputs(len(sl), 8, d, 0, 2100, seed=500 + Hkv + d, Hkv=Hkv,
                                         seqlens=sl, Lcap=2100)
    o, lse = fa_mod.decode(q.cuda(), kc.cuda(), vc.cuda(), sl.cuda())
    torch.cuda.synchronize()
    assert fa_mod.get_device_error() == 0
    ref_o, ref_l = oracle.decode_forward(inputs.to_f64(q), inputs.to_f64(kc), inputs.to_f64(vc),
                                         sl.tolist(), 1 / np.sqrt(d))
    check_o(o.cpu(), ref_o)
    check_lse(lse.cpu(), ref_l)


@pytest.mark.parametrize("d", [128, 64])
@pytest.mark.parametrize("H,Hkv", [(9, 3), (12, 2), (48, 3), (32, 1), (24, 1), (20, 1)],
                         ids=lambda x: str(x))
def test_gqa_decode_group_sizes(fa_mod, cuda_device, H, Hkv, d):
    """Groups of 3, 6 and 16 query heads (one CTA per cached head, padded
    head rows), 32 and 24 (16 or 8 heads per CTA, several CTAs per cached
    head) and 20 (one CTA per query head); lengths inside and across 16-key
    steps and 512-key splits."""
    sl = [0, 1, 15, 16, 17, 100, 513, 1300]
    q, kc, vc, sl = inputs.decode_inputs(len(sl), H, d, 0, 1300, seed=600 + H + Hkv + d,
                                         Hkv=Hkv, seqlens=sl, Lcap=1300)
    o, lse = fa_mod.decode(q.cuda(), kc.cuda(), vc.cuda(), sl.cuda())
    torch.cuda.synchronize()
    assert fa_mod.get_device_error() == 0
    ref_o, ref_l = oracle.decode_forward(inputs.to_f64(q), inputs.to_f64(kc), inputs.to_f64(vc),
                                         sl.tolist(), 1 / np.sqrt(d))
    check_o(o.cpu(), ref_o)
    check_lse(lse.cpu(), ref_l)


def test_gqa_workload_forward_B4_H32_Hkv8_N2048_sampled(fa_mod, cuda_device):
    w = inputs.WORKLOADS["fwd_causal_gqa_B4_H32_Hkv8_N2048_d128"]
    q, k, v = inputs.workload_inputs(w)
    o, lse = fa_mod.fwd(q.cuda(), k.cuda(), v.cuda(), causal=True)
    torch.cuda.synchronize()
    rows = inputs.sample_rows(w.N, 64, seed=w.seed)
    for b, h in ((0, 0), (3, 31), (1, 9)):
        ro, rl = oracle.attention_forward_rows(inputs.to_f64(q[b, h]), inputs.to_f64(k[b, h // 4]),
                                               inputs.to_f64(v[b, h // 4]), True, w.scale, rows)
        check_o(o[b, h, rows].cpu(), ro)
        check_lse(lse[b, h, rows].cpu(), rl)
