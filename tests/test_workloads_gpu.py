"""Full-size parity of the benchmark's remaining workloads (the grouped
backward, the grouped decode, the ragged prefill and the e4m3 prefill),
run in the configuration bench.py times and checked against the fp64
oracle on sampled heads, sequences or rows."""
import numpy as np
import pytest
import torch

import oracle
from io_aware_exact_35_b200 import inputs
from tests._parity import check_grad, check_lse, check_o, rel_l2, as_f64
from tests.test_fp8_gpu import FP8_O_REL_L2, _fp8_o_bound

pytestmark = pytest.mark.gpu

DEV = torch.device("cuda:0")


def test_bwd_gqa_workload_B2_H32_Hkv8_N4096_sampled_groups(fa_mod, cuda_device):
    """All 32 query heads share 8 key/value heads; the gradients of two whole
    groups (four query heads and their shared K/V head each) vs the oracle."""
    w = inputs.WORKLOADS["bwd_causal_gqa_B2_H32_Hkv8_N4096_d128"]
    q, k, v, do = inputs.workload_inputs(w)
    g = w.H // w.kv_heads
    qd, kd, vd, dod = (t.to(DEV) for t in (q, k, v, do))
    o, lse = fa_mod.fwd(qd, kd, vd, causal=True, scale=w.scale)
    dq, dk, dv = fa_mod.bwd(qd, kd, vd, o, dod, lse, causal=True, scale=w.scale)
    torch.cuda.synchronize()
    assert fa_mod.get_device_error() == 0
    dq, dk, dv = dq.cpu(), dk.cpu(), dv.cpu()
    for t in (dq, dk, dv):
        assert torch.isfinite(t.float()).all()
    for b, hk in ((0, 0), (1, w.kv_heads - 1)):
        hs = slice(g * hk, g * hk + g)
        rq, rk, rv, _ = oracle.attention_backward(
            inputs.to_f64(q[b:b + 1, hs]), inputs.to_f64(k[b:b + 1, hk:hk + 1]),
            inputs.to_f64(v[b:b + 1, hk:hk + 1]), inputs.to_f64(do[b:b + 1, hs]), True, w.scale)
        for i in range(g):
            check_grad(dq[b, g * hk + i], rq[0, i], f"dQ[{b},{g * hk + i}]")
        check_grad(dk[b, hk], rk[0, 0], f"dK[{b},{hk}]")
        check_grad(dv[b, hk], rv[0, 0], f"dV[{b},{hk}]")


def test_decode_gqa_workload_B16_H32_Hkv8_sampled_heads(fa_mod, cuda_device):
    """Grouped decode on the tensor cores, full-size caches with NaN tails."""
    w = inputs.WORKLOADS["decode_gqa_B16_H32_Hkv8_d128_L4096-16384"]
    q, kc, vc, sl = inputs.workload_inputs(w)
    o, lse = fa_mod.decode(q.to(DEV), kc.to(DEV), vc.to(DEV), sl.to(DEV), scale=w.scale)
    torch.cuda.synchronize()
    assert fa_mod.get_device_error() == 0
    o, lse = o.cpu(), lse.cpu()
    assert torch.isfinite(o.float()).all() and torch.isfinite(lse).all()
    g = w.H // w.kv_heads
    rng = np.random.default_rng(w.seed)
    pairs = [(0, 0), (w.B - 1, w.H - 1)] + [tuple(x) for x in
                                            zip(rng.integers(0, w.B, 10), rng.integers(0, w.H, 10))]
    for b, h in pairs:
        L = int(sl[b])
        hk = h // g
        o_ref, lse_ref = oracle.decode_forward(inputs.to_f64(q[b:b + 1, h:h + 1]),
                                               inputs.to_f64(kc[b:b + 1, hk:hk + 1, :L]),
                                               inputs.to_f64(vc[b:b + 1, hk:hk + 1, :L]), [L],
                                               w.scale)
        check_o(o[b, h], o_ref[0, 0], f"o[{b},{h}]")
        check_lse(lse[b, h], lse_ref[0, 0], f"lse[{b},{h}]")


def test_fwd_varlen_workload_B16_H16_sampled(fa_mod, cuda_device):
    """The ragged prefill batch (16 sequences of U{512..4096} tokens, packed):
    sampled rows of the shortest and the longest sequence and two others,
    on three heads each."""
    w = inputs.WORKLOADS["fwd_varlen_causal_B16_H16_d128_L512-4096"]
    lens = inputs.varlen_lengths(w)
    q, k, v, cu_q, cu_k = inputs.workload_inputs(w)
    o, lse = fa_mod.fwd_varlen(q.to(DEV), k.to(DEV), v.to(DEV), cu_q.to(DEV), cu_k.to(DEV),
                               max(lens), causal=True, scale=w.scale)
    torch.cuda.synchronize()
    assert fa_mod.get_device_error() == 0
    o, lse = o.cpu(), lse.cpu()
    order = np.argsort(lens)
    seqs = sorted({int(order[0]), int(order[-1]), 3, 11})
    for s in seqs:
        q0, q1 = int(cu_q[s]), int(cu_q[s + 1])
        n = q1 - q0
        rows = inputs.sample_rows(n, 48, seed=w.seed + s)
        for h in (0, 7, w.H - 1):
            ro, rl = oracle.attention_forward_rows(inputs.to_f64(q[q0:q1, h]),
                                                   inputs.to_f64(k[q0:q1, h]),
                                                   inputs.to_f64(v[q0:q1, h]), True, w.scale, rows)
            idx = torch.as_tensor(q0 + rows, dtype=torch.long)
            check_o(o[idx, h], ro, f"O seq {s} head {h}")
            check_lse(lse[h, idx], rl, f"LSE seq {s} head {h}")


def test_fwd_fp8_workload_B4_H16_N2048_sampled_heads(fa_mod, cuda_device):
    """The e4m3 prefill at full size: three whole heads against the oracle on
    the descaled inputs, with the e4m3 tolerance and worst-case bound."""
    w = inputs.WORKLOADS["fwd_fp8_causal_B4_H16_N2048_d128"]
    q8, k8, vt8, (qs, ks, vs) = inputs.workload_inputs(w)
    o, lse = fa_mod.fwd_fp8(q8.to(DEV), k8.to(DEV), vt8.to(DEV), qs, ks, vs, causal=True,
                            scale=w.scale)
    torch.cuda.synchronize()
    assert fa_mod.get_device_error() == 0
    o, lse = o.cpu(), lse.cpu()
    for b, h in ((0, 0), (1, 9), (w.B - 1, w.H - 1)):
        qh = inputs.fp8_to_f64(q8[b:b + 1, h:h + 1], qs)
        kh = inputs.fp8_to_f64(k8[b:b + 1, h:h + 1], ks)
        vh = inputs.fp8_to_f64(vt8[b:b + 1, h:h + 1].transpose(-1, -2).contiguous(), vs)
        o_ref, lse_ref = oracle.attention_forward(qh, kh, vh, True, w.scale)
        got = as_f64(o[b:b + 1, h:h + 1])
        assert np.isfinite(got).all()
        rl = rel_l2(got, o_ref)
        assert rl <= FP8_O_REL_L2, f"O[{b},{h}] relative L2 {rl:.3e} > {FP8_O_REL_L2}"
        check_lse(lse[b:b + 1, h:h + 1], lse_ref, f"LSE[{b},{h}]")
        bound = _fp8_o_bound(qh, kh, vh, o_ref, True, w.scale)
        worst = float(np.max(np.abs(got - o_ref) - bound))
        assert worst <= 0.0, f"O[{b},{h}] exceeds the e4m3 worst-case bound by {worst:.3e}"
