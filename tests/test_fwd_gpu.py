"""GPU parity of the forward kernel against the fp64 oracle (through the C ABI)."""
import numpy as np
import pytest
import torch

import oracle
from io_aware_exact_35_b200 import inputs
from tests._parity import check_lse, check_o

pytestmark = pytest.mark.gpu


def _run(fa_mod, q, k, v, causal, scale):
    dev = torch.device("cuda:0")
    o, lse = fa_mod.fwd(q.to(dev), k.to(dev), v.to(dev), causal=causal, scale=scale)
    torch.cuda.synchronize()
    assert fa_mod.get_device_error() == 0
    return o.cpu(), lse.cpu()


SMALL = [
    # (B, H, N, d): several tiles, ragged tails, sub-tile sizes
    (1, 2, 1, 64), (1, 1, 7, 128), (2, 3, 64, 64), (1, 2, 128, 128), (1, 2, 129, 128),
    (2, 2, 255, 64), (1, 3, 256, 128), (2, 1, 401, 128), (1, 1, 1000, 64), (1, 2, 1153, 128),
]


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("shape", SMALL, ids=lambda s: "B%dH%dN%dd%d" % s)
def test_fwd_small_shapes(fa_mod, cuda_device, shape, causal):
    B, H, N, d = shape
    q, k, v = inputs.fwd_inputs(B, H, N, d, seed=1000 + N + d + causal)
    scale = 1.0 / np.sqrt(d)
    o, lse = _run(fa_mod, q, k, v, causal, scale)
    o_ref, lse_ref = oracle.attention_forward(inputs.to_f64(q), inputs.to_f64(k),
                                              inputs.to_f64(v), causal, scale)
    check_o(o, o_ref)
    check_lse(lse, lse_ref)


def test_fwd_large_scores_and_rescaling(fa_mod, cuda_device):
    """Keys ramped from 0.1x to 4x make every row's running maximum grow by far
    more than the 2^8 rescale threshold across the key tiles, so O and l are
    rescaled many times.  The rows end up dominated by a few keys; V is scaled
    by 1/4 so that |O| stays below 1 and bf16 rounding of P and of O (2^-9
    relative each) stays inside the absolute tolerance."""
    B, H, N, d = 1, 2, 777, 128
    q, k, v = inputs.fwd_inputs(B, H, N, d, seed=7, std=1.0)
    ramp = torch.linspace(0.1, 4.0, N).view(1, 1, N, 1)
    k = (k.float() * ramp).to(torch.bfloat16)
    v = (v.float() * 0.25).to(torch.bfloat16)
    for causal in (False, True):
        o, lse = _run(fa_mod, q, k, v, causal, 0.3)
        o_ref, lse_ref = oracle.attention_forward(inputs.to_f64(q), inputs.to_f64(k),
                                                  inputs.to_f64(v), causal, 0.3)
        check_o(o, o_ref)
        check_lse(lse, lse_ref)


def test_fwd_workload_noncausal_B1_H2_N256_d64(fa_mod, cuda_device):
    w = inputs.WORKLOADS["fwd_noncausal_B1_H2_N256_d64"]
    q, k, v = inputs.workload_inputs(w)
    o, lse = _run(fa_mod, q, k, v, w.causal, w.scale)
    o_ref, lse_ref = oracle.attention_forward(inputs.to_f64(q), inputs.to_f64(k),
                                              inputs.to_f64(v), w.causal, w.scale)
    check_o(o, o_ref)
    check_lse(lse, lse_ref)


def test_fwd_workload_causal_B4_H16_N2048_d128(fa_mod, cuda_device):
    w = inputs.WORKLOADS["fwd_causal_B4_H16_N2048_d128"]
    q, k, v = inputs.workload_inputs(w)
    o, lse = _run(fa_mod, q, k, v, w.causal, w.scale)
    o_ref, lse_ref = oracle.attention_forward(inputs.to_f64(q), inputs.to_f64(k),
                                              inputs.to_f64(v), w.causal, w.scale)
    check_o(o, o_ref)
    check_lse(lse, lse_ref)


def test_fwd_workload_causal_B1_H32_N32768_d128_sampled(fa_mod, cuda_device):
    """Full-size long-context run: every head, on its first and last 64 rows
    and 64 random rows (a different random set per head), vs the oracle."""
    w = inputs.WORKLOADS["fwd_causal_B1_H32_N32768_d128"]
    q, k, v = inputs.workload_inputs(w)
    o, lse = _run(fa_mod, q, k, v, w.causal, w.scale)
    assert torch.isfinite(o.float()).all() and torch.isfinite(lse).all()
    for h in range(w.H):
        rows = inputs.sample_rows(w.N, 64, seed=w.seed + 100 * h, edge=64)
        qh, kh, vh = (inputs.to_f64(t[0, h]) for t in (q, k, v))
        o_ref, lse_ref = oracle.attention_forward_rows(qh, kh, vh, True, w.scale, rows)
        check_o(o[0, h, rows], o_ref, f"O head {h}")
        check_lse(lse[0, h, rows], lse_ref, f"LSE head {h}")


def test_fwd_output_buffers_and_streams(fa_mod, cuda_device):
    B, H, N, d = 1, 2, 300, 64
    q, k, v = (t.cuda() for t in inputs.fwd_inputs(B, H, N, d, seed=3))
    out = torch.full_like(q, float("nan"))
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        o, lse = fa_mod.fwd(q, k, v, causal=True, out=out, want_lse=False)
    s.synchronize()
    assert lse is None and o.data_ptr() == out.data_ptr()
    o_ref, _ = oracle.attention_forward(*(inputs.to_f64(t) for t in (q, k, v)), True,
                                        1 / np.sqrt(d))
    check_o(o.cpu(), o_ref)


# (B, H, Hkv, Nq, Nk, d, causal); with Nq > Nk many work items have halves
# that see the same number of key tiles, with Nq < Nk none do
_SCHEDULE_CASES = [(2, 3, 3, 1000, 1000, 128, True), (1, 5, 5, 777, 777, 64, True),
                   (3, 2, 2, 513, 513, 128, False), (2, 4, 4, 2048, 2048, 128, True),
                   (1, 4, 2, 3000, 1000, 128, True), (2, 2, 1, 1500, 4000, 64, True),
                   (1, 3, 3, 2900, 2900, 128, True)]


@pytest.mark.parametrize("schedule", ["persistent", "grid"])
def test_fwd_both_work_schedules(fa_mod, cuda_device, schedule):
    """The forward runs either one CTA per 256-row tile or persistently (each
    CTA loops over several tiles, barrier phases carried across them); both
    must give the oracle's result, also for unequal query / key lengths."""
    fa_mod.set_schedule(fwd=schedule)
    try:
        for (B, H, Hkv, N, Nk, d, causal) in _SCHEDULE_CASES:
            q, k, v = inputs.fwd_inputs(B, H, N, d, seed=N + d, Hkv=Hkv, Nk=Nk)
            o, lse = fa_mod.fwd(q.cuda(), k.cuda(), v.cuda(), causal=causal)
            torch.cuda.synchronize()
            assert fa_mod.get_device_error() == 0
            ref_o, ref_l = oracle.attention_forward(*(inputs.to_f64(t) for t in (q, k, v)),
                                                    causal, 1 / np.sqrt(d))
            check_o(o.cpu(), ref_o)
            check_lse(lse.cpu(), ref_l)
    finally:
        fa_mod.set_schedule()
