"""fa_decode_static: the decode entry point that allocates nothing.

It exists for callers that cannot call cudaMalloc, such as a plug-in whose
host program has reserved nearly all device memory for its own pool, or a
latency-critical loop that must not trigger the device-wide synchronisation
an allocation can cause.  Its scratch is a fixed library-owned device array,
shared by every call.  These tests compare it with fa_decode (caller-provided
workspace) and with the fp64 oracle on two different problems in a row, so
that a stale array from the first call would show up in the second.  This file is collected last on
purpose: a failure here comes after every other test has run.
"""
import numpy as np
import pytest
import torch

import oracle
from io_aware_exact_35_b200 import inputs
from tests._parity import check_lse, check_o


def test_static_decode_rejects_problems_beyond_its_scratch(fa_mod):
    # 64 x 32 heads x 32 splits x 130 floats (34 MB) exceeds the 16 MiB
    # array: rejected on the host before any CUDA call.
    P = 1 << 20
    B, H, Lmax, d = 64, 32, 16384, 128
    assert fa_mod.decode_workspace_size(B, H, Lmax, d) > fa_mod.DECODE_STATIC_SCRATCH_BYTES
    st = fa_mod.lib().fa_decode_static(P, P, P, P, P, None, B, H, Lmax, d, 0.1, None)
    assert st == 3  # FA_ERR_WORKSPACE


@pytest.mark.gpu
def test_static_decode_matches_workspace_decode_twice(fa_mod, cuda_device):
    dev = torch.device("cuda:0")
    problems = [
        # (B, H, d, Lmin, Lmax, seed): a large one, then a smaller one with
        # different lengths, so leftovers of the first call would be visible
        (16, 32, 128, 4096, 16384, 91),
        (3, 5, 64, 1, 3000, 92),
    ]
    for (B, H, d, lo, hi, seed) in problems:
        assert fa_mod.decode_workspace_size(B, H, hi, d) <= fa_mod.DECODE_STATIC_SCRATCH_BYTES
        q, kc, vc, sl = (t.to(dev) for t in inputs.decode_inputs(B, H, d, lo, hi, seed=seed))
        o_ref, lse_ref = fa_mod.decode(q, kc, vc, sl)
        o_st = torch.full_like(o_ref, float("nan"))
        lse_st = torch.full_like(lse_ref, float("nan"))
        fa_mod.decode_static(q, kc, vc, sl, out=o_st, lse=lse_st)
        torch.cuda.synchronize()
        assert fa_mod.get_device_error() == 0
        check_o(o_st.cpu(), o_ref.cpu().double().numpy(), "static-scratch O")
        check_lse(lse_st.cpu(), lse_ref.cpu().double().numpy(), "static-scratch LSE")
        # and against the fp64 oracle itself
        o_or, lse_or = oracle.decode_forward(*(inputs.to_f64(t) for t in (q, kc, vc)),
                                             sl.cpu().tolist(), 1 / np.sqrt(d))
        check_o(o_st.cpu(), o_or, "static-scratch O vs oracle")
        check_lse(lse_st.cpu(), lse_or, "static-scratch LSE vs oracle")
