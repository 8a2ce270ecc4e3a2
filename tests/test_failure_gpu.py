"""Failure detection on the GPU without a fault: a bounded wait on a barrier
that nothing completes gives up after its limit, the host reads FA_ERR_TIMEOUT
from the device error word, and the context keeps working afterwards."""
import time

import numpy as np
import pytest
import torch

import oracle
from io_aware_exact_35_b200 import inputs
from tests._parity import check_lse, check_o

pytestmark = pytest.mark.gpu

FA_ERR_TIMEOUT = 5


def test_bounded_wait_reports_timeout_and_context_survives(fa_mod, cuda_device):
    dev = torch.device("cuda:0")
    assert fa_mod.get_device_error() == 0  # start from a clear error word
    gave_up = torch.zeros(1, dtype=torch.int32, device=dev)
    t0 = time.monotonic()
    fa_mod.check_bounded_wait(gave_up)
    status = fa_mod.get_device_error()
    elapsed = time.monotonic() - t0
    assert status == FA_ERR_TIMEOUT
    # both waits (single-thread and warp-collective) returned false
    assert int(gave_up.item()) == 2
    # the limit is 2 s: the wait neither returned early nor ran on unbounded
    assert 1.5 < elapsed < 30.0, elapsed
    # reading the word cleared it
    assert fa_mod.get_device_error() == 0

    # the context is still usable: a forward on the same stream is correct
    B, H, N, d = 1, 2, 300, 128
    q, k, v = inputs.fwd_inputs(B, H, N, d, seed=4242)
    scale = 1.0 / np.sqrt(d)
    o, lse = fa_mod.fwd(q.to(dev), k.to(dev), v.to(dev), causal=True, scale=scale)
    assert fa_mod.get_device_error() == 0
    o_ref, lse_ref = oracle.attention_forward(inputs.to_f64(q), inputs.to_f64(k),
                                              inputs.to_f64(v), True, scale)
    check_o(o.cpu(), o_ref)
    check_lse(lse.cpu(), lse_ref)


def test_bounded_wait_rejects_bad_pointer(fa_mod, cuda_device):
    with pytest.raises((TypeError, ValueError)):
        fa_mod.check_bounded_wait(torch.zeros(1, dtype=torch.int64, device="cuda:0"))
