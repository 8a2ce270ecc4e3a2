"""The autograd wrapper: forward and the gradients it returns through
loss.backward() match the fp64 oracle (the upstream gradient of
loss = sum(O * W) is W)."""
import numpy as np
import pytest
import torch

import oracle
from io_aware_exact_35_b200 import inputs
from tests._parity import check_grad, check_o

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("hkv", [4, 2])
def test_attention_autograd_matches_oracle(fa_mod, cuda_device, causal, hkv):
    from io_aware_exact_35_b200.autograd import attention
    B, H, N, d = 2, 4, 333, 128
    q, k, v, w = inputs.bwd_inputs(B, H, N, d, seed=77 + hkv + causal, Hkv=hkv)
    tq, tk, tv = (t.cuda().requires_grad_() for t in (q, k, v))
    o = attention(tq, tk, tv, causal=causal)
    loss = (o.float() * w.cuda().float()).sum()
    loss.backward()
    torch.cuda.synchronize()
    assert fa_mod.get_device_error() == 0
    f64 = [inputs.to_f64(t) for t in (q, k, v, w)]
    ro, _ = oracle.attention_forward(f64[0], f64[1], f64[2], causal, 1 / np.sqrt(d))
    check_o(o.detach().cpu(), ro)
    rq, rk, rv, _ = oracle.attention_backward(*f64, causal, 1 / np.sqrt(d))
    check_grad(tq.grad.cpu(), rq, "dQ")
    check_grad(tk.grad.cpu(), rk, "dK")
    check_grad(tv.grad.cpu(), rv, "dV")


def test_attention_autograd_chunk_over_longer_keys(fa_mod, cuda_device):
    """Nq = 200 queries over Nk = 450 keys, causal (bottom-right aligned)."""
    from io_aware_exact_35_b200.autograd import attention
    B, H, Hkv, Nq, Nk, d = 1, 4, 2, 200, 450, 64
    q, k, v, w = inputs.bwd_inputs(B, H, Nq, d, seed=91, Hkv=Hkv, Nk=Nk)
    tq, tk, tv = (t.cuda().requires_grad_() for t in (q, k, v))
    o = attention(tq, tk, tv, causal=True)
    (o.float() * w.cuda().float()).sum().backward()
    torch.cuda.synchronize()
    assert fa_mod.get_device_error() == 0
    f64 = [inputs.to_f64(t) for t in (q, k, v, w)]
    ro, _ = oracle.attention_forward(f64[0], f64[1], f64[2], True, 1 / np.sqrt(d))
    check_o(o.detach().cpu(), ro)
    rq, rk, rv, _ = oracle.attention_backward(*f64, True, 1 / np.sqrt(d))
    check_grad(tq.grad.cpu(), rq, "dQ")
    check_grad(tk.grad.cpu(), rk, "dK")
    check_grad(tv.grad.cpu(), rv, "dV")
