"""GPU parity of the split-KV decode kernels against the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle
from io_aware_exact_35_b200 import inputs
from tests._parity import check_lse, check_o

pytestmark = pytest.mark.gpu


def _run(fa_mod, q, kc, vc, seqlens, scale):
    dev = torch.device("cuda:0")
    o, lse = fa_mod.decode(q.to(dev), kc.to(dev), vc.to(dev), seqlens.to(dev), scale=scale)
    torch.cuda.synchronize()
    assert fa_mod.get_device_error() == 0
    return o.cpu(), lse.cpu()


def _oracle(q, kc, vc, seqlens, scale):
    return oracle.decode_forward(inputs.to_f64(q), inputs.to_f64(kc), inputs.to_f64(vc),
                                 seqlens.tolist(), scale)


@pytest.mark.parametrize("d", [64, 128])
def test_decode_edge_lengths(fa_mod, cuda_device, d):
    # empty prefix, single key, chunk boundaries, ragged tails, full capacity
    Lcap = 1537
    seqlens = [0, 1, 2, 511, 512, 513, 1024, 1536, 1537]
    q, kc, vc, sl = inputs.decode_inputs(len(seqlens), 3, d, 0, Lcap, seed=11 + d,
                                         Lcap=Lcap, seqlens=seqlens)
    o, lse = _run(fa_mod, q, kc, vc, sl, 1 / np.sqrt(d))
    o_ref, lse_ref = _oracle(q, kc, vc, sl, 1 / np.sqrt(d))
    assert np.all(o[0].float().numpy() == 0) and torch.isneginf(lse[0]).all()
    check_o(o, o_ref)
    check_lse(lse, lse_ref)


@pytest.mark.parametrize("d,H,Hkv,L", [(64, 2, 2, 40000), (128, 2, 2, 70000),
                                         (128, 8, 1, 70000), (64, 16, 1, 33000)])
def test_decode_more_splits_than_combine_threads(fa_mod, cuda_device, d, H, Hkv, L):
    """Long contexts give more 512-key splits than the combine kernel has
    threads (d), so its weights are gathered in several chunks; per head,
    grouped (8 and 16 query heads per cached head) and not."""
    seqlens = [L, L // 3 + 5]
    q, kc, vc, sl = inputs.decode_inputs(2, H, d, 0, L, seed=900 + d + H + L % 97, Lcap=L,
                                         seqlens=seqlens, Hkv=Hkv)
    o, lse = _run(fa_mod, q, kc, vc, sl, 1 / np.sqrt(d))
    o_ref, lse_ref = _oracle(q, kc, vc, sl, 1 / np.sqrt(d))
    check_o(o, o_ref)
    check_lse(lse, lse_ref)


def test_decode_small_random(fa_mod, cuda_device):
    q, kc, vc, sl = inputs.decode_inputs(4, 8, 128, 100, 3000, seed=5)
    o, lse = _run(fa_mod, q, kc, vc, sl, 0.1)
    o_ref, lse_ref = _oracle(q, kc, vc, sl, 0.1)
    check_o(o, o_ref)
    check_lse(lse, lse_ref)


def test_decode_workload_B16_H32_d128_full_size(fa_mod, cuda_device):
    """Full-size decode (caches 16 x 32 x 16384 x 128, NaN tails) vs the oracle on
    sampled (batch, head) pairs."""
    w = inputs.WORKLOADS["decode_B16_H32_d128_L4096-16384"]
    q, kc, vc, sl = inputs.workload_inputs(w)
    o, lse = _run(fa_mod, q, kc, vc, sl, w.scale)
    assert torch.isfinite(o.float()).all() and torch.isfinite(lse).all()
    rng = np.random.default_rng(w.seed)
    pairs = [(0, 0), (w.B - 1, w.H - 1)] + [tuple(x) for x in
                                            zip(rng.integers(0, w.B, 10), rng.integers(0, w.H, 10))]
    for b, h in pairs:
        L = int(sl[b])
        o_ref, lse_ref = oracle.decode_forward(inputs.to_f64(q[b:b + 1, h:h + 1]),
                                               inputs.to_f64(kc[b:b + 1, h:h + 1, :L]),
                                               inputs.to_f64(vc[b:b + 1, h:h + 1, :L]), [L],
                                               w.scale)
        check_o(o[b, h], o_ref[0, 0], f"o[{b},{h}]")
        check_lse(lse[b, h], lse_ref[0, 0], f"lse[{b},{h}]")
