"""Decode over a paged KV cache (fa_decode_paged) against the fp64 oracle.

The pages name PagedAttention without describing it; paging changes only
where a position's key and value live, so the oracle is the plain decode
definition on the contiguous cache and the paged kernel must also match the
library's contiguous decode bit for bit (same arithmetic, other addresses).
Page pools are filled in a random order with NaN in every row and page that no
sequence owns, so any stray read shows up in the outputs."""
import numpy as np
import pytest
import torch

import oracle
from io_aware_exact_35_b200 import inputs
from tests._parity import check_lse, check_o

pytestmark = pytest.mark.gpu

DEV = torch.device("cuda:0")


def _decode_both(fa_mod, B, H, Hkv, d, seqlens, Lcap, page_size, seed):
    q, kc, vc, sl = inputs.decode_inputs(B, H, d, 0, Lcap, seed, Lcap=Lcap, seqlens=seqlens,
                                         Hkv=Hkv)
    kp, vp, table = inputs.page_cache(kc, vc, sl, page_size, seed + 1)
    o_p, lse_p = fa_mod.decode_paged(q.to(DEV), kp.to(DEV), vp.to(DEV), table.to(DEV),
                                     sl.to(DEV))
    o_c, lse_c = fa_mod.decode(q.to(DEV), kc.to(DEV), vc.to(DEV), sl.to(DEV))
    torch.cuda.synchronize()
    assert fa_mod.get_device_error() == 0
    return (q, kc, vc, sl), (o_p.cpu(), lse_p.cpu()), (o_c.cpu(), lse_c.cpu())


@pytest.mark.parametrize("page_size", [1, 16, 64, 256, 1024])
@pytest.mark.parametrize("hkv,d", [(4, 128), (1, 64), (2, 128)])
def test_paged_decode_matches_oracle_and_contiguous(fa_mod, cuda_device, page_size, hkv, d):
    B, H, Lcap = 4, 4, 1500
    seqlens = [0, 1, 1024, 1500]  # empty, one key, page/split aligned, ragged
    (q, kc, vc, sl), (o_p, lse_p), (o_c, lse_c) = _decode_both(
        fa_mod, B, H, hkv, d, seqlens, Lcap, page_size, seed=500 + page_size + d + hkv)
    assert torch.equal(o_p, o_c), "paged and contiguous decode differ"
    assert torch.equal(lse_p, lse_c)
    scale = 1.0 / np.sqrt(d)
    o_ref, lse_ref = oracle.decode_forward(inputs.to_f64(q), inputs.to_f64(kc), inputs.to_f64(vc),
                                           sl.tolist(), scale)
    check_o(o_p, o_ref)
    check_lse(lse_p, lse_ref)


@pytest.mark.parametrize("page_size", [1, 16, 128])
@pytest.mark.parametrize("H,hkv,d", [(16, 1, 128), (12, 2, 64)])
def test_paged_grouped_decode_large_groups(fa_mod, cuda_device, page_size, H, hkv, d):
    """Groups of 16 and 6 query heads per cached head (all 16 head rows of the
    tensor-core decode in use, and a padded group) over pages."""
    B, Lcap = 3, 1300
    seqlens = [17, 1300, 529]
    (q, kc, vc, sl), (o_p, lse_p), (o_c, lse_c) = _decode_both(
        fa_mod, B, H, hkv, d, seqlens, Lcap, page_size, seed=700 + page_size + H + d)
    assert torch.equal(o_p, o_c), "paged and contiguous decode differ"
    assert torch.equal(lse_p, lse_c)
    o_ref, lse_ref = oracle.decode_forward(inputs.to_f64(q), inputs.to_f64(kc), inputs.to_f64(vc),
                                           sl.tolist(), 1.0 / np.sqrt(d))
    check_o(o_p, o_ref)
    check_lse(lse_p, lse_ref)


def test_paged_decode_workload_shape(fa_mod, cuda_device):
    """B16 H32 (and 8 shared K/V heads) d128, lengths U{4096..16384}, 16-row
    pages: bit-exact against the contiguous kernel on the full batch, and
    against the oracle on three sequences."""
    for hkv in (32, 8):
        w = inputs.WORKLOADS["decode_B16_H32_d128_L4096-16384"]
        q, kc, vc, sl = inputs.decode_inputs(w.B, w.H, w.d, w.Lmin, w.Lmax, w.seed, Hkv=hkv)
        kp, vp, table = inputs.page_cache(kc, vc, sl, 16, w.seed + 1)
        o_p, lse_p = fa_mod.decode_paged(q.to(DEV), kp.to(DEV), vp.to(DEV), table.to(DEV),
                                         sl.to(DEV))
        o_c, lse_c = fa_mod.decode(q.to(DEV), kc.to(DEV), vc.to(DEV), sl.to(DEV))
        torch.cuda.synchronize()
        assert fa_mod.get_device_error() == 0
        assert torch.equal(o_p.cpu(), o_c.cpu()) and torch.equal(lse_p.cpu(), lse_c.cpu())
        for b in (0, 7, 15):
            L = int(sl[b])
            o_ref, lse_ref = oracle.decode_forward(
                inputs.to_f64(q[b:b + 1]), inputs.to_f64(kc[b:b + 1, :, :L]),
                inputs.to_f64(vc[b:b + 1, :, :L]), [L], w.scale)
            check_o(o_p[b:b + 1].cpu(), o_ref)
            check_lse(lse_p[b:b + 1].cpu(), lse_ref)


def test_paged_decode_bad_table_entry_is_reported(fa_mod, cuda_device):
    """A table entry outside the pool is never dereferenced: its positions are
    masked and FA_ERR_INVALID_ARG (1) is recorded in the device error word."""
    B, H, d, Lcap, ps = 2, 2, 128, 256, 16
    q, kc, vc, sl = inputs.decode_inputs(B, H, d, 0, Lcap, 42, Lcap=Lcap, seqlens=[256, 256])
    kp, vp, table = inputs.page_cache(kc, vc, sl, ps, 43)
    bad = table.clone()
    bad[1, 3] = kp.shape[0] + 1000  # past the pool
    o, lse = fa_mod.decode_paged(q.to(DEV), kp.to(DEV), vp.to(DEV), bad.to(DEV), sl.to(DEV))
    assert fa_mod.get_device_error() == 1
    assert torch.isfinite(o.float()).all()
    # sequence 0 is untouched; sequence 1 equals attention without page 3's rows
    keep = np.r_[0:3 * ps, 4 * ps:256]
    o_ref, _ = oracle.decode_forward(inputs.to_f64(q[1:]), inputs.to_f64(kc[1:, :, keep]),
                                     inputs.to_f64(vc[1:, :, keep]), [len(keep)], 1 / np.sqrt(d))
    check_o(o[1:].cpu(), o_ref)
    o_ref0, _ = oracle.decode_forward(inputs.to_f64(q[:1]), inputs.to_f64(kc[:1]),
                                      inputs.to_f64(vc[:1]), [256], 1 / np.sqrt(d))
    check_o(o[:1].cpu(), o_ref0)
    assert fa_mod.get_device_error() == 0
