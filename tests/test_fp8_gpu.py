"""GPU parity of the e4m3 forward (fa_fwd_fp8) against the fp64 oracle.

The oracle runs on the exact real values of the 8-bit inputs (stored value x
descale factor), so the only differences are the kernel's own roundings:
f32 accumulation (negligible), P rounded to e4m3 before the P V product, and
O rounded to bf16.  The pages give no FP8 tolerance; the one used here is
derived from the e4m3 rounding of P: each probability carries an independent
relative error of at most 2^-4 (uniform, sigma = 2^-4 / sqrt(3) = 0.036), and
with O = sum P v / l that makes the relative L2 error of O about sigma.  The
test allows 6e-2.  LSE comes from the f32 scores alone (products of e4m3
values are exact in f32), so it keeps the bf16 path's 1e-3.

Each output element must also lie within a worst-case bound derived from the
same arithmetic.  Write P_ij = p_ij / l_i for the exact probabilities.  The
kernel exponentiates against a running maximum that is at most the row's
true maximum, so its unnormalised p lie at or above p_ij / max_j p_ij and its
row sum l is at least 1 / max_j P_ij.  Rounding one p to e4m3 errs by at most
2^-4 of it in the normal range (>= 2^-6) and by at most 2^-10 below it
(subnormal spacing 2^-9; values under 2^-10 flush to 0).  Hence
  |O_ic - O*_ic| <= 2^-4 sum_j P_ij |v_jc|
                    + 2^-10 max_j P_ij sum_{j: P_ij < 2^-6 max_j P_ij} |v_jc|
                    + 2^-8 |O*_ic| (bf16 output) + 1e-5 (f32 sums),
evaluated from the oracle's P (read out through V = identity)."""
import numpy as np
import pytest
import torch

import oracle
from io_aware_exact_35_b200 import inputs
from tests._parity import LSE_MAX_ABS, as_f64, check_lse, rel_l2

pytestmark = pytest.mark.gpu

FP8_O_REL_L2 = 6e-2
DEV = torch.device("cuda:0")


def _check(q8, k8, vt8, scales, causal, fa_mod, scale=None):
    qs, ks, vs = scales
    d = q8.shape[-1]
    scale = 1.0 / np.sqrt(d) if scale is None else scale
    o, lse = fa_mod.fwd_fp8(q8.to(DEV), k8.to(DEV), vt8.to(DEV), qs, ks, vs, causal=causal,
                            scale=scale)
    torch.cuda.synchronize()
    assert fa_mod.get_device_error() == 0
    q = inputs.fp8_to_f64(q8, qs)
    k = inputs.fp8_to_f64(k8, ks)
    v = inputs.fp8_to_f64(vt8.transpose(-1, -2).contiguous(), vs)
    o_ref, lse_ref = oracle.attention_forward(q, k, v, causal, scale)
    g = as_f64(o.cpu())
    assert np.isfinite(g).all()
    rl = rel_l2(g, o_ref)
    assert rl <= FP8_O_REL_L2, f"O relative L2 {rl:.3e} > {FP8_O_REL_L2}"
    check_lse(lse.cpu(), lse_ref)
    bound = _fp8_o_bound(q, k, v, o_ref, causal, scale)
    err = np.abs(g - o_ref)
    worst = float(np.max(err - bound))
    assert worst <= 0.0, f"O exceeds the e4m3 worst-case bound by {worst:.3e}"
    return rl


def _fp8_o_bound(q, k, v, o_ref, causal, scale):
    """Element-wise worst-case error bound of the e4m3 forward (module doc)."""
    nk, hkv, H = k.shape[-2], k.shape[1], q.shape[1]
    eye = np.broadcast_to(np.eye(nk), (k.shape[0], hkv, nk, nk)).copy()
    P, _ = oracle.attention_forward(q, k, eye, causal, scale)   # [B, H, Nq, Nk]
    absv = oracle.expand_kv_heads(np.abs(v), H)                 # [B, H, Nk, d]
    pmax = P.max(axis=-1, keepdims=True)
    small = (P < 2.0 ** -6 * pmax).astype(np.float64)
    return (2.0 ** -4 * (P @ absv) + 2.0 ** -10 * pmax * (small @ absv)
            + 2.0 ** -8 * np.abs(o_ref) + 1e-5)


CASES = [  # (B, H, Hkv, Nq, Nk); Nk is a multiple of 16 (rows of vt)
    (1, 2, 2, 256, 256), (2, 2, 1, 513, 512), (1, 4, 2, 1000, 1024), (1, 2, 2, 300, 1200),
    (1, 2, 2, 1200, 304), (1, 1, 1, 1, 16),
]


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("case", CASES, ids=lambda c: "B%dH%dHkv%dNq%dNk%d" % c)
def test_fwd_fp8_matches_oracle(fa_mod, cuda_device, case, causal):
    B, H, Hkv, Nq, Nk = case
    q8, k8, vt8, sc = inputs.fp8_inputs(B, H, Nq, 128, seed=7000 + Nq + Nk + causal, Hkv=Hkv,
                                        Nk=Nk)
    rl = _check(q8, k8, vt8, sc, causal, fa_mod)
    # the error model says about 0.036; far below that would mean P is not
    # rounded to e4m3 at all, far above a wrong layout or scale
    assert rl > 5e-3


def test_fwd_fp8_scales_are_applied(fa_mod, cuda_device):
    """The V descale factor multiplies O and nothing else: four times the
    factor gives exactly four times O (a power of two commutes with every
    rounding) and the same LSE."""
    q8, k8, vt8, (qs, ks, vs) = inputs.fp8_inputs(1, 2, 384, 128, seed=7100, Nk=384)
    o1, l1 = fa_mod.fwd_fp8(q8.to(DEV), k8.to(DEV), vt8.to(DEV), qs, ks, vs, causal=True)
    o2, l2 = fa_mod.fwd_fp8(q8.to(DEV), k8.to(DEV), vt8.to(DEV), qs, ks, 4.0 * vs, causal=True)
    torch.cuda.synchronize()
    assert torch.equal(o2.float(), (4.0 * o1.float()).to(torch.bfloat16).float())
    assert torch.equal(l1, l2)


def test_fwd_fp8_rejects_unsupported_shapes(fa_mod, cuda_device):
    q8, k8, vt8, sc = inputs.fp8_inputs(1, 1, 64, 128, seed=7200, Nk=40)  # Nk % 16 != 0
    with pytest.raises(fa_mod.FAError):
        fa_mod.fwd_fp8(q8.to(DEV), k8.to(DEV), vt8.to(DEV), *sc)
