"""Shared comparison helpers for the GPU parity tests (tolerances of the spec).

Forward / decode outputs (bf16): max-abs error <= 1e-2 and relative L2 error
<= 5e-3 against the unrounded fp64 oracle.  LSE (fp32): max-abs <= 1e-3.
Gradients (bf16): relative L2 <= 1e-2.
"""
import numpy as np
import torch

O_MAX_ABS = 1e-2
O_REL_L2 = 5e-3
LSE_MAX_ABS = 1e-3
GRAD_REL_L2 = 1e-2


def as_f64(t):
    if isinstance(t, torch.Tensor):
        return t.detach().to("cpu").to(torch.float64).numpy()
    return np.asarray(t, dtype=np.float64)


def rel_l2(a, b):
    a, b = as_f64(a), as_f64(b)
    den = np.linalg.norm(b.ravel())
    return float(np.linalg.norm((a - b).ravel()) / (den if den > 0 else 1.0))


def check_o(got, ref, what="O"):
    g, r = as_f64(got), as_f64(ref)
    assert g.shape == r.shape, (g.shape, r.shape)
    assert np.isfinite(g).all(), f"{what}: non-finite values"
    err = float(np.max(np.abs(g - r))) if g.size else 0.0
    rl = rel_l2(g, r) if g.size else 0.0
    assert err <= O_MAX_ABS, f"{what}: max-abs error {err:.3e} > {O_MAX_ABS}"
    assert rl <= O_REL_L2, f"{what}: relative L2 error {rl:.3e} > {O_REL_L2}"
    return err, rl


def check_lse(got, ref, what="LSE"):
    g, r = as_f64(got), as_f64(ref)
    assert g.shape == r.shape
    both_inf = np.isneginf(g) & np.isneginf(r)
    diff = np.where(both_inf, 0.0, np.abs(g - r))
    err = float(np.max(diff)) if g.size else 0.0
    assert err <= LSE_MAX_ABS, f"{what}: max-abs error {err:.3e} > {LSE_MAX_ABS}"
    return err


def check_grad(got, ref, what):
    rl = rel_l2(got, ref)
    assert np.isfinite(as_f64(got)).all(), f"{what}: non-finite values"
    assert rl <= GRAD_REL_L2, f"{what}: relative L2 error {rl:.3e} > {GRAD_REL_L2}"
    return rl

