"""The debug build (FA_DEBUG): the same kernels with a bounds check on every
computed global address and TMA coordinate.  A failed check would record
FA_ERR_BOUNDS in the device error word and skip the access; on correct inputs
no check may fail and the results must still be the oracle's.  The library is
built as lib/libfa_b200_debug.so and loaded in a child process (a process
loads one build of the library)."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

_SCRIPT = r"""
import sys
import numpy as np, torch
sys.path.insert(0, {root!r})
import oracle
from io_aware_exact_35_b200 import fa, inputs
from tests._parity import check_o, check_lse, check_grad
assert fa.library_path().endswith("libfa_b200_debug.so"), fa.library_path()
dev = torch.device("cuda:0")
f64 = inputs.to_f64

def clean():
    torch.cuda.synchronize()
    err = fa.get_device_error()
    assert err == 0, f"device error word {{err}} (6 = a bounds check failed)"

# forward and backward, padded layout, ragged lengths, both head dims, grouped heads
for (B, H, Hkv, N, d, causal) in [(1, 2, 2, 200, 128, True), (2, 2, 1, 333, 64, False),
                                  (1, 4, 2, 700, 128, True), (2, 1, 1, 1, 64, True)]:
    q, k, v, do = inputs.bwd_inputs(B, H, N, d, seed=N + d, Hkv=Hkv)
    qd, kd, vd, dod = (t.to(dev) for t in (q, k, v, do))
    o, lse = fa.fwd(qd, kd, vd, causal=causal)
    dq, dk, dv = fa.bwd(qd, kd, vd, o, dod, lse, causal=causal)
    clean()
    ro, rl = oracle.attention_forward(f64(q), f64(k), f64(v), causal, 1 / np.sqrt(d))
    check_o(o.cpu(), ro)
    check_lse(lse.cpu(), rl)
    rq, rk, rv, _ = oracle.attention_backward(f64(q), f64(k), f64(v), f64(do), causal, 1 / np.sqrt(d))
    check_grad(dq.cpu(), rq, "dQ"); check_grad(dk.cpu(), rk, "dK"); check_grad(dv.cpu(), rv, "dV")

# unequal query / key lengths
q, k, v = inputs.fwd_inputs(1, 2, 300, 128, seed=7, Nk=900)
o, lse = fa.fwd(q.to(dev), k.to(dev), v.to(dev), causal=True)
clean()
ro, rl = oracle.attention_forward(f64(q), f64(k), f64(v), True, 1 / np.sqrt(128))
check_o(o.cpu(), ro)

# ragged batch, forward and backward
lens = [1, 130, 257, 600]
q, k, v, do, cu_q, cu_k = inputs.varlen_inputs(lens, lens, 2, 1, 128, seed=11, with_do=True)
qd, kd, vd, dod, cqd, ckd = (t.to(dev) for t in (q, k, v, do, cu_q, cu_k))
o, lse = fa.fwd_varlen(qd, kd, vd, cqd, ckd, max(lens), causal=True)
dq, dk, dv = fa.bwd_varlen(qd, kd, vd, o, dod, lse, cqd, ckd, max(lens), causal=True)
clean()
for b, L in enumerate(lens):
    a, e = int(cu_q[b]), int(cu_q[b + 1])
    t = [f64(x[a:e].transpose(0, 1)[None]) for x in (q, k, v)]
    ro, _ = oracle.attention_forward(*t, True, 1 / np.sqrt(128))
    check_o(o[a:e].transpose(0, 1).cpu(), ro[0], f"varlen O seq {{b}}")

# decode, contiguous and paged, with NaN tails
sl = [0, 1, 511, 513, 2000]
qq, kc, vc, sld = inputs.decode_inputs(len(sl), 4, 128, 0, 2000, seed=13, seqlens=sl, Lcap=2000,
                                       Hkv=2)
od, ld = fa.decode(qq.to(dev), kc.to(dev), vc.to(dev), sld.to(dev))
kp, vp, table = inputs.page_cache(kc, vc, sld, 16, 14)
op, lp = fa.decode_paged(qq.to(dev), kp.to(dev), vp.to(dev), table.to(dev), sld.to(dev))
clean()
ro, rl = oracle.decode_forward(f64(qq), f64(kc), f64(vc), sl, 1 / np.sqrt(128))
check_o(od.cpu(), ro); check_lse(ld.cpu(), rl)
check_o(op.cpu(), ro); check_lse(lp.cpu(), rl)

# e4m3 forward
q8, k8, vt8, (qs, ks, vs) = inputs.fp8_inputs(1, 2, 300, 128, seed=15, Nk=304)
o8, _ = fa.fwd_fp8(q8.to(dev), k8.to(dev), vt8.to(dev), qs, ks, vs, causal=True)
clean()
print("debug build ok")
"""


def test_debug_build_small_cases_have_a_clean_error_word(cuda_device):
    from io_aware_exact_35_b200 import build
    lib = build.build(debug=True)
    env = dict(os.environ, FA_B200_LIBRARY=lib)
    r = subprocess.run([sys.executable, "-c", _SCRIPT.format(root=ROOT)], env=env,
                       capture_output=True, text=True, timeout=900, cwd=ROOT)
    assert r.returncode == 0 and "debug build ok" in r.stdout, r.stdout[-3000:] + r.stderr[-3000:]
