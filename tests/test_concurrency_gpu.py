"""Calls from several host threads at once, each on its own CUDA stream.

The library opts each kernel in to its shared-memory size once per device
(the first launch on that device).  Here, in a fresh process, the first call
of every entry point happens on four threads at the same time; every result
must equal the one the same call gives when run alone afterwards (the
forward, the e4m3 forward and decode are deterministic, so bit for bit; the
backward's dQ accumulates in L2 in an order that varies, so dK and dV bit for
bit and dQ to its fp32 rounding)."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

SCRIPT = r"""
import sys, threading
sys.path.insert(0, {root!r})
import torch
from io_aware_exact_35_b200 import fa, inputs

dev = torch.device("cuda:0")
q, k, v = (t.to(dev) for t in inputs.fwd_inputs(2, 4, 700, 128, seed=1, Hkv=2))
qb, kb, vb, dob = (t.to(dev) for t in inputs.bwd_inputs(1, 2, 520, 128, seed=2))
q8, k8, vt8, sc = inputs.fp8_inputs(1, 2, 384, 128, seed=3, Nk=384)
q8, k8, vt8 = q8.to(dev), k8.to(dev), vt8.to(dev)
qd, kc, vc, sl = inputs.decode_inputs(4, 8, 128, 100, 3000, seed=4)
qd, kc, vc, sl = qd.to(dev), kc.to(dev), vc.to(dev), sl.to(dev)
ob, lseb = fa.fwd(qb, kb, vb, causal=True)  # inputs of the backward (not timed)
torch.cuda.synchronize()

def run(kind, stream):
    if kind == "fwd":
        return fa.fwd(q, k, v, causal=True, stream=stream)
    if kind == "fp8":
        return fa.fwd_fp8(q8, k8, vt8, *sc, causal=True, stream=stream)
    if kind == "bwd":
        return fa.bwd(qb, kb, vb, ob, dob, lseb, causal=True, stream=stream)
    return fa.decode(qd, kc, vc, sl, stream=stream)

kinds = ["fwd", "fp8", "bwd", "decode"]
results, errors = {{}}, []
start = threading.Barrier(len(kinds))
def worker(kind):
    try:
        s = torch.cuda.Stream()
        start.wait()
        with torch.cuda.stream(s):
            r = run(kind, s)
        s.synchronize()
        results[kind] = [t.clone() for t in r]
    except Exception as e:  # reported below
        errors.append(repr(e))
threads = [threading.Thread(target=worker, args=(kd,)) for kd in kinds]
for t in threads: t.start()
for t in threads: t.join()
assert not errors, errors
assert fa.get_device_error() == 0
for kind in kinds:
    ref = run(kind, None)
    torch.cuda.synchronize()
    for i, (a, b) in enumerate(zip(results[kind], ref)):
        if kind == "bwd" and i == 0:
            err = (a.float() - b.float()).abs().max().item()
            scale = b.float().abs().max().item()
            assert err <= 1e-2 * scale, (kind, i, err, scale)
        else:
            assert torch.equal(a, b), (kind, i)
print("ok")
"""


def test_first_calls_from_several_threads(cuda_device, fa_mod):
    out = subprocess.run([sys.executable, "-c", SCRIPT.format(root=ROOT)], capture_output=True,
                         text=True, timeout=600)
    assert out.returncode == 0 and out.stdout.strip().endswith("ok"), out.stdout + out.stderr
