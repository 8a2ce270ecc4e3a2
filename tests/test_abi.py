"""CPU checks of the C ABI: the library builds for sm_100a, loads, exports every
entry point declared in include/*.h, and sizes workspaces / rejects bad
arguments on the host before touching a device."""
import ctypes
import glob
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        for m in re.finditer(r"\b(fa_\w+)\s*\(", text):
            names.add(m.group(1))
    return names


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("fa_fwd", "fa_bwd", "fa_decode", "fa_bwd_workspace_size",
                     "fa_decode_workspace_size", "fa_get_device_error", "fa_status_string"):
        assert required in names


def test_library_exports_every_declared_symbol(fa_mod):
    lib = ctypes.CDLL(fa_mod.library_path())
    for name in declared_functions():
        assert hasattr(lib, name), f"{name} declared in include/ but not exported"
    assert set(fa_mod.SIGNATURES) <= declared_functions()


def test_status_strings(fa_mod):
    for code in range(7):
        assert fa_mod.status_string(code)
    assert fa_mod.lib().fa_version() >= 100


def test_workspace_sizes(fa_mod):
    B, H, N, d = 2, 16, 8192, 128
    ws = fa_mod.bwd_workspace_size(B, H, N, d)
    rows = B * H * N
    assert ws >= rows * 4 + rows * d * 4
    assert ws % 256 == 0
    # D and log2(e) LSE on 128-padded rows, the fp32 dQ accumulator and one
    # uint32 completion counter per (batch, head), each 256-byte aligned
    up = lambda x: (x + 255) // 256 * 256
    padded = B * H * ((N + 127) // 128 * 128)
    assert ws == 2 * up(padded * 4) + up(rows * d * 4) + up(B * H * 4)
    assert fa_mod.bwd_workspace_size(1, 3, 1, 64) == 2 * up(3 * 128 * 4) + up(3 * 64 * 4) + up(12)
    assert fa_mod.bwd_workspace_size(0, 1, 1, 128) == 0
    assert fa_mod.bwd_workspace_size(1, 1, 1, 96) == 0
    wd = fa_mod.decode_workspace_size(16, 32, 16384, 128)
    assert wd >= 16 * 32 * (d + 2) * 4 and wd % 256 == 0
    assert fa_mod.decode_workspace_size(1, 1, 0, 128) == 0
    assert fa_mod.decode_workspace_size(1, 1, 10, 80) == 0


def test_host_validation_rejects_bad_arguments(fa_mod):
    lib = fa_mod.lib()
    P = 1 << 20  # a fake, aligned address: never dereferenced on these paths
    INVALID, UNSUPPORTED, WORKSPACE = 1, 2, 3
    # null pointers, negative sizes, misalignment, bad flags, bad head dims
    assert lib.fa_fwd(None, P, P, P, None, 1, 1, 8, 64, 0, 1.0, None) == INVALID
    assert lib.fa_fwd(P, P, P, P, None, 0, 1, 8, 64, 0, 1.0, None) == INVALID
    assert lib.fa_fwd(P, P, P, P, None, 1, 1, -1, 64, 0, 1.0, None) == INVALID
    assert lib.fa_fwd(P + 8, P, P, P, None, 1, 1, 8, 64, 0, 1.0, None) == INVALID
    assert lib.fa_fwd(P, P, P, P, P + 2, 1, 1, 8, 64, 0, 1.0, None) == INVALID
    assert lib.fa_fwd(P, P, P, P, None, 1, 1, 8, 64, 2, 1.0, None) == INVALID
    assert lib.fa_fwd(P, P, P, P, None, 1, 1, 8, 64, 0, float("nan"), None) == INVALID
    assert lib.fa_fwd(P, P, P, P, None, 1, 1, 8, 96, 0, 1.0, None) == UNSUPPORTED
    assert lib.fa_fwd(P, P, P, P, None, 1024, 1024, 1 << 20, 64, 0, 1.0, None) == INVALID
    # backward: workspace checks
    args = [P] * 6 + [P, P, P]
    assert lib.fa_bwd(*args, None, 0, 1, 1, 8, 64, 0, 1.0, None) == WORKSPACE
    assert lib.fa_bwd(*args, P, 16, 1, 1, 8, 64, 0, 1.0, None) == WORKSPACE
    assert lib.fa_bwd(*args, P + 16, 1 << 20, 1, 1, 8, 64, 0, 1.0, None) == WORKSPACE
    assert lib.fa_bwd(None, *args[1:], P, 1 << 20, 1, 1, 8, 64, 0, 1.0, None) == INVALID
    # decode
    assert lib.fa_decode(P, P, P, P, P, None, 1, 1, 1024, 128, 1.0, None, 0, None) == WORKSPACE
    assert lib.fa_decode(P, P, P, P + 2, P, None, 1, 1, 1024, 128, 1.0, P, 1 << 20, None) == INVALID
    assert lib.fa_decode(P, P, P, P, P, None, 1, 1, 1024, 80, 1.0, P, 1 << 20, None) == UNSUPPORTED
    assert lib.fa_decode(P, P, None, P, P, None, 1, 1, 1024, 128, 1.0, P, 1 << 20, None) == INVALID
    # separate query / key lengths
    ext = lib.fa_fwd_ext
    assert ext(P, P, P, P, None, 1, 2, 3, 8, 8, 64, 0, 1.0, None) == INVALID    # 3 does not divide 2
    assert ext(P, P, P, P, None, 1, 2, 1, -1, 8, 64, 0, 1.0, None) == INVALID   # Nq < 0
    assert ext(P, P, P, P, None, 1, 2, 1, 8, -1, 64, 0, 1.0, None) == INVALID   # Nk < 0
    assert ext(P, None, P, P, None, 1, 2, 1, 8, 8, 64, 0, 1.0, None) == INVALID  # k null, Nk > 0
    assert ext(P, P, P, P, None, 1, 1, 1, (1 << 30) + 1, 1 << 30, 64, 0, 1.0, None) == INVALID
    bext = lib.fa_bwd_ext
    assert bext(*args, None, 0, 1, 1, 1, 8, 5, 64, 1, 1.0, None) == WORKSPACE
    assert bext(P, P, P, P, P, P, P, None, P, P, 1 << 20, 1, 1, 1, 8, 5, 64, 1, 1.0,
                None) == INVALID                                                # dk null
    # ragged batch
    vl = lib.fa_fwd_varlen
    assert vl(P, P, P, P, None, None, P, 2, 4, 2, 100, 100, 64, 128, 1, 1.0, None) == INVALID  # cu_q null
    assert vl(P, P, P, P, None, P, P, 2, 4, 3, 100, 100, 64, 128, 1, 1.0, None) == INVALID    # Hkv
    assert vl(P, P, P, P, None, P, P, 0, 4, 2, 100, 100, 64, 128, 1, 1.0, None) == INVALID    # B < 1
    assert vl(P, P, P, P, None, P, P, 2, 4, 2, -1, 100, 64, 128, 1, 1.0, None) == INVALID     # total_q
    assert vl(P, P, P, P, None, P + 2, P, 2, 4, 2, 100, 100, 64, 128, 1, 1.0, None) == INVALID
    assert vl(P, P, P, P, None, P, P, 2, 4, 2, 100, 100, 64, 80, 1, 1.0, None) == UNSUPPORTED
    assert vl(P, None, P, P, None, P, P, 2, 4, 2, 100, 100, 64, 128, 1, 1.0, None) == INVALID  # k null
    bvl = lib.fa_bwd_varlen
    ten = [P] * 9 + [P, P]  # q k v o dout lse dq dk dv cu_q cu_k
    assert bvl(*ten, None, 0, 2, 4, 2, 100, 100, 64, 128, 1, 1.0, None) == WORKSPACE
    assert bvl(*ten[:9], None, P, P, 1 << 30, 2, 4, 2, 100, 100, 64, 128, 1, 1.0, None) == INVALID
    assert bvl(*ten, P, 1 << 30, 2, 4, 2, 100, 100, 64, 96, 1, 1.0, None) == UNSUPPORTED
    assert lib.fa_bwd_varlen_workspace_size(2, 4, 100, 128) > 0
    assert lib.fa_bwd_varlen_workspace_size(0, 4, 100, 128) == 0
    f8 = lib.fa_fwd_fp8
    assert f8(P, P, P, P, None, 1.0, 1.0, 1.0, 1, 2, 2, 64, 64, 64, 0, 1.0, None) == UNSUPPORTED   # d
    assert f8(P, P, P, P, None, 1.0, 1.0, 1.0, 1, 2, 2, 64, 40, 128, 0, 1.0, None) == UNSUPPORTED  # Nk % 16
    assert f8(P, P, P, P, None, float("nan"), 1.0, 1.0, 1, 2, 2, 64, 64, 128, 0, 1.0, None) == INVALID
    assert f8(P, P, None, P, None, 1.0, 1.0, 1.0, 1, 2, 2, 64, 64, 128, 0, 1.0, None) == INVALID
    assert f8(P, P, P, P, None, 1.0, 1.0, 1.0, 1, 2, 3, 64, 64, 128, 0, 1.0, None) == INVALID
    # paged decode: page size must be a power of two, table needed
    dp = lib.fa_decode_paged
    assert dp(P, P, P, P, P, P, None, 2, 4, 2, 24, 8, 16, 128, 1.0, P, 1 << 20, None) == INVALID
    assert dp(P, P, P, P, P, P, None, 2, 4, 2, 0, 8, 16, 128, 1.0, P, 1 << 20, None) == INVALID
    assert dp(P, P, P, None, P, P, None, 2, 4, 2, 16, 8, 16, 128, 1.0, P, 1 << 20, None) == INVALID
    assert dp(P, P, P, P, P, P, None, 2, 4, 3, 16, 8, 16, 128, 1.0, P, 1 << 20, None) == INVALID
    assert dp(P, P, P, P, P, P, None, 2, 4, 2, 16, 8, 16, 96, 1.0, P, 1 << 20, None) == UNSUPPORTED
    assert dp(P, P, P, P, P, P, None, 2, 4, 2, 16, 8, 16, 128, 1.0, None, 0, None) == WORKSPACE
    assert dp(P, P, P, P, P, P, None, 2, 4, 2, 1 << 16, 1 << 15, 16, 128, 1.0, P, 1 << 20,
              None) == INVALID                                                  # Lmax > INT_MAX


def test_binding_fails_loudly_without_cuda_tensors(fa_mod):
    import torch
    x = torch.zeros(1, 1, 8, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        fa_mod.fwd(x, x, x)


def test_bounded_wait_check_validates_pointer(fa_mod):
    lib = fa_mod.lib()
    INVALID = 1
    assert lib.fa_check_bounded_wait(None, None) == INVALID
    assert lib.fa_check_bounded_wait((1 << 20) + 2, None) == INVALID


def test_set_schedule_validates_and_resets(fa_mod):
    lib = fa_mod.lib()
    assert lib.fa_set_schedule(3, 0) == 1 and lib.fa_set_schedule(0, -1) == 1
    for f in (0, 1, 2):
        for b in (0, 1, 2):
            assert lib.fa_set_schedule(f, b) == 0
    fa_mod.set_schedule("grid", "persistent")
    fa_mod.set_schedule()  # back to the library's own choice
    with pytest.raises(KeyError):
        fa_mod.set_schedule("sideways")
