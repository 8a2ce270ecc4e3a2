"""Python binding of libfa_b200.so (argument marshalling only).

Every function takes torch CUDA tensors, checks dtype / shape / contiguity,
allocates outputs when none are given, and calls the C ABI of
include/fa_b200.h with raw device pointers and the current CUDA stream.  All
arithmetic happens in the library's sm_100a kernels; there is no fallback:
if the library is missing or the device is unsupported, the call raises.
"""

from __future__ import annotations

import ctypes
import math
import os
from typing import Optional

import torch

# The in-tree build; FA_B200_LIBRARY may point at another build of the same library.
_LIB_PATH = os.environ.get("FA_B200_LIBRARY") or os.path.join(
    os.path.dirname(os.path.abspath(__file__)), "lib", "libfa_b200.so")
_lib = None

FA_OK = 0
STATUS_NAMES = {0: "FA_OK", 1: "FA_ERR_INVALID_ARG", 2: "FA_ERR_UNSUPPORTED",
                3: "FA_ERR_WORKSPACE", 4: "FA_ERR_CUDA", 5: "FA_ERR_TIMEOUT",
                6: "FA_ERR_BOUNDS"}

# Public entry points and their C signatures (restype, argtypes).
_P, _I, _F, _S = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
SIGNATURES = {
    "fa_fwd": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _F, _P]),
    "fa_fwd_gqa": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _P]),
    "fa_fwd_ext": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _F, _P]),
    "fa_fwd_varlen": (_I, [_P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _F,
                           _P]),
    "fa_fwd_fp8": (_I, [_P, _P, _P, _P, _P, _F, _F, _F, _I, _I, _I, _I, _I, _I, _I, _F, _P]),
    "fa_bwd_workspace_size": (_S, [_I, _I, _I, _I]),
    "fa_bwd_varlen_workspace_size": (_S, [_I, _I, _I, _I]),
    "fa_bwd_varlen": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _S, _I, _I, _I, _I, _I,
                           _I, _I, _I, _F, _P]),
    "fa_bwd": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _S, _I, _I, _I, _I, _I, _F, _P]),
    "fa_bwd_gqa": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _S, _I, _I, _I, _I, _I, _I, _F,
                        _P]),
    "fa_bwd_ext": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _S, _I, _I, _I, _I, _I, _I, _I,
                        _F, _P]),
    "fa_decode_workspace_size": (_S, [_I, _I, _I, _I]),
    "fa_decode": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _F, _P, _S, _P]),
    "fa_decode_gqa": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _F, _P, _S, _P]),
    "fa_decode_static": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _F, _P]),
    "fa_decode_paged": (_I, [_P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _F, _P, _S,
                             _P]),
    "fa_get_device_error": (_I, [_P]),
    "fa_check_bounded_wait": (_I, [_P, _P]),
    "fa_set_timing_events": (_I, [_P, _P]),
    "fa_set_schedule": (_I, [_I, _I]),
    "fa_status_string": (ctypes.c_char_p, [_I]),
    "fa_version": (_I, []),
}


class FAError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        name = STATUS_NAMES.get(status, str(status))
        super().__init__(f"{fn} failed: {name} ({status_string(status)})")


def library_path() -> str:
    return _LIB_PATH


def lib():
    """Load libfa_b200.so once; raise if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise RuntimeError(f"{_LIB_PATH} is missing: build it with "
                               "`python -m io_aware_exact_35_b200.build`")
        handle = ctypes.CDLL(_LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(handle, name)
            fn.restype, fn.argtypes = res, args
        _lib = handle
    return _lib


def status_string(status: int) -> str:
    return lib().fa_status_string(int(status)).decode()


def _check(fn: str, status: int) -> None:
    if status != FA_OK:
        raise FAError(fn, status)


def _stream_ptr(stream: Optional[torch.cuda.Stream]) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _req(t: torch.Tensor, name: str, dtype: torch.dtype, ndim: int) -> None:
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, causal: bool = False,
        scale: Optional[float] = None, out: Optional[torch.Tensor] = None,
        lse: Optional[torch.Tensor] = None, want_lse: bool = True, stream=None):
    """Exact attention forward.  q: bf16 [B, H, Nq, d]; k, v: bf16 [B, Hkv, Nk, d]
    with Hkv dividing H (Hkv < H: grouped-query attention).  With Nq != Nk the
    queries are the last Nq positions of the key sequence (causal mask
    j <= i + Nk - Nq).  Returns (o [B, H, Nq, d], lse [B, H, Nq])."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _req(t, n, torch.bfloat16, 4)
    B, H, N, d = q.shape
    Hkv, Nk = k.shape[1], k.shape[2]
    if (tuple(k.shape) != (B, Hkv, Nk, d) or v.shape != k.shape or Hkv < 1 or H % Hkv):
        raise ValueError("k and v must be [B, Hkv, Nk, d] with Hkv dividing q's H")
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    if out is None:
        out = torch.empty_like(q)
    _req(out, "out", torch.bfloat16, 4)
    if out.shape != q.shape:
        raise ValueError("out must match q")
    if lse is None and want_lse:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    if lse is not None:
        _req(lse, "lse", torch.float32, 3)
        if tuple(lse.shape) != (B, H, N):
            raise ValueError("lse must be [B, H, N]")
    st = lib().fa_fwd_ext(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), _ptr(lse),
                          B, H, Hkv, N, Nk, d, int(bool(causal)), scale, _stream_ptr(stream))
    _check("fa_fwd_ext", st)
    return out, lse


def fwd_varlen(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, cu_seqlens_q: torch.Tensor,
               cu_seqlens_k: torch.Tensor, max_seqlen_q: int, causal: bool = False,
               scale: Optional[float] = None, out: Optional[torch.Tensor] = None,
               lse: Optional[torch.Tensor] = None, want_lse: bool = True, stream=None):
    """Forward over a ragged batch packed token-major: q [total_q, H, d],
    k, v [total_k, Hkv, d] bf16; cu_seqlens_q / cu_seqlens_k int32 [B + 1] on
    the device; max_seqlen_q bounds the query lengths.  Returns
    (o [total_q, H, d], lse [H, total_q])."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _req(t, n, torch.bfloat16, 3)
    _req(cu_seqlens_q, "cu_seqlens_q", torch.int32, 1)
    _req(cu_seqlens_k, "cu_seqlens_k", torch.int32, 1)
    total_q, H, d = q.shape
    total_k, Hkv = k.shape[0], k.shape[1]
    if tuple(k.shape) != (total_k, Hkv, d) or v.shape != k.shape or Hkv < 1 or H % Hkv:
        raise ValueError("k and v must be [total_k, Hkv, d] with Hkv dividing q's H")
    B = cu_seqlens_q.shape[0] - 1
    if B < 1 or cu_seqlens_k.shape[0] != B + 1:
        raise ValueError("cu_seqlens_q and cu_seqlens_k must both have B + 1 entries")
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    if out is None:
        out = torch.empty_like(q)
    _req(out, "out", torch.bfloat16, 3)
    if out.shape != q.shape:
        raise ValueError("out must match q")
    if lse is None and want_lse:
        lse = torch.empty((H, total_q), dtype=torch.float32, device=q.device)
    if lse is not None:
        _req(lse, "lse", torch.float32, 2)
        if tuple(lse.shape) != (H, total_q):
            raise ValueError("lse must be [H, total_q]")
    st = lib().fa_fwd_varlen(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), _ptr(lse),
                             cu_seqlens_q.data_ptr(), cu_seqlens_k.data_ptr(), B, H, Hkv, total_q,
                             total_k, int(max_seqlen_q), d, int(bool(causal)), scale,
                             _stream_ptr(stream))
    _check("fa_fwd_varlen", st)
    return out, lse


def fwd_fp8(q: torch.Tensor, k: torch.Tensor, vt: torch.Tensor, q_scale: float,
            k_scale: float, v_scale: float, causal: bool = False, scale: Optional[float] = None,
            out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
            want_lse: bool = True, stream=None):
    """Forward with e4m3 inputs: q [B, H, Nq, 128], k [B, Hkv, Nk, 128] and V
    transposed, vt [B, Hkv, 128, Nk] (torch.float8_e4m3fn), one descale factor
    per tensor.  Returns (o [B, H, Nq, 128] bf16, lse [B, H, Nq])."""
    for t, n in ((q, "q"), (k, "k"), (vt, "vt")):
        _req(t, n, torch.float8_e4m3fn, 4)
    B, H, N, d = q.shape
    Hkv, Nk = k.shape[1], k.shape[2]
    if tuple(k.shape) != (B, Hkv, Nk, d) or tuple(vt.shape) != (B, Hkv, d, Nk) or H % Hkv:
        raise ValueError("k must be [B, Hkv, Nk, d] and vt [B, Hkv, d, Nk], Hkv dividing H")
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    if out is None:
        out = torch.empty((B, H, N, d), dtype=torch.bfloat16, device=q.device)
    _req(out, "out", torch.bfloat16, 4)
    if lse is None and want_lse:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    st = lib().fa_fwd_fp8(q.data_ptr(), k.data_ptr(), vt.data_ptr(), out.data_ptr(), _ptr(lse),
                          float(q_scale), float(k_scale), float(v_scale), B, H, Hkv, N, Nk, d,
                          int(bool(causal)), scale, _stream_ptr(stream))
    _check("fa_fwd_fp8", st)
    return out, lse


def bwd_workspace_size(B: int, H: int, N: int, d: int) -> int:
    return int(lib().fa_bwd_workspace_size(B, H, N, d))


def bwd(q, k, v, o, do, lse, causal: bool = False, scale: Optional[float] = None,
        dq=None, dk=None, dv=None, workspace: Optional[torch.Tensor] = None, stream=None):
    """Backward with recomputation.  Returns (dq, dk, dv); dk and dv have k's
    shape [B, Hkv, Nk, d] (grouped heads accumulate over their query heads)."""
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (o, "o"), (do, "do")):
        _req(t, n, torch.bfloat16, 4)
    B, H, N, d = q.shape
    Hkv, Nk = k.shape[1], k.shape[2]
    if o.shape != q.shape or do.shape != q.shape:
        raise ValueError("o and do must match q's shape")
    if tuple(k.shape) != (B, Hkv, Nk, d) or v.shape != k.shape or H % Hkv:
        raise ValueError("k and v must be [B, Hkv, Nk, d] with Hkv dividing q's H")
    _req(lse, "lse", torch.float32, 3)
    if tuple(lse.shape) != (B, H, N):
        raise ValueError("lse must be [B, H, N]")
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    for t, n in ((dq, "dq"), (dk, "dk"), (dv, "dv")):
        _req(t, n, torch.bfloat16, 4)
    need = bwd_workspace_size(B, H, N, d)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    if dq.shape != q.shape or dk.shape != k.shape or dv.shape != v.shape:
        raise ValueError("gradient buffers must match q, k, v")
    st = lib().fa_bwd_ext(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), do.data_ptr(),
                          lse.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(),
                          workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                          B, H, Hkv, N, Nk, d, int(bool(causal)), scale, _stream_ptr(stream))
    _check("fa_bwd_ext", st)
    return dq, dk, dv


def bwd_varlen(q, k, v, o, do, lse, cu_seqlens_q, cu_seqlens_k, max_seqlen_k: int,
               causal: bool = False, scale: Optional[float] = None, dq=None, dk=None, dv=None,
               workspace: Optional[torch.Tensor] = None, stream=None):
    """Backward over a ragged batch packed token-major (layouts of
    fwd_varlen; lse [H, total_q]).  Returns (dq, dk, dv)."""
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (o, "o"), (do, "do")):
        _req(t, n, torch.bfloat16, 3)
    _req(lse, "lse", torch.float32, 2)
    _req(cu_seqlens_q, "cu_seqlens_q", torch.int32, 1)
    _req(cu_seqlens_k, "cu_seqlens_k", torch.int32, 1)
    total_q, H, d = q.shape
    total_k, Hkv = k.shape[0], k.shape[1]
    if o.shape != q.shape or do.shape != q.shape:
        raise ValueError("o and do must match q's shape")
    if tuple(k.shape) != (total_k, Hkv, d) or v.shape != k.shape or H % Hkv:
        raise ValueError("k and v must be [total_k, Hkv, d] with Hkv dividing q's H")
    if tuple(lse.shape) != (H, total_q):
        raise ValueError("lse must be [H, total_q]")
    B = cu_seqlens_q.shape[0] - 1
    if B < 1 or cu_seqlens_k.shape[0] != B + 1:
        raise ValueError("cu_seqlens_q and cu_seqlens_k must both have B + 1 entries")
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    for t, n in ((dq, "dq"), (dk, "dk"), (dv, "dv")):
        _req(t, n, torch.bfloat16, 3)
    if dq.shape != q.shape or dk.shape != k.shape or dv.shape != v.shape:
        raise ValueError("gradient buffers must match q, k, v")
    need = int(lib().fa_bwd_varlen_workspace_size(B, H, total_q, d))
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    st = lib().fa_bwd_varlen(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                             do.data_ptr(), lse.data_ptr(), dq.data_ptr(), dk.data_ptr(),
                             dv.data_ptr(), cu_seqlens_q.data_ptr(), cu_seqlens_k.data_ptr(),
                             workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                             B, H, Hkv, total_q, total_k, int(max_seqlen_k), d,
                             int(bool(causal)), scale, _stream_ptr(stream))
    _check("fa_bwd_varlen", st)
    return dq, dk, dv


def decode_workspace_size(B: int, H: int, Lmax: int, d: int) -> int:
    return int(lib().fa_decode_workspace_size(B, H, Lmax, d))


def decode(q, kcache, vcache, seqlens, scale: Optional[float] = None, out=None, lse=None,
           want_lse: bool = True, workspace: Optional[torch.Tensor] = None, stream=None):
    """Split-KV decode.  q [B,H,d], caches [B,H,Lmax,d] bf16, seqlens int32 [B]
    on the device.  Returns (o [B,H,d] bf16, lse [B,H] fp32)."""
    _req(q, "q", torch.bfloat16, 3)
    _req(kcache, "kcache", torch.bfloat16, 4)
    _req(vcache, "vcache", torch.bfloat16, 4)
    _req(seqlens, "seqlens", torch.int32, 1)
    B, H, d = q.shape
    Hkv, Lmax = kcache.shape[1], kcache.shape[2]
    if tuple(kcache.shape) != (B, Hkv, Lmax, d) or vcache.shape != kcache.shape or H % Hkv:
        raise ValueError("caches must be [B, Hkv, Lmax, d] with Hkv dividing q's H")
    if seqlens.shape[0] != B:
        raise ValueError("seqlens must have B entries")
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    out = torch.empty_like(q) if out is None else out
    _req(out, "out", torch.bfloat16, 3)
    if lse is None and want_lse:
        lse = torch.empty((B, H), dtype=torch.float32, device=q.device)
    need = decode_workspace_size(B, H, Lmax, d)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    st = lib().fa_decode_gqa(q.data_ptr(), kcache.data_ptr(), vcache.data_ptr(),
                             seqlens.data_ptr(), out.data_ptr(), _ptr(lse), B, H, Hkv, Lmax, d,
                             scale, workspace.data_ptr(),
                             workspace.numel() * workspace.element_size(), _stream_ptr(stream))
    _check("fa_decode_gqa", st)
    return out, lse


def decode_paged(q, kpages, vpages, block_table, seqlens, scale: Optional[float] = None,
                 out=None, lse=None, want_lse: bool = True,
                 workspace: Optional[torch.Tensor] = None, stream=None):
    """Decode over a paged cache.  q [B,H,d] bf16; kpages/vpages
    [num_pages, Hkv, page_size, d] bf16; block_table int32 [B, pages_per_seq]
    and seqlens int32 [B] on the device.  Returns (o [B,H,d], lse [B,H])."""
    _req(q, "q", torch.bfloat16, 3)
    _req(kpages, "kpages", torch.bfloat16, 4)
    _req(vpages, "vpages", torch.bfloat16, 4)
    _req(block_table, "block_table", torch.int32, 2)
    _req(seqlens, "seqlens", torch.int32, 1)
    B, H, d = q.shape
    num_pages, Hkv, page_size = kpages.shape[0], kpages.shape[1], kpages.shape[2]
    if (tuple(kpages.shape) != (num_pages, Hkv, page_size, d) or vpages.shape != kpages.shape
            or H % Hkv):
        raise ValueError("page pools must be [num_pages, Hkv, page_size, d] with Hkv dividing H")
    if block_table.shape[0] != B or seqlens.shape[0] != B:
        raise ValueError("block_table and seqlens must have B rows")
    pages_per_seq = block_table.shape[1]
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    out = torch.empty_like(q) if out is None else out
    _req(out, "out", torch.bfloat16, 3)
    if lse is None and want_lse:
        lse = torch.empty((B, H), dtype=torch.float32, device=q.device)
    need = decode_workspace_size(B, H, pages_per_seq * page_size, d)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    st = lib().fa_decode_paged(q.data_ptr(), kpages.data_ptr(), vpages.data_ptr(),
                               block_table.data_ptr(), seqlens.data_ptr(), out.data_ptr(),
                               _ptr(lse), B, H, Hkv, page_size, pages_per_seq, num_pages, d,
                               scale, workspace.data_ptr(),
                               workspace.numel() * workspace.element_size(), _stream_ptr(stream))
    _check("fa_decode_paged", st)
    return out, lse


# Bytes of the library-owned scratch array behind fa_decode_static.
DECODE_STATIC_SCRATCH_BYTES = 16 * 1024 * 1024


def decode_static(q, kcache, vcache, seqlens, scale: Optional[float] = None, out=None,
                  lse=None, want_lse: bool = True, stream=None):
    """Split-KV decode that allocates nothing: the library keeps the scratch in
    a fixed device array (see fa_decode_static in include/fa_b200.h).  For
    callers that cannot allocate device memory, e.g. inside a host program
    that owns all of it.  Outputs must be passed in (or are created here by
    torch when omitted, which is an allocation of the caller's own).  Calls
    that overlap on the GPU share the scratch and race."""
    _req(q, "q", torch.bfloat16, 3)
    _req(kcache, "kcache", torch.bfloat16, 4)
    _req(vcache, "vcache", torch.bfloat16, 4)
    _req(seqlens, "seqlens", torch.int32, 1)
    B, H, d = q.shape
    Lmax = kcache.shape[2]
    if tuple(kcache.shape) != (B, H, Lmax, d) or vcache.shape != kcache.shape:
        raise ValueError("caches must be [B, H, Lmax, d] matching q")
    if seqlens.shape[0] != B:
        raise ValueError("seqlens must have B entries")
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    out = torch.empty_like(q) if out is None else out
    _req(out, "out", torch.bfloat16, 3)
    if lse is None and want_lse:
        lse = torch.empty((B, H), dtype=torch.float32, device=q.device)
    st = lib().fa_decode_static(q.data_ptr(), kcache.data_ptr(), vcache.data_ptr(),
                                seqlens.data_ptr(), out.data_ptr(), _ptr(lse), B, H, Lmax, d,
                                scale, _stream_ptr(stream))
    _check("fa_decode_static", st)
    return out, lse


def get_device_error(stream=None) -> int:
    """Synchronise the stream and return (and clear) the device error word."""
    return int(lib().fa_get_device_error(_stream_ptr(stream)))


def check_bounded_wait(gave_up: torch.Tensor, stream=None) -> None:
    """Launch the bounded-wait self-check: one CTA waits on a barrier that
    never completes, gives up after the wait limit and records FA_ERR_TIMEOUT
    in the device error word; 2 is added to ``gave_up`` (an int32 CUDA tensor)."""
    _req(gave_up, "gave_up", torch.int32, 1)
    _check("fa_check_bounded_wait", lib().fa_check_bounded_wait(gave_up.data_ptr(),
                                                                _stream_ptr(stream)))


def set_timing_events(start=None, stop=None) -> None:
    """Record ``start`` / ``stop`` (torch.cuda.Event, already recorded once so
    that their CUDA events exist) around the dominant kernel of every later
    call; ``None, None`` turns this off."""
    def handle(ev):
        if ev is None:
            return None
        if not ev.cuda_event:
            raise ValueError("record the event once before passing it")
        return ev.cuda_event
    _check("fa_set_timing_events", lib().fa_set_timing_events(handle(start), handle(stop)))


SCHEDULES = {"auto": 0, "grid": 1, "persistent": 2}


def set_schedule(fwd: str = "auto", bwd: str = "auto") -> None:
    """Force the work distribution of later calls (process-wide; results do
    not change): forward ``"grid"`` (one CTA per 256-row query tile) or
    ``"persistent"`` (CTAs looping over tiles); backward ``"grid"``
    (head-major) or ``"persistent"`` (longest key tiles first); ``"auto"``
    restores the library's own choice."""
    _check("fa_set_schedule", lib().fa_set_schedule(SCHEDULES[fwd], SCHEDULES[bwd]))
