"""Seeded synthetic inputs shared by the tests, the benchmark and the oracle checks.

This module draws random numbers and rounds them to bf16; it holds none of the
attention arithmetic.  Every draw uses a CPU ``torch.Generator`` seeded
explicitly, so both the CUDA path and the fp64 oracle see bit-identical inputs.

Recipe (the pages' seed 42 is the base; each workload adds its index):

* forward:  q, k, v ~ iid N(0,1) * std, drawn in that order as float32, then
  rounded to bf16 (round-to-nearest-even); k and v may have fewer heads
  (grouped queries) and another length than q;
* backward: q, k, v, dO drawn in that order the same way;
* decode:   seqlens ~ U{Lmin .. Lmax} (both ends inclusive) first, then
  q ~ N(0,1) [B, H, d], then for each sequence b in order: K_b, V_b ~ N(0,1)
  of shape [H, L_b, d].  Cache rows at or beyond L_b hold NaN so that any
  read past the prefix shows up in the outputs.
"""

from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np
import torch

BASE_SEED = 42


@dataclass(frozen=True)
class Workload:
    name: str
    kind: str            # "fwd" | "bwd" | "decode" | "fwd_varlen" | "fwd_fp8"
    B: int
    H: int
    d: int
    N: int = 0           # sequence length (fwd / bwd)
    causal: bool = False
    std: float = 1.0
    Lmin: int = 0        # decode / ragged batch: length range, inclusive
    Lmax: int = 0
    seed: int = BASE_SEED
    Hkv: int = 0         # key/value heads (0: same as H; fewer: grouped-query attention)
    page: int = 0        # decode: rows per cache page (0: contiguous cache)

    @property
    def kv_heads(self) -> int:
        return self.Hkv or self.H

    @property
    def scale(self) -> float:
        return 1.0 / float(np.sqrt(self.d))


# The five workloads: the shapes of a 2K-context prefill layer, a 32K
# long-context prefill, an 8K causal backward and a batched KV-cache decode,
# plus a small non-causal case that the oracle finishes instantly.
WORKLOADS = {
    w.name: w for w in (
        Workload("fwd_noncausal_B1_H2_N256_d64", "fwd", 1, 2, 64, N=256,
                 causal=False, seed=BASE_SEED + 0),
        Workload("fwd_causal_B4_H16_N2048_d128", "fwd", 4, 16, 128, N=2048,
                 causal=True, seed=BASE_SEED + 1),
        Workload("fwd_causal_B1_H32_N32768_d128", "fwd", 1, 32, 128, N=32768,
                 causal=True, std=0.5, seed=BASE_SEED + 2),
        Workload("bwd_causal_B2_H16_N8192_d128", "bwd", 2, 16, 128, N=8192,
                 causal=True, seed=BASE_SEED + 3),
        Workload("decode_B16_H32_d128_L4096-16384", "decode", 16, 32, 128,
                 Lmin=4096, Lmax=16384, seed=BASE_SEED + 4),
        # grouped-query variants (8 key/value heads shared by 32 query heads)
        Workload("fwd_causal_gqa_B4_H32_Hkv8_N2048_d128", "fwd", 4, 32, 128, N=2048,
                 causal=True, seed=BASE_SEED + 5, Hkv=8),
        Workload("bwd_causal_gqa_B2_H32_Hkv8_N4096_d128", "bwd", 2, 32, 128, N=4096,
                 causal=True, seed=BASE_SEED + 6, Hkv=8),
        Workload("decode_gqa_B16_H32_Hkv8_d128_L4096-16384", "decode", 16, 32, 128,
                 Lmin=4096, Lmax=16384, seed=BASE_SEED + 7, Hkv=8),
        # a ragged prefill batch: 16 sequences of U{512..4096} tokens, packed
        Workload("fwd_varlen_causal_B16_H16_d128_L512-4096", "fwd_varlen", 16, 16, 128,
                 causal=True, Lmin=512, Lmax=4096, seed=BASE_SEED + 9),
        # the 2K-context prefill with e4m3 inputs (V supplied transposed)
        Workload("fwd_fp8_causal_B4_H16_N2048_d128", "fwd_fp8", 4, 16, 128, N=2048,
                 causal=True, seed=BASE_SEED + 10),
        # the decode workload over a paged cache (16-row pages, random page order)
        Workload("decode_paged_B16_H32_d128_L4096-16384_p16", "decode", 16, 32, 128,
                 Lmin=4096, Lmax=16384, seed=BASE_SEED + 8, page=16),
    )
}


def _gen(seed: int) -> torch.Generator:
    return torch.Generator(device="cpu").manual_seed(int(seed))


def _randn_bf16(g: torch.Generator, shape, std: float = 1.0) -> torch.Tensor:
    x = torch.randn(shape, generator=g, dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    return x.to(torch.bfloat16)


def fwd_inputs(B: int, H: int, N: int, d: int, seed: int, std: float = 1.0,
               Hkv: int | None = None, Nk: int | None = None):
    """q [B, H, N, d] and k, v [B, Hkv, Nk, d] (Hkv defaults to H, Nk to N) as
    contiguous bf16 CPU tensors."""
    g = _gen(seed)
    hk = Hkv or H
    nk = N if Nk is None else Nk
    return (_randn_bf16(g, (B, H, N, d), std), _randn_bf16(g, (B, hk, nk, d), std),
            _randn_bf16(g, (B, hk, nk, d), std))


def bwd_inputs(B: int, H: int, N: int, d: int, seed: int, std: float = 1.0,
               Hkv: int | None = None, Nk: int | None = None):
    """q, k, v, dO as contiguous bf16 CPU tensors (k, v with Hkv heads of Nk
    rows)."""
    g = _gen(seed)
    hk = Hkv or H
    nk = N if Nk is None else Nk
    return (_randn_bf16(g, (B, H, N, d), std), _randn_bf16(g, (B, hk, nk, d), std),
            _randn_bf16(g, (B, hk, nk, d), std), _randn_bf16(g, (B, H, N, d), std))


def decode_inputs(B: int, H: int, d: int, Lmin: int, Lmax: int, seed: int,
                  Lcap: int | None = None, seqlens=None, poison: bool = True,
                  Hkv: int | None = None):
    """q [B,H,d], kcache/vcache [B,Hkv,Lcap,d] bf16 (Hkv defaults to H),
    seqlens int32 [B].

    ``seqlens`` may be given explicitly (edge-case tests); otherwise it is
    drawn first from the generator.  ``Lcap`` (the cache capacity) defaults
    to Lmax.
    """
    g = _gen(seed)
    if seqlens is None:
        seqlens = torch.randint(Lmin, Lmax + 1, (B,), generator=g, dtype=torch.int64)
    seqlens = torch.as_tensor(seqlens, dtype=torch.int64)
    Lcap = int(Lcap if Lcap is not None else max(Lmax, int(seqlens.max().item()) if B else 0))
    q = _randn_bf16(g, (B, H, d))
    hk = Hkv or H
    fill = float("nan") if poison else 0.0
    kc = torch.full((B, hk, Lcap, d), fill, dtype=torch.bfloat16)
    vc = torch.full((B, hk, Lcap, d), fill, dtype=torch.bfloat16)
    for b in range(B):
        L = int(seqlens[b])
        kc[b, :, :L] = _randn_bf16(g, (hk, L, d))
        vc[b, :, :L] = _randn_bf16(g, (hk, L, d))
    return q, kc, vc, seqlens.to(torch.int32)


def varlen_inputs(seqlens_q, seqlens_k, H: int, Hkv: int, d: int, seed: int,
                  std: float = 1.0, with_do: bool = False):
    """A ragged batch packed without padding, token-major: q [total_q, H, d],
    k, v [total_k, Hkv, d] (and dO like q when ``with_do``) as bf16 CPU
    tensors, plus cu_seqlens_q / cu_seqlens_k int32 [B + 1] (prefix sums of
    the lengths, starting at 0).  Draw order: q, k, v, dO, each over the
    packed rows."""
    g = _gen(seed)
    lq = [int(x) for x in seqlens_q]
    lk = [int(x) for x in seqlens_k]
    cu_q = torch.tensor([0] + list(np.cumsum(lq)), dtype=torch.int32)
    cu_k = torch.tensor([0] + list(np.cumsum(lk)), dtype=torch.int32)
    tq, tk = int(cu_q[-1]), int(cu_k[-1])
    out = [_randn_bf16(g, (tq, H, d), std), _randn_bf16(g, (tk, Hkv, d), std),
           _randn_bf16(g, (tk, Hkv, d), std)]
    if with_do:
        out.append(_randn_bf16(g, (tq, H, d), std))
    return (*out, cu_q, cu_k)


E4M3_MAX = 448.0


def fp8_inputs(B: int, H: int, Nq: int, d: int, seed: int, Hkv: int | None = None,
               Nk: int | None = None, std: float = 1.0):
    """e4m3 inputs for the FP8 forward: q [B, H, Nq, d], k [B, Hkv, Nk, d] and
    V transposed, vt [B, Hkv, d, Nk], as torch.float8_e4m3fn CPU tensors, with
    one descale factor per tensor (real value = stored value x factor).

    q, k, v ~ N(0,1) * std are drawn as float32 in that order; each tensor is
    divided by its factor amax / 448 and rounded to e4m3 (round to nearest
    even) -- data preparation, no attention arithmetic.  Returns
    (q8, k8, vt8, (q_scale, k_scale, v_scale))."""
    g = _gen(seed)
    hk = Hkv or H
    nk = Nq if Nk is None else Nk
    out, scales = [], []
    for shape in ((B, H, Nq, d), (B, hk, nk, d), (B, hk, nk, d)):
        x = torch.randn(shape, generator=g, dtype=torch.float32) * std
        amax = float(x.abs().max()) if x.numel() else 1.0
        sc = max(amax, 1e-30) / E4M3_MAX
        out.append((x / sc).to(torch.float8_e4m3fn))
        scales.append(sc)
    q8, k8, v8 = out
    return q8, k8, v8.transpose(-1, -2).contiguous(), tuple(scales)


def fp8_to_f64(t: torch.Tensor, scale: float) -> np.ndarray:
    """Exact real values of an e4m3 tensor: stored value x descale factor."""
    return t.to(torch.float64).numpy() * scale


def page_cache(kc: torch.Tensor, vc: torch.Tensor, seqlens, page_size: int, seed: int,
               spare_pages: int = 3):
    """Scatter contiguous caches [B, Hkv, Lcap, d] into page pools
    [num_pages, Hkv, page_size, d] in a seeded random page order.

    Returns (kpages, vpages, block_table int32 [B, pages_per_seq]).  Logical
    page p of sequence b goes to pool page block_table[b, p]; table entries
    past a sequence's last page are -1, and the ``spare_pages`` pool pages
    that no sequence uses, like the rows past a sequence's end, hold NaN.
    Pure data movement: no attention arithmetic."""
    B, hk, Lcap, d = kc.shape
    pps = -(-Lcap // page_size)
    seqlens = torch.as_tensor(seqlens, dtype=torch.int64)
    used = [int(-(-int(seqlens[b]) // page_size)) for b in range(B)]
    num_pages = sum(used) + spare_pages
    perm = torch.randperm(num_pages, generator=_gen(seed))
    kp = torch.full((num_pages, hk, page_size, d), float("nan"), dtype=kc.dtype)
    vp = torch.full((num_pages, hk, page_size, d), float("nan"), dtype=vc.dtype)
    table = torch.full((B, pps), -1, dtype=torch.int32)
    nxt = 0
    for b in range(B):
        for p in range(used[b]):
            page = int(perm[nxt])
            nxt += 1
            table[b, p] = page
            r0, r1 = p * page_size, min((p + 1) * page_size, Lcap)
            kp[page, :, :r1 - r0] = kc[b, :, r0:r1]
            vp[page, :, :r1 - r0] = vc[b, :, r0:r1]
    return kp, vp, table


def varlen_lengths(w: Workload) -> list:
    """Sequence lengths of a ragged-batch workload, drawn first from its seed."""
    g = _gen(w.seed)
    return torch.randint(w.Lmin, w.Lmax + 1, (w.B,), generator=g).tolist()


def workload_inputs(w: Workload):
    if w.kind == "fwd_fp8":
        return fp8_inputs(w.B, w.H, w.N, w.d, w.seed, Hkv=w.kv_heads, std=w.std)
    if w.kind == "fwd_varlen":
        lens = varlen_lengths(w)
        return varlen_inputs(lens, lens, w.H, w.kv_heads, w.d, w.seed + 1, w.std)
    if w.kind == "fwd":
        return fwd_inputs(w.B, w.H, w.N, w.d, w.seed, w.std, Hkv=w.kv_heads)
    if w.kind == "bwd":
        return bwd_inputs(w.B, w.H, w.N, w.d, w.seed, w.std, Hkv=w.kv_heads)
    return decode_inputs(w.B, w.H, w.d, w.Lmin, w.Lmax, w.seed, Hkv=w.kv_heads)


def sample_rows(N: int, n_random: int, seed: int, edge: int = 128) -> np.ndarray:
    """Sorted row indices: the first and last ``edge`` rows plus random ones."""
    rng = np.random.default_rng(seed)
    head = np.arange(min(edge, N))
    tail = np.arange(max(0, N - edge), N)
    mid = rng.integers(0, N, size=n_random) if N else np.zeros(0, np.int64)
    return np.unique(np.concatenate([head, tail, mid]))


def to_f64(t: torch.Tensor) -> np.ndarray:
    """Exact conversion of a (bf16 / fp32) tensor to a float64 numpy array."""
    return t.detach().to("cpu").to(torch.float64).numpy()
