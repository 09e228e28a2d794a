"""Seeded synthetic inputs for the attention workloads.

This module only draws random numbers and lays them out; it holds none of the
attention arithmetic, so both the fp64 oracle (``oracle/``) and the CUDA path
(``exact_io_aware_75_b200``) can take their inputs from it without sharing any
of the method.

Recipe (same for every workload):
  * values are iid N(0, 1), drawn in fp32 by a ``torch.Generator('cpu')`` seeded
    with ``manual_seed(seed)`` and rounded to bf16 (round-to-nearest-even);
  * draw order: sequence lengths, then the page permutation, then Q, then K,
    then V;
  * large tensors are drawn in fixed chunks of ``CHUNK`` elements, so the values
    depend only on the seed and the shape;
  * the workloads follow the shapes the pages discuss: an 8B-class GQA layer
    (32 query heads, 8 KV heads, head dim 128; "What attention costs", "MQA and
    GQA"), long context with a 4,096-token sliding window ("Sliding windows and
    local:global layers"), packed documents, and a 16-token paged KV cache
    ("Paging and prefix sharing").
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

CHUNK = 1 << 26  # elements per randn call for large tensors

#: The workloads. ``scale`` is the softmax temperature 1/sqrt(d).
CONFIGS = {
    "tiny": dict(kind="dense", B=1, Hq=2, Hkv=2, N=128, d=64, causal=False,
                 window=0, o_dtype="fp32"),
    "gqa4k": dict(kind="dense", B=1, Hq=32, Hkv=8, N=4096, d=128, causal=True,
                  window=0, o_dtype="bf16"),
    "long32k": dict(kind="dense", B=1, Hq=32, Hkv=8, N=32768, d=128,
                    causal=True, window=0, o_dtype="bf16"),
    "long32k_w4096": dict(kind="dense", B=1, Hq=32, Hkv=8, N=32768, d=128,
                          causal=True, window=4096, o_dtype="bf16"),
    "varlen16": dict(kind="varlen", num_seqs=16, len_lo=256, len_hi=8192,
                     Hq=32, Hkv=8, d=128, causal=True, window=0,
                     o_dtype="bf16"),
    "decode64": dict(kind="decode", num_seqs=64, len_lo=4096, len_hi=32768,
                     Hq=32, Hkv=8, d=128, page_size=16),
}


def default_scale(d: int) -> float:
    return 1.0 / math.sqrt(d)


def randn_bf16(shape, gen: torch.Generator) -> torch.Tensor:
    """iid N(0,1) drawn in fp32 chunks, rounded to bf16 (CPU tensor)."""
    n = 1
    for s in shape:
        n *= int(s)
    out = torch.empty(n, dtype=torch.bfloat16)
    for lo in range(0, n, CHUNK):
        hi = min(n, lo + CHUNK)
        out[lo:hi] = torch.randn(hi - lo, generator=gen,
                                 dtype=torch.float32).to(torch.bfloat16)
    return out.view(*shape)


def draw_lengths(num: int, lo: int, hi: int, gen: torch.Generator) -> list[int]:
    """Integer lengths uniform on the inclusive range [lo, hi]."""
    return [int(x) for x in torch.randint(lo, hi + 1, (num,), generator=gen)]


@dataclass
class Dense:
    q: torch.Tensor  # [B, N, Hq, d] bf16
    k: torch.Tensor  # [B, N, Hkv, d] bf16
    v: torch.Tensor  # [B, N, Hkv, d] bf16
    causal: bool
    window: int
    scale: float


@dataclass
class Varlen:
    q: torch.Tensor  # [total, Hq, d] bf16
    k: torch.Tensor  # [total, Hkv, d] bf16
    v: torch.Tensor  # [total, Hkv, d] bf16
    lens: list
    cu_seqlens: torch.Tensor  # [num_seqs + 1] int32
    causal: bool
    window: int
    scale: float

    @property
    def max_seqlen(self) -> int:
        return max(self.lens) if self.lens else 0


@dataclass
class Paged:
    q: torch.Tensor            # [S, Hq, d] bf16
    k_cache: torch.Tensor      # [num_pages, page_size, Hkv, d] bf16
    v_cache: torch.Tensor      # [num_pages, page_size, Hkv, d] bf16
    block_table: torch.Tensor  # [S, max_pages] int32
    seq_lens: torch.Tensor     # [S] int32
    page_size: int
    scale: float
    pages_used: int = 0
    extra: dict = field(default_factory=dict)


def dense(B, Hq, Hkv, N, d, causal=False, window=0, seed=0, scale=None) -> Dense:
    g = torch.Generator("cpu").manual_seed(seed)
    q = randn_bf16((B, N, Hq, d), g)
    k = randn_bf16((B, N, Hkv, d), g)
    v = randn_bf16((B, N, Hkv, d), g)
    return Dense(q, k, v, bool(causal), int(window),
                 default_scale(d) if scale is None else float(scale))


def varlen(lens=None, num_seqs=16, len_lo=256, len_hi=8192, Hq=32, Hkv=8, d=128,
           causal=True, window=0, seed=0, scale=None) -> Varlen:
    g = torch.Generator("cpu").manual_seed(seed)
    if lens is None:
        lens = draw_lengths(num_seqs, len_lo, len_hi, g)
    lens = [int(x) for x in lens]
    total = sum(lens)
    cu = [0]
    for L in lens:
        cu.append(cu[-1] + L)
    q = randn_bf16((total, Hq, d), g)
    k = randn_bf16((total, Hkv, d), g)
    v = randn_bf16((total, Hkv, d), g)
    return Varlen(q, k, v, lens, torch.tensor(cu, dtype=torch.int32),
                  bool(causal), int(window),
                  default_scale(d) if scale is None else float(scale))


def paged(lens=None, num_seqs=64, len_lo=4096, len_hi=32768, Hq=32, Hkv=8,
          d=128, page_size=16, seed=0, scale=None, poison=False,
          spare_pages=0) -> Paged:
    """A paged KV cache whose pages are scattered by a random permutation.

    With ``poison`` the unused tail slots of each sequence's last page and the
    ``spare_pages`` pages that no sequence references are filled with NaN, so
    any read of them into a result shows up.
    """
    g = torch.Generator("cpu").manual_seed(seed)
    if lens is None:
        lens = draw_lengths(num_seqs, len_lo, len_hi, g)
    lens = [int(x) for x in lens]
    S = len(lens)
    npages = [(L + page_size - 1) // page_size for L in lens]
    used = sum(npages)
    perm = torch.randperm(used, generator=g)
    max_pages = max(max(npages) if npages else 1, 1)
    table = torch.zeros((S, max_pages), dtype=torch.int32)
    off = 0
    for s, n in enumerate(npages):
        table[s, :n] = perm[off:off + n].to(torch.int32)
        off += n
    q = randn_bf16((S, Hq, d), g)
    total_pages = used + int(spare_pages)
    kc = randn_bf16((total_pages, page_size, Hkv, d), g)
    vc = randn_bf16((total_pages, page_size, Hkv, d), g)
    if poison:
        nan = torch.tensor(float("nan"), dtype=torch.bfloat16)
        for s, L in enumerate(lens):
            tail = L % page_size
            if npages[s] and tail:
                p = int(table[s, npages[s] - 1])
                kc[p, tail:] = nan
                vc[p, tail:] = nan
        if spare_pages:
            kc[used:] = nan
            vc[used:] = nan
    return Paged(q, kc, vc, table, torch.tensor(lens, dtype=torch.int32),
                 page_size, default_scale(d) if scale is None else float(scale),
                 pages_used=used)


@dataclass
class PagedPrefill:
    q: torch.Tensor            # [total_q, Hq, d] bf16: each sequence's last L_q tokens
    k_cache: torch.Tensor      # [num_pages, page_size, Hkv, d] bf16
    v_cache: torch.Tensor
    block_table: torch.Tensor  # [S, max_pages] int32
    cu_seqlens_q: torch.Tensor  # [S + 1] int32
    seq_lens_k: torch.Tensor   # [S] int32
    lens_q: list
    scale: float

    @property
    def max_seqlen_q(self) -> int:
        return max(self.lens_q) if self.lens_q else 0


def paged_prefill(lens_k, lens_q, Hq=32, Hkv=8, d=128, seed=0, scale=None, poison=False,
                  spare_pages=0) -> PagedPrefill:
    """A chunked-prefill batch: the paged cache of ``paged(lens=lens_k)`` and,
    per sequence, L_q new query tokens (its last L_q positions), drawn from a
    generator of their own (seed + 2)."""
    base = paged(lens=lens_k, Hq=Hq, Hkv=Hkv, d=d, seed=seed, scale=scale, poison=poison,
                 spare_pages=spare_pages)
    lens_q = [int(x) for x in lens_q]
    g = torch.Generator("cpu").manual_seed(seed + 2)
    q = randn_bf16((sum(lens_q), Hq, d), g)
    cu = [0]
    for L in lens_q:
        cu.append(cu[-1] + L)
    return PagedPrefill(q, base.k_cache, base.v_cache, base.block_table,
                        torch.tensor(cu, dtype=torch.int32), base.seq_lens, lens_q, base.scale)


@dataclass
class PagedFP8:
    q: torch.Tensor            # [S, Hq, d] bf16
    k_codes: torch.Tensor      # [num_pages, page_size, Hkv, d] uint8 (FP8 E4M3 codes)
    v_codes: torch.Tensor
    k_scale: torch.Tensor      # [num_pages, Hkv] fp32
    v_scale: torch.Tensor
    block_table: torch.Tensor
    seq_lens: torch.Tensor
    page_size: int
    scale: float
    pages_used: int = 0


def _quantize_e4m3(x: torch.Tensor, pow2: bool):
    """Per-(page, KV head) scale = amax / 448 (rounded up to a power of two
    with ``pow2``), codes = the round-to-nearest-even E4M3 of x / scale
    (torch's float8_e4m3fn conversion).  NaN inputs stay NaN codes."""
    xf = x.float()
    amax = torch.nan_to_num(xf.abs(), nan=0.0).amax(dim=(1, 3))          # [P, Hkv]
    sc = torch.where(amax > 0, amax / 448.0, torch.ones_like(amax))
    if pow2:
        sc = torch.exp2(torch.ceil(torch.log2(sc)))
    codes = (xf / sc[:, None, :, None]).to(torch.float8_e4m3fn).view(torch.uint8)
    return codes, sc.to(torch.float32).contiguous()


def paged_fp8(pow2_scales=False, **kw) -> PagedFP8:
    """The paged workload of ``paged(**kw)`` with its cache stored as FP8
    E4M3 codes and one fp32 scale per (page, KV head): the same draws, then
    quantised (a storage format of the input, not attention arithmetic)."""
    b = paged(**kw)
    kc, ks = _quantize_e4m3(b.k_cache, pow2_scales)
    vc, vs = _quantize_e4m3(b.v_cache, pow2_scales)
    return PagedFP8(b.q, kc, vc, ks, vs, b.block_table, b.seq_lens, b.page_size, b.scale,
                    b.pages_used)


def make(name: str, seed: int = 0, **over):
    """Inputs of one named workload (CPU tensors)."""
    cfg = dict(CONFIGS[name])
    cfg.update(over)
    kind = cfg.pop("kind")
    cfg.pop("o_dtype", None)
    if kind == "dense":
        return dense(seed=seed, **cfg)
    if kind == "varlen":
        return varlen(seed=seed, **cfg)
    if kind == "decode":
        return paged(seed=seed, **cfg)
    raise ValueError(kind)


def grad_out(shape, seed=0) -> torch.Tensor:
    """The upstream gradient dO of a backward workload: iid N(0,1) in bf16
    from a generator of its own, seeded with ``seed + 1`` (so the forward
    inputs drawn with ``seed`` are unchanged)."""
    g = torch.Generator("cpu").manual_seed(seed + 1)
    return randn_bf16(tuple(shape), g)


def hadamard_signs(d: int, seed=0) -> torch.Tensor:
    """The random +-1 per channel of the FP8 prefill's rotation (fp32 [d]),
    from a generator of its own seeded with ``seed + 4``."""
    g = torch.Generator("cpu").manual_seed(seed + 4)
    return torch.where(torch.rand(d, generator=g) < 0.5, -1.0, 1.0).to(torch.float32)


def bf16_bits(t: torch.Tensor):
    """The raw bf16 bit patterns of a CPU bf16 tensor as a numpy uint16 array."""
    import numpy as np
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)
