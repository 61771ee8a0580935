"""Seeded synthetic inputs for the attention workloads.

This module draws random numbers and lays them out; it holds none of the
attention arithmetic, so both the float64 oracle (under ``oracle/``) and the
CUDA path can be fed from it without sharing any method code.

Every tensor is drawn on the CPU as float32 N(0, 1) from a
``torch.Generator`` seeded per tensor, then rounded to the storage dtype
(round-to-nearest-even for bf16).  The oracle consumes exactly those rounded
values, upcast to float64.

Layouts (all contiguous, row-major):

* prefill: ``q`` is ``[B, Hq, Sq, D]``, ``k`` and ``v`` are ``[B, Hkv, Skv, D]``
  (the ``(batch, n_heads, seq_len, d)`` order of the Attention-mechanism
  explainer, "Scaled Dot-Product Attention" section 2.2).
* paged decode: ``q`` is ``[N, Hq, D]``; ``k_pool`` and ``v_pool`` are
  ``[num_pages, Hkv, page_size, D]``; ``page_table`` is ``[N, max_pages]``
  int32 padded with -1; ``seq_lens`` is ``[N]`` int32.  Token ``t`` of
  sequence ``b`` lives in physical page ``page_table[b, t // page_size]`` at
  slot ``t % page_size`` (the page table of the "Paged KV Cache" item of the
  Attention-From-Scratch project README, with its default page size 16).
"""
from __future__ import annotations

from dataclasses import dataclass

import torch

_DTYPES = {"bf16": torch.bfloat16, "f32": torch.float32}


def _gen(seed: int) -> torch.Generator:
    return torch.Generator("cpu").manual_seed(int(seed))


def normal(shape, seed: int, dtype: str = "bf16") -> torch.Tensor:
    """N(0, 1) float32 draws from ``seed``, rounded to ``dtype`` ("bf16" or "f32")."""
    x = torch.randn(tuple(shape), generator=_gen(seed), dtype=torch.float32)
    return x.to(_DTYPES[dtype]).contiguous()


@dataclass
class PrefillInputs:
    q: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    seed: int


def prefill_inputs(B, Hq, Hkv, Sq, Skv, D, seed: int, dtype: str = "bf16") -> PrefillInputs:
    """Q ``[B,Hq,Sq,D]``, K/V ``[B,Hkv,Skv,D]``, each an independent seeded stream."""
    base = int(seed) * 16
    q = normal((B, Hq, Sq, D), base + 0, dtype)
    k = normal((B, Hkv, Skv, D), base + 1, dtype)
    v = normal((B, Hkv, Skv, D), base + 2, dtype)
    return PrefillInputs(q, k, v, seed)


@dataclass
class PagedInputs:
    q: torch.Tensor            # [N, Hq, D]
    k_pool: torch.Tensor       # [num_pages, Hkv, page_size, D]
    v_pool: torch.Tensor       # [num_pages, Hkv, page_size, D]
    page_table: torch.Tensor   # [N, max_pages] int32, -1 padded
    seq_lens: torch.Tensor     # [N] int32
    page_size: int
    used_pages: int            # pages referenced by some sequence
    seed: int

    @property
    def num_pages(self) -> int:
        return int(self.k_pool.shape[0])

    @property
    def max_pages(self) -> int:
        return int(self.page_table.shape[1])

    @property
    def max_seq_len(self) -> int:
        return int(self.seq_lens.max().item()) if self.seq_lens.numel() else 0


def draw_seq_lens(N: int, seed: int, len_range=(512, 8192)) -> torch.Tensor:
    """The sequence lengths ``paged_inputs`` draws for ``seed``: integers uniform in ``len_range`` (inclusive)."""
    lo, hi = len_range
    return torch.randint(int(lo), int(hi) + 1, (N,), generator=_gen(int(seed) * 16 + 3), dtype=torch.int64)


def paged_inputs(N, Hq, Hkv, D, page_size: int, seed: int, *, seq_lens=None,
                 len_range=(512, 8192), spare_pages: int = 0, poison: bool = False,
                 max_pages: int | None = None, dtype: str = "bf16") -> PagedInputs:
    """A shared page pool with per-sequence page tables.

    ``seq_lens`` defaults to integers drawn uniformly from ``len_range``
    (inclusive).  Each sequence owns ``ceil(L / page_size)`` pages; all pages
    (plus ``spare_pages`` unreferenced ones) are scattered over the pool by
    a seeded random permutation.  With ``poison`` the unreferenced pages and
    the slots past each sequence's last token are filled with NaN, so that a
    kernel that lets them reach an output shows up as NaN there.
    """
    base = int(seed) * 16
    if seq_lens is None:
        seq_lens = draw_seq_lens(N, seed, len_range)
    seq_lens = torch.as_tensor(seq_lens, dtype=torch.int64).reshape(-1)
    assert seq_lens.numel() == N
    n_pages_seq = [(int(L) + page_size - 1) // page_size for L in seq_lens.tolist()]
    used = sum(n_pages_seq)
    total = used + int(spare_pages)
    mp = max(n_pages_seq) if N and max(n_pages_seq) > 0 else 1
    if max_pages is not None:
        assert max_pages >= mp
        mp = int(max_pages)
    perm = torch.randperm(total, generator=_gen(base + 4)) if total else torch.zeros(0, dtype=torch.int64)
    table = torch.full((N, mp), -1, dtype=torch.int32)
    off = 0
    for b, npg in enumerate(n_pages_seq):
        table[b, :npg] = perm[off:off + npg].to(torch.int32)
        off += npg
    q = normal((N, Hq, D), base + 0, dtype)
    k_pool = normal((total, Hkv, page_size, D), base + 1, dtype)
    v_pool = normal((total, Hkv, page_size, D), base + 2, dtype)
    if poison and total:
        nan = float("nan")
        valid = torch.zeros(total, page_size, dtype=torch.bool)
        for b, npg in enumerate(n_pages_seq):
            L = int(seq_lens[b])
            for p in range(npg):
                phys = int(table[b, p])
                n_tok = min(page_size, L - p * page_size)
                valid[phys, :n_tok] = True
        bad = ~valid  # [total, page_size]
        k_pool = k_pool.masked_fill(bad[:, None, :, None].expand(total, Hkv, page_size, D), nan)
        v_pool = v_pool.masked_fill(bad[:, None, :, None].expand(total, Hkv, page_size, D), nan)
    return PagedInputs(q, k_pool.contiguous(), v_pool.contiguous(), table,
                       seq_lens.to(torch.int32), page_size, used, seed)


def e4m3_codes(shape, seed: int, scale: float) -> torch.Tensor:
    """N(0, 1) float32 draws from ``seed``, divided by ``scale`` and rounded to FP8 E4M3 codes (uint8).

    The rounding is torch's float8_e4m3fn conversion, saturated at +-448; a
    code stands for ``scale * value(code)``.
    """
    x = torch.randn(tuple(shape), generator=_gen(seed), dtype=torch.float32) / float(scale)
    return x.clamp(-448.0, 448.0).to(torch.float8_e4m3fn).view(torch.uint8).contiguous()


NAN_E4M3 = 0x7F


def paged_inputs_fp8(N, Hq, Hkv, D, page_size: int, seed: int, *, k_scale: float, v_scale: float, **kw):
    """``paged_inputs`` with the pools replaced by E4M3 codes (``k_scale``, ``v_scale`` per pool).

    The page tables, lengths and bf16 queries are those of ``paged_inputs``
    with the same arguments; with ``poison`` every slot that must never be
    read holds the NaN code 0x7F.
    """
    p = paged_inputs(N, Hq, Hkv, D, page_size, seed, **kw)
    base = int(seed) * 16
    k = e4m3_codes(p.k_pool.shape, base + 5, k_scale)
    v = e4m3_codes(p.v_pool.shape, base + 6, v_scale)
    bad = torch.isnan(p.k_pool.float())
    k = torch.where(bad, torch.full_like(k, NAN_E4M3), k)
    v = torch.where(bad, torch.full_like(v, NAN_E4M3), v)
    return PagedInputs(p.q, k, v, p.page_table, p.seq_lens, page_size, p.used_pages, seed)
