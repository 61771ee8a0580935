"""The five benchmark workloads and their work/byte accounting.

Accounting conventions:

* Prefill work counts only visible (query, key) pairs, at 4*D floating-point
  operations per pair (2*D for the q.k dot product, 2*D for adding p*v):
      flops = 4 * D * sum over (b, h, i) of |visible keys of row i|.
  This is the attention-core term of the per-step FLOP table of "Taking LLMs
  apart (2): attention by hand" (section "KV cache", last-step FLOP table):
  its no-cache column is 6nD^2 + 4n^2 D + 2D^2 and its cache column is
  4nD + 8D^2 for D = 64, i.e. projections plus 4 * n_q * n_k * D.
* Paged decode bytes are the K and V bytes that must be read once per kv
  head: sum_b L_b * Hkv * D * 2 (K and V) * element size, plus q, out and
  the page-table entries touched.  The KV-cache byte column of the same page
  (65,536 B for n = 128 at D = 64 in fp32) and its 7B projection (512 KB per
  token for 32 layers x 32 heads x 128 in fp16) follow the same formula.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np


@dataclass(frozen=True)
class PrefillSpec:
    name: str
    B: int
    Hq: int
    Hkv: int
    Sq: int
    Skv: int
    D: int
    causal: bool
    window: int
    dtype: str            # "bf16" or "f32" (storage and I/O type)
    seed: int
    desc: str = ""

    @property
    def scale(self) -> float:
        return 1.0 / float(np.sqrt(self.D))


@dataclass(frozen=True)
class DecodeSpec:
    name: str
    N: int
    Hq: int
    Hkv: int
    D: int
    page_size: int
    len_range: tuple
    window: int
    seed: int
    desc: str = ""

    @property
    def scale(self) -> float:
        return 1.0 / float(np.sqrt(self.D))


@dataclass(frozen=True)
class PagedPrefillSpec:
    """Chunked prefill over a paged cache: B sequences of L cached tokens each, the last Sq of them new."""
    name: str
    B: int
    Hq: int
    Hkv: int
    L: int
    Sq: int
    D: int
    page_size: int
    seed: int
    desc: str = ""

    @property
    def scale(self) -> float:
        return 1.0 / float(np.sqrt(self.D))


WORKLOADS = {
    "single_head_f32": PrefillSpec(
        "single_head_f32", 1, 1, 1, 256, 256, 64, False, 0, "f32", 1000,
        "single-head non-causal attention, fp32, B=1 H=1 S=256 D=64"),
    "mha_causal_gpt2s": PrefillSpec(
        "mha_causal_gpt2s", 8, 12, 12, 1024, 1024, 64, True, 0, "bf16", 1001,
        "causal MHA prefill, GPT-2-small shape, B=8 H=12 S=1024 D=64, bf16"),
    "gqa_causal_4k": PrefillSpec(
        "gqa_causal_4k", 4, 32, 8, 4096, 4096, 128, True, 0, "bf16", 1002,
        "causal GQA prefill, B=4 Hq=32 Hkv=8 S=4096 D=128, bf16"),
    "gqa_swa_16k": PrefillSpec(
        "gqa_swa_16k", 1, 32, 8, 16384, 16384, 128, True, 4096, "bf16", 1003,
        "causal sliding-window GQA prefill, B=1 Hq=32 Hkv=8 S=16384 W=4096 D=128, bf16"),
    "paged_decode_gqa": DecodeSpec(
        "paged_decode_gqa", 64, 32, 8, 128, 16, (512, 8192), 0, 1004,
        "paged-KV GQA decode, 64 seqs x 1 token, Hq=32 Hkv=8 D=128, L~U[512,8192], page 16, bf16"),
}


def visible_per_row(Sq: int, Skv: int, causal: bool, window: int = 0) -> np.ndarray:
    """Number of visible keys of each query row (int64 [Sq]), closed form."""
    if not causal:
        return np.full(Sq, Skv, dtype=np.int64)
    i = np.arange(Sq, dtype=np.int64)
    last = np.minimum(i + (Skv - Sq), Skv - 1)
    first = np.zeros_like(i)
    if window and window > 0:
        first = np.maximum(0, i + (Skv - Sq) - window + 1)
    return np.maximum(0, last - first + 1)


def visible_pairs(Sq: int, Skv: int, causal: bool, window: int = 0) -> int:
    return int(visible_per_row(Sq, Skv, causal, window).sum())


def attention_flops(B: int, Hq: int, Sq: int, Skv: int, D: int, causal: bool, window: int = 0) -> int:
    """4 * D per visible (query, key) pair, over every batch and query head."""
    return 4 * D * B * Hq * visible_pairs(Sq, Skv, causal, window)


def prefill_flops(spec: PrefillSpec) -> int:
    return attention_flops(spec.B, spec.Hq, spec.Sq, spec.Skv, spec.D, spec.causal, spec.window)


def kv_bytes(seq_lens, Hkv: int, D: int, elem_bytes: int = 2, window: int = 0) -> int:
    """K plus V bytes one decode step must read: each visible token once per kv head."""
    L = np.asarray(seq_lens, dtype=np.int64)
    if window and window > 0:
        L = np.minimum(L, window)
    return int(L.sum()) * Hkv * D * 2 * elem_bytes


def decode_bytes(seq_lens, Hq: int, Hkv: int, D: int, page_size: int, elem_bytes: int = 2,
                 window: int = 0) -> int:
    """Algorithmic bytes of one paged decode step: K/V + q + out + page-table entries read."""
    L = np.asarray(seq_lens, dtype=np.int64)
    n = L.size
    Lw = np.minimum(L, window) if window and window > 0 else L
    pages = int(((Lw + page_size - 1) // page_size).sum())
    return kv_bytes(L, Hkv, D, elem_bytes, window) + 2 * n * Hq * D * elem_bytes + 4 * pages


# Measurement cases beyond the five above (their rows of the scope table are built on top of them).
EXTRA_WORKLOADS = {
    "chunked_prefill_paged_gqa": PagedPrefillSpec(
        "chunked_prefill_paged_gqa", 4, 32, 8, 4096, 1024, 128, 16, 1005,
        "chunked prefill over a paged cache: 4 sequences of 4096 cached tokens, the last 1024 new, "
        "Hq=32 Hkv=8 D=128, page 16, pages scattered over the pool, bf16"),
}


def paged_prefill_flops(spec: PagedPrefillSpec) -> int:
    """The Sq new rows attend causally (bottom-right) over the L cached keys."""
    return attention_flops(spec.B, spec.Hq, spec.Sq, spec.L, spec.D, True)
