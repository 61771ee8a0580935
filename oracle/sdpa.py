"""Plain float64 scaled-dot-product attention (the definition, materialised).

Test infrastructure only (see ``oracle/__init__.py``).

Readings taken where the pages are silent or disagree (each also listed in
the design notes):

* Visibility.  The causal mask is a lower-triangular boolean with True =
  visible ([ANAT] "full implementation", ``causal_mask``); masked logits are
  set to -inf *before* the softmax so their weight is exactly 0 ([AME] 2.2
  ``masked_fill(mask == 0, -inf)``; [ANAT] pitfalls 1 and 2).
* Causal alignment when Sq != Skv: bottom-right, offset = Skv - Sq, key j is
  visible to query i iff j <= i + offset.  The pages only show square masks
  and a decode query that "sees only the past" with no mask ([ANAT] "KV
  cache"); bottom-right is the one alignment that makes both agree.
* Sliding window of W: key j is visible iff i + off - W < j <= i + off,
  i.e. exactly W keys including the query's own position ([LCT] "Sliding
  Window Attention" gives O(n*w) and the 16k/4k example; [ANAT] "try it"
  keeps the last 256 keys as ``K[max(0, t-256):t]``, which is t's own key
  plus the 255 before it).
* A row with no visible key (possible only for Sq > Skv under a causal
  mask, or an empty cache) has output 0 and lse -inf.  The pages' stable
  softmax would return NaN there ([ANAT] pitfall 3 only covers rows with at
  least one finite logit).
* GQA head map: query head h reads kv head ``h // (Hq // Hkv)``, the order
  produced by ``repeat_interleave(n_rep, dim=1)`` ([AME] 5.2; [LCT] "GQA
  implementation logic", ``repeat_kv``).
* Default scale 1/sqrt(D) ([AME] 2.1; [ANAT] "sqrt(d)").
"""
from __future__ import annotations

import numpy as np

NEG_INF = -np.inf


def _f64(x) -> np.ndarray:
    """Upcast to float64 (exact for bf16/fp32 inputs); accepts numpy or torch CPU tensors."""
    if hasattr(x, "detach"):
        import torch  # only for the dtype conversion of the caller's tensor

        return x.detach().to("cpu", dtype=torch.float64).numpy()
    return np.asarray(x, dtype=np.float64)


def default_scale(D: int) -> float:
    """1/sqrt(d_k) ([AME] 2.1: the variance of q.k is d_k for unit-variance components)."""
    return 1.0 / np.sqrt(D)


def visible(Sq: int, Skv: int, causal: bool, window: int = 0, rows=None) -> np.ndarray:
    """Boolean [len(rows), Skv]: True where query row i may attend key j.

    ``rows`` selects query positions (default all Sq).  Non-causal: every key
    is visible.  Causal: j <= i + (Skv - Sq).  Window W > 0 additionally
    requires j > i + (Skv - Sq) - W.
    """
    i = np.arange(Sq) if rows is None else np.asarray(rows, dtype=np.int64)
    i = i[:, None]
    j = np.arange(Skv)[None, :]
    if not causal:
        return np.ones((i.shape[0], Skv), dtype=bool)
    off = Skv - Sq
    vis = j <= i + off
    if window and window > 0:
        vis &= j > i + off - window
    return vis


def softmax_rows(logits: np.ndarray):
    """Max-subtracted softmax along the last axis ([ANAT] "softmax").

    Returns (weights, lse).  Subtracting the row max leaves the result
    unchanged (softmax is shift invariant) and keeps exp() <= 1.  Rows whose
    logits are all -inf get weights 0 and lse -inf.
    """
    m = logits.max(axis=-1, keepdims=True)
    empty = ~np.isfinite(m)
    m_safe = np.where(empty, 0.0, m)
    e = np.exp(logits - m_safe)            # exp(-inf) == 0 exactly
    s = e.sum(axis=-1, keepdims=True)
    w = np.where(empty, 0.0, e / np.where(empty, 1.0, s))
    with np.errstate(divide="ignore"):
        lse = np.where(empty, NEG_INF, m_safe + np.log(np.where(empty, 1.0, s)))
    return w, lse[..., 0]


def weights(q, k, scale: float, causal: bool, window: int = 0, rows=None, Sq=None):
    """Attention weights softmax(q k^T * scale + mask) for one head.

    q: [n, D] (the query rows ``rows`` of a length-``Sq`` sequence, or all of
    them), k: [Skv, D].  Returns (P [n, Skv], lse [n]).
    """
    q = _f64(q)
    k = _f64(k)
    if Sq is None:
        Sq = q.shape[0]
    logits = (q @ k.T) * scale
    vis = visible(Sq, k.shape[0], causal, window, rows)
    logits = np.where(vis, logits, NEG_INF)
    return softmax_rows(logits)


def kv_head(h: int, Hq: int, Hkv: int) -> int:
    """kv head serving query head h: contiguous groups of Hq // Hkv ([AME] 5.2)."""
    return h // (Hq // Hkv)


def attention(q, k, v, scale=None, causal=False, window=0, return_lse=False):
    """O = softmax(Q K^T * scale + mask) V for every batch and query head.

    q: [B, Hq, Sq, D]; k, v: [B, Hkv, Skv, D]; returns float64 [B, Hq, Sq, D]
    (and lse [B, Hq, Sq] with ``return_lse``).  Each (b, h) materialises
    the full Sq x Skv score matrix ([AME] 2.2; [ANAT] "full implementation").
    """
    q = _f64(q)
    k = _f64(k)
    v = _f64(v)
    B, Hq, Sq, D = q.shape
    Hkv, Skv = k.shape[1], k.shape[2]
    if Hq % Hkv:
        raise ValueError("Hq must be a multiple of Hkv")
    if scale is None:
        scale = default_scale(D)
    out = np.zeros((B, Hq, Sq, v.shape[-1]), dtype=np.float64)
    lse = np.zeros((B, Hq, Sq), dtype=np.float64)
    for b in range(B):
        for h in range(Hq):
            g = kv_head(h, Hq, Hkv)
            P, l = weights(q[b, h], k[b, g], scale, causal, window)
            out[b, h] = P @ v[b, g]
            lse[b, h] = l
    return (out, lse) if return_lse else out


def attention_rows(q_rows, k, v, rows, Sq: int, scale: float, causal: bool, window: int = 0):
    """Selected output rows of one head: the definition evaluated at query positions ``rows``.

    q_rows: [n, D] (the queries at those positions); k, v: [Skv, D].
    Used to check full-size launches on sampled outputs.
    """
    P, _ = weights(q_rows, k, scale, causal, window, rows=rows, Sq=Sq)
    return P @ _f64(v)


def gather_pages(pool, page_table_row, seq_len: int, page_size: int) -> np.ndarray:
    """Contiguous [L, Hkv, D] cache of one sequence from a paged pool.

    pool: [num_pages, Hkv, page_size, D]; token t is slot t % page_size of
    physical page page_table_row[t // page_size] ([AFS] "Paged KV Cache":
    fixed-size pages, a per-sequence page table over a shared pool; [LCT]
    "PagedAttention": the same cache stored non-contiguously).
    """
    pool = _f64(pool)
    pt = np.asarray(page_table_row, dtype=np.int64)
    Hkv, D = pool.shape[1], pool.shape[3]
    out = np.zeros((seq_len, Hkv, D), dtype=np.float64)
    for t in range(seq_len):
        phys = pt[t // page_size]
        if phys < 0 or phys >= pool.shape[0]:
            raise IndexError(f"page table entry {phys} for token {t} is outside the pool")
        out[t] = pool[phys, :, t % page_size, :]
    return out


def append_pages(pool, page_table, seq_lens, new, page_size: int) -> np.ndarray:
    """The paged cache after writing S_new new tokens of every sequence into it.

    pool: [num_pages, Hkv, page_size, D]; new: [B, Hkv, S_new, D];
    page_table [B, max_pages]; seq_lens [B] are the lengths AFTER the append.
    Token i of sequence b is the cache's position p = seq_lens[b] - S_new + i
    and goes to slot p % page_size of page page_table[b][p // page_size]
    ([ANAT] "KV cache": the new token's k and v are stored before the step's
    attention; [AFS] "Paged KV Cache": that store goes through the page table
    into the shared pool).  Positions below 0 (a cache shorter than the chunk)
    have no slot and are skipped.  Returns a new array in the pool's dtype;
    every other slot keeps its value.
    """
    out = np.array(pool, copy=True)
    new = np.asarray(new)
    pt = np.asarray(page_table, dtype=np.int64)
    B, Hkv, S_new, D = new.shape
    for b in range(B):
        L = int(seq_lens[b])
        for i in range(S_new):
            p = L - S_new + i
            if p < 0:
                continue
            phys = pt[b, p // page_size]
            if phys < 0 or phys >= out.shape[0]:
                raise IndexError(f"page table entry {phys} for position {p} is outside the pool")
            out[phys, :, p % page_size, :] = new[b, :, i, :]
    return out


def decode_paged(q, k_pool, v_pool, page_table, seq_lens, page_size: int, scale=None, window: int = 0):
    """One decode step per sequence over a paged KV cache.

    q: [N, Hq, D]; pools [num_pages, Hkv, page_size, D]; page_table [N, max_pages];
    seq_lens [N].  ``seq_lens[b]`` counts the new token itself: the cache is
    appended before the scores are taken ([ANAT] "KV cache": ``K[t-1] = ...``
    then ``s = K[:t] @ q / sqrt(D)``), so the query at position L-1 attends to
    all L cached keys (or the last ``window`` of them), with no further mask.
    Returns float64 [N, Hq, D].
    """
    q = _f64(q)
    N, Hq, D = q.shape
    Hkv = int(np.asarray(k_pool.shape)[1])
    if scale is None:
        scale = default_scale(D)
    seq_lens = np.asarray(seq_lens, dtype=np.int64).reshape(-1)
    page_table = np.asarray(page_table, dtype=np.int64)
    out = np.zeros((N, Hq, D), dtype=np.float64)
    for b in range(N):
        L = int(seq_lens[b])
        if L <= 0:
            continue
        K = gather_pages(k_pool, page_table[b], L, page_size)
        V = gather_pages(v_pool, page_table[b], L, page_size)
        for h in range(Hq):
            g = kv_head(h, Hq, Hkv)
            out[b, h] = attention_rows(q[b, h][None, :], K[:, g], V[:, g], [L - 1], L,
                                       scale, True, window)[0]
    return out
