"""Pure-Python brute-force attention for tiny shapes.

Test infrastructure only (see ``oracle/__init__.py``).  A second, independent
statement of the definition: nested loops over nested lists, ``math.exp``,
no numpy, and the visibility rule written as explicit comparisons rather
than the array predicate of ``oracle.sdpa``.  It exists to check that
module on shapes up to a few dozen rows.

For each batch b, query head h (kv head g = floor(h * Hkv / Hq)) and query
row i:
    s_j  = scale * sum_d q[b][h][i][d] * k[b][g][j][d]     for visible j
    p_j  = exp(s_j - max_j s_j) / sum_j exp(s_j - max_j s_j)
    o[d] = sum_j p_j * v[b][g][j][d]
([AME] 2.1-2.2; [ANAT] "softmax" and "full implementation").  A row with no
visible key returns zeros.
"""
from __future__ import annotations

import math


def _to_list(x):
    if hasattr(x, "detach"):
        import torch

        return x.detach().to("cpu", dtype=torch.float64).tolist()
    if hasattr(x, "tolist"):
        return x.astype("float64").tolist()
    return x


def _is_visible(i, j, Sq, Skv, causal, window):
    if not causal:
        return True
    last = i + Skv - Sq            # newest key this query may see
    if j > last:
        return False
    if window > 0 and j <= last - window:
        return False
    return True


def attention(q, k, v, scale, causal=False, window=0):
    """Nested-list attention; q [B][Hq][Sq][D], k/v [B][Hkv][Skv][D]."""
    q, k, v = _to_list(q), _to_list(k), _to_list(v)
    B, Hq, Sq, D = len(q), len(q[0]), len(q[0][0]), len(q[0][0][0])
    Hkv, Skv, Dv = len(k[0]), len(k[0][0]), len(v[0][0][0])
    out = []
    for b in range(B):
        ob = []
        for h in range(Hq):
            g = (h * Hkv) // Hq
            oh = []
            for i in range(Sq):
                scores = []
                for j in range(Skv):
                    if _is_visible(i, j, Sq, Skv, causal, window):
                        dot = 0.0
                        for d in range(D):
                            dot += q[b][h][i][d] * k[b][g][j][d]
                        scores.append((j, dot * scale))
                row = [0.0] * Dv
                if scores:
                    mx = max(s for _, s in scores)
                    ex = [(j, math.exp(s - mx)) for j, s in scores]
                    tot = sum(e for _, e in ex)
                    for j, e in ex:
                        p = e / tot
                        for d in range(Dv):
                            row[d] += p * v[b][g][j][d]
                oh.append(row)
            ob.append(oh)
        out.append(ob)
    return out


def decode_paged(q, k_pool, v_pool, page_table, seq_lens, page_size, scale, window=0):
    """Nested-list paged decode: q [N][Hq][D], pools [P][Hkv][page_size][D]."""
    q, kp, vp = _to_list(q), _to_list(k_pool), _to_list(v_pool)
    pt = page_table.tolist() if hasattr(page_table, "tolist") else page_table
    sl = seq_lens.tolist() if hasattr(seq_lens, "tolist") else seq_lens
    N, Hq, D = len(q), len(q[0]), len(q[0][0])
    Hkv = len(kp[0])
    out = []
    for b in range(N):
        L = int(sl[b])
        ob = []
        for h in range(Hq):
            g = (h * Hkv) // Hq
            first = 0 if window <= 0 else max(0, L - window)
            scores = []
            for t in range(first, L):
                page = pt[b][t // page_size]
                slot = t % page_size
                dot = 0.0
                for d in range(D):
                    dot += q[b][h][d] * kp[page][g][slot][d]
                scores.append((page, slot, dot * scale))
            row = [0.0] * D
            if scores:
                mx = max(s for _, _, s in scores)
                ex = [(p, s_, math.exp(s - mx)) for p, s_, s in scores]
                tot = sum(e for _, _, e in ex)
                for page, slot, e in ex:
                    for d in range(D):
                        row[d] += (e / tot) * vp[page][g][slot][d]
            ob.append(row)
        out.append(ob)
    return out
