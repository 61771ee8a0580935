"""The blocked, head-parallel evaluation of tests/oracle_blocks.py equals the oracle itself.

Runs on CPU.  Small shapes cover every mask mode, ragged row blocks,
Sq < Skv (a chunk at the end of a cache), Sq > Skv (leading rows with no
visible key), windows narrower and wider than a block, and GQA head maps;
one case goes through the spawned worker pool.
"""
import numpy as np
import pytest

import oracle_blocks
from oracle import sdpa
from scaled_dot_product_prefill_b200 import inputs

CASES = [
    # B, Hq, Hkv, Sq, Skv, D, causal, window, block
    (1, 2, 1, 70, 70, 16, True, 0, 16),
    (1, 2, 2, 70, 70, 16, True, 9, 16),       # window narrower than a block
    (1, 2, 2, 70, 70, 16, True, 40, 16),      # window wider than a block
    (2, 4, 2, 33, 90, 8, True, 0, 8),         # chunk at the end of a cache
    (1, 2, 2, 33, 90, 8, True, 20, 8),
    (1, 2, 1, 90, 33, 8, True, 0, 16),        # leading rows see no key
    (1, 2, 1, 90, 33, 8, True, 5, 16),
    (1, 3, 3, 50, 61, 8, False, 0, 16),
    (1, 2, 2, 64, 64, 8, True, 1, 7),         # window 1, blocks not dividing Sq
]


@pytest.mark.parametrize("case", CASES, ids=[str(c) for c in CASES])
def test_blocked_rows_equal_the_oracle(case):
    B, Hq, Hkv, Sq, Skv, D, causal, window, block = case
    inp = inputs.prefill_inputs(B, Hq, Hkv, Sq, Skv, D, seed=sum(case))
    scale = 1 / np.sqrt(D)
    want = sdpa.attention(inp.q, inp.k, inp.v, scale, causal, window)
    got = oracle_blocks.attention_all_rows(inp.q, inp.k, inp.v, scale, causal, window, block=block, procs=1)
    assert np.abs(got - want).max() <= 1e-12


def test_worker_pool_gives_the_same_rows():
    inp = inputs.prefill_inputs(2, 4, 2, 100, 100, 16, seed=3)
    want = sdpa.attention(inp.q, inp.k, inp.v, 0.25, True, 30)
    got = oracle_blocks.attention_all_rows(inp.q, inp.k, inp.v, 0.25, True, 30, block=32, procs=2)
    assert np.abs(got - want).max() <= 1e-12
