"""attn_decode_paged_noalloc: the paged decode for callers that cannot allocate device memory.

Such callers (code behind an interface with no workspace argument, or a
serving loop whose device memory is planned once at start-up) get the
split-KV scratch from a fixed array inside the library instead of a
workspace they allocate.  The GPU test calls the entry point through the C
ABI twice in a row, on different inputs.  It runs the same kernels on the
same inputs as attn_decode_paged with a workspace, so each result must equal
that call's bit for bit (a second call overwriting part of the first one's
partials would show up here); each is also compared with the float64 oracle
at the bf16 tolerance of the other tests.  This file is named to be
collected last.
"""
import ctypes

import numpy as np
import pytest
import torch

from conftest import assert_parity
from oracle import sdpa
from scaled_dot_product_prefill_b200 import _lib, api, inputs


def test_sizes_over_the_scratch_limit_are_rejected_before_launch():
    lib = _lib.load()
    fake = ctypes.c_void_p(0x10000)
    # 4096 sequences x 64 heads x up to 16k keys needs far more than the 32 MiB scratch
    assert lib.attn_decode_paged_workspace_size(4096, 64, 128, 16384, 16) > 32 << 20
    st = lib.attn_decode_paged_noalloc(fake, fake, fake, fake, fake, 16, 4096, 64, 8, 128, 1 << 20, 1024, 16384,
                                       0.1, 0, fake, None)
    assert st == 6  # ATTN_ERR_WORKSPACE


@pytest.mark.gpu
def test_noalloc_decode_matches_workspace_decode_twice_in_a_row(cuda_device):
    cases = [
        dict(N=64, Hq=32, Hkv=8, D=128, page=16, seed=1004, len_range=(512, 8192)),   # the decode workload
        dict(N=5, Hq=16, Hkv=4, D=64, page=32, seed=77, len_range=(1, 3000)),
    ]
    devs, refs, hosts = [], [], []
    for c in cases:
        p = inputs.paged_inputs(c["N"], c["Hq"], c["Hkv"], c["D"], c["page"], c["seed"], len_range=c["len_range"],
                                spare_pages=2, poison=True)
        dev = [t.to(cuda_device) for t in (p.q, p.k_pool, p.v_pool, p.page_table, p.seq_lens)]
        devs.append((dev, p.max_seq_len))
        hosts.append(p)
        refs.append(api.attn_decode_paged(*dev, max_seq_len=p.max_seq_len))
    # two no-allocation calls back to back: the second reuses the scratch the first just wrote
    outs = [api.attn_decode_paged_noalloc(*dev, max_seq_len=msl) for dev, msl in devs]
    torch.cuda.synchronize()
    assert api.attn_device_status(clear=True) == 0
    for c, p, got, ref in zip(cases, hosts, outs, refs):
        assert torch.equal(got, ref), c
        want = sdpa.decode_paged(p.q, p.k_pool, p.v_pool, p.page_table, p.seq_lens, c["page"], 1 / np.sqrt(c["D"]))
        assert_parity(got, want, "bf16", f"noalloc {c}")
