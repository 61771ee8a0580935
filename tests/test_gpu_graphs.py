"""The entry points inside CUDA graphs: a serving loop captures its decode step once and replays it.

Each call is captured after a warm-up call (which sets the kernels up on the device), then the
graph is replayed with new values in the same buffers; every replay must equal an eager call
and the oracle.
"""
import numpy as np
import pytest
import torch

from conftest import assert_parity
from oracle import sdpa
from scaled_dot_product_prefill_b200 import api, inputs

pytestmark = pytest.mark.gpu


def capture(fn):
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        fn()                                   # warm-up outside the graph
    torch.cuda.current_stream().wait_stream(s)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    return g


def test_decode_step_with_append_replays_from_a_graph():
    N, Hq, Hkv, D, page = 4, 16, 4, 128, 16
    p = inputs.paged_inputs(N, Hq, Hkv, D, page, seed=12, seq_lens=[300, 1000, 17, 2500], max_pages=200)
    q = p.q.cuda()
    kp, vp, pt = p.k_pool.cuda(), p.v_pool.cuda(), p.page_table.cuda()
    # every sequence has room for 8 more tokens in its pages (page tables padded with spare pages)
    lens0 = p.seq_lens.clone()
    spare = torch.arange(p.num_pages, p.num_pages + 4 * N, dtype=torch.int32)
    kp = torch.cat([kp, torch.zeros((4 * N, Hkv, page, D), dtype=torch.bfloat16, device="cuda")])
    vp = torch.cat([vp, torch.zeros_like(kp[:4 * N])])
    table = p.page_table.clone()
    for b in range(N):
        used = (int(lens0[b]) + page - 1) // page
        table[b, used:used + 4] = spare[4 * b:4 * b + 4]
    pt = table.cuda()
    sl = lens0.cuda()
    k_new = torch.zeros((N, Hkv, 1, D), dtype=torch.bfloat16, device="cuda")
    v_new = torch.zeros_like(k_new)
    out = torch.empty_like(q)
    ws = torch.empty(api.attn_decode_paged_workspace_size(N, Hq, D, 4096, page), dtype=torch.uint8, device="cuda")

    def step():
        api.attn_kv_append(k_new, v_new, kp, vp, pt, sl)
        api.attn_decode_paged(q, kp, vp, pt, sl, max_seq_len=4096, workspace=ws, out=out)

    sl += 1                                    # the warm-up step appends at the first new position
    g = capture(step)
    K_hist = [sdpa.gather_pages(p.k_pool, table[b].numpy(), int(lens0[b]), page) for b in range(N)]
    V_hist = [sdpa.gather_pages(p.v_pool, table[b].numpy(), int(lens0[b]), page) for b in range(N)]
    for t in range(3):                          # three decode steps replayed from the graph
        kn = inputs.normal((N, Hkv, 1, D), seed=100 + t)
        vn = inputs.normal((N, Hkv, 1, D), seed=200 + t)
        qn = inputs.normal((N, Hq, D), seed=300 + t)
        k_new.copy_(kn)
        v_new.copy_(vn)
        q.copy_(qn)
        sl.copy_((lens0 + 1 + t).cuda())
        g.replay()
        torch.cuda.synchronize()
        assert api.attn_device_status(clear=True) == 0
        for b in range(N):
            K_hist[b] = np.concatenate([K_hist[b][: int(lens0[b]) + t], kn[b].double().numpy().transpose(1, 0, 2)])
            V_hist[b] = np.concatenate([V_hist[b][: int(lens0[b]) + t], vn[b].double().numpy().transpose(1, 0, 2)])
            ref = sdpa.attention(qn[b][None, :, None, :], K_hist[b].transpose(1, 0, 2)[None],
                                 V_hist[b].transpose(1, 0, 2)[None], 1 / np.sqrt(D), causal=True)[0, :, 0]
            assert_parity(out[b], ref, "bf16", f"graph step {t} seq {b}")
        # the eager call on the same state gives the same bits
        eager = api.attn_decode_paged(q, kp, vp, pt, sl, max_seq_len=4096)
        torch.cuda.synchronize()
        assert torch.equal(eager, out)
    del g


def test_paged_prefill_and_fp8_decode_replay_from_graphs():
    p = inputs.paged_inputs(2, 8, 2, 64, 16, seed=21, seq_lens=[300, 700])
    q = inputs.normal((2, 8, 128, 64), seed=22).cuda()
    dev = [t.cuda() for t in (p.k_pool, p.v_pool, p.page_table, p.seq_lens)]
    out = torch.empty_like(q)
    g = capture(lambda: api.attn_prefill_paged(q, *dev, max_seq_len=700, causal=True, out=out))
    for t in range(2):
        qn = inputs.normal((2, 8, 128, 64), seed=30 + t)
        q.copy_(qn)
        g.replay()
        torch.cuda.synchronize()
        eager = api.attn_prefill_paged(q, *dev, max_seq_len=700, causal=True)
        torch.cuda.synchronize()
        assert torch.equal(eager, out)
    del g
    ks = vs = 0.02
    p8 = inputs.paged_inputs_fp8(3, 8, 2, 128, 16, seed=23, k_scale=ks, v_scale=vs, seq_lens=[50, 900, 4000])
    q8 = p8.q.cuda()
    dev8 = [t.cuda() for t in (p8.k_pool, p8.v_pool, p8.page_table, p8.seq_lens)]
    out8 = torch.empty_like(q8)
    ws = torch.empty(api.attn_decode_paged_workspace_size(3, 8, 128, 4000, 16), dtype=torch.uint8, device="cuda")
    g8 = capture(lambda: api.attn_decode_paged_fp8(q8, *dev8, max_seq_len=4000, k_scale=ks, v_scale=vs,
                                                   workspace=ws, out=out8))
    g8.replay()
    torch.cuda.synchronize()
    assert api.attn_device_status(clear=True) == 0
    eager = api.attn_decode_paged_fp8(q8, *dev8, max_seq_len=4000, k_scale=ks, v_scale=vs)
    torch.cuda.synchronize()
    assert torch.equal(eager, out8)
    del g8
