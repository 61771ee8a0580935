"""GPU parity of the paged decode over an 8-bit (FP8 E4M3) cache against the float64 oracle."""
import numpy as np
import pytest
import torch

from conftest import assert_parity
from oracle import fp8, sdpa
from scaled_dot_product_prefill_b200 import api, inputs, workloads

pytestmark = pytest.mark.gpu


def oracle_fp8(p, k_scale, v_scale, scale, window):
    """Decode each code to the value it stands for, then the plain definition."""
    K = fp8.dequantize(p.k_pool, k_scale)
    V = fp8.dequantize(p.v_pool, v_scale)
    return sdpa.decode_paged(p.q, K, V, p.page_table, p.seq_lens, p.page_size, scale, window)


def run_fp8(p, k_scale, v_scale, window=0, scale=None):
    dev = [t.cuda() for t in (p.q, p.k_pool, p.v_pool, p.page_table, p.seq_lens)]
    out = api.attn_decode_paged_fp8(*dev, max_seq_len=max(p.max_seq_len, 1), k_scale=k_scale, v_scale=v_scale,
                                    scale=scale, window=window)
    torch.cuda.synchronize()
    return out


CASES = [
    # N, Hq, Hkv, D, page, seq_lens, window, k_scale, v_scale
    (4, 8, 2, 128, 16, [1, 16, 17, 300], 0, 1 / 64, 1 / 64),
    (3, 4, 4, 64, 16, [5, 513, 1000], 0, 0.02, 0.03),
    (2, 8, 1, 128, 32, [700, 33], 0, 1 / 32, 0.011),            # MQA, 32-token pages
    (3, 16, 2, 128, 64, [2000, 64, 65], 0, 0.015, 0.015),       # group of 8
    (3, 16, 2, 64, 16, [900, 1, 130], 0, 0.05, 0.01),           # group of 8 at D = 64
    (4, 8, 2, 128, 16, [300, 1200, 20, 4000], 100, 1 / 64, 0.02),   # sliding window
    (2, 8, 4, 64, 16, [1, 0], 0, 1.0, 1.0),                     # an empty cache gives zeros
]


@pytest.mark.parametrize("case", CASES, ids=[str(c[:6]) for c in CASES])
def test_fp8_decode_matches_oracle(case):
    N, Hq, Hkv, D, page, lens, window, ks, vs = case
    p = inputs.paged_inputs_fp8(N, Hq, Hkv, D, page, seed=len(lens) * 11 + D, k_scale=ks, v_scale=vs,
                                seq_lens=lens, spare_pages=3, poison=True)
    out = run_fp8(p, ks, vs, window)
    assert api.attn_device_status(clear=True) == 0
    ref = oracle_fp8(p, ks, vs, 1 / np.sqrt(D), window)
    assert_parity(out, ref, "bf16", str(case))


@pytest.mark.parametrize("Hq,Hkv,D", [(32, 8, 128), (16, 4, 64), (8, 4, 64), (16, 2, 128)],
                         ids=["G4-D128", "G4-D64", "G2-D64", "G8-D128"])
def test_fp8_decode_equals_bf16_decode_of_the_decoded_cache(Hq, Hkv, D):
    """With power-of-two scales every decoded element is exact in bf16 and every scaling is exact in fp32:
    the 8-bit path must then return the bf16 path's output bit for bit, and both match the oracle.  The
    cases cover both lane maps of the scores (two pieces per lane up to 4 heads per group, one for 8)
    and, at D = 64, the rows whose lanes read their second piece first."""
    ks, vs = 1 / 64, 1 / 128
    p = inputs.paged_inputs_fp8(6, Hq, Hkv, D, 16, seed=5, k_scale=ks, v_scale=vs,
                                seq_lens=[33, 1000, 17, 4097, 250, 64])
    K = torch.from_numpy(fp8.dequantize(p.k_pool, ks)).to(torch.bfloat16)
    V = torch.from_numpy(fp8.dequantize(p.v_pool, vs)).to(torch.bfloat16)
    assert torch.equal(K.double(), torch.from_numpy(fp8.dequantize(p.k_pool, ks)))   # exact in bf16
    out8 = run_fp8(p, ks, vs)
    dev = [t.cuda() for t in (p.q, K, V, p.page_table, p.seq_lens)]
    out16 = api.attn_decode_paged(*dev, max_seq_len=p.max_seq_len)
    torch.cuda.synchronize()
    assert api.attn_device_status(clear=True) == 0
    assert torch.equal(out8, out16)
    assert_parity(out8, oracle_fp8(p, ks, vs, 1 / np.sqrt(D), 0), "bf16", "8-bit cache")


def test_fp8_decode_workload_every_sequence():
    """The decode workload over an 8-bit cache, all 64 sequences x 32 heads x 128 outputs against the oracle."""
    spec = workloads.WORKLOADS["paged_decode_gqa"]
    ks, vs = 1 / 64, 1 / 64
    p = inputs.paged_inputs_fp8(spec.N, spec.Hq, spec.Hkv, spec.D, spec.page_size, spec.seed, k_scale=ks,
                                v_scale=vs, len_range=spec.len_range)
    out = run_fp8(p, ks, vs, spec.window, spec.scale).cpu()
    assert api.attn_device_status(clear=True) == 0
    ref = np.zeros(out.shape)
    for b in range(spec.N):
        L = int(p.seq_lens[b])
        K = fp8.dequantize(sdpa.gather_pages(p.k_pool.numpy(), p.page_table[b].numpy(), L, spec.page_size), ks)
        V = fp8.dequantize(sdpa.gather_pages(p.v_pool.numpy(), p.page_table[b].numpy(), L, spec.page_size), vs)
        ref[b] = sdpa.attention(p.q[b][None, :, None, :], K.transpose(1, 0, 2)[None], V.transpose(1, 0, 2)[None],
                                spec.scale, causal=True)[0, :, 0]
    assert_parity(out, ref, "bf16", f"{spec.name} (8-bit cache)", report=True)


def test_fp8_decode_rejects_bad_scales_and_dtypes():
    p = inputs.paged_inputs_fp8(2, 8, 2, 128, 16, seed=1, k_scale=1.0, v_scale=1.0, seq_lens=[20, 40])
    with pytest.raises(api.AttnError):
        run_fp8(p, 0.0, 1.0)
    with pytest.raises(api.AttnError):
        run_fp8(p, 1.0, float("inf"))
    with pytest.raises(ValueError):
        api.attn_decode_paged_fp8(p.q.cuda(), p.k_pool.cuda().view(torch.int8), p.v_pool.cuda(),
                                  p.page_table.cuda(), p.seq_lens.cuda(), max_seq_len=40, k_scale=1, v_scale=1)


def bits8(t):
    return t.cpu().numpy()


@pytest.mark.parametrize("ks,vs", [(0.05, 0.013), (1 / 64, 1 / 32)])
def test_fp8_append_matches_the_oracle_quantizer_bit_for_bit(ks, vs):
    B, Hkv, S_new, D, page = 3, 2, 40, 128, 16
    lens = [40, 100, 23]                       # sequence 2 is shorter than the chunk
    p = inputs.paged_inputs_fp8(B, 1, Hkv, D, page, seed=17, k_scale=1.0, v_scale=1.0, seq_lens=lens,
                                spare_pages=2, poison=True)
    k_new = (inputs.normal((B, Hkv, S_new, D), seed=3).float() * 4).to(torch.bfloat16)   # some saturate
    v_new = inputs.normal((B, Hkv, S_new, D), seed=4)
    kp, vp = p.k_pool.cuda(), p.v_pool.cuda()
    api.attn_device_status(clear=True)
    api.attn_kv_append_fp8(k_new.cuda(), v_new.cuda(), kp, vp, p.page_table.cuda(), p.seq_lens.cuda(),
                           k_scale=ks, v_scale=vs)
    torch.cuda.synchronize()
    assert api.attn_device_status(clear=True) == 0
    table, sl = p.page_table.numpy(), p.seq_lens.numpy()
    want_k = sdpa.append_pages(p.k_pool.numpy(), table, sl, fp8.quantize(k_new, ks), page)
    want_v = sdpa.append_pages(p.v_pool.numpy(), table, sl, fp8.quantize(v_new, vs), page)
    np.testing.assert_array_equal(bits8(kp), want_k)
    np.testing.assert_array_equal(bits8(vp), want_v)


def test_fp8_cache_filled_by_the_append_decodes_like_the_oracle():
    """Prefill-time append of whole caches into 8-bit pools, then a decode step against them."""
    N, Hq, Hkv, D, page, L = 4, 16, 4, 128, 16, 777
    ks, vs = 0.02, 0.02
    p = inputs.paged_inputs_fp8(N, Hq, Hkv, D, page, seed=23, k_scale=ks, v_scale=vs, seq_lens=[L] * N,
                                poison=True)
    k_new = inputs.normal((N, Hkv, L, D), seed=8)
    v_new = inputs.normal((N, Hkv, L, D), seed=9)
    kp = torch.full_like(p.k_pool, inputs.NAN_E4M3).cuda()
    vp = torch.full_like(p.v_pool, inputs.NAN_E4M3).cuda()
    pt, sl = p.page_table.cuda(), p.seq_lens.cuda()
    api.attn_kv_append_fp8(k_new.cuda(), v_new.cuda(), kp, vp, pt, sl, k_scale=ks, v_scale=vs)
    out = api.attn_decode_paged_fp8(p.q.cuda(), kp, vp, pt, sl, max_seq_len=L, k_scale=ks, v_scale=vs)
    torch.cuda.synchronize()
    assert api.attn_device_status(clear=True) == 0
    K = fp8.dequantize(fp8.quantize(k_new, ks), ks)          # [N, Hkv, L, D]
    V = fp8.dequantize(fp8.quantize(v_new, vs), vs)
    ref = sdpa.attention(p.q.double().numpy()[:, :, None, :], K, V, 1 / np.sqrt(D), causal=True)[:, :, 0]
    assert_parity(out, ref, "bf16", "fp8 cache from the append")


def test_fp8_long_context_decode():
    ks, vs = 0.02, 0.02
    p = inputs.paged_inputs_fp8(2, 8, 2, 128, 16, seed=78, k_scale=ks, v_scale=vs, seq_lens=[33333, 50000],
                                poison=True)
    out = run_fp8(p, ks, vs)
    assert api.attn_device_status(clear=True) == 0
    assert_parity(out, oracle_fp8(p, ks, vs, 1 / np.sqrt(128), 0), "bf16", "fp8 long context")
