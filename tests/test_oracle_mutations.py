"""Plant plausible mistakes in the oracle (CPU only) and check that the pins catch each one.

Every mutation below replaces one piece of ``oracle.sdpa`` with a subtly
wrong version -- a dropped term, a wrong index, an off-by-one bound, a
transposed operand -- and asserts that at least one of the pin tests in
``test_oracle_pins`` fails while it is in place.
"""
import numpy as np
import pytest

import test_oracle_pins as pins
from oracle import fp8, sdpa

_orig_visible = sdpa.visible
_orig_softmax = sdpa.softmax_rows
_orig_weights = sdpa.weights
_orig_append = sdpa.append_pages


def _visible_window_off_by_one(Sq, Skv, causal, window=0, rows=None):
    vis = _orig_visible(Sq, Skv, causal, 0, rows)
    if causal and window > 0:
        i = (np.arange(Sq) if rows is None else np.asarray(rows))[:, None]
        vis &= np.arange(Skv)[None, :] >= i + (Skv - Sq) - window
    return vis


def _visible_top_left(Sq, Skv, causal, window=0, rows=None):
    return _orig_visible(Skv, Skv, causal, window, rows if rows is not None else np.arange(Sq))


def _softmax_no_max_subtraction(logits):
    e = np.exp(logits)
    s = e.sum(-1, keepdims=True)
    return e / s, np.log(s[..., 0])


def _softmax_unnormalised(logits):
    P, lse = _orig_softmax(logits)
    return P * 1.0001, lse


def _weights_mask_after_softmax(q, k, scale, causal, window=0, rows=None, Sq=None):
    q, k = sdpa._f64(q), sdpa._f64(k)
    Sq = q.shape[0] if Sq is None else Sq
    P, lse = _orig_softmax((q @ k.T) * scale)
    return np.where(sdpa.visible(Sq, k.shape[0], causal, window, rows), P, 0.0), lse


def _weights_scale_by_d(q, k, scale, causal, window=0, rows=None, Sq=None):
    return _orig_weights(q, k, scale * scale, causal, window, rows, Sq)


def _weights_keys_reversed(q, k, scale, causal, window=0, rows=None, Sq=None):
    P, lse = _orig_weights(q, k, scale, causal, window, rows, Sq)
    return P[:, ::-1], lse


def _append_one_slot_late(pool, page_table, seq_lens, new, page_size):
    return _orig_append(pool, page_table, [int(L) + 1 for L in seq_lens], new, page_size)


def _append_chunk_reversed(pool, page_table, seq_lens, new, page_size):
    return _orig_append(pool, page_table, seq_lens, np.asarray(new)[:, :, ::-1], page_size)


def _e4m3_bias_8(codes):
    return fp8.__dict__["_orig_e4m3"](codes) / 2.0


def _e4m3_subnormals_as_normals(codes):
    c = np.asarray(codes.numpy() if hasattr(codes, "numpy") else codes, dtype=np.uint8)
    v = fp8.__dict__["_orig_e4m3"](c)
    sub = ((c >> 3) & 0xF) == 0
    return np.where(sub, np.where(c & 0x80, -1.0, 1.0) * (1 + (c & 7) / 8.0) * 2.0 ** -7, v)


def _e4m3_ties_away(x):
    x = np.asarray(x, dtype=np.float64)
    got = fp8.__dict__["_orig_round"](x)
    up = fp8.__dict__["_orig_round"](np.nextafter(np.abs(x), np.inf)) & 0x7F
    v = fp8.e4m3_value(got & 0x7F)
    nxt = fp8.e4m3_value(np.minimum((got & 0x7F) + 1, 0x7E))
    tie = np.abs(np.abs(x) - (v + nxt) / 2) == 0
    return np.where(tie, up | (got & 0x80), got).astype(np.uint8)


fp8.__dict__.setdefault("_orig_e4m3", fp8.e4m3_value)
fp8.__dict__.setdefault("_orig_round", fp8.e4m3_round)

MUTATIONS = {
    "kv_head round robin": ("kv_head", lambda h, Hq, Hkv: h % Hkv),
    "window off by one": ("visible", _visible_window_off_by_one),
    "causal top-left alignment": ("visible", _visible_top_left),
    "no max subtraction": ("softmax_rows", _softmax_no_max_subtraction),
    "unnormalised softmax": ("softmax_rows", _softmax_unnormalised),
    "mask after softmax": ("weights", _weights_mask_after_softmax),
    "scale squared": ("weights", _weights_scale_by_d),
    "value rows reversed": ("weights", _weights_keys_reversed),
    "append one slot late": ("append_pages", _append_one_slot_late),
    "append chunk reversed": ("append_pages", _append_chunk_reversed),
    "e4m3 exponent bias 8": ("fp8.e4m3_value", _e4m3_bias_8),
    "e4m3 subnormals read as normals": ("fp8.e4m3_value", _e4m3_subnormals_as_normals),
    "e4m3 ties rounded away from zero": ("fp8.e4m3_round", _e4m3_ties_away),
}

PIN_TESTS = [getattr(pins, n) for n in dir(pins) if n.startswith("test_")]


def _run_pin(fn):
    import inspect

    params = inspect.signature(fn).parameters
    if not params:
        fn()
        return
    # parametrised brute-force pin: run it over its whole grid
    for shape in pins.TINY:
        for causal, window in [(False, 0), (True, 0), (True, 1), (True, 3)]:
            fn(shape, causal, window)


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_catch_planted_mistake(name, monkeypatch):
    attr, bad = MUTATIONS[name]
    if attr.startswith("fp8."):
        monkeypatch.setattr(fp8, attr[4:], bad)
    else:
        monkeypatch.setattr(sdpa, attr, bad)
    caught = []
    for fn in PIN_TESTS:
        if fn.__name__ in ("test_scale_table_statistics",):
            continue  # slow; the other pins suffice
        try:
            with np.errstate(all="ignore"):
                _run_pin(fn)
        except (AssertionError, FloatingPointError, IndexError, ValueError):
            caught.append(fn.__name__)
    assert caught, f"no pin caught the planted mistake '{name}'"
