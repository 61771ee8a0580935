"""Every output row of a large prefill from the float64 oracle, in reasonable time.

Test infrastructure only.  The oracle (``oracle.sdpa``) materialises one
score row per query over all keys; for 4k-16k-token sequences with 32-128
(batch, head) pairs that is minutes of work in one process.  This module
evaluates the same definition:

* head by head, in worker processes started with ``spawn`` (a pool forked
  after the GPU context exists can hang);
* within a head, block by block of query rows, each block over only the key
  range ``[k0, k1)`` that can be visible to any of its rows.

The second point changes nothing in the result.  Under the causal mask with
bottom-right alignment (offset ``off = Skv - Sq``), row ``i`` sees keys
``j <= i + off``, and with a window ``W`` also ``j > i + off - W``; so no row
of ``[r0, r1)`` sees a key at or past ``k1 = r1 + off`` or before
``k0 = r0 + off - W + 1``.  Those keys get weight exactly 0 in every row of
the block.  Both conditions depend on ``i - j`` only, so the block is the
oracle's own problem on the key slice with positions shifted by ``k0``:
``Sq' = r1 - r0`` queries, ``Skv' = k1 - k0`` keys, rows ``i - r0``; its
offset ``Skv' - Sq'`` equals ``off + r0 - k0``, which maps every (row, key)
pair to the same visibility.  ``tests/test_oracle_blocks.py`` checks this
against ``oracle.sdpa.attention`` on small cases in every mask mode.
"""
from __future__ import annotations

import concurrent.futures as cf
import multiprocessing as mp
import os

import numpy as np


def head_rows(q, k, v, scale, causal, window, block=512):
    """Every output row of one head: q [Sq, D], k/v [Skv, D] -> float64 [Sq, Dv]."""
    from oracle import sdpa

    q = np.asarray(q)
    k = np.asarray(k)
    v = np.asarray(v)
    Sq, Skv = q.shape[0], k.shape[0]
    off = Skv - Sq
    out = np.zeros((Sq, v.shape[1]), dtype=np.float64)
    for r0 in range(0, Sq, block):
        r1 = min(Sq, r0 + block)
        if causal:
            k1 = r1 + off
            k0 = max(0, r0 + off - window + 1) if window and window > 0 else 0
        else:
            k0, k1 = 0, Skv
        if k1 <= k0:
            continue   # no row of the block sees a key: its rows are 0
        n = r1 - r0
        out[r0:r1] = sdpa.attention_rows(q[r0:r1], k[k0:k1], v[k0:k1], np.arange(n), n, scale, causal, window)
    return out


def _task(args):
    idx, q, k, v, scale, causal, window, block = args
    return idx, head_rows(q, k, v, scale, causal, window, block)


def _f32(t):
    """bf16/fp32 torch tensor or array -> float32 numpy (exact for bf16 values)."""
    if hasattr(t, "detach"):
        import torch

        return t.detach().to("cpu", dtype=torch.float32).numpy()
    return np.asarray(t, dtype=np.float32)


def workers():
    try:
        n = len(os.sched_getaffinity(0))
    except AttributeError:
        n = os.cpu_count() or 1
    return max(1, n)


def attention_all_rows(q, k, v, scale, causal, window=0, block=512, procs=None):
    """oracle.sdpa.attention for [B, Hq, Sq, D] / [B, Hkv, Skv, D], head-parallel and blocked.

    Returns float64 [B, Hq, Sq, Dv].  ``procs`` worker processes (default:
    the CPUs this process may run on), each with one BLAS thread.
    """
    B, Hq, Sq, _ = q.shape
    Hkv = k.shape[1]
    G = Hq // Hkv
    qf, kf, vf = _f32(q), _f32(k), _f32(v)
    out = np.zeros((B, Hq, Sq, vf.shape[-1]), dtype=np.float64)
    tasks = [((b, h), qf[b, h], kf[b, h // G], vf[b, h // G], scale, causal, window, block)
             for b in range(B) for h in range(Hq)]
    procs = procs or workers()
    if procs == 1 or len(tasks) == 1:
        for t in tasks:
            (b, h), o = _task(t)
            out[b, h] = o
        return out
    saved = {name: os.environ.get(name) for name in ("OPENBLAS_NUM_THREADS", "OMP_NUM_THREADS", "MKL_NUM_THREADS")}
    for name in saved:
        os.environ[name] = "1"   # read by the spawned interpreters when they load numpy
    try:
        # a worker that dies makes the executor raise (BrokenProcessPool) instead of waiting for ever
        with cf.ProcessPoolExecutor(min(procs, len(tasks)), mp_context=mp.get_context("spawn")) as pool:
            for (b, h), o in pool.map(_task, tasks):
                out[b, h] = o
    finally:
        for name, val in saved.items():
            if val is None:
                os.environ.pop(name, None)
            else:
                os.environ[name] = val
    return out
