"""Benchmark of the attention hot path on B200: prefill TFLOP/s and paged-decode KV GB/s.

One step = one pass of the whole path over one batch of synthetic input:
  1. attn_prefill on the causal sliding-window GQA prefill, the largest
     prefill workload (B=1, Hq=32, Hkv=8, S=16384, W=4096, D=128, bf16;
     962 GFLOP; 335 MB of q, k, v and out, and a 256 MiB write before it
     flushes L2), and
  2. attn_decode_paged on the paged GQA decode batch (64 sequences, Hq=32,
     Hkv=8, D=128, L ~ U[512, 8192], 16-token pages; 1.1 GB of K/V, larger
     than L2).
`value` is the prefill throughput in TFLOP/s (4*D flops per visible
(query, key) pair); the decode throughput (algorithmic K/V bytes per
second) is reported beside it with its own roofline.  Each kernel is timed
with CUDA events on the stream it is launched on.  The other prefill
workloads are timed after the steps, each with its own roofline entry.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
Under torchrun each rank runs the same per-GPU workload (weak scaling, no
collective on the data path); the time is the max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from scaled_dot_product_prefill_b200 import inputs, workloads  # noqa: E402

PREFILL = workloads.WORKLOADS["gqa_swa_16k"]
DECODE = workloads.WORKLOADS["paged_decode_gqa"]
METRIC = "prefill TFLOP/s & paged-decode KV GB/s on 1 B200, % of roofline"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


def tensor_peak(peaks, clocks):
    """(peak TFLOP/s, kind) for the prefill roofline.

    The burst GEMM figure is the peak of a kernel timed in a short run; when the
    power cap held the SM clock below 97 % of its maximum during the timed steps
    (a long run), the figure measured the same way, seconds under the cap, is
    the comparable one.
    """
    burst = float(peaks["bf16_tflops"])
    sustained = float(peaks.get("bf16_tflops_sustained", burst))
    capped = bool("sw_power_cap" in clocks.get("reasons", []) and clocks.get("sm_mhz") and clocks.get("sm_max_mhz")
                  and clocks["sm_mhz"] < 0.97 * clocks["sm_max_mhz"])
    if capped:
        return sustained, "bf16 sustained (power-capped clocks in the timed steps)"
    return burst, "bf16 burst"


def code_of(text):
    """C++/CUDA source with comments removed and each line's whitespace trimmed (string literals kept)."""
    import re

    pattern = re.compile(r'//[^\n]*|/\*.*?\*/|"(?:\\.|[^"\\])*"', re.S)
    text = pattern.sub(lambda m: m.group(0) if m.group(0).startswith('"') else " ", text)
    return "\n".join(line.strip() for line in text.splitlines() if line.strip())


def source_sha(name):
    """First 16 hex digits of the sha256 of a kernel source's code (comments and layout ignored)."""
    p = os.path.join(ROOT, "scaled_dot_product_prefill_b200", "csrc", name)
    with open(p, encoding="utf-8") as f:
        return hashlib.sha256(code_of(f.read()).encode()).hexdigest()[:16]


def recorded_traffic(kernel, workload, src):
    """DRAM bytes per launch from the committed ncu summary, if the kernel source is unchanged since."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.txt")
    if not os.path.exists(path):
        return None
    sha = source_sha(src)
    with open(path) as f:
        for line in f:
            parts = line.split("#", 1)[0].split()
            if len(parts) == 4 and parts[0] == kernel and parts[1] == workload and parts[2] == sha:
                return int(parts[3])
    return None


# ---------------------------------------------------------------- clocks


class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        self.out = ""
        if self.proc is not None:
            time.sleep(0.2)
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.out, _ = self.proc.communicate()

    def summary(self):
        rows = []
        for line in (getattr(self, "out", "") or "").splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                rows.append((float(f[1]), float(f[2]), f[5:9]))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        mx = max(r[1] for r in rows)
        load = [r for r in rows if r[0] > 0.5 * mx] or rows
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in load for i, v in enumerate(r[2]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(r[0] for r in load), "sm_max_mhz": mx, "reasons": reasons,
                "samples": len(load)}


# ---------------------------------------------------------------- CPU (oracle) legs


def cpu_threads():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


ORACLE_ROWS = 256   # query rows per oracle call in the CPU sample


def oracle_prefill_sample(budget_s=8.0):
    """Float64 oracle on blocks of query rows of the prefill workload until the budget is spent.

    Each call is the oracle's attention_rows for ORACLE_ROWS consecutive rows of
    one head against all of that head's keys, as the oracle computes them;
    the blocks walk the rows of head 0 from the end (the rows with the most
    visible keys first).  Work is counted as in the GPU leg: 4*D flops per
    visible (query, key) pair of the rows done.
    """
    from oracle import sdpa

    spec = PREFILL
    inp = inputs.prefill_inputs(1, 1, 1, spec.Sq, spec.Skv, spec.D, spec.seed)
    q, k, v = inp.q[0, 0], inp.k[0, 0], inp.v[0, 0]
    per_row = workloads.visible_per_row(spec.Sq, spec.Skv, spec.causal, spec.window)
    flops = done = 0
    n_blocks = (spec.Sq + ORACLE_ROWS - 1) // ORACLE_ROWS
    t0 = time.perf_counter()
    while time.perf_counter() - t0 < budget_s or done == 0:
        blk = n_blocks - 1 - done % n_blocks
        rows = list(range(blk * ORACLE_ROWS, min(spec.Sq, (blk + 1) * ORACLE_ROWS)))
        sdpa.attention_rows(q[rows], k, v, rows, spec.Sq, spec.scale, spec.causal, spec.window)
        flops += 4 * spec.D * int(per_row[rows].sum())
        done += 1
    dt = time.perf_counter() - t0
    return (flops / dt / 1e12,
            f"{done} blocks of {ORACLE_ROWS} query rows of one head of {spec.name} ({spec.Sq}x{spec.Skv}, "
            f"D={spec.D}, W={spec.window}), each against all {spec.Skv} keys as the oracle evaluates them", dt)


def oracle_decode_sample(budget_s=6.0):
    from oracle import sdpa

    spec = DECODE
    p = inputs.paged_inputs(4, spec.Hq, spec.Hkv, spec.D, spec.page_size, spec.seed, len_range=spec.len_range)
    nbytes = done = 0
    t0 = time.perf_counter()
    while time.perf_counter() - t0 < budget_s or done == 0:
        b = done % 4
        sdpa.decode_paged(p.q[b:b + 1], p.k_pool, p.v_pool, p.page_table[b:b + 1], p.seq_lens[b:b + 1],
                          spec.page_size, spec.scale, spec.window)
        nbytes += workloads.kv_bytes(p.seq_lens[b:b + 1].numpy(), spec.Hkv, spec.D)
        done += 1
    dt = time.perf_counter() - t0
    return nbytes / dt / 1e9, f"{done} sequences of {spec.name}", dt


# ---------------------------------------------------------------- GPU leg


def max_over_ranks(values, dist, device):
    """Element-wise maximum of ``values`` over all ranks (each rank's own list when ``dist`` is None).

    Every rank must call it at the same point with the same number of values.
    """
    values = [float(v) for v in values]
    if dist is None:
        return values
    import torch

    t = torch.tensor(values, dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def job_rate(units_per_rank, world, ms):
    """Whole-job throughput: the units all ranks processed over the slowest rank's time (weak scaling)."""
    return world * float(units_per_rank) / (ms * 1e-3)


def arm_config(world, seq_lens):
    """The workload description both arms print (decode sequence lengths of rank 0's seed)."""
    spec, dspec = PREFILL, DECODE
    return {
        "workload": f"{spec.name} + {dspec.name}",
        "prefill": {"B": spec.B, "Hq": spec.Hq, "Hkv": spec.Hkv, "S": spec.Sq, "D": spec.D,
                    "causal": spec.causal, "window": spec.window, "flops": workloads.prefill_flops(spec)},
        "decode": {"N": dspec.N, "Hq": dspec.Hq, "Hkv": dspec.Hkv, "D": dspec.D,
                   "page_size": dspec.page_size, "len_range": list(dspec.len_range),
                   "sum_len": int(np.sum(seq_lens)),
                   "kv_bytes": workloads.kv_bytes(seq_lens, dspec.Hkv, dspec.D),
                   "bytes": workloads.decode_bytes(seq_lens, dspec.Hq, dspec.Hkv, dspec.D, dspec.page_size)},
        "l2": "prefill: 256 MiB write before each call (and 335 MB of q/k/v/out > 126 MB L2); "
              "decode: 1.1 GB K/V > 126 MB L2",
        "parallelism": f"replicas x{world}",
    }


def run_ours(args, rank, world, local_rank):
    import torch

    from scaled_dot_product_prefill_b200 import api

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    peaks, peak_kind = load_peaks()
    spec = PREFILL
    pi = inputs.prefill_inputs(spec.B, spec.Hq, spec.Hkv, spec.Sq, spec.Skv, spec.D, spec.seed + rank)
    q, k, v = pi.q.to(dev), pi.k.to(dev), pi.v.to(dev)
    out = torch.empty_like(q)
    dspec = DECODE
    pd = inputs.paged_inputs(dspec.N, dspec.Hq, dspec.Hkv, dspec.D, dspec.page_size, dspec.seed + rank,
                             len_range=dspec.len_range)
    dq, kp, vp, pt, sl = (t.to(dev) for t in (pd.q, pd.k_pool, pd.v_pool, pd.page_table, pd.seq_lens))
    dout = torch.empty_like(dq)
    msl = pd.max_seq_len
    ws = torch.empty(api.attn_decode_paged_workspace_size(dspec.N, dspec.Hq, dspec.D, msl, dspec.page_size),
                     dtype=torch.uint8, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    p_flops = workloads.prefill_flops(spec)
    d_bytes = workloads.decode_bytes(pd.seq_lens.numpy(), dspec.Hq, dspec.Hkv, dspec.D, dspec.page_size)

    def step(ev=None):
        flush.zero_()
        if ev is not None:
            ev[0].record()
        api.attn_prefill(q, k, v, causal=spec.causal, window=spec.window, scale=spec.scale, out=out)
        if ev is not None:
            ev[1].record()
            ev[2].record()
        api.attn_decode_paged(dq, kp, vp, pt, sl, max_seq_len=msl, scale=dspec.scale, window=dspec.window,
                              workspace=ws, out=dout)
        if ev is not None:
            ev[3].record()

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    assert api.attn_device_status(clear=True) == 0
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local_rank) as clk:
        for i in range(args.steps):
            step(evs[i])
        torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    assert api.attn_device_status(clear=True) == 0
    t_pre = [e[0].elapsed_time(e[1]) for e in evs]
    t_dec = [e[2].elapsed_time(e[3]) for e in evs]
    pre_ms, dec_ms = float(np.mean(t_pre)), float(np.mean(t_dec))
    stats = {name: {"median": round(float(np.median(t)), 5), "mean": round(float(np.mean(t)), 5),
                    "std": round(float(np.std(t)), 5)} for name, t in (("prefill_ms", t_pre), ("decode_ms", t_dec))}
    step_ms = pre_ms + dec_ms
    pre_ms, dec_ms, step_ms = max_over_ranks([pre_ms, dec_ms, step_ms], dist, dev)

    # ---- end to end through the public API: pinned host inputs -> device -> kernel -> host result
    hq, hk, hv = (t.pin_memory() for t in (pi.q, pi.k, pi.v))
    hout = torch.empty_like(pi.q).pin_memory()
    e_steps = max(10, args.steps // 10)
    e_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(e_steps)]
    for i in range(e_steps + 3):
        flush.zero_()
        ev = e_ev[i - 3] if i >= 3 else None
        if ev:
            ev[0].record()
        # one call: host-to-device copies, kernels and the copy back, overlapped piece by piece
        api.attn_prefill_host(hq, hk, hv, causal=spec.causal, window=spec.window, scale=spec.scale, out=hout,
                              device_buffers=(q, k, v, out))
        if ev:
            ev[1].record()
    torch.cuda.synchronize()
    e2e_ms = float(np.mean([e[0].elapsed_time(e[1]) for e in e_ev]))
    (e2e_ms,) = max_over_ranks([e2e_ms], dist, dev)
    h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv))
    d2h = hout.numel() * hout.element_size()

    # ---- the decode half end to end: the step's query and new key/value from pinned host memory, appended
    # to the resident cache, decoded, and the output read back, in one attn_decode_step_host call
    gen = np.random.default_rng(rank)
    dq_h = pd.q.pin_memory()
    kn_h = torch.from_numpy(gen.standard_normal((dspec.N, dspec.Hkv, 1, dspec.D), dtype=np.float32)).to(
        torch.bfloat16).pin_memory()
    vn_h = torch.from_numpy(gen.standard_normal((dspec.N, dspec.Hkv, 1, dspec.D), dtype=np.float32)).to(
        torch.bfloat16).pin_memory()
    dout_h = torch.empty_like(pd.q).pin_memory()
    dbufs = (torch.empty_like(dq), torch.empty(kn_h.shape, dtype=torch.bfloat16, device=dev),
             torch.empty(vn_h.shape, dtype=torch.bfloat16, device=dev), torch.empty_like(dq))
    d_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(e_steps)]
    for i in range(e_steps + 3):
        ev = d_ev[i - 3] if i >= 3 else None
        if ev:
            ev[0].record()
        api.attn_decode_step_host(dq_h, kn_h, vn_h, kp, vp, pt, sl, max_seq_len=msl, scale=dspec.scale,
                                  window=dspec.window, out=dout_h, device_buffers=dbufs, workspace=ws)
        if ev:
            ev[1].record()
    torch.cuda.synchronize()
    assert api.attn_device_status(clear=True) == 0
    e2e_dec_ms = float(np.mean([e[0].elapsed_time(e[1]) for e in d_ev]))
    (e2e_dec_ms,) = max_over_ranks([e2e_dec_ms], dist, dev)
    h2d_dec = sum(t.numel() * t.element_size() for t in (dq_h, kn_h, vn_h))
    d2h_dec = dout_h.numel() * dout_h.element_size()

    # ---- the prefill replayed from a CUDA graph: the same kernel without the host launch path
    graph_ms = None
    if rank == 0 and not args.no_extra:
        graph_ms = graph_prefill_ms(lambda: api.attn_prefill(q, k, v, causal=spec.causal, window=spec.window,
                                                             scale=spec.scale, out=out), flush, args.steps)

    # ---- the other workloads, one line each (parity cases, reported for context)
    extra = {}
    if rank == 0 and not args.no_extra:
        extra = other_workloads(dev, peaks)
        extra.update(append_workloads(dev, peaks))
        extra.update(fp8_decode_workload(dev, peaks))
        extra.update(paged_prefill_workload(dev, peaks))

    result = None
    if rank == 0:
        tflops = job_rate(p_flops, world, pre_ms) / 1e12
        clocks = clk.summary()
        peak_t, kind_t = tensor_peak(peaks, clocks)   # both fractions are reported below
        peak_burst = float(peaks["bf16_tflops"])
        peak_sust = float(peaks.get("bf16_tflops_sustained", peak_burst))
        peak_h = float(peaks["hbm_gbs"])
        ach_t = p_flops / (pre_ms * 1e-3) / 1e12
        ach_d = d_bytes / (dec_ms * 1e-3) / 1e9
        traffic = recorded_traffic("prefill_tc_kernel", spec.name, "prefill_sm100.cu")
        traffic_d = recorded_traffic("decode_split_kernel", dspec.name, "decode_paged.cu")
        result = {
            "metric": METRIC,
            "value": round(tflops, 3),
            "unit": "TFLOP/s",
            "n_gpus": world,
            "steps": args.steps,
            "warmup": max(3, args.warmup),
            "ms_per_step": round(step_ms, 5),
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "bf16",
            "data": "synthetic (seeded N(0,1), bf16)",
            "config": arm_config(world, pd.seq_lens.numpy()),
            "roofline": {"bound": "tensor", "achieved": round(ach_t, 2), "peak": peak_t, "unit": "TFLOP/s",
                         "frac": round(ach_t / peak_t, 4), "traffic": traffic,
                         "algorithmic_flops": p_flops, "ms": round(pre_ms, 5),
                         "kernel": f"prefill_tc_kernel<{spec.D}, false>", "peak_kind": f"{kind_t}, {peak_kind}",
                         "frac_of_burst": round(ach_t / peak_burst, 4),
                         "frac_of_sustained": round(ach_t / peak_sust, 4)},
            "roofline_decode": {"bound": "hbm", "achieved": round(ach_d, 1), "peak": peak_h, "unit": "GB/s",
                                "frac": round(ach_d / peak_h, 4), "traffic": traffic_d, "algorithmic_bytes": d_bytes,
                                "ms": round(dec_ms, 5),
                                "kernel": "decode_split_kernel<128,4,false> + decode_combine_kernel<128>",
                                "peak_kind": f"HBM copy, {peak_kind}"},
            "decode": {"value": round(job_rate(d_bytes, world, dec_ms) / 1e9, 1), "unit": "GB/s",
                       "ms": round(dec_ms, 5)},
            "prefill_ms": round(pre_ms, 5),
            "timing": dict(stats, prefill_graph_ms=None if graph_ms is None else round(graph_ms, 5)),
            "e2e": {"value": round(job_rate(p_flops, world, e2e_ms) / 1e12, 3), "unit": "TFLOP/s",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms": round(e2e_ms, 5),
                    "path": "attn_prefill_host: pinned host q/k/v -> device -> kernels -> pinned host out, "
                            "in pieces whose copies overlap the kernels"},
            "e2e_decode": {"value": round(job_rate(d_bytes, world, e2e_dec_ms) / 1e9, 1), "unit": "GB/s",
                           "h2d_bytes_per_step": h2d_dec, "d2h_bytes_per_step": d2h_dec,
                           "ms": round(e2e_dec_ms, 5),
                           "path": "attn_decode_step_host: pinned host q and new k/v -> device -> append -> "
                                   "decode -> pinned host out"},
            "gpu_launches": 3 * args.steps,
            "clocks": clocks,
            "workloads": extra,
        }
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return result


def time_call(fn, reps, flush=None, clean_flush=None):
    import torch

    for _ in range(3):
        fn()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(reps)]
    for e in ev:
        if flush is not None:
            flush.zero_()
        if clean_flush is not None:
            clean_flush.sum()
        e[0].record()
        fn()
        e[1].record()
    torch.cuda.synchronize()
    return float(np.median([a.elapsed_time(b) for a, b in ev]))


def graph_prefill_ms(fn, flush, reps):
    """Median time of fn replayed from a CUDA graph (captured once), with an L2 flush before each replay."""
    import torch

    reps = max(10, min(reps, 200))
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        fn()
    torch.cuda.current_stream().wait_stream(s)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, capture_error_mode="relaxed"):
        fn()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(reps)]
    for _ in range(3):
        g.replay()
    for e in ev:
        flush.zero_()
        e[0].record()
        g.replay()
        e[1].record()
    torch.cuda.synchronize()
    ms = float(np.median([a.elapsed_time(b) for a, b in ev]))
    del g
    return ms


def fp8_decode_workload(dev, peaks):
    """attn_decode_paged_fp8 on the paged_decode_gqa shape with an E4M3 cache (1 byte per K/V element)."""
    import torch

    from scaled_dot_product_prefill_b200 import api

    dspec = DECODE
    ks = vs = 1.0 / 64
    pd = inputs.paged_inputs_fp8(dspec.N, dspec.Hq, dspec.Hkv, dspec.D, dspec.page_size, dspec.seed, k_scale=ks,
                                 v_scale=vs, len_range=dspec.len_range)
    dq, kp, vp, pt, sl = (t.to(dev) for t in (pd.q, pd.k_pool, pd.v_pool, pd.page_table, pd.seq_lens))
    out = torch.empty_like(dq)
    msl = pd.max_seq_len
    ws = torch.empty(api.attn_decode_paged_workspace_size(dspec.N, dspec.Hq, dspec.D, msl, dspec.page_size),
                     dtype=torch.uint8, device=dev)
    ms = time_call(lambda: api.attn_decode_paged_fp8(dq, kp, vp, pt, sl, max_seq_len=msl, k_scale=ks, v_scale=vs,
                                                     scale=dspec.scale, workspace=ws, out=out), 100)
    lens = pd.seq_lens.numpy()
    kv = int(lens.sum()) * dspec.Hkv * dspec.D * 2          # K and V, one byte each
    nbytes = kv + workloads.decode_bytes(lens, dspec.Hq, dspec.Hkv, dspec.D, dspec.page_size) - \
        workloads.kv_bytes(lens, dspec.Hkv, dspec.D)
    gbs = nbytes / (ms * 1e-3) / 1e9
    res = {"decode_fp8_" + dspec.name: {"ms": round(ms, 5), "GB/s": round(gbs, 1), "bytes": int(nbytes),
                                        "frac_of_hbm": round(gbs / float(peaks["hbm_gbs"]), 4),
                                        "tokens_per_s": round(int(lens.sum()) / (ms * 1e-3), 1),
                                        "l2": "none (0.57 GB of K/V > L2)"}}
    del kp, vp
    torch.cuda.empty_cache()
    return res


def append_workloads(dev, peaks):
    """attn_kv_append on a decode step, a prefill chunk and a copy larger than L2.

    HBM-bound copies: bytes = 2 (K, V) x 2 (read + write) x B x Hkv x S_new x D x 2 B.  The two serving
    shapes run after a 256 MB read, which leaves L2 holding clean lines (a write flush would leave dirty
    lines whose write-back lands inside the timed copy); the large one needs no flush.
    """
    import torch

    from scaled_dot_product_prefill_b200 import api

    clean = torch.ones(64 << 20, device=dev)
    res = {}
    shapes = {"kv_append_decode_step": (64, 8, 1, 128, 16, 4096, True),       # paged_decode_gqa's new tokens
              "kv_append_prefill_chunk": (8, 12, 1024, 64, 16, 1024, True),   # mha_causal_gpt2s's K/V
              "kv_append_large": (8, 8, 8192, 128, 16, 8192, False)}         # 537 MB moved, > L2
    for name, (B, Hkv, S_new, D, page, L, flush) in shapes.items():
        npg = -(-L // page)
        perm = torch.randperm(B * npg, generator=torch.Generator().manual_seed(B)).to(torch.int32)
        table = perm.reshape(B, npg).to(dev)
        lens = torch.full((B,), L, dtype=torch.int32, device=dev)
        kp = torch.zeros((B * npg, Hkv, page, D), dtype=torch.bfloat16, device=dev)
        vp = torch.zeros_like(kp)
        kn = torch.randn((B, Hkv, S_new, D), device=dev).to(torch.bfloat16)
        vn = torch.randn_like(kn)
        ms = time_call(lambda: api.attn_kv_append(kn, vn, kp, vp, table, lens), 50,
                       clean_flush=clean if flush else None)
        nbytes = 4 * B * Hkv * S_new * D * 2
        gbs = nbytes / (ms * 1e-3) / 1e9
        res[name] = {"ms": round(ms, 5), "GB/s": round(gbs, 1), "bytes": nbytes,
                     "frac_of_hbm": round(gbs / float(peaks["hbm_gbs"]), 4),
                     "l2": "256 MB read before each call" if flush else "none (data > L2)"}
        del kp, vp, kn, vn
    torch.cuda.empty_cache()
    return res


def other_workloads(dev, peaks):
    """The other prefill workloads, each timed on its own with a roofline entry of its own.

    Median of 20 CUDA-event timed calls, a 256 MiB write before each.  ``traffic`` is the DRAM
    bytes per launch from the committed ncu record for this kernel source and workload, or null.
    """
    import torch

    from scaled_dot_product_prefill_b200 import api

    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    res = {}
    for name, spec in workloads.WORKLOADS.items():
        if not isinstance(spec, workloads.PrefillSpec) or name == PREFILL.name:
            continue
        pi = inputs.prefill_inputs(spec.B, spec.Hq, spec.Hkv, spec.Sq, spec.Skv, spec.D, spec.seed, spec.dtype)
        q, k, v = pi.q.to(dev), pi.k.to(dev), pi.v.to(dev)
        out = torch.empty_like(q)
        fn = api.attn_prefill if spec.dtype == "bf16" else api.attn_prefill_f32
        ms = time_call(lambda: fn(q, k, v, causal=spec.causal, window=spec.window, scale=spec.scale, out=out),
                       20, flush)
        fl = workloads.prefill_flops(spec)
        ach = fl / (ms * 1e-3) / 1e12
        entry = {"ms": round(ms, 5), "TFLOP/s": round(ach, 2), "flops": fl}
        if spec.dtype == "bf16":
            peak = float(peaks["bf16_tflops"])
            entry["roofline"] = {"bound": "tensor", "achieved": round(ach, 2), "peak": peak, "unit": "TFLOP/s",
                                 "frac": round(ach / peak, 4),
                                 "traffic": recorded_traffic("prefill_tc_kernel", name, "prefill_sm100.cu"),
                                 "kernel": f"prefill_tc_kernel<{spec.D}, false>"}
        else:
            entry["traffic"] = recorded_traffic("prefill_f32_kernel", name, "prefill_f32.cu")
        res[name] = entry
        del q, k, v, out
    torch.cuda.empty_cache()
    return res


def paged_prefill_workload(dev, peaks):
    """The chunked prefill over a paged cache (bottom-right causal), one timing."""
    import torch

    from scaled_dot_product_prefill_b200 import api

    spec = workloads.EXTRA_WORKLOADS["chunked_prefill_paged_gqa"]
    p = inputs.paged_inputs(spec.B, spec.Hq, spec.Hkv, spec.D, spec.page_size, spec.seed, seq_lens=[spec.L] * spec.B)
    q = inputs.normal((spec.B, spec.Hq, spec.Sq, spec.D), seed=spec.seed + 1).to(dev)
    kp, vp, pt, sl = (t.to(dev) for t in (p.k_pool, p.v_pool, p.page_table, p.seq_lens))
    out = torch.empty_like(q)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    ms = time_call(lambda: api.attn_prefill_paged(q, kp, vp, pt, sl, max_seq_len=spec.L, causal=True,
                                                  scale=spec.scale, out=out), 20, flush)
    ach = workloads.paged_prefill_flops(spec) / (ms * 1e-3) / 1e12
    res = {spec.name: {"ms": round(ms, 5), "TFLOP/s": round(ach, 2),
                       "frac_of_bf16_peak": round(ach / float(peaks["bf16_tflops"]), 4),
                       "l2": "256 MB write before each call"}}
    del q, kp, vp, pt, sl, out, flush
    torch.cuda.empty_cache()
    return res


def profile_case(name, calls):
    """Run one workload ``calls`` times and nothing else, for a profiler capture of its kernels.

    ``name`` is a prefill workload of ``workloads.WORKLOADS``, ``paged_decode_gqa``,
    ``paged_decode_gqa_fp8`` (the same decode over an 8-bit cache), or ``chunked_prefill_paged_gqa``.  Prints one line with the
    mean CUDA-event time, which is not a benchmark number when taken under a profiler.
    """
    import torch

    from scaled_dot_product_prefill_b200 import api

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    if name.startswith("paged_decode_gqa"):
        spec = workloads.WORKLOADS["paged_decode_gqa"]
        fp8 = name.endswith("_fp8")
        if fp8:
            pd = inputs.paged_inputs_fp8(spec.N, spec.Hq, spec.Hkv, spec.D, spec.page_size, spec.seed,
                                         k_scale=1 / 64, v_scale=1 / 64, len_range=spec.len_range)
        else:
            pd = inputs.paged_inputs(spec.N, spec.Hq, spec.Hkv, spec.D, spec.page_size, spec.seed,
                                     len_range=spec.len_range)
        dq, kp, vp, pt, sl = (t.to(dev) for t in (pd.q, pd.k_pool, pd.v_pool, pd.page_table, pd.seq_lens))
        ws = torch.empty(api.attn_decode_paged_workspace_size(spec.N, spec.Hq, spec.D, pd.max_seq_len,
                                                              spec.page_size), dtype=torch.uint8, device=dev)
        out = torch.empty_like(dq)
        if fp8:
            fn = lambda: api.attn_decode_paged_fp8(dq, kp, vp, pt, sl, max_seq_len=pd.max_seq_len, k_scale=1 / 64,
                                                   v_scale=1 / 64, scale=spec.scale, workspace=ws, out=out)
        else:
            fn = lambda: api.attn_decode_paged(dq, kp, vp, pt, sl, max_seq_len=pd.max_seq_len, scale=spec.scale,
                                               workspace=ws, out=out)
    elif name in workloads.EXTRA_WORKLOADS:
        spec = workloads.EXTRA_WORKLOADS[name]
        pp = inputs.paged_inputs(spec.B, spec.Hq, spec.Hkv, spec.D, spec.page_size, spec.seed,
                                 seq_lens=[spec.L] * spec.B)
        q = inputs.normal((spec.B, spec.Hq, spec.Sq, spec.D), seed=spec.seed + 1).to(dev)
        kp, vp, pt, sl = (t.to(dev) for t in (pp.k_pool, pp.v_pool, pp.page_table, pp.seq_lens))
        out = torch.empty_like(q)
        fn = lambda: api.attn_prefill_paged(q, kp, vp, pt, sl, max_seq_len=spec.L, causal=True, scale=spec.scale,
                                            out=out)
    else:
        spec = workloads.WORKLOADS[name]
        pi = inputs.prefill_inputs(spec.B, spec.Hq, spec.Hkv, spec.Sq, spec.Skv, spec.D, spec.seed, spec.dtype)
        q, k, v = pi.q.to(dev), pi.k.to(dev), pi.v.to(dev)
        out = torch.empty_like(q)
        call = api.attn_prefill if spec.dtype == "bf16" else api.attn_prefill_f32
        fn = lambda: call(q, k, v, causal=spec.causal, window=spec.window, scale=spec.scale, out=out)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    ev[0].record()
    for _ in range(calls):
        fn()
    ev[1].record()
    torch.cuda.synchronize()
    assert api.attn_device_status(clear=True) == 0
    print(json.dumps({"profile_case": name, "calls": calls, "ms_per_call": ev[0].elapsed_time(ev[1]) / calls}))


def reference_line(args, rank, world):
    """The float64 oracle on the host cores, on a bounded sample of the same workload."""
    if rank != 0:
        return None
    threads = cpu_threads()
    per_step = []
    for _ in range(max(1, args.steps) + max(0, min(args.warmup, 1))):
        v, sample, dt = oracle_prefill_sample(budget_s=min(10.0, 60.0 / max(1, args.steps)))
        per_step.append(v)
    v = float(np.mean(per_step[-max(1, args.steps):]))
    return {
        "impl": "reference", "metric": METRIC, "value": round(v, 6), "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded N(0,1), bf16 values upcast)",
        "config": arm_config(world, inputs.draw_seq_lens(DECODE.N, DECODE.seed, DECODE.len_range).numpy()),
        "cpu_baseline": {"value": round(v, 6), "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(v, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra", action="store_true")
    ap.add_argument("--profile", default=None,
                    help="run only this workload --steps times, for a profiler capture (prints no bench line)")
    args = ap.parse_args()
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", args.gpus if args.gpus == 1 else 1))
    local_rank = int(os.environ.get("LOCAL_RANK", 0))
    threads = cpu_threads()
    os.environ.setdefault("OMP_NUM_THREADS", str(threads))

    if args.profile is not None:
        profile_case(args.profile, max(1, args.steps))
        return

    if args.impl == "reference":
        line = reference_line(args, rank, world)
        if line is not None:
            print(json.dumps(line))
        return

    result = run_ours(args, rank, world, local_rank)
    if rank == 0:
        if not args.no_cpu_baseline and world == 1:
            v, sample, dt = oracle_prefill_sample()
            vd, sample_d, dtd = oracle_decode_sample()
            result["cpu_baseline"] = {"value": round(v, 6), "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                                      "sample": sample, "seconds": round(dt, 2),
                                      "decode": {"value": round(vd, 4), "unit": "GB/s", "sample": sample_d,
                                                 "seconds": round(dtd, 2)}}
        print(json.dumps(result))


if __name__ == "__main__":
    main()
