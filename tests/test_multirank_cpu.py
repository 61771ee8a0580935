"""The multi-rank path of bench.py on CPU: two gloo ranks, no GPU.

The attention path has no exchange step; with N GPUs every rank runs its own
replica of the per-GPU workload, the times are reduced with a maximum over
ranks, and the whole-job rate counts the work of all ranks over that time.
These tests run those host steps as world-size-2 gloo process groups.
"""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from conftest import ROOT

sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, queue):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    try:
        import datetime

        dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
        # each rank reports its own times; every rank must see the maximum
        mine = [1.0 + rank, 10.0 - rank, 0.5 * (rank + 1)]
        got = bench.max_over_ranks(mine, dist, "cpu")
        # the reference arm runs on rank 0 only: the other ranks return without work
        args = type("A", (), {"steps": 1, "warmup": 0})()
        ref = bench.reference_line(args, rank, world) if rank != 0 else "rank0"
        dist.barrier()
        queue.put((rank, got, ref))
        dist.destroy_process_group()
    except Exception as e:  # report instead of hanging the parent
        queue.put((rank, repr(e), None))


def test_two_gloo_ranks_take_the_maximum_time_and_only_rank_0_runs_the_reference():
    world = 2
    ctx = mp.get_context("spawn")
    queue = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, queue)) for r in range(world)]
    for p in procs:
        p.start()
    results = {}
    for _ in range(world):
        rank, got, ref = queue.get(timeout=120)
        results[rank] = (got, ref)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank in range(world):
        got, ref = results[rank]
        assert got == [2.0, 10.0, 1.0], got
    assert results[1][1] is None


def test_single_process_keeps_its_own_times_and_rates_count_every_rank():
    assert bench.max_over_ranks([3.0, 4.0], None, "cpu") == [3.0, 4.0]
    # 2 ranks, 10 GFLOP each, slowest rank 5 ms: 4 TFLOP/s for the job
    assert bench.job_rate(10e9, 2, 5.0) == pytest.approx(4e12)
    assert bench.job_rate(10e9, 1, 5.0) == pytest.approx(2e12)


def test_gloo_is_available():
    assert dist.is_available() and dist.is_gloo_available()
    assert torch.multiprocessing.get_all_start_methods()


def test_both_arms_describe_the_same_workload():
    """The reference arm draws the decode lengths without building the pools; they must be the lengths the
    timed arm's generated cache has."""
    import numpy as np

    from scaled_dot_product_prefill_b200 import inputs

    for seed, rng in ((5, (512, 8192)), (1234, (1, 40))):
        p = inputs.paged_inputs(6, 8, 2, 64, 16, seed=seed, len_range=rng)
        assert np.array_equal(p.seq_lens.numpy(), inputs.draw_seq_lens(6, seed, rng).numpy())
    d = bench.DECODE
    lens = inputs.draw_seq_lens(d.N, d.seed, d.len_range).numpy()
    cfg = bench.arm_config(1, lens)
    assert cfg["decode"]["sum_len"] == int(lens.sum()) and cfg["workload"].startswith(bench.PREFILL.name)


def test_tensor_peak_follows_the_clock_record():
    """Burst peak for a short run at full clock; the sustained peak when the power cap held the clock down."""
    peaks = {"bf16_tflops": 1650.8, "bf16_tflops_sustained": 1354.4, "hbm_gbs": 6535.7}
    assert bench.tensor_peak(peaks, {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": []})[0] == 1650.8
    # the cap was active but did not pull the clock down: still the burst figure
    assert bench.tensor_peak(peaks, {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"]})[0] == 1650.8
    assert bench.tensor_peak(peaks, {"sm_mhz": 1770.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"]})[0] == 1354.4
    # a clock held down with no reason (a lock) is not a power cap
    assert bench.tensor_peak(peaks, {"sm_mhz": 1500.0, "sm_max_mhz": 1965.0, "reasons": []})[0] == 1650.8
    assert bench.tensor_peak(peaks, {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]})[0] == 1650.8
    assert bench.tensor_peak({"bf16_tflops": 1590.0}, {"sm_mhz": 1300.0, "sm_max_mhz": 1965.0,
                                                        "reasons": ["sw_power_cap"]})[0] == 1590.0
