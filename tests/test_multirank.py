"""The replicas path of bench.py on two CPU ranks (gloo): every rank takes the
same collective steps (barrier, max of the elapsed time), the slowest rank's
time is what all ranks see, and the job value sums the per-GPU work."""

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        bench.barrier(world)
        # rank r "measured" 10 + r ms; every rank must see the slowest
        got = bench.max_over_ranks(10.0 + rank, world, torch.device("cpu"))
        bench.barrier(world)
        out[rank] = got
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_barrier_two_gloo_ranks():
    world = 2
    out = mp.Manager().dict()
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    assert dict(out) == {0: 11.0, 1: 11.0}


def test_single_rank_needs_no_process_group():
    import bench
    assert bench.max_over_ranks(3.5, 1, torch.device("cpu")) == 3.5
    bench.barrier(1)  # a no-op without a process group


@pytest.mark.parametrize("world", [1, 2, 8])
def test_job_value_is_summed_over_replicas(world):
    """A step at half the roofline rate scores 50 % per GPU, summed over the
    replicas (weak scaling)."""
    import bench
    peaks = {"hbm_gbs": 6456.5, "bf16_tflops": 1698.5, "bf16_tflops_sustained": 1422.0,
             "source": "test"}
    table = bench.op_table(peaks, peaks["bf16_tflops"])
    roof_ms = sum(v["t_roof"] for v in table.values()) * 1e3
    assert bench.job_value(table, 2 * roof_ms, world) == pytest.approx(50.0 * world)


def test_tensor_peak_follows_the_recorded_clocks():
    """The bf16 denominator is the burst figure unless the timed region's own
    clock record shows the power cap or clocks well below maximum."""
    import bench
    peaks = {"hbm_gbs": 6456.5, "bf16_tflops": 1698.5, "bf16_tflops_sustained": 1422.0}
    assert bench.tensor_peak(peaks, {"sm_mhz": 1965, "sm_max_mhz": 1965, "reasons": []}) == (
        1698.5, "burst")
    assert bench.tensor_peak(peaks, {"sm_mhz": 1965, "sm_max_mhz": 1965,
                                     "reasons": ["sw_power_cap"]}) == (1422.0, "sustained")
    assert bench.tensor_peak(peaks, {"sm_mhz": 1372, "sm_max_mhz": 1965, "reasons": []}) == (
        1422.0, "sustained")
    assert bench.tensor_peak(peaks, {"sm_mhz": None, "sm_max_mhz": None,
                                     "reasons": ["unavailable"]}) == (1698.5, "burst")
