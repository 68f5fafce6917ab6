"""Host-side logic of bench.py on CPU: the max-over-ranks timing reduction with
two gloo ranks (the data path has no collective), the clock-sample summary, the
FLOP convention and when the stored dK/dV DRAM figure is reported."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, values, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        out[rank] = bench.max_over_ranks(values[rank], world)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    world = 2
    values = [3.5, 7.25]
    out = mp.get_context("spawn").Manager().dict()
    mp.spawn(_worker, args=(world, _free_port(), values, out), nprocs=world, join=True)
    assert out[0] == out[1] == max(values)


def test_max_over_ranks_single_rank_is_identity():
    assert bench.max_over_ranks(4.0, 1) == 4.0


def test_clock_summary():
    lines = ["1965, 1965, 0x0, Not Active, Not Active, Not Active, Not Active",
             "1800, 1965, 0x4, Not Active, Not Active, Not Active, Active",
             "1900, 1965, 0x0, Not Active, Not Active, Not Active, Not Active",
             "garbage"]
    s = bench.summarize_clock_lines(lines)
    assert s["sm_mhz"] == 1900 and s["sm_max_mhz"] == 1965
    assert s["reasons"] == ["sw_power_cap"] and s["samples"] == 3
    assert bench.summarize_clock_lines([])["reasons"] == ["unsampled"]


def test_flop_convention():
    w = dict(B=1, S=16384, Hq=32, D=128, causal=True)
    assert bench.flops_fwd(w) == 4 * 32 * 16384 ** 2 * 128 / 2
    w["causal"] = False
    assert bench.flops_fwd(w) == 4 * 32 * 16384 ** 2 * 128


def test_dkdv_traffic_is_reported_only_for_its_sources_and_workload(monkeypatch):
    """The stored ncu DRAM figure of the dK/dV kernel is reported for the workload it
    was captured on while the kernel's sources hash to what was captured, else null."""
    rec = dict(bench.DKDV_TRAFFIC)
    assert bench.dkdv_traffic("some_other_workload") is None
    monkeypatch.setattr(bench, "DKDV_TRAFFIC", dict(rec, sources_sha256="0" * 64))
    assert bench.dkdv_traffic(rec["workload"]) is None
    monkeypatch.setattr(bench, "DKDV_TRAFFIC", dict(rec, sources_sha256=bench.dkdv_sources_sha256()))
    assert bench.dkdv_traffic(rec["workload"]) == rec["bytes"]
