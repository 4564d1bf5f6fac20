"""The benchmark's multi-rank bookkeeping on CPU (gloo, world size 2): every
rank processes its own sequence (no data-path collective); the job time is
the slowest rank's, and the whole-job throughput counts all ranks' tokens."""
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


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = 100.0 + 50.0 * rank                    # rank 1 is slower
        m = bench.max_over_ranks(ms, dist, torch.device("cpu"))
        v = bench.weak_scaling_value(65536, 10, world, m)
        again = bench.any_rank(rank == 1, dist, torch.device("cpu"))   # one rank saw throttling
        q.put((rank, m, v, again))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_weak_scaling_with_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    assert [r[1] for r in res] == [150.0, 150.0]
    assert res[0][2] == res[1][2] == pytest.approx(2 * 65536 * 10 / 0.150)
    assert res[0][3] is True and res[1][3] is True          # both ranks measure again together


def test_single_rank_is_identity():
    assert bench.max_over_ranks(12.5) == 12.5
    assert bench.weak_scaling_value(1000, 4, 1, 2000.0) == pytest.approx(2000.0)


def test_clock_records_that_force_a_second_measurement():
    ok = {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": [], "samples": 10}
    assert not bench.clocks_rejected(ok)
    assert not bench.clocks_rejected(dict(ok, sm_mhz=1300.0, reasons=["sw_power_cap"]))   # power cap: kept
    for r in ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"):
        assert bench.clocks_rejected(dict(ok, reasons=[r]))
    assert bench.clocks_rejected(dict(ok, sm_mhz=1200.0))                                 # held low, no reason
    assert not bench.clocks_rejected({"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]})
    assert bench.any_rank(True) and not bench.any_rank(False)

