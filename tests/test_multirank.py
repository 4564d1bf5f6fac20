"""Multi-rank paths on CPU (gloo, world size 2): the benchmark's bookkeeping
(every rank processes its own sequence, no data-path collective; the job time is
the slowest rank's, the whole-job throughput counts all ranks' tokens; a
re-measurement decided by any rank is taken by all), and sharding one sequence
by GQA group, which needs no exchange and reproduces the single-rank result."""
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



def _group_worker(rank, world, port, q):
    import numpy as np

    import oracle
    from sparse_attention_long_phi_b200 import inputs as I
    from sparse_attention_long_phi_b200 import shard
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        c = dict(B=1, T=200, H=8, G=4, dk=16, dv=8, l=8, d=4, lp=16, n=4, fi=1, fl=2, w=24,
                 phi="linear", seed=21)
        x = {k: (I.bits(v) if v.dtype == torch.bfloat16 else v.numpy())
             for k, v in I.make_forward_inputs(c, "cpu").items()}
        g0, g1 = shard.group_range(c["G"], rank, world)
        cs, xs = shard.slice_groups(c, x, g0, g1)
        kc, vc = oracle.phi(cs, xs["k"], xs["v"], xs["wk"], xs["ek"], xs["wv"], xs["ev"])
        r = oracle.forward_rows(cs, xs["q"], xs["k"], xs["v"], xs["gates"], kc, vc, np.arange(200))
        parts = [None] * world
        dist.all_gather_object(parts, (g0, g1, r["out"], r["idx"]))   # no data-path exchange: results only
        if rank == 0:
            kc, vc = oracle.phi(c, x["k"], x["v"], x["wk"], x["ek"], x["wv"], x["ev"])
            full = oracle.forward_rows(c, x["q"], x["k"], x["v"], x["gates"], kc, vc, np.arange(200))
            out = np.concatenate([p[2] for p in parts], axis=1)
            idx = np.concatenate([p[3] for p in parts], axis=1)
            q.put((np.array_equal(out, full["out"]), np.array_equal(idx, full["idx"]),
                   [p[:2] for p in parts]))
    finally:
        dist.destroy_process_group()


def test_group_sharding_is_exact_with_two_gloo_ranks():
    # the operator splits by GQA group with no exchange: two ranks' outputs, concatenated
    # along the heads, are bit for bit the single-rank result (fp64 oracle as the compute)
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_group_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(180)
        assert p.exitcode == 0
    same_out, same_idx, ranges = q.get(timeout=10)
    assert ranges == [(0, 2), (2, 4)]
    assert same_out and same_idx


def test_group_ranges_cover_every_group_once():
    from sparse_attention_long_phi_b200 import shard
    for G in (1, 2, 3, 4, 7, 8):
        for world in range(1, G + 1):
            rs = [shard.group_range(G, r, world) for r in range(world)]
            assert rs[0][0] == 0 and rs[-1][1] == G
            assert all(a[1] == b[0] for a, b in zip(rs, rs[1:]))
            assert max(g1 - g0 for g0, g1 in rs) - min(g1 - g0 for g0, g1 in rs) <= 1
    with pytest.raises(ValueError):
        shard.group_range(2, 0, 3)


def test_slice_groups_on_torch_tensors():
    from sparse_attention_long_phi_b200 import inputs as I
    from sparse_attention_long_phi_b200 import shard
    c = dict(I.WORKLOADS["prefill_fwd_T8192"], T=64)
    x = I.make_forward_inputs(c, "cpu", with_dout=True)
    cs, xs = shard.slice_groups(c, x, 1, 3)
    assert (cs["G"], cs["H"]) == (2, 32)
    assert xs["q"].shape == (1, 64, 32, 192) and xs["q"].is_contiguous()
    assert torch.equal(xs["q"], x["q"][:, :, 16:48]) and torch.equal(xs["k"], x["k"][:, :, 1:3])
    assert torch.equal(xs["gates"], x["gates"][:, :, 16:48]) and torch.equal(xs["dout"], x["dout"][:, :, 16:48])
    assert xs["wk"] is x["wk"]                       # the phi parameters are shared by every group
