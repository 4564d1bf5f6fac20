"""bench.py's host flow on the CPU, with fakes in place of the CUDA runtime and
the library: the warm-up and timed steps, the second measurement after a
throttled timed region, the roofline of the dominant kernel and the keys of the
JSON line the benchmark contract asks for."""
import contextlib
import io
import json
import sys
import types

import pytest
import torch

import bench
from sparse_attention_long_phi_b200 import inputs as I


class _Event:
    def __init__(self, enable_timing=False):
        pass

    def record(self, stream=None):
        pass

    def synchronize(self):
        pass

    def elapsed_time(self, other):
        return 660.0          # 20 steps of 33 ms


def _run(monkeypatch, clock_records, argv, inputs=None):
    calls = {"forward": 0, "regions": 0}
    monkeypatch.setattr(torch.cuda, "Event", _Event)
    monkeypatch.setattr(torch.cuda, "synchronize", lambda *a, **k: None)
    monkeypatch.setattr(torch.cuda, "set_device", lambda *a, **k: None)
    monkeypatch.setattr(torch.cuda, "current_stream", lambda *a, **k: None)
    fake = types.ModuleType("sparse_attention_long_phi_b200.nsa")
    fake.forward_buffers = lambda c, dev, want_lse=False: object()

    def forward_into(*a, **k):
        calls["forward"] += 1
    fake.forward_into = forward_into
    fake.sync_status = lambda *a: None
    fake.profile_enable = lambda on=True: None
    fake.profile_read = lambda *a: {"attn_sel_kernel": (20, 341.0), "attn_cmp_pv_scores": (20, 145.0),
                                    "attn_cmp_lse": (20, 65.0), "attn_window": (20, 64.0),
                                    "topn_kernel": (20, 7.0)}
    import sparse_attention_long_phi_b200 as pkg
    monkeypatch.setattr(pkg, "nsa", fake, raising=False)
    monkeypatch.setitem(sys.modules, "sparse_attention_long_phi_b200.nsa", fake)
    monkeypatch.setattr(I, "make_forward_inputs", inputs or
                        (lambda c, dev, with_dout=False: {k: torch.zeros(1) for k in
                                                          ("q", "k", "v", "gates", "wk", "ek", "wv", "ev")}))
    records = list(clock_records)

    def stop(self):
        calls["regions"] += 1
        return records.pop(0)
    monkeypatch.setattr(bench.ClockSampler, "__init__", lambda self, dev: None)
    monkeypatch.setattr(bench.ClockSampler, "start", lambda self: None)
    monkeypatch.setattr(bench.ClockSampler, "stop", stop)
    monkeypatch.setattr(sys, "argv", ["bench.py"] + argv)
    out = io.StringIO()
    with contextlib.redirect_stdout(out):
        bench.main()
    return json.loads(out.getvalue().strip().splitlines()[-1]), calls


CLEAN = {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": [], "samples": 10}


def test_line_has_the_contract_keys(monkeypatch):
    line, calls = _run(monkeypatch, [CLEAN], ["--no-extras", "--steps", "20", "--warmup", "5"])
    assert calls == {"forward": 25, "regions": 1}
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "roofline", "clocks", "gpu_launches"):
        assert key in line, key
    assert line["steps"] == 20 and line["warmup"] == 5 and line["n_gpus"] == 1
    assert line["ms_per_step"] == pytest.approx(33.0)
    assert line["value"] == pytest.approx(65536 / 0.033, rel=1e-4)
    assert line["scaling"] == "weak" and line["higher_is_better"] is True
    assert line["config"]["workload"] == "prefill_fwd_T65536"
    roof = line["roofline"]
    assert roof["kernel"] == "attn_sel_kernel" and roof["bound"] == "tensor" and roof["unit"] == "TFLOP/s"
    assert roof["frac"] == pytest.approx(roof["achieved"] / roof["peak"], rel=1e-3)
    assert line["gpu_launches"] == 100
    assert "remeasured_after" not in line["clocks"]


def test_throttled_region_is_measured_again(monkeypatch):
    hot = dict(CLEAN, reasons=["hw_thermal_slowdown"])
    line, calls = _run(monkeypatch, [hot, CLEAN], ["--no-extras", "--steps", "20", "--warmup", "5"])
    assert calls == {"forward": 45, "regions": 2}
    assert line["clocks"]["reasons"] == [] and line["clocks"]["remeasured_after"]["reasons"] == [
        "hw_thermal_slowdown"]


def test_warmup_below_three_is_refused(monkeypatch):
    with pytest.raises(AssertionError):
        _run(monkeypatch, [CLEAN], ["--no-extras", "--steps", "20", "--warmup", "2"])


def test_reference_arm_runs_on_rank_zero_only(monkeypatch):
    # under torchrun every rank but 0 leaves at once, without work or output
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setattr(sys, "argv", ["bench.py", "--impl", "reference", "--steps", "2", "--warmup", "3"])
    monkeypatch.setattr(I, "make_forward_inputs", lambda *a, **k: pytest.fail("rank 1 did work"))
    out = io.StringIO()
    with contextlib.redirect_stdout(out):
        bench.main()
    assert out.getvalue() == ""


def test_roofline_reports_burst_and_sustained(monkeypatch):
    line, _ = _run(monkeypatch, [CLEAN], ["--no-extras", "--steps", "20", "--warmup", "5"])
    roof = line["roofline"]
    peaks, _ = bench.load_peaks()
    assert roof["peak"] == peaks.get("bf16_tflops", bench.FALLBACK_PEAKS["bf16_tflops"])
    assert roof["frac_sustained"] == pytest.approx(roof["achieved"] / roof["peak_sustained"], rel=1e-3)
    assert roof["frac_sustained"] > roof["frac"]


def test_group_sharding_is_strong_scaling_over_one_sequence(monkeypatch):
    # rank 1 of 2 takes groups [2, 4) of the one sequence; the job's tokens per step are
    # the sequence's, counted once, over the slowest rank's time
    monkeypatch.setenv("RANK", "0")
    monkeypatch.setenv("WORLD_SIZE", "1")
    shapes = {"q": (1, 2, 64, 1), "gates": (1, 2, 64, 3), "k": (1, 2, 4, 1), "v": (1, 2, 4, 1),
              "wk": (1,), "ek": (1,), "wv": (1,), "ev": (1,)}
    line, _ = _run(monkeypatch, [CLEAN], ["--no-extras", "--steps", "20", "--warmup", "5",
                                          "--shard", "groups"],
                   inputs=lambda c, dev, with_dout=False: {k: torch.zeros(v) for k, v in shapes.items()})
    assert line["scaling"] == "strong"
    assert line["value"] == pytest.approx(65536 / 0.033, rel=1e-4)
    assert bench.strong_scaling_value(65536, 20, 660.0) == pytest.approx(65536 * 20 / 0.66)
    from sparse_attention_long_phi_b200 import shard
    assert shard.group_range(4, 1, 2) == (2, 4) and shard.group_range(4, 3, 4) == (3, 4)
