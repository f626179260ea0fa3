"""The bench's JSON line, assembled on the CPU: bench.main() runs with its
GPU measurement legs replaced by stubs that return fixed figures, so that
the line's layout (the keys the benchmark contract requires, the tile-plan
figures, the CPU-baseline leg at one GPU, the decode headline) is checked
without a device.  The figures themselves are measured only on a GPU."""
import io
import json
import sys
from contextlib import redirect_stdout

import pytest
import torch

import bench

REQUIRED = {"metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
            "vs_baseline", "dtype", "data", "config", "roofline", "cpu_baseline", "e2e", "gpu_launches", "clocks"}


def _roofline():
    return {"bound": "tensor", "achieved": 1.0, "peak": 2.0, "unit": "TFLOP/s", "frac": 0.5, "traffic": 123}


@pytest.fixture
def stubbed(monkeypatch):
    def prefill(w, args, world, rank, peaks, with_e2e=True):
        out = {"ms_per_step": 1.0, "tflops": 7.0, "flops_per_step": 7e9, "roofline": _roofline(),
               "roofline_exp": {"bound": "alu"}, "gpu_launches": args.steps, "wall_s": 0.1, "eager_ms_per_step": 1.1,
               "timing": "stub"}
        if with_e2e:
            out["e2e"] = {"value": 3.0, "unit": "TFLOP/s", "h2d_bytes_per_step": 10, "d2h_bytes_per_step": 5}
        return out

    def decode(w, args, world, rank, peaks, with_e2e=True):
        return {"metric": "decode KV GB/s", "value": 6000.0, "unit": "GB/s", "ms_per_step": 0.2, "steps": 20,
                "config": {"workload": w["desc"]}, "roofline": _roofline(),
                "e2e": {"value": 5900.0, "unit": "GB/s", "h2d_bytes_per_step": 1, "d2h_bytes_per_step": 1},
                "gpu_launches": 40}

    def other(w, args, world, rank, peaks):
        return {"metric": "stub", "value": 1.0, "unit": "TFLOP/s", "roofline": _roofline()}

    class Clocks:
        def __init__(self, index):
            pass

        def __enter__(self):
            return self

        def __exit__(self, *a):
            return False

        def summary(self):
            return {"sm_mhz": 1965.0, "sm_max_mhz": 1965, "reasons": [], "samples": 1, "source": "stub"}

    real_sample = bench.oracle_prefill_sample
    monkeypatch.setattr(bench, "bench_prefill", prefill)
    monkeypatch.setattr(bench, "bench_decode", decode)
    monkeypatch.setattr(bench, "bench_backward", other)
    monkeypatch.setattr(bench, "bench_bound", other)
    monkeypatch.setattr(bench, "ClockSampler", Clocks)
    monkeypatch.setattr(bench, "oracle_prefill_sample", lambda w, seed: real_sample(w, seed, min_seconds=0.2))
    monkeypatch.setattr(bench, "oracle_decode_baseline", lambda w, seed: {"value": 1.0, "unit": "GB/s", "cores": 1,
                                                                         "kind": "oracle", "sample": "stub"})
    monkeypatch.setattr(torch.cuda, "is_available", lambda: True)
    monkeypatch.setattr(torch.cuda, "set_device", lambda i: None)
    monkeypatch.setattr(torch.cuda, "current_device", lambda: 0)


def _run(argv):
    old = sys.argv
    sys.argv = ["bench.py"] + argv
    buf = io.StringIO()
    try:
        with redirect_stdout(buf):
            bench.main()
    finally:
        sys.argv = old
    lines = [ln for ln in buf.getvalue().splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    return json.loads(lines[0])


def test_headline_line_carries_the_contract(stubbed):
    d = _run(["--steps", "4", "--warmup", "3"])
    assert REQUIRED <= set(d), REQUIRED - set(d)
    assert d["n_gpus"] == 1 and d["steps"] == 4 and d["warmup"] == 3 and d["scaling"] == "weak"
    assert d["higher_is_better"] is True and d["vs_baseline"] is None and d["data"] == "synthetic"
    assert "workload" in d["config"] and set(d["roofline"]) >= {"bound", "achieved", "peak", "unit", "frac",
                                                                 "traffic"}
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1 and d["cpu_baseline"]["value"] > 0
    assert set(d["e2e"]) >= {"value", "unit", "h2d_bytes_per_step", "d2h_bytes_per_step"}
    assert d["plan"]["q_tiles"] == 8 and d["plan"]["partial_visits"] == 8
    for extra in ("decode", "backward", "bound", "long", "frame"):
        assert extra in d
    assert d["frame"]["plan"]["partial_visits"] == 0


def test_warmup_below_three_is_raised_to_three(stubbed):
    d = _run(["--steps", "2", "--warmup", "1", "--no-extra", "--no-cpu-baseline"])
    assert d["warmup"] == 3 and d["cpu_baseline"] is None and "decode" not in d


def test_decode_headline_line(stubbed):
    d = _run(["--workload", "decode", "--steps", "4", "--warmup", "3"])
    assert REQUIRED <= set(d), REQUIRED - set(d)
    assert d["metric"] == "decode KV GB/s" and d["unit"] == "GB/s" and d["cpu_baseline"]["kind"] == "oracle"
