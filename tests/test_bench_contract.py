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
    # figures with as many digits as measured ones, so that the line's length is realistic
    return {"bound": "tensor", "achieved": 1123.456789, "peak": 1640.7, "unit": "TFLOP/s", "frac": 0.684712345,
            "traffic": 441834752}


@pytest.fixture
def stubbed(monkeypatch):
    def prefill(w, args, world, rank, peaks, with_e2e=True):
        out = {"ms_per_step": 1.0, "ms_median": 0.99, "tflops": 7.0, "flops_per_step": 7e9,
               "roofline": dict(_roofline(), peak_source="stub"),
               "roofline_exp": {"bound": "alu"}, "gpu_launches": args.steps, "wall_s": 0.1, "eager_ms_per_step": 1.1,
               "timing": "stub"}
        if with_e2e:
            out["e2e"] = {"value": 345.678912, "unit": "TFLOP/s", "h2d_bytes_per_step": 201326592,
                          "d2h_bytes_per_step": 136314880}
        return out

    def decode(w, args, world, rank, peaks, with_e2e=True):
        return {"metric": "decode KV GB/s", "value": 6000.0, "unit": "GB/s", "ms_per_step": 0.2, "ms_median": 0.2,
                "steps": 20, "config": {"workload": w["desc"]}, "roofline": dict(_roofline(), peak_source="stub"),
                "e2e": {"value": 5912.345678, "unit": "GB/s", "h2d_bytes_per_step": 524288,
                        "d2h_bytes_per_step": 532480},
                "gpu_launches": 40, "multi_token_2": {"value": 5900.0, "unit": "GB/s", "ms_per_step": 0.21}}

    def other(w, args, world, rank, peaks):
        return {"metric": "stub", "value": 1.0, "unit": "TFLOP/s", "ms_per_step": 0.1, "ms_median": 0.1,
                "key_stats_ms": 0.03, "roofline": dict(_roofline(), executed_frac=0.7)}

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
    monkeypatch.setattr(bench, "oracle_prefill_sample",
                        lambda w, seed, min_seconds=0: real_sample(w, seed, min_seconds=0.05, max_passes=1))
    monkeypatch.setattr(bench, "oracle_decode_baseline", lambda w, seed: {"value": 1.0, "unit": "GB/s", "cores": 1,
                                                                         "kind": "oracle", "sample": "stub",
                                                                         "cpu": "stub"})
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
    return json.loads(lines[0]), lines[0]


def test_headline_line_carries_the_contract(stubbed):
    d, raw = _run(["--steps", "4", "--warmup", "3"])
    assert REQUIRED <= set(d), REQUIRED - set(d)
    assert d["n_gpus"] == 1 and d["steps"] == 4 and d["warmup"] == 3 and d["scaling"] == "weak"
    assert d["higher_is_better"] is True and d["vs_baseline"] is None and d["data"] == "synthetic"
    assert "N=16384" in d["config"]["workload"]  # the largest single-GPU workload is the headline
    assert set(d["roofline"]) >= {"bound", "achieved", "peak", "unit", "frac", "traffic"}
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] > 0 and cb["cpu"]
    assert set(d["e2e"]) >= {"value", "unit", "h2d_bytes_per_step", "d2h_bytes_per_step"}
    assert "ms_median" in d
    # every other workload: its roofline fraction, the oracle's rate and the end-to-end rate
    for name in ("gpt2", "frame", "decode"):
        x = d[name]
        assert set(x["roofline"]) >= {"bound", "achieved", "peak", "unit", "frac", "traffic"}, name
        assert x["cpu_baseline"]["kind"] == "oracle" and x["cpu_baseline"]["value"] > 0, name
        assert set(x["e2e"]) >= {"value", "unit"}, name
        assert "ms" in x and "ms_median" in x
    assert "backward" in d and "bound" in d
    # the main legs close the line
    assert list(d)[-2:] == ["long", "decode"] or list(d)[-1] == "decode"
    # the whole line fits in the few KB of output a driver keeps
    assert len(raw) < 2800, len(raw)


def test_warmup_below_three_is_raised_to_three(stubbed):
    d, _ = _run(["--steps", "2", "--warmup", "1", "--no-extra", "--no-cpu-baseline"])
    assert d["warmup"] == 3 and d["cpu_baseline"] is None and "decode" not in d


def test_decode_headline_line(stubbed):
    d, raw = _run(["--workload", "decode", "--steps", "4", "--warmup", "3"])
    assert REQUIRED <= set(d), REQUIRED - set(d)
    assert d["metric"] == "decode KV GB/s" and d["unit"] == "GB/s" and d["cpu_baseline"]["kind"] == "oracle"
    assert "long" in d and "gpt2" in d and len(raw) < 2800
