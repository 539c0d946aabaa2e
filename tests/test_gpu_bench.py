"""Bench smoke: every workload runs through bench.py's own code path once, at
a reduced batch and a few steps, and its JSON line carries every field the
measurement contract needs (the numbers themselves are not checked here)."""
from __future__ import annotations

import argparse
import importlib.util
import json
import os

import pytest
import torch

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    assert torch.cuda.is_available()
    return mod


def _args(**kw):
    base = dict(gpus=1, steps=3, warmup=3, workload="llama7b", impl="ours", partition=0, batch=None,
                no_cpu_baseline=True, op="decode", no_other_workloads=True)
    base.update(kw)
    return argparse.Namespace(**base)


def _line(capsys):
    lines = [l for l in capsys.readouterr().out.splitlines() if l.startswith("{")]
    assert len(lines) == 1, lines
    return json.loads(lines[0])


@pytest.mark.parametrize("workload,batch", [("tiny", None), ("llama7b", 8), ("gqa", 16), ("cow", 16),
                                            ("long16", 1), ("long32", 1)])
def test_decode_bench_line_has_the_contract_fields(bench, capsys, workload, batch):
    bench.run_ours(_args(workload=workload, batch=batch))
    d = _line(capsys)
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "roofline", "e2e", "gpu_launches", "clocks",
                "cpu_baseline", "paging_overhead", "tokens_per_s", "cache_part"):
        assert key in d, key
    assert d["value"] > 0 and d["ms_per_step"] > 0 and d["n_gpus"] == 1 and d["steps"] == 3
    assert d["unit"] == "GB/s" and d["higher_is_better"] is True and d["scaling"] == "weak"
    assert d["dtype"] == ("f32" if workload == "tiny" else "bf16")
    assert d["config"]["workload"] and d["config"]["kv_bytes_per_step"] > 0
    r = d["roofline"]
    assert r["bound"] == "hbm" and r["unit"] == "GB/s" and r["achieved"] > 0 and r["peak"] > 0
    assert abs(r["frac"] - r["achieved"] / r["peak"]) < 1e-9
    assert r["traffic"] is None  # the committed traffic record is for the full-size batches
    e = d["e2e"]
    assert e["value"] > 0 and e["h2d_bytes_per_step"] > 0 and e["d2h_bytes_per_step"] > 0
    assert d["gpu_launches"] >= 2 * d["steps"]
    assert d["cache_part"]["ms"] > 0 and d["cache_part"]["bytes"] > 0
    assert {"sm_mhz", "sm_max_mhz", "reasons"} <= set(d["clocks"])
    for k in ("step_ms", "decode_attention_ms"):
        st = d[k]
        assert st["p10"] <= st["median"] <= st["p90"] and st["n"] >= 3
    assert d["decode_attention_ms"]["n"] >= 100
    assert r["read_ceiling_gbs"] > 0 and abs(r["frac_of_read_ceiling"] - r["achieved"] / r["read_ceiling_gbs"]) < 1e-9
    assert e["device_ms_per_step"] > 0 and e["ms_stats"]["n"] == d["steps"]
    assert d["other_workloads"] is None
    if workload == "cow":
        assert d["unique_kv"]["bytes_per_step"] < d["config"]["kv_bytes_per_step"]
    else:
        assert d["unique_kv"] is None


def test_default_run_times_the_other_workloads(bench, capsys):
    """The driver's default run (Llama-7B-shaped headline) also times the
    GQA, long-context and shared-prefix decode calls in the same line."""
    bench.run_ours(_args(steps=3, warmup=3, no_other_workloads=False))
    d = _line(capsys)
    o = d["other_workloads"]
    for name in ("gqa", "long16", "cow"):
        assert o[name]["gbs"] > 0 and o[name]["decode_ms"]["n"] >= 100, name
        assert abs(o[name]["frac"] - o[name]["gbs"] / d["roofline"]["peak"]) < 1e-9
    assert o["cow"]["unique_kv"]["bytes"] < o["cow"]["kv_bytes"]
    assert "unique_kv" not in o["gqa"]


def test_prefill_bench_line(bench, capsys):
    bench.run_prefill(_args(op="prefill", steps=2))
    d = _line(capsys)
    assert d["unit"] == "TFLOP/s" and d["value"] > 0
    r = d["roofline"]
    assert r["bound"] == "tensor" and abs(r["frac"] - r["achieved"] / r["peak"]) < 1e-9
    assert d["cpu_baseline"] is None  # skipped with --no-cpu-baseline


def test_blocks_bench_line(bench, capsys):
    bench.run_blocks(_args(op="blocks", steps=2, warmup=1))
    d = _line(capsys)
    assert d["unit"] == "GB/s" and d["value"] > 0 and d["roofline"]["bound"] == "hbm"
    assert d["swap_out"]["gbs"] > 0 and d["swap_in"]["gbs"] > 0
    assert d["host_link"]["d2h_gbs"] > 0 and d["host_link"]["h2d_gbs"] > 0
