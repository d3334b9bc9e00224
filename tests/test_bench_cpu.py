"""The bench's reference arm: the fp64 oracle timed on host cores, and the JSON line it
prints.  Run here on a small prefill workload so that it takes seconds; the arm itself and
the line's fields are the ones `bench.py --impl reference` uses."""
import json
import types

import torch

import bench
from gated_linear_attention_liger_b200 import inputs

REQUIRED = ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
            "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e")


def small_prefill():
    return inputs.small("bench_reference_small", B=2, Hq=4, Hkv=2, T=256, d=64, dtype=torch.bfloat16, seed=3)


def test_reference_arm_prints_one_contract_line(monkeypatch, capsys):
    wl = small_prefill()
    monkeypatch.setattr(bench, "PREFILL", wl)
    sample = bench.oracle_prefill_sample
    monkeypatch.setattr(bench, "oracle_prefill_sample", lambda target_s: sample(0.2))
    bench.run_reference(types.SimpleNamespace(gpus=1, steps=2, warmup=1), 1, 0)
    out = capsys.readouterr().out.strip().splitlines()
    assert len(out) == 1
    line = json.loads(out[0])
    for key in REQUIRED:
        assert key in line, key
    assert line["impl"] == "reference"
    assert line["unit"] == "tokens/s" and line["higher_is_better"] is True
    assert line["dtype"] == "f64" and line["value"] > 0
    assert abs(line["ms_per_step"] - wl.tokens / line["value"] * 1e3) <= 1e-9 * line["ms_per_step"]
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == line["value"] and cb["cores"] >= 1
    assert isinstance(cb["cpu_model"], str) and cb["cpu_model"]
    assert f"all {wl.B} sequences x {wl.Hq} q heads" in cb["sample"]
    assert line["e2e"] == {"value": line["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}
    assert line["config"]["prefill"]["T"] == wl.T


def test_reference_arm_runs_on_rank_zero_only(capsys):
    bench.run_reference(types.SimpleNamespace(gpus=2, steps=1, warmup=0), 2, 1)
    assert capsys.readouterr().out == ""


def test_oracle_sample_covers_whole_small_workload():
    """A workload the oracle finishes within the target is run whole, repeated."""
    wl = small_prefill()
    old = bench.PREFILL
    bench.PREFILL = wl
    try:
        tps, secs, desc, nthr = bench.oracle_prefill_sample(0.2)
    finally:
        bench.PREFILL = old
    assert tps > 0 and secs >= 0.2 and nthr >= 1
    assert f"first {wl.T} of {wl.T} tokens" in desc


def test_algorithmic_work_matches_the_stated_figures():
    """The roofline numerators: 339.7 MB and 47.4 GFLOP per Llama-3-8B prefill call, 286.8 MB per
    decode step at B = 64 (state 268.4, ring 16.8, q/k/v/out and the ring slot 1.6)."""
    b, f = bench.prefill_algorithmic()
    assert abs(b / 1e6 - 339.7) < 0.05 and abs(f / 1e9 - 47.4) < 0.05
    assert abs(bench.decode_algorithmic() / 1e6 - 286.8) < 0.05
    shared = bench.decode_algorithmic(bench.DECODE_KV, kvshared=True)
    wl = bench.DECODE_KV
    assert shared == (wl.B * wl.Hkv * wl.d * wl.d * 8 + wl.B * wl.Hkv * 2 * (wl.w + 1) * wl.d * 2
                      + wl.B * (2 * wl.Hq + 2 * wl.Hkv) * wl.d * 2)
