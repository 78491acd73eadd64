"""The reference arm of bench.py (the fp64 oracle timed on the host cores) on
a tiny configuration: it prints one JSON line with the keys, metric, unit and
direction of the GPU arm's line and its own cpu_baseline and e2e objects.
Under torchrun only rank 0 works and prints.  No GPU involved."""
import argparse
import json

import bench
import workloads as W

TINY = W.Prefill("ring_bf16_causal_zigzag_tiny_B1_Hq2_Hkv1_S512_D64_P2", "bf16", True, "zigzag", 1, 2, 1, 512, 64,
                 2, 3)


def _args(**kw):
    a = dict(warmup=3, steps=2, cpu_seconds=0.4)
    a.update(kw)
    return argparse.Namespace(**a)


def test_reference_line(monkeypatch, capsys):
    monkeypatch.setattr(bench.W, "CFG4", TINY)
    monkeypatch.delenv("RANK", raising=False)
    monkeypatch.delenv("WORLD_SIZE", raising=False)
    bench.run_reference(_args())
    out = capsys.readouterr().out.strip().splitlines()
    assert len(out) == 1
    line = json.loads(out[0])
    assert line["impl"] == "reference"
    assert line["metric"] == "causal-adjusted attention TFLOP/s at S=128k (1 GPU); split-KV decode GB/s"
    assert line["unit"] == "TFLOP/s" and line["higher_is_better"] is True and line["vs_baseline"] is None
    assert line["n_gpus"] == 1 and line["steps"] == 2 and line["warmup"] == 3 and line["ms_per_step"] > 0
    assert line["value"] > 0 and line["dtype"] == "f64" and line["scaling"] == "weak"
    assert line["config"]["workload"] == TINY.name and line["config"]["S"] == 512
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == line["value"] and cb["cores"] >= 1 and cb["sample"]
    e2e = line["e2e"]
    assert e2e == {"value": line["value"], "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_reference_other_ranks_print_nothing(monkeypatch, capsys):
    monkeypatch.setattr(bench.W, "CFG4", TINY)
    monkeypatch.setenv("RANK", "1")
    bench.run_reference(_args())
    assert capsys.readouterr().out == ""
