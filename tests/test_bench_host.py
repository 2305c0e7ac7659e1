"""Host-side accounting of bench.py (CPU only): the B = 1 roofline's
algorithmic bytes, counted a second way from the weight table's shapes."""

import os
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402
import synth  # noqa: E402


def _bytes_from_weight_table(g, seq, K):
    """Every step streams each bf16 weight matrix that the loop multiplies by,
    for one category: all block matrices except the cross layers' K/V
    projections (applied once per call to the backbone), the action encoder
    with only the action half of W2 (its timestep half is a per-K table),
    proj_out and the decoder.  Plus the cross layers' K/V cache reads."""
    shapes = synth.weight_shapes(g)
    n = 0
    for name, shp in shapes.items():
        parts = name.split(".")
        if name.startswith("blk") and name.endswith(".w") and parts[1] in ("q", "k", "v", "o", "ff1", "ff2"):
            layer = int(parts[0][3:])
            if layer % 2 == 0 and parts[1] in ("k", "v"):
                continue
            n += int(np.prod(shp))
        elif name in ("act_enc.W1.W", "act_enc.W3.W", "act_dec.l1.W", "act_dec.l2.W"):
            n += int(np.prod(shp[1:]))
        elif name == "act_enc.W2.W":
            n += int(np.prod(shp[1:])) // 2
        elif name == "out.proj.w":
            n += int(np.prod(shp))
    kv = (g.num_layers // 2) * 2 * seq * g.hidden * 2
    return K * (2 * n + kv)


@pytest.mark.parametrize("name", ["latency", "tiny"])
def test_b1_algorithmic_bytes_match_the_weight_table(name):
    w = synth.WORKLOADS[name]
    assert bench.b1_algorithmic_bytes(w.geom, w.seq, w.num_steps) == _bytes_from_weight_table(w.geom, w.seq, w.num_steps)


def test_b1_bytes_of_the_latency_workload():
    w = synth.WORKLOADS["latency"]
    b = bench.b1_algorithmic_bytes(w.geom, w.seq, w.num_steps)
    assert b == 3_065_511_936            # 4 x (746.7 MB weights + 19.7 MB K/V)
    r = bench.latency_roofline(w.geom, w.seq, w.num_steps, 4.73, 6452.8)
    assert r["frac"] == pytest.approx(b / 4.73e-3 / 1e9 / 6452.8)
    assert r["bound"] == "hbm" and r["unit"] == "GB/s"


def test_reference_arm_prints_one_complete_line(monkeypatch, capsys):
    """`bench.py --impl reference` times the oracle and prints one JSON line
    with the contract's keys (run here on the tiny workload)."""
    import argparse
    import json
    monkeypatch.setattr(bench, "THROUGHPUT", "tiny")
    args = argparse.Namespace(gpus=1, steps=2, warmup=1)
    bench.run_reference(args, rank=0)
    lines = [l for l in capsys.readouterr().out.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["value"] > 0 and d["unit"] == bench.UNIT
    assert d["metric"] == bench.METRIC and d["higher_is_better"] is True
    # the same workload description as our arm's line
    assert d["config"] == bench.throughput_config(synth.WORKLOADS["tiny"], 1)
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    bench.run_reference(args, rank=1)                     # other ranks print nothing
    assert capsys.readouterr().out.strip() == ""
