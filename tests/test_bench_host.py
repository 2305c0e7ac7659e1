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


def _count_from_weight_table(g, batch, tok, K, used):
    """Bytes and GEMM FLOPs of one call, counted matrix by matrix from the
    weight table.  Every step streams each bf16 weight matrix that the loop
    multiplies by (category matrices once per used category): all block
    matrices except the cross layers' K/V projections (applied once per call to
    the valid backbone tokens), the action encoder with only the action half
    of W2 (its timestep half is a per-K table), proj_out and the decoder.  Once
    per call: the cross K/V weights and the state encoder.  Plus the valid
    backbone tokens, the K/V cache written once and read every step, and the
    f32 noise, output and state.  FLOPs are 2 x rows x params of every
    matrix, rows being the valid tokens (K/V), the B x N token rows (block
    matrices), B (state encoder) or the B x H action rows (the rest)."""
    shapes = synth.weight_shapes(g)
    N, H = g.action_horizon + 1, g.action_horizon
    step = once = 0
    flops = 0
    for name, shp in shapes.items():
        parts = name.split(".")
        if name.startswith("blk") and name.endswith(".w") and parts[1] in ("q", "k", "v", "o", "ff1", "ff2"):
            n = int(np.prod(shp))
            if int(parts[0][3:]) % 2 == 0 and parts[1] in ("k", "v"):
                once += n
                flops += 2 * tok * n
            else:
                step += n
                flops += K * 2 * batch * N * n
        elif name in ("act_enc.W1.W", "act_enc.W3.W", "act_dec.l1.W", "act_dec.l2.W"):
            n = int(np.prod(shp[1:]))
            step += used * n
            flops += K * 2 * batch * H * n
        elif name == "act_enc.W2.W":
            n = int(np.prod(shp[1:])) // 2
            step += used * n
            flops += K * 2 * batch * H * n
        elif name == "out.proj.w":
            n = int(np.prod(shp))
            step += n
            flops += K * 2 * batch * H * n
        elif name in ("state_enc.l1.W", "state_enc.l2.W"):
            n = int(np.prod(shp[1:]))
            once += used * n
            flops += 2 * batch * n
    kv = tok * (g.num_layers // 2) * 2 * g.hidden * 2
    io = 2 * batch * H * g.action_dim * 4 + batch * g.state_dim * 4
    nbytes = 2 * (K * step + once) + tok * g.backbone_dim * 2 + (1 + K) * kv + io
    return nbytes, flops


@pytest.mark.parametrize("name", ["latency", "tiny", "sweep256", "batched", "long_chunk"])
def test_call_work_matches_the_weight_table(name):
    w = synth.WORKLOADS[name]
    inp = synth.make_inputs(w) if name != "sweep256" else None
    B = w.batch
    tok = int(inp["vl_mask"].sum()) if inp is not None else B * w.seq
    used = len(set(inp["embodiment_id"].tolist())) if inp is not None else 32
    got = bench.call_work(w.geom, B, tok, w.num_steps, used)
    nbytes, flops = _count_from_weight_table(w.geom, B, tok, w.num_steps, used)
    assert got["bytes"] == nbytes
    assert got["gemm_flops"] == flops


def test_b1_bytes_of_the_latency_workload():
    """4 x 746.7 MB of step weights + 134.2 MB of cross K/V weights + 2.2 MB of
    state encoder + 1.2 MB of backbone tokens + the K/V cache (19.7 MB) written
    once and read 4 times."""
    w = synth.WORKLOADS["latency"]
    b = bench.b1_algorithmic_bytes(w.geom, w.seq, w.num_steps)
    assert b == 3_222_851_840
    r = bench.latency_roofline(w.geom, w.seq, w.num_steps, 4.73, 6452.8)
    assert r["frac"] == pytest.approx(b / 4.73e-3 / 1e9 / 6452.8)
    assert r["bound"] == "hbm" and r["unit"] == "GB/s"


def test_sweep256_flops_split():
    """B = 256, S = 256: the K/V projection is 2 x 65536 x 32768 x 2048 =
    8.80 TFLOP and the whole call 21.79 TFLOP of dense GEMM."""
    w = synth.WORKLOADS["sweep256"]
    got = bench.call_work(w.geom, 256, 256 * 256, 4, 32)
    assert 2 * 65536 * 32768 * 2048 == 8_796_093_022_208
    assert got["gemm_flops"] == pytest.approx(21.787e12, rel=1e-3)


def test_workload_roofline_picks_the_bound():
    peaks = (6452.8, 1676.2, 1404.4, "measured")
    work = {"bytes": 3.2e9, "gemm_flops": 2.0e13}
    r = bench.workload_roofline(work, 8, 2.0, peaks)
    assert r["bound"] == "hbm" and r["frac"] == pytest.approx(3.2e9 / 2e-3 / 1e9 / 6452.8)
    r = bench.workload_roofline(work, 32, 20.0, peaks)
    assert r["bound"] == "tensor" and r["frac"] == pytest.approx(2e13 / 20e-3 / 1e12 / 1676.2)
    assert r["frac_of_nominal"] == pytest.approx(2e13 / 20e-3 / 1e12 / 2250.0)


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
