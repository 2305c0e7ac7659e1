#!/usr/bin/env python
"""Benchmark of the flow-matching DiT action head (get_action) on B200.

One step = one gdit_get_action call over a batch of synthetic inputs:
B = 256 action chunks, backbone features [256, 256, 2048] bf16 (all valid),
embodiment ids uniform over 32 categories, K = 4 Euler steps, 32-layer DiT
(hidden 1024, 16 x 64 heads, MLP 4096), inputs resident in HBM.
value = chunks/s of the whole job (all ranks).  Also reported: p50/p99
latency of a B = 1 call (backbone [1, 300, 2048], K = 4), the dominant
kernel's roofline, an end-to-end number through the host-buffer entry point,
and the CPU oracle timed on a bounded sample.

    python bench.py [--gpus N --steps K --warmup W] [--impl reference]

For N > 1 launch with torch.distributed.run; every rank runs its own replica
on its own batch (the samples are independent: no collective on the data
path), timing is taken as the max over ranks.
"""

from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "DiT action chunks/s at B=256 and p50 get_action latency at B=1 (4 steps)"
UNIT = "chunks/s"
THROUGHPUT = "sweep256"
LATENCY = "latency"


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--latency-calls", type=int, default=200)
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-profile", action="store_true")
    p.add_argument("--no-workloads", action="store_true", help="skip the per-workload table")
    p.add_argument("--workload-calls", type=int, default=30)
    p.add_argument("--oracle-samples", type=int, default=4)
    p.add_argument("--batch", type=int, default=None, help="override the throughput batch (profiling runs)")
    p.add_argument("--seq", type=int, default=None, help="override the throughput backbone length (profiling runs)")
    return p.parse_args()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return d.get("hbm_gbs", 6650.0), d.get("bf16_tflops", 1590.0), d.get("bf16_tflops_sustained", 1400.0), "measured"
    return 6650.0, 1590.0, 1400.0, "fallback"


# ------------------------------------------------------------------ clocks

class Clocks:
    """nvidia-smi sampling during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device: int):
        self.device = device
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-lms", "200", "-i", str(self.device)],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) >= 9:
                rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        smax = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": reasons, "samples": len(rows)}


# ------------------------------------------------------------------ CPU oracle

def time_oracle(W, w, samples: int):
    """The C++ CPU oracle (its float instantiation, as it stands) on `samples`
    batch rows of workload w, on all host cores.  The weights are converted to
    float once, outside the timed region.  Returns (chunks/s, threads, s)."""
    from oracle import cpp_oracle
    inp = synth.make_inputs(w)
    prep = cpp_oracle.Weights(W, w.geom, np.float32)
    args = (W, w.geom, inp["backbone_features"], inp["vl_mask"], inp["state"], inp["embodiment_id"],
            inp["init_noise"], w.num_steps)
    rows = list(range(samples))
    t0 = time.perf_counter()
    cpp_oracle.get_action(*args, samples=rows, dtype=np.float32, prepared=prep)
    dt = time.perf_counter() - t0
    return samples / dt, cpp_oracle.max_threads(), dt


# ------------------------------------------------------------------ algorithmic work of one call

NOMINAL_BF16_TFLOPS = 2250.0   # B200 dense bf16 tensor peak (spec sheet), for context beside the measured peaks


def call_work(g, batch: int, valid_tokens: int, num_steps: int, used_categories: int) -> dict:
    """Minimum HBM bytes and dense FLOPs of one get_action call.

    Bytes: the bf16 weights each Euler step multiplies by (the 32 DiT blocks
    without the cross layers' K/V projections, proj_out, and the action
    encoder and decoder of every category used), once per step; the cross
    K/V weights and the state encoder (per used category) once per call; the
    valid backbone tokens read once; the K/V cache written once and read every
    step; x, the output and the state.  The per-K AdaLN tables and the
    timestep half of the action encoder's W2 are cached, so not counted.
    FLOPs: 2 M N K of every dense contraction over the rows that need it
    (valid tokens for the K/V projection, the B x N token rows in the blocks,
    the B x H action rows in the encoder, proj_out and decoder), plus
    attention 4 N Sv D per sample and cross layer and 4 N^2 D per sample and
    self layer."""
    D, F, A, L = g.hidden, g.mlp_hidden, g.action_dim, g.num_layers
    Dvl, Sd, H = g.backbone_dim, g.state_dim, g.action_horizon
    N = H + 1
    Lc = L // 2
    B, tok, K, C = batch, valid_tokens, num_steps, used_categories
    self_w = 3 * D * D + D * D + 2 * F * D
    cross_w = 2 * D * D + 2 * F * D
    enc_w = A * D + D * D + D * D          # W1, W2 (action half), W3
    dec_w = D * D + D * A
    step_w = Lc * (self_w + cross_w) + D * D + C * (enc_w + dec_w)
    once_w = Lc * 2 * D * Dvl + C * (Sd * D + D * D)
    kv_cache = tok * Lc * 2 * D * 2
    io = B * H * A * 4 * 2 + B * Sd * 4
    nbytes = K * step_w * 2 + once_w * 2 + tok * Dvl * 2 + kv_cache * (1 + K) + io
    rows, arows = B * N, B * H
    gemm = 2 * tok * (Lc * 2 * D) * Dvl + 2 * B * (Sd * D + D * D)
    gemm += K * (2 * rows * Lc * (self_w + cross_w) + 2 * arows * (enc_w + D * D + dec_w))
    attn = K * (Lc * 4 * N * tok * D + Lc * 4 * B * N * N * D)
    return {"bytes": int(nbytes), "gemm_flops": int(gemm), "attn_flops": int(attn), "weights_per_step": int(step_w * 2)}


def b1_algorithmic_bytes(g, seq: int, num_steps: int) -> int:
    """Minimum HBM bytes of one single-sample call (one category, `seq` valid
    backbone tokens): call_work's count."""
    return call_work(g, 1, seq, num_steps, 1)["bytes"]


def latency_roofline(g, seq: int, num_steps: int, p50_ms: float, hbm_gbs: float) -> dict:
    """HBM roofline of the B = 1 call at its p50 latency."""
    b = b1_algorithmic_bytes(g, seq, num_steps)
    ach = b / (p50_ms / 1e3) / 1e9
    return {"bound": "hbm", "algorithmic_bytes": b, "achieved": ach, "peak": hbm_gbs, "unit": "GB/s",
            "frac": ach / hbm_gbs}


def workload_roofline(work: dict, batch: int, mean_ms: float, peaks) -> dict:
    """Roofline of a whole call: weight streaming (HBM) for batches of at most
    8 samples, tensor cores (dense bf16 GEMM FLOPs) from 32 up."""
    hbm, tf_burst, tf_sus, src = peaks
    sec = mean_ms / 1e3
    if batch <= 8:
        ach = work["bytes"] / sec / 1e9
        return {"bound": "hbm", "achieved": ach, "peak": hbm, "unit": "GB/s", "frac": ach / hbm,
                "peak_kind": f"HBM copy ({src})"}
    ach = work["gemm_flops"] / sec / 1e12
    return {"bound": "tensor", "achieved": ach, "peak": tf_burst, "unit": "TFLOP/s", "frac": ach / tf_burst,
            "frac_of_sustained": ach / tf_sus, "frac_of_nominal": ach / NOMINAL_BF16_TFLOPS,
            "peak_kind": f"burst bf16 ({src})"}


# ------------------------------------------------------------------ replicas (one per GPU, no data-path collective)

def ranks_from_env():
    """(rank, world, local rank) as torchrun sets them; (0, 1, 0) without it."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def max_over_ranks(x: float, world: int, device) -> float:
    """The largest value of x over all ranks (every rank gets it).  Timings of
    the replicas are reported as their maximum: the job is as slow as its
    slowest replica."""
    if world <= 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def shard_rows(global_batch: int, rank: int, world: int):
    """Rows [start, stop) of a global batch that `rank` serves: contiguous,
    sizes differing by at most one, earlier ranks taking the extra rows."""
    base, extra = divmod(global_batch, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def gather_rows(local, global_batch: int, world: int):
    """The ranks' slices of a batch-major tensor (rows as shard_rows gives
    them) put back together on every rank: one all_gather of equal-sized,
    zero-padded slices.  Samples are independent, so this is the only
    collective the batch-sharded path needs, and it is outside the timed
    region."""
    import torch
    import torch.distributed as dist
    if world <= 1:
        return local
    cap = -(-global_batch // world)
    pad = torch.zeros((cap,) + tuple(local.shape[1:]), dtype=local.dtype, device=local.device)
    pad[: local.shape[0]] = local
    parts = [torch.empty_like(pad) for _ in range(world)]
    dist.all_gather(parts, pad)
    out = []
    for r in range(world):
        a, b = shard_rows(global_batch, r, world)
        out.append(parts[r][: b - a])
    return torch.cat(out)


def whole_job_rate(world: int, units_per_rank_step: int, steps: int, seconds: float) -> float:
    """Units per second of the whole job: every rank processed
    units_per_rank_step units in each of `steps` steps, within `seconds`."""
    return world * units_per_rank_step * steps / seconds


# ------------------------------------------------------------------ the workload both arms report

def throughput_config(w, world: int) -> dict:
    """The `config` of the JSON line, the same for our arm and the reference arm."""
    g = w.geom
    return {"workload": f"DiT action head B={w.batch} S={w.seq} K={w.num_steps} (throughput sweep)",
            "batch": w.batch, "seq": w.seq, "num_steps": w.num_steps, "layers": g.num_layers, "hidden": g.hidden,
            "embodiments": g.num_embodiments, "parallelism": f"replicas x{world}",
            "l2": "inputs larger than L2 (1.36 GB bf16 weights, 4.3 GB KV cache per call)"}


# ------------------------------------------------------------------ reference arm

def run_reference(args, rank):
    """The reference arm: the C++ CPU oracle (float instantiation, all host
    cores), one chunk of the throughput workload per step."""
    if rank != 0:
        return
    from oracle import cpp_oracle
    w = synth.WORKLOADS[THROUGHPUT]
    W = synth.make_weights(w.geom)
    inp = synth.make_inputs(w)
    prep = cpp_oracle.Weights(W, w.geom, np.float32)
    a = (W, w.geom, inp["backbone_features"], inp["vl_mask"], inp["state"], inp["embodiment_id"],
         inp["init_noise"], w.num_steps)
    times = []
    for i in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        cpp_oracle.get_action(*a, samples=[i % w.batch], dtype=np.float32, prepared=prep)
        if i >= args.warmup:
            times.append(time.perf_counter() - t0)
    per = float(np.mean(times))
    value = 1.0 / per
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": per * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": throughput_config(w, args.gpus),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cpp_oracle.max_threads(), "kind": "oracle",
                         "sample": f"1 chunk of the B={w.batch} workload per step ({args.steps} steps), "
                                   "C++ oracle, float"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ our arm

# every workload of the task, timed one call after the other (inputs resident in HBM)
WORKLOAD_TABLE = ("latency", "sweep1", "sweep2", "sweep4", "sweep8", "sweep32", "sweep128", "sweep256", "batched",
                  "long_chunk")


def time_calls(head, d, K, out, stream, calls: int, warmup: int):
    """Device time of each of `calls` consecutive calls (CUDA events on the
    launching stream between calls) and of all of them together, in ms."""
    import torch
    for _ in range(warmup):
        head.get_action(*d, num_steps=K, out=out)
    torch.cuda.synchronize()
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(calls + 1)]
    evs[0].record(stream)
    for i in range(calls):
        head.get_action(*d, num_steps=K, out=out)
        evs[i + 1].record(stream)
    torch.cuda.synchronize()
    per = [evs[i].elapsed_time(evs[i + 1]) for i in range(calls)]
    return per, evs[0].elapsed_time(evs[-1])


def main():
    args = parse()
    rank, world, local = ranks_from_env()
    if args.impl == "reference":
        return run_reference(args, rank)

    import torch
    import torch.distributed as dist
    from flow_matching_dit_b200 import ActionHead

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", device_id=dev)

    w = synth.WORKLOADS[THROUGHPUT]
    if args.batch or args.seq:
        w = synth.workload(THROUGHPUT, batch=args.batch or w.batch, seq=args.seq or w.seq)
    wl = synth.WORKLOADS[LATENCY]
    g = w.geom
    W = synth.make_weights(g)
    max_seq = max(w.seq, wl.seq) if args.latency_calls > 0 else w.seq
    if not args.no_workloads:
        max_seq = max(max_seq, max(synth.WORKLOADS[n].seq for n in WORKLOAD_TABLE if n != "long_chunk"))
    head = ActionHead(g, W, max_batch=max(w.batch, 256 if not args.no_workloads else 1), max_seq=max_seq,
                      device=local)

    def dev_inputs(wk, seed):
        inp = synth.make_inputs(wk, seed=seed)
        f = torch.from_numpy(inp["backbone_features"].view(np.int16)).to(dev).view(torch.bfloat16)
        return inp, (f, torch.from_numpy(inp["vl_mask"]).to(dev), torch.from_numpy(inp["state"]).to(dev),
                     torch.from_numpy(inp["embodiment_id"]).to(dev), torch.from_numpy(inp["init_noise"]).to(dev))

    inp, d = dev_inputs(w, 1 + rank)
    out = torch.empty_like(d[4])
    stream = torch.cuda.current_stream(dev)
    K = w.num_steps
    for _ in range(max(args.warmup, 1)):
        head.get_action(*d, num_steps=K, out=out)
    assert head.sync_status() == 0

    # ---- timed region: K steps, device-resident inputs
    clocks = Clocks(local)
    clocks.start()
    time.sleep(0.3)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for _ in range(args.steps):
        head.get_action(*d, num_steps=K, out=out)
    ev1.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clk = clocks.stop()
    ms = max_over_ranks(ev0.elapsed_time(ev1), world, dev)
    assert head.sync_status() == 0
    ms_per_step = ms / args.steps
    value = whole_job_rate(world, w.batch, args.steps, ms / 1e3)
    if world > 1:
        # the job's global batch is world x B rows, rank r serving rows
        # shard_rows(world * B, r, world); its actions are gathered once,
        # outside the timed region
        gathered = gather_rows(out, world * w.batch, world)
        assert gathered.shape[0] == world * w.batch

    # ---- B = 1 latency (device inputs, one call at a time)
    lat = None
    if rank == 0 and args.latency_calls > 0:
        _, dl = dev_inputs(wl, 7)
        outl = torch.empty_like(dl[4])
        for _ in range(20):
            head.get_action(*dl, num_steps=wl.num_steps, out=outl)
        torch.cuda.synchronize()
        ts = []
        for _ in range(args.latency_calls):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            head.get_action(*dl, num_steps=wl.num_steps, out=outl)
            b.record(stream)
            b.synchronize()
            ts.append(a.elapsed_time(b))
        ts = np.array(ts)
        lat = {"p50_ms": float(np.percentile(ts, 50)), "p99_ms": float(np.percentile(ts, 99)),
               "mean_ms": float(ts.mean()), "calls": int(len(ts)),
               "workload": "B=1, backbone [1,300,2048] bf16 all valid, id 0, K=4"}
        lat["roofline"] = latency_roofline(wl.geom, wl.seq, wl.num_steps, lat["p50_ms"], load_peaks()[0])

    # ---- every workload: chunks/s, p50/p99 per call, roofline of the whole call
    table = None
    if rank == 0 and not args.no_workloads:
        table = {}
        peaks = load_peaks()
        for name in WORKLOAD_TABLE:
            wk = synth.WORKLOADS[name]
            hw = head
            if wk.geom != g:     # another horizon: a handle of its own
                hw = ActionHead(wk.geom, W, max_batch=wk.batch, max_seq=wk.seq, device=local)
            winp, dw = dev_inputs(wk, 1)
            outw = torch.empty_like(dw[4])
            per, total_ms = time_calls(hw, dw, wk.num_steps, outw, stream, args.workload_calls, 5)
            assert hw.sync_status() == 0
            if hw is not head:
                hw.close()
            work = call_work(wk.geom, wk.batch, int(winp["vl_mask"].sum()), wk.num_steps,
                             len(set(winp["embodiment_id"].tolist())))
            mean_ms = total_ms / len(per)
            table[name] = {
                "workload": wk.description, "batch": wk.batch, "seq": wk.seq, "horizon": wk.geom.action_horizon,
                "num_steps": wk.num_steps, "chunks_per_s": wk.batch / (mean_ms / 1e3),
                "p50_ms": float(np.percentile(per, 50)), "p99_ms": float(np.percentile(per, 99)),
                "mean_ms": mean_ms, "calls": len(per), "algorithmic_bytes": work["bytes"],
                "gemm_flops": work["gemm_flops"], "attn_flops": work["attn_flops"],
                "roofline": workload_roofline(work, wk.batch, mean_ms, peaks)}

    # ---- end to end through the host-buffer entry point (pinned host memory)
    e2e = None
    if not args.no_e2e:
        pin = {k: torch.from_numpy(np.ascontiguousarray(v)).pin_memory() for k, v in inp.items()}
        hf = pin["backbone_features"].numpy()
        hout = torch.empty(d[4].shape, dtype=torch.float32).pin_memory().numpy()
        hargs = (hf, pin["vl_mask"].numpy(), pin["state"].numpy(), pin["embodiment_id"].numpy(),
                 pin["init_noise"].numpy())
        st = stream.cuda_stream
        for _ in range(2):
            head.get_action_host(*hargs, num_steps=K, out=hout, stream=st)
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        n_e2e = max(3, args.steps // 2)
        for _ in range(n_e2e):
            head.get_action_host(*hargs, num_steps=K, out=hout, stream=st)
        sec = max_over_ranks(time.perf_counter() - t0, world, dev)
        h2d = sum(int(v.nbytes) for v in hargs)
        e2e = {"value": whole_job_rate(world, w.batch, n_e2e, sec), "unit": UNIT, "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": int(hout.nbytes), "steps": n_e2e,
               "api": "gdit_get_action_host (pinned host buffers, copies and sync inside)"}

    # ---- per-kernel-class timing of one instrumented (eager) call
    roof = None
    launches_per_call = None
    kstats = None
    if rank == 0 and not args.no_profile:
        kstats = head.profile(*d, num_steps=K, out=out)
        launches_per_call = sum(k["launches"] for k in kstats) + 1    # + the pointer-setting kernel
        top = max(kstats, key=lambda k: k["total_ms"])
        hbm, tf_burst, tf_sus, src = load_peaks()
        traffic = None
        tpath = os.path.join(ROOT, "profiles", "traffic.json")
        if os.path.exists(tpath):
            traffic = json.load(open(tpath)).get(top["name"])
        if top["name"].startswith("gemm"):
            ach = top["flops"] / (top["total_ms"] / 1e3) / 1e12
            # each launch is timed on its own (events around it, one eager call of
            # about 40 ms): the burst peak is the denominator
            roof = {"bound": "tensor", "kernel": top["name"], "achieved": ach, "peak": tf_burst, "unit": "TFLOP/s",
                    "frac": ach / tf_burst, "frac_of_sustained": ach / tf_sus,
                    "frac_of_nominal": ach / NOMINAL_BF16_TFLOPS, "peak_kind": f"burst bf16 ({src})",
                    "traffic": traffic, "launches": top["launches"], "ms": top["total_ms"]}
        else:
            ach = top["bytes"] / (top["total_ms"] / 1e3) / 1e9
            roof = {"bound": "hbm", "kernel": top["name"], "achieved": ach, "peak": hbm, "unit": "GB/s",
                    "frac": ach / hbm, "peak_kind": f"HBM copy ({src})", "traffic": traffic,
                    "launches": top["launches"], "ms": top["total_ms"]}

    # ---- CPU oracle on a bounded sample
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, cores, secs = time_oracle(W, w, args.oracle_samples)
        cpu = {"value": v, "unit": UNIT, "cores": cores, "kind": "oracle",
               "sample": f"{args.oracle_samples} chunks of the B={w.batch} workload (rows 0..{args.oracle_samples - 1}), "
                         f"C++ oracle (float, OpenMP), {secs:.1f} s"}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": throughput_config(w, world),
            "latency_b1": lat, "roofline": roof, "cpu_baseline": cpu, "e2e": e2e, "workloads": table,
            "gpu_launches": (launches_per_call * args.steps) if launches_per_call else None,
            "clocks": clk,
        }
        if kstats is not None:
            line["kernel_classes"] = [{k: (round(v, 4) if isinstance(v, float) else v) for k, v in s.items()}
                                      for s in kstats]
        print(json.dumps(line), flush=True)
    head.close()
    if world > 1:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
