"""Seeded synthetic inputs for the flow-matching action head.

This module is shared by the CPU oracle (``oracle/``) and by the GPU path's
tests and benchmark.  It draws numbers and lays out shapes; it holds none of
the action head's arithmetic.

Generator
---------
Every tensor is drawn from its own counter-based stream: SplitMix64 (Steele,
Lea & Flood, "Fast splittable pseudorandom number generators", OOPSLA 2014)
evaluated at counters 1, 2, 3, ... of a per-tensor seed, turned into 53-bit
uniforms, and into normals by the Box-Muller transform (Box & Muller, 1958).
The per-tensor seed mixes the base seed with the FNV-1a hash of the tensor's
name, so adding a tensor never changes another one.

Weights use base seed 0 and N(0, 0.02) (every bias included, so bias paths
are exercised); the affine LayerNorm gain is 1 + N(0, 0.02).  Inputs use base
seed 1.  The pages give the model's parameters in bf16 (GR00T-N1.7 model card
on the PhyAI "Single-GPU inference" page; "~12 GB for inference (bfloat16)"
under "Memory and computation" on the Isaac-GR00T architecture page), so the
full-size workloads draw their weights and backbone features as bf16 bit
patterns (uint16 arrays).  The tiny oracle-check workload keeps fp32.
"""

from __future__ import annotations

import math
import os
import threading
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, replace
from typing import Dict, Optional, Tuple

import numpy as np

__all__ = [
    "Geometry", "Workload", "GEOM_FULL", "GEOM_TINY", "WORKLOADS", "workload", "make_image_mask",
    "splitmix64_stream", "uniform53", "normal", "randint", "tensor_seed", "fnv1a64",
    "f32_to_bf16_bits", "bf16_bits_to_f32", "weight_shapes", "make_weights",
    "make_inputs", "make_training_inputs",
]

_GOLDEN = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)


# --------------------------------------------------------------------------
# counter-based generator
# --------------------------------------------------------------------------

def _mix64(z: np.ndarray) -> np.ndarray:
    z = (z ^ (z >> np.uint64(30))) * _M1
    z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def splitmix64_stream(seed: int, n: int, offset: int = 0) -> np.ndarray:
    """Outputs ``offset .. offset+n-1`` of the SplitMix64 stream of ``seed``."""
    with np.errstate(over="ignore"):
        ctr = np.arange(offset + 1, offset + n + 1, dtype=np.uint64)
        state = np.uint64(seed & 0xFFFFFFFFFFFFFFFF) + ctr * _GOLDEN
        return _mix64(state)


def fnv1a64(text: str) -> int:
    """64-bit FNV-1a hash of the UTF-8 bytes of `text`."""
    h = 0xCBF29CE484222325
    for byte in text.encode():
        h ^= byte
        h = (h * 0x100000001B3) & 0xFFFFFFFFFFFFFFFF
    return h


def tensor_seed(base_seed: int, name: str) -> int:
    """Per-tensor seed: SplitMix64 finaliser of (base * golden) xor FNV-1a(name)."""
    h = fnv1a64(name)
    with np.errstate(over="ignore"):
        z = (np.uint64(base_seed & 0xFFFFFFFFFFFFFFFF) * _GOLDEN) ^ np.uint64(h)
        return int(_mix64(np.array([z], dtype=np.uint64))[0])


def uniform53(seed: int, n: int) -> np.ndarray:
    """n uniforms in [0, 1) with 53 random bits each."""
    return (splitmix64_stream(seed, n) >> np.uint64(11)).astype(np.float64) * (2.0 ** -53)


def _normal_pairs(seed: int, first_pair: int, m: int) -> np.ndarray:
    bits = splitmix64_stream(seed, 2 * m, offset=2 * first_pair) >> np.uint64(11)
    u1 = (bits[0::2].astype(np.float64) + 1.0) * (2.0 ** -53)   # (0, 1]
    u2 = bits[1::2].astype(np.float64) * (2.0 ** -53)           # [0, 1)
    r = np.sqrt(-2.0 * np.log(u1))
    ang = 2.0 * math.pi * u2
    z = np.empty(2 * m, dtype=np.float64)
    z[0::2] = r * np.cos(ang)
    z[1::2] = r * np.sin(ang)
    return z


def _parallel_ok() -> bool:
    return threading.current_thread() is threading.main_thread()


def _threads() -> int:
    return max(1, min(16, os.cpu_count() or 1))


def normal(seed: int, n: int, std: float = 1.0, mean: float = 0.0,
           chunk: int = 1 << 21) -> np.ndarray:
    """n normals (float64) by Box-Muller on consecutive uniform pairs.

    Pair j uses stream outputs 2j and 2j+1; chunks are drawn on worker threads,
    which does not change any value."""
    out = np.empty(n, dtype=np.float64)
    npairs = (n + 1) // 2
    starts = list(range(0, npairs, chunk))

    def work(p0: int) -> None:
        m = min(chunk, npairs - p0)
        z = _normal_pairs(seed, p0, m)
        lo = 2 * p0
        hi = min(n, lo + 2 * m)
        out[lo:hi] = z[: hi - lo] * std + mean

    if len(starts) == 1 or not _parallel_ok():
        for p0 in starts:
            work(p0)
    else:
        with ThreadPoolExecutor(_threads()) as ex:
            list(ex.map(work, starts))
    return out


def randint(seed: int, n: int, low: int, high: int) -> np.ndarray:
    """n integers uniform in [low, high] (inclusive), as int64."""
    u = uniform53(seed, n)
    return (low + np.floor(u * (high - low + 1))).astype(np.int64)


# --------------------------------------------------------------------------
# bf16 bit patterns (round to nearest even)
# --------------------------------------------------------------------------

def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bf16 (ties to even); uint16 bits."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    lsb = (b >> np.uint32(16)) & np.uint32(1)
    r = (b + np.uint32(0x7FFF) + lsb) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


# --------------------------------------------------------------------------
# geometry and workloads
# --------------------------------------------------------------------------

@dataclass(frozen=True)
class Geometry:
    num_layers: int = 32
    hidden: int = 1024
    num_heads: int = 16
    head_dim: int = 64
    mlp_hidden: int = 4096
    backbone_dim: int = 2048
    action_dim: int = 32
    state_dim: int = 64
    action_horizon: int = 16
    num_embodiments: int = 32
    time_freq_dim: int = 256
    num_timestep_buckets: int = 1000
    ln_eps: float = 1e-5
    weight_dtype: str = "bf16"      # "bf16" -> uint16 bit patterns, "f32" -> float32
    attend_text_every_n_blocks: int = 0   # 0: every cross layer attends to all valid tokens
    vlln: bool = False              # vision-language LayerNorm (vlln.g, vlln.b) on the backbone features


GEOM_FULL = Geometry()
GEOM_TINY = Geometry(num_layers=2, hidden=128, num_heads=4, head_dim=32, mlp_hidden=512,
                     backbone_dim=256, num_embodiments=2, weight_dtype="f32")


@dataclass(frozen=True)
class Workload:
    name: str
    geom: Geometry
    batch: int
    seq: int                      # padded backbone length S
    num_steps: int                # Euler steps K
    valid_min: Optional[int] = None   # None: every token valid; else Sv ~ U{valid_min..seq}
    id_low: int = 0
    id_high: int = 0              # embodiment ids ~ U{id_low..id_high}
    fixed_ids: Optional[Tuple[int, ...]] = None
    feature_dtype: str = "bf16"
    description: str = ""


WORKLOADS: Dict[str, Workload] = {
    "tiny": Workload("tiny", GEOM_TINY, batch=1, seq=64, num_steps=4, fixed_ids=(0,),
                     feature_dtype="f32",
                     description="2-layer hidden-128 DiT, B=1, backbone [1,64,256] all valid, K=4"),
    "latency": Workload("latency", GEOM_FULL, batch=1, seq=300, num_steps=4, fixed_ids=(0,),
                        description="32-layer DiT, B=1, backbone [1,300,2048] all valid, id 0, K=4"),
    "batched": Workload("batched", GEOM_FULL, batch=32, seq=600, num_steps=4, valid_min=200,
                        id_low=0, id_high=31,
                        description="B=32, Sv~U{200..600} padded to 600, ids~U{0..31}, K=4"),
    "long_chunk": Workload("long_chunk", replace(GEOM_FULL, action_horizon=50), batch=8, seq=512,
                           num_steps=8, id_low=0, id_high=7,
                           description="B=8, H=50, backbone [8,512,2048] all valid, ids~U{0..7}, K=8"),
    "sweep256": Workload("sweep256", GEOM_FULL, batch=256, seq=256, num_steps=4, id_low=0, id_high=31,
                         description="B=256, S=256 all valid, ids~U{0..31}, K=4"),
}
for _b in (1, 2, 4, 8, 32, 128):
    WORKLOADS[f"sweep{_b}"] = Workload(
        f"sweep{_b}", GEOM_FULL, batch=_b, seq=256, num_steps=4, id_low=0, id_high=31,
        fixed_ids=(0,) if _b == 1 else None,
        description=f"B={_b}, S=256 all valid, ids~U{{0..31}}, K=4")


def workload(name: str, **overrides) -> Workload:
    return replace(WORKLOADS[name], **overrides)


# --------------------------------------------------------------------------
# weights
# --------------------------------------------------------------------------

def weight_shapes(g: Geometry) -> Dict[str, Tuple[int, ...]]:
    """Canonical weight table.

    Plain linears are PyTorch-style ``[out, in]`` (y = x W^T + b).  The
    per-embodiment (CategorySpecificLinear) weights keep the pages' layout
    ``W [C, in, out]``, ``b [C, out]`` (y = x W[c] + b[c]).
    """
    D, F, C = g.hidden, g.mlp_hidden, g.num_embodiments
    s: Dict[str, Tuple[int, ...]] = {
        "t_enc.l1.w": (D, g.time_freq_dim), "t_enc.l1.b": (D,),
        "t_enc.l2.w": (D, D), "t_enc.l2.b": (D,),
    }
    for l in range(g.num_layers):
        din = g.backbone_dim if l % 2 == 0 else D
        p = f"blk{l}."
        s.update({
            p + "ada.w": (2 * D, D), p + "ada.b": (2 * D,),
            p + "q.w": (D, D), p + "q.b": (D,),
            p + "k.w": (D, din), p + "k.b": (D,),
            p + "v.w": (D, din), p + "v.b": (D,),
            p + "o.w": (D, D), p + "o.b": (D,),
            p + "ln3.g": (D,), p + "ln3.b": (D,),
            p + "ff1.w": (F, D), p + "ff1.b": (F,),
            p + "ff2.w": (D, F), p + "ff2.b": (D,),
        })
    s.update({
        "out.ada.w": (2 * D, D), "out.ada.b": (2 * D,),
        "out.proj.w": (D, D), "out.proj.b": (D,),
        "state_enc.l1.W": (C, g.state_dim, D), "state_enc.l1.b": (C, D),
        "state_enc.l2.W": (C, D, D), "state_enc.l2.b": (C, D),
        "act_enc.W1.W": (C, g.action_dim, D), "act_enc.W1.b": (C, D),
        "act_enc.W2.W": (C, 2 * D, D), "act_enc.W2.b": (C, D),
        "act_enc.W3.W": (C, D, D), "act_enc.W3.b": (C, D),
        "act_dec.l1.W": (C, D, D), "act_dec.l1.b": (C, D),
        "act_dec.l2.W": (C, D, g.action_dim), "act_dec.l2.b": (C, g.action_dim),
    })
    if g.vlln:
        s["vlln.g"] = (g.backbone_dim,)
        s["vlln.b"] = (g.backbone_dim,)
    return s


def _draw(name: str, shape, base_seed: int, dtype: str, mean: float = 0.0, std: float = 0.02):
    n = int(np.prod(shape))
    v = normal(tensor_seed(base_seed, name), n, std=std, mean=mean).astype(np.float32).reshape(shape)
    return f32_to_bf16_bits(v) if dtype == "bf16" else v


def make_weights(g: Geometry, seed: int = 0) -> Dict[str, np.ndarray]:
    """All weights, N(0, 0.02); LayerNorm gains 1 + N(0, 0.02).

    bf16 geometries return uint16 bf16 bit patterns, fp32 ones float32.  Tensors
    are drawn on worker threads; each has its own stream, so values do not
    depend on the order."""
    shapes = weight_shapes(g)

    def work(name: str):
        mean = 1.0 if name.endswith("ln3.g") or name == "vlln.g" else 0.0
        return name, _draw(name, shapes[name], seed, g.weight_dtype, mean=mean)

    with ThreadPoolExecutor(_threads()) as ex:
        drawn = dict(ex.map(work, list(shapes)))
    return {name: drawn[name] for name in shapes}


# --------------------------------------------------------------------------
# per-call inputs
# --------------------------------------------------------------------------

def make_image_mask(w: Workload, seed: int = 1, batch: Optional[int] = None) -> np.ndarray:
    """image_mask [B,S] uint8 (1 = image token) for the image/text split of the
    cross layers: sample b's first n_b backbone tokens are image tokens, n_b
    uniform in 0..S (image tokens lead a VLM prompt; padding positions may be
    marked too and must not matter)."""
    B = w.batch if batch is None else batch
    n = randint(tensor_seed(seed, "image_len"), B, 0, w.seq)
    m = np.zeros((B, w.seq), dtype=np.uint8)
    for b in range(B):
        m[b, : n[b]] = 1
    return m


def make_inputs(w: Workload, seed: int = 1, batch: Optional[int] = None) -> Dict[str, np.ndarray]:
    """Inputs of one get_action call.

    backbone_features [B,S,Dvl] (uint16 bf16 bits or float32), vl_mask [B,S] uint8
    (1 = valid, a valid prefix of length Sv_b; padding holds N(0,1) values that must
    not matter), state [B,1,Sd] float32, embodiment_id [B] int32, init_noise [B,H,A]
    float32.
    """
    g = w.geom
    B = w.batch if batch is None else batch
    S, Dvl = w.seq, g.backbone_dim
    feats = normal(tensor_seed(seed, "backbone_features"), B * S * Dvl).astype(np.float32)
    feats = feats.reshape(B, S, Dvl)
    if w.feature_dtype == "bf16":
        feats = f32_to_bf16_bits(feats)
    mask = np.zeros((B, S), dtype=np.uint8)
    if w.valid_min is None:
        mask[:] = 1
    else:
        sv = randint(tensor_seed(seed, "valid_len"), B, w.valid_min, S)
        for b in range(B):
            mask[b, : sv[b]] = 1
    if w.fixed_ids is not None:
        ids = np.resize(np.asarray(w.fixed_ids, dtype=np.int32), B)
    else:
        ids = randint(tensor_seed(seed, "embodiment_id"), B, w.id_low, w.id_high).astype(np.int32)
    state = normal(tensor_seed(seed, "state"), B * g.state_dim).astype(np.float32)
    noise = normal(tensor_seed(seed, "init_noise"), B * g.action_horizon * g.action_dim)
    return {
        "backbone_features": feats,
        "vl_mask": mask,
        "state": state.reshape(B, 1, g.state_dim),
        "embodiment_id": ids,
        "init_noise": noise.astype(np.float32).reshape(B, g.action_horizon, g.action_dim),
    }


def make_training_inputs(w: Workload, seed: int = 2, batch: Optional[int] = None,
                         alpha: float = 1.5) -> Dict[str, np.ndarray]:
    """The random draws of one training step of the action head, which the
    training objective takes as inputs.

    actions [B,H,A] float32 ~ N(0, 1) (synthetic ground-truth chunks);
    noise [B,H,A] float32 ~ N(0, 1); t [B] float64 ~ Beta(alpha, 1) (the
    architecture page draws t from Beta(1.5, 1)), by inverse CDF: Beta(alpha, 1)
    has CDF x^alpha, so t = u^(1/alpha) for u uniform in [0, 1);
    action_mask [B,H,A] float32: 1 on the first a_b action dimensions of sample
    b, a_b uniform in 1..A (embodiments with fewer action dimensions are
    padded to A, and the padding is masked)."""
    g = w.geom
    B = w.batch if batch is None else batch
    H, A = g.action_horizon, g.action_dim
    n = B * H * A
    acts = normal(tensor_seed(seed, "train_actions"), n).astype(np.float32).reshape(B, H, A)
    noise = normal(tensor_seed(seed, "train_noise"), n).astype(np.float32).reshape(B, H, A)
    t = uniform53(tensor_seed(seed, "train_t"), B) ** (1.0 / alpha)
    dims = randint(tensor_seed(seed, "train_action_dims"), B, 1, A)
    mask = np.zeros((B, H, A), dtype=np.float32)
    for b in range(B):
        mask[b, :, : dims[b]] = 1.0
    return {"actions": acts, "noise": noise, "t": t, "action_mask": mask}
