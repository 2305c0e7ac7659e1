"""B200 (sm_100a) flow-matching DiT action head behind a C ABI.

The compute path is ``libgdit.so`` (hand-written CUDA in ``csrc/``); this
package only marshals arguments.  PyTorch supplies device memory and streams.
``ActionHead`` wraps one ``gdit_handle``:

    head = ActionHead(geom, weights, max_batch=256, max_seq=300)
    out = head.get_action(features, vl_mask, state, embodiment_id, init_noise, num_steps=4)

``geom`` is any object with the fields of ``gdit_config`` (for example
``synth.Geometry``); ``weights`` maps the names of ``include/gdit.h`` to numpy
arrays (float32, or uint16 holding bf16 bit patterns).
"""

from __future__ import annotations

import ctypes
from typing import Dict, List, Optional

import numpy as np

from . import _lib
from ._lib import (GDIT_BF16, GDIT_F32, GDIT_FLAG_NO_GRAPH, GDIT_FLAG_NO_PAIR, GDIT_FLAG_NO_SKINNY,  # noqa: F401
                   GDIT_FLAG_NO_SMALL, GDIT_FLAG_NO_TMA_STORE, GDIT_FLAG_STRICT_PROFILES,
                   GditError, check, lib)
from .build import build  # noqa: F401

__all__ = ["ActionHead", "GditError", "lib", "build", "check_io_shapes", "is_checked", "GDIT_BF16", "GDIT_F32",
           "GDIT_FLAG_NO_GRAPH", "GDIT_FLAG_NO_SMALL", "GDIT_FLAG_STRICT_PROFILES"]


def is_checked() -> bool:
    """Whether the loaded library is the range-checked build (GDIT_CHECKED=1)."""
    return bool(_lib.gdit_is_checked())


def _ptr(t) -> int:
    return int(t.data_ptr())


def check_io_shapes(cfg, feats, mask, state, ids, noise, out, image_mask=None):
    """The library reads and writes the I/O buffers by the batch and sequence
    it is given, so every buffer must have the shape that implies (a smaller
    one would be read or written past its end).  Raises ValueError.

    feats [B, S, backbone_dim]; vl_mask and image_mask [B, S]; state
    [B, 1, state_dim] (or [B, state_dim]); embodiment_id [B];
    init_noise and out [B, action_horizon, action_dim]."""
    shp = lambda t: tuple(int(d) for d in t.shape)
    if len(shp(feats)) != 3:
        raise ValueError(f"backbone_features must be [batch, seq, {cfg.backbone_dim}], got {shp(feats)}")
    B, S, dvl = shp(feats)
    if dvl != cfg.backbone_dim:
        raise ValueError(f"backbone_features last dim {dvl} != backbone_dim {cfg.backbone_dim}")
    want = {"vl_mask": (mask, [(B, S)]),
            "state": (state, [(B, 1, cfg.state_dim), (B, cfg.state_dim)]),
            "embodiment_id": (ids, [(B,)]),
            "init_noise": (noise, [(B, cfg.action_horizon, cfg.action_dim)]),
            "out": (out, [(B, cfg.action_horizon, cfg.action_dim)])}
    if image_mask is not None:
        want["image_mask"] = (image_mask, [(B, S)])
    for name, (t, shapes) in want.items():
        if shp(t) not in shapes:
            raise ValueError(f"{name} has shape {shp(t)}, expected {' or '.join(map(str, shapes))}")
    return B, S


def make_config(geom, max_batch: int, max_seq: int, device: int = 0, flags: int = 0):
    """The gdit_config of a model geometry (any object with the config's
    geometry fields as attributes) and a capacity."""
    cfg = _lib.gdit_config()
    for name in ("num_layers", "hidden", "num_heads", "head_dim", "mlp_hidden", "backbone_dim",
                 "action_dim", "state_dim", "action_horizon", "num_embodiments", "time_freq_dim",
                 "num_timestep_buckets"):
        setattr(cfg, name, int(getattr(geom, name)))
    cfg.ln_eps = float(geom.ln_eps)
    cfg.max_batch = int(max_batch)
    cfg.max_backbone_seq = int(max_seq)
    cfg.flags = int(flags)
    cfg.device = int(device)
    cfg.attend_text_every_n_blocks = int(getattr(geom, "attend_text_every_n_blocks", 0))
    return cfg


class ActionHead:
    def __init__(self, geom, weights: Dict[str, np.ndarray], max_batch: int, max_seq: int,
                 device: int = 0, flags: int = 0):
        cfg = make_config(geom, max_batch, max_seq, device, flags)
        self.cfg = cfg
        keep = []
        arr = (_lib.gdit_tensor * len(weights))()
        for i, (name, a) in enumerate(weights.items()):
            a = np.ascontiguousarray(a)
            if a.dtype == np.uint16:
                dt = GDIT_BF16
            elif a.dtype == np.float32:
                dt = GDIT_F32
            else:
                raise TypeError(f"weight {name}: dtype {a.dtype} (need float32 or uint16 bf16 bits)")
            shape = (ctypes.c_int64 * a.ndim)(*a.shape)
            nm = name.encode()
            keep += [a, shape, nm]
            arr[i].name = nm
            arr[i].dtype = dt
            arr[i].ndim = a.ndim
            arr[i].shape = shape
            arr[i].host_ptr = a.ctypes.data
        h = ctypes.c_void_p()
        rc = _lib.gdit_create(ctypes.byref(cfg), arr, len(weights), ctypes.byref(h))
        check(rc, None)
        self.h = h
        del keep

    # ------------------------------------------------------------------ calls
    def _args(self, feats, mask, state, ids, noise, out):
        import torch
        if feats.dtype == torch.bfloat16:
            bb = GDIT_BF16
        elif feats.dtype == torch.float32:
            bb = GDIT_F32
        else:
            raise TypeError("backbone_features must be bfloat16 or float32")
        if out is None:
            out = torch.empty_like(noise)
        for t, dt in ((mask, torch.uint8), (state, torch.float32), (ids, torch.int32), (noise, torch.float32),
                      (out, torch.float32)):
            if t.dtype != dt or not t.is_contiguous() or not t.is_cuda:
                raise TypeError(f"expected a contiguous CUDA tensor of {dt}")
        if not feats.is_contiguous() or not feats.is_cuda:
            raise TypeError("backbone_features must be a contiguous CUDA tensor")
        for t in (feats, mask, state, ids, noise, out):
            if t.device.index != self.cfg.device:
                raise ValueError(f"tensor on {t.device}, the head is on cuda:{self.cfg.device}")
        B, S = check_io_shapes(self.cfg, feats, mask, state, ids, noise, out)
        return bb, B, S, out

    def get_action(self, feats, mask, state, ids, noise, num_steps: int = 4, out=None, stream=None,
                   image_mask=None):
        """Asynchronous on ``stream`` (default: torch's current stream).  ``image_mask``
        (uint8 [B, S] CUDA tensor, 1 = image token) feeds the image/text split of the
        cross layers when the geometry's attend_text_every_n_blocks > 0."""
        import torch
        bb, B, S, out = self._args(feats, mask, state, ids, noise, out)
        st = stream if stream is not None else torch.cuda.current_stream().cuda_stream
        if image_mask is None:
            check(_lib.gdit_get_action(self.h, _ptr(feats), bb, _ptr(mask), _ptr(state), _ptr(ids), _ptr(noise),
                                       int(num_steps), _ptr(out), B, S, st), self.h)
            return out
        if image_mask.dtype != torch.uint8 or not image_mask.is_contiguous() or not image_mask.is_cuda \
                or image_mask.device.index != self.cfg.device:
            raise TypeError("image_mask must be a contiguous uint8 tensor on the head's device")
        check_io_shapes(self.cfg, feats, mask, state, ids, noise, out, image_mask)
        check(_lib.gdit_get_action_vl(self.h, _ptr(feats), bb, _ptr(mask), _ptr(image_mask), _ptr(state), _ptr(ids),
                                      _ptr(noise), int(num_steps), _ptr(out), B, S, st), self.h)
        return out

    def get_action_host(self, feats: np.ndarray, mask: np.ndarray, state: np.ndarray, ids: np.ndarray,
                        noise: np.ndarray, num_steps: int = 4, out: Optional[np.ndarray] = None, stream=None):
        """Host buffers in and out (uint16 features are bf16 bits); synchronous."""
        feats = np.ascontiguousarray(feats)
        bb = GDIT_BF16 if feats.dtype == np.uint16 else GDIT_F32
        if bb == GDIT_F32 and feats.dtype != np.float32:
            raise TypeError("features must be float32 or uint16 (bf16 bits)")
        mask = np.ascontiguousarray(mask, dtype=np.uint8)
        state = np.ascontiguousarray(state, dtype=np.float32)
        ids = np.ascontiguousarray(ids, dtype=np.int32)
        noise = np.ascontiguousarray(noise, dtype=np.float32)
        if out is None:
            out = np.empty_like(noise)
        if out.dtype != np.float32 or not out.flags.c_contiguous or not out.flags.writeable:
            raise TypeError("out must be a writable contiguous float32 array")
        B, S = check_io_shapes(self.cfg, feats, mask, state, ids, noise, out)
        check(_lib.gdit_get_action_host(self.h, feats.ctypes.data, bb, mask.ctypes.data, state.ctypes.data,
                                        ids.ctypes.data, noise.ctypes.data, int(num_steps), out.ctypes.data,
                                        B, S, stream or 0), self.h)
        return out

    def prepare(self, batch: int, seq: int, num_steps: int, bf16: bool = True, stream=None):
        check(_lib.gdit_prepare(self.h, batch, seq, num_steps, GDIT_BF16 if bf16 else GDIT_F32, stream or 0), self.h)

    def sync_status(self) -> int:
        """0, or the (negative) device status code of the last call."""
        return _lib.gdit_sync_status(self.h)

    def check_canaries(self) -> int:
        """Range-checked build only: the number of guard bytes of this handle's
        device allocations that were overwritten (0 when nothing wrote past a
        buffer).  Synchronizes the device."""
        n = ctypes.c_longlong()
        check(_lib.gdit_check_canaries(self.h, ctypes.byref(n)), self.h)
        return n.value

    def debug_poke_guard(self, which: int = 0):
        """Range-checked build only (test hook): overwrite the first guard byte
        after allocation `which`, as a one-element overrun would."""
        check(_lib.gdit_debug_poke_guard(self.h, which), self.h)

    def routing(self, batch: int):
        perm = np.zeros(batch, np.int32)
        seg = np.zeros(self.cfg.num_embodiments + 1, np.int32)
        vofs = np.zeros(batch + 1, np.int32)
        check(_lib.gdit_debug_routing(self.h, perm.ctypes.data, seg.ctypes.data, vofs.ctypes.data), self.h)
        return perm, seg, vofs

    def debug_kv(self, layer: int):
        n = ctypes.c_int()
        check(_lib.gdit_debug_kv(self.h, layer, None, None, ctypes.byref(n)), self.h)
        k = np.zeros((n.value, self.cfg.hidden), np.float32)
        v = np.zeros((n.value, self.cfg.hidden), np.float32)
        check(_lib.gdit_debug_kv(self.h, layer, k.ctypes.data, v.ctypes.data, ctypes.byref(n)), self.h)
        return k, v

    def profile(self, feats, mask, state, ids, noise, num_steps: int = 4, out=None, stream=None) -> List[dict]:
        """Per-kernel-class CUDA-event timing of one eager run (same kernels)."""
        import torch
        bb, B, S, out = self._args(feats, mask, state, ids, noise, out)
        st = stream if stream is not None else torch.cuda.current_stream().cuda_stream
        stats = (_lib.gdit_kernel_stat * 32)()
        n = check(_lib.gdit_profile_get_action(self.h, _ptr(feats), bb, _ptr(mask), _ptr(state), _ptr(ids),
                                               _ptr(noise), int(num_steps), _ptr(out), B, S, st, stats, 32), self.h)
        return [dict(name=stats[i].name.decode(), launches=stats[i].launches, total_ms=stats[i].total_ms,
                     flops=stats[i].flops, bytes=stats[i].bytes) for i in range(n)]

    def close(self):
        if getattr(self, "h", None):
            _lib.gdit_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()


def test_gemm(A, B, bias, bn: int = 128, splits: int = 1, stream=None):
    """C = A B^T + bias through the tcgen05 GEMM (A [M,K], B [N,K] bf16 CUDA tensors)."""
    import torch
    M, K = A.shape
    N = B.shape[0]
    C = torch.empty((M, N), dtype=torch.float32, device=A.device)
    st = stream if stream is not None else torch.cuda.current_stream().cuda_stream
    check(_lib.gdit_test_gemm(_ptr(A), _ptr(B), _ptr(bias) if bias is not None else None, _ptr(C),
                              M, N, K, bn, splits, st), None)
    return C


def gemm_static_scratch(A, B, bias, C=None, bn: int = 64, splits: int = 1, stream=None):
    """Same as test_gemm, through the entry point that allocates no device
    memory (its scratch is a fixed array inside the library).  C may be given."""
    import torch
    M, K = A.shape
    N = B.shape[0]
    if C is None:
        C = torch.empty((M, N), dtype=torch.float32, device=A.device)
    st = stream if stream is not None else torch.cuda.current_stream().cuda_stream
    check(_lib.gdit_gemm_static_scratch(_ptr(A), _ptr(B), _ptr(bias) if bias is not None else None, _ptr(C),
                                        M, N, K, bn, splits, st), None)
    return C


def debug_small_plan(geom, batch: int, num_steps: int = 4, num_sms: int = 148, max_seq: int = 600,
                     flags: int = 0):
    """Whether a call of `batch` samples runs the persistent loop
    (gdit_debug_small_plan): dict(group_ctas, grouped), or None for the
    per-layer kernels."""
    cfg = make_config(geom, max(batch, 1), max_seq, 0, flags)
    g, gr = ctypes.c_int(), ctypes.c_int()
    check(_lib.gdit_debug_small_plan(ctypes.byref(cfg), int(batch), int(num_steps), int(num_sms),
                                     ctypes.byref(g), ctypes.byref(gr)))
    return None if g.value == 0 else {"group_ctas": g.value, "grouped": bool(gr.value)}


def debug_skinny_plan(M: int, N: int, K: int, num_sms: int = 148):
    """The skinny-M GEMM's plan for an [M, K] x [N, K]^T product
    (gdit_debug_skinny_plan): dict(mt, nu, stages, ctas, smem_bytes), or None
    when the shape runs on the tensor-core GEMM."""
    out = [ctypes.c_int() for _ in range(5)]
    rc = _lib.gdit_debug_skinny_plan(int(M), int(N), int(K), int(num_sms), *[ctypes.byref(o) for o in out])
    if rc != 0:
        return None
    return dict(zip(("mt", "nu", "stages", "ctas", "smem_bytes"), (o.value for o in out)))


def debug_wait_expiry(device: int = 0, limit_ns: int = 1_000_000) -> int:
    """Status of one bounded wait on an mbarrier that nothing arrives at
    (gdit_debug_wait_expiry): GDIT_ETIMEOUT is the expected result."""
    return _lib.gdit_debug_wait_expiry(int(device), int(limit_ns))
