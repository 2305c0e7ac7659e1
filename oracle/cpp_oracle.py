"""Python side of the C++ CPU oracle (``oracle/cpp/gdit_oracle.cpp``).

TEST INFRASTRUCTURE ONLY: used by ``tests/`` and by the CPU-baseline leg of
``bench.py``.  The C++ oracle is a second restatement of the pages, written as
naive loops (float and double instantiations, OpenMP over samples or over the
outputs of a linear).  It shares no code with the GPU library or with the
numpy oracle (``oracle/dit.py``); this module only converts the inputs and
passes pointers.

Weight order passed to the library (canonical names, ``include/gdit.h``):
t_enc.l1.w, t_enc.l1.b, t_enc.l2.w, t_enc.l2.b; for every block l:
blk{l}.ada.w, .ada.b, .q.w, .q.b, .k.w, .k.b, .v.w, .v.b, .o.w, .o.b, .ln3.g,
.ln3.b, .ff1.w, .ff1.b, .ff2.w, .ff2.b; out.ada.w, out.ada.b, out.proj.w,
out.proj.b; state_enc.l1.W, .l1.b, .l2.W, .l2.b; act_enc.W1.W, .W1.b, .W2.W,
.W2.b, .W3.W, .W3.b; act_dec.l1.W, .l1.b, .l2.W, .l2.b.
"""

from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from typing import Dict, List, Optional, Sequence

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "cpp", "gdit_oracle.cpp")
LIB = os.path.join(HERE, "cpp", "libgdit_oracle.so")


class _Geom(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in (
        "num_layers", "hidden", "num_heads", "head_dim", "mlp_hidden", "backbone_dim", "action_dim",
        "state_dim", "action_horizon", "num_embodiments", "time_freq_dim", "num_timestep_buckets")] + [
        ("ln_eps", ctypes.c_double)]


def build(force: bool = False) -> str:
    """Compile the C++ oracle with g++ (OpenMP) into oracle/cpp/."""
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    tmp = LIB + ".tmp"
    cmd = ["g++", "-O3", "-fopenmp", "-fPIC", "-shared", "-std=c++17", "-Wall", "-o", tmp, SRC]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError("g++ failed:\n" + r.stdout + r.stderr)
    os.replace(tmp, LIB)
    return LIB


_lock = threading.Lock()
_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    with _lock:
        if _lib is None:
            L = ctypes.CDLL(build())
            for name, T in (("oracle_get_action_f64", ctypes.c_double), ("oracle_get_action_f32", ctypes.c_float)):
                f = getattr(L, name)
                f.restype = ctypes.c_int
                P = ctypes.POINTER(T)
                f.argtypes = [ctypes.POINTER(_Geom), ctypes.POINTER(P), ctypes.c_int, P, ctypes.c_void_p, P,
                              ctypes.c_void_p, P, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, P]
            L.oracle_max_threads.restype = ctypes.c_int
            _lib = L
        return _lib


def weight_order(geom) -> List[str]:
    names = ["t_enc.l1.w", "t_enc.l1.b", "t_enc.l2.w", "t_enc.l2.b"]
    for l in range(geom.num_layers):
        names += [f"blk{l}.{t}" for t in ("ada.w", "ada.b", "q.w", "q.b", "k.w", "k.b", "v.w", "v.b", "o.w",
                                          "o.b", "ln3.g", "ln3.b", "ff1.w", "ff1.b", "ff2.w", "ff2.b")]
    names += ["out.ada.w", "out.ada.b", "out.proj.w", "out.proj.b",
              "state_enc.l1.W", "state_enc.l1.b", "state_enc.l2.W", "state_enc.l2.b",
              "act_enc.W1.W", "act_enc.W1.b", "act_enc.W2.W", "act_enc.W2.b", "act_enc.W3.W", "act_enc.W3.b",
              "act_dec.l1.W", "act_dec.l1.b", "act_dec.l2.W", "act_dec.l2.b"]
    return names


def _as(a, dtype) -> np.ndarray:
    """Contiguous copy in `dtype`; uint16 arrays hold bf16 bit patterns."""
    a = np.asarray(a)
    if a.dtype == np.uint16:
        a = (a.astype(np.uint32) << np.uint32(16)).view(np.float32)
    return np.ascontiguousarray(a, dtype=dtype)


class Weights:
    """The weight table converted once to float64 or float32, in the library's order."""

    def __init__(self, weights: Dict[str, np.ndarray], geom, dtype=np.float64):
        self.dtype = np.dtype(dtype)
        self.arrays = [_as(weights[n], self.dtype) for n in weight_order(geom)]
        T = ctypes.c_double if self.dtype == np.float64 else ctypes.c_float
        self.ptrs = (ctypes.POINTER(T) * len(self.arrays))(*[a.ctypes.data_as(ctypes.POINTER(T))
                                                             for a in self.arrays])


def get_action(weights, geom, backbone_features, vl_mask, state, embodiment_id, init_noise, num_steps: int,
               samples: Optional[Sequence[int]] = None, dtype=np.float64, threads: int = 0,
               prepared: Optional[Weights] = None) -> np.ndarray:
    """x = init_noise; K Euler steps of the velocity field; returns [B, H, A]
    (or the rows `samples`, in that order) in `dtype`."""
    if getattr(geom, "attend_text_every_n_blocks", 0) or getattr(geom, "vlln", False):
        raise ValueError("the C++ oracle covers neither the image/text split nor vlln")
    W = prepared if prepared is not None else Weights(weights, geom, dtype)
    dt = W.dtype
    rows = list(range(len(embodiment_id))) if samples is None else list(samples)
    feats = _as(np.asarray(backbone_features)[rows], dt)
    mask = np.ascontiguousarray(np.asarray(vl_mask)[rows], dtype=np.uint8)
    st = _as(np.asarray(state)[rows], dt)
    ids = np.ascontiguousarray(np.asarray(embodiment_id).reshape(-1)[rows], dtype=np.int32)
    noise = _as(np.asarray(init_noise)[rows], dt)
    B, S = mask.shape
    out = np.zeros((B, geom.action_horizon, geom.action_dim), dtype=dt)
    g = _Geom(*[int(getattr(geom, f)) for f, _ in _Geom._fields_[:-1]], float(geom.ln_eps))
    T = ctypes.c_double if dt == np.float64 else ctypes.c_float
    P = ctypes.POINTER(T)
    fn = lib().oracle_get_action_f64 if dt == np.float64 else lib().oracle_get_action_f32
    rc = fn(ctypes.byref(g), W.ptrs, len(W.arrays), feats.ctypes.data_as(P), mask.ctypes.data, st.ctypes.data_as(P),
            ids.ctypes.data, noise.ctypes.data_as(P), B, S, int(num_steps), int(threads), out.ctypes.data_as(P))
    if rc == -2:
        raise ValueError("embodiment_id out of range")
    if rc != 0:
        raise ValueError(f"C++ oracle rejected its arguments ({rc})")
    return out


def max_threads() -> int:
    return int(lib().oracle_max_threads())
