"""ctypes binding of include/gdit.h: argument marshalling only.

Every function here forwards to the entry point of the same name in
``libgdit.so`` (or, with the environment variable ``GDIT_CHECKED=1`` set
before the first call, in the range-checked build ``libgdit_checked.so``).
There is no fallback: if the library is missing or cannot be loaded, ``lib()``
raises.
"""

from __future__ import annotations

import ctypes
import os
import threading

from .build import LIB, LIB_CHECKED

GDIT_OK = 0
GDIT_EINVAL = -1
GDIT_ENOMEM = -2
GDIT_ECUDA = -3
GDIT_EPROFILE = -4
GDIT_ETIMEOUT = -5
GDIT_EDEVICE = -6
GDIT_ENODEV = -7
GDIT_F32 = 0
GDIT_BF16 = 1
GDIT_FLAG_STRICT_PROFILES = 1
GDIT_FLAG_NO_GRAPH = 2
GDIT_FLAG_NO_SMALL = 4
GDIT_FLAG_NO_TMA_STORE = 8
GDIT_FLAG_NO_PAIR = 16
GDIT_FLAG_NO_SKINNY = 32


class gdit_config(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in (
        "num_layers", "hidden", "num_heads", "head_dim", "mlp_hidden", "backbone_dim",
        "action_dim", "state_dim", "action_horizon", "num_embodiments",
        "max_batch", "max_backbone_seq", "time_freq_dim", "num_timestep_buckets")] + [
        ("ln_eps", ctypes.c_float), ("flags", ctypes.c_uint), ("device", ctypes.c_int),
        ("attend_text_every_n_blocks", ctypes.c_int)]


class gdit_tensor(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char_p), ("dtype", ctypes.c_int), ("ndim", ctypes.c_int),
                ("shape", ctypes.POINTER(ctypes.c_int64)), ("host_ptr", ctypes.c_void_p)]


class gdit_kernel_stat(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char * 32), ("launches", ctypes.c_int), ("total_ms", ctypes.c_double),
                ("flops", ctypes.c_double), ("bytes", ctypes.c_double)]


_P = ctypes.c_void_p
_I = ctypes.c_int
_SIGS = {
    "gdit_create": (_I, [ctypes.POINTER(gdit_config), ctypes.POINTER(gdit_tensor), _I, ctypes.POINTER(_P)]),
    "gdit_destroy": (None, [_P]),
    "gdit_get_action": (_I, [_P, _P, _I, _P, _P, _P, _P, _I, _P, _I, _I, _P]),
    "gdit_get_action_host": (_I, [_P, _P, _I, _P, _P, _P, _P, _I, _P, _I, _I, _P]),
    "gdit_prepare": (_I, [_P, _I, _I, _I, _I, _P]),
    "gdit_sync_status": (_I, [_P]),
    "gdit_strerror": (ctypes.c_char_p, [_I]),
    "gdit_last_error": (ctypes.c_char_p, [_P]),
    "gdit_version": (ctypes.c_char_p, []),
    "gdit_debug_routing": (_I, [_P, _P, _P, _P]),
    "gdit_debug_kv": (_I, [_P, _I, _P, _P, ctypes.POINTER(_I)]),
    "gdit_profile_get_action": (_I, [_P, _P, _I, _P, _P, _P, _P, _I, _P, _I, _I, _P,
                                     ctypes.POINTER(gdit_kernel_stat), _I]),
    "gdit_test_gemm": (_I, [_P, _P, _P, _P, _I, _I, _I, _I, _I, _P]),
    "gdit_gemm_static_scratch": (_I, [_P, _P, _P, _P, _I, _I, _I, _I, _I, _P]),
    "gdit_debug_wait_expiry": (_I, [_I, ctypes.c_ulonglong]),
    "gdit_debug_skinny_plan": (_I, [ctypes.c_longlong, _I, _I, _I] + [ctypes.POINTER(_I)] * 5),
    "gdit_debug_small_plan": (_I, [ctypes.POINTER(gdit_config), _I, _I, _I, ctypes.POINTER(_I), ctypes.POINTER(_I)]),
    "gdit_get_action_vl": (_I, [_P, _P, _I, _P, _P, _P, _P, _P, _I, _P, _I, _I, _P]),
    "gdit_is_checked": (_I, []),
    "gdit_check_canaries": (_I, [_P, ctypes.POINTER(ctypes.c_longlong)]),
    "gdit_debug_poke_guard": (_I, [_P, _I]),
}

_lock = threading.Lock()
_lib = None


def default_path() -> str:
    return LIB_CHECKED if os.environ.get("GDIT_CHECKED") == "1" else LIB


def lib(path: str = None) -> ctypes.CDLL:
    """The loaded library (raises if it is missing: build it first)."""
    global _lib
    with _lock:
        if _lib is None:
            path = path or default_path()
            if not os.path.exists(path):
                raise RuntimeError(f"{path} not found: run flow_matching_dit_b200.build.build() first")
            L = ctypes.CDLL(path)
            for name, (res, args) in _SIGS.items():
                f = getattr(L, name)
                f.restype = res
                f.argtypes = args
            _lib = L
        return _lib


def exported_names():
    return list(_SIGS)


class GditError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"{msg} (code {code})")
        self.code = code


def check(code: int, handle=None) -> int:
    if code < 0:
        L = lib()
        detail = L.gdit_last_error(handle)
        raise GditError(code, (detail or L.gdit_strerror(code)).decode())
    return code


# thin forwarding functions, same names as the C ABI
def gdit_create(cfg, weights, n, out):
    return lib().gdit_create(cfg, weights, n, out)


def gdit_destroy(h):
    return lib().gdit_destroy(h)


def gdit_get_action(*a):
    return lib().gdit_get_action(*a)


def gdit_get_action_vl(*a):
    return lib().gdit_get_action_vl(*a)


def gdit_get_action_host(*a):
    return lib().gdit_get_action_host(*a)


def gdit_prepare(*a):
    return lib().gdit_prepare(*a)


def gdit_sync_status(h):
    return lib().gdit_sync_status(h)


def gdit_strerror(c):
    return lib().gdit_strerror(c)


def gdit_last_error(h):
    return lib().gdit_last_error(h)


def gdit_version():
    return lib().gdit_version()


def gdit_debug_routing(*a):
    return lib().gdit_debug_routing(*a)


def gdit_debug_kv(*a):
    return lib().gdit_debug_kv(*a)


def gdit_profile_get_action(*a):
    return lib().gdit_profile_get_action(*a)


def gdit_test_gemm(*a):
    return lib().gdit_test_gemm(*a)


def gdit_gemm_static_scratch(*a):
    return lib().gdit_gemm_static_scratch(*a)


def gdit_debug_wait_expiry(device, limit_ns):
    return lib().gdit_debug_wait_expiry(device, limit_ns)


def gdit_debug_skinny_plan(*a):
    return lib().gdit_debug_skinny_plan(*a)


def gdit_debug_small_plan(*a):
    return lib().gdit_debug_small_plan(*a)


def gdit_is_checked():
    return lib().gdit_is_checked()


def gdit_check_canaries(h, out):
    return lib().gdit_check_canaries(h, out)


def gdit_debug_poke_guard(h, which):
    return lib().gdit_debug_poke_guard(h, which)
