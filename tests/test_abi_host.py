"""The C-ABI library builds, loads and exports every entry point that
include/gdit.h declares; host-side argument validation works without a GPU."""

import ctypes
import os
import re

import numpy as np
import pytest

import synth
from flow_matching_dit_b200 import _lib
from flow_matching_dit_b200.build import HEADER, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    build()
    return _lib.lib()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(gdit_[a-z_]+)\s*\(", src)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("gdit_create", "gdit_get_action", "gdit_destroy", "gdit_sync_status", "gdit_strerror"):
        assert required in names


def test_library_exports_every_declared_symbol(L):
    for name in declared_functions():
        assert hasattr(L, name), name
    assert set(declared_functions()) == set(_lib.exported_names())


def test_range_checked_build_exports_the_same_symbols_and_says_so(L):
    """libgdit_checked.so (GDIT_CHECKED=1: guard bands, index checks) has the
    same entry points; gdit_is_checked tells the two builds apart.  Neither
    call touches a GPU."""
    path = build(checked=True)
    C = ctypes.CDLL(path)
    for name in declared_functions():
        assert hasattr(C, name), name
    C.gdit_is_checked.restype = ctypes.c_int
    assert C.gdit_is_checked() == 1
    L.gdit_is_checked.restype = ctypes.c_int
    assert L.gdit_is_checked() == 0
    # a regular-build handle has no guard bands: the canary check refuses a NULL handle either way
    assert L.gdit_check_canaries(None, None) == _lib.GDIT_EINVAL
    assert L.gdit_debug_poke_guard(None, 0) == _lib.GDIT_EINVAL


def test_strings(L):
    assert L.gdit_version().startswith(b"gdit")
    assert L.gdit_strerror(_lib.GDIT_EINVAL) == b"invalid argument"
    assert L.gdit_strerror(-1234) == b"unknown error"


def _cfg(g, **over):
    c = _lib.gdit_config()
    for f in ("num_layers", "hidden", "num_heads", "head_dim", "mlp_hidden", "backbone_dim", "action_dim",
              "state_dim", "action_horizon", "num_embodiments", "time_freq_dim", "num_timestep_buckets"):
        setattr(c, f, getattr(g, f))
    c.ln_eps = g.ln_eps
    c.max_batch = 4
    c.max_backbone_seq = 64
    for k, v in over.items():
        setattr(c, k, v)
    return c


def _tensors(W):
    keep = []
    arr = (_lib.gdit_tensor * len(W))()
    for i, (n, a) in enumerate(W.items()):
        a = np.ascontiguousarray(a)
        shp = (ctypes.c_int64 * a.ndim)(*a.shape)
        nm = n.encode()
        keep += [a, shp, nm]
        arr[i].name, arr[i].ndim, arr[i].shape, arr[i].host_ptr = nm, a.ndim, shp, a.ctypes.data
        arr[i].dtype = _lib.GDIT_BF16 if a.dtype == np.uint16 else _lib.GDIT_F32
    return arr, keep


@pytest.fixture(scope="module")
def tinyW():
    return synth.make_weights(synth.GEOM_TINY)


def _create(L, cfg, W):
    arr, keep = _tensors(W)
    h = ctypes.c_void_p()
    rc = L.gdit_create(ctypes.byref(cfg), arr, len(W), ctypes.byref(h))
    return rc, h, L.gdit_last_error(None).decode()


@pytest.mark.parametrize("field,value,msg", [
    ("num_layers", 3, "num_layers"),
    ("head_dim", 48, "head_dim"),
    ("hidden", 96, "hidden"),
    ("action_dim", 30, "action_dim"),
    ("action_horizon", 64, "action_horizon"),
    ("num_embodiments", 65, "num_embodiments"),
    ("max_batch", 0, "max_batch"),
    ("attend_text_every_n_blocks", -1, "attend_text_every_n_blocks"),
    ("max_backbone_seq", 65537, "max_backbone_seq"),
    ("num_timestep_buckets", 0, "num_timestep_buckets"),
    ("ln_eps", 0.0, "ln_eps"),
    ("time_freq_dim", 255, "time_freq_dim"),
    ("head_dim", 128, "head_dim"),
    ("state_dim", 48, "state_dim"),
])
def test_bad_config_rejected_on_host(L, tinyW, field, value, msg):
    cfg = _cfg(synth.GEOM_TINY, **{field: value})
    rc, h, err = _create(L, cfg, tinyW)
    assert rc == _lib.GDIT_EINVAL and not h.value
    assert msg in err


def test_missing_weight_is_named(L, tinyW):
    W = dict(tinyW)
    del W["blk1.ff2.b"]
    rc, h, err = _create(L, _cfg(synth.GEOM_TINY), W)
    assert rc == _lib.GDIT_EINVAL and "blk1.ff2.b" in err


def test_misshaped_weight_is_named(L, tinyW):
    W = dict(tinyW)
    W["act_enc.W2.W"] = np.zeros((2, 128, 128), np.float32)
    rc, h, err = _create(L, _cfg(synth.GEOM_TINY), W)
    assert rc == _lib.GDIT_EINVAL and "act_enc.W2.W" in err


def test_unknown_weight_rejected(L, tinyW):
    W = dict(tinyW)
    W["blk9.extra"] = np.zeros(3, np.float32)
    rc, h, err = _create(L, _cfg(synth.GEOM_TINY), W)
    assert rc == _lib.GDIT_EINVAL and "unknown" in err


def test_valid_table_without_gpu_reports_no_device(L, tinyW):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    rc, h, err = _create(L, _cfg(synth.GEOM_TINY), tinyW)
    assert rc in (_lib.GDIT_ENODEV, _lib.GDIT_ECUDA) and not h.value


def test_null_handle_calls_are_rejected(L):
    assert L.gdit_get_action(None, None, 0, None, None, None, None, 4, None, 1, 1, None) == _lib.GDIT_EINVAL
    assert L.gdit_get_action_vl(None, None, 0, None, None, None, None, None, 4, None, 1, 1, None) == _lib.GDIT_EINVAL
    assert L.gdit_get_action_host(None, None, 0, None, None, None, None, 4, None, 1, 1, None) == _lib.GDIT_EINVAL
    assert L.gdit_sync_status(None) == _lib.GDIT_EINVAL
    L.gdit_destroy(None)


def test_wait_expiry_check_validates_on_host(L):
    from flow_matching_dit_b200._lib import GDIT_EINVAL, GDIT_ENODEV
    assert L.gdit_debug_wait_expiry(0, 10) == GDIT_EINVAL              # below 1 us
    assert L.gdit_debug_wait_expiry(0, 5_000_000_000) == GDIT_EINVAL   # above 1 s
    import torch
    if not torch.cuda.is_available():
        assert L.gdit_debug_wait_expiry(0, 1_000_000) == GDIT_ENODEV


def test_vlln_weights_come_in_pairs_of_the_backbone_width(L, tinyW):
    """The optional vision-language layer norm: vlln.g and vlln.b together, [Dvl] each."""
    dvl = synth.GEOM_TINY.backbone_dim
    only_g = dict(tinyW)
    only_g["vlln.g"] = np.ones(dvl, np.float32)
    rc, _, msg = _create(L, _cfg(synth.GEOM_TINY), only_g)
    assert rc == _lib.GDIT_EINVAL and "together" in msg
    bad = dict(only_g)
    bad["vlln.b"] = np.zeros(dvl + 1, np.float32)
    rc, _, msg = _create(L, _cfg(synth.GEOM_TINY), bad)
    assert rc == _lib.GDIT_EINVAL and "vlln.b" in msg


def test_io_shapes_are_checked_before_any_pointer_is_passed():
    """The binding refuses buffers whose shapes disagree with the batch and
    sequence of the features: the library would read or write past them."""
    from flow_matching_dit_b200 import check_io_shapes
    g = synth.GEOM_TINY
    cfg = _cfg(g)
    B, S = 3, 40
    ok = dict(feats=np.zeros((B, S, g.backbone_dim), np.float32), mask=np.zeros((B, S), np.uint8),
              state=np.zeros((B, 1, g.state_dim), np.float32), ids=np.zeros(B, np.int32),
              noise=np.zeros((B, g.action_horizon, g.action_dim), np.float32),
              out=np.zeros((B, g.action_horizon, g.action_dim), np.float32))
    assert check_io_shapes(cfg, **ok) == (B, S)
    assert check_io_shapes(cfg, **dict(ok, state=np.zeros((B, g.state_dim), np.float32))) == (B, S)
    assert check_io_shapes(cfg, **ok, image_mask=np.zeros((B, S), np.uint8)) == (B, S)
    bad = {
        "feats": np.zeros((B, S, g.backbone_dim + 1), np.float32),
        "mask": np.zeros((B, S - 1), np.uint8),
        "state": np.zeros((B - 1, 1, g.state_dim), np.float32),
        "ids": np.zeros(B + 1, np.int32),
        "noise": np.zeros((B, g.action_horizon - 1, g.action_dim), np.float32),
        "out": np.zeros((B - 1, g.action_horizon, g.action_dim), np.float32),
    }
    for name, arr in bad.items():
        with pytest.raises(ValueError):
            check_io_shapes(cfg, **dict(ok, **{name: arr}))
    with pytest.raises(ValueError):
        check_io_shapes(cfg, **ok, image_mask=np.zeros((B, S + 1), np.uint8))
    with pytest.raises(ValueError):
        check_io_shapes(cfg, **dict(ok, feats=np.zeros((B * S, g.backbone_dim), np.float32)))


class _FakeCuda:
    """Stands in for a contiguous CUDA tensor: dtype, shape and device only
    (the pointer is never dereferenced: the handle below is NULL)."""

    def __init__(self, shape, dtype, index=0):
        import torch
        self.shape, self.dtype, self.is_cuda = tuple(shape), dtype, True
        self.device = torch.device("cuda", index)

    def is_contiguous(self):
        return True

    def data_ptr(self):
        return 0


def test_device_call_path_validates_then_reaches_the_library(L):
    """ActionHead.get_action's Python path on realistic inputs: it accepts
    them, passes them to the library (a NULL handle: GDIT_EINVAL, nothing is
    dereferenced), and rejects wrong shapes, dtypes and devices first."""
    import torch
    from flow_matching_dit_b200 import ActionHead, GditError
    g = synth.GEOM_TINY
    head = object.__new__(ActionHead)
    head.cfg = _cfg(g)
    head.cfg.device = 0
    head.h = None
    B, S = 2, 64
    args = [_FakeCuda((B, S, g.backbone_dim), torch.bfloat16), _FakeCuda((B, S), torch.uint8),
            _FakeCuda((B, 1, g.state_dim), torch.float32), _FakeCuda((B,), torch.int32),
            _FakeCuda((B, g.action_horizon, g.action_dim), torch.float32)]
    out = _FakeCuda((B, g.action_horizon, g.action_dim), torch.float32)
    for kw in ({}, {"image_mask": _FakeCuda((B, S), torch.uint8)}):
        with pytest.raises(GditError) as e:
            head.get_action(*args, num_steps=4, out=out, stream=0, **kw)
        assert e.value.code == _lib.GDIT_EINVAL
    with pytest.raises(ValueError):
        head.get_action(*args[:4], _FakeCuda((B, g.action_horizon + 1, g.action_dim), torch.float32),
                        out=out, stream=0)
    with pytest.raises(TypeError):
        head.get_action(args[0], args[1], args[2], _FakeCuda((B,), torch.int64), args[4], out=out, stream=0)
    with pytest.raises(ValueError):
        head.get_action(*args, out=_FakeCuda(out.shape, torch.float32, index=1), stream=0)
    with pytest.raises(TypeError):
        head.get_action(*args, out=out, stream=0, image_mask=_FakeCuda((B, S), torch.bool))
    with pytest.raises(ValueError):
        head.get_action(*args, out=out, stream=0, image_mask=_FakeCuda((B, S - 1), torch.uint8))
    # the host-buffer path on numpy inputs of the same shapes
    inp = synth.make_inputs(synth.workload("tiny", batch=B, fixed_ids=(0, 1)))
    with pytest.raises(GditError) as e:
        head.get_action_host(inp["backbone_features"], inp["vl_mask"], inp["state"], inp["embodiment_id"],
                             inp["init_noise"], 4)
    assert e.value.code == _lib.GDIT_EINVAL
    with pytest.raises(ValueError):
        head.get_action_host(inp["backbone_features"], inp["vl_mask"][:, :-1], inp["state"],
                             inp["embodiment_id"], inp["init_noise"], 4)


def test_binding_flags_and_codes_equal_the_header():
    """Every GDIT_FLAG_* and status code the header defines has the same value
    in the binding (the C ABI passes them as plain integers)."""
    src = open(HEADER).read()
    defs = dict((n, int(v)) for n, v in re.findall(r"#define\s+(GDIT_FLAG_[A-Z_]+)\s+(\d+)u", src))
    assert len(defs) >= 6
    codes = dict((n, int(v)) for n, v in re.findall(r"#define\s+(GDIT_(?:OK|E[A-Z]+))\s+\(?(-?\d+)\)?", src))
    assert codes["GDIT_OK"] == 0 and len(codes) >= 8
    for name, value in {**defs, **codes}.items():
        assert getattr(_lib, name) == value, name


def test_binding_forwards_every_entry_point_under_its_own_name():
    for name in _lib.exported_names():
        assert callable(getattr(_lib, name, None)), name


def test_every_handle_entry_point_rejects_a_null_handle(L):
    """Checked before anything else (no pointer is dereferenced, no CUDA call)."""
    E = _lib.GDIT_EINVAL
    assert L.gdit_prepare(None, 1, 1, 4, _lib.GDIT_BF16, None) == E
    assert L.gdit_debug_routing(None, None, None, None) == E
    n = ctypes.c_int()
    assert L.gdit_debug_kv(None, 0, None, None, ctypes.byref(n)) == E
    stats = (_lib.gdit_kernel_stat * 4)()
    assert L.gdit_profile_get_action(None, None, 0, None, None, None, None, 4, None, 1, 1, None, stats, 4) == E


def test_gemm_hooks_reject_null_matrices_on_the_host(L):
    for f in (L.gdit_test_gemm, L.gdit_gemm_static_scratch):
        assert f(None, None, None, None, 128, 128, 64, 128, 1, None) == _lib.GDIT_EINVAL
        assert "NULL matrix" in L.gdit_last_error(None).decode()


@pytest.mark.parametrize("spec", ["alloc", "alloc:0", "alloc:x", "disk:3", "graph:2,upload:-1"])
def test_malformed_fault_injection_spec_is_rejected(L, tinyW, monkeypatch, spec):
    """GDIT_FAULT (host-side fault injection) is parsed before any device
    call: a malformed value is an invalid argument, named in the message."""
    monkeypatch.setenv("GDIT_FAULT", spec)
    rc, h, err = _create(L, _cfg(synth.GEOM_TINY), tinyW)
    assert rc == _lib.GDIT_EINVAL and not h.value
    assert "GDIT_FAULT" in err
