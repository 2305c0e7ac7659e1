"""Host-side fault injection (GDIT_FAULT=alloc:N | upload:N | graph:N): the
N-th device allocation, weight upload or CUDA-graph instantiation of a handle
fails as the real call would.  Nothing on the GPU is made to fail.  Each
failure must come back as the right status, leave no device memory behind once
the handle is gone, and leave the library usable."""

import numpy as np
import pytest

import oracle
import synth
from tests.gpu_util import MAX_ABS, REL_L2, parity_stats, require_gpu, to_dev

pytestmark = pytest.mark.gpu


def _free_bytes():
    import torch
    torch.cuda.synchronize()
    return torch.cuda.mem_get_info()[0]


@pytest.fixture(scope="module")
def tiny_weights():
    W = synth.make_weights(synth.GEOM_TINY)
    require_gpu()
    from flow_matching_dit_b200 import ActionHead
    # one clean create and destroy first: the CUDA context and the library's
    # kernels are loaded once per process and stay, which is not a leak
    ActionHead(synth.GEOM_TINY, W, max_batch=4, max_seq=64).close()
    return W


@pytest.mark.parametrize("spec,code", [
    ("alloc:1", "GDIT_ENOMEM"),      # the first device allocation of create
    ("alloc:60", "GDIT_ENOMEM"),     # one inside the workspace (the weights take the first 45)
    ("upload:1", "GDIT_ECUDA"),      # the first weight upload
    ("upload:25", "GDIT_ECUDA"),     # one in the middle of the block weights
])
def test_create_fails_cleanly(tiny_weights, monkeypatch, spec, code):
    require_gpu()
    from flow_matching_dit_b200 import ActionHead, GditError, _lib
    before = _free_bytes()
    monkeypatch.setenv("GDIT_FAULT", spec)
    with pytest.raises(GditError) as e:
        ActionHead(synth.GEOM_TINY, tiny_weights, max_batch=4, max_seq=64)
    assert e.value.code == getattr(_lib, code)
    assert "injected fault" in str(e.value)
    # everything create allocated before the failure is released
    assert abs(_free_bytes() - before) < 8 << 20


def test_graph_instantiation_failure_then_recovery(tiny_weights, monkeypatch):
    """The first profile's graph fails to instantiate: the call reports
    GDIT_ECUDA; the next call of the same profile builds it again and runs
    normally; destroying the handle returns its memory."""
    require_gpu()
    from flow_matching_dit_b200 import ActionHead, GditError, _lib
    before = _free_bytes()
    monkeypatch.setenv("GDIT_FAULT", "graph:1")
    w = synth.workload("tiny", batch=2, fixed_ids=(0, 1))
    inp = synth.make_inputs(w, seed=3)
    head = ActionHead(synth.GEOM_TINY, tiny_weights, max_batch=2, max_seq=64)
    try:
        with pytest.raises(GditError) as e:
            head.get_action(*to_dev(inp), num_steps=4)
        assert e.value.code == _lib.GDIT_ECUDA and "injected fault" in str(e.value)
        out = head.get_action(*to_dev(inp), num_steps=4).cpu().numpy()
        assert head.sync_status() == 0
        ref = oracle.get_action(tiny_weights, w.geom, inp["backbone_features"], inp["vl_mask"], inp["state"],
                                inp["embodiment_id"], inp["init_noise"], 4)
        max_abs, rel, _ = parity_stats(out, ref, inp["init_noise"])
        assert max_abs <= MAX_ABS and rel <= REL_L2
    finally:
        head.close()
    assert abs(_free_bytes() - before) < 8 << 20


def test_a_clean_create_after_injected_failures(tiny_weights, monkeypatch):
    require_gpu()
    from flow_matching_dit_b200 import ActionHead
    monkeypatch.delenv("GDIT_FAULT", raising=False)
    w = synth.workload("tiny", fixed_ids=(1,))
    inp = synth.make_inputs(w, seed=4)
    with ActionHead(synth.GEOM_TINY, tiny_weights, max_batch=1, max_seq=64) as head:
        out = head.get_action(*to_dev(inp), num_steps=4).cpu().numpy()
        assert head.sync_status() == 0
    ref = oracle.get_action(tiny_weights, w.geom, inp["backbone_features"], inp["vl_mask"], inp["state"],
                            inp["embodiment_id"], inp["init_noise"], 4)
    assert np.abs(out - ref).max() <= MAX_ABS
