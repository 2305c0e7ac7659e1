"""The range-checked build (libgdit_checked.so, GDIT_CHECKED=1).

It is the same library with guard bands around every device allocation of a
handle and index checks on what the kernels derive from the inputs (packed
token rows, key spans, the sample permutation).  On valid inputs it must give
the regular build's results bit for bit, report a clean status and leave every
guard byte intact; a guard byte overwritten from the host (what a one-element
overrun would do) must be counted.  The checked library runs in a child
process (the binding loads one library per process).
"""

import json
import os
import subprocess
import sys

import numpy as np
import pytest

import synth
from tests.gpu_util import require_gpu

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _cases():
    """Ragged tiny batches of 3 (the persistent loop, one CTA group per
    sample) and 6 (the per-layer path), one tiny sample (the loop, one group)
    and the full-size batched workload (ragged keys, 32 embodiments)."""
    tiny = synth.workload("tiny", batch=3, fixed_ids=(1, 0, 1), valid_min=1)
    tiny_w = synth.make_weights(tiny.geom)
    return [("tiny", tiny, tiny_w, 5),
            ("tiny6", synth.workload("tiny", batch=6, fixed_ids=(1, 0), valid_min=1), tiny_w, 8),
            ("tiny_b1", synth.workload("tiny", batch=1, fixed_ids=(1,), valid_min=1), tiny_w, 6),
            ("batched", synth.WORKLOADS["batched"], synth.make_weights(synth.GEOM_FULL), 7)]


def _run(case, weights, seed):
    import torch
    from flow_matching_dit_b200 import ActionHead
    inp = synth.make_inputs(case, seed=seed)
    feats = inp["backbone_features"]
    f = torch.from_numpy(feats.view(np.int16)).cuda().view(torch.bfloat16) if feats.dtype == np.uint16 \
        else torch.from_numpy(feats).cuda()
    d = [f] + [torch.from_numpy(inp[k]).cuda() for k in ("vl_mask", "state", "embodiment_id", "init_noise")]
    head = ActionHead(case.geom, weights, max_batch=case.batch, max_seq=case.seq)
    out = head.get_action(*d, num_steps=case.num_steps).cpu().numpy()
    return head, out, head.sync_status()


def _child(outdir):
    """Runs in the child process, on the range-checked library."""
    import flow_matching_dit_b200 as fm
    res = {"checked": fm.is_checked()}
    for name, case, weights, seed in _cases():
        head, out, st = _run(case, weights, seed)
        res[name] = {"status": st, "canaries": head.check_canaries()}
        np.save(os.path.join(outdir, name + ".npy"), out)
        if name == "tiny":
            head.debug_poke_guard(0)
            res["poked"] = head.check_canaries()
        head.close()
    json.dump(res, open(os.path.join(outdir, "res.json"), "w"))


def test_checked_build_equals_regular_build_and_keeps_its_guards(tmp_path):
    require_gpu()
    env = dict(os.environ, GDIT_CHECKED="1")
    code = f"import sys; sys.path.insert(0, {ROOT!r}); import tests.test_gpu_checked as t; t._child({str(tmp_path)!r})"
    r = subprocess.run([sys.executable, "-c", code], cwd=ROOT, env=env, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stderr[-3000:]
    res = json.load(open(tmp_path / "res.json"))
    assert res["checked"] is True
    for name, case, weights, seed in _cases():
        assert res[name]["status"] == 0, name
        assert res[name]["canaries"] == 0, name
        head, ref, st = _run(case, weights, seed)    # the regular build, in this process
        head.close()
        assert st == 0
        np.testing.assert_array_equal(np.load(tmp_path / (name + ".npy")), ref, err_msg=name)
    assert res["poked"] == 1
