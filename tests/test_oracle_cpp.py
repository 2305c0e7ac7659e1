"""Pins of the C++ oracle (oracle/cpp/gdit_oracle.cpp, float and double).

It is a second restatement of the pages, sharing no code with the numpy
oracle: the double instantiation must agree with the numpy oracle to rounding
on the tiny workload (every edge case the GPU tests use) and on a full-size
row, the float instantiation with the double one within float rounding, and
closed forms must hold exactly."""

import dataclasses

import numpy as np
import pytest

import oracle
import synth
from oracle import cpp_oracle as co


def _run(fn, W, w, inp, K, **kw):
    return fn(W, w.geom, inp["backbone_features"], inp["vl_mask"], inp["state"], inp["embodiment_id"],
              inp["init_noise"], K, **kw)


@pytest.fixture(scope="module")
def tiny():
    w = synth.workload("tiny", batch=6, fixed_ids=(1, 0, 0, 1, 1, 0), valid_min=1)
    W = synth.make_weights(w.geom)
    inp = synth.make_inputs(w, seed=7)
    inp["vl_mask"][2] = 0                 # no valid token
    inp["vl_mask"][3] = 0
    inp["vl_mask"][3, 17] = 1             # exactly one
    inp["vl_mask"][4, ::2] = 0            # not a prefix
    return w, W, inp


@pytest.mark.parametrize("K", [1, 3, 4, 8])
def test_double_matches_the_numpy_oracle(tiny, K):
    w, W, inp = tiny
    a = _run(oracle.get_action, W, w, inp, K)
    b = _run(co.get_action, W, w, inp, K)
    np.testing.assert_allclose(b, a, rtol=0, atol=1e-12 * max(1.0, float(np.abs(a).max())))


def test_float_is_within_float_rounding_of_double(tiny):
    w, W, inp = tiny
    a = _run(co.get_action, W, w, inp, 4)
    b = _run(co.get_action, W, w, inp, 4, dtype=np.float32)
    assert b.dtype == np.float32
    assert float(np.linalg.norm(b - a) / np.linalg.norm(a)) < 1e-5


def test_samples_are_independent(tiny):
    w, W, inp = tiny
    whole = _run(co.get_action, W, w, inp, 4)
    part = _run(co.get_action, W, w, inp, 4, samples=[4, 1])
    np.testing.assert_array_equal(part, whole[[4, 1]])


def test_zero_velocity_head_returns_the_noise():
    """act_dec.l2 weights and bias zero: every velocity is 0 and x stays the
    initial noise, bit for bit."""
    w = synth.workload("tiny", batch=2, fixed_ids=(0, 1))
    W = synth.make_weights(w.geom)
    W["act_dec.l2.W"][:] = 0
    W["act_dec.l2.b"][:] = 0
    inp = synth.make_inputs(w, seed=2)
    out = _run(co.get_action, W, w, inp, 4)
    np.testing.assert_array_equal(out, inp["init_noise"].astype(np.float64))


def test_decoder_signature_names_the_category():
    """Decoder weights zero and b2[c] = c: every sample moves by exactly its
    category index (K steps of c / K, exact for these values)."""
    g = dataclasses.replace(synth.GEOM_TINY, num_embodiments=6)
    W = synth.make_weights(g)
    for n in ("act_dec.l1.W", "act_dec.l1.b", "act_dec.l2.W"):
        W[n][:] = 0
    for c in range(6):
        W["act_dec.l2.b"][c] = c
    ids = (5, 0, 3, 1, 4, 2)
    w = synth.workload("tiny", geom=g, batch=6, fixed_ids=ids)
    inp = synth.make_inputs(w, seed=11)
    out = _run(co.get_action, W, w, inp, 4)
    moved = out - inp["init_noise"].astype(np.float64)
    np.testing.assert_array_equal(moved, np.broadcast_to(np.asarray(ids, np.float64)[:, None, None], moved.shape))


def test_masked_tokens_do_not_matter(tiny):
    w, W, inp = tiny
    a = _run(co.get_action, W, w, inp, 4)
    f = inp["backbone_features"].copy()
    f[inp["vl_mask"] == 0] = 1e3
    b = _run(co.get_action, W, w, dict(inp, backbone_features=f), 4)
    np.testing.assert_array_equal(a, b)


def test_bad_embodiment_id_is_rejected(tiny):
    w, W, inp = tiny
    bad = dict(inp, embodiment_id=np.array([0, 1, 9, 0, 1, 0], np.int32))
    with pytest.raises(ValueError):
        _run(co.get_action, W, w, bad, 4)


@pytest.mark.slow
def test_full_size_row_matches_the_numpy_oracle():
    """The latency workload (32 layers, hidden 1024, backbone [1, 300, 2048]):
    double against the numpy oracle to rounding, float within 1e-5."""
    W = synth.make_weights(synth.GEOM_FULL)
    w = synth.WORKLOADS["latency"]
    inp = synth.make_inputs(w)
    a = _run(oracle.get_action, W, w, inp, 4)
    b = _run(co.get_action, W, w, inp, 4)
    np.testing.assert_allclose(b, a, rtol=0, atol=1e-11)
    c = _run(co.get_action, W, w, inp, 4, dtype=np.float32)
    assert float(np.linalg.norm(c - a) / np.linalg.norm(a)) < 1e-5
