"""Pins of the gradient oracle (``oracle.grad``), CPU only.

The expected side never uses torch: the loss comes from the numpy oracle,
directional derivatives from central finite differences of the numpy oracle's
loss, and the decoder's last bias from its closed form."""

import dataclasses

import numpy as np
import pytest

import oracle
import synth
from oracle.grad import training_loss_and_grads

G = synth.GEOM_TINY


def _case(g=G, ids=(0, 1), seed=3, vlln=False):
    g = dataclasses.replace(g, vlln=vlln)
    W = {k: np.asarray(v, np.float64) for k, v in synth.make_weights(g).items()}
    w = dataclasses.replace(synth.WORKLOADS["tiny"], geom=g, batch=len(ids), fixed_ids=tuple(ids))
    inp = synth.make_inputs(w, seed=seed)
    r = np.random.default_rng(seed)
    acts = r.standard_normal(inp["init_noise"].shape)
    mask = (r.uniform(size=acts.shape) < 0.7).astype(np.float64)
    t = r.uniform(0.05, 0.95, size=len(ids))
    return g, W, inp, acts, mask, t


def _np_loss(g, W, inp, acts, mask, t, image_mask=None):
    return oracle.training_loss(W, g, inp["backbone_features"], inp["vl_mask"], inp["state"], inp["embodiment_id"],
                                acts, inp["init_noise"], t, mask, image_mask=image_mask)


def _grads(g, W, inp, acts, mask, t, image_mask=None):
    return training_loss_and_grads(W, g, inp["backbone_features"], inp["vl_mask"], inp["state"],
                                   inp["embodiment_id"], acts, inp["init_noise"], t, mask, image_mask=image_mask)


@pytest.mark.parametrize("variant", ["plain", "vlln", "split"])
def test_loss_equals_the_numpy_oracle(variant):
    g = dataclasses.replace(G, num_layers=4, attend_text_every_n_blocks=1) if variant == "split" else G
    g, W, inp, acts, mask, t = _case(g, vlln=variant == "vlln")
    img = None
    if variant == "split":
        img = synth.make_image_mask(dataclasses.replace(synth.WORKLOADS["tiny"], geom=g, batch=2), seed=8)
    want, _ = _np_loss(g, W, inp, acts, mask, t, img)
    got, _ = _grads(g, W, inp, acts, mask, t, img)
    assert got == pytest.approx(want, rel=1e-12)


GROUPS = [None, "t_enc.", "blk0.ada.", "blk0.k.", "blk0.v.", "blk1.q.", "blk1.ff1.", "blk0.ln3.", "out.",
          "state_enc.", "act_enc.W2.", "act_dec.l1.", "vlln."]


@pytest.mark.parametrize("group", GROUPS)
def test_directional_derivative_matches_central_differences(group):
    """(L(W + h d) - L(W - h d)) / 2h of the numpy oracle equals sum(grad * d)
    for a random direction d over all weights or one group of them."""
    g, W, inp, acts, mask, t = _case(vlln=group == "vlln.", seed=5)
    _, grads = _grads(g, W, inp, acts, mask, t)
    r = np.random.default_rng(17)
    d = {k: (r.standard_normal(v.shape) * (np.std(v) + 1e-3) if group is None or k.startswith(group)
             else np.zeros(v.shape)) for k, v in W.items()}
    assert any(np.any(v) for v in d.values())
    h = 1e-5
    lp, _ = _np_loss(g, {k: W[k] + h * d[k] for k in W}, inp, acts, mask, t)
    lm, _ = _np_loss(g, {k: W[k] - h * d[k] for k in W}, inp, acts, mask, t)
    fd = (lp - lm) / (2 * h)
    an = sum(float((grads[k] * d[k]).sum()) for k in W)
    assert abs(an) > 1e-8
    # the difference quotient carries the rounding of two O(|L|) losses in
    # double divided by 2h (about 1e-11 here), and an O(h^2) truncation term
    tol_abs = 100 * np.finfo(np.float64).eps * max(abs(lp), abs(lm)) / (2 * h)
    assert fd == pytest.approx(an, rel=2e-6, abs=tol_abs)


def test_decoder_output_bias_has_the_closed_form_gradient():
    """d L / d act_dec.l2.b[c] = 2 sum over category-c samples and action
    tokens of mask (pred - (a - e)), divided by sum(mask) + 1e-6."""
    g, W, inp, acts, mask, t = _case(ids=(1, 0, 1), seed=9)
    _, pred = _np_loss(g, W, inp, acts, mask, t)
    _, grads = _grads(g, W, inp, acts, mask, t)
    r = mask * (pred - (acts - inp["init_noise"].astype(np.float64)))
    denom = mask.sum() + 1e-6
    ids = inp["embodiment_id"]
    for c in range(g.num_embodiments):
        want = 2.0 * r[ids == c].sum(axis=(0, 1)) / denom
        np.testing.assert_allclose(grads["act_dec.l2.b"][c], want, rtol=1e-10, atol=1e-14)


def test_parameters_off_the_path_get_zero_gradient():
    g, W, inp, acts, mask, t = _case(ids=(0, 0))
    _, grads = _grads(g, W, inp, acts, mask, t)
    for name, v in grads.items():
        if name.split(".")[0] in ("state_enc", "act_enc", "act_dec"):
            assert not np.any(v[1]), name          # category 1 is never used
            assert np.any(v[0]), name
    loss, grads = _grads(g, W, inp, acts, np.zeros_like(mask), t)
    assert loss == 0.0
    assert all(not np.any(v) for v in grads.values())


def test_gradient_on_the_generators_training_draws():
    """The training recipe of the input generator (t ~ Beta(1.5, 1), masked
    action-dimension padding): the gradient still matches central differences."""
    w = dataclasses.replace(synth.WORKLOADS["tiny"], batch=3, fixed_ids=(1, 0, 1))
    g = w.geom
    W = {k: np.asarray(v, np.float64) for k, v in synth.make_weights(g).items()}
    inp = synth.make_inputs(w, seed=12)
    tr = synth.make_training_inputs(w, seed=12)
    args = (g, inp["backbone_features"], inp["vl_mask"], inp["state"], inp["embodiment_id"],
            tr["actions"], tr["noise"], tr["t"], tr["action_mask"])
    loss, grads = training_loss_and_grads(W, *args)
    assert np.isfinite(loss) and loss > 0
    r = np.random.default_rng(2)
    d = {k: r.standard_normal(v.shape) * (np.std(v) + 1e-3) for k, v in W.items()}
    h = 1e-5
    lp, _ = oracle.training_loss({k: W[k] + h * d[k] for k in W}, *args)
    lm, _ = oracle.training_loss({k: W[k] - h * d[k] for k in W}, *args)
    an = sum(float((grads[k] * d[k]).sum()) for k in W)
    tol_abs = 100 * np.finfo(np.float64).eps * max(abs(lp), abs(lm)) / (2 * h)
    assert (lp - lm) / (2 * h) == pytest.approx(an, rel=2e-6, abs=tol_abs)
