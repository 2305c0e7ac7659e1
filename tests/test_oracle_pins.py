"""Pins of the oracle's elementary functions (CPU only).

Each test checks an oracle function against something other than its own
formula: a closed form, a mathematical identity, a different library's routine
(torch in float64), brute force on tiny inputs, or a value the pages print.
"""

import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
rng = np.random.default_rng(1234)


# ---------------------------------------------------------------- sinusoid

def test_sinusoid_at_zero_is_zeros_then_ones():
    e = oracle.sinusoidal_embedding(0.0, 256)
    assert e.shape == (256,)
    assert np.array_equal(e[:128], np.zeros(128))
    assert np.array_equal(e[128:], np.ones(128))


def test_sinusoid_pairs_lie_on_unit_circle():
    p = rng.uniform(0, 1000, size=7)
    e = oracle.sinusoidal_embedding(p, 64)
    np.testing.assert_allclose(e[:, :32] ** 2 + e[:, 32:] ** 2, 1.0, atol=1e-14)


def test_sinusoid_angle_addition():
    # sin(a+b) = sin a cos b + cos a sin b and cos(a+b) = cos a cos b - sin a sin b
    # hold feature by feature only if both halves use the same frequency at the
    # same index and the sin half comes first.
    a, b = 123.0, 456.0
    ea, eb, eab = (oracle.sinusoidal_embedding(x, 128) for x in (a, b, a + b))
    sa, ca, sb, cb = ea[:64], ea[64:], eb[:64], eb[64:]
    np.testing.assert_allclose(eab[:64], sa * cb + ca * sb, atol=1e-9)
    np.testing.assert_allclose(eab[64:], ca * cb - sa * sb, atol=1e-9)


def test_sinusoid_frequencies():
    # feature 0 has unit frequency; frequencies fall geometrically from 1 to
    # 10000^(-(h-1)/h): read them off with small arguments (sin x ~ x).
    h = 64
    eps = 1e-7
    e = oracle.sinusoidal_embedding(eps, 2 * h)
    freq = e[:h] / eps
    assert abs(freq[0] - 1.0) < 1e-12
    ratios = freq[1:] / freq[:-1]
    np.testing.assert_allclose(ratios, 10000.0 ** (-1.0 / h), rtol=1e-9)
    assert math.isclose(float(oracle.sinusoidal_embedding(math.pi / 2, 2 * h)[0]), 1.0, abs_tol=1e-15)


# ---------------------------------------------------------------- schedule

def test_euler_schedule_matches_page_k4():
    gold = json.load(open(os.path.join(GOLDEN, "euler_schedule_k4.json")))
    t, td, dt = oracle.euler_schedule(gold["num_steps"])
    assert t == gold["t_cont"]
    assert dt == gold["dt"]
    assert td == [0.0, 250.0, 500.0, 750.0]


def test_euler_schedule_k8_and_k1():
    t, td, dt = oracle.euler_schedule(8)
    assert td == [0.0, 125.0, 250.0, 375.0, 500.0, 625.0, 750.0, 875.0]
    assert dt == 0.125
    assert oracle.euler_schedule(1) == ([0.0], [0.0], 1.0)
    # step sizes always integrate to 1 over [0, 1)
    for k in (1, 2, 3, 5, 7, 16):
        _, _, dt = oracle.euler_schedule(k)
        assert abs(dt * k - 1.0) < 1e-15


# ---------------------------------------------------------------- linear layers

def test_linear_is_pytorch_nn_linear():
    x = rng.normal(size=(5, 7))
    w = rng.normal(size=(3, 7))
    b = rng.normal(size=3)
    ref = torch.nn.functional.linear(torch.from_numpy(x), torch.from_numpy(w), torch.from_numpy(b))
    np.testing.assert_allclose(oracle.linear(x, w, b), ref.numpy(), rtol=1e-13, atol=1e-13)


def test_category_linear_brute_force_and_bmm():
    gold = json.load(open(os.path.join(GOLDEN, "category_linear_example.json")))
    C, din, dout = gold["num_categories"], gold["input_dim"], 6   # small out for the loop
    W = rng.normal(size=(C, din, dout))
    b = rng.normal(size=(C, dout))
    ids = [3, 0, 9, 3]
    x = rng.normal(size=(len(ids), 2, din))
    ours = np.stack([oracle.category_linear(x[i], W, b, c) for i, c in enumerate(ids)])
    # per-element triple loop over the pages' [C, in, out] layout
    brute = np.zeros_like(ours)
    for i, c in enumerate(ids):
        for t in range(x.shape[1]):
            for o in range(dout):
                brute[i, t, o] = sum(x[i, t, j] * W[c, j, o] for j in range(din)) + b[c, o]
    np.testing.assert_allclose(ours, brute, rtol=1e-12, atol=1e-12)
    # the page's expression: bmm(x, W[ids]) + b[ids].unsqueeze(1)
    tW, tb, tx = (torch.from_numpy(a) for a in (W, b, x))
    tids = torch.tensor(ids)
    ref = torch.bmm(tx, tW[tids]) + tb[tids].unsqueeze(1)
    np.testing.assert_allclose(ours, ref.numpy(), rtol=1e-12, atol=1e-12)


def test_category_linear_layout_of_page_example():
    gold = json.load(open(os.path.join(GOLDEN, "category_linear_example.json")))
    C, din, dout = gold["num_categories"], gold["input_dim"], gold["hidden_dim"]
    W = np.zeros(gold["W_shape"])
    b = np.zeros(gold["b_shape"])
    assert W[0].shape == tuple(gold["matrix_shape"])
    # category c is selected as a whole [in, out] matrix: put a marker in W[c]
    W[7, 2, 5] = 1.0
    x = np.zeros((1, din)); x[0, 2] = 1.0
    y7 = oracle.category_linear(x, W, b, 7)
    y6 = oracle.category_linear(x, W, b, 6)
    assert y7.shape == (1, dout) and y7[0, 5] == 1.0 and y7.sum() == 1.0
    assert not y6.any()


def test_synth_weight_layout_matches_pages():
    g = synth.GEOM_FULL
    s = synth.weight_shapes(g)
    assert s["act_enc.W1.W"] == (32, g.action_dim, g.hidden)
    assert s["act_enc.W2.W"] == (32, 2 * g.hidden, g.hidden)     # cat([a, tau]) -> hidden
    assert s["state_enc.l1.W"] == (32, g.state_dim, g.hidden)
    assert s["act_dec.l2.W"] == (32, g.hidden, g.action_dim)
    assert s["blk0.k.w"] == (g.hidden, g.backbone_dim)            # even: cross to backbone
    assert s["blk1.k.w"] == (g.hidden, g.hidden)                  # odd: self


# ---------------------------------------------------------------- norms, activations

@pytest.mark.parametrize("affine", [False, True])
def test_layer_norm_vs_torch(affine):
    x = rng.normal(loc=0.3, scale=2.0, size=(9, 40))
    g = rng.normal(size=40) if affine else None
    bt = rng.normal(size=40) if affine else None
    ours = oracle.layer_norm(x, 1e-5, g, bt)
    ref = torch.nn.functional.layer_norm(torch.from_numpy(x), (40,),
                                         None if g is None else torch.from_numpy(g),
                                         None if bt is None else torch.from_numpy(bt), eps=1e-5)
    np.testing.assert_allclose(ours, ref.numpy(), rtol=1e-12, atol=1e-12)
    if not affine:
        np.testing.assert_allclose(ours.mean(-1), 0.0, atol=1e-13)
        np.testing.assert_allclose(ours.var(-1), 1.0 / (1.0 + 1e-5 / x.var(-1)), rtol=1e-12)


def test_gelu_vs_torch_and_identity():
    x = np.linspace(-8, 8, 1001)
    ref = torch.nn.functional.gelu(torch.from_numpy(x), approximate="none").numpy()
    np.testing.assert_allclose(oracle.gelu(x), ref, rtol=1e-13, atol=1e-15)
    # Phi(x) + Phi(-x) = 1  =>  gelu(x) - gelu(-x) = x
    np.testing.assert_allclose(oracle.gelu(x) - oracle.gelu(-x), x, atol=1e-14)
    assert oracle.gelu(np.array([0.0]))[0] == 0.0


def test_silu_vs_torch():
    x = np.linspace(-30, 30, 601)
    ref = torch.nn.functional.silu(torch.from_numpy(x)).numpy()
    np.testing.assert_allclose(oracle.silu(x), ref, rtol=1e-13, atol=1e-15)
    np.testing.assert_array_equal(oracle.relu(np.array([-1.0, 0.0, 2.5])), [0.0, 0.0, 2.5])


# ---------------------------------------------------------------- attention

def _sdpa(q, k, v, nh, mask=None):
    Nq, W = q.shape
    dh = W // nh
    tq = torch.from_numpy(q).view(Nq, nh, dh).transpose(0, 1)
    tk = torch.from_numpy(k).view(-1, nh, dh).transpose(0, 1)
    tv = torch.from_numpy(v).view(-1, nh, dh).transpose(0, 1)
    am = None if mask is None else torch.from_numpy(mask.astype(bool))[None, None, :]
    o = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, attn_mask=am)
    return o.transpose(0, 1).reshape(Nq, W).numpy()


def test_attention_vs_torch_sdpa():
    nh, dh = 4, 8
    q = rng.normal(size=(17, nh * dh))
    k = rng.normal(size=(23, nh * dh))
    v = rng.normal(size=(23, nh * dh))
    ours, probs = oracle.attention(q, k, v, nh, return_probs=True)
    np.testing.assert_allclose(ours, _sdpa(q, k, v, nh), rtol=1e-12, atol=1e-12)
    for p in probs:
        np.testing.assert_allclose(p.sum(axis=1), 1.0, atol=1e-12)
        assert (p >= 0).all()


def test_attention_masked_matches_sdpa_with_mask():
    nh, dh = 2, 16
    q = rng.normal(size=(5, nh * dh))
    k = rng.normal(size=(11, nh * dh))
    v = rng.normal(size=(11, nh * dh))
    mask = np.array([1, 0, 1, 1, 0, 0, 1, 0, 1, 1, 0], dtype=np.uint8)
    ours = oracle.attention(q, k[mask == 1], v[mask == 1], nh)
    np.testing.assert_allclose(ours, _sdpa(q, k, v, nh, mask), rtol=1e-12, atol=1e-12)


def test_attention_single_key_returns_its_value_row():
    nh, dh = 4, 8
    q = rng.normal(size=(6, nh * dh))
    k = rng.normal(size=(1, nh * dh))
    v = rng.normal(size=(1, nh * dh))
    np.testing.assert_array_equal(oracle.attention(q, k, v, nh), np.repeat(v, 6, axis=0))


def test_attention_no_keys_gives_zero():
    nh, dh = 4, 8
    q = rng.normal(size=(3, nh * dh))
    z = np.zeros((0, nh * dh))
    assert not oracle.attention(q, z, z, nh).any()


def test_attention_identical_keys_average_values():
    nh, dh = 2, 4
    q = rng.normal(size=(3, nh * dh))
    k = np.repeat(rng.normal(size=(1, nh * dh)), 5, axis=0)
    v = rng.normal(size=(5, nh * dh))
    np.testing.assert_allclose(oracle.attention(q, k, v, nh), np.repeat(v.mean(0, keepdims=True), 3, 0),
                               atol=1e-14)


# ---------------------------------------------------------------- bf16 decoding

def test_bf16_decode_exact():
    vals = np.array([1.0, -2.5, 0.0078125, 3.140625, -0.0], dtype=np.float32)
    bits = synth.f32_to_bf16_bits(vals)
    assert bits.tolist() == [0x3F80, 0xC020, 0x3C00, 0x4049, 0x8000]
    np.testing.assert_array_equal(oracle.to_f64(bits), vals.astype(np.float64))
    # round to nearest even at a tie: 1 + 2^-8 lies halfway between 1 and 1 + 2^-7
    assert synth.f32_to_bf16_bits(np.array([1.0 + 2 ** -8], np.float32))[0] == 0x3F80
    assert synth.f32_to_bf16_bits(np.array([1.0 + 3 * 2 ** -8], np.float32))[0] == 0x3F82
