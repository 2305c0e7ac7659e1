"""Model-level pins of the oracle (CPU only): invariants and closed forms.

Each test would fail under a plausible mistake in the composition: a dropped
residual, a wrong AdaLN order, a swapped concatenation, a wrong category index,
a wrong self/cross alternation, an Euler step of the wrong size or sign.
"""

import dataclasses

import numpy as np
import pytest

import oracle
import synth

TINY = synth.WORKLOADS["tiny"]
G = TINY.geom
rng = np.random.default_rng(77)


@pytest.fixture(scope="module")
def W():
    return synth.make_weights(G)


def _inputs(batch=1, seq=64, ids=None, seed=1):
    w = dataclasses.replace(TINY, batch=batch, seq=seq,
                            fixed_ids=tuple(ids) if ids is not None else (0,))
    return synth.make_inputs(w, seed=seed)


def _run(W, inp, K=4, g=G, **kw):
    return oracle.get_action(W, g, inp["backbone_features"], inp["vl_mask"], inp["state"],
                             inp["embodiment_id"], inp["init_noise"], K, **kw)


def _copy(W):
    return {k: np.array(v, copy=True) for k, v in W.items()}


# ---------------------------------------------------------------- invariants

def test_masked_backbone_tokens_have_no_influence(W):
    inp = _inputs(batch=2, ids=[0, 1])
    inp["vl_mask"][0, 40:] = 0
    inp["vl_mask"][1, ::3] = 0
    out = _run(W, inp)
    feats = inp["backbone_features"].copy()
    feats[inp["vl_mask"] == 0] = rng.normal(size=(int((inp["vl_mask"] == 0).sum()), G.backbone_dim)) * 100
    out2 = _run(W, dict(inp, backbone_features=feats))
    np.testing.assert_array_equal(out, out2)
    # a valid token does matter
    feats[0, 0] += 1.0
    assert not np.array_equal(out, _run(W, dict(inp, backbone_features=feats)))


def test_zero_velocity_head_leaves_noise(W):
    W0 = _copy(W)
    W0["act_dec.l2.W"][:] = 0
    W0["act_dec.l2.b"][:] = 0
    inp = _inputs(batch=2, ids=[1, 0])
    np.testing.assert_array_equal(_run(W0, inp), inp["init_noise"].astype(np.float64))


def test_one_step_is_noise_plus_velocity(W):
    inp = _inputs()
    m = oracle.Model(W, G)
    s, kvs = oracle.prepare_sample(m, inp["backbone_features"][0], inp["vl_mask"][0], inp["state"][0], 0)
    x0 = inp["init_noise"][0].astype(np.float64)
    v = oracle.velocity(m, x0, 0.0, s, kvs, 0)
    np.testing.assert_array_equal(_run(W, inp, K=1)[0], x0 + v)


def test_decoder_bias_signature_routes_by_category():
    g = dataclasses.replace(G, num_embodiments=4)
    Wg = synth.make_weights(g)
    Wg["act_dec.l1.W"][:] = 0
    Wg["act_dec.l1.b"][:] = 0
    Wg["act_dec.l2.W"][:] = 0
    for c in range(4):
        Wg["act_dec.l2.b"][c] = c
    inp = _inputs(batch=4, ids=[2, 0, 3, 1])
    out = _run(Wg, inp, g=g)
    expect = inp["init_noise"].astype(np.float64) + np.array([2, 0, 3, 1], np.float64)[:, None, None]
    np.testing.assert_array_equal(out, expect)


def test_routing_equals_running_alone_with_category_moved_to_zero(W):
    inp = _inputs(batch=2, ids=[1, 0])
    mixed = _run(W, inp)
    # sample 0 (category 1) alone, in a model whose category 0 holds category 1's weights
    Wm = _copy(W)
    for name, v in Wm.items():
        if v.ndim >= 2 and v.shape[0] == G.num_embodiments and name.split(".")[0] in (
                "state_enc", "act_enc", "act_dec"):
            v[0] = W[name][1]
    alone = {k: v[:1] for k, v in inp.items()}
    alone["embodiment_id"] = np.array([0], np.int32)
    np.testing.assert_array_equal(_run(Wm, alone)[0], mixed[0])
    # and the category matters
    other = dict(alone, embodiment_id=np.array([0], np.int32))
    assert not np.array_equal(_run(W, other)[0], mixed[0])


def test_batch_permutation_equivariance(W):
    inp = _inputs(batch=3, ids=[0, 1, 1])
    inp["vl_mask"][1, 10:] = 0
    out = _run(W, inp)
    perm = [2, 0, 1]
    pinp = {k: v[perm] for k, v in inp.items()}
    np.testing.assert_array_equal(_run(W, pinp), out[perm])


def test_horizon_permutation_equivariance(W):
    # no positional encoding over the horizon: permuting noise rows permutes the output
    inp = _inputs()
    out = _run(W, inp)
    perm = rng.permutation(G.action_horizon)
    pinp = dict(inp, init_noise=inp["init_noise"][:, perm])
    np.testing.assert_allclose(_run(W, pinp), out[:, perm], rtol=0, atol=1e-13)


def test_constant_velocity_integrates_exactly(W):
    # all DiT and encoder matrices zero: v no longer depends on x or t, and K
    # Euler steps of size 1/K add exactly v for every K
    Wz = _copy(W)
    for name, v in Wz.items():
        if name.endswith((".w", ".W")) and not name.startswith("act_dec"):
            v[:] = 0
    inp = _inputs()
    deltas = [(_run(Wz, inp, K=K) - inp["init_noise"])[0] for K in (1, 2, 3, 4, 8)]
    for d in deltas[1:]:
        np.testing.assert_allclose(d, deltas[0], rtol=0, atol=1e-14)
    assert np.abs(deltas[0]).max() > 1e-3


def test_alternation_even_layers_cross_odd_layers_self():
    g = dataclasses.replace(G, num_layers=4)
    Wg = synth.make_weights(g)
    inp = _inputs()
    feats2 = inp["backbone_features"] + 1.0
    # silence the attention outputs of the even layers: the backbone no longer matters
    We = _copy(Wg)
    for l in (0, 2):
        We[f"blk{l}.o.w"][:] = 0
    np.testing.assert_array_equal(_run(We, inp, g=g), _run(We, dict(inp, backbone_features=feats2), g=g))
    # silence only layer 0: layer 2 still reads the backbone
    W0 = _copy(Wg)
    W0["blk0.o.w"][:] = 0
    assert not np.array_equal(_run(W0, inp, g=g), _run(W0, dict(inp, backbone_features=feats2), g=g))
    # silence the odd layers: the backbone still matters
    Wo = _copy(Wg)
    for l in (1, 3):
        Wo[f"blk{l}.o.w"][:] = 0
    assert not np.array_equal(_run(Wo, inp, g=g), _run(Wo, dict(inp, backbone_features=feats2), g=g))


def test_sample_without_valid_tokens_sees_zero_attention(W):
    inp = _inputs()
    inp["vl_mask"][:] = 0
    out = _run(W, inp)
    assert np.isfinite(out).all()
    # same as one valid token whose values are all zero (cross V weights and biases zeroed)
    Wv = _copy(W)
    Wv["blk0.v.w"][:] = 0
    Wv["blk0.v.b"][:] = 0
    one = dict(inp, vl_mask=inp["vl_mask"].copy())
    one["vl_mask"][0, 5] = 1
    np.testing.assert_array_equal(_run(Wv, one), out)


# ---------------------------------------------------------------- closed forms

def _zero_block(W, layer):
    Wb = _copy(W)
    for n in ("q", "k", "v", "o", "ff1", "ff2", "ada"):
        Wb[f"blk{layer}.{n}.w"][:] = 0
    return Wb


@pytest.mark.parametrize("layer", [0, 1])
def test_block_residuals_closed_form(W, layer):
    # Q = K = 0 (uniform attention), V = b_v for every key, O = identity:
    # attention adds b_v + b_o; the MLP adds GELU(b_1) W_2 + b_2 = b_2 with W_2 = 0.
    Wb = _zero_block(W, layer)
    D = G.hidden
    Wb[f"blk{layer}.o.w"][:] = np.eye(D, dtype=np.float32)
    m = oracle.Model(Wb, G)
    h = rng.normal(size=(G.action_horizon + 1, D))
    temb = rng.normal(size=D)
    kv = None
    if layer % 2 == 0:
        bv = m[f"blk{layer}.v.b"]
        kv = (np.zeros((9, D)), np.repeat(bv[None], 9, axis=0))
    out = oracle.dit_block(m, layer, h, temb, kv)
    expect = h + m[f"blk{layer}.v.b"] + m[f"blk{layer}.o.b"] + m[f"blk{layer}.ff2.b"]
    np.testing.assert_allclose(out, expect, rtol=0, atol=1e-12)


def test_adaln_scale_then_shift_closed_form():
    D = 8
    a = 3.0
    h = np.tile(np.array([a, -a] * (D // 2)), (2, 1))       # mean 0, variance a^2
    s = rng.normal(size=D)
    t = rng.normal(size=D)
    out = oracle.ada_layer_norm(h, rng.normal(size=5), np.zeros((2 * D, 5)), np.concatenate([s, t]), 1e-5)
    n = a / np.sqrt(a * a + 1e-5)
    expect = np.array([n, -n] * (D // 2)) * (1.0 + s) + t
    np.testing.assert_allclose(out, np.tile(expect, (2, 1)), rtol=1e-14, atol=1e-14)


def test_timestep_embedding_with_zero_weights_is_output_bias(W):
    Wz = _copy(W)
    Wz["t_enc.l1.w"][:] = 0
    Wz["t_enc.l1.b"][:] = 0
    Wz["t_enc.l2.w"][:] = 0
    m = oracle.Model(Wz, G)
    np.testing.assert_array_equal(oracle.timestep_embedding(m, 250.0), m["t_enc.l2.b"])


def test_action_encoder_concatenates_actions_first(W):
    D = G.hidden
    x = rng.normal(size=(G.action_horizon, G.action_dim))
    # zero the first D input rows of W2: only the timestep half remains
    Wa = _copy(W)
    Wa["act_enc.W2.W"][:, :D, :] = 0
    m = oracle.Model(Wa, G)
    e1 = oracle.action_encoder(m, x, 250.0, 1)
    e2 = oracle.action_encoder(m, x + 5.0, 250.0, 1)
    np.testing.assert_array_equal(e1, e2)
    assert not np.array_equal(e1, oracle.action_encoder(m, x, 500.0, 1))
    # zero the last D rows: only the action half remains
    Wt = _copy(W)
    Wt["act_enc.W2.W"][:, D:, :] = 0
    m = oracle.Model(Wt, G)
    np.testing.assert_array_equal(oracle.action_encoder(m, x, 250.0, 1), oracle.action_encoder(m, x, 750.0, 1))
    assert not np.array_equal(oracle.action_encoder(m, x, 250.0, 1), oracle.action_encoder(m, x + 5.0, 250.0, 1))


def test_category_mlp_relu_between_layers(W):
    D = G.hidden
    Wr = _copy(W)
    Wr["state_enc.l1.W"][:] = 0
    b1 = np.where(np.arange(D) % 2 == 0, -1.0, 2.0).astype(np.float32)
    Wr["state_enc.l1.b"][1] = b1
    Wr["state_enc.l2.W"][1] = np.eye(D, dtype=np.float32)
    m = oracle.Model(Wr, G)
    out = oracle.state_encoder(m, rng.normal(size=(1, G.state_dim)), 1)
    expect = np.where(np.arange(D) % 2 == 0, 0.0, 2.0) + m.cat("state_enc.l2.b", 1)
    np.testing.assert_array_equal(out[0], expect)


def test_state_token_comes_first(W):
    # the decoder output of row 0 is dropped: zero the action encoder (all action
    # tokens equal) and the state feature still reaches the actions only through
    # attention; changing the state changes the output
    inp = _inputs()
    out = _run(W, inp)
    inp2 = dict(inp, state=inp["state"] + 1.0)
    assert not np.array_equal(out, _run(W, inp2))
    assert out.shape == (1, G.action_horizon, G.action_dim)


def test_bad_embodiment_id_rejected(W):
    inp = _inputs()
    inp["embodiment_id"] = np.array([G.num_embodiments], np.int32)
    with pytest.raises(ValueError):
        _run(W, inp)


def test_dropped_row_is_the_state_token(W):
    # With every attention and MLP output silenced and proj_out the identity, a
    # token's velocity depends on that token alone.  Perturbing noise row i must
    # then change output row i only: this fails if the state token were not the
    # first row or if the wrong decoded row were dropped.
    Wi = _copy(W)
    for l in range(G.num_layers):
        for n in ("o", "ff2"):
            Wi[f"blk{l}.{n}.w"][:] = 0
            Wi[f"blk{l}.{n}.b"][:] = 0
    Wi["out.proj.w"][:] = np.eye(G.hidden, dtype=np.float32)
    inp = _inputs()
    out = _run(Wi, inp, K=1)
    for i in (0, 3, G.action_horizon - 1):
        noise = inp["init_noise"].copy()
        noise[0, i] += 0.5
        out2 = _run(Wi, dict(inp, init_noise=noise), K=1)
        changed = np.nonzero(np.abs(out2 - out)[0].max(axis=1) > 0)[0].tolist()
        assert changed == [i]


def test_loop_feeds_discretised_timesteps(W):
    # K = 2: t = 0, 0.5 -> t_discretized = 0, 500 (1000 buckets); dt = 0.5
    inp = _inputs()
    m = oracle.Model(W, G)
    s, kvs = oracle.prepare_sample(m, inp["backbone_features"][0], inp["vl_mask"][0], inp["state"][0], 0)
    x = inp["init_noise"][0].astype(np.float64)
    x = x + 0.5 * oracle.velocity(m, x, 0.0, s, kvs, 0)
    x = x + 0.5 * oracle.velocity(m, x, 500.0, s, kvs, 0)
    np.testing.assert_array_equal(_run(W, inp, K=2)[0], x)
    # the timestep does reach the network
    x1 = inp["init_noise"][0].astype(np.float64)
    assert not np.array_equal(oracle.velocity(m, x1, 0.0, s, kvs, 0), oracle.velocity(m, x1, 0.5, s, kvs, 0))


def test_mlp_branch_is_gelu_of_affine_layer_norm(W):
    # attention silenced, FF1/FF2 = identity embeddings: the block adds
    # GELU(LN3(h)) with LN3's gain and bias (expected value from torch)
    import torch
    layer = 1
    D, F = G.hidden, G.mlp_hidden
    Wb = _copy(W)
    p = f"blk{layer}."
    Wb[p + "o.w"][:] = 0
    Wb[p + "o.b"][:] = 0
    Wb[p + "ff1.w"][:] = np.eye(F, D, dtype=np.float32)
    Wb[p + "ff1.b"][:] = 0
    Wb[p + "ff2.w"][:] = np.eye(D, F, dtype=np.float32)
    Wb[p + "ff2.b"][:] = 0
    m = oracle.Model(Wb, G)
    h = rng.normal(size=(5, D))
    out = oracle.dit_block(m, layer, h, rng.normal(size=D), None)
    th = torch.from_numpy(h)
    ln = torch.nn.functional.layer_norm(th, (D,), torch.from_numpy(m[p + "ln3.g"]),
                                        torch.from_numpy(m[p + "ln3.b"]), eps=G.ln_eps)
    expect = (th + torch.nn.functional.gelu(ln)).numpy()
    np.testing.assert_allclose(out, expect, rtol=1e-12, atol=1e-12)


def test_timestep_encoder_is_linear_silu_linear(W):
    import torch
    D = G.hidden
    Wt = _copy(W)
    Wt["t_enc.l1.w"][:] = 0
    Wt["t_enc.l2.w"][:] = np.eye(D, dtype=np.float32)
    m = oracle.Model(Wt, G)
    expect = torch.nn.functional.silu(torch.from_numpy(m["t_enc.l1.b"])).numpy() + m["t_enc.l2.b"]
    np.testing.assert_allclose(oracle.timestep_embedding(m, 750.0), expect, rtol=1e-13, atol=1e-15)


def test_action_encoder_applies_swish_to_w2(W):
    import torch
    D = G.hidden
    Wa = _copy(W)
    for n in ("W1", "W2", "W3"):
        Wa[f"act_enc.{n}.W"][:] = 0
        Wa[f"act_enc.{n}.b"][:] = 0
    Wa["act_enc.W2.W"][0, D:, :] = np.eye(D, dtype=np.float32)    # tau half -> identity
    Wa["act_enc.W3.W"][0] = np.eye(D, dtype=np.float32)
    m = oracle.Model(Wa, G)
    x = rng.normal(size=(G.action_horizon, G.action_dim))
    tau = oracle.sinusoidal_embedding(250.0, D)
    expect = torch.nn.functional.silu(torch.from_numpy(tau)).numpy()
    out = oracle.action_encoder(m, x, 250.0, 0)
    np.testing.assert_allclose(out, np.broadcast_to(expect, out.shape), rtol=1e-13, atol=1e-15)


# ---------------------------------------------------------------- image/text split of the cross layers

G4 = dataclasses.replace(G, num_layers=4)


@pytest.fixture(scope="module")
def W4():
    return synth.make_weights(G4)


def _split_inputs(seed=3):
    w = dataclasses.replace(TINY, geom=G4, batch=2, seq=64, valid_min=40, fixed_ids=(0, 1))
    inp = synth.make_inputs(w, seed=seed)
    img = np.zeros_like(inp["vl_mask"])
    img[:, :20] = 1   # the first 20 tokens of every sample are image tokens
    return inp, img


def test_split_layer_kinds_follow_the_page_rule():
    """Cross block idx attends to text when idx % (2 n) == 0, else to images
    ([ARCH] "AlternateVLDiT variant"): for 8 layers, blocks 0, 2, 4, 6 are
    text/text/text/text (n = 1), text/image/text/image (n = 2) and
    text/image/image/text (n = 3)."""
    mask = np.ones(6, dtype=np.uint8)
    img = np.array([1, 1, 1, 0, 0, 0], dtype=np.uint8)
    text_keys, image_keys = [False] * 3 + [True] * 3, [True] * 3 + [False] * 3
    expect = {1: "TTTT", 2: "TITI", 3: "TIIT"}
    for n, kinds in expect.items():
        for idx, kind in zip((0, 2, 4, 6), kinds):
            got = list(oracle.cross_key_mask(idx, mask, img, n))
            assert got == (text_keys if kind == "T" else image_keys), (n, idx)
    # n = 0: no split, every valid token
    assert list(oracle.cross_key_mask(2, mask, img, 0)) == [True] * 6
    # padding never enters, image or not
    pad = np.array([1, 1, 0, 1, 0, 1], dtype=np.uint8)
    assert list(oracle.cross_key_mask(2, pad, img, 2)) == [True, True, False, False, False, False]


def test_split_off_is_the_plain_model(W4):
    inp, img = _split_inputs()
    a = _run(W4, inp, g=G4)
    b = _run(W4, inp, g=G4, image_mask=img)
    np.testing.assert_array_equal(a, b)


def test_split_n1_image_tokens_have_no_influence(W4):
    """n = 1: every cross block attends to text, so image-token features do not
    matter; text-token features do."""
    g1 = dataclasses.replace(G4, attend_text_every_n_blocks=1)
    inp, img = _split_inputs()
    base = _run(W4, inp, g=g1, image_mask=img)
    pert = dict(inp)
    f = inp["backbone_features"].copy()
    f[:, :20] += np.float32(3.0)        # image tokens only
    pert["backbone_features"] = f
    np.testing.assert_array_equal(_run(W4, pert, g=g1, image_mask=img), base)
    f2 = inp["backbone_features"].copy()
    f2[:, 25] += np.float32(3.0)        # one valid text token
    pert["backbone_features"] = f2
    assert np.abs(_run(W4, pert, g=g1, image_mask=img) - base).max() > 1e-6


def test_split_n2_alternates_text_and_image(W4):
    """n = 2 with 4 layers: block 0 attends to text, block 2 to images; each
    kind of token then changes the output, and each block's K/V holds exactly
    its kind of valid token."""
    g2 = dataclasses.replace(G4, attend_text_every_n_blocks=2)
    inp, img = _split_inputs()
    m = oracle.Model(W4, g2)
    sv = int(inp["vl_mask"][0].sum())
    _, kvs = oracle.prepare_sample(m, inp["backbone_features"][0], inp["vl_mask"][0], inp["state"][0], 0,
                                   img[0], 2)
    assert kvs[0][0].shape[0] == sv - 20 and kvs[2][0].shape[0] == 20
    base = _run(W4, inp, g=g2, image_mask=img)
    for cols in (slice(0, 20), slice(25, 26)):
        pert = dict(inp)
        f = inp["backbone_features"].copy()
        f[:, cols] += np.float32(3.0)
        pert["backbone_features"] = f
        assert np.abs(_run(W4, pert, g=g2, image_mask=img) - base).max() > 1e-6
    # with no image token, block 2 has no key: its attention output is zero and
    # only its bias reaches the residual, whatever the features
    none = np.zeros_like(img)
    r0 = _run(W4, inp, g=g2, image_mask=none)
    zero_k = _copy(W4)
    zero_k["blk2.k.w"][:] = 0
    zero_k["blk2.v.w"][:] = 0
    zero_k["blk2.o.w"][:] = 0
    zero_k["blk2.k.b"][:] = 0
    zero_k["blk2.v.b"][:] = 0
    g0 = dataclasses.replace(G4, attend_text_every_n_blocks=0)
    np.testing.assert_allclose(r0, _run(zero_k, inp, g=g0), rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------- vision-language layer norm (vlln)

GV = dataclasses.replace(G, vlln=True)


@pytest.fixture(scope="module")
def WV():
    return synth.make_weights(GV)


def _token_affine(feats, seed=5):
    """Each token's features scaled by a_t in [0.5, 3] and shifted by c_t in [-2, 2]."""
    r = np.random.default_rng(seed)
    B, S, _ = feats.shape
    a = r.uniform(0.5, 3.0, size=(B, S, 1)).astype(np.float32)
    c = r.uniform(-2.0, 2.0, size=(B, S, 1)).astype(np.float32)
    return (feats * a + c).astype(np.float32)


def test_vlln_makes_the_head_blind_to_each_tokens_scale_and_shift(WV):
    """A LayerNorm over each token's features removes that token's mean and
    scale: with vlln the actions do not change (up to the eps under the square
    root, relative 1e-5, and the fp32 rounding of the moved features); without
    it they change by more than 1e-3."""
    inp = _inputs(seed=9)
    base = _run(WV, inp, g=GV)
    moved = dict(inp)
    moved["backbone_features"] = _token_affine(inp["backbone_features"])
    np.testing.assert_allclose(_run(WV, moved, g=GV), base, rtol=1e-4, atol=1e-5)
    plain = {k: v for k, v in WV.items() if not k.startswith("vlln.")}
    assert np.abs(_run(plain, moved, g=G) - _run(plain, inp, g=G)).max() > 1e-3


def test_vlln_zero_gain_leaves_only_its_bias(WV):
    """vlln.g = 0: every token becomes vlln.b, so the features do not matter."""
    W0 = _copy(WV)
    W0["vlln.g"][:] = 0
    inp = _inputs(seed=9)
    other = dict(inp)
    other["backbone_features"] = -3.0 * inp["backbone_features"] + 1.0
    np.testing.assert_allclose(_run(W0, other, g=GV), _run(W0, inp, g=GV), rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------- training objective (forward)

def _train_inputs(seed=21, batch=2):
    inp = _inputs(batch=batch, ids=(0, 1)[:batch], seed=seed)
    r = np.random.default_rng(seed)
    shape = inp["init_noise"].shape
    acts = r.standard_normal(shape).astype(np.float32)
    mask = (r.uniform(size=shape) < 0.7).astype(np.float32)
    return inp, acts, mask


def _loss(W, inp, acts, noise, t, mask, g=G):
    return oracle.training_loss(W, g, inp["backbone_features"], inp["vl_mask"], inp["state"],
                                inp["embodiment_id"], acts, noise, np.asarray(t, np.float64), mask)


def test_training_loss_of_a_zero_velocity_head_is_the_masked_target_energy(W):
    """pred = 0 (decoder output layer zeroed): the loss is
    sum(mask * (a - e)^2) / (sum(mask) + 1e-6), whatever t."""
    W0 = _copy(W)
    W0["act_dec.l2.W"][:] = 0
    W0["act_dec.l2.b"][:] = 0
    inp, acts, mask = _train_inputs()
    noise = inp["init_noise"]
    target = acts.astype(np.float64) - noise.astype(np.float64)
    m64 = mask.astype(np.float64)
    want = float((m64 * target ** 2).sum() / (m64.sum() + 1e-6))
    for t in ([0.3, 0.9], [0.0, 1.0]):
        loss, pred = _loss(W0, inp, acts, noise, t, mask)
        assert np.all(pred == 0)
        assert loss == pytest.approx(want, rel=1e-12)


def test_training_prediction_at_t0_is_the_first_euler_velocity(W):
    """t = 0: x_t is the noise and t_discretized is 0, so the predicted velocity
    is v(noise, 0) = get_action(K = 1) - noise."""
    inp, acts, mask = _train_inputs()
    _, pred = _loss(W, inp, acts, inp["init_noise"], [0.0, 0.0], mask)
    ref = _run(W, inp, K=1) - inp["init_noise"].astype(np.float64)
    np.testing.assert_allclose(pred, ref, rtol=1e-12, atol=1e-12)


def test_training_prediction_at_t_half_is_the_second_euler_velocity(W):
    """With actions = noise = x1 (so x_t = x1 for every t) and t = 0.5
    (t_discretized 500), the prediction is the velocity of the second step of
    the K = 2 loop: (x2 - x1) / 0.5, with x1 = noise + 0.5 v(noise, 0)."""
    inp, _, mask = _train_inputs()
    e = inp["init_noise"].astype(np.float64)
    v0 = _run(W, inp, K=1) - e
    x1 = e + 0.5 * v0
    x2 = _run(W, inp, K=2)
    _, pred = _loss(W, inp, x1, x1, [0.5, 0.5], mask)
    np.testing.assert_allclose(pred, (x2 - x1) / 0.5, rtol=1e-9, atol=1e-10)


def test_training_loss_interpolates_noise_and_actions(W):
    """x_t = (1 - t) noise + t actions: at t = 1 the prediction depends on the
    actions only (changing the noise changes only the target), at t = 0 on the
    noise only."""
    inp, acts, mask = _train_inputs()
    e = inp["init_noise"]
    _, p1 = _loss(W, inp, acts, e, [1.0, 1.0], mask)
    _, p1b = _loss(W, inp, acts, (e + 1.0).astype(np.float32), [1.0, 1.0], mask)
    np.testing.assert_array_equal(p1, p1b)
    _, p0 = _loss(W, inp, acts, e, [0.0, 0.0], mask)
    _, p0b = _loss(W, inp, (acts + 1.0).astype(np.float32), e, [0.0, 0.0], mask)
    np.testing.assert_array_equal(p0, p0b)


def test_training_loss_of_a_perfect_predictor_is_zero(W):
    """At t = 0 the prediction is v(noise, 0) whatever the actions are; with
    actions = noise + v(noise, 0) the target actions - noise equals that
    prediction, so the loss vanishes (and a flipped target would give 4 v^2)."""
    inp, _, mask = _train_inputs()
    e = inp["init_noise"].astype(np.float64)
    v0 = _run(W, inp, K=1) - e
    loss, pred = _loss(W, inp, e + v0, inp["init_noise"], [0.0, 0.0], mask)
    np.testing.assert_allclose(pred, v0, rtol=1e-12, atol=1e-12)
    assert loss < 1e-20
    loss_off, _ = _loss(W, inp, e + v0 + 0.5, inp["init_noise"], [0.0, 0.0], mask)
    m64 = mask.astype(np.float64)
    assert loss_off == pytest.approx(0.25 * m64.sum() / (m64.sum() + 1e-6), rel=1e-9)


def test_training_time_is_truncated_to_its_bucket(W):
    """t_discretized = floor(t * buckets): with actions = noise (x_t the same
    for every t) the prediction depends on the bucket alone, so t = 0.5009
    predicts as t = 0.5 (bucket 500) and t = 0.4999 as t = 0.499 (bucket 499),
    and buckets 499 and 500 predict differently."""
    inp, _, mask = _train_inputs()
    e = inp["init_noise"]

    def pred(t):
        return _loss(W, inp, e, e, [t, t], mask)[1]

    p500 = pred(0.5)
    np.testing.assert_array_equal(pred(0.5009), p500)
    p499 = pred(0.499)
    np.testing.assert_array_equal(pred(0.4999), p499)
    assert np.abs(p500 - p499).max() > 1e-6


# ---------------------------------------------------------------- composition of the pieces

def test_action_encoder_ends_in_its_third_layer(W):
    """W3[c] = 0 leaves b3[c] on every action token, whatever the actions and t
    (the encoder's last step is the W3 layer, [ARCH] multi-embodiment action
    encoder)."""
    W0 = _copy(W)
    W0["act_enc.W3.W"][1] = 0
    m = oracle.Model(W0, G)
    x = rng.normal(size=(G.action_horizon, G.action_dim))
    for td in (0.0, 750.0):
        out = oracle.action_encoder(m, x, td, 1)
        np.testing.assert_array_equal(out, np.broadcast_to(W0["act_enc.W3.b"][1].astype(np.float64), out.shape))
    assert not np.allclose(oracle.action_encoder(oracle.Model(W, G), x, 0.0, 1), W["act_enc.W3.b"][1])


def test_final_layer_is_output_adaln_then_proj_out_then_decoder(W):
    """out.ada.w = 0 with bias (scale = -1, shift = sigma) turns the final AdaLN
    into the constant sigma, so each step's velocity is
    decoder_c(proj_out(sigma)) for every token and input, and the K-step loop
    adds it once: x_K = noise + v (computed here with torch's linear and bmm)."""
    import torch
    W0 = _copy(W)
    D = G.hidden
    sigma = rng.normal(size=D).astype(np.float32)
    W0["out.ada.w"][:] = 0
    W0["out.ada.b"][:D] = -1.0
    W0["out.ada.b"][D:] = sigma
    inp = _inputs(batch=2, ids=[1, 0], seed=9)
    out = _run(W0, inp, K=4)
    t = lambda a: torch.from_numpy(np.asarray(a, np.float64))
    y = torch.nn.functional.linear(t(sigma), t(W0["out.proj.w"]), t(W0["out.proj.b"]))
    for b, c in enumerate((1, 0)):
        h1 = torch.relu(torch.bmm(y.view(1, 1, D), t(W0["act_dec.l1.W"][c:c + 1])) + t(W0["act_dec.l1.b"][c]))
        v = torch.bmm(h1, t(W0["act_dec.l2.W"][c:c + 1])) + t(W0["act_dec.l2.b"][c])
        want = inp["init_noise"][b].astype(np.float64) + v.numpy().reshape(1, G.action_dim)
        np.testing.assert_allclose(out[b], want, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("layer", [0, 1])
def test_attention_branch_sees_h_only_through_its_adaln(W, layer):
    """With the MLP branch zeroed, block(h) - h is the attention branch, whose
    queries (and, in self layers, keys and values) come from AdaLN(h).  A layer
    norm without eps ignores a per-row scale and shift of h, so the branch is
    the same for h and alpha_row * h + beta_row."""
    g = dataclasses.replace(G, ln_eps=0.0)
    W0 = _copy(W)
    W0[f"blk{layer}.ff2.w"][:] = 0
    W0[f"blk{layer}.ff2.b"][:] = 0
    m = oracle.Model(W0, g)
    inp = _inputs(seed=4)
    _, kvs = oracle.prepare_sample(m, inp["backbone_features"][0], inp["vl_mask"][0], inp["state"][0], 0)
    h = rng.normal(size=(G.action_horizon + 1, G.hidden))
    temb = oracle.timestep_embedding(m, 250.0)
    alpha = rng.uniform(0.5, 3.0, size=(h.shape[0], 1))
    beta = rng.normal(size=(h.shape[0], 1))
    h2 = alpha * h + beta
    kv = None if layer % 2 else kvs[layer]
    br = oracle.dit_block(m, layer, h, temb, kv) - h
    br2 = oracle.dit_block(m, layer, h2, temb, kv) - h2
    np.testing.assert_allclose(br2, br, rtol=1e-9, atol=1e-12)
    assert np.abs(br).max() > 1e-3


def test_modulation_sees_temb_only_through_silu(W):
    """t_enc.l2 = (0, -60) makes temb = -60, where SiLU is below 1e-24: every
    AdaLN (blocks and output) is then left with its bias, so zeroing all AdaLN
    weights changes nothing (AdaLN input SiLU(temb), [ARCH] norm1(h, temb))."""
    W1 = _copy(W)
    W1["t_enc.l2.w"][:] = 0
    W1["t_enc.l2.b"][:] = -60.0
    W2 = _copy(W1)
    for name in W2:
        if name.endswith("ada.w"):
            W2[name][:] = 0
    inp = _inputs(batch=2, ids=[0, 1], seed=6)
    np.testing.assert_allclose(_run(W1, inp, K=2), _run(W2, inp, K=2), rtol=1e-12, atol=1e-12)
    W3 = _copy(W1)
    W3["t_enc.l2.b"][:] = 2.0
    assert not np.allclose(_run(W3, inp, K=2), _run(dict(W3, **{k: W2[k] for k in W2 if k.endswith("ada.w")}), inp, K=2))
