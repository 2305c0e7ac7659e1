"""Pins of the seeded input generator that both the oracle and the GPU path
consume (CPU only).  It holds none of the model's arithmetic; these tests tie
it to the published definitions it implements."""

import numpy as np
import pytest
import torch

import synth


def test_splitmix64_published_sequence():
    """SplitMix64 (Steele, Lea and Flood 2014; Vigna's splitmix64.c): state +=
    0x9E3779B97F4A7C15, then the two xor-shift-multiply rounds.  The first five
    outputs from state 1234567 are the widely published example values (Rosetta
    Code, "Pseudo-random numbers/Splitmix64")."""
    want = [6457827717110365317, 3203168211198807973, 9817491932198370423,
            4593380528125082431, 16408922859458223821]
    assert [int(v) for v in synth.splitmix64_stream(1234567, 5)] == want


def test_splitmix64_offsets_are_positions_in_one_stream():
    full = synth.splitmix64_stream(99, 1000)
    np.testing.assert_array_equal(synth.splitmix64_stream(99, 10, offset=500), full[500:510])


def test_fnv1a64_published_vectors():
    """FNV-1a 64 (Fowler, Noll, Vo): offset basis 0xcbf29ce484222325, prime
    0x100000001b3; test vectors of the reference distribution."""
    assert synth.fnv1a64("") == 0xCBF29CE484222325
    assert synth.fnv1a64("a") == 0xAF63DC4C8601EC8C
    assert synth.fnv1a64("foobar") == 0x85944171F73967E8


def test_tensor_seeds_differ_by_name_and_base():
    a = synth.tensor_seed(0, "blk0.q.w")
    assert a != synth.tensor_seed(0, "blk0.k.w")
    assert a != synth.tensor_seed(1, "blk0.q.w")
    assert a == synth.tensor_seed(0, "blk0.q.w")


def test_uniforms_have_53_bits_in_unit_interval():
    u = synth.uniform53(5, 1 << 16)
    assert u.min() >= 0.0 and u.max() < 1.0
    assert np.all(u * 2.0 ** 53 == np.floor(u * 2.0 ** 53))
    assert abs(u.mean() - 0.5) < 5 * (1 / 12) ** 0.5 / 256


def test_normals_do_not_depend_on_chunking_and_have_unit_moments():
    n = 200_001
    z = synth.normal(11, n)
    np.testing.assert_array_equal(synth.normal(11, n, chunk=1 << 12), z)
    np.testing.assert_array_equal(synth.normal(11, 1001), z[:1001])
    assert abs(z.mean()) < 5 / n ** 0.5
    assert abs(z.var() - 1.0) < 5 * (2 / n) ** 0.5
    # Box-Muller pairs: z0^2 + z1^2 = -2 log(u1), an exponential of mean 2
    r2 = z[0:n - 1:2] ** 2 + z[1::2] ** 2
    assert abs(r2.mean() - 2.0) < 5 * 2 / (n / 2) ** 0.5


def test_randint_covers_its_inclusive_range():
    v = synth.randint(3, 20000, 0, 31)
    assert v.min() == 0 and v.max() == 31
    counts = np.bincount(v, minlength=32)
    assert counts.min() > 20000 / 32 * 0.8


def test_bf16_rounding_matches_torch():
    """Round to nearest, ties to even, as torch's float32 -> bfloat16 cast."""
    r = np.random.default_rng(0)
    x = np.concatenate([
        r.standard_normal(50000).astype(np.float32) * np.float32(3.0),
        # exact ties: the low 16 bits 0x8000 on even and odd bf16 mantissas
        (np.arange(1000, dtype=np.uint32) << np.uint32(16) | np.uint32(0x3F800000 + 0x8000)).view(np.float32),
        np.array([0.0, -0.0, 1e-40, -1e-40, 3.0e38, np.inf, -np.inf], np.float32),
    ])
    want = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(synth.f32_to_bf16_bits(x), want)
    back = synth.bf16_bits_to_f32(want)
    np.testing.assert_array_equal(back, torch.from_numpy(want.view(np.int16)).view(torch.bfloat16).float().numpy())


@pytest.mark.parametrize("name", ["tiny", "latency", "batched"])
def test_inputs_follow_the_workload_recipe(name):
    w = synth.workload(name, batch=min(synth.WORKLOADS[name].batch, 4))
    inp = synth.make_inputs(w)
    B, S = w.batch, w.seq
    assert inp["backbone_features"].shape == (B, S, w.geom.backbone_dim)
    assert inp["vl_mask"].shape == (B, S) and inp["vl_mask"].dtype == np.uint8
    assert inp["init_noise"].shape == (B, w.geom.action_horizon, w.geom.action_dim)
    ids = inp["embodiment_id"]
    assert ids.dtype == np.int32 and ids.min() >= 0 and ids.max() < w.geom.num_embodiments
    m = inp["vl_mask"].astype(bool)
    for b in range(B):
        sv = int(m[b].sum())
        assert m[b, :sv].all() and not m[b, sv:].any()      # valid prefix
        if name == "batched":
            assert 200 <= sv <= 600
        else:
            assert sv == S


def test_training_times_follow_beta_one_and_a_half_one():
    """t ~ Beta(1.5, 1): CDF x^1.5, mean 1.5 / 2.5 = 0.6, variance
    1.5 / (2.5^2 * 3.5)."""
    w = synth.workload("tiny", batch=40000)
    t = synth.make_training_inputs(w)["t"]
    n = len(t)
    assert t.min() >= 0.0 and t.max() < 1.0
    var = 1.5 / (2.5 ** 2 * 3.5)
    assert abs(t.mean() - 0.6) < 5 * (var / n) ** 0.5
    assert abs(t.var() - var) < 0.01 * var + 5e-4
    for x in (0.1, 0.25, 0.5, 0.75, 0.9):
        p = x ** 1.5
        assert abs((t <= x).mean() - p) < 5 * (p * (1 - p) / n) ** 0.5


def test_training_inputs_shapes_and_action_mask_prefixes():
    w = synth.workload("tiny", batch=64)
    d = synth.make_training_inputs(w)
    g = w.geom
    assert d["actions"].shape == d["noise"].shape == d["action_mask"].shape == (64, g.action_horizon, g.action_dim)
    assert d["t"].shape == (64,)
    assert not np.array_equal(d["actions"], d["noise"])
    dims = d["action_mask"][:, 0, :].sum(axis=1).astype(int)
    assert dims.min() >= 1 and dims.max() <= g.action_dim and len(set(dims)) > 10
    for b in range(64):
        assert d["action_mask"][b, :, : dims[b]].all() and not d["action_mask"][b, :, dims[b]:].any()
    again = synth.make_training_inputs(w)
    for k in d:
        np.testing.assert_array_equal(d[k], again[k])


def test_training_draw_uses_the_pages_beta_parameters():
    """The generator's default t distribution is the printed config's
    Beta(noise_beta_alpha, noise_beta_beta); its inverse-CDF draw needs beta = 1."""
    import inspect
    import json
    import os
    path = os.path.join(os.path.dirname(__file__), "golden", "training_time_beta.json")
    cfg = json.load(open(path))
    assert cfg["noise_beta_beta"] == 1.0
    assert inspect.signature(synth.make_training_inputs).parameters["alpha"].default == cfg["noise_beta_alpha"]
    assert synth.GEOM_FULL.num_timestep_buckets == cfg["num_timestep_buckets"]
    assert synth.WORKLOADS["sweep256"].num_steps == cfg["num_inference_timesteps"]
