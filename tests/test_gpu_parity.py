"""End-to-end parity of gdit_get_action (CUDA, through the C ABI) with the fp64
CPU oracle on the same seeded inputs, for every workload, plus edge cases.

Samples are independent, so at full batch sizes the oracle is run on a few
sampled batch rows (covering different embodiments) and compared row by row.
"""

import dataclasses

import numpy as np
import pytest

import oracle
import synth
from tests.gpu_util import DELTA_REL_L2, MAX_ABS, REL_L2, parity_stats, require_gpu, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def full_weights():
    return synth.make_weights(synth.GEOM_FULL)


@pytest.fixture(scope="module")
def full_model(full_weights):
    return oracle.Model(full_weights, synth.GEOM_FULL)


@pytest.fixture(scope="module")
def head_full(full_weights):
    require_gpu()
    from flow_matching_dit_b200 import ActionHead
    h = ActionHead(synth.GEOM_FULL, full_weights, max_batch=256, max_seq=600)
    yield h
    h.close()


@pytest.fixture(scope="module")
def tiny_weights():
    return synth.make_weights(synth.GEOM_TINY)


@pytest.fixture(scope="module")
def head_tiny(tiny_weights):
    require_gpu()
    from flow_matching_dit_b200 import ActionHead
    h = ActionHead(synth.GEOM_TINY, tiny_weights, max_batch=8, max_seq=64)
    yield h
    h.close()


def run_gpu(head, inp, K):
    out = head.get_action(*to_dev(inp), num_steps=K)
    st = head.sync_status()
    return out.cpu().numpy(), st


def run_oracle(W, g, inp, K, samples=None, model=None):
    return oracle.get_action(W, g, inp["backbone_features"], inp["vl_mask"], inp["state"], inp["embodiment_id"],
                             inp["init_noise"], K, samples=samples, model=model)


def assert_parity(gpu, ref, noise, what):
    max_abs, rel, drel = parity_stats(gpu, ref, noise)
    print(f"{what}: max_abs={max_abs:.3e} rel_l2={rel:.3e} delta_rel_l2={drel:.3e}")
    assert np.isfinite(gpu).all(), what
    assert max_abs <= MAX_ABS, (what, max_abs)
    assert rel <= REL_L2, (what, rel)
    assert drel <= DELTA_REL_L2, (what, drel)


# ---------------------------------------------------------------- tiny workload

@pytest.mark.parametrize("emb", [0, 1])
def test_tiny_parity(head_tiny, tiny_weights, emb):
    w = synth.workload("tiny", fixed_ids=(emb,))
    inp = synth.make_inputs(w)
    gpu, st = run_gpu(head_tiny, inp, 4)
    assert st == 0
    ref = run_oracle(tiny_weights, w.geom, inp, 4)
    assert_parity(gpu, ref, inp["init_noise"], f"tiny id={emb}")


def test_tiny_mixed_batch_ragged_masks(head_tiny, tiny_weights):
    w = synth.workload("tiny", batch=5, valid_min=1, fixed_ids=None, id_low=0, id_high=1)
    inp = synth.make_inputs(w, seed=5)
    inp["vl_mask"][2] = 0                          # a sample with no valid token
    inp["vl_mask"][3] = 0
    inp["vl_mask"][3, 17] = 1                      # exactly one valid token
    inp["vl_mask"][4, ::2] = 0                     # not a prefix
    gpu, st = run_gpu(head_tiny, inp, 4)
    assert st == 0
    ref = run_oracle(tiny_weights, w.geom, inp, 4)
    assert_parity(gpu, ref, inp["init_noise"], "tiny mixed")


@pytest.mark.parametrize("K", [1, 3, 8])
def test_tiny_step_counts(head_tiny, tiny_weights, K):
    w = synth.workload("tiny", batch=2, fixed_ids=(1, 0))
    inp = synth.make_inputs(w, seed=9)
    gpu, st = run_gpu(head_tiny, inp, K)
    ref = run_oracle(tiny_weights, w.geom, inp, K)
    assert_parity(gpu, ref, inp["init_noise"], f"tiny K={K}")


def test_tiny_masked_tokens_do_not_matter(head_tiny):
    w = synth.workload("tiny", batch=2, fixed_ids=(0, 1))
    inp = synth.make_inputs(w, seed=3)
    inp["vl_mask"][:, 40:] = 0
    a, _ = run_gpu(head_tiny, inp, 4)
    inp2 = dict(inp, backbone_features=inp["backbone_features"].copy())
    inp2["backbone_features"][:, 40:] = 1e3
    b, _ = run_gpu(head_tiny, inp2, 4)
    np.testing.assert_array_equal(a, b)


def test_bad_embodiment_id_gives_nan_and_status(head_tiny, tiny_weights):
    from flow_matching_dit_b200._lib import GDIT_EDEVICE
    w = synth.workload("tiny", batch=3, fixed_ids=(0, 7, 1))
    inp = synth.make_inputs(w, seed=4)
    gpu, st = run_gpu(head_tiny, inp, 4)
    assert st == GDIT_EDEVICE
    assert np.isnan(gpu[1]).all()
    ok = dict(inp)
    for k in ok:
        ok[k] = ok[k][[0, 2]]
    ref = run_oracle(tiny_weights, w.geom, ok, 4)
    assert_parity(gpu[[0, 2]], ref, ok["init_noise"], "tiny valid rows next to a bad id")
    assert head_tiny.sync_status() == 0   # cleared


def test_decoder_signature_routes_exactly():
    """act_dec weights zero and b2[c] = c: every sample moves by exactly its
    category index, so the output names the category that was used."""
    require_gpu()
    from flow_matching_dit_b200 import ActionHead
    g = dataclasses.replace(synth.GEOM_TINY, num_embodiments=6)
    W = synth.make_weights(g)
    W["act_dec.l1.W"][:] = 0
    W["act_dec.l1.b"][:] = 0
    W["act_dec.l2.W"][:] = 0
    for c in range(6):
        W["act_dec.l2.b"][c] = c
    ids = np.array([5, 0, 3, 3, 1, 4, 2, 0], np.int32)
    w = synth.workload("tiny", geom=g, batch=8, fixed_ids=tuple(ids))
    inp = synth.make_inputs(w, seed=11)
    with ActionHead(g, W, max_batch=8, max_seq=64) as head:
        gpu, st = run_gpu(head, inp, 4)
        perm, seg, vofs = head.routing(8)
    assert st == 0
    moved = gpu - inp["init_noise"]
    np.testing.assert_allclose(moved, np.broadcast_to(ids[:, None, None].astype(np.float64), moved.shape),
                               rtol=0, atol=1e-5)
    # routing arrays: stable counting sort by id
    assert perm.tolist() == np.argsort(ids, kind="stable").tolist()
    assert seg.tolist() == [int((ids < c).sum()) for c in range(7)]
    assert vofs.tolist() == [64 * i for i in range(9)]


def test_host_buffer_entry_point_matches_device_entry_point(head_tiny):
    w = synth.workload("tiny", batch=3, fixed_ids=(1, 0, 1))
    inp = synth.make_inputs(w, seed=21)
    dev, _ = run_gpu(head_tiny, inp, 4)
    host = head_tiny.get_action_host(inp["backbone_features"], inp["vl_mask"], inp["state"],
                                     inp["embodiment_id"], inp["init_noise"], 4)
    np.testing.assert_array_equal(dev, host)


def test_eager_and_graph_paths_agree(tiny_weights):
    require_gpu()
    from flow_matching_dit_b200 import GDIT_FLAG_NO_GRAPH, ActionHead
    w = synth.workload("tiny", batch=2, fixed_ids=(0, 1))
    inp = synth.make_inputs(w, seed=2)
    with ActionHead(synth.GEOM_TINY, tiny_weights, max_batch=2, max_seq=64, flags=GDIT_FLAG_NO_GRAPH) as eager:
        a, _ = run_gpu(eager, inp, 4)
    with ActionHead(synth.GEOM_TINY, tiny_weights, max_batch=2, max_seq=64) as graph:
        b, _ = run_gpu(graph, inp, 4)
        c, _ = run_gpu(graph, inp, 4)     # graph replay
    np.testing.assert_array_equal(a, b)
    np.testing.assert_array_equal(b, c)


def test_strict_profiles(tiny_weights):
    require_gpu()
    from flow_matching_dit_b200 import GDIT_FLAG_STRICT_PROFILES, ActionHead, GditError
    from flow_matching_dit_b200._lib import GDIT_EPROFILE
    w = synth.workload("tiny", batch=2, fixed_ids=(0, 1))
    inp = synth.make_inputs(w, seed=2)
    with ActionHead(synth.GEOM_TINY, tiny_weights, max_batch=2, max_seq=64, flags=GDIT_FLAG_STRICT_PROFILES) as h:
        with pytest.raises(GditError) as e:
            run_gpu(h, inp, 4)
        assert e.value.code == GDIT_EPROFILE
        h.prepare(2, 64, 4, bf16=False)
        run_gpu(h, inp, 4)


# ---------------------------------------------------------------- full-size workloads

def test_latency_workload_full_oracle(head_full, full_weights, full_model):
    w = synth.WORKLOADS["latency"]
    inp = synth.make_inputs(w)
    gpu, st = run_gpu(head_full, inp, w.num_steps)
    assert st == 0
    ref = run_oracle(full_weights, w.geom, inp, w.num_steps, model=full_model)
    assert_parity(gpu, ref, inp["init_noise"], "latency B=1 S=300")


def test_cross_kv_projection_matches_oracle(head_full, full_model):
    w = synth.WORKLOADS["latency"]
    inp = synth.make_inputs(w)
    run_gpu(head_full, inp, w.num_steps)
    valid = oracle.to_f64(inp["backbone_features"][0])[inp["vl_mask"][0] == 1]
    for layer in (0, 30):
        k, v = head_full.debug_kv(layer)
        kr, vr = oracle.cross_kv(full_model, layer, valid)
        for got, ref in ((k, kr), (v, vr)):
            # bf16 storage of f32-accumulated exact products: <= 2^-8 relative
            np.testing.assert_allclose(got, ref, rtol=2 ** -8, atol=1e-3)


def rows_one_per_embodiment(ids):
    """The first batch row of every embodiment id present, in row order: each
    category's segment of the grouped GEMMs is compared at least once."""
    ids = np.asarray(ids).reshape(-1)
    first = {}
    for r, c in enumerate(ids.tolist()):
        first.setdefault(c, r)
    return sorted(first.values())


def test_batched_workload_every_row(head_full, full_weights, full_model):
    """B = 32, ragged valid lengths 200..600 padded to 600: every row, so every
    sample's packed key range and every category segment is compared."""
    w = synth.WORKLOADS["batched"]
    inp = synth.make_inputs(w)
    gpu, st = run_gpu(head_full, inp, w.num_steps)
    assert st == 0
    rows = list(range(w.batch))
    ref = run_oracle(full_weights, w.geom, inp, w.num_steps, samples=rows, model=full_model)
    assert_parity(gpu, ref, inp["init_noise"], "batched B=32 S<=600 (all rows)")


@pytest.mark.parametrize("name", ["sweep8", "sweep32", "sweep128", "sweep256"])
def test_sweep_workloads(head_full, full_weights, full_model, name):
    """The throughput sweep at S = 256: every row up to B = 32; at B = 128 and
    256 one row of every embodiment (all 32 categories occur), so every
    segment of the grouped per-embodiment GEMMs, and the 128-row tiles that
    straddle segment boundaries, feed a compared row."""
    w = synth.WORKLOADS[name]
    inp = synth.make_inputs(w)
    gpu, st = run_gpu(head_full, inp, w.num_steps)
    assert st == 0
    assert np.isfinite(gpu).all()
    if w.batch <= 32:
        rows = list(range(w.batch))
    else:
        rows = rows_one_per_embodiment(inp["embodiment_id"])
        assert sorted(set(inp["embodiment_id"][rows].tolist())) == list(range(32))
    ref = run_oracle(full_weights, w.geom, inp, w.num_steps, samples=rows, model=full_model)
    assert_parity(gpu[rows], ref, inp["init_noise"][rows], f"{name} ({len(rows)} rows)")


def test_long_chunk_workload_every_row(full_weights, full_model):
    """B = 8, H = 50 (51 tokens per sample), S = 512, K = 8: every row."""
    require_gpu()
    from flow_matching_dit_b200 import ActionHead
    w = synth.WORKLOADS["long_chunk"]
    inp = synth.make_inputs(w)
    with ActionHead(w.geom, full_weights, max_batch=8, max_seq=512) as head:
        gpu, st = run_gpu(head, inp, w.num_steps)
    assert st == 0
    rows = list(range(w.batch))
    model = oracle.Model(full_weights, w.geom)
    ref = run_oracle(full_weights, w.geom, inp, w.num_steps, samples=rows, model=model)
    assert_parity(gpu, ref, inp["init_noise"], "long chunk B=8 H=50 K=8 (all rows)")


# ---------------------------------------------------------------- single-sample persistent loop

def test_single_sample_loop_matches_general_path_and_oracle(full_weights, full_model, head_full):
    """B = 1 runs the whole K-step loop as one persistent kernel; the general
    per-layer path (GDIT_FLAG_NO_SMALL) and the oracle must agree with it."""
    from flow_matching_dit_b200 import GDIT_FLAG_NO_SMALL, ActionHead
    w = synth.WORKLOADS["latency"]
    inp = synth.make_inputs(w, seed=13)
    small, st = run_gpu(head_full, inp, w.num_steps)
    assert st == 0
    with ActionHead(w.geom, full_weights, max_batch=1, max_seq=w.seq, flags=GDIT_FLAG_NO_SMALL) as general:
        gen, st2 = run_gpu(general, inp, w.num_steps)
    assert st2 == 0
    ref = run_oracle(full_weights, w.geom, inp, w.num_steps, model=full_model)
    assert_parity(small, ref, inp["init_noise"], "single-sample loop vs oracle")
    assert_parity(gen, ref, inp["init_noise"], "general path B=1 vs oracle")
    assert_parity(small, gen, inp["init_noise"], "single-sample loop vs general path")


def test_single_sample_loop_eager_equals_graph(tiny_weights):
    require_gpu()
    from flow_matching_dit_b200 import GDIT_FLAG_NO_GRAPH, ActionHead
    w = synth.workload("tiny", fixed_ids=(1,))
    inp = synth.make_inputs(w, seed=17)
    with ActionHead(synth.GEOM_TINY, tiny_weights, max_batch=1, max_seq=64, flags=GDIT_FLAG_NO_GRAPH) as eager:
        a, _ = run_gpu(eager, inp, 4)
    with ActionHead(synth.GEOM_TINY, tiny_weights, max_batch=1, max_seq=64) as graph:
        b, _ = run_gpu(graph, inp, 4)
        c, _ = run_gpu(graph, inp, 4)
    np.testing.assert_array_equal(a, b)
    np.testing.assert_array_equal(b, c)


def test_grouped_loop_matches_general_path_and_oracle(full_weights, full_model, head_full):
    """2 <= B <= 4 run the same persistent loop with one group of CTAs per
    sample (each CTA takes its units of a linear in several passes).  At
    full size, mixed embodiments and ragged valid lengths, it must agree with
    the per-layer path (GDIT_FLAG_NO_SMALL) and, on sampled rows, the oracle."""
    from flow_matching_dit_b200 import GDIT_FLAG_NO_SMALL, ActionHead
    for B, seed in ((2, 61), (4, 62)):
        w = synth.workload("sweep8", batch=B, valid_min=40, id_low=0, id_high=31)
        inp = synth.make_inputs(w, seed=seed)
        grouped, st = run_gpu(head_full, inp, w.num_steps)
        assert st == 0
        with ActionHead(w.geom, full_weights, max_batch=B, max_seq=w.seq, flags=GDIT_FLAG_NO_SMALL) as general:
            gen, st2 = run_gpu(general, inp, w.num_steps)
        assert st2 == 0
        assert_parity(grouped, gen, inp["init_noise"], f"grouped loop vs general path, B={B}")
        rows = [0, B - 1]
        ref = run_oracle(full_weights, w.geom, inp, w.num_steps, samples=rows, model=full_model)
        assert_parity(grouped[rows], ref, inp["init_noise"][rows], f"grouped loop vs oracle, B={B}")


@pytest.mark.parametrize("B", [2, 3, 4, 5, 6, 7, 8])
def test_grouped_loop_every_batch_size(head_tiny, tiny_weights, B):
    """Every group count of the loop (B <= 4) and the per-layer path just
    above it, on the tiny DiT: both embodiments, ragged (and one empty) key
    lists, one out-of-range id (its row NaN, the others unaffected), every
    row against the oracle."""
    from flow_matching_dit_b200._lib import GDIT_EDEVICE
    w = synth.workload("tiny", batch=B, valid_min=1, fixed_ids=None, id_low=0, id_high=1)
    inp = synth.make_inputs(w, seed=70 + B)
    inp["vl_mask"][B - 1] = 0                          # a sample with no valid key
    bad = B // 2 if B >= 3 else None
    if bad is not None:
        inp["embodiment_id"][bad] = 9
    gpu, st = run_gpu(head_tiny, inp, 4)
    assert st == (GDIT_EDEVICE if bad is not None else 0)
    rows = [b for b in range(B) if b != bad]
    if bad is not None:
        assert np.isnan(gpu[bad]).all()
    ok = {k: v[rows] for k, v in inp.items()}
    ref = run_oracle(tiny_weights, w.geom, ok, 4)
    assert_parity(gpu[rows], ref, ok["init_noise"], f"grouped loop B={B}")
    assert head_tiny.sync_status() == 0


def test_skinny_gemms_match_tensor_core_gemms_and_oracle(full_weights, full_model):
    """The per-layer path at a few samples (B = 6, 102 rows) runs its DiT
    linears on the skinny-M kernel; against the same path on the tensor-core
    GEMM (GDIT_FLAG_NO_SKINNY) and, on sampled rows, the oracle."""
    require_gpu()
    from flow_matching_dit_b200 import GDIT_FLAG_NO_SKINNY, GDIT_FLAG_NO_SMALL, ActionHead
    w = synth.workload("sweep8", batch=6, valid_min=40, id_low=0, id_high=31)
    inp = synth.make_inputs(w, seed=63)
    with ActionHead(w.geom, full_weights, max_batch=6, max_seq=w.seq, flags=GDIT_FLAG_NO_SMALL) as sk:
        a, st = run_gpu(sk, inp, w.num_steps)
    assert st == 0
    with ActionHead(w.geom, full_weights, max_batch=6, max_seq=w.seq,
                    flags=GDIT_FLAG_NO_SMALL | GDIT_FLAG_NO_SKINNY) as tc:
        b, st2 = run_gpu(tc, inp, w.num_steps)
    assert st2 == 0
    assert_parity(a, b, inp["init_noise"], "skinny-M GEMMs vs tensor-core GEMMs, B=6")
    rows = [0, 5]
    ref = run_oracle(full_weights, w.geom, inp, w.num_steps, samples=rows, model=full_model)
    assert_parity(a[rows], ref, inp["init_noise"][rows], "skinny-M GEMMs vs oracle, B=6")


def test_grouped_loop_eager_equals_graph(tiny_weights):
    require_gpu()
    from flow_matching_dit_b200 import GDIT_FLAG_NO_GRAPH, ActionHead
    w = synth.workload("tiny", batch=6, fixed_ids=None, id_low=0, id_high=1, valid_min=10)
    inp = synth.make_inputs(w, seed=23)
    with ActionHead(synth.GEOM_TINY, tiny_weights, max_batch=6, max_seq=64, flags=GDIT_FLAG_NO_GRAPH) as eager:
        a, _ = run_gpu(eager, inp, 4)
    with ActionHead(synth.GEOM_TINY, tiny_weights, max_batch=6, max_seq=64) as graph:
        b, _ = run_gpu(graph, inp, 4)
        c, _ = run_gpu(graph, inp, 4)
    np.testing.assert_array_equal(a, b)
    np.testing.assert_array_equal(b, c)


@pytest.mark.parametrize("case", ["empty", "one_token", "bad_id"])
def test_single_sample_loop_edge_cases(head_tiny, tiny_weights, case):
    from flow_matching_dit_b200._lib import GDIT_EDEVICE
    w = synth.workload("tiny", fixed_ids=(1,))
    inp = synth.make_inputs(w, seed=19)
    if case == "empty":
        inp["vl_mask"][:] = 0
    elif case == "one_token":
        inp["vl_mask"][:] = 0
        inp["vl_mask"][0, 33] = 1
    else:
        inp["embodiment_id"][:] = 5
    gpu, st = run_gpu(head_tiny, inp, 4)
    if case == "bad_id":
        assert st == GDIT_EDEVICE and np.isnan(gpu).all()
        return
    assert st == 0
    ref = run_oracle(tiny_weights, w.geom, inp, 4)
    assert_parity(gpu, ref, inp["init_noise"], f"single-sample loop, {case}")


def test_tma_store_epilogue_is_bitwise_equal_to_thread_stores(full_weights):
    """The DiT GEMMs' TMA store / reduce-add epilogue computes the same f32
    values as the per-thread stores (same adds, same roundings)."""
    require_gpu()
    from flow_matching_dit_b200 import GDIT_FLAG_NO_TMA_STORE, ActionHead
    w = synth.WORKLOADS["batched"]
    inp = synth.make_inputs(w, seed=23)
    with ActionHead(w.geom, full_weights, max_batch=32, max_seq=600) as a:
        x, _ = run_gpu(a, inp, w.num_steps)
    with ActionHead(w.geom, full_weights, max_batch=32, max_seq=600, flags=GDIT_FLAG_NO_TMA_STORE) as b:
        y, _ = run_gpu(b, inp, w.num_steps)
    np.testing.assert_array_equal(x, y)


def test_host_entry_point_matches_device_entry_point_at_full_size(head_full):
    """The host-buffer entry point packs and projects the features in four
    sample chunks (the K/V projection of each chunk starts at a device-side
    row); the device entry point projects all packed rows at once.  With
    ragged key counts the chunk boundaries fall inside row tiles.  Every
    output element is accumulated in the same order either way: equal bit
    for bit."""
    w = synth.WORKLOADS["batched"]
    inp = synth.make_inputs(w, seed=53)
    dev, st = run_gpu(head_full, inp, w.num_steps)
    assert st == 0
    host = head_full.get_action_host(inp["backbone_features"], inp["vl_mask"], inp["state"],
                                     inp["embodiment_id"], inp["init_noise"], w.num_steps)
    np.testing.assert_array_equal(dev, host)


def test_pair_gemms_match_single_cta_gemms(head_full, full_weights):
    """At B = 256 the DiT GEMMs run on CTA pairs (cta_group::2, 256-row tiles);
    with GDIT_FLAG_NO_PAIR they run on single CTAs.  Both sum the same bf16
    products in f32 in the same K order, so the actions agree to rounding."""
    from flow_matching_dit_b200 import GDIT_FLAG_NO_PAIR, ActionHead
    w = synth.WORKLOADS["sweep256"]
    inp = synth.make_inputs(w, seed=37)
    x, st = run_gpu(head_full, inp, w.num_steps)
    assert st == 0
    with ActionHead(w.geom, full_weights, max_batch=256, max_seq=256, flags=GDIT_FLAG_NO_PAIR) as b:
        y, st2 = run_gpu(b, inp, w.num_steps)
    assert st2 == 0
    print("pair vs single-CTA max |diff|", float(np.abs(x - y).max()))
    np.testing.assert_allclose(x, y, rtol=0, atol=1e-3)


def test_cross_attention_on_ragged_keys_at_64_samples(head_full, full_weights, full_model):
    """64 samples with valid lengths 200..600 padded to 600: 1024 (sample,
    head) items, the warp schedule of the cross attention over ragged key
    lists, against the oracle on rows spread over the batch."""
    w = synth.workload("batched", batch=64)
    inp = synth.make_inputs(w, seed=43)
    x, st = run_gpu(head_full, inp, w.num_steps)
    assert st == 0
    rows = [0, 9, 33, 63]
    ref = run_oracle(full_weights, w.geom, inp, w.num_steps, samples=rows, model=full_model)
    assert_parity(x[rows], ref, inp["init_noise"][rows], "cross attention, B=64 ragged")


def test_bounded_wait_expiry_is_reported_and_the_device_stays_usable(head_tiny, tiny_weights):
    """A wait on an mbarrier that nothing arrives at, through the library's
    bounded wait with a 1 ms limit: it gives up, reports GDIT_ETIMEOUT, and the
    next call on the same device runs normally."""
    import time
    from flow_matching_dit_b200 import debug_wait_expiry
    from flow_matching_dit_b200._lib import GDIT_ETIMEOUT
    t0 = time.perf_counter()
    assert debug_wait_expiry(0, 1_000_000) == GDIT_ETIMEOUT
    assert time.perf_counter() - t0 >= 1e-3
    w = synth.workload("tiny", fixed_ids=(1,))
    inp = synth.make_inputs(w, seed=29)
    gpu, st = run_gpu(head_tiny, inp, 4)
    assert st == 0
    assert_parity(gpu, run_oracle(tiny_weights, w.geom, inp, 4), inp["init_noise"], "after a wait expiry")


# ---------------------------------------------------------------- image/text split of the cross layers

@pytest.mark.parametrize("n", [1, 2])
# 1, 3: the persistent loop (one and three CTA groups); 12: per-layer kernels, split attention
# schedule; 160 (x 4 heads >= 4 x SMs): per-layer kernels, warp attention schedule (rows sampled)
@pytest.mark.parametrize("batch", [1, 3, 12, 160])
def test_image_text_split_matches_oracle(n, batch):
    """AlternateVLDiT with attend_text_every_n_blocks = n on a 4-layer tiny DiT
    (cross blocks 0 and 2): ragged valid lengths and seeded image masks; the
    cross layers keep only their kind of key, as the oracle's per-layer masks."""
    require_gpu()
    import torch
    from flow_matching_dit_b200 import ActionHead
    g = dataclasses.replace(synth.GEOM_TINY, num_layers=4, attend_text_every_n_blocks=n)
    W = synth.make_weights(g)
    w = dataclasses.replace(synth.WORKLOADS["tiny"], geom=g, batch=batch, seq=64, valid_min=30,
                            fixed_ids=(1, 0, 1)[:min(batch, 3)])
    inp = synth.make_inputs(w, seed=31 + n)
    img = synth.make_image_mask(w, seed=41 + n)
    with ActionHead(g, W, max_batch=batch, max_seq=64) as head:
        out = head.get_action(*to_dev(inp), num_steps=4, image_mask=torch.from_numpy(img).cuda())
        st = head.sync_status()
        gpu = out.cpu().numpy()
        plain = head.get_action(*to_dev(inp), num_steps=4).cpu().numpy()   # no image mask: no image token
    assert st == 0
    rows = list(range(batch)) if batch <= 3 else [0, batch // 2, batch - 1]
    ref = oracle.get_action(W, g, inp["backbone_features"], inp["vl_mask"], inp["state"], inp["embodiment_id"],
                            inp["init_noise"], 4, image_mask=img, samples=rows)
    assert_parity(gpu[rows], ref, inp["init_noise"][rows], f"image/text split n={n} B={batch}")
    ref0 = oracle.get_action(W, g, inp["backbone_features"], inp["vl_mask"], inp["state"], inp["embodiment_id"],
                             inp["init_noise"], 4, samples=rows)
    assert_parity(plain[rows], ref0, inp["init_noise"][rows], f"split on, no image mask, n={n} B={batch}")


# ---------------------------------------------------------------- vision-language layer norm (vlln)

@pytest.mark.parametrize("batch", [1, 3])
def test_vlln_matches_oracle_and_removes_token_scale(batch):
    """With vlln weights the packed backbone tokens are layer-normalised before
    the K/V projection.  Each token's features get a random scale in [0.5, 3]
    and shift in [-2, 2] (which vlln removes and the parity would otherwise
    show); the device must match the oracle and not see the transform."""
    require_gpu()
    from flow_matching_dit_b200 import ActionHead
    g = dataclasses.replace(synth.GEOM_TINY, vlln=True)
    W = synth.make_weights(g)
    w = dataclasses.replace(synth.WORKLOADS["tiny"], geom=g, batch=batch, seq=64, valid_min=30,
                            fixed_ids=(0, 1, 1)[:batch])
    inp = synth.make_inputs(w, seed=51)
    r = np.random.default_rng(52)
    f = inp["backbone_features"].astype(np.float32)
    a = r.uniform(0.5, 3.0, size=(batch, 64, 1)).astype(np.float32)
    c = r.uniform(-2.0, 2.0, size=(batch, 64, 1)).astype(np.float32)
    moved = dict(inp)
    moved["backbone_features"] = (f * a + c).astype(np.float32)
    with ActionHead(g, W, max_batch=batch, max_seq=64) as head:
        got, st = run_gpu(head, moved, 4)
        same, st2 = run_gpu(head, inp, 4)
    assert st == 0 and st2 == 0
    ref = run_oracle(W, g, moved, 4)
    assert_parity(got, ref, inp["init_noise"], f"vlln B={batch}")
    assert_parity(same, ref, inp["init_noise"], f"vlln B={batch}, untransformed features")
