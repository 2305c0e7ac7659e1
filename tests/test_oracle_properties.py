"""Property pins of the oracle's building blocks over random shapes and
values (CPU only, hypothesis): facts that hold at any size, checked against
the definitions rather than another implementation."""

import numpy as np
from hypothesis import given, settings
from hypothesis import strategies as st

import oracle

SETTINGS = settings(max_examples=40, deadline=None)


def _rng(seed):
    return np.random.default_rng(seed)


@SETTINGS
@given(nq=st.integers(1, 20), nk=st.integers(1, 40), heads=st.sampled_from([1, 2, 4]),
       dh=st.sampled_from([4, 8, 16]), seed=st.integers(0, 2 ** 31 - 1))
def test_attention_rows_are_convex_combinations_of_values(nq, nk, heads, dh, seed):
    """Each head's output row is a probability-weighted mean of that head's
    value rows, so it lies between the columns' min and max."""
    r = _rng(seed)
    q, k, v = (r.standard_normal((n, heads * dh)) * 3 for n in (nq, nk, nk))
    out, probs = oracle.attention(q, k, v, heads, return_probs=True)
    for h, p in enumerate(probs):
        assert np.all(p >= 0) and np.allclose(p.sum(axis=1), 1.0, atol=1e-12)
        cols = slice(h * dh, (h + 1) * dh)
        assert np.all(out[:, cols] <= v[:, cols].max(axis=0) + 1e-12)
        assert np.all(out[:, cols] >= v[:, cols].min(axis=0) - 1e-12)


@SETTINGS
@given(nq=st.integers(1, 12), nk=st.integers(1, 30), heads=st.sampled_from([1, 2, 4]),
       seed=st.integers(0, 2 ** 31 - 1))
def test_attention_ignores_a_shift_of_the_keys_along_the_query(nq, nk, heads, seed):
    """Adding the same vector c to every key adds q.c to all of a query's
    scores, which the softmax ignores; the output is unchanged."""
    r = _rng(seed)
    dh = 8
    q, k, v = (r.standard_normal((n, heads * dh)) for n in (nq, nk, nk))
    c = r.standard_normal(heads * dh) * 2
    np.testing.assert_allclose(oracle.attention(q, k + c, v, heads), oracle.attention(q, k, v, heads),
                               rtol=1e-10, atol=1e-12)


@SETTINGS
@given(nk=st.integers(1, 30), seed=st.integers(0, 2 ** 31 - 1))
def test_attention_is_invariant_to_key_order(nk, seed):
    r = _rng(seed)
    q, k, v = (r.standard_normal((n, 16)) for n in (5, nk, nk))
    perm = r.permutation(nk)
    np.testing.assert_allclose(oracle.attention(q, k[perm], v[perm], 2), oracle.attention(q, k, v, 2),
                               rtol=1e-12, atol=1e-13)


@SETTINGS
@given(rows=st.integers(1, 10), width=st.sampled_from([2, 7, 64, 128]), seed=st.integers(0, 2 ** 31 - 1))
def test_layer_norm_without_eps_ignores_a_row_affine_map(rows, width, seed):
    r = _rng(seed)
    x = r.standard_normal((rows, width))
    if width > 1:
        x[:, 0] += 1.0                                   # no constant row
    a = r.uniform(0.1, 10.0, size=(rows, 1))
    b = r.standard_normal((rows, 1)) * 5
    y = oracle.layer_norm(x, 0.0)
    np.testing.assert_allclose(oracle.layer_norm(a * x + b, 0.0), y, rtol=1e-9, atol=1e-10)
    np.testing.assert_allclose(y.mean(axis=1), 0.0, atol=1e-12)
    np.testing.assert_allclose((y ** 2).mean(axis=1), 1.0, rtol=1e-10)


@SETTINGS
@given(C=st.integers(1, 5), din=st.integers(1, 12), dout=st.integers(1, 12), n=st.integers(1, 6),
       seed=st.integers(0, 2 ** 31 - 1))
def test_category_linear_is_the_selected_affine_map(C, din, dout, n, seed):
    """x W[c] + b[c] is affine in x and selects category c only."""
    r = _rng(seed)
    W = r.standard_normal((C, din, dout))
    b = r.standard_normal((C, dout))
    x1, x2 = r.standard_normal((n, din)), r.standard_normal((n, din))
    c = int(r.integers(C))
    lhs = oracle.category_linear(0.3 * x1 + 0.7 * x2, W, b, c)
    rhs = 0.3 * oracle.category_linear(x1, W, b, c) + 0.7 * oracle.category_linear(x2, W, b, c)
    np.testing.assert_allclose(lhs, rhs, rtol=1e-12, atol=1e-12)
    W2 = W.copy()
    for other in range(C):
        if other != c:
            W2[other] = r.standard_normal((din, dout))
    np.testing.assert_array_equal(oracle.category_linear(x1, W2, b, c), oracle.category_linear(x1, W, b, c))
