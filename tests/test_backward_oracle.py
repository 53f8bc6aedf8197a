"""Pins of the backward oracle (oracle/backward.py), on the CPU.

The gradient formula is derived from the alpha-entmax Jacobian, not printed on the pages, so it is
pinned by what does not depend on it:
  * central finite differences of L = sum(dout * out) through the forward oracle's exact tau, on
    tiny fixed-length, non-causal and packed problems, for alpha in {1.333, 1.5, 2, 3};
  * invariants: the key gradients of a head sum to zero (a common shift of all keys moves every
    score of a row alike, which entmax ignores); values constant over the keys give zero query
    and key gradients; dv sums p over rows, so the total of dv equals the total of dout summed
    over each group's query heads.
"""
import numpy as np
import pytest

from oracle import backward as bwd


def _problem(rng, B, Hq, Hkv, T, d, packed=None):
    if packed is not None:
        Tt = int(sum(packed))
        q = rng.standard_normal((Hq, Tt, d))
        k = rng.standard_normal((Hkv, Tt, d))
        v = rng.standard_normal((Hkv, Tt, d))
        g = rng.standard_normal((Hq, Tt, d))
        cu = np.concatenate([[0], np.cumsum(packed)]).astype(np.int32)
        return q, k, v, g, cu
    q = rng.standard_normal((B, Hq, T, d))
    k = rng.standard_normal((B, Hkv, T, d))
    v = rng.standard_normal((B, Hkv, T, d))
    g = rng.standard_normal((B, Hq, T, d))
    return q, k, v, g, None


def _loss(q, k, v, g, alpha, causal, cu):
    return float((bwd.attention_forward_fp64(q, k, v, alpha, causal, cu) * g).sum())


def _fd(arr, f, h=1e-6):
    grad = np.zeros_like(arr)
    it = np.nditer(arr, flags=["multi_index"])
    for _ in it:
        i = it.multi_index
        keep = arr[i]
        arr[i] = keep + h
        lp = f()
        arr[i] = keep - h
        lm = f()
        arr[i] = keep
        grad[i] = (lp - lm) / (2 * h)
    return grad


CASES = [
    ("causal_a1.5", dict(B=1, Hq=2, Hkv=1, T=6, d=4), 1.5, True, None),
    ("causal_a2", dict(B=1, Hq=2, Hkv=1, T=6, d=4), 2.0, True, None),
    ("causal_a1.333", dict(B=1, Hq=2, Hkv=2, T=5, d=4), 1.333, True, None),
    ("noncausal_a3", dict(B=2, Hq=1, Hkv=1, T=5, d=3), 3.0, False, None),
    ("packed_a1.5", dict(B=None, Hq=2, Hkv=1, T=None, d=4), 1.5, True, (3, 1, 4)),
]


@pytest.mark.parametrize("name,shape,alpha,causal,packed", CASES, ids=[c[0] for c in CASES])
def test_backward_matches_finite_differences(name, shape, alpha, causal, packed):
    rng = np.random.default_rng(7)
    # scores scaled up so that supports are small and no score sits at a kink of p
    q, k, v, g, cu = _problem(rng, packed=packed, **shape)
    q *= 2.0
    dq, dk, dv, _ = bwd.attention_backward(q, k, v, g, alpha, causal, cu)
    f = lambda: _loss(q, k, v, g, alpha, causal, cu)  # noqa: E731
    for got, arr in ((dq, q), (dk, k), (dv, v)):
        want = _fd(arr, f)
        np.testing.assert_allclose(got, want, rtol=1e-5, atol=1e-6, err_msg=name)


def test_key_gradients_sum_to_zero():
    """Adding one vector c to every key adds q_i . c / sqrt(d) to all scores of row i alike, which
    entmax ignores: L does not move, so sum_j dk_j . c = 0 for every c, i.e. sum_j dk_j = 0 (the
    score gradients of each row sum to zero)."""
    rng = np.random.default_rng(3)
    for causal in (True, False):
        q, k, v, g, _ = _problem(rng, B=1, Hq=2, Hkv=1, T=9, d=5)
        _, dk, _, _ = bwd.attention_backward(q, k, v, g, 1.5, causal, None)
        np.testing.assert_allclose(dk.sum(axis=2), 0.0, atol=1e-10)


def test_constant_values_give_zero_query_and_key_gradients():
    rng = np.random.default_rng(5)
    q, k, v, g, _ = _problem(rng, B=1, Hq=2, Hkv=1, T=7, d=4)
    v[:] = rng.standard_normal(4)  # every value row the same: out = v_0 whatever p is
    dq, dk, dv, _ = bwd.attention_backward(q, k, v, g, 1.5, True, None)
    np.testing.assert_allclose(dq, 0.0, atol=1e-12)
    np.testing.assert_allclose(dk, 0.0, atol=1e-12)


def test_value_gradient_total_equals_dout_total():
    rng = np.random.default_rng(9)
    q, k, v, g, _ = _problem(rng, B=2, Hq=4, Hkv=2, T=6, d=3)
    _, _, dv, _ = bwd.attention_backward(q, k, v, g, 1.333, True, None)
    # sum_j dv_j = sum_i (sum_j p_ij) g_i = sum_i g_i, per (batch, kv head) over its query heads
    want = g.reshape(2, 2, 2, 6, 3).sum(axis=(2, 3))
    np.testing.assert_allclose(dv.sum(axis=2), want, atol=1e-12)


@pytest.mark.parametrize("packed", [None, (5, 1, 9)], ids=["fixed", "packed"])
@pytest.mark.parametrize("causal", [True, False])
def test_row_gradients_equal_the_full_backward(packed, causal):
    """row_gradients (dq and delta of chosen rows, for sampled checks at large sizes) equals
    the full backward oracle on every row of small problems, GQA and packed included."""
    rng = np.random.default_rng(11)
    q, k, v, g, cu = _problem(rng, 2, 4, 2, 12, 8, packed)
    dq, _, _, delta = bwd.attention_backward(q, k, v, g, 1.5, causal, cu)
    rows = np.arange(dq.reshape(-1, dq.shape[-1]).shape[0])[::-1]  # every row, in reverse
    rdq, rdelta = bwd.row_gradients(q, k, v, g, 1.5, causal, cu, rows)
    np.testing.assert_allclose(rdq, dq.reshape(-1, dq.shape[-1])[rows], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(rdelta, delta.reshape(-1)[rows], rtol=1e-12, atol=1e-12)
