"""Pins of the entmax block-routing oracle (oracle/routing.py), on the CPU.

The router is alpha-entmax over query-to-summary scores (MiniCPM-4-8B-NSA page, DashAttention,
"How it works", stage 2).  Checked against what the mathematics fixes, not against the oracle:
  * chunks of one token with the keys as summaries turn routing into entmax attention's p, so it
    must equal the explicit-loop brute force of tests/test_oracle_pins.py (bisection on every
    score, no sort);
  * alpha = 2 routes by sparsemax: Duchi et al.'s sort-based simplex projection of the scores;
  * priors sum to 1 over the visible chunks and vanish elsewhere, the top-scoring chunk is always
    in the support, tau lies in its bracket [m - 1, m - n^(1-alpha)];
  * adding one vector to every summary shifts all scores of a row alike and leaves the priors
    unchanged (catches a summary indexed by the wrong chunk or head);
  * the visibility rule (causal, own chunk with estimate_diagonal or not, non-causal) and the
    GQA head map, chunk by chunk.
"""
import math

import numpy as np
import pytest

from oracle import routing
from test_oracle_pins import brute_attention, duchi_simplex_projection


def _inputs(rng, B, Hq, Hkv, T, d, C, scale=2.0):
    q = rng.standard_normal((B, Hq, T, d)) * scale
    nc = -(-T // C)
    sig = rng.standard_normal((B, Hkv, nc, d))
    return q, sig


@pytest.mark.parametrize("alpha", [1.333, 1.5, 2.0, 3.0])
@pytest.mark.parametrize("causal", [True, False])
def test_single_token_chunks_equal_entmax_attention(oracle, alpha, causal):
    rng = np.random.default_rng(21)
    Hq, Hkv, T, d = 4, 2, 9, 5
    q = rng.standard_normal((Hq, T, d)) * 2.0
    k = rng.standard_normal((Hkv, T, d))
    v = np.zeros((Hkv, T, d))
    _, _, p = brute_attention(q, k, v, alpha, causal, Hq // Hkv)
    pi, _ = routing.route_chunks(q[None], k[None], alpha, chunk_size=1, causal=causal)
    np.testing.assert_allclose(pi[0], p, atol=1e-10)


def test_alpha2_routes_by_simplex_projection(oracle):
    rng = np.random.default_rng(22)
    q, sig = _inputs(rng, 2, 2, 1, 200, 8, 16)
    pi, tau = routing.route_chunks(q, sig, 2.0, chunk_size=16)
    for b in range(2):
        for h in range(2):
            for i in range(0, 200, 7):
                n = i // 16 + 1
                s = sig[b, 0, :n] @ q[b, h, i] / math.sqrt(8)
                want, theta = duchi_simplex_projection(s)
                np.testing.assert_allclose(pi[b, h, i, :n], want, atol=1e-12)
                assert abs(tau[b, h, i] - theta) <= 1e-12
                assert np.all(pi[b, h, i, n:] == 0.0)


@pytest.mark.parametrize("alpha", [1.333, 1.5, 3.0])
def test_priors_are_a_distribution_with_the_top_chunk_in_support(oracle, alpha):
    rng = np.random.default_rng(23)
    C, T, d = 8, 100, 6
    q, sig = _inputs(rng, 1, 2, 2, T, d, C)
    pi, tau = routing.route_chunks(q, sig, alpha, chunk_size=C, scaling_factor=1.7)
    for h in range(2):
        for i in range(T):
            n = i // C + 1
            row = pi[0, h, i]
            assert abs(row[:n].sum() - 1.0) <= 1e-12
            assert np.all(row >= 0.0) and np.all(row[n:] == 0.0)
            z = (alpha - 1.0) * 1.7 * (sig[0, h, :n] @ q[0, h, i]) / math.sqrt(d)
            assert row[int(np.argmax(z))] > 0.0
            m = z.max()
            assert m - 1.0 - 1e-12 <= tau[0, h, i] <= m - n ** (1.0 - alpha) + 1e-12


def test_common_shift_of_the_summaries_leaves_priors_unchanged(oracle):
    rng = np.random.default_rng(24)
    q, sig = _inputs(rng, 1, 4, 2, 60, 5, 8)
    pi, _ = routing.route_chunks(q, sig, 1.5, chunk_size=8)
    shifted = sig + rng.standard_normal(5)[None, None, None, :]
    pi2, _ = routing.route_chunks(q, shifted, 1.5, chunk_size=8)
    np.testing.assert_allclose(pi2, pi, atol=1e-10)


def test_visibility_rule_and_gqa_map(oracle):
    rng = np.random.default_rng(25)
    C, T = 4, 14  # four chunks, the last one ragged (2 tokens)
    q, sig = _inputs(rng, 1, 4, 2, T, 3, C)
    for causal, diag in ((True, True), (True, False), (False, True)):
        pi, tau = routing.route_chunks(q, sig, 1.5, chunk_size=C, causal=causal,
                                       estimate_diagonal=diag)
        for h in range(4):
            for i in range(T):
                own = i // C
                n = 4 if not causal else (own + 1 if diag else own)
                assert np.all(pi[0, h, i, n:] == 0.0)
                if n == 0:
                    assert np.isinf(tau[0, h, i]) and np.all(pi[0, h, i] == 0.0)
                else:
                    assert abs(pi[0, h, i, :n].sum() - 1.0) <= 1e-12
    # GQA: kv head floor(h / 2) -- the same as two query heads per repeated kv head
    pi, _ = routing.route_chunks(q, sig, 1.5, chunk_size=C)
    pi_rep, _ = routing.route_chunks(q, np.repeat(sig, 2, axis=1), 1.5, chunk_size=C)
    np.testing.assert_array_equal(pi, pi_rep)


def test_rejects_summary_count_that_does_not_match_the_chunks(oracle):
    rng = np.random.default_rng(26)
    q, sig = _inputs(rng, 1, 1, 1, 20, 4, 8)
    with pytest.raises(ValueError):
        routing.route_chunks(q, sig[:, :, :2], 1.5, chunk_size=8)
