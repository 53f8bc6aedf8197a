"""Pins for the fp64 oracle, against facts fixed by the mathematics rather than by the oracle.

The attention computed is alpha-entmax attention (AdaSplash: Adaptive Sparse Flash Attention,
sections "AdaSplash with Block Masking", "Adaptive Sparsity Control", "Variable Length
Sequences", "Causal and Non-causal Masking"), with the alpha-entmax closed form of Peters,
Niculae & Martins 2019.  Each test states what it pins:

* alpha = 2 is the Euclidean projection onto the simplex (sparsemax): checked against the
  sort-based projection of Duchi et al. 2008 and against its KKT conditions;
* alpha = 1.5's closed form against the general root-finder and against brute-force bisection;
* any alpha against brute-force bisection on all keys (tiny inputs, explicit loops), including
  causal / non-causal, GQA and the block-mask tiles;
* alpha -> 1 approaches softmax; shift and permutation invariances; sum-to-one; the tau bracket;
* hand-derived worked examples under tests/golden/.
"""
import math
import os

import numpy as np
import pytest

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------- independent helpers (tests) --

def duchi_simplex_projection(z):
    """Euclidean projection onto the probability simplex, Duchi et al. 2008 (sort-based)."""
    u = np.sort(z)[::-1]
    css = np.cumsum(u)
    j = np.arange(1, z.size + 1)
    rho = np.nonzero(u - (css - 1.0) / j > 0)[0][-1]
    theta = (css[rho] - 1.0) / (rho + 1.0)
    return np.maximum(z - theta, 0.0), theta


def bisect_tau(z, alpha, halvings=200):
    """Brute force: bisection of sum_j [z_j - t]_+^beta = 1 over all entries of z."""
    beta = 1.0 / (alpha - 1.0)
    m = float(np.max(z))
    lo, hi = m - 1.0, m - z.size ** (1.0 - alpha)
    for _ in range(halvings):
        mid = 0.5 * (lo + hi)
        total = 0.0
        for x in z:
            if x > mid:
                total += (x - mid) ** beta
        if total > 1.0:
            lo = mid
        else:
            hi = mid
    return 0.5 * (lo + hi)


def brute_attention(q, k, v, alpha, causal, G):
    """Explicit-loop alpha-entmax attention for tiny [H, T, d] problems (one sequence).
    Returns tau [Hq, T], o [Hq, T, d], p [Hq, T, T]."""
    Hq, T, d = q.shape
    beta = 1.0 / (alpha - 1.0)
    tau = np.zeros((Hq, T))
    o = np.zeros((Hq, T, d))
    p = np.zeros((Hq, T, T))
    for h in range(Hq):
        hk = h // G
        for i in range(T):
            keys = range(i + 1) if causal else range(T)
            z = []
            for j in keys:
                dot = 0.0
                for c in range(d):
                    dot += float(q[h, i, c]) * float(k[hk, j, c])
                z.append((alpha - 1.0) * dot / math.sqrt(d))
            z = np.array(z)
            t = bisect_tau(z, alpha)
            tau[h, i] = t
            for jj, j in enumerate(keys):
                if z[jj] > t:
                    p[h, i, j] = (z[jj] - t) ** beta
                    o[h, i] += p[h, i, j] * v[hk, j].astype(np.float64)
    return tau, o, p


# ------------------------------------------------------------------------------------ pins --

@pytest.mark.parametrize("n,scale,seed", [(1, 1.0, 0), (2, 0.1, 1), (7, 1.0, 2), (50, 0.3, 3),
                                          (50, 3.0, 4), (300, 1.0, 5), (1000, 10.0, 6)])
def test_sparsemax_is_simplex_projection(oracle, n, scale, seed):
    z = np.random.default_rng(seed).standard_normal(n) * scale
    p, tau = oracle.entmax_vec(z, 2.0)
    pd, theta = duchi_simplex_projection(z)
    assert np.max(np.abs(p - pd)) <= 1e-12
    assert abs(tau - theta) <= 1e-12 * max(1.0, abs(theta))
    # KKT of min ||p - z||^2 on the simplex: p_j = z_j - tau on the support, z_j <= tau off it.
    on = p > 0
    assert np.all(np.abs(p[on] - (z[on] - tau)) <= 1e-12)
    assert np.all(z[~on] <= tau + 1e-12)
    assert abs(p.sum() - 1.0) <= 1e-12


def test_sparsemax_is_nearest_point_of_simplex(oracle):
    rng = np.random.default_rng(11)
    z = rng.standard_normal(20)
    p, _ = oracle.entmax_vec(z, 2.0)
    best = np.sum((p - z) ** 2)
    for _ in range(2000):  # random points of the simplex are never closer
        x = rng.dirichlet(np.full(20, 0.3))
        assert np.sum((x - z) ** 2) >= best - 1e-12


@pytest.mark.parametrize("seed", range(6))
def test_entmax15_closed_form_matches_root_finder_and_bisection(oracle, seed):
    rng = np.random.default_rng(100 + seed)
    z = rng.standard_normal(40) * (0.5 + seed)
    p, tau = oracle.entmax_vec(z, 1.5)
    pg, taug = oracle.entmax_vec(z, 1.5, force_general=True)
    assert abs(tau - taug) <= 1e-12 * max(1.0, abs(tau))
    assert np.max(np.abs(p - pg)) <= 1e-12
    assert abs(tau - bisect_tau(z, 1.5)) <= 1e-12 * max(1.0, abs(tau))


@pytest.mark.parametrize("alpha", [1.1, 1.25, 1.333, 1.5, 1.75, 2.0, 3.0])
def test_entmax_vec_matches_bisection(oracle, alpha):
    rng = np.random.default_rng(int(alpha * 1000))
    for n in (1, 2, 3, 8, 33):
        z = rng.standard_normal(n) * 2.0
        p, tau = oracle.entmax_vec(z, alpha)
        tb = bisect_tau(z, alpha)
        assert abs(tau - tb) <= 1e-12 * max(1.0, abs(tb)), (n, tau, tb)
        assert abs(p.sum() - 1.0) <= 1e-12
        assert np.all(p >= 0)


def _read_cases(path):
    cases = []
    for line in open(path):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        a, z, t, p = [s.strip() for s in line.split("|")]
        cases.append((float(a), np.array(z.split(), dtype=float), float(t),
                      np.array(p.split(), dtype=float)))
    return cases


def test_hand_worked_examples(oracle):
    cases = _read_cases(os.path.join(GOLDEN, "entmax_hand_examples.txt"))
    assert len(cases) >= 6
    for alpha, z, tau_ref, p_ref in cases:
        p, tau = oracle.entmax_vec(z, alpha)
        assert abs(tau - tau_ref) <= 1e-12, (alpha, z, tau, tau_ref)
        assert np.max(np.abs(p - p_ref)) <= 1e-12, (alpha, z, p, p_ref)


def test_hand_worked_attention(oracle):
    rows = {}
    for line in open(os.path.join(GOLDEN, "attention_hand_example.txt")):
        if line.startswith("#") or ":" not in line:
            continue
        key, val = line.split(":", 1)
        rows[key.strip()] = np.array([[float(x) for x in r.split()] for r in val.split(";")])
    q, k, v = (rows[n].astype(np.float32)[None, None] for n in ("q", "k", "v"))
    r = oracle.attention_rows(q, k, v, alpha=2.0, causal=True)
    assert np.max(np.abs(r["tau"] - rows["tau"].ravel())) <= 1e-15
    assert np.max(np.abs(r["out"] - rows["o"])) <= 1e-15


def test_softmax_limit(oracle):
    s = np.random.default_rng(5).standard_normal(64) * 1.5
    soft = np.exp(s - s.max())
    soft /= soft.sum()
    errs = []
    for alpha in (1.1, 1.01, 1.001):
        p, _ = oracle.entmax_vec((alpha - 1.0) * s, alpha)
        errs.append(np.max(np.abs(p - soft)))
    assert errs[0] > errs[1] > errs[2]
    assert errs[2] < 5e-3
    # roughly proportional to (alpha - 1): each tenfold step shrinks the error severalfold
    assert errs[1] < errs[0] / 4 and errs[2] < errs[1] / 4


def test_shift_and_permutation_invariance(oracle):
    rng = np.random.default_rng(9)
    z = rng.standard_normal(30)
    for alpha in (1.333, 1.5, 2.0):
        p, tau = oracle.entmax_vec(z, alpha)
        p2, tau2 = oracle.entmax_vec(z + 3.25, alpha)
        assert np.max(np.abs(p - p2)) <= 1e-12 and abs(tau2 - tau - 3.25) <= 1e-12
        perm = rng.permutation(30)
        p3, tau3 = oracle.entmax_vec(z[perm], alpha)
        assert np.max(np.abs(p3 - p[perm])) <= 1e-12 and abs(tau3 - tau) <= 1e-12


@pytest.mark.parametrize("alpha", [1.333, 1.5, 2.0, 3.0])
@pytest.mark.parametrize("causal", [True, False])
def test_attention_matches_brute_force_8x8(oracle, alpha, causal):
    """Seeded 8 x 8 inputs, GQA with 2 q heads per kv head: tau, o against explicit loops +
    bisection over all keys."""
    rng = np.random.default_rng(int(alpha * 100) + causal)
    Hq, Hkv, T, d = 4, 2, 8, 8
    q = rng.standard_normal((1, Hq, T, d)).astype(np.float32) * 2
    k = rng.standard_normal((1, Hkv, T, d)).astype(np.float32) * 2
    v = rng.standard_normal((1, Hkv, T, d)).astype(np.float32)
    tau_b, o_b, _ = brute_attention(q[0], k[0], v[0], alpha, causal, G=Hq // Hkv)
    r = oracle.attention_rows(q, k, v, alpha=alpha, causal=causal)
    assert np.max(np.abs(r["tau"] - tau_b.ravel())) <= 1e-12
    assert np.max(np.abs(r["out"] - o_b.reshape(-1, d))) <= 1e-12


def test_block_mask_tiles_match_brute_force(oracle):
    """T = 300 spans three 128-key tiles with a ragged tail; the per-tile max p of every row
    must equal the brute-force p, grouped by tile."""
    rng = np.random.default_rng(21)
    T, d = 300, 4
    q = rng.standard_normal((1, 1, T, d)).astype(np.float32) * 3
    k = rng.standard_normal((1, 1, T, d)).astype(np.float32) * 3
    v = rng.standard_normal((1, 1, T, d)).astype(np.float32)
    r = oracle.attention_rows(q, k, v, alpha=1.5, causal=True)
    _, _, p = brute_attention(q[0], k[0], v[0], 1.5, True, G=1)
    assert r["maxp"].shape == (T, 3)
    for kt in range(3):
        ref = p[0][:, kt * 128:(kt + 1) * 128].max(axis=1)
        assert np.max(np.abs(r["maxp"][:, kt] - ref)) <= 1e-12


def test_one_hot_values_read_back_p_and_rows_sum_to_one(oracle):
    """v = identity (T <= d) makes o_i = p_i; every row sums to one and tau lies in
    [m - 1, m - n^(1 - alpha)]."""
    rng = np.random.default_rng(3)
    T = d = 64
    for alpha in (1.333, 1.5, 2.0):
        q = rng.standard_normal((1, 1, T, d)).astype(np.float32)
        k = rng.standard_normal((1, 1, T, d)).astype(np.float32)
        v = np.eye(T, d, dtype=np.float32)[None, None]
        r = oracle.attention_rows(q, k, v, alpha=alpha, causal=True)
        p = r["out"]
        assert np.all(p >= 0)
        assert np.max(np.abs(p.sum(axis=1) - 1.0)) <= 1e-12
        assert np.all(p[np.triu_indices(T, 1)] == 0.0)  # causal: nothing above the diagonal
        s = (q[0, 0].astype(np.float64) @ k[0, 0].astype(np.float64).T) / math.sqrt(d)
        for i in range(T):
            z = (alpha - 1.0) * s[i, :i + 1]
            m = z.max()
            assert m - 1.0 - 1e-12 <= r["tau"][i] <= m - (i + 1) ** (1.0 - alpha) + 1e-12
            pv, tv = oracle.entmax_vec(z, alpha)
            assert np.max(np.abs(pv - p[i, :i + 1])) <= 1e-12


def test_constant_values_give_constant_output_and_single_key_row(oracle):
    rng = np.random.default_rng(4)
    q = rng.standard_normal((1, 2, 40, 16)).astype(np.float32)
    k = rng.standard_normal((1, 2, 40, 16)).astype(np.float32)
    v = np.full((1, 2, 40, 16), 0.375, dtype=np.float32)
    r = oracle.attention_rows(q, k, v, alpha=1.5, causal=True)
    assert np.max(np.abs(r["out"] - 0.375)) <= 1e-12
    # row 0 of each head has a single key: p = 1, tau = z - 1
    z00 = 0.5 * float(q[0, 0, 0].astype(np.float64) @ k[0, 0, 0].astype(np.float64)) / 4.0
    assert abs(r["tau"][0] - (z00 - 1.0)) <= 1e-12
    assert r["maxp"][0, 0] == 1.0


@pytest.mark.parametrize("alpha", [1.333, 1.5, 2.0, 3.0])
def test_equal_scores_give_uniform_rows_and_the_value_prefix_mean(oracle, alpha):
    """q = 0: every score of a row is 0, so p is uniform over the row's n valid keys.  From
    sum_j (-tau)^(1/(alpha-1)) = 1: tau = -n^(1-alpha), and o_i is the mean of the first n value
    rows (causal) or of all of them (non-causal)."""
    rng = np.random.default_rng(6)
    T, d = 37, 8
    q = np.zeros((1, 2, T, d), dtype=np.float32)
    k = rng.standard_normal((1, 1, T, d)).astype(np.float32)
    v = rng.standard_normal((1, 1, T, d)).astype(np.float32)
    a = float(np.float32(alpha))
    for causal in (True, False):
        r = oracle.attention_rows(q, k, v, alpha=a, causal=causal)
        n = np.arange(1, T + 1, dtype=np.float64) if causal else np.full(T, float(T))
        vf = v[0, 0].astype(np.float64)
        mean = np.cumsum(vf, axis=0) / n[:, None] if causal else np.tile(vf.mean(axis=0), (T, 1))
        assert np.max(np.abs(r["out"] - np.concatenate([mean, mean]))) <= 1e-12
        assert np.max(np.abs(r["tau"] - np.concatenate([-(n ** (1.0 - a))] * 2))) <= 1e-12


def test_gqa_equals_repeated_kv_heads(oracle):
    """The kv head of q head h is floor(h / G): GQA equals MHA with each kv head repeated G
    times in a row."""
    rng = np.random.default_rng(8)
    q = rng.standard_normal((2, 8, 50, 16)).astype(np.float32)
    k = rng.standard_normal((2, 2, 50, 16)).astype(np.float32)
    v = rng.standard_normal((2, 2, 50, 16)).astype(np.float32)
    a = oracle.attention_rows(q, k, v, alpha=1.333, causal=True)
    b = oracle.attention_rows(q, np.repeat(k, 4, axis=1), np.repeat(v, 4, axis=1), alpha=1.333,
                              causal=True)
    assert np.array_equal(a["tau"], b["tau"]) and np.array_equal(a["out"], b["out"])


@pytest.mark.parametrize("causal", [True, False])
def test_varlen_equals_separate_sequences(oracle, causal):
    rng = np.random.default_rng(12)
    lens = [5, 130, 1, 260]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    T = int(cu[-1])
    q = rng.standard_normal((4, T, 8)).astype(np.float32)
    k = rng.standard_normal((2, T, 8)).astype(np.float32)
    v = rng.standard_normal((2, T, 8)).astype(np.float32)
    r = oracle.attention_rows(q, k, v, alpha=1.5, causal=causal, cu_seqlens=cu)
    tau = r["tau"].reshape(4, T)
    out = r["out"].reshape(4, T, 8)
    maxp = r["maxp"].reshape(4, T, -1)
    for s, L in enumerate(lens):
        a, b = cu[s], cu[s + 1]
        rs = oracle.attention_rows(q[None, :, a:b], k[None, :, a:b], v[None, :, a:b], alpha=1.5,
                                   causal=causal)
        assert np.array_equal(tau[:, a:b].ravel(), rs["tau"])
        assert np.array_equal(out[:, a:b].reshape(-1, 8), rs["out"])
        nkt = rs["maxp"].shape[1]
        assert np.array_equal(maxp[:, a:b, :nkt].reshape(-1, nkt), rs["maxp"])
        assert np.all(maxp[:, a:b, nkt:] == 0)


def test_tau_given_reproduces_p_at_that_tau(oracle):
    rng = np.random.default_rng(13)
    q = rng.standard_normal((1, 1, 200, 8)).astype(np.float32)
    k = rng.standard_normal((1, 1, 200, 8)).astype(np.float32)
    v = np.zeros((1, 1, 200, 8), dtype=np.float32)
    r = oracle.attention_rows(q, k, v, alpha=2.0, causal=True)
    shifted = r["tau"] + 0.01
    r2 = oracle.attention_rows(q, k, v, alpha=2.0, causal=True, tau_given=shifted)
    assert np.array_equal(r2["tau"], shifted)
    # raising tau by 0.01 lowers every positive p by exactly 0.01 (beta = 1), floor 0
    assert np.all(r2["maxp"] <= np.maximum(r["maxp"] - 0.01, 0.0) + 1e-12)
    assert np.all(r2["maxp"] >= r["maxp"] - 0.01 - 1e-12)


@pytest.mark.parametrize("alpha,n_iter", [(1.1, 10), (1.333, 10), (1.5, 10), (1.75, 10),
                                          (2.0, 10), (3.0, 20), (5.0, 20)])
def test_fixed_iteration_halley_search_converges(oracle, alpha, n_iter):
    """The bracketed Halley + bisection search of the "Triton Entmax" section reaches the exact
    tau on rows shaped like the attention rows (a few large scores over a Gaussian bulk): to
    fp64 rounding after n_iter steps (10 for alpha <= 2; 20 for alpha > 2, where the infinite
    slope at support edges leaves bisection to do part of the work), and to 1e-12 after 80."""
    rng = np.random.default_rng(int(alpha * 77))
    for trial in range(60):
        n = int(rng.integers(1, 3000))
        z = (alpha - 1.0) * rng.standard_normal(n) * rng.choice([0.3, 1.0, 3.0])
        spikes = rng.choice(n, size=max(1, n // 50), replace=False)
        z[spikes] *= 4.0
        _, tau = oracle.entmax_vec(z, alpha)
        scale = max(1.0, abs(tau))
        assert abs(oracle.tau_halley(z, alpha, 80) - tau) <= 1e-12 * scale
        assert abs(oracle.tau_halley(z, alpha, n_iter) - tau) <= 1e-10 * scale, (trial, n)


def test_halley_progress_test_breaks_two_cycle(oracle):
    """beta = 1/2 (alpha = 3) with the root just below a support edge: without the progress test
    the Halley steps alternate around the edge and never reach the root."""
    z = np.array([5.68103051, 5.22318906, 5.16629349, 4.49633861, 3.0, 2.0])
    _, tau = oracle.entmax_vec(z, 3.0)
    assert abs(oracle.tau_halley(z, 3.0, 25) - tau) <= 1e-12


def test_rejects_malformed_arguments(oracle):
    q = np.zeros((1, 3, 4, 2), dtype=np.float32)
    k = np.zeros((1, 2, 4, 2), dtype=np.float32)
    with pytest.raises(ValueError):  # Hq not a multiple of Hkv
        oracle.attention_rows(q, k, k, alpha=1.5)
    with pytest.raises(ValueError):
        oracle.attention_rows(q[:, :2], k, k, alpha=1.0)
    with pytest.raises(ValueError):
        oracle.attention_rows(q[:, :2], k, k, alpha=1.5, rows=[8])
