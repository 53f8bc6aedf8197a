"""GPU parity of entmax block routing (entmax_attn_route_chunks) against the fp64 routing oracle
(oracle/routing.py) on the same seeded inputs: tau within 1e-4 max(1, |tau|) (+inf where a row
sees no chunk), priors within 1e-4 (plus the derived 2^(-20 beta) for beta < 1, as for the
row-wise entmax: the kernel scores in fp32 from the exact inputs)."""
import numpy as np
import pytest
import torch

import adaptive_sparse_attention_b200 as ea
from oracle import oracle as orc
from oracle import routing

pytestmark = pytest.mark.gpu


def _case(B, Hq, Hkv, T, d, C, dtype, seed):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, Hq, T, d, generator=g) * 2.0
    nc = -(-T // C)
    sig = torch.randn(B, Hkv, nc, d, generator=g)
    sig[:, :, ::7] *= 3.0  # a few loud summaries: peaked rows
    dt = torch.bfloat16 if dtype == "bf16" else torch.float32
    return q.to(dt), sig.to(dt)


def _check(q, sig, alpha, n_iter, C, causal, diag, scaling=1.0):
    a32 = orc.alpha_as_float32(alpha)
    pi, tau = ea.route_chunks(q.cuda(), sig.cuda(), a32, C, n_iter, causal, diag, scaling)
    torch.cuda.synchronize()
    assert ea.status() == 0
    want_pi, want_tau = routing.route_chunks(q, sig, a32, C, causal, diag, scaling)
    got_pi, got_tau = pi.cpu().double().numpy(), tau.cpu().double().numpy()
    empty = np.isinf(want_tau)
    assert np.array_equal(np.isinf(got_tau), empty)
    assert np.all(got_pi[empty] == 0.0)
    ok = ~empty
    err_t = np.abs(got_tau[ok] - want_tau[ok]) / np.maximum(1.0, np.abs(want_tau[ok]))
    assert float(err_t.max(initial=0.0)) <= 1e-4, float(err_t.max())
    beta = 1.0 / (a32 - 1.0)
    bar = 1e-4 + (2.0 ** (-20.0 * beta) if beta < 1.0 else 0.0)
    err_p = float(np.abs(got_pi - want_pi).max())
    assert err_p <= bar, err_p


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
@pytest.mark.parametrize("alpha,n_iter", [(1.333, 10), (1.5, 10), (2.0, 10), (3.0, 40)])
@pytest.mark.parametrize("causal,diag", [(True, True), (True, False), (False, True)],
                         ids=["causal_diag", "causal_nodiag", "noncausal"])
def test_routing_matches_oracle(oracle, dtype, alpha, n_iter, causal, diag):
    q, sig = _case(2, 4, 2, 300, 64, 16, dtype, seed=40)
    _check(q, sig, alpha, n_iter, 16, causal, diag)


@pytest.mark.parametrize("C", [1, 64, 300, 512])
def test_routing_chunk_sizes(oracle, C):
    """One-token chunks (routing = entmax attention over the keys), the default 64, one chunk
    for the whole sequence, and a chunk longer than the sequence."""
    q, sig = _case(1, 2, 1, 300, 32, C, "fp32", seed=41)
    _check(q, sig, 1.5, 10, C, True, True, scaling=0.7)


def test_routing_4k_heads(oracle):
    """4096 tokens, eight query heads over two kv heads, d = 128, chunks of 64 (64 chunks)."""
    q, sig = _case(1, 8, 2, 4096, 128, 64, "bf16", seed=42)
    _check(q, sig, 1.5, 10, 64, True, True)


@pytest.mark.parametrize("T,d,C", [(1000, 128, 7), (2304, 64, 16), (8192, 128, 16)],
                         ids=["ragged_nc143", "d64_nc144", "nc512"])
def test_routing_tensor_core_scores(oracle, T, d, C):
    """bf16 with d = 64 or 128: the chunk scores come from the tensor cores (128-row x 128-chunk
    tiles), the search from the CUDA cores.  Ragged row and chunk counts (a chunk count that is
    not a multiple of 4 takes the element-wise store), and 512 chunks per row."""
    q, sig = _case(1, 4, 2, T, d, C, "bf16", seed=43)
    _check(q, sig, 1.5, 10, C, True, True)
    _check(q, sig, 2.0, 10, C, False, True)


@pytest.mark.parametrize("dtype,d", [("fp32", 32), ("bf16", 64)])
def test_routing_many_chunks(oracle, dtype, d):
    """Rows that see up to 600 chunks (two-token chunks of 1200 tokens): 19 per lane of the
    row's warp, past the 512 of the other cases."""
    q, sig = _case(1, 2, 1, 1200, d, 2, dtype, seed=44)
    _check(q, sig, 1.5, 10, 2, True, True)
    _check(q, sig, 2.0, 10, 2, False, True)
