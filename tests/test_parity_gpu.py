"""GPU parity: the CUDA library through its C ABI against the fp64 oracle, element by element,
on the same seeded inputs.  See parity.py for the tolerances.

Covered: the five named workloads (whole at the small sizes; at the large sizes, whole query
tiles sampled two-sided plus loose rows one-sided, through the same entry points bench.py
times), ragged and tiny sequence lengths, non-causal attention, GQA, packed batches with empty
and one-token sequences, d = 64 and 128, alpha in {1.333, 1.5, 2, 3}, the CUDA-core path for
bf16, the multi-sweep overflow path forced on every tile, and inputs that overflow the
candidate buffers naturally, and the degenerate rows: all scores equal (uniform p, tau at the
upper end of the search bracket) and scores far apart (one-hot p).
"""
import numpy as np
import pytest
import torch

import adaptive_sparse_attention_b200 as ea
from adaptive_sparse_attention_b200 import _native
from adaptive_sparse_attention_b200.workloads import WORKLOADS, make_inputs, random_case
import parity

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.fail("a CUDA device is required for -m gpu tests")
    _native.lib()


def _sample_tiles(w, cu, per_head, rng, include_ends=True):
    tiles = []
    table = parity.seq_table(w, cu)
    nb = 1 if cu is not None else w.B
    for b in range(nb):
        for h in range(w.Hq):
            seqs = range(len(table)) if cu is not None else [b]
            for s in seqs:
                nqt = table[s][1]
                if nqt == 0:
                    continue
                pick = set(rng.choice(nqt, size=min(per_head, nqt), replace=False).tolist())
                if include_ends:
                    pick |= {0, nqt - 1}
                tiles += [(b, h, s, int(qt)) for qt in sorted(pick)]
    return tiles


@pytest.mark.parametrize("path", parity.PATHS)
@pytest.mark.parametrize("name", ["t256_fp32_d64_a1.5", "t4k_bf16_d64_a1.5"])
def test_small_workloads_every_row(oracle, name, path):
    w = WORKLOADS[name]
    inputs = make_inputs(w)
    g = parity.run_gpu(w, inputs, path=path)
    s = parity.compare(w, inputs, g, parity.all_tiles(w, inputs[3]), label=name)
    print(name, s, "fallback tiles", g.fallback_tiles)


def test_small_workload_full_forward_entry_point(oracle):
    w = WORKLOADS["t4k_bf16_d64_a1.5"]
    inputs = make_inputs(w)
    g = parity.run_gpu(w, inputs, use_fwd=True)
    parity.compare(w, inputs, g, parity.all_tiles(w, inputs[3]), label="fwd")


@pytest.mark.parametrize("path", parity.PATHS)
def test_16k_gqa_sparsemax_sampled(oracle, path):
    w = WORKLOADS["b2_t16k_gqa4_bf16_d128_a2"]
    inputs = make_inputs(w)
    g = parity.run_gpu(w, inputs, path=path)
    rng = np.random.default_rng(1000)
    tiles = _sample_tiles(w, None, 1, rng, include_ends=False)
    tiles += [(b, h, 0, 127) for b in range(2) for h in (0, 31)]  # longest rows
    loose = rng.choice(w.B * w.Hq * w.T, size=2048, replace=False)
    s = parity.compare(w, inputs, g, tiles, loose, label=w.name)
    print(w.name, s, "fallback tiles", g.fallback_tiles)


@pytest.mark.parametrize("path", parity.PATHS)
def test_varlen_gqa_alpha1333_sampled(oracle, path):
    w = WORKLOADS["varlen4_32k_gqa4_bf16_d128_a1.333"]
    inputs = make_inputs(w)
    g = parity.run_gpu(w, inputs, path=path)
    rng = np.random.default_rng(1001)
    tiles = _sample_tiles(w, inputs[3], 1, rng, include_ends=True)
    loose = rng.choice(w.Hq * w.T, size=2048, replace=False)
    s = parity.compare(w, inputs, g, tiles, loose, label=w.name)
    print(w.name, s, "fallback tiles", g.fallback_tiles)


@pytest.mark.parametrize("path", parity.PATHS)
def test_128k_sampled_rows(oracle, path):
    """512 seeded rows per head (one-sided mask) plus 4 whole query tiles per head
    (two-sided)."""
    w = WORKLOADS["t128k_gqa4_bf16_d128_a1.5"]
    inputs = make_inputs(w)
    g = parity.run_gpu(w, inputs, path=path)
    loose, tiles = [], []
    for h in range(w.Hq):
        rng = np.random.default_rng(1000 + h)
        loose.append(h * w.T + rng.choice(w.T, size=512, replace=False))
        tiles += [(0, h, 0, int(qt)) for qt in rng.choice(w.T // 128, size=4, replace=False)]
    s = parity.compare(w, inputs, g, tiles, np.concatenate(loose), label=w.name)
    print(w.name, s, "fallback tiles", g.fallback_tiles)


SMALL = [
    # name, kwargs for random_case
    ("t1", dict(B=1, Hq=1, Hkv=1, T=1, d=64)),
    ("t2_gqa", dict(B=2, Hq=4, Hkv=1, T=2, d=128)),
    ("t127", dict(B=1, Hq=2, Hkv=2, T=127, d=64, alpha=2.0)),
    ("t129", dict(B=1, Hq=2, Hkv=1, T=129, d=128, alpha=1.333)),
    ("t300_a3", dict(B=2, Hq=2, Hkv=2, T=300, d=64, alpha=3.0, spike_frac=0.05, spike_scale=4.0,
                     n_iter=20)),
    ("t1000_spk", dict(B=1, Hq=4, Hkv=2, T=1000, d=128, alpha=1.5, spike_frac=0.02,
                       spike_scale=4.0)),
    ("noncausal", dict(B=1, Hq=2, Hkv=1, T=333, d=64, alpha=1.5, causal=False)),
    ("noncausal_a2", dict(B=2, Hq=4, Hkv=4, T=520, d=128, alpha=2.0, causal=False,
                          spike_frac=0.02, spike_scale=4.0)),
    ("varlen_ragged", dict(B=None, Hq=4, Hkv=2, T=None, d=128, alpha=1.5,
                           seqlens=(5, 0, 300, 1, 129, 256))),
    ("varlen_noncausal", dict(B=None, Hq=2, Hkv=1, T=None, d=64, alpha=1.333, causal=False,
                              seqlens=(130, 7, 250))),
]


@pytest.mark.parametrize("path", parity.PATHS)
@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
@pytest.mark.parametrize("name,kw", SMALL, ids=[s[0] for s in SMALL])
def test_small_cases(oracle, name, kw, dtype, path):
    w, inputs = random_case(dtype=dtype, name=name, seed=7, **kw)
    g = parity.run_gpu(w, inputs, path=path)
    parity.compare(w, inputs, g, parity.all_tiles(w, inputs[3]), label=f"{name}/{dtype}")


@pytest.mark.parametrize("flags", [_native.FLAG_CUDA_CORES, _native.FLAG_ALL_FALLBACK,
                                   _native.FLAG_CUDA_CORES | _native.FLAG_ALL_FALLBACK],
                         ids=["cuda_cores", "all_fallback", "cuda_cores_all_fallback"])
@pytest.mark.parametrize("name,kw", [SMALL[5], SMALL[7], SMALL[8]],
                         ids=[SMALL[5][0], SMALL[7][0], SMALL[8][0]])
@pytest.mark.parametrize("path", parity.PATHS)
def test_alternate_paths(oracle, name, kw, flags, path):
    w, inputs = random_case(dtype="bf16", name=name, seed=11, **kw)
    g = parity.run_gpu(w, inputs, flags=flags, path=path)
    if flags & _native.FLAG_ALL_FALLBACK:
        assert g.fallback_tiles == sum(1 for _ in parity.all_tiles(w, inputs[3]))
    parity.compare(w, inputs, g, parity.all_tiles(w, inputs[3]), label=f"{name}/{flags}")


@pytest.mark.parametrize("alpha", [1.333, 1.5, 2.0])
@pytest.mark.parametrize("path", parity.PATHS)
def test_candidate_overflow_is_exact(oracle, alpha, path):
    """Tiny score spread (q, k scaled by 1/16) puts hundreds of keys within 1 of the row max, so
    rows overflow the 64-slot candidate buffers; tied keys (repeated rows of k) defeat the
    pruning too.  The result must stay exact."""
    w, (q, k, v, cu) = random_case(B=1, Hq=2, Hkv=1, T=700, d=64, dtype="bf16", alpha=alpha,
                                   name="overflow", seed=3)
    q = (q.float() / 16).to(torch.bfloat16)
    k = (k.float() / 16).to(torch.bfloat16)
    k[:, :, 200:400] = k[:, :, 200:201]  # 200 identical keys
    inputs = (q, k, v, cu)
    g = parity.run_gpu(w, inputs, path=path)
    assert g.fallback_tiles > 0
    parity.compare(w, inputs, g, parity.all_tiles(w, cu), label=f"overflow/{alpha}")


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
@pytest.mark.parametrize("alpha", [1.5, 2.0])
@pytest.mark.parametrize("path", parity.PATHS)
def test_equal_scores_give_uniform_rows(oracle, alpha, dtype, path):
    """q = 0 makes every score of a row equal, so p is uniform over the row's valid keys
    (p_j = 1/n for all j, tau = -n^(1-alpha)) and o is the mean of the value prefix.  Every key
    is then a candidate: rows longer than the buffers take the overflow path.  Checked against
    the oracle and against that closed form."""
    w, (q, k, v, cu) = random_case(B=1, Hq=4, Hkv=2, T=300, d=128, dtype=dtype, alpha=alpha,
                                   name="equal_scores", seed=13)
    q = torch.zeros_like(q)
    inputs = (q, k, v, cu)
    g = parity.run_gpu(w, inputs, path=path)
    assert g.fallback_tiles > 0
    parity.compare(w, inputs, g, parity.all_tiles(w, cu), label=f"equal_scores/{dtype}/{alpha}")
    vf = v.double().numpy()
    n = np.arange(1, w.T + 1, dtype=np.float64)
    G = w.Hq // w.Hkv
    want = np.stack([np.cumsum(vf[0, h // G], axis=0) / n[:, None] for h in range(w.Hq)])
    want = want.reshape(-1, w.d)
    bar = parity.out_bar(w, want)
    assert np.all(np.abs(g.out - want) <= bar), "output is not the mean of the value prefix"
    want_tau = -(n ** (1.0 - float(np.float32(alpha))))
    np.testing.assert_allclose(g.tau.reshape(w.Hq, w.T), np.broadcast_to(want_tau, (w.Hq, w.T)),
                               rtol=parity.TAU_RTOL, atol=parity.TAU_RTOL)


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
@pytest.mark.parametrize("path", parity.PATHS)
def test_far_apart_scores_give_one_hot_rows(oracle, dtype, path):
    """q scaled by 16 against spiked keys spreads the scores of a row over hundreds of units, so
    most rows put all their mass on one key (p one-hot, o = that key's value row).  The mask then
    holds few tiles per row; the result must match the oracle, including rows whose support
    still has two or more keys."""
    w, (q, k, v, cu) = random_case(B=2, Hq=4, Hkv=1, T=400, d=64, dtype=dtype, alpha=1.5,
                                   spike_frac=0.02, spike_scale=4.0, name="one_hot", seed=17)
    q = (q.float() * 16).to(q.dtype)
    inputs = (q, k, v, cu)
    g = parity.run_gpu(w, inputs, path=path)
    parity.compare(w, inputs, g, parity.all_tiles(w, cu), label=f"one_hot/{dtype}")


@pytest.mark.parametrize("name,kw", [SMALL[5], SMALL[8]], ids=[SMALL[5][0], SMALL[8][0]])
def test_support_path_without_room_for_the_lists(oracle, name, kw):
    """ENTMAX_ATTN_FLAG_SUPPORT on a workspace with the warm-up sections but no room for the
    support lists: every query tile takes the tile output pass, with the same results."""
    w, inputs = random_case(dtype="bf16", name=name, seed=19, **kw)
    q, k, v, cu = (t.cuda() if t is not None else None for t in inputs)
    B, Hq, Hkv, T, d = ea.api.problem_dims(q, k, cu)
    full = ea.workspace_bytes(B, Hq, T, cu is not None)
    ws = torch.empty(full, dtype=torch.uint8, device="cuda")
    room = ws[:full - 256]  # one byte short of the support lists' end: no support lists
    out, tau, mask, _ = ea.entmax_attn_fused(q, k, v, oracle.alpha_as_float32(w.alpha),
                                             w.n_iter, w.causal, cu, workspace=room)
    torch.cuda.synchronize()
    assert ea.status() == 0
    g = parity.GpuResult(out.float().cpu().numpy().reshape(-1, w.d), tau.cpu().numpy().ravel(),
                         ea.decode_block_mask(mask.cpu().numpy(), w.B, w.Hq, w.T, inputs[3]), -1)
    parity.compare(w, inputs, g, parity.all_tiles(w, inputs[3]), label=f"support_noroom/{name}")


@pytest.mark.parametrize("path", parity.PATHS)
def test_large_supports(oracle, path):
    """Near-flat scores at alpha = 1.333 (q scaled by 1/4) give supports of tens of keys per
    row: query tiles whose rows need more entries than a tile's support list holds, or more
    candidates than the buffers hold, take the tile output pass; every row must still match."""
    w, (q, k, v, cu) = random_case(B=1, Hq=4, Hkv=2, T=1500, d=128, dtype="bf16", alpha=1.333,
                                   name="large_supports", seed=37)
    q = (q.float() / 4).to(q.dtype)
    inputs = (q, k, v, cu)
    g = parity.run_gpu(w, inputs, path=path)
    parity.compare(w, inputs, g, parity.all_tiles(w, cu), label=f"large_supports/{path}")
