"""GPU parity of the backward pass (entmax_attn_bwd) against the fp64 backward oracle.

The forward runs first on the GPU (tau pass + output pass: tau, the compact lists and, on the
support path, the support lists the backward reuses); the oracle computes the gradients from
the same stored inputs with its exact tau.  Both paths: "support" (forward and backward with
ENTMAX_ATTN_FLAG_SUPPORT: rows with a recorded support from their supports, the other query
tiles over their listed key tiles) and "tile" (every query tile over its listed key tiles).
Bar: max-abs error <= 1e-3 * max(1, max |reference|) per gradient.  Derivation: the kernels
compute in fp32 from the exact stored values, with the GPU's tau (within ~1e-7 of the exact one)
and without the key tiles the mask may skip (max p < 1e-6); dk and dv sum up to a few thousand
fp32 terms per element (rows x query heads), whose rounding stays near 1e-6 relative, and ds
scales differences of u by w <= 1 for alpha <= 2, so 1e-3 leaves two orders of margin while a
wrong term, sign or index moves results by O(1).
"""
import numpy as np
import pytest
import torch

from adaptive_sparse_attention_b200 import _native
import adaptive_sparse_attention_b200 as ea
from adaptive_sparse_attention_b200.workloads import WORKLOADS, make_inputs, random_case
from oracle import backward as obwd
from oracle import oracle as orc

pytestmark = pytest.mark.gpu

CASES = [
    ("t300_d64_a1.5", dict(B=1, Hq=2, Hkv=2, T=300, d=64, alpha=1.5, spike_frac=0.02,
                           spike_scale=4.0), "bf16", 0),
    ("t200_gqa_d128_a2", dict(B=2, Hq=4, Hkv=2, T=200, d=128, alpha=2.0), "bf16", 0),
    ("varlen_a1.333", dict(B=None, Hq=2, Hkv=1, T=None, d=128, alpha=1.333, spike_frac=0.02,
                           spike_scale=4.0, seqlens=[130, 5, 260]), "bf16", 0),
    ("noncausal_d64", dict(B=1, Hq=2, Hkv=1, T=150, d=64, alpha=1.5, causal=False), "bf16", 0),
    ("fp32_t129", dict(B=1, Hq=2, Hkv=2, T=129, d=64, alpha=1.5), "fp32", 0),
    ("no_block_mask", dict(B=1, Hq=2, Hkv=1, T=260, d=128, alpha=1.5), "bf16",
     _native.FLAG_NO_BLOCK_MASK),
    # every query tile through the overflow kernel: on the support path its lists come from that
    # kernel's extra sweep
    ("all_fallback_varlen", dict(B=None, Hq=4, Hkv=2, T=None, d=128, alpha=1.5,
                                 seqlens=[200, 1, 330]), "bf16", _native.FLAG_ALL_FALLBACK),
]


PATHS = ("support", "tile")


def _gpu_backward(w, inputs, g, flags=0, path="support"):
    q, k, v, cu = inputs
    dev = torch.device("cuda:0")
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    cud = cu.to(dev) if cu is not None else None
    alpha = orc.alpha_as_float32(w.alpha)
    if path == "support":
        flags |= _native.FLAG_SUPPORT
    out, tau, mask, ws = ea.entmax_attn_two_pass(qd, kd, vd, alpha, w.n_iter, w.causal, cud,
                                                 flags=flags)
    dq, dk, dv, delta = ea.entmax_attn_bwd(qd, kd, vd, g.to(dev), tau, ws, alpha, w.causal, cud,
                                           flags=flags)
    torch.cuda.synchronize()
    assert ea.status() == 0
    return dq.cpu().numpy(), dk.cpu().numpy(), dv.cpu().numpy(), delta.cpu().numpy()


def _check(name, got, want, labels=("dq", "dk", "dv", "delta")):
    for label, a, b in zip(labels, got, want):
        bar = 1e-3 * max(1.0, float(np.abs(b).max()))
        err = float(np.abs(a - b).max())
        assert err <= bar, f"{name}: {label} max-abs error {err:.3e} > {bar:.3e}"


@pytest.mark.parametrize("path", PATHS)
@pytest.mark.parametrize("name,kw,dtype,flags", CASES, ids=[c[0] for c in CASES])
def test_backward_matches_oracle(oracle, name, kw, dtype, flags, path):
    kw = dict(kw)
    w, inputs = random_case(dtype=dtype, name=name, seed=31, **kw)
    q, k, v, cu = inputs
    gen = torch.Generator().manual_seed(32)
    g = torch.randn(q.shape, generator=gen).to(q.dtype)
    got = _gpu_backward(w, inputs, g, flags, path)
    want = obwd.attention_backward(q, k, v, g, orc.alpha_as_float32(w.alpha), w.causal,
                                   None if cu is None else cu.numpy())
    _check(name, got, want)


@pytest.mark.parametrize("path", PATHS)
def test_backward_4k_workload(oracle, path):
    """The 4K workload (B=1, Hq=Hkv=8, T=4096, d=64, bf16, alpha 1.5, key spikes) in full."""
    w = WORKLOADS["t4k_bf16_d64_a1.5"]
    inputs = make_inputs(w, 0)
    gen = torch.Generator().manual_seed(33)
    g = torch.randn(inputs[0].shape, generator=gen).to(inputs[0].dtype)
    got = _gpu_backward(w, inputs, g, path=path)
    q, k, v, _ = inputs
    want = obwd.attention_backward(q, k, v, g, orc.alpha_as_float32(w.alpha), w.causal, None)
    _check(w.name, got, want)


def test_backward_16k_sampled_rows_and_sums(oracle):
    """The 16K GQA sparsemax workload on the support path: dq and delta of sampled rows against
    the oracle's per-row gradients (bar as above, from the sampled rows' magnitudes), and the
    properties that fix dk and dv at any size: a common shift of a sequence's keys leaves every
    row's p unchanged, so each kv head's dk sums to zero over the keys; every row's p sums to
    one, so each kv head's dv sums to the sum of dout over its query heads."""
    w = WORKLOADS["b2_t16k_gqa4_bf16_d128_a2"]
    inputs = make_inputs(w, 0)
    q, k, v, _ = inputs
    gen = torch.Generator().manual_seed(34)
    g = torch.randn(q.shape, generator=gen).to(q.dtype)
    dq, dk, dv, delta = _gpu_backward(w, inputs, g, path="support")
    rng = np.random.default_rng(35)
    rows = rng.choice(w.B * w.Hq * w.T, size=256, replace=False)
    want_dq, want_delta = obwd.row_gradients(q, k, v, g, orc.alpha_as_float32(w.alpha), w.causal,
                                             None, rows)
    _check("16k rows", (dq.reshape(-1, w.d)[rows], delta.reshape(-1)[rows]),
           (want_dq, want_delta), labels=("dq", "delta"))
    G = w.Hq // w.Hkv
    gsum = g.double().numpy().reshape(w.B, w.Hkv, G, w.T, w.d).sum(axis=(2, 3))  # [B, Hkv, d]
    dvsum = dv.astype(np.float64).sum(axis=2)
    np.testing.assert_allclose(dvsum, gsum, rtol=0, atol=1e-3 * max(1.0, np.abs(gsum).max()))
    dksum = dk.astype(np.float64).sum(axis=2)
    assert np.abs(dksum).max() <= 1e-3 * max(1.0, np.abs(dk).sum(axis=2).max())
