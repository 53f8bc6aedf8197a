"""GPU parity of the backward pass (entmax_attn_bwd) against the fp64 backward oracle.

The forward runs first on the GPU (tau pass + output pass: tau and the compact lists the
backward reuses); the oracle computes the gradients from the same stored inputs with its exact
tau.  Bar: max-abs error <= 1e-3 * max(1, max |reference|) per gradient.  Derivation: the kernels
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
]


def _gpu_backward(w, inputs, g, flags=0):
    q, k, v, cu = inputs
    dev = torch.device("cuda:0")
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    cud = cu.to(dev) if cu is not None else None
    alpha = orc.alpha_as_float32(w.alpha)
    out, tau, mask, ws = ea.entmax_attn_two_pass(qd, kd, vd, alpha, w.n_iter, w.causal, cud,
                                                 flags=flags)
    dq, dk, dv, delta = ea.entmax_attn_bwd(qd, kd, vd, g.to(dev), tau, ws, alpha, w.causal, cud,
                                           flags=flags)
    torch.cuda.synchronize()
    assert ea.status() == 0
    return dq.cpu().numpy(), dk.cpu().numpy(), dv.cpu().numpy(), delta.cpu().numpy()


def _check(name, got, want):
    for label, a, b in zip(("dq", "dk", "dv", "delta"), got, want):
        bar = 1e-3 * max(1.0, float(np.abs(b).max()))
        err = float(np.abs(a - b).max())
        assert err <= bar, f"{name}: {label} max-abs error {err:.3e} > {bar:.3e}"


@pytest.mark.parametrize("name,kw,dtype,flags", CASES, ids=[c[0] for c in CASES])
def test_backward_matches_oracle(oracle, name, kw, dtype, flags):
    kw = dict(kw)
    w, inputs = random_case(dtype=dtype, name=name, seed=31, **kw)
    q, k, v, cu = inputs
    gen = torch.Generator().manual_seed(32)
    g = torch.randn(q.shape, generator=gen).to(q.dtype)
    got = _gpu_backward(w, inputs, g, flags)
    want = obwd.attention_backward(q, k, v, g, orc.alpha_as_float32(w.alpha), w.causal,
                                   None if cu is None else cu.numpy())
    _check(name, got, want)


def test_backward_4k_workload(oracle):
    """The 4K workload (B=1, Hq=Hkv=8, T=4096, d=64, bf16, alpha 1.5, key spikes) in full."""
    w = WORKLOADS["t4k_bf16_d64_a1.5"]
    inputs = make_inputs(w, 0)
    gen = torch.Generator().manual_seed(33)
    g = torch.randn(inputs[0].shape, generator=gen).to(inputs[0].dtype)
    got = _gpu_backward(w, inputs, g)
    q, k, v, _ = inputs
    want = obwd.attention_backward(q, k, v, g, orc.alpha_as_float32(w.alpha), w.causal, None)
    _check(w.name, got, want)
