"""GPU parity of the variant without block mask (AdaSplash page, "adasplash_no_block_mask"): the
output pass visits every causally valid key tile.  Its tau and out must match the oracle with the
same tolerances as the masked pass.  Its tau comes from the same search as the masked pass's, up
to the fp32 rounding of the candidate sums (the order in which candidates sit in their buffers
depends on when the warps of a row publish its running max), and its out may differ from the
masked pass's only where a key tile the mask skips would add p > 0, which the mask rule allows
for p < 1e-6."""
import numpy as np
import pytest
import torch

from adaptive_sparse_attention_b200 import _native
import adaptive_sparse_attention_b200 as ea
from adaptive_sparse_attention_b200.workloads import WORKLOADS, make_inputs, random_case
from oracle import oracle as orc
import parity

pytestmark = pytest.mark.gpu

CASES = [
    ("t127", dict(B=1, Hq=2, Hkv=2, T=127, d=64, alpha=2.0), "bf16"),
    ("t129", dict(B=1, Hq=2, Hkv=1, T=129, d=128, alpha=1.333), "bf16"),
    ("t1000_spk", dict(B=1, Hq=4, Hkv=2, T=1000, d=128, alpha=1.5, spike_frac=0.02,
                       spike_scale=4.0), "bf16"),
    ("noncausal", dict(B=1, Hq=2, Hkv=1, T=333, d=64, alpha=1.5, causal=False), "bf16"),
    ("varlen_ragged", dict(B=None, Hq=4, Hkv=2, T=None, d=128, alpha=1.5,
                           seqlens=(1, 200, 0, 129, 300)), "bf16"),
    ("t300_fp32", dict(B=2, Hq=2, Hkv=2, T=300, d=64, alpha=1.5), "fp32"),
]


def _no_mask_result(w, inputs, g_masked, two_pass):
    q, k, v, cu = inputs
    dev = torch.device("cuda:0")
    q, k, v = q.to(dev), k.to(dev), v.to(dev)
    cu_d = cu.to(dev) if cu is not None else None
    alpha = orc.alpha_as_float32(w.alpha)
    if two_pass:
        out, tau, _, ws = ea.entmax_attn_two_pass(q, k, v, alpha, w.n_iter, w.causal, cu_d,
                                                  flags=_native.FLAG_NO_BLOCK_MASK)
    else:
        out, tau = ea.entmax_attn_fwd_no_block_mask(q, k, v, alpha, w.n_iter, w.causal, cu_d)
    torch.cuda.synchronize()
    assert ea.status() == 0
    return parity.GpuResult(out.float().cpu().numpy().reshape(-1, w.d), tau.cpu().numpy().ravel(),
                            g_masked.bits, g_masked.fallback_tiles)


@pytest.mark.parametrize("two_pass", [False, True], ids=["fwd", "two_pass"])
@pytest.mark.parametrize("name,kw,dtype", CASES, ids=[c[0] for c in CASES])
def test_no_block_mask_small(oracle, name, kw, dtype, two_pass):
    kw = dict(kw)
    if "seqlens" in kw:
        kw["seqlens"] = list(kw["seqlens"])
    w, inputs = random_case(dtype=dtype, name=name, seed=13, **kw)
    g = parity.run_gpu(w, inputs, path="tile")  # the same output kernel over fewer tiles
    n = _no_mask_result(w, inputs, g, two_pass)
    np.testing.assert_allclose(n.tau, g.tau, rtol=1e-6, atol=1e-6)  # the same search
    parity.compare(w, inputs, n, parity.all_tiles(w, inputs[3]), label=f"nomask/{name}")


def test_no_block_mask_16k_sampled(oracle):
    w = WORKLOADS["b2_t16k_gqa4_bf16_d128_a2"]
    inputs = make_inputs(w, seed=0)
    g = parity.run_gpu(w, inputs, path="tile")  # the same output kernel over fewer tiles
    n = _no_mask_result(w, inputs, g, two_pass=True)
    np.testing.assert_allclose(n.tau, g.tau, rtol=1e-6, atol=1e-6)
    assert float(np.max(np.abs(n.out - g.out))) <= 2e-2
    rng = np.random.default_rng(21)
    tiles = [(b, h, b, int(qt)) for b in range(w.B) for h in (0, 13, 31)
             for qt in sorted(set(rng.choice(w.T // 128, size=3, replace=False).tolist()) | {0, 127})]
    parity.compare(w, inputs, n, tiles, label="nomask/16k")
