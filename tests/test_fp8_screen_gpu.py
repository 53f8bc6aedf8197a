"""GPU parity of the FP8-screened tau pass (entmax_attn_tau_pass_screened) against the fp64
oracle, on the bars of parity.py.  The screen only removes key tiles that cannot hold a
candidate, so every output must match as for the unscreened pass: small fixed-length, GQA,
packed ragged and non-causal problems on every row, with and without the support lists, and the
16K and 128K workloads on sampled query tiles and rows (the 128K one also reports how many key
tiles the screen kept)."""
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


def _screen_counts(w, screen, cu):
    """The per-query-tile counts of screened key tiles, read from the documented order of the
    screen buffer's sections (q8, q statistics, k8, key-tile statistics, lists, counts)."""
    up = lambda x: (x + 255) // 256 * 256  # noqa: E731
    nb = 1 if cu is not None else w.B
    slots, _ = ea.mask_layout(w.B, w.Hq, w.T, cu is not None)
    nkt = -(-w.T // 128)
    tiles = nb * w.Hq * slots
    off = (up(nb * w.Hq * w.T * 128) + up(nb * w.Hq * w.T * 16) + up(nb * w.Hkv * w.T * 128)
           + up(nb * w.Hkv * slots * 16) + up(4 * tiles * nkt))
    return screen[off:off + 4 * tiles].view(torch.int32).cpu().numpy()


def _run(w, inputs, flags=0):
    q, k, v, cu = inputs
    dev = torch.device("cuda:0")
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    cud = cu.to(dev) if cu is not None else None
    alpha = float(np.float32(w.alpha))
    out, tau, mask, ws, scr = ea.entmax_attn_screened(qd, kd, vd, alpha, w.n_iter, w.causal, cud,
                                                      flags=flags)
    torch.cuda.synchronize()
    assert ea.status() == 0
    g = parity.GpuResult(out.float().cpu().numpy().reshape(-1, w.d), tau.cpu().numpy().ravel(),
                         ea.decode_block_mask(mask.cpu().numpy(), w.B, w.Hq, w.T, cu),
                         ea.fallback_tiles(ws))
    return g, _screen_counts(w, scr, cu)


CASES = [
    ("t1000_spk", dict(B=1, Hq=4, Hkv=2, T=1000, d=128, alpha=1.5, spike_frac=0.02,
                       spike_scale=4.0)),
    ("gqa_a2", dict(B=2, Hq=4, Hkv=1, T=700, d=128, alpha=2.0, spike_frac=0.02, spike_scale=4.0)),
    ("varlen_ragged", dict(B=None, Hq=4, Hkv=2, T=None, d=128, alpha=1.333,
                           seqlens=(5, 0, 300, 1, 129, 256))),
    ("noncausal", dict(B=1, Hq=2, Hkv=2, T=520, d=128, alpha=1.5, causal=False, spike_frac=0.02,
                       spike_scale=4.0)),
]


@pytest.mark.parametrize("flags", [0, _native.FLAG_SUPPORT], ids=["tile", "support"])
@pytest.mark.parametrize("name,kw", CASES, ids=[c[0] for c in CASES])
def test_screened_small_cases(oracle, name, kw, flags):
    w, inputs = random_case(dtype="bf16", name=name, seed=51, **kw)
    g, _ = _run(w, inputs, flags)
    parity.compare(w, inputs, g, parity.all_tiles(w, inputs[3]), label=f"fp8/{name}")


def test_screened_16k_sampled(oracle):
    w = WORKLOADS["b2_t16k_gqa4_bf16_d128_a2"]
    inputs = make_inputs(w)
    g, counts = _run(w, inputs, _native.FLAG_SUPPORT)
    rng = np.random.default_rng(52)
    tiles = [(b, h, b, int(qt)) for b in range(w.B) for h in (0, 9, 31)
             for qt in sorted(set(rng.choice(w.T // 128, size=2, replace=False).tolist()) | {127})]
    loose = rng.choice(w.B * w.Hq * w.T, size=1024, replace=False)
    parity.compare(w, inputs, g, tiles, loose, label="fp8/16k")
    nkt = w.T // 128
    total = w.B * w.Hq * nkt * (nkt + 1) // 2
    print("16K: key tiles kept by the screen", int(counts.sum()), "of", total)


def test_screened_128k_sampled(oracle):
    w = WORKLOADS["t128k_gqa4_bf16_d128_a1.5"]
    inputs = make_inputs(w)
    g, counts = _run(w, inputs, _native.FLAG_SUPPORT)
    loose, tiles = [], []
    for h in range(0, w.Hq, 4):
        rng = np.random.default_rng(2000 + h)
        loose.append(h * w.T + rng.choice(w.T, size=256, replace=False))
        tiles += [(0, h, 0, int(qt)) for qt in rng.choice(w.T // 128, size=2, replace=False)]
    parity.compare(w, inputs, g, tiles, np.concatenate(loose), label="fp8/128k")
    nkt = w.T // 128
    total = w.Hq * nkt * (nkt + 1) // 2
    kept = int(counts.sum())
    print("128K: key tiles kept by the screen", kept, "of", total, f"({kept / total:.3f})")
    assert 0 < kept < total
