"""GPU checks of the tau pass's warm-up keys.

The bf16 tau pass starts every query tile with one product against the 128 keys of largest norm
in a prefix of the tile's visible keys; their scores only raise the candidate threshold, so the
results must not depend on them.  Checked here:
  * parity with the oracle both with the full workspace (warm-up keys used) and with the
    smallest one the passes accept (no warm-up keys), and the same tau from both;
  * the workspace sections themselves: the squared norms against fp64 norms of the same keys,
    and every warm-up tile against the definition -- 128 distinct rows of the level's key
    range, copied bit for bit, whose norms are the 128 largest of the range.
"""
import numpy as np
import pytest
import torch

import adaptive_sparse_attention_b200 as ea
from adaptive_sparse_attention_b200.workloads import random_case
from oracle import oracle as orc
import parity

pytestmark = pytest.mark.gpu

CASES = [
    ("t2500_spk_a1.5", dict(B=1, Hq=4, Hkv=2, T=2500, d=128, alpha=1.5, spike_frac=0.02,
                            spike_scale=4.0)),
    ("t3000_d64_a2", dict(B=2, Hq=2, Hkv=1, T=3000, d=64, alpha=2.0)),
    ("varlen_a1.333", dict(B=None, Hq=4, Hkv=2, T=None, d=128, alpha=1.333, spike_frac=0.02,
                           spike_scale=4.0, seqlens=[1500, 40, 3100, 1200])),
    ("noncausal_d64", dict(B=1, Hq=2, Hkv=2, T=2100, d=64, alpha=1.5, causal=False,
                           spike_frac=0.01, spike_scale=5.0)),
]


def _case(name, kw):
    return random_case(dtype="bf16", name=name, seed=21, **dict(kw))


def _run(w, inputs, ws_bytes):
    q, k, v, cu = inputs
    dev = torch.device("cuda:0")
    q, k, v = q.to(dev), k.to(dev), v.to(dev)
    cu_d = cu.to(dev) if cu is not None else None
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    out, tau, mask, _ = ea.entmax_attn_two_pass(q, k, v, orc.alpha_as_float32(w.alpha), w.n_iter,
                                                w.causal, cu_d, workspace=ws)
    torch.cuda.synchronize()
    assert ea.status() == 0
    bits = ea.decode_block_mask(mask.cpu().numpy(), w.B, w.Hq, w.T, cu)
    g = parity.GpuResult(out.float().cpu().numpy().reshape(-1, w.d), tau.cpu().numpy().ravel(),
                         bits, ea.fallback_tiles(ws))
    return g, ws


@pytest.mark.parametrize("name,kw", CASES, ids=[c[0] for c in CASES])
def test_results_do_not_depend_on_warm_up_keys(oracle, name, kw):
    w, inputs = _case(name, kw)
    packed = inputs[3] is not None
    full = ea.workspace_bytes(w.B, w.Hq, w.T, packed)
    small = ea.workspace_min_bytes(w.B, w.Hq, w.T, packed)
    assert small < full
    g_full, _ = _run(w, inputs, full)
    g_small, _ = _run(w, inputs, small)
    # the same search over the same candidates, up to the order of fp32 sums
    np.testing.assert_allclose(g_full.tau, g_small.tau, rtol=1e-6, atol=1e-6)
    tiles = parity.all_tiles(w, inputs[3])
    parity.compare(w, inputs, g_full, tiles, label=f"warm/{name}")
    parity.compare(w, inputs, g_small, tiles, label=f"nowarm/{name}")


def _levels(n):
    j = 0
    while (1024 << j) <= n:
        j += 1
    return j


@pytest.mark.parametrize("name,kw", CASES, ids=[c[0] for c in CASES])
def test_warm_up_sections_follow_their_definition(name, kw):
    w, inputs = _case(name, kw)
    q, k, v, cu = inputs
    packed = cu is not None
    full = ea.workspace_bytes(w.B, w.Hq, w.T, packed)
    small = ea.workspace_min_bytes(w.B, w.Hq, w.T, packed)
    _, ws = _run(w, inputs, full)
    raw = ws.cpu().numpy()
    kk = k.float().numpy().reshape(-1, w.d).astype(np.float64)   # [kv rows, d]
    kbits = k.view(torch.int16).numpy().reshape(-1, w.d)
    rows = kk.shape[0]
    norms_gpu = raw[small:small + 4 * rows].view(np.float32)
    norms_ref = (kk * kk).sum(axis=1)
    np.testing.assert_allclose(norms_gpu, norms_ref, rtol=1e-5, atol=1e-6)

    norm_rows = (1 if packed else w.B) * w.Hq * w.T
    warm_off = small + (4 * norm_rows + 255) // 256 * 256
    J = _levels(w.T)
    tile_elems = 128 * w.d
    warm = raw[warm_off:warm_off + 2 * w.B * w.Hq * J * tile_elems].view(np.int16)
    cu_l = cu.tolist() if packed else None
    checked = 0
    for grp in range(w.B * w.Hkv):
        s, kvh = divmod(grp, w.Hkv)
        if packed:
            base, length = kvh * w.T + cu_l[s], cu_l[s + 1] - cu_l[s]
        else:
            base, length = grp * w.T, w.T
        usable = 128 * (-(-length // 128) - 1) if w.causal else length
        for lvl in range(J):
            n = 1024 << lvl
            if n > usable:
                continue
            tile = warm[(grp * J + lvl) * tile_elems:(grp * J + lvl + 1) * tile_elems]
            tile = tile.reshape(128, w.d)
            rng = kbits[base:base + n]
            # every warm-up row is one of the range's key rows, bit for bit, each at most once
            lookup = {rng[i].tobytes(): i for i in range(n)}
            picked = [lookup.get(tile[r].tobytes(), -1) for r in range(128)]
            assert min(picked) >= 0, f"{name}: group {grp} level {lvl}: a row not in the range"
            assert len(set(picked)) == 128
            # ... and their norms are the 128 largest of the range (fp32 ties: within rounding)
            rn = norms_ref[base:base + n]
            kth = np.sort(rn)[::-1][127]
            assert rn[picked].min() >= kth * (1 - 1e-5), f"{name}: group {grp} level {lvl}"
            checked += 1
    assert checked > 0
