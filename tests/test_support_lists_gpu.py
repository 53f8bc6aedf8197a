"""The support lists the tau pass records (ENTMAX_ATTN_FLAG_SUPPORT), on EVERY row of the large
workloads, by the properties that fix them at any size.

Row i's support is {j : p_ij > 0} with p_ij = [z_ij - tau_i]_+^(1/(alpha-1)), and p_i is a
probability vector (AdaSplash page, "Triton Entmax": tau is the root of sum_j p_ij = 1), so a
correctly recorded list has at least one entry, distinct keys inside the row's causal range,
p > 0 and sum p = 1.  The sampled oracle tiles of the parity tests cover a few thousand rows of
the 16K, packed 32K and 128K workloads; a fault that corrupts the lists of a handful of rows out
of millions (an entry written into the next row's part of its tile's list) slips past them, and
it is what this test catches: such a row loses a key, and with it the key's share of the sum.

Bar: |sum p - 1| <= 1e-3.  Each p is computed in fp32 from the stored raw score and the GPU's
tau (within ~1e-6 relative of the exact root, the oracle pins of the parity tests), a sum of at
most a few thousand terms; the sum at a tau off by d is 1 - beta * sum (z - tau)^(beta - 1) * d,
whose error stays near 1e-5 for these workloads, while a lost key moves the sum by its p, which
for the rows whose lists can be corrupted this way (rows with a key within rounding of tau) is
the share of a key well above tau.  Rows of query tiles left to the tile output pass (pending:
overflowed candidate buffers or lists) have no list and are skipped; the parity tests cover them.

The workspace sections read here follow the library's documented layout (the size identities of
test_abi_host.test_workspace_sizes_nest): the pending flags after the fallback counter, queue
and counts; the support index per query row and the entries per query tile last.
"""
import numpy as np
import pytest
import torch

import adaptive_sparse_attention_b200 as ea
from adaptive_sparse_attention_b200 import _native
from adaptive_sparse_attention_b200.workloads import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu

SUP_PER_TILE = 2048


def _up(x):
    return (x + 255) // 256 * 256


def _sections(ws: torch.Tensor, w, cu):
    packed = cu is not None
    nb = 1 if packed else w.B
    slots = (w.T // 128 + w.B) if packed else -(-w.T // 128)
    tiles = nb * w.Hq * slots
    qrows = nb * w.Hq * w.T
    b = ws.cpu().numpy()
    p0 = 256 + 2 * _up(4 * tiles)
    pending = b[p0:p0 + 4 * tiles].view(np.int32)
    sup_bytes = _up(8 * SUP_PER_TILE * tiles)
    sup = b[b.size - sup_bytes:].view(np.int32).reshape(tiles * SUP_PER_TILE, 2)
    i0 = b.size - sup_bytes - _up(4 * qrows)
    sup_idx = b[i0:i0 + 4 * qrows].view(np.int32)
    return slots, pending, sup_idx, sup


def _row_layout(w, cu, slots):
    """Per flat query row: its tile id, its position in its sequence, and whether it exists."""
    if cu is None:
        rows = np.arange(w.B * w.Hq * w.T, dtype=np.int64)
        t = rows % w.T
        bh = rows // w.T
        return bh * slots + t // 128, t, np.ones(rows.size, bool)
    cuv = cu.numpy().astype(np.int64)
    g = np.arange(w.T, dtype=np.int64)
    s = np.searchsorted(cuv, g, side="right") - 1
    ok = g < cuv[-1]
    s = np.clip(s, 0, cuv.size - 2)
    pos = g - cuv[s]
    slot = cuv[s] // 128 + s + pos // 128
    h = np.arange(w.Hq, dtype=np.int64)[:, None]
    return ((h * slots + slot[None, :]).ravel(), np.tile(pos, w.Hq), np.tile(ok, w.Hq))


@pytest.mark.parametrize("name", ["b2_t16k_gqa4_bf16_d128_a2",
                                  "varlen4_32k_gqa4_bf16_d128_a1.333",
                                  "t128k_gqa4_bf16_d128_a1.5"])
def test_every_recorded_support_sums_to_one(name):
    w = WORKLOADS[name]
    q, k, v, cu = make_inputs(w, 0)
    dev = torch.device("cuda:0")
    qd, kd = q.to(dev), k.to(dev)
    cud = cu.to(dev) if cu is not None else None
    out, tau, mask = ea.alloc_outputs(qd, kd, cud)
    ws = ea.alloc_workspace(qd, kd, cud)
    alpha = float(np.float32(w.alpha))
    ea.tau_pass(qd, kd, tau, mask, ws, alpha, w.n_iter, w.causal, cud, flags=_native.FLAG_SUPPORT)
    torch.cuda.synchronize()
    assert ea.status() == 0
    slots, pending, sup_idx, sup = _sections(ws, w, cu)
    tile, pos, exists = _row_layout(w, cu, slots)
    rec = exists & (pending[tile] == 0)
    rows = np.nonzero(rec)[0]
    # not vacuous: most query tiles keep their lists (the packed alpha = 1.333 workload leaves
    # about a sixth of them to the overflow path)
    assert rows.size > 0.75 * exists.sum(), "most query tiles keep their lists"
    first = (sup_idx[rows] & 0xffff).astype(np.int64)
    n = (sup_idx[rows] >> 16).astype(np.int64)
    assert n.min() >= 1 and np.all(first + n <= SUP_PER_TILE), name
    # every entry of every recorded row
    start = tile[rows] * SUP_PER_TILE + first
    owner = np.repeat(np.arange(rows.size), n)
    at = np.repeat(start - np.cumsum(n) + n, n) + np.arange(n.sum())
    key = sup[at, 0].astype(np.int64)
    p = sup[at, 1].view(np.float32).astype(np.float64)
    hi = pos[rows][owner] if w.causal else np.full(owner.size, w.T)
    assert np.all((key >= 0) & (key <= hi)), f"{name}: a key outside its row's range"
    assert np.all(p > 0) and np.all(np.isfinite(p)), f"{name}: an entry without positive p"
    # distinct keys per row: sorted by (row, key), no equal neighbours
    order = np.lexsort((key, owner))
    same = (owner[order][1:] == owner[order][:-1]) & (key[order][1:] == key[order][:-1])
    assert not same.any(), f"{name}: a key listed twice in one row"
    psum = np.bincount(owner, weights=p, minlength=rows.size)
    bad = np.abs(psum - 1.0) > 1e-3
    assert not bad.any(), (f"{name}: {int(bad.sum())} of {rows.size} rows with sum p off 1, "
                           f"first rows {rows[bad][:5].tolist()} sums {psum[bad][:5].tolist()}")
    print(name, "recorded rows", rows.size, "entries", int(n.sum()),
          "max |sum p - 1|", float(np.abs(psum - 1).max()))
