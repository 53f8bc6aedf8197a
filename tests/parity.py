"""Parity harness: the CUDA library (through its C ABI) against the fp64 oracle on the same
seeded inputs.

Tolerances (the acceptance bar of the forward pass):
  out   max-abs error <= 1e-4 for fp32 inputs, <= 2e-2 for bf16 inputs (fp32 accumulate); a bf16
        output is stored in bf16, which adds up to half a unit in its last place, 2^-9 |o|, to
        the error of the accumulated value: its bar is 2e-2 + 2^-9 |o_ref| per element
  tau   |tau_gpu - tau_ref| <= 1e-4 * max(1, |tau_ref|)
  mask  bit-exact per (query tile, key tile), except tiles whose largest p is below 1e-6 both at
        the exact tau and at the GPU's tau (p evaluated in fp64 on the host by the oracle).
Rows are compared one by one; the block mask is compared two-sided on whole query tiles and
one-sided (every tile holding a p > 1e-6 of a checked row must be set) on loose rows.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np
import torch

import adaptive_sparse_attention_b200 as ea
from adaptive_sparse_attention_b200.workloads import Workload
from oracle import oracle

TILE = 128
OUT_TOL = {"fp32": 1e-4, "bf16": 2e-2}


def out_tolerance(w: Workload) -> float:
    """Max-abs bar for o.  For alpha > 2 (beta < 1) the map x -> x^beta has unbounded slope at
    0, so a rounding error delta of an fp32 score moves p by up to delta^beta near a support
    edge; with delta <= 2^-20 (a few ulps of |z| <= 8) the fp32 bar becomes
    1e-4 + 2^(-20 beta).  bf16 inputs keep 2e-2."""
    tol = OUT_TOL[w.dtype]
    beta = 1.0 / (oracle.alpha_as_float32(w.alpha) - 1.0)
    if w.dtype == "fp32" and beta < 1.0:
        tol += 2.0 ** (-20.0 * beta)
    return tol
def out_bar(w: Workload, ref_out: np.ndarray) -> np.ndarray:
    """Per-element bar on |o_gpu - o_ref|: out_tolerance, plus for bf16 the rounding of the
    stored output (round to nearest with 8 significant bits: at most 2^-9 |o|)."""
    bar = np.full(ref_out.shape, out_tolerance(w))
    if w.dtype == "bf16":
        bar += 2.0 ** -9 * np.abs(ref_out)
    return bar


TAU_RTOL = 1e-4
MASK_EXEMPT_P = 1e-6


@dataclass
class GpuResult:
    out: np.ndarray    # [rows, d] fp32 copy
    tau: np.ndarray    # [rows]
    bits: np.ndarray   # decoded mask [nb, Hq, slots, nkt]
    fallback_tiles: int


# The forward pass's paths through the C ABI's two passes:
#   "fused": with ENTMAX_ATTN_FLAG_SUPPORT: the tau pass records each row's support, the output
#            pass computes o from the supports (tile pass for the query tiles without one) --
#            the path entmax_attn_fwd takes and bench.py times;
#   "tile":  without it: the output pass over every query tile's active key tiles.
PATHS = ("fused", "tile")


def run_gpu(w: Workload, inputs, flags: int = 0, use_fwd: bool = False,
            path: str = "fused") -> GpuResult:
    q, k, v, cu = inputs
    dev = torch.device("cuda:0")
    q, k, v = q.to(dev), k.to(dev), v.to(dev)
    cu_d = cu.to(dev) if cu is not None else None
    alpha = oracle.alpha_as_float32(w.alpha)
    if use_fwd:
        out, tau, mask = ea.entmax_attn_fwd(q, k, v, alpha, w.n_iter, w.causal, cu_d)
        nfb = -1
    else:
        run = ea.entmax_attn_fused if path == "fused" else ea.entmax_attn_two_pass
        out, tau, mask, ws = run(q, k, v, alpha, w.n_iter, w.causal, cu_d, flags=flags)
        nfb = ea.fallback_tiles(ws)
    torch.cuda.synchronize()
    st = ea.status()
    assert st == 0, f"device status {st}"
    bits = ea.decode_block_mask(mask.cpu().numpy(), w.B, w.Hq, w.T, cu)
    return GpuResult(out.float().cpu().numpy().reshape(-1, w.d), tau.cpu().numpy().ravel(),
                     bits, nfb)


def seq_table(w: Workload, cu):
    """[(first slot, n query tiles, first token, length)] per sequence (fixed length: per batch
    row, which all share slot numbering)."""
    return ea.tile_slot_table(w.B, w.T, None if cu is None else cu.tolist())


def tile_rows(w: Workload, cu, b: int, h: int, s: int, qt: int) -> np.ndarray:
    """Flat row ids of query tile qt of sequence s (fixed length: batch row b) of head h."""
    slot0, nqt, start, length = seq_table(w, cu)[s if cu is not None else b]
    pos = np.arange(qt * TILE, min((qt + 1) * TILE, length))
    if cu is None:
        return (b * w.Hq + h) * w.T + pos
    return h * w.T + start + pos


def row_coords(w: Workload, cu, rows: np.ndarray):
    """(b, h, sequence, position) of flat row ids."""
    if cu is None:
        t = rows % w.T
        h = (rows // w.T) % w.Hq
        b = rows // (w.T * w.Hq)
        return b, h, b, t
    h = rows // w.T
    g = rows % w.T
    cuv = cu.numpy()
    s = np.searchsorted(cuv, g, side="right") - 1
    return np.zeros_like(rows), h, s, g - cuv[s]


def all_tiles(w: Workload, cu):
    tiles = []
    nb = 1 if cu is not None else w.B
    for b in range(nb):
        for h in range(w.Hq):
            for s, (slot0, nqt, start, length) in enumerate(seq_table(w, cu)):
                if cu is None and s != b:
                    continue
                for qt in range(nqt):
                    tiles.append((b, h, s, qt))
    return tiles


def compare(w: Workload, inputs, g: GpuResult, whole_tiles, loose_rows=None, label="",
            flat_bar: bool = False):
    """Asserts parity on the given whole query tiles and loose rows.  Returns a summary dict.
    flat_bar: o was stored in fp32 (ENTMAX_ATTN_FLAG_OUT_FP32), so its bar is the flat
    out_tolerance, without the bf16 rounding of a stored bf16 output."""
    q, k, v, cu = inputs
    alpha = oracle.alpha_as_float32(w.alpha)
    groups = [tile_rows(w, cu, *t) for t in whole_tiles]
    rows = np.concatenate(groups + ([np.asarray(loose_rows, dtype=np.int64)]
                                    if loose_rows is not None and len(loose_rows) else []))
    ref = oracle.attention_rows(q, k, v, alpha, w.causal, cu, rows)
    err_out = np.abs(g.out[rows] - ref["out"])
    bar = (np.full(ref["out"].shape, out_tolerance(w)) if flat_bar else out_bar(w, ref["out"]))
    max_out = float(err_out.max()) if err_out.size else 0.0
    over = float((err_out / bar).max()) if err_out.size else 0.0
    tau_g = g.tau[rows].astype(np.float64)
    err_tau = np.abs(tau_g - ref["tau"]) / np.maximum(1.0, np.abs(ref["tau"]))
    max_tau = float(err_tau.max()) if err_tau.size else 0.0
    worst = int(np.argmax((err_out / bar).max(axis=1))) if err_out.size else 0
    assert over <= 1.0, (f"{label}: out error {err_out[worst].max():.3e} above its bar "
                         f"{bar[worst][np.argmax(err_out[worst] / bar[worst])]:.3e} at row "
                         f"{rows[worst]}")
    assert max_tau <= TAU_RTOL, (f"{label}: tau rel err {max_tau:.3e} at row "
                                 f"{rows[int(np.argmax(err_tau))]}")

    nkt = ref["nkt"]
    table = seq_table(w, cu)
    mismatched = exempt = 0
    off = 0
    for t, grp in zip(whole_tiles, groups):
        b, h, s, qt = t
        n = grp.size
        mp_ref = ref["maxp"][off:off + n].max(axis=0)
        slot = table[s if cu is not None else b][0] + qt
        bits = g.bits[b, h, slot, :nkt]
        bad = np.nonzero(bits != (mp_ref > 0))[0]
        if bad.size:
            # p at the GPU's tau (fp64, host), for the exemption rule
            at_gpu = oracle.attention_rows(q, k, v, alpha, w.causal, cu, grp,
                                           tau_given=tau_g[off:off + n], want_out=False)
            mp_gpu = at_gpu["maxp"].max(axis=0)
        for kt in bad:
            mismatched += 1
            if mp_ref[kt] < MASK_EXEMPT_P and mp_gpu[kt] < MASK_EXEMPT_P:
                exempt += 1
            else:
                raise AssertionError(
                    f"{label}: mask bit (b={b}, h={h}, seq={s}, qt={qt}, kt={kt}) gpu={bits[kt]} "
                    f"oracle max p={mp_ref[kt]:.3e}, p at gpu tau={mp_gpu[kt]:.3e}")
        off += n
    # loose rows: one-sided
    if loose_rows is not None and len(loose_rows):
        lr = np.asarray(loose_rows, dtype=np.int64)
        b, h, s, pos = row_coords(w, cu, lr)
        mp = ref["maxp"][off:]
        for i in range(lr.size):
            need = np.nonzero(mp[i] > MASK_EXEMPT_P)[0]
            slot = table[int(s[i]) if cu is not None else int(b[i])][0] + int(pos[i]) // TILE
            got = g.bits[int(b[i]), int(h[i]), slot]
            assert np.all(got[need]), (f"{label}: row {lr[i]} has p > 1e-6 in key tiles "
                                       f"{need[~got[need]]} whose bit is clear")
    return {"rows": int(rows.size), "max_out_err": max_out, "max_tau_rel_err": max_tau,
            "mask_mismatch_exempt": exempt, "mask_mismatch": mismatched}
