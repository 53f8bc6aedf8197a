"""fp64 CPU oracle of the backward pass of causal alpha-entmax attention -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg use this module;
the CUDA library never does, and this module imports nothing from it.

The pages say the block mask of the forward pass also serves the backward pass ("AdaSplash with
Block Masking", AdaSplash: Adaptive Sparse Flash Attention) but print no gradient formula.  It is
derived here from the Jacobian of alpha-entmax (Peters, Niculae & Martins 2019, "Sparse
Sequence-to-Sequence Models", Proposition 2): for p = entmax_alpha(s),

    dp/ds = diag(w) - w w^T / sum(w),   w_j = p_j^(2 - alpha) = [z_j - tau]_+^(beta - 1)

(w_j = 0 off the support).  With s_ij = q_i . k_j / sqrt(d), o_i = sum_j p_ij v_j and an upstream
gradient g_i = dL/do_i, per query row i:

    u_ij     = g_i . v_j                                   (dL/dp_ij)
    delta_i  = sum_j w_ij u_ij / sum_j w_ij
    ds_ij    = w_ij (u_ij - delta_i)                       (dL/ds_ij)
    dq_i     = sum_j ds_ij k_j / sqrt(d)
    dk_j    += ds_ij q_i / sqrt(d)        (summed over the rows and the query heads of the group)
    dv_j    += p_ij g_i

p comes from the forward oracle's exact tau (``oracle.entmax_vec``).  Everything is fp64; the
inputs are used as given (fp64 arrays stay fp64, so the tests can differentiate numerically).
"""
from __future__ import annotations

import numpy as np

from . import oracle


def _f64(x) -> np.ndarray:
    if hasattr(x, "detach"):  # torch tensor, without importing torch here
        x = x.detach().cpu().double().numpy()
    return np.asarray(x, dtype=np.float64)


def _sequences(T: int, cu_seqlens):
    if cu_seqlens is None:
        return [(0, T)]
    cu = [int(c) for c in np.asarray(cu_seqlens).ravel()]
    return [(cu[s], cu[s + 1] - cu[s]) for s in range(len(cu) - 1)]


def attention_backward(q, k, v, dout, alpha: float, causal: bool = True, cu_seqlens=None):
    """Gradients of L = sum(dout * out) with respect to q, k and v, in fp64.

    Layouts as the forward: q, dout [B, Hq, T, d] and k, v [B, Hkv, T, d], or [Hq, T, d] /
    [Hkv, T, d] with cu_seqlens.  alpha is used as given.  Returns (dq, dk, dv, delta) with
    delta [B, Hq, T] (or [Hq, T]) the per-row sum(w u) / sum(w).
    """
    qf, kf, vf, gf = _f64(q), _f64(k), _f64(v), _f64(dout)
    packed = cu_seqlens is not None
    if packed:
        qf, kf, vf, gf = qf[None], kf[None], vf[None], gf[None]
    B, Hq, T, d = qf.shape
    Hkv = kf.shape[1]
    G = Hq // Hkv
    scale = 1.0 / np.sqrt(d)
    beta = 1.0 / (alpha - 1.0)
    dq = np.zeros_like(qf)
    dk = np.zeros_like(kf)
    dv = np.zeros_like(vf)
    delta = np.zeros(qf.shape[:3])
    seqs = _sequences(T, cu_seqlens)
    for b in range(B):
        for h in range(Hq):
            hk = h // G
            for start, length in seqs:
                K = kf[b, hk, start:start + length]
                V = vf[b, hk, start:start + length]
                for t in range(length):
                    n = t + 1 if causal else length
                    qi, gi = qf[b, h, start + t], gf[b, h, start + t]
                    s = K[:n] @ qi * scale
                    p, tau = oracle.entmax_vec((alpha - 1.0) * s, alpha)
                    x = (alpha - 1.0) * s - tau
                    w = np.zeros_like(p)
                    w[p > 0.0] = x[p > 0.0] ** (beta - 1.0)
                    u = V[:n] @ gi
                    dl = float(w @ u) / float(w.sum())
                    ds = w * (u - dl)
                    delta[b, h, start + t] = dl
                    dq[b, h, start + t] = (ds @ K[:n]) * scale
                    dk[b, hk, start:start + n] += np.outer(ds, qi) * scale
                    dv[b, hk, start:start + n] += np.outer(p, gi)
    if packed:
        return dq[0], dk[0], dv[0], delta[0]
    return dq, dk, dv, delta


def row_gradients(q, k, v, dout, alpha: float, causal: bool = True, cu_seqlens=None, rows=()):
    """dq and delta of the given query rows only, in fp64: the same formulas as
    ``attention_backward`` (each row's dq and delta depend on that row alone), for checking
    sampled rows of problems too large for the full oracle.  rows are flat indices into
    q.reshape(-1, d) (fixed length: (b * Hq + h) * T + t; packed: h * T + token).  Returns
    (dq [len(rows), d], delta [len(rows)])."""
    qf, kf, vf, gf = _f64(q), _f64(k), _f64(v), _f64(dout)
    packed = cu_seqlens is not None
    if packed:
        qf, kf, vf, gf = qf[None], kf[None], vf[None], gf[None]
    B, Hq, T, d = qf.shape
    G = Hq // kf.shape[1]
    scale = 1.0 / np.sqrt(d)
    beta = 1.0 / (alpha - 1.0)
    seqs = _sequences(T, cu_seqlens)
    starts = np.array([st for st, _ in seqs])
    rows = np.asarray(rows, dtype=np.int64)
    dq = np.zeros((rows.size, d))
    delta = np.zeros(rows.size)
    for n_, row in enumerate(rows):
        tok = int(row % T)
        h = int((row // T) % Hq)
        b = int(row // (T * Hq))
        sidx = int(np.searchsorted(starts, tok, side="right") - 1)
        start, length = seqs[sidx]
        t = tok - start
        n = t + 1 if causal else length
        K = kf[b, h // G, start:start + n]
        V = vf[b, h // G, start:start + n]
        qi, gi = qf[b, h, tok], gf[b, h, tok]
        s = K @ qi * scale
        p, tau = oracle.entmax_vec((alpha - 1.0) * s, alpha)
        x = (alpha - 1.0) * s - tau
        w = np.zeros_like(p)
        w[p > 0.0] = x[p > 0.0] ** (beta - 1.0)
        u = V @ gi
        dl = float(w @ u) / float(w.sum())
        delta[n_] = dl
        dq[n_] = (w * (u - dl)) @ K * scale
    return dq, delta


def attention_forward_fp64(q, k, v, alpha: float, causal: bool = True, cu_seqlens=None):
    """The forward output in fp64 from fp64 inputs (exact tau per row), for numerical
    differentiation in the tests: the same definition as ``oracle.attention_rows`` without its
    fp32 input conversion."""
    qf, kf, vf = _f64(q), _f64(k), _f64(v)
    packed = cu_seqlens is not None
    if packed:
        qf, kf, vf = qf[None], kf[None], vf[None]
    B, Hq, T, d = qf.shape
    G = Hq // kf.shape[1]
    scale = 1.0 / np.sqrt(d)
    out = np.zeros_like(qf)
    for b in range(B):
        for h in range(Hq):
            for start, length in _sequences(T, cu_seqlens):
                K = kf[b, h // G, start:start + length]
                V = vf[b, h // G, start:start + length]
                for t in range(length):
                    n = t + 1 if causal else length
                    p, _ = oracle.entmax_vec((alpha - 1.0) * (K[:n] @ qf[b, h, start + t]) * scale,
                                             alpha)
                    out[b, h, start + t] = p @ V[:n]
    return out[0] if packed else out
