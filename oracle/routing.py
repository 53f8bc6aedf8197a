"""fp64 CPU oracle of entmax block routing over chunk summaries -- TEST INFRASTRUCTURE.

Only ``tests/`` uses this module; the CUDA library never does, and this module imports nothing
from it.

What it computes (MiniCPM-4-8B-NSA page, DashAttention, "How it works", stage 2 "Entmax block
routing", with the "Core API" arguments chunk_size, enable_gqa, estimate_diagonal and
scaling_factor).  Keys are cut into chunks of C tokens; each kv head has one summary vector per
chunk, sigma[b, hk, c] (the page builds it from learned weights, which are not available, so the
summaries here are inputs).  Each query row scores the summaries it may see and routes by
alpha-entmax over those scores:

    s_ic  = scaling_factor * q_i . sigma_{kv(h), c} / sqrt(d)      kv(h) = floor(h / (Hq / Hkv))
    pi_i  = entmax_alpha(s_i) over the visible chunks               (routing priors, sum to 1)
    support_i = { c : pi_ic > 0 }                                   (sparse chunk support)

Visible chunks of row i: causal -- every chunk before the row's own chunk floor(i / C), and the
own (diagonal) chunk too when estimate_diagonal is set, its summary standing in for the keys of
that chunk the row cannot see yet; not causal -- every chunk.  The pages do not say how the
router treats the diagonal chunk without estimate_diagonal; the plainest reading is that it then
takes no part in routing, so the rows of the first chunk route nowhere (pi = 0, tau = +inf).
The pages give no alpha for the router; it is an argument.  alpha-entmax itself is the oracle's
exact one (``oracle.entmax_vec``; Peters, Niculae & Martins 2019).
"""
from __future__ import annotations

import math

import numpy as np

from . import oracle


def _f64(x) -> np.ndarray:
    if hasattr(x, "detach"):  # torch tensor, without importing torch here
        x = x.detach().cpu().double().numpy()
    return np.asarray(x, dtype=np.float64)


def visible_chunks(i: int, chunk_size: int, n_chunks: int, causal: bool,
                   estimate_diagonal: bool) -> int:
    """Number of chunks row i routes over (always the chunks 0 .. n - 1)."""
    if not causal:
        return n_chunks
    own = i // chunk_size
    return min(n_chunks, own + 1 if estimate_diagonal else own)


def route_chunks(q, summaries, alpha: float, chunk_size: int = 64, causal: bool = True,
                 estimate_diagonal: bool = True, scaling_factor: float = 1.0):
    """Routing priors of every query row.

    q: [B, Hq, T, d]; summaries: [B, Hkv, Nc, d] with Nc = ceil(T / chunk_size).  alpha is used
    as given.  Returns (pi [B, Hq, T, Nc] fp64, zero outside the visible chunks; tau [B, Hq, T]
    in the units of z = (alpha - 1) s, +inf for a row with no visible chunk).
    """
    qf, sf = _f64(q), _f64(summaries)
    B, Hq, T, d = qf.shape
    Hkv, Nc = sf.shape[1], sf.shape[2]
    if Nc != -(-T // chunk_size):
        raise ValueError("one summary per chunk of chunk_size tokens is required")
    G = Hq // Hkv
    scale = scaling_factor / math.sqrt(d)
    pi = np.zeros((B, Hq, T, Nc))
    tau = np.full((B, Hq, T), np.inf)
    for b in range(B):
        for h in range(Hq):
            S = sf[b, h // G]
            for i in range(T):
                n = visible_chunks(i, chunk_size, Nc, causal, estimate_diagonal)
                if n == 0:
                    continue
                s = S[:n] @ qf[b, h, i] * scale
                p, t = oracle.entmax_vec((alpha - 1.0) * s, alpha)
                pi[b, h, i, :n] = p
                tau[b, h, i] = t
    return pi, tau
