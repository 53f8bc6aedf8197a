"""Torch-facing binding of the entmax attention C ABI: argument marshalling only.

Every step of the computation runs in the CUDA kernels of libentmax_attn.so; this module checks
tensor shapes and dtypes, allocates outputs with torch (device memory only) and passes raw
pointers and the current CUDA stream through ctypes.

Layouts (AdaSplash: Adaptive Sparse Flash Attention, "AdaSplash with Block Masking" and
"Variable Length Sequences"): fixed length q [B, Hq, T, d], k, v [B, Hkv, T, d]; packed varlen
q [Hq, T_total, d], k, v [Hkv, T_total, d] with int32 cu_seqlens [B + 1] on the device.
"""
from __future__ import annotations

import ctypes

import numpy as np
import torch

from . import _native as N

TILE = 128
_DT = {torch.float32: N.FP32, torch.bfloat16: N.BF16}


def _ptr(t) -> int | None:
    return None if t is None else t.data_ptr()


def _stream(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def problem_dims(q, k, cu_seqlens):
    """(B, Hq, Hkv, T, d) of a fixed-length or packed problem."""
    if cu_seqlens is None:
        if q.dim() != 4 or k.dim() != 4:
            raise ValueError("fixed-length q, k must be [B, H, T, d]")
        B, Hq, T, d = q.shape
        if k.shape[0] != B or k.shape[2] != T or k.shape[3] != d:
            raise ValueError("k does not match q")
        return B, Hq, k.shape[1], T, d
    if q.dim() != 3 or k.dim() != 3:
        raise ValueError("packed q, k must be [H, T_total, d]")
    Hq, T, d = q.shape
    if k.shape[1] != T or k.shape[2] != d:
        raise ValueError("k does not match q")
    return cu_seqlens.numel() - 1, Hq, k.shape[0], T, d


def _check_inputs(q, k, v, cu_seqlens):
    for name, t in (("q", q), ("k", k), ("v", v)):
        if t is None:
            continue
        if not t.is_cuda:
            raise ValueError(f"{name} must be a CUDA tensor")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
        if t.dtype not in _DT:
            raise ValueError(f"{name} must be float32 or bfloat16")
    if k.dtype != q.dtype or (v is not None and v.dtype != q.dtype):
        raise ValueError("q, k, v must share one dtype")
    if v is not None and v.shape != k.shape:
        raise ValueError("v must have the shape of k")
    if cu_seqlens is not None:
        if not cu_seqlens.is_cuda or cu_seqlens.dtype != torch.int32 or cu_seqlens.dim() != 1:
            raise ValueError("cu_seqlens must be a 1-D int32 CUDA tensor")


def mask_layout(B, Hq, T, packed: bool):
    """(query tiles per head, words per query tile) of the block-mask layout."""
    a, b = ctypes.c_int(), ctypes.c_int()
    N.check(N.lib().entmax_attn_mask_layout(B, Hq, T, int(packed), ctypes.byref(a),
                                            ctypes.byref(b)), "entmax_attn_mask_layout")
    return a.value, b.value


def mask_words(B, Hq, T, packed: bool) -> int:
    return int(N.lib().entmax_attn_mask_words(B, Hq, T, int(packed)))


def workspace_bytes(B, Hq, T, packed: bool) -> int:
    return int(N.lib().entmax_attn_workspace_bytes(B, Hq, T, int(packed)))


def workspace_min_bytes(B, Hq, T, packed: bool) -> int:
    """The smallest workspace the passes accept (the tau pass then runs without warm-up keys)."""
    return int(N.lib().entmax_attn_workspace_min_bytes(B, Hq, T, int(packed)))


def alloc_outputs(q, k, cu_seqlens):
    B, Hq, Hkv, T, d = problem_dims(q, k, cu_seqlens)
    packed = cu_seqlens is not None
    out = torch.empty_like(q)
    tau = torch.empty(q.shape[:-1], dtype=torch.float32, device=q.device)
    mask = torch.empty(mask_words(B, Hq, T, packed), dtype=torch.int32, device=q.device)
    return out, tau, mask


def entmax_attn_fwd(q, k, v, alpha: float = 1.5, n_iter: int = 10, causal: bool = True,
                    cu_seqlens=None, out=None, tau=None, block_mask=None, stream=None):
    """Forward pass.  Returns (out, tau, block_mask); block_mask holds the uint32 words of the
    documented layout in an int32 tensor."""
    _check_inputs(q, k, v, cu_seqlens)
    B, Hq, Hkv, T, d = problem_dims(q, k, cu_seqlens)
    o2, t2, m2 = alloc_outputs(q, k, cu_seqlens) if None in (out, tau, block_mask) else (None,) * 3
    out = o2 if out is None else out
    tau = t2 if tau is None else tau
    block_mask = m2 if block_mask is None else block_mask
    rc = N.lib().entmax_attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(tau),
                                 _ptr(block_mask), B, Hq, Hkv, T, d, float(alpha), int(n_iter),
                                 int(bool(causal)), _ptr(cu_seqlens), _DT[q.dtype],
                                 _stream(stream))
    N.check(rc, "entmax_attn_fwd")
    return out, tau, block_mask


def entmax_attn_fwd_no_block_mask(q, k, v, alpha: float = 1.5, n_iter: int = 10,
                                  causal: bool = True, cu_seqlens=None, out=None, tau=None,
                                  stream=None):
    """Forward pass without the block mask (the output pass visits every causally valid key
    tile).  Returns (out, tau)."""
    _check_inputs(q, k, v, cu_seqlens)
    B, Hq, Hkv, T, d = problem_dims(q, k, cu_seqlens)
    o2, t2, _ = alloc_outputs(q, k, cu_seqlens) if None in (out, tau) else (None,) * 3
    out = o2 if out is None else out
    tau = t2 if tau is None else tau
    rc = N.lib().entmax_attn_fwd_no_block_mask(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(tau),
                                               B, Hq, Hkv, T, d, float(alpha), int(n_iter),
                                               int(bool(causal)), _ptr(cu_seqlens), _DT[q.dtype],
                                               _stream(stream))
    N.check(rc, "entmax_attn_fwd_no_block_mask")
    return out, tau


def entmax_rows(x, alpha: float = 1.5, n_iter: int = 10, out=None, tau=None, stream=None):
    """Row-wise alpha-entmax over the last dimension of x (fp32 or bf16, contiguous rows).
    Returns (p, tau): p like x, tau fp32 with x's leading shape."""
    if x.dtype not in _DT:
        raise TypeError("x must be float32 or bfloat16")
    if x.dim() < 1 or x.numel() == 0 or x.stride(-1) != 1:
        raise ValueError("x needs a non-empty, unit-stride last dimension")
    n = x.shape[-1]
    x2 = x.reshape(-1, n)  # a view when the rows have one stride, else a contiguous copy
    rows = x2.shape[0]
    p = (torch.empty((rows, n), dtype=x.dtype, device=x.device) if out is None
         else out.view(rows, n))
    if p.stride(1) != 1 or p.dtype != x.dtype:
        raise ValueError("out must have x's dtype and unit-stride rows")
    t = torch.empty(rows, dtype=torch.float32, device=x.device) if tau is None else tau.view(rows)
    rc = N.lib().entmax_attn_rows(_ptr(x2), x2.stride(0), _ptr(p), p.stride(0), _ptr(t), rows, n,
                                  float(alpha), int(n_iter), _DT[x.dtype], _stream(stream))
    N.check(rc, "entmax_attn_rows")
    return p.reshape(x.shape), t.reshape(x.shape[:-1])


def route_chunks(q, summaries, alpha: float = 1.5, chunk_size: int = 64, n_iter: int = 10,
                 causal: bool = True, estimate_diagonal: bool = True, scaling_factor: float = 1.0,
                 stream=None):
    """Entmax block routing of every query row over the chunk summaries it may see.
    q [B, Hq, T, d] and summaries [B, Hkv, ceil(T / chunk_size), d], same dtype, contiguous.
    Returns (pi fp32 [B, Hq, T, n_chunks], tau fp32 [B, Hq, T])."""
    if q.dtype not in _DT or summaries.dtype != q.dtype:
        raise TypeError("q and summaries must both be float32 or both bfloat16")
    if q.dim() != 4 or summaries.dim() != 4 or not q.is_contiguous() or \
            not summaries.is_contiguous():
        raise ValueError("q [B, Hq, T, d] and summaries [B, Hkv, n_chunks, d], contiguous")
    B, Hq, T, d = q.shape
    Hkv, nc = summaries.shape[1], summaries.shape[2]
    if summaries.shape[0] != B or summaries.shape[3] != d or nc != -(-T // chunk_size):
        raise ValueError("summaries must be [B, Hkv, ceil(T / chunk_size), d]")
    pi = torch.empty((B, Hq, T, nc), dtype=torch.float32, device=q.device)
    tau = torch.empty((B, Hq, T), dtype=torch.float32, device=q.device)
    rc = N.lib().entmax_attn_route_chunks(_ptr(q), _ptr(summaries), _ptr(pi), _ptr(tau), B, Hq,
                                          Hkv, T, d, int(chunk_size), float(alpha), int(n_iter),
                                          int(bool(causal)), int(bool(estimate_diagonal)),
                                          float(scaling_factor), _DT[q.dtype], _stream(stream))
    N.check(rc, "entmax_attn_route_chunks")
    return pi, tau


def entmax_attn_fwd_noalloc(q, k, v, alpha: float = 1.5, n_iter: int = 10, causal: bool = True,
                            cu_seqlens=None, out=None, tau=None, block_mask=None, stream=None):
    """Forward pass through the allocation-free entry point: the library's scratch is a fixed
    device array (ENTMAX_ATTN_NOALLOC_SCRATCH_BYTES), so the call allocates no device memory.
    The outputs are allocated here by torch only when not passed in."""
    _check_inputs(q, k, v, cu_seqlens)
    B, Hq, Hkv, T, d = problem_dims(q, k, cu_seqlens)
    o2, t2, m2 = alloc_outputs(q, k, cu_seqlens) if None in (out, tau, block_mask) else (None,) * 3
    out = o2 if out is None else out
    tau = t2 if tau is None else tau
    block_mask = m2 if block_mask is None else block_mask
    rc = N.lib().entmax_attn_fwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(tau),
                                         _ptr(block_mask), B, Hq, Hkv, T, d, float(alpha),
                                         int(n_iter), int(bool(causal)), _ptr(cu_seqlens),
                                         _DT[q.dtype], _stream(stream))
    N.check(rc, "entmax_attn_fwd_noalloc")
    return out, tau, block_mask


def entmax_attn_fwd_host(q, k, v, alpha: float = 1.5, n_iter: int = 10, causal: bool = True,
                         cu_seqlens=None, out=None, tau=None, block_mask=None, stream=None,
                         synchronize: bool = True):
    """Forward pass on CPU tensors (pin them for asynchronous, full-speed copies): the library
    streams the problem through the GPU in chunks, the copies in and out overlapping the
    computation.  cu_seqlens is an int32 CPU tensor.  Outputs are CPU tensors (allocated
    pinned here unless passed in); with synchronize=False they are complete only once `stream`
    has finished.  Returns (out, tau, block_mask)."""
    for name, t in (("q", q), ("k", k), ("v", v)):
        if t.is_cuda or not t.is_contiguous() or t.dtype not in _DT:
            raise ValueError(f"{name} must be a contiguous float32 or bfloat16 CPU tensor")
    if k.dtype != q.dtype or v.dtype != q.dtype or v.shape != k.shape:
        raise ValueError("q, k, v must share one dtype; v must have the shape of k")
    if cu_seqlens is not None and (cu_seqlens.is_cuda or cu_seqlens.dtype != torch.int32 or
                                   not cu_seqlens.is_contiguous()):
        raise ValueError("cu_seqlens must be a contiguous int32 CPU tensor")
    B, Hq, Hkv, T, d = problem_dims(q, k, cu_seqlens)
    pin = torch.cuda.is_available()
    if out is None:
        out = torch.empty(q.shape, dtype=q.dtype, pin_memory=pin)
    if tau is None:
        tau = torch.empty(q.shape[:-1], dtype=torch.float32, pin_memory=pin)
    if block_mask is None:
        block_mask = torch.empty(mask_words(B, Hq, T, cu_seqlens is not None), dtype=torch.int32,
                                 pin_memory=pin)
    rc = N.lib().entmax_attn_fwd_host(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(tau),
                                      _ptr(block_mask), B, Hq, Hkv, T, d, float(alpha),
                                      int(n_iter), int(bool(causal)), _ptr(cu_seqlens),
                                      _DT[q.dtype], _stream(stream))
    N.check(rc, "entmax_attn_fwd_host")
    if synchronize:
        (torch.cuda.current_stream() if stream is None else stream).synchronize()
    return out, tau, block_mask


def tau_pass(q, k, tau, block_mask, workspace, alpha=1.5, n_iter=10, causal=True,
             cu_seqlens=None, flags=0, stream=None):
    _check_inputs(q, k, None, cu_seqlens)
    B, Hq, Hkv, T, d = problem_dims(q, k, cu_seqlens)
    rc = N.lib().entmax_attn_tau_pass(_ptr(q), _ptr(k), _ptr(tau), _ptr(block_mask),
                                      _ptr(workspace), workspace.numel() * workspace.element_size(),
                                      B, Hq, Hkv, T, d, float(alpha), int(n_iter),
                                      int(bool(causal)), _ptr(cu_seqlens), _DT[q.dtype],
                                      int(flags), _stream(stream))
    N.check(rc, "entmax_attn_tau_pass")


def screen_bytes(B, Hq, Hkv, T, packed: bool) -> int:
    return int(N.lib().entmax_attn_screen_bytes(B, Hq, Hkv, T, int(packed)))


def alloc_screen(q, k, cu_seqlens):
    B, Hq, Hkv, T, d = problem_dims(q, k, cu_seqlens)
    n = screen_bytes(B, Hq, Hkv, T, cu_seqlens is not None)
    return torch.empty(n, dtype=torch.uint8, device=q.device)


def tau_pass_screened(q, k, tau, block_mask, workspace, screen, alpha=1.5, n_iter=10,
                      causal=True, cu_seqlens=None, flags=0, stream=None):
    """The tau pass with the FP8 screen of its key tiles (bf16, d = 128); same outputs as
    tau_pass.  screen: a uint8 device buffer of screen_bytes(...) bytes."""
    _check_inputs(q, k, None, cu_seqlens)
    B, Hq, Hkv, T, d = problem_dims(q, k, cu_seqlens)
    rc = N.lib().entmax_attn_tau_pass_screened(
        _ptr(q), _ptr(k), _ptr(tau), _ptr(block_mask), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _ptr(screen),
        screen.numel() * screen.element_size(), B, Hq, Hkv, T, d, float(alpha), int(n_iter),
        int(bool(causal)), _ptr(cu_seqlens), _DT[q.dtype], int(flags), _stream(stream))
    N.check(rc, "entmax_attn_tau_pass_screened")


def entmax_attn_screened(q, k, v, alpha=1.5, n_iter=10, causal=True, cu_seqlens=None, flags=0,
                         workspace=None, screen=None, stream=None):
    """The forward pass with the FP8-screened tau pass (and the same flags for the output pass).
    Returns (out, tau, block_mask, workspace, screen)."""
    out, tau, mask = alloc_outputs(q, k, cu_seqlens)
    ws = alloc_workspace(q, k, cu_seqlens) if workspace is None else workspace
    scr = alloc_screen(q, k, cu_seqlens) if screen is None else screen
    tau_pass_screened(q, k, tau, mask, ws, scr, alpha, n_iter, causal, cu_seqlens, flags, stream)
    out_pass(q, k, v, tau, ws, out, alpha, causal, cu_seqlens, flags, stream)
    return out, tau, mask, ws, scr


def out_pass(q, k, v, tau, workspace, out, alpha=1.5, causal=True, cu_seqlens=None, flags=0,
             stream=None):
    _check_inputs(q, k, v, cu_seqlens)
    B, Hq, Hkv, T, d = problem_dims(q, k, cu_seqlens)
    rc = N.lib().entmax_attn_out_pass(_ptr(q), _ptr(k), _ptr(v), _ptr(tau), _ptr(workspace),
                                      workspace.numel() * workspace.element_size(), _ptr(out),
                                      B, Hq, Hkv, T, d, float(alpha), int(bool(causal)),
                                      _ptr(cu_seqlens), _DT[q.dtype], int(flags),
                                      _stream(stream))
    N.check(rc, "entmax_attn_out_pass")


def entmax_attn_bwd(q, k, v, dout, tau, workspace, alpha=1.5, causal=True, cu_seqlens=None,
                    flags=0, stream=None):
    """Backward pass (gradients of sum(dout * out)) for the forward whose tau and workspace are
    given.  Returns fp32 (dq, dk, dv, delta), dq / dk / dv in the layouts of q / k / v."""
    _check_inputs(q, k, v, cu_seqlens)
    if dout.shape != q.shape or dout.dtype != q.dtype or not dout.is_contiguous():
        raise ValueError("dout must be a contiguous tensor with q's shape and dtype")
    B, Hq, Hkv, T, d = problem_dims(q, k, cu_seqlens)
    dq = torch.empty(q.shape, dtype=torch.float32, device=q.device)
    dk = torch.empty(k.shape, dtype=torch.float32, device=q.device)
    dv = torch.empty(v.shape, dtype=torch.float32, device=q.device)
    delta = torch.empty(q.shape[:-1], dtype=torch.float32, device=q.device)
    rc = N.lib().entmax_attn_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(dout), _ptr(tau),
                                 _ptr(workspace), workspace.numel() * workspace.element_size(),
                                 _ptr(delta), _ptr(dq), _ptr(dk), _ptr(dv), B, Hq, Hkv, T, d,
                                 float(alpha), int(bool(causal)), _ptr(cu_seqlens), _DT[q.dtype],
                                 int(flags), _stream(stream))
    N.check(rc, "entmax_attn_bwd")
    return dq, dk, dv, delta


def alloc_workspace(q, k, cu_seqlens):
    B, Hq, Hkv, T, d = problem_dims(q, k, cu_seqlens)
    n = workspace_bytes(B, Hq, T, cu_seqlens is not None)
    return torch.empty(n, dtype=torch.uint8, device=q.device)


def entmax_attn_two_pass(q, k, v, alpha=1.5, n_iter=10, causal=True, cu_seqlens=None, flags=0,
                         workspace=None, stream=None):
    """Both passes through the two-pass entry points with a torch-allocated workspace.
    Returns (out, tau, block_mask, workspace)."""
    out, tau, mask = alloc_outputs(q, k, cu_seqlens)
    if flags & N.FLAG_OUT_FP32:
        out = torch.empty(q.shape, dtype=torch.float32, device=q.device)
    ws = alloc_workspace(q, k, cu_seqlens) if workspace is None else workspace
    tau_pass(q, k, tau, mask, ws, alpha, n_iter, causal, cu_seqlens, flags, stream)
    out_pass(q, k, v, tau, ws, out, alpha, causal, cu_seqlens, flags, stream)
    return out, tau, mask, ws


def entmax_attn_fused(q, k, v, alpha=1.5, n_iter=10, causal=True, cu_seqlens=None, flags=0,
                      workspace=None, stream=None):
    """The forward pass of entmax_attn_fwd through the two-pass entry points with a
    torch-allocated workspace and ENTMAX_ATTN_FLAG_SUPPORT: the tau pass records each row's
    support, the output pass computes o from the supports (tile pass for the other query tiles).
    Returns (out, tau, block_mask, workspace)."""
    return entmax_attn_two_pass(q, k, v, alpha, n_iter, causal, cu_seqlens,
                                flags | N.FLAG_SUPPORT, workspace, stream)


def fallback_tiles(workspace, stream=None) -> int:
    return int(N.lib().entmax_attn_fallback_tiles(_ptr(workspace), _stream(stream)))


def status(stream=None) -> int:
    return int(N.lib().entmax_attn_status(_stream(stream)))


# ------------------------------------------------------------------ host-side mask decoding --

def tile_slot_table(B, T, cu_seqlens=None):
    """Per sequence: (first slot, number of query tiles, first token, length).  Fixed length:
    one entry per batch row with slot 0.  Follows the documented layout."""
    if cu_seqlens is None:
        nqt = (T + TILE - 1) // TILE
        return [(0, nqt, 0, T) for _ in range(B)]
    cu = [int(x) for x in cu_seqlens]
    return [(cu[s] // TILE + s, (cu[s + 1] - cu[s] + TILE - 1) // TILE, cu[s], cu[s + 1] - cu[s])
            for s in range(len(cu) - 1)]


def decode_block_mask(words, B, Hq, T, cu_seqlens=None):
    """Unpacks the mask words into a bool array [B, Hq, tiles_per_head, nkt]: entry
    [b, h, slot, kt] is the bit of key tile kt.  For a packed batch b = 0 only (B rows are
    sequences, not batch rows) and the array is [1, Hq, slots, nkt]."""
    w = np.asarray(words).astype(np.uint32, copy=False)
    packed = cu_seqlens is not None
    nt = (T + TILE - 1) // TILE
    slots = T // TILE + B if packed else nt
    nw = (nt + 31) // 32
    nb = 1 if packed else B
    w = w.reshape(nb, Hq, slots, nw)
    bits = np.unpackbits(w.view(np.uint8).reshape(nb, Hq, slots, nw, 4), axis=-1,
                         bitorder="little").reshape(nb, Hq, slots, nw * 32)
    return bits[..., :nt].astype(bool)
