"""Seeded synthetic inputs for causal alpha-entmax attention.

This module only draws random tensors; it holds none of the attention arithmetic, and both the
CUDA library's tests and the oracle's are fed from it.

Shapes and value distributions follow the workloads the attention is measured on: q, k, v iid
N(0, 1) in the heads-before-tokens layout [B, H, T, d] of the "AdaSplash with Block Masking"
example (AdaSplash: Adaptive Sparse Flash Attention), or packed [H, T_total, d] with
``cu_seqlens`` for a variable-length batch ("Variable Length Sequences" section).  "Key spikes"
make rows peaked and sparse: in each kv head (and each sequence of a packed batch) a fraction of
the key positions, drawn uniformly without replacement, has its fp32 key row multiplied by a
factor before the cast to the storage dtype.

Draw order, from one ``torch.Generator`` seeded with ``seed``: q, k, v as fp32 ``randn`` in that
order, then the spike positions with ``randperm`` per (batch, kv head) -- per (sequence, kv head)
for a packed batch -- then the cast.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int                    # batch (number of sequences when seqlens is set)
    Hq: int
    Hkv: int
    T: int                    # tokens per sequence, or total packed tokens when seqlens is set
    d: int
    dtype: str                # "fp32" or "bf16"
    alpha: float
    n_iter: int = 10
    causal: bool = True
    spike_frac: float = 0.0
    spike_scale: float = 1.0
    seqlens: tuple[int, ...] | None = None
    note: str = field(default="", compare=False)

    @property
    def varlen(self) -> bool:
        return self.seqlens is not None


def _packed(name, seqlens, **kw):
    return Workload(name=name, B=len(seqlens), T=int(sum(seqlens)), seqlens=tuple(seqlens), **kw)


# The five workloads the forward pass is measured and checked on (sizes, dtypes, alpha and spike
# recipes).
WORKLOADS: dict[str, Workload] = {w.name: w for w in [
    Workload("t256_fp32_d64_a1.5", B=1, Hq=2, Hkv=2, T=256, d=64, dtype="fp32", alpha=1.5,
             note="small fp32 case, no spikes"),
    Workload("t4k_bf16_d64_a1.5", B=1, Hq=8, Hkv=8, T=4096, d=64, dtype="bf16", alpha=1.5,
             spike_frac=0.02, spike_scale=4.0),
    Workload("b2_t16k_gqa4_bf16_d128_a2", B=2, Hq=32, Hkv=8, T=16384, d=128, dtype="bf16",
             alpha=2.0, spike_frac=0.02, spike_scale=4.0),
    _packed("varlen4_32k_gqa4_bf16_d128_a1.333", (1000, 3000, 8192, 20000), Hq=32, Hkv=8, d=128,
            dtype="bf16", alpha=1.333, spike_frac=0.02, spike_scale=4.0),
    Workload("t128k_gqa4_bf16_d128_a1.5", B=1, Hq=32, Hkv=8, T=131072, d=128, dtype="bf16",
             alpha=1.5, spike_frac=0.01, spike_scale=5.0),
]}
WORKLOAD_ORDER = list(WORKLOADS)


def storage_dtype(name: str) -> torch.dtype:
    return {"fp32": torch.float32, "bf16": torch.bfloat16}[name]


def cu_seqlens_of(seqlens) -> torch.Tensor:
    cu = [0]
    for n in seqlens:
        cu.append(cu[-1] + int(n))
    return torch.tensor(cu, dtype=torch.int32)


def make_inputs(w: Workload, seed: int = 0):
    """Draw (q, k, v, cu_seqlens) on the CPU; cu_seqlens is None for fixed-length batches."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    if w.varlen:
        qshape, kshape = (w.Hq, w.T, w.d), (w.Hkv, w.T, w.d)
    else:
        qshape, kshape = (w.B, w.Hq, w.T, w.d), (w.B, w.Hkv, w.T, w.d)
    q = torch.randn(qshape, generator=g, dtype=torch.float32)
    k = torch.randn(kshape, generator=g, dtype=torch.float32)
    v = torch.randn(kshape, generator=g, dtype=torch.float32)
    cu = cu_seqlens_of(w.seqlens) if w.varlen else None
    if w.spike_frac > 0.0:
        if w.varlen:
            for s in range(w.B):
                lo, hi = int(cu[s]), int(cu[s + 1])
                n = round(w.spike_frac * (hi - lo))
                for h in range(w.Hkv):
                    pos = torch.randperm(hi - lo, generator=g)[:n] + lo
                    k[h, pos] *= w.spike_scale
        else:
            n = round(w.spike_frac * w.T)
            for b in range(w.B):
                for h in range(w.Hkv):
                    pos = torch.randperm(w.T, generator=g)[:n]
                    k[b, h, pos] *= w.spike_scale
    dt = storage_dtype(w.dtype)
    return q.to(dt), k.to(dt), v.to(dt), cu


def random_case(B, Hq, Hkv, T, d, dtype="bf16", alpha=1.5, causal=True, seqlens=None,
                spike_frac=0.0, spike_scale=1.0, n_iter=10, seed=0, name="case"):
    """An ad-hoc workload plus its inputs, for parity cases off the five named workloads."""
    if seqlens is not None:
        w = _packed(name, seqlens, Hq=Hq, Hkv=Hkv, d=d, dtype=dtype, alpha=alpha, causal=causal,
                    spike_frac=spike_frac, spike_scale=spike_scale, n_iter=n_iter)
    else:
        w = Workload(name, B=B, Hq=Hq, Hkv=Hkv, T=T, d=d, dtype=dtype, alpha=alpha, causal=causal,
                     spike_frac=spike_frac, spike_scale=spike_scale, n_iter=n_iter)
    return w, make_inputs(w, seed)
