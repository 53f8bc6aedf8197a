"""The allocation-free entry point, entmax_attn_fwd_noalloc, against entmax_attn_fwd.

It exists for callers that cannot allocate device memory while they run (code inside an
allocator or memory-pool callback, runtimes with a fixed post-start-up footprint, replayed
launch sequences); its scratch is a fixed device array shared by all calls.  Two calls in a row
on different problems check that what the first call leaves in the shared array does not leak
into the second.  This file sorts last so that a failure here, with -x, comes after every other
test has run; it also passes on its own in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

import adaptive_sparse_attention_b200 as ea
from adaptive_sparse_attention_b200 import _native
from adaptive_sparse_attention_b200.workloads import WORKLOADS, make_inputs, random_case

pytestmark = pytest.mark.gpu

OUT_TOL = {"fp32": 1e-4, "bf16": 2e-2}  # the parity bar of the forward pass
TAU_RTOL = 1e-4


def _run_both(w, inputs):
    q, k, v, cu = inputs
    dev = torch.device("cuda:0")
    q, k, v = q.to(dev), k.to(dev), v.to(dev)
    cud = cu.to(dev) if cu is not None else None
    alpha = float(np.float32(w.alpha))
    ref = ea.entmax_attn_fwd(q, k, v, alpha, w.n_iter, w.causal, cud)
    got = ea.entmax_attn_fwd_noalloc(q, k, v, alpha, w.n_iter, w.causal, cud)
    torch.cuda.synchronize()
    assert ea.status() == 0
    return [t.float().cpu().numpy() for t in ref], [t.float().cpu().numpy() for t in got]


def _check(w, ref, got):
    (o_r, t_r, m_r), (o_g, t_g, m_g) = ref, got
    assert np.max(np.abs(o_g - o_r)) <= OUT_TOL[w.dtype]
    assert np.max(np.abs(t_g - t_r) / np.maximum(1.0, np.abs(t_r))) <= TAU_RTOL
    assert np.array_equal(m_g.view(np.int32), m_r.view(np.int32))


def test_noalloc_matches_fwd_on_two_calls_in_a_row():
    if not torch.cuda.is_available():
        pytest.fail("a CUDA device is required for -m gpu tests")
    # first a large packed problem (fills more of the shared scratch), then a smaller one
    w1, in1 = random_case(B=None, Hq=8, Hkv=2, T=None, d=128, dtype="bf16", alpha=1.5,
                          seqlens=(3000, 1, 700, 4100), spike_frac=0.02, spike_scale=4.0,
                          name="noalloc1", seed=5)
    w2 = WORKLOADS["t4k_bf16_d64_a1.5"]
    in2 = make_inputs(w2)
    for w, inputs in ((w1, in1), (w2, in2)):
        need = ea.workspace_min_bytes(w.B, w.Hq, w.T, w.varlen)
        assert need <= _native.NOALLOC_SCRATCH_BYTES
        ref, got = _run_both(w, inputs)
        _check(w, ref, got)


def test_noalloc_rejects_problems_beyond_its_scratch():
    if not torch.cuda.is_available():
        pytest.fail("a CUDA device is required for -m gpu tests")
    lib = _native.lib()
    w = WORKLOADS["t128k_gqa4_bf16_d128_a1.5"]
    assert ea.workspace_min_bytes(w.B, w.Hq, w.T, False) > _native.NOALLOC_SCRATCH_BYTES
    fake = ctypes.c_void_p(0x10000)  # never dereferenced: the size check comes first
    rc = lib.entmax_attn_fwd_noalloc(fake, fake, fake, fake, fake, fake, w.B, w.Hq, w.Hkv, w.T,
                                     w.d, 1.5, 10, 1, None, _native.BF16, None)
    assert rc == _native.ENOMEM
