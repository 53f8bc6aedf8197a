"""The allocation-free entry point, entmax_attn_fwd_noalloc, against entmax_attn_fwd and the
oracle.

It exists for callers that cannot allocate device memory while they run (code inside an
allocator or memory-pool callback, runtimes with a fixed post-start-up footprint, replayed
launch sequences); its scratch is a fixed device array shared by all calls.  Two calls in a row
on different problems check that what the first call leaves in the shared array does not leak
into the second: each call's output is compared with the fp64 oracle on every row (tau, output
and the block mask under the exemption rule; tau may differ between runs by an ulp, so no
bit-equality is asked of the masks of two runs), and with entmax_attn_fwd's within twice the
forward pass's parity bar.  A last test checks the property itself: after a first call, further calls
leave the device's free memory unchanged.  This file sorts last so that a failure here, with -x,
comes after every other test has run; it also passes on its own in a fresh process.
"""
import ctypes

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


def _problems():
    # first a large packed problem (fills more of the shared scratch), then a smaller one
    w1, in1 = random_case(B=None, Hq=8, Hkv=2, T=None, d=128, dtype="bf16", alpha=1.5,
                          seqlens=(3000, 1, 700, 4100), spike_frac=0.02, spike_scale=4.0,
                          name="noalloc1", seed=5)
    w2 = WORKLOADS["t4k_bf16_d64_a1.5"]
    return [(w1, in1), (w2, make_inputs(w2))]


def _result(w, out, tau, mask, cu):
    bits = ea.decode_block_mask(mask.cpu().numpy(), w.B, w.Hq, w.T, cu)
    return parity.GpuResult(out.float().cpu().numpy().reshape(-1, w.d),
                            tau.cpu().numpy().ravel(), bits, -1)


def test_noalloc_matches_fwd_and_oracle_on_two_calls_in_a_row(oracle):
    dev = torch.device("cuda:0")
    for w, inputs in _problems():
        need = ea.workspace_min_bytes(w.B, w.Hq, w.T, w.varlen)
        assert need <= _native.NOALLOC_SCRATCH_BYTES
        q, k, v, cu = inputs
        qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
        cud = cu.to(dev) if cu is not None else None
        alpha = oracle.alpha_as_float32(w.alpha)
        ref = ea.entmax_attn_fwd(qd, kd, vd, alpha, w.n_iter, w.causal, cud)
        got = ea.entmax_attn_fwd_noalloc(qd, kd, vd, alpha, w.n_iter, w.causal, cud)
        torch.cuda.synchronize()
        assert ea.status() == 0
        r = _result(w, *ref, cu)
        g = _result(w, *got, cu)
        # against the oracle, every row
        parity.compare(w, inputs, g, parity.all_tiles(w, cu), label=f"noalloc {w.name}")
        # against the existing entry point: each lies within the parity bar of the exact value,
        # so the two lie within twice the bar of each other.  (Without room for the warm-up keys
        # the allocation-free call may send other query tiles through the overflow path, whose
        # output comes from the tile pass with p rounded to bf16 rather than from the tau pass's
        # fp32 gather, so the two need not round alike.)
        ref_o = r.out.astype(np.float64)
        assert np.all(np.abs(g.out - r.out) <= 2 * parity.out_bar(w, ref_o)), w.name
        assert np.max(np.abs(g.tau - r.tau) / np.maximum(1.0, np.abs(r.tau))) <= parity.TAU_RTOL


def test_noalloc_allocates_no_device_memory(oracle):
    """After a first call (which may load the library's kernels), further calls change the
    device's free memory by nothing: the outputs were allocated before, and the scratch is the
    library's fixed array."""
    dev = torch.device("cuda:0")
    w, inputs = _problems()[0]
    q, k, v, cu = inputs
    qd, kd, vd, cud = q.to(dev), k.to(dev), v.to(dev), cu.to(dev)
    out = torch.empty_like(qd)
    tau = torch.empty(qd.shape[:-1], dtype=torch.float32, device=dev)
    mask = torch.empty(ea.mask_words(w.B, w.Hq, w.T, True), dtype=torch.int32, device=dev)
    lib = _native.lib()
    args = [ctypes.c_void_p(t.data_ptr()) for t in (qd, kd, vd, out, tau, mask)]
    call = lambda: lib.entmax_attn_fwd_noalloc(  # noqa: E731
        *args, w.B, w.Hq, w.Hkv, w.T, w.d, oracle.alpha_as_float32(w.alpha), w.n_iter,
        int(w.causal), ctypes.c_void_p(cud.data_ptr()), _native.BF16, None)
    assert call() == 0
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info(dev)
    for _ in range(2):
        assert call() == 0
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info(dev)
    assert ea.status() == 0
    assert free1 == free0, (free0, free1)


def test_noalloc_rejects_problems_beyond_its_scratch():
    lib = _native.lib()
    w = WORKLOADS["t128k_gqa4_bf16_d128_a1.5"]
    assert ea.workspace_min_bytes(w.B, w.Hq, w.T, False) > _native.NOALLOC_SCRATCH_BYTES
    fake = ctypes.c_void_p(0x10000)  # never dereferenced: the size check comes first
    rc = lib.entmax_attn_fwd_noalloc(fake, fake, fake, fake, fake, fake, w.B, w.Hq, w.Hkv, w.T,
                                     w.d, 1.5, 10, 1, None, _native.BF16, None)
    assert rc == _native.ENOMEM
