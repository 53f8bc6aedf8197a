"""Failure detection on the GPU without a fault: the tensor-core tau pass, given the test hook
ENTMAX_ATTN_FLAG_TEST_STALL, never requests its query tile, so its waits run out.  Every role of
the CTA must leave, the pass must report ENTMAX_ATTN_ETIMEOUT through the status word, and the
context must stay usable: the next, normal call matches the oracle."""
import time

import pytest
import torch

from adaptive_sparse_attention_b200 import _native
from adaptive_sparse_attention_b200 import api as ea
from adaptive_sparse_attention_b200.workloads import random_case
import parity

pytestmark = pytest.mark.gpu


def test_stalled_tau_pass_times_out_and_recovers(oracle):
    if not torch.cuda.is_available():
        pytest.fail("a CUDA device is required for -m gpu tests")
    # one query tile: a single CTA waits out one limit
    w, inputs = random_case(B=1, Hq=1, Hkv=1, T=128, d=64, dtype="bf16", alpha=1.5,
                            name="stall", seed=5)
    q, k, v, cu = (x.cuda() if x is not None else None for x in inputs)
    assert ea.status() == _native.OK
    out, tau, mask = ea.alloc_outputs(q, k, None)
    ws = ea.alloc_workspace(q, k, None)
    t0 = time.monotonic()
    ea.tau_pass(q, k, tau, mask, ws, 1.5, 10, True, None, _native.FLAG_TEST_STALL)
    code = ea.status()  # synchronises: the CTA has returned
    elapsed = time.monotonic() - t0
    assert code == _native.ETIMEOUT
    assert elapsed < 30.0
    assert ea.status() == _native.OK  # the word was cleared

    g = parity.run_gpu(w, inputs)
    assert ea.status() == _native.OK
    parity.compare(w, inputs, g, parity.all_tiles(w, inputs[3]), label="after-timeout")
