"""GPU parity of the host-memory entry point entmax_attn_fwd_host (inputs and outputs in pinned
host memory, streamed through the GPU in chunks of whole (batch row, kv head) groups) against the
fp64 oracle, on the same seeded inputs and bars as the device entry points (parity.py): small
fixed-length and packed problems on every row, the 16K workload on sampled query tiles and rows,
and two calls in a row of different problems (the staging buffer and events are reused)."""
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


def _host_run(w, inputs):
    q, k, v, cu = inputs
    pinned = [t.pin_memory() for t in (q, k, v)]
    out, tau, mask = ea.entmax_attn_fwd_host(*pinned, oracle_alpha(w), w.n_iter, w.causal, cu)
    assert ea.status() == 0
    bits = ea.decode_block_mask(mask.numpy(), w.B, w.Hq, w.T, cu)
    return parity.GpuResult(out.float().numpy().reshape(-1, w.d), tau.numpy().ravel(), bits, -1)


def oracle_alpha(w):
    return float(np.float32(w.alpha))


CASES = [
    ("fixed_gqa", dict(B=2, Hq=8, Hkv=2, T=700, d=128, alpha=1.5, spike_frac=0.02,
                       spike_scale=4.0)),
    ("fixed_many_groups", dict(B=3, Hq=34, Hkv=17, T=129, d=64, alpha=2.0)),
    ("packed_ragged", dict(B=None, Hq=4, Hkv=2, T=None, d=128, alpha=1.333,
                           seqlens=(5, 0, 300, 1, 129, 256))),
    ("fp32", dict(B=1, Hq=2, Hkv=1, T=300, d=64, alpha=1.5, dtype="fp32")),
]


@pytest.mark.parametrize("name,kw", CASES, ids=[c[0] for c in CASES])
def test_host_entry_matches_oracle(oracle, name, kw):
    kw = dict(kw)
    dtype = kw.pop("dtype", "bf16")
    w, inputs = random_case(dtype=dtype, name=name, seed=23, **kw)
    g = _host_run(w, inputs)
    parity.compare(w, inputs, g, parity.all_tiles(w, inputs[3]), label=f"host/{name}")


def test_host_entry_16k_and_a_second_call(oracle):
    """The 16K workload (16 chunks of one (batch row, kv head) group each), then a small packed
    problem through the same pipeline."""
    w = WORKLOADS["b2_t16k_gqa4_bf16_d128_a2"]
    inputs = make_inputs(w)
    g = _host_run(w, inputs)
    rng = np.random.default_rng(77)
    tiles = [(b, h, b, int(qt)) for b in range(w.B) for h in (0, 5, 31)
             for qt in rng.choice(w.T // 128, size=2, replace=False)]
    loose = rng.choice(w.B * w.Hq * w.T, size=1024, replace=False)
    parity.compare(w, inputs, g, tiles, loose, label="host/16k")
    # the device entry point on the same inputs gives the same result within the bars
    dev = [t.cuda() for t in inputs[:3]]
    o_d, t_d, _ = ea.entmax_attn_fwd(*dev, oracle_alpha(w), w.n_iter, w.causal)
    torch.cuda.synchronize()
    o_d = o_d.float().cpu().numpy().reshape(-1, w.d)
    assert np.all(np.abs(g.out - o_d) <= parity.out_bar(w, o_d.astype(np.float64)))
    w2, in2 = random_case(B=None, Hq=4, Hkv=1, T=None, d=128, dtype="bf16", alpha=1.5,
                          seqlens=(1000, 17, 2100), name="host_second", seed=29)
    g2 = _host_run(w2, in2)
    parity.compare(w2, in2, g2, parity.all_tiles(w2, in2[3]), label="host/second")
