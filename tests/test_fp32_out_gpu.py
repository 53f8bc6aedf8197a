"""The fp32-accumulated output of bf16 inputs against the flat bar.

The forward pass's bf16 bar is 2e-2 on the fp32-accumulated value; a bf16-stored output adds
the half-ulp rounding of the store (parity.py).  With ENTMAX_ATTN_FLAG_OUT_FP32 the passes store
the fp32 accumulations themselves, so here every checked element must lie within the flat 2e-2
of the fp64 oracle: on both forward paths (the tau pass's gather and the tile output pass), on
the 16K sparsemax workload and the packed 32K alpha = 1.333 workload (sampled query tiles and
rows, the launch configuration bench.py times), and on small cases with every row."""
import numpy as np
import pytest
import torch

from adaptive_sparse_attention_b200 import _native
from adaptive_sparse_attention_b200.workloads import WORKLOADS, make_inputs, random_case
import adaptive_sparse_attention_b200 as ea
import parity

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.fail("a CUDA device is required for -m gpu tests")
    _native.lib()


def _run(w, inputs, path):
    g = parity.run_gpu(w, inputs, flags=_native.FLAG_OUT_FP32, path=path)
    return g


@pytest.mark.parametrize("path", parity.PATHS)
@pytest.mark.parametrize("name", ["b2_t16k_gqa4_bf16_d128_a2",
                                  "varlen4_32k_gqa4_bf16_d128_a1.333"])
def test_fp32_out_flat_bar_workloads(oracle, name, path):
    w = WORKLOADS[name]
    inputs = make_inputs(w)
    g = _run(w, inputs, path)
    rng = np.random.default_rng(2024)
    table = parity.seq_table(w, inputs[3])
    tiles = []
    nb = 1 if inputs[3] is not None else w.B
    for b in range(nb):
        for h in (0, 7, 30):
            for s in (range(len(table)) if inputs[3] is not None else [b]):
                nqt = table[s][1]
                tiles += [(b, h, s, int(qt)) for qt in
                          sorted(set(rng.choice(nqt, size=min(2, nqt), replace=False).tolist())
                                 | {nqt - 1})]
    rows = w.Hq * w.T * (1 if inputs[3] is not None else w.B)
    loose = rng.choice(rows, size=1024, replace=False)
    s = parity.compare(w, inputs, g, tiles, loose, label=f"fp32out/{name}/{path}",
                       flat_bar=True)
    assert s["max_out_err"] <= 2e-2


SMALL = [
    ("t1000_spk", dict(B=1, Hq=4, Hkv=2, T=1000, d=128, alpha=1.5, spike_frac=0.02,
                       spike_scale=4.0)),
    ("varlen_ragged", dict(B=None, Hq=4, Hkv=2, T=None, d=128, alpha=1.333,
                           seqlens=(5, 0, 300, 1, 129, 256))),
    ("t300_d64_a2", dict(B=2, Hq=2, Hkv=1, T=300, d=64, alpha=2.0)),
]


@pytest.mark.parametrize("path", parity.PATHS)
@pytest.mark.parametrize("name,kw", SMALL, ids=[c[0] for c in SMALL])
def test_fp32_out_flat_bar_small(oracle, name, kw, path):
    w, inputs = random_case(dtype="bf16", name=name, seed=31, **kw)
    g = _run(w, inputs, path)
    parity.compare(w, inputs, g, parity.all_tiles(w, inputs[3]), label=f"fp32out/{name}",
                   flat_bar=True)


def test_fp32_out_needs_the_tensor_core_path():
    w, inputs = random_case(B=1, Hq=2, Hkv=1, T=200, d=64, dtype="fp32", alpha=1.5,
                            name="fp32in", seed=3)
    q, k, v = (t.cuda() for t in inputs[:3])
    with pytest.raises(_native.EntmaxAttnError) as e:
        ea.entmax_attn_fused(q, k, v, 1.5, 10, True, flags=_native.FLAG_OUT_FP32)
    assert e.value.code == _native.EINVAL
