"""The seeded input generator (adaptive_sparse_attention_b200/workloads.py), on the CPU: the
recipe the parity tests and bench.py rely on.  Key spikes: round(frac * L) distinct positions per
kv head (per sequence of a packed batch), the fp32 key row multiplied by the factor before the
cast to the storage dtype, values and queries untouched; the same seed gives the same tensors."""
import dataclasses

import pytest
import torch

from adaptive_sparse_attention_b200.workloads import WORKLOADS, Workload, make_inputs


def _spiked_rows(k_spiked, k_plain):
    """Boolean [..., T]: rows of k that differ from the unspiked draw."""
    return (k_spiked != k_plain).any(dim=-1)


@pytest.mark.parametrize("seqlens", [None, (37, 0, 300, 1, 129)])
def test_spikes_scale_the_fp32_rows_of_distinct_positions(seqlens):
    kw = dict(name="w", Hq=4, Hkv=2, d=16, dtype="fp32", alpha=1.5, spike_frac=0.05,
              spike_scale=4.0)
    if seqlens is None:
        w = Workload(B=2, T=300, **kw)
    else:
        w = Workload(B=len(seqlens), T=sum(seqlens), seqlens=seqlens, **kw)
    plain = dataclasses.replace(w, spike_frac=0.0, spike_scale=1.0)
    q, k, v, cu = make_inputs(w, seed=3)
    q0, k0, v0, _ = make_inputs(plain, seed=3)
    assert torch.equal(q, q0) and torch.equal(v, v0)  # only keys are spiked
    rows = _spiked_rows(k, k0)
    assert torch.equal(k[rows], k0[rows] * 4.0)  # exact in fp32
    assert torch.equal(k[~rows], k0[~rows])
    if seqlens is None:
        for b in range(2):
            for h in range(2):
                assert int(rows[b, h].sum()) == round(0.05 * 300)
    else:
        bounds = cu.tolist()
        for s in range(len(seqlens)):
            lo, hi = bounds[s], bounds[s + 1]
            for h in range(2):
                assert int(rows[h, lo:hi].sum()) == round(0.05 * (hi - lo))


def test_bf16_keys_are_cast_after_the_spike():
    """x5 is not exact in bf16: casting first and then scaling would round differently."""
    w = Workload(name="w", B=1, Hq=2, Hkv=1, T=500, d=32, dtype="fp32", alpha=1.5,
                 spike_frac=0.02, spike_scale=5.0)
    _, k32, _, _ = make_inputs(w, seed=5)
    _, kbf, _, _ = make_inputs(dataclasses.replace(w, dtype="bf16"), seed=5)
    assert kbf.dtype == torch.bfloat16
    assert torch.equal(kbf, k32.to(torch.bfloat16))
    _, k0, _, _ = make_inputs(dataclasses.replace(w, spike_frac=0.0, spike_scale=1.0), seed=5)
    rows = _spiked_rows(k32, k0)
    cast_first = (k0[rows].to(torch.bfloat16).float() * 5.0).to(torch.bfloat16)
    assert not torch.equal(kbf[rows], cast_first)


def test_same_seed_same_tensors_other_seed_other_tensors():
    w = WORKLOADS["t4k_bf16_d64_a1.5"]
    a = make_inputs(w, seed=0)
    b = make_inputs(w, seed=0)
    c = make_inputs(w, seed=1)
    for x, y, z in zip(a[:3], b[:3], c[:3]):
        assert torch.equal(x, y) and not torch.equal(x, z)


@pytest.mark.parametrize("name", ["t256_fp32_d64_a1.5", "t4k_bf16_d64_a1.5"])
def test_small_workload_shapes_and_dtypes(name):
    w = WORKLOADS[name]
    q, k, v, cu = make_inputs(w)
    assert cu is None
    assert q.shape == (w.B, w.Hq, w.T, w.d) and k.shape == v.shape == (w.B, w.Hkv, w.T, w.d)
    want = torch.float32 if w.dtype == "fp32" else torch.bfloat16
    assert q.dtype == k.dtype == v.dtype == want


def test_named_workloads_have_the_stated_sizes():
    w = WORKLOADS["b2_t16k_gqa4_bf16_d128_a2"]
    assert (w.B, w.Hq, w.Hkv, w.T, w.d, w.alpha, w.spike_frac, w.spike_scale) == \
        (2, 32, 8, 16384, 128, 2.0, 0.02, 4.0)
    w = WORKLOADS["varlen4_32k_gqa4_bf16_d128_a1.333"]
    assert w.seqlens == (1000, 3000, 8192, 20000) and w.T == 32192 and w.B == 4
    assert (w.Hq, w.Hkv, w.d, w.alpha) == (32, 8, 128, 1.333)
    w = WORKLOADS["t128k_gqa4_bf16_d128_a1.5"]
    assert (w.B, w.Hq, w.Hkv, w.T, w.d, w.alpha, w.spike_frac, w.spike_scale) == \
        (1, 32, 8, 131072, 128, 1.5, 0.01, 5.0)
