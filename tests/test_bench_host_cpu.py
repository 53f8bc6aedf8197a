"""Host-side arithmetic of bench.py, on the CPU: the valid-pair counts behind the effective-FLOP
metric, the DRAM-traffic record that is reported only while the kernel sources are unchanged,
the clock summary taken from nvidia-smi samples, and the kernel count per step."""
import numpy as np
import pytest

import bench
from adaptive_sparse_attention_b200.workloads import WORKLOADS


@pytest.mark.parametrize("L", [1, 2, 127, 128, 129, 300, 1000])
def test_pair_matrix_counts_every_valid_pair_once(L):
    causal = bench.pair_matrix(L, True)
    full = bench.pair_matrix(L, False)
    assert int(causal.sum()) == L * (L + 1) // 2
    assert int(full.sum()) == L * L
    nt = (L + 127) // 128
    assert causal.shape == full.shape == (nt, nt)
    assert np.all(np.triu(causal, 1) == 0)  # no key tile after the query tile
    # brute force over positions
    qt = np.arange(L) // 128
    want = np.zeros((nt, nt), dtype=np.int64)
    for i in range(L):
        np.add.at(want[qt[i]], qt[: i + 1], 1)
    assert np.array_equal(causal, want)


def test_traffic_is_reported_only_for_the_captured_sources(monkeypatch):
    h = bench.kernel_sources_hash()
    table = {("wl", "out_pass"): (123.0e6, h, "capture"),
             ("wl", "tau_pass"): (456.0e6, "0" * 16, "capture")}
    monkeypatch.setattr(bench, "NCU_TRAFFIC", table)
    assert bench.ncu_traffic("wl", "out_pass") == 123.0e6
    assert bench.ncu_traffic("wl", "tau_pass") is None  # sources changed since the capture
    assert bench.ncu_traffic("other", "out_pass") is None


def test_capture_hash_ignores_comments_but_not_code():
    src = "int f(int x) {  // the tile count\n  /* two\n lines */ return x + 1;\n}\n"
    assert bench._code_only(src) == bench._code_only(src.replace("the tile count", "rows"))
    assert bench._code_only(src) == bench._code_only(src.replace("\n  ", "\n\n      "))
    assert bench._code_only(src) != bench._code_only(src.replace("x + 1", "x + 2"))


def test_clock_summary_reads_median_clock_and_active_reasons():
    s = bench.ClockSampler(0)
    row = "0, {sm}, 1965, 900.5, 0x0, Not Active, Not Active, Not Active, {cap}"
    s.lines = [row.format(sm=120, cap="Not Active"),   # idle sample before the load
               row.format(sm=1965, cap="Not Active"),
               row.format(sm=1870, cap="Active"),
               row.format(sm=1900, cap="Not Active"),
               "garbage line"]
    got = s.summary()
    assert got["sm_max_mhz"] == 1965.0
    assert got["sm_mhz"] == 1900.0  # median of the loaded samples (idle one left out)
    assert got["reasons"] == ["sw_power_cap"]
    assert got["samples"] == 4
    s.lines = []
    assert s.summary() is None


def test_launches_per_step():
    assert bench.launches_per_step(WORKLOADS["t256_fp32_d64_a1.5"]) == 3
    assert bench.launches_per_step(WORKLOADS["t4k_bf16_d64_a1.5"]) == 6
    assert bench.launches_per_step(WORKLOADS["b2_t16k_gqa4_bf16_d128_a2"]) == 6
    assert bench.launches_per_step(WORKLOADS["b2_t16k_gqa4_bf16_d128_a2"], "tile") == 5
    assert bench.launches_per_step(WORKLOADS["b2_t16k_gqa4_bf16_d128_a2"], "nomask") == 5
