"""GPU parity of the standalone row-wise alpha-entmax (AdaSplash page, "Triton Entmax (Optimized
Entmax Activation)") against the oracle's exact alpha-entmax of each row: tau within
1e-4 max(1, |tau|), p within the output tolerance of the attention passes (fp32: 1e-4, plus the
derived 2^(-20 beta) for beta < 1; bf16 p is stored rounded to bf16: 2^-8 relative + 1e-4)."""
import numpy as np
import pytest
import torch

import adaptive_sparse_attention_b200 as ea
from oracle import oracle as orc

pytestmark = pytest.mark.gpu


def _check(x, p, tau, alpha, dtype):
    a32 = orc.alpha_as_float32(alpha)
    beta = 1.0 / (a32 - 1.0)
    xs = x.float().cpu().numpy().astype(np.float64)
    ps = p.float().cpu().numpy()
    ts = tau.cpu().numpy()
    ptol = 1e-4 + (2.0 ** (-20.0 * beta) if beta < 1.0 else 0.0)
    for r in range(xs.shape[0]):
        z = (a32 - 1.0) * xs[r]
        pr, tr = orc.entmax_vec(z, a32)
        assert abs(ts[r] - tr) <= 1e-4 * max(1.0, abs(tr)), (r, ts[r], tr)
        if dtype == "bf16":
            err = np.abs(ps[r] - pr) - 2.0 ** -8 * np.abs(pr)
            assert float(err.max()) <= 1e-4, (r, float(err.max()))
        else:
            assert float(np.abs(ps[r] - pr).max()) <= ptol, (r, float(np.abs(ps[r] - pr).max()))
            assert abs(float(ps[r].sum()) - 1.0) <= 1e-3


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
# alpha > 2: a near-uniform row puts tau within n^(1 - alpha) of the bracket end, where the
# Halley proposals overshoot and the search bisects; 40 steps resolve that for n up to 10^6.
@pytest.mark.parametrize("alpha,n_iter", [(1.333, 10), (1.5, 10), (2.0, 10), (3.0, 40)])
@pytest.mark.parametrize("n", [1, 5, 33, 1000, 4099])
def test_rows_match_oracle(oracle, dtype, alpha, n_iter, n):
    g = torch.Generator().manual_seed(1000 + n)
    x = torch.randn(24, n, generator=g) * 2.0
    x[3] = 0.0                      # all-equal row: uniform p
    if n > 1:
        x[5, n // 2] += 40.0        # one dominant entry: p = one-hot
        x[7, : n // 2] = x[7, n // 2]  # ties
    x = x.to(torch.bfloat16 if dtype == "bf16" else torch.float32).cuda()
    p, tau = ea.entmax_rows(x, orc.alpha_as_float32(alpha), n_iter)
    torch.cuda.synchronize()
    _check(x, p, tau, alpha, dtype)


def test_rows_strided_and_batched(oracle):
    """Rows taken from a wider matrix (row stride > n) and a 3-D input."""
    g = torch.Generator().manual_seed(7)
    wide = (torch.randn(16, 300, generator=g) * 3.0).cuda()
    x = wide[:, :257]  # row stride 300
    p, tau = ea.entmax_rows(x, 1.5, 10)
    torch.cuda.synchronize()
    _check(x, p, tau, 1.5, "fp32")
    x3 = (torch.randn(2, 3, 77, generator=g)).to(torch.bfloat16).cuda()
    p3, t3 = ea.entmax_rows(x3, 2.0, 10)
    torch.cuda.synchronize()
    assert p3.shape == x3.shape and t3.shape == (2, 3)
    _check(x3.reshape(-1, 77), p3.reshape(-1, 77), t3.reshape(-1), 2.0, "bf16")


@pytest.mark.parametrize("alpha", [1.5, 2.0])
def test_tied_rows_every_length(oracle, alpha):
    """Rows whose entries all tie have tau = m - n^(1 - alpha) exactly, the upper end of the
    search bracket, and p = 1/n.  Whether an fp32 search step lands inside or just outside that
    end depends on the rounding at each n, so every n from 2 to 1200 is checked against the
    closed forms, at three offsets m."""
    a32 = orc.alpha_as_float32(alpha)
    for n in range(2, 1201):
        x = torch.tensor([0.0, 3.25, -7.5], dtype=torch.float32)[:, None].repeat(1, n).cuda()
        p, tau = ea.entmax_rows(x, a32, 10)
        torch.cuda.synchronize()
        z = (a32 - 1.0) * np.array([0.0, 3.25, -7.5])
        want = z - float(n) ** (1.0 - a32)
        got = tau.cpu().numpy().astype(np.float64)
        assert np.all(np.abs(got - want) <= 1e-4 * np.maximum(1.0, np.abs(want))), (n, got, want)
        assert float((p.cpu().double() - 1.0 / n).abs().max()) <= 1e-4, n
