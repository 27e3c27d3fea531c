"""GPU parity of cadd_cost_fit (the non-negative fit of the verification cost).

CaDDTree summary (gist.science), "Method: CaDDTree": C_v(n; l) profiled offline
as a convex, non-decreasing cost, i.e. a + b l + c n + e n^2 with a, b, c, e >= 0
fitted to latency samples. The device fit is compared with oracle.cost_fit (the
exhaustive free-set search) on synthetic samples: noisy convex costs with some
coefficients truly zero, concave data that pins e at zero, and the noiseless
cost of the configurations. Both sides work in float64 from the same float32
samples; the coefficients agree to 1e-6 relative.
"""
import numpy as np
import pytest
import torch

import oracle
import speculative_decoding_draft_07_b200 as pct

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda")


def _fit(n, ell, t):
    f = lambda x: torch.as_tensor(np.asarray(x, np.float32), device=DEV)
    out, st = pct.cadd_cost_fit(f(n), f(ell), f(t))
    torch.cuda.synchronize()
    return out.cpu().numpy(), int(st.cpu()[0])


def _check(n, ell, t):
    n32, l32, t32 = (np.asarray(x, np.float32) for x in (n, ell, t))
    got, st = _fit(n32, l32, t32)
    ref = np.array(oracle.cost_fit(n32, l32, t32))
    assert st == 0
    scale = np.array([1.0, 1e-4, 1e-3, 1e-5])      # coefficient magnitudes of the model
    np.testing.assert_allclose(got[:4], ref[:4], rtol=1e-6, atol=1e-9 * scale.max())
    np.testing.assert_allclose(got[4], ref[4], rtol=1e-4, atol=1e-5)
    return got, ref


@pytest.mark.parametrize("seed", range(12))
def test_noisy_convex_costs(seed):
    rng = np.random.default_rng(5000 + seed)
    m = int(rng.integers(8, 3000))
    n = rng.integers(1, 512, m)
    ell = rng.choice([512, 4096, 32768], m)
    coef = rng.uniform(0, 1, 4) * np.array([2.0, 1e-4, 5e-3, 1e-5])
    coef[rng.random(4) < 0.3] = 0.0
    t = coef[0] + coef[1] * ell + coef[2] * n + coef[3] * n * n + rng.normal(0, 0.02, m)
    _check(n, ell, t)


def test_noiseless_configuration_cost():
    n = np.repeat(np.arange(1, 513, 7), 3)
    ell = np.tile([512, 4096, 32768], len(n) // 3)
    t = 2.0 + 1e-4 * ell + 5e-3 * n + 1e-5 * n * n
    got, _ = _check(n, ell, t)
    np.testing.assert_allclose(got[:4], [2.0, 1e-4, 5e-3, 1e-5], rtol=1e-4)


def test_concave_data_keeps_e_at_zero():
    n = np.arange(1, 400)
    ell = np.where(n % 2 == 0, 4096, 32768)
    t = 3.0 + 2e-5 * ell + 0.02 * n - 4e-5 * n * n
    got, ref = _check(n, ell, t)
    assert got[3] == 0.0 and ref[3] == 0.0


def test_non_finite_sample_is_reported():
    n = np.arange(1, 50, dtype=np.float32)
    ell = np.full_like(n, 4096.0)
    t = 1.0 + 0.01 * n
    t[7] = np.nan
    _, st = _fit(n, ell, t)
    assert st == pct.DEV_BAD_COST
