"""Pins of the oracle's synthetic write-back studies (oracle/simulate.py):
the autocorrelation estimator on series of known correlation, the
independent-noise readout model against its closed form and a Monte Carlo
of the same noise, the Gramian diagonal against closed forms and the
pages' worked example, and the allocation comparison's invariances."""
import math

import numpy as np
import pytest

from bit_recurrent_state_b200 import synth
from conftest import golden


@pytest.fixture(scope="module")
def sim():
    from oracle import simulate
    return simulate


def _running_sums(E):
    """Running sums of a series E [n][...] as the studies accumulate them."""
    n = E.shape[0]
    s1 = E.sum(0)
    s2 = (E * E).sum(0)
    cr = (E[:-1] * E[1:]).sum(0)
    return s1, s2, cr, E[0], E[-1], n


@pytest.mark.parametrize("phi", [0.0, 0.23, 0.7, -0.4])
def test_lag1_estimator_recovers_ar1(sim, phi):
    rng = np.random.default_rng(1)
    n, m = 4000, 400
    E = np.zeros((n, m))
    E[0] = rng.standard_normal(m) / math.sqrt(1 - phi * phi)
    for t in range(1, n):
        E[t] = phi * E[t - 1] + rng.standard_normal(m)
    E += 3.0                                             # a mean the estimator must remove
    r = sim.lag1_autocorrelation(*_running_sums(E))
    assert abs(r.mean() - phi) < 4 * math.sqrt((1 - phi * phi) / (n * m)) + 2.0 / n
    # the centred textbook form, element by element
    Ec = E - E.mean(0)
    ref = (Ec[:-1] * Ec[1:]).sum(0) / (Ec * Ec).sum(0)
    np.testing.assert_allclose(r, ref, rtol=1e-9, atol=1e-12)


def test_readout_model_closed_form(sim):
    """No writes (beta = 0), one decay a: the noise covariance settles at
    sigma^2 / (1 - a^2) and a unit readout sees a^2 sigma^2 / (1 - a^2) per
    value column."""
    d, T, a, s2 = 8, 3000, 0.97, 0.3
    F = np.repeat((a * np.eye(d))[None], T, axis=0)
    q = np.zeros((T, d)); q[:, 2] = 1.0
    out = sim.readout_model(F, q, np.full((T, d), s2), d_v=5)
    assert out[0] == 0.0
    assert out[-1] == pytest.approx(5 * a * a * s2 / (1 - a * a), rel=1e-9)


def test_readout_model_matches_monte_carlo(sim):
    """Non-symmetric F_t = (I - beta k k^T) diag(a) with per-row decays and
    row variances: the model's expected readout error equals the mean over
    many independent noise draws propagated the same way (a transposed F or
    a misplaced noise term fails)."""
    rng = np.random.default_rng(2)
    d, T, N = 6, 40, 40000
    a = np.exp(-rng.uniform(0.01, 0.5, (T, d)))
    k = rng.standard_normal((T, d)); k /= np.linalg.norm(k, axis=1, keepdims=True)
    beta = rng.uniform(0.2, 0.9, T)
    F = (np.eye(d)[None] - beta[:, None, None] * k[:, :, None] * k[:, None, :]) * a[:, None, :]
    q = rng.standard_normal((T, d))
    s2 = rng.uniform(0.1, 1.0, (T, d))
    model = sim.readout_model(F, q, s2, d_v=1)
    E = np.zeros((N, d))
    mc = np.zeros(T)
    for t in range(T):
        pre = E @ F[t].T                                  # F_t E_(t-1), one column per draw
        mc[t] = np.mean((pre @ q[t]) ** 2)
        E = pre + rng.standard_normal((N, d)) * np.sqrt(s2[t])
    sel = slice(5, None)
    assert np.all(np.abs(mc[sel] / model[sel] - 1) < 0.06), np.max(np.abs(mc[sel] / model[sel] - 1))


def test_gramian_diag_closed_forms(sim):
    """beta = 0: the diagonal is sum_l a_i^(2l); the pages' fixed-key example
    (k = (1, 1)/sqrt 2, a = k/2, s = 0.01) gives the exact rate 24.9."""
    d, L = 5, 600
    a = np.exp(-np.array([0.01, 0.05, 0.2, 0.5, 1.0]))
    F = np.repeat(np.diag(a)[None], L + 1, axis=0)
    g = sim.gramian_diag(F, [0], L)
    ref = np.array([sum(x ** (2 * l) for l in range(1, L + 1)) for x in a])
    np.testing.assert_allclose(g, ref, rtol=1e-12)
    gold = golden("erasure_rate_example.txt")
    s = float(gold["s"])
    k = np.array([1.0, 1.0]) / math.sqrt(2)
    Fx = (np.eye(2) - np.outer(k, k / 2)) * math.exp(-s)
    g2 = sim.gramian_diag(np.repeat(Fx[None], 6001, axis=0), [0], 6000)
    assert round(g2[0], 1) == float(gold["gamma_exact"])


def test_approx_gamma_of_constant_inputs(sim, orc):
    w = synth.Workload("g", B=1, H=2, d=16, T=4, seed=3)
    inp = synth.run_inputs(w, 0, 4)
    inp["decay"][:] = np.float32(0.9)
    inp["beta"][:] = np.float32(0.5)
    g = sim.approx_gamma(inp, 0, 1, 2, 2)
    kf = (inp["k"][:, 0, 1].astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    K = (0.75 * kf * kf).mean(0)
    A = float(np.float32(0.9)) ** 2
    np.testing.assert_allclose(g, [orc.gamma_hat(A, float(x), 1) for x in K], rtol=1e-14)


def test_allocation_excess_invariances(sim):
    rng = np.random.default_rng(4)
    g = np.exp(rng.normal(0, 2, 256))
    assert sim.allocation_excess(g, g, 4.0, 1, 8)[2] == 0.0
    assert sim.allocation_excess(g, 7.5 * g, 4.0, 1, 8)[2] == 0.0          # allocation is scale-free
    be, ba, ex = sim.allocation_excess(g, g * np.exp(rng.normal(0, 1, 256)), 4.0, 1, 8)
    assert be.sum() == ba.sum() == 4 * 256 and ex > 0


def test_rounding_study_runs_and_is_consistent(sim):
    """A tiny study: the quantized run's readout equals the FP32 step from
    its own stored state (checked inside), the errors are bounded by half a
    step, and the readout ratio is a finite positive number."""
    w = synth.Workload("sim", B=1, H=2, d=32, T=48, s_min=1e-4, seed=5)
    r = sim.rounding_study(w, 48, 4, burn_in=8)
    assert np.all(np.isfinite(r["corr"])) and np.all(np.abs(r["corr"]) <= 1.0)
    ratio = r["readout"] / r["model"]
    assert np.all((ratio > 0.05) & (ratio < 20.0))
    assert r["s"].shape == (1, 2, 32) and np.all(r["s"] > 0)
