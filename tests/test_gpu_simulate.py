"""The synthetic write-back studies on the GPU (bit_recurrent_state_b200.
simulate: trajectories from the library's kernels, FP64 statistics in torch)
against the same studies computed from the oracle (oracle/simulate.py).
The trajectories are bit-identical, so the statistics agree to FP64
reduction order; the allocator's widths are identical."""
import numpy as np
import pytest

from bit_recurrent_state_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("bits,persistent", [(4, 0), (3, 1), (6, 0)])
def test_rounding_study_matches_oracle(bits, persistent):
    from bit_recurrent_state_b200 import simulate as G
    from oracle import simulate as S
    w = synth.Workload("sim", B=1, H=2, d=128, T=40, s_min=1e-4, persistent_keys=persistent, seed=9)
    g = G.rounding_study(w, 40, bits, burn_in=8)
    o = S.rounding_study(w, 40, bits, burn_in=8)
    np.testing.assert_allclose(g["s"], o["s"], rtol=1e-12)
    np.testing.assert_allclose(g["corr"], o["corr"], rtol=1e-9, atol=1e-12)
    np.testing.assert_allclose(g["readout"], o["readout"], rtol=1e-12)
    np.testing.assert_allclose(g["model"], o["model"], rtol=1e-9)


@pytest.mark.parametrize("persistent", [0, 1])
def test_erasure_study_matches_oracle(persistent):
    from bit_recurrent_state_b200 import simulate as G
    from oracle import simulate as S
    w = synth.Workload("sim_erasure", B=1, H=2, d=64, T=700, s_min=1e-2, persistent_keys=persistent, seed=13)
    starts, lags = [0, 150, 299], 400
    g = G.erasure_study(w, 700, starts, lags, avg_bits=4.0, b_min=1, b_max=8)
    inp = synth.run_inputs(w, 0, 700)
    gam = np.stack([S.gramian_diag(S.transitions(inp, 0, h, 2, 2), starts, lags) for h in range(2)])
    ghat = np.stack([S.approx_gamma(inp, 0, h, 2, 2) for h in range(2)])
    np.testing.assert_allclose(g["gamma"], gam, rtol=1e-9)
    np.testing.assert_allclose(g["gamma_hat"], ghat, rtol=1e-12)
    be, ba, ex = S.allocation_excess(gam.ravel(), ghat.ravel(), 4.0, 1, 8)
    np.testing.assert_array_equal(g["bits_exact"], be)
    np.testing.assert_array_equal(g["bits_approx"], ba)
    assert g["excess"] == pytest.approx(ex, rel=1e-9, abs=1e-12)
