"""Pin of the DAMP protected-row selection against an FP64 recomputation of
the risk score C_u = E_u * P_u."""
import numpy as np

from bit_recurrent_state_b200 import synth
from ref64 import dense_step, hadamard_n, int8_nearest64, token_vectors


def test_calibration_matches_fp64_score(orc):
    d, H, k_hi, block = 16, 2, 4, 16
    w = synth.Workload("t", B=1, H=H, d=d, T=1, k_hi=k_hi, block=block, seed=40)
    Bc, T, every = 4, 32, 8
    inp = synth.calibration_inputs(w, batch=Bc, tokens=T)
    cfg = orc.Config(B=1, H=H, d=d, storage=orc.STORE_DAMP, k_hi=k_hi, block=block)
    perm, score = orc.calibrate(cfg, inp, every=every, tau=1e-3)
    Hn = hadamard_n(d)
    ident = np.arange(d)
    for h in range(H):
        E = np.zeros(d)
        n = 0
        for b in range(Bc):
            S = np.zeros((d, d))
            for t in range(T):
                k, q, v, a, beta = token_vectors(inp, t, b, h, H, H, ident, True)
                S, _ = dense_step(S, k, q, v, a, beta)
                if (t + 1) % every == 0:
                    n += 1
                    R = S @ Hn
                    for u in range(d):
                        c, s, z, _ = int8_nearest64(R[u])
                        E[u] += np.sum((R[u] - (c * s + z)) ** 2)
        a_eff = np.exp(np.mean(np.log(inp["decay"][:, :, h].astype(np.float64)), axis=(0, 1)))
        P = 1.0 / np.maximum(1.0 - a_eff ** 2, 1e-3)
        C = E / n * P
        np.testing.assert_allclose(score[h], C, rtol=1e-3)
        top = set(np.argsort(-C, kind="stable")[:k_hi])
        assert set(perm[h, d - k_hi:]) == top            # protected rows last
        assert list(perm[h, d - k_hi:]) == sorted(perm[h, d - k_hi:])
        assert list(perm[h, :d - k_hi]) == sorted(perm[h, :d - k_hi])
        assert sorted(perm[h]) == list(range(d))


def test_calibration_protects_persistent_high_error_rows(orc):
    """A row that decays slowly (P large) outranks an equally noisy fast one."""
    d, H, k_hi = 16, 1, 2
    w = synth.Workload("t", B=1, H=H, d=d, T=1, k_hi=k_hi, block=16, seed=41)
    inp = synth.calibration_inputs(w, batch=2, tokens=64)
    inp["decay"][:] = np.float32(np.exp(-1.0))
    inp["decay"][..., 5] = np.float32(np.exp(-1e-3))
    inp["decay"][..., 9] = np.float32(np.exp(-2e-3))
    cfg = orc.Config(B=1, H=H, d=d, storage=orc.STORE_DAMP, k_hi=k_hi, block=16)
    perm, _ = orc.calibrate(cfg, inp)
    assert list(perm[0, d - 2:]) == [5, 9]
