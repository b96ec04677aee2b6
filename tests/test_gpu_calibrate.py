"""GPU parity of the protected-row selection (brs_calibrate) against the
oracle's calibration: the permutation must be identical and the FP64 scores
within 1e-12 relative.  Both sides sum in the same order; the FP32
recurrence is bit-identical; only the library log/exp of the mean decay
may differ in the last bit.  Where two scores of a head are that close, the
test accepts either order (both selections are valid)."""
import numpy as np
import pytest

from bit_recurrent_state_b200 import synth
from parity import oracle_cfg, to_dev

pytestmark = pytest.mark.gpu
RTOL = 1e-12


def _gpu_calibrate(w, inp, every, tau):
    import torch
    from bit_recurrent_state_b200 import brs
    L = brs.layout_of(w)
    T, Bc = inp["q"].shape[0], inp["q"].shape[1]
    nb = brs.calibrate_workspace_bytes(L, Bc, T, every)
    ws = torch.zeros(nb, dtype=torch.uint8, device="cuda")
    perm = torch.zeros((w.H, w.d), dtype=torch.int16, device="cuda")
    score = torch.zeros((w.H, w.d), dtype=torch.float64, device="cuda")
    dev = to_dev(inp)
    brs.calibrate(L, Bc, T, every, tau, dev["q"], dev["k"], dev["v"], dev["beta"], dev["decay"], ws, perm,
                  score_out=score)
    assert brs.fetch_errors(ws) == 0
    return perm.cpu().numpy(), score.cpu().numpy()


def _oracle_calibrate(w, inp, every, tau):
    from oracle import oracle as O
    return O.calibrate(oracle_cfg(w), inp, every=every, tau=tau)


def _compare(perm_g, score_g, perm_o, score_o, k_hi):
    np.testing.assert_allclose(score_g, score_o, rtol=RTOL, atol=0)
    d = perm_o.shape[1]
    for h in range(perm_o.shape[0]):
        assert sorted(perm_g[h]) == list(range(d))
        if np.array_equal(perm_g[h], perm_o[h]):
            continue
        # a near-tie at the k_hi-th score: both protected sets must be valid
        prot_g, prot_o = set(perm_g[h, d - k_hi:]), set(perm_o[h, d - k_hi:])
        kth = np.sort(score_o[h])[::-1][k_hi - 1]
        for u in prot_g ^ prot_o:
            assert abs(score_o[h, u] - kth) <= 4 * RTOL * abs(kth), (h, u)


@pytest.mark.parametrize("name,kw,Bc,T,every", [
    ("kda32", dict(B=1, H=2, d=32, k_hi=4, block=32), 4, 32, 8),
    ("kda64_b16_nohad", dict(B=1, H=3, d=64, k_hi=8, block=16, hadamard=0), 3, 40, 8),
    ("gdn128", dict(B=1, H=4, Hk=2, d=128, k_hi=16, block=128, decay_per_key=0), 4, 48, 8),
    ("kda128_every5", dict(B=1, H=2, d=128, k_hi=24, block=32), 2, 33, 5),
    ("kda128_int4", dict(B=1, H=2, d=128, k_hi=16, block=32, low_bits=4), 2, 24, 8),
    ("kda32_int4_nohad", dict(B=1, H=2, d=32, k_hi=4, block=16, hadamard=0, low_bits=4), 3, 24, 6),
])
def test_small_configs(name, kw, Bc, T, every):
    w = synth.Workload(name, T=1, seed=11, **kw)
    inp = synth.calibration_inputs(w, batch=Bc, tokens=T)
    pg, sg = _gpu_calibrate(w, inp, every, 1e-3)
    po, so = _oracle_calibrate(w, inp, every, 1e-3)
    _compare(pg, sg, po, so, w.k_hi)


def test_tau_binds():
    """Slow decays (1 - a^2 below tau) take the cap on both sides."""
    w = synth.Workload("kda32_tau", B=1, H=2, d=32, T=1, k_hi=4, block=32, seed=12)
    inp = synth.calibration_inputs(w, batch=2, tokens=16)
    inp["decay"][..., :8] = np.float32(1.0 - 1e-5)
    pg, sg = _gpu_calibrate(w, inp, 8, 1e-2)
    po, so = _oracle_calibrate(w, inp, 8, 1e-2)
    _compare(pg, sg, po, so, w.k_hi)


def test_kda_decode_full_calibration_sampled_heads():
    """The KDA decode layer's calibration (H=32, d=128, 16 protected rows,
    32 sequences x 256 tokens, a sample every 8 tokens) in one GPU call; the
    oracle recomputes the first 4 heads (heads are scored independently)."""
    w = synth.WORKLOADS["kda_decode"]
    inp = synth.calibration_inputs(w, batch=32, tokens=256)
    pg, sg = _gpu_calibrate(w, inp, 8, 1e-3)
    nh = 4
    sub = {key: np.ascontiguousarray(val[:, :, :nh]) for key, val in inp.items()}
    ws = w.with_(H=nh)
    po, so = _oracle_calibrate(ws, sub, 8, 1e-3)
    _compare(pg[:nh], sg[:nh], po, so, w.k_hi)
