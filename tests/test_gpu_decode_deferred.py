"""GPU parity of decode with deferred write-back (write-back every C tokens,
the state between write-backs carried in FP32) against the oracle's run
with the same interval, through the C ABI.  The interval state keeps each
tier in the basis of the token arithmetic, exactly as the oracle's FP32
state between write-backs, so outputs, stored bytes and residuals are
expected identical."""
import numpy as np
import pytest

from bit_recurrent_state_b200 import synth
from parity import MODE, oracle_cfg, random_perm, to_dev

pytestmark = pytest.mark.gpu


def _interval_inputs(w, t0, C):
    toks = [synth.token_inputs(w, t) for t in range(t0, t0 + C)]
    return {k: np.stack([tk[k] for tk in toks]) for k in toks[0]}


def _run(w, C, T, perm=None, units=None, init_scale=0.05):
    import torch
    from bit_recurrent_state_b200 import brs
    from bit_recurrent_state_b200.state import LayerState
    from oracle import oracle as O

    assert T % C == 0
    cfg = oracle_cfg(w)
    L = brs.layout_of(w)
    wb = brs.writeback_of(w, C=C)
    st = LayerState(L, perm=perm)
    S0 = (np.random.default_rng(9).standard_normal((w.B, w.H, w.d, w.d)) * init_scale).astype(np.float32)
    st.pack(torch.from_numpy(S0).cuda())
    packed_o, _ = O.state_pack(cfg, S0, perm)
    _, aux_o, stats_o = O.new_state(cfg)
    s32 = torch.zeros(brs.decode_state32_bytes(L) // 4, dtype=torch.float32, device="cuda")
    o_gpu = torch.zeros((w.B, w.H, w.d), dtype=torch.float32, device="cuda")
    hb = packed_o.size // (w.B * w.H)
    sel = np.arange(w.B * w.H) if units is None else np.arange(*units)
    for t0 in range(0, T, C):
        og = []
        for t in range(t0, t0 + C):
            dev = to_dev(synth.token_inputs(w, t))
            brs.decode_step_deferred(L, wb, t, st.packed, st.aux, st.workspace, s32, st.perm, dev["q"], dev["k"],
                                     dev["v"], dev["beta"], dev["decay"], o_gpu)
            og.append(o_gpu.cpu().numpy().copy())
        oo, fl, _ = O.run_parallel(cfg, MODE[w.mode], w.seed, C, t0, _interval_inputs(w, t0, C), packed_o,
                                   aux=aux_o, stats=stats_o, perm=perm, units=units)
        assert fl == 0
        for c in range(C):
            g = og[c].reshape(w.B * w.H, w.d)[sel]
            r = oo[c].reshape(w.B * w.H, w.d)[sel]
            np.testing.assert_array_equal(g.view(np.uint32), r.view(np.uint32), err_msg=f"o of token {t0 + c}")
        pg = st.packed.cpu().numpy().reshape(w.B * w.H, hb)[sel]
        np.testing.assert_array_equal(pg, packed_o.reshape(w.B * w.H, hb)[sel], err_msg=f"state after {t0 + C}")
        if w.mode == "errfeedback":
            ag = st.aux.cpu().numpy()[: aux_o.nbytes]
            per = ag.size // (w.B * w.H)
            np.testing.assert_array_equal(ag.reshape(w.B * w.H, per)[sel],
                                          aux_o.view(np.uint8).reshape(w.B * w.H, per)[sel])
    assert st.errors() == 0


@pytest.mark.parametrize("name,C,kw", [
    ("kda128_c2", 2, dict(B=2, H=3, d=128, k_hi=16, block=128)),
    ("kda128_c8", 8, dict(B=2, H=3, d=128, k_hi=16, block=128)),
    ("kda128_b32_sr_c4", 4, dict(B=2, H=2, d=128, k_hi=16, block=32, mode="stochastic")),
    ("kda128_ef_c4", 4, dict(B=2, H=3, d=128, k_hi=16, block=128, mode="errfeedback")),
    ("kda64_c3", 3, dict(B=2, H=3, d=64, k_hi=8, block=64)),
    ("kda32_nohad_c2", 2, dict(B=2, H=2, d=32, k_hi=4, block=32, hadamard=0)),
    ("gdn128_c4", 4, dict(B=3, H=4, Hk=2, d=128, k_hi=0, block=128, decay_per_key=0)),
    ("kda128_int4_c4", 4, dict(B=2, H=3, d=128, k_hi=16, block=128, low_bits=4)),
    ("kda32_int4_ef_c3", 3, dict(B=2, H=2, d=32, k_hi=4, block=32, mode="errfeedback", low_bits=4)),
])
def test_deferred_small_bit_exact(name, C, kw):
    w = synth.Workload(name, T=2 * C, seed=11, **kw)
    _run(w, C, 2 * C, perm=random_perm(w, seed=4))


def test_deferred_c1_is_decode_step():
    """C = 1 through the deferred entry is the ordinary decode step (the
    interval state is not touched and may be absent)."""
    w = synth.Workload("c1", B=2, H=3, d=128, k_hi=16, block=128, T=3, seed=2)
    _run(w, 1, 3, perm=random_perm(w, seed=1))


def test_deferred_kda_decode_full_size_sampled():
    """The KDA decode configuration (B=64, H=32, d=128) with write-back every
    8 tokens for 16 tokens; the oracle runs 64 of the 2048 heads."""
    w = synth.WORKLOADS["kda_decode"]
    _run(w, 8, 16, perm=random_perm(w, seed=5), units=(1000, 1064), init_scale=0.0)
