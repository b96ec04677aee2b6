"""GPU parity of the chunked prefill (WY form, write-back once per 64-token
chunk) against the oracle's token-by-token recurrence, teacher-forced per
chunk: both start every chunk from the same stored state.  Outputs and the
pre-write-back state within 2e-3 x RMS; the stored codes equal the oracle
quantizer applied to the GPU's own pre-write-back state (replay)."""
import numpy as np
import pytest

from bit_recurrent_state_b200 import synth
from oracle import oracle as O
from parity import MODE, random_perm

pytestmark = pytest.mark.gpu


def _tok_major(inp):
    """[B][T][...] -> [T][B][...] for the oracle."""
    return {k: np.ascontiguousarray(np.swapaxes(v, 0, 1)) for k, v in inp.items()}


def _seq_major(w, t0, T):
    """Inputs of tokens [t0, t0+T) laid out [B][T][...] for the prefill call."""
    r = synth.run_inputs(w, t0, T)
    return {k: np.ascontiguousarray(np.swapaxes(v, 0, 1)) for k, v in r.items()}


def _dev(a):
    import torch
    a = np.ascontiguousarray(a)
    return torch.from_numpy(a.view(np.int16) if a.dtype == np.uint16 else a).cuda()


def _run_chunks(w, nchunks, units=None, mode="nearest"):
    import torch
    from bit_recurrent_state_b200 import brs
    from bit_recurrent_state_b200.state import LayerState
    perm = random_perm(w, seed=11)
    cfg = O.Config(B=w.B, H=w.H, Hk=w.hk, d=w.d, storage=O.STORE_DAMP, k_hi=w.k_hi, block=w.block,
                   hadamard=w.hadamard, decay_per_key=w.decay_per_key, low_bits=w.low_bits,
                   domain=O.DOMAIN_CANONICAL)
    L, wb = brs.layout_of(w), brs.writeback_of(w, C=64, mode=brs.MODES[mode])
    rng = np.random.default_rng(5)
    S0 = (rng.standard_normal((w.B, w.H, w.d, w.d)) * 0.05).astype(np.float32)
    packed_o, _ = O.state_pack(cfg, S0, perm)
    _, aux_o, _ = O.new_state(cfg)
    st = LayerState(L, perm=perm)
    hb = packed_o.size // (w.B * w.H)
    sel = np.arange(w.B * w.H) if units is None else np.arange(*units)
    for c in range(nchunks):
        t0 = 64 * c
        inp = _seq_major(w, t0, 64)
        st.packed.copy_(torch.from_numpy(packed_o))
        st.aux.copy_(torch.from_numpy(np.pad(aux_o.view(np.uint8), (0, st.aux.numel() - aux_o.nbytes))))
        before_p, before_a = packed_o.copy(), aux_o.copy()
        o = torch.zeros((w.B, 64, w.H, w.d), device="cuda")
        dump = torch.zeros((w.B, w.H, w.d, w.d), device="cuda")
        d = {k: _dev(v) for k, v in inp.items()}
        st.prefill(wb, t0, 64, d["q"], d["k"], d["v"], d["beta"], d["decay"], o, state_dump=dump)
        assert st.errors() == 0
        og = o.cpu().numpy()
        sg = dump.cpu().numpy()
        pg = st.packed.cpu().numpy()
        oo, fl, _, so = O.run(cfg, MODE[mode], w.seed, 64, t0, _tok_major(inp), packed_o, aux=aux_o,
                              perm=perm, units=units, dump_s=True)
        assert fl == 0
        # outputs and pre-write-back state, over the compared heads
        og_u = np.swapaxes(og, 1, 2).reshape(w.B * w.H, 64, w.d)[sel]
        oo_u = np.swapaxes(oo, 0, 1).swapaxes(1, 2).reshape(w.B * w.H, 64, w.d)[sel]
        rms_o = np.sqrt(np.mean(oo_u.astype(np.float64) ** 2))
        assert np.max(np.abs(og_u - oo_u)) <= 2e-3 * rms_o, (c, np.max(np.abs(og_u - oo_u)) / rms_o)
        sg_u = sg.reshape(w.B * w.H, w.d, w.d)[sel]
        so_u = so.reshape(w.B * w.H, w.d, w.d)[sel]
        rms_s = np.sqrt(np.mean(so_u.astype(np.float64) ** 2))
        assert np.max(np.abs(sg_u - so_u)) <= 2e-3 * rms_s, (c, np.max(np.abs(sg_u - so_u)) / rms_s)
        # replay: the oracle's write-back (mode, seed, step, residuals) of the
        # GPU's own pre-write-back state gives the GPU's codes and residuals
        fl = O.damp_writeback(cfg, MODE[mode], w.seed, t0 + 63, sg, before_p, before_a)
        assert fl == 0
        np.testing.assert_array_equal(pg.reshape(w.B * w.H, hb)[sel], before_p.reshape(w.B * w.H, hb)[sel])
        if mode == "errfeedback":
            ag = st.aux.cpu().numpy()[: aux_o.nbytes].view(np.uint16)
            np.testing.assert_array_equal(ag, before_a)


@pytest.mark.parametrize("kw,mode", [
    (dict(B=2, H=3, d=128, k_hi=16, block=128), "nearest"),
    (dict(B=1, H=2, d=128, k_hi=16, block=32), "nearest"),
    (dict(B=2, H=4, Hk=2, d=128, k_hi=0, block=128, decay_per_key=0), "nearest"),
    (dict(B=1, H=2, d=128, k_hi=16, block=128), "errfeedback"),
    (dict(B=1, H=2, d=128, k_hi=16, block=128), "stochastic"),
    # the 4-bit low tier
    (dict(B=2, H=3, d=128, k_hi=16, block=128, low_bits=4), "nearest"),
    (dict(B=1, H=2, d=128, k_hi=16, block=32, low_bits=4), "errfeedback"),
    (dict(B=1, H=2, d=128, k_hi=0, block=128, decay_per_key=0, low_bits=4), "stochastic"),
])
def test_prefill_teacher_forced(kw, mode):
    w = synth.Workload("pf", T=192, C=64, seed=60, **kw)
    _run_chunks(w, 3, mode=mode)


@pytest.mark.parametrize("kw,mode,ctas", [
    (dict(B=2, H=3, d=128, k_hi=16, block=128), "nearest", 0),
    (dict(B=1, H=4, Hk=2, d=128, k_hi=0, block=128, decay_per_key=0), "nearest", 0),
    (dict(B=1, H=2, d=128, k_hi=16, block=32), "errfeedback", 0),
    (dict(B=2, H=3, d=128, k_hi=16, block=128), "nearest", 5),
    (dict(B=2, H=3, d=128, k_hi=16, block=128), "stochastic", 4),
    (dict(B=1, H=4, Hk=2, d=128, k_hi=0, block=128, decay_per_key=0), "nearest", 3),
    (dict(B=1, H=2, d=128, k_hi=16, block=32), "errfeedback", 1),
    (dict(B=2, H=3, d=128, k_hi=16, block=128, low_bits=4), "nearest", 4),
])
def test_prefill_multi_chunk_one_launch(kw, mode, ctas):
    """Four chunks in ONE launch (the chunk-to-chunk hand-over inside the
    kernel) equal, bit for bit, four one-chunk launches (each of which the
    teacher-forced tests compare with the oracle): the same outputs, the same
    stored state and residuals, the same state before the last write-back.
    With the CTAs capped below the heads (`ctas`), the one launch cuts heads
    between CTAs, which hand them over through the scratch state."""
    import torch
    from bit_recurrent_state_b200 import brs
    from bit_recurrent_state_b200.state import LayerState
    brs.test_prefill_ctas(ctas)
    try:
        _multi_chunk_compare(kw, mode)
    finally:
        brs.test_prefill_ctas(0)


def _multi_chunk_compare(kw, mode):
    import torch
    from bit_recurrent_state_b200 import brs
    from bit_recurrent_state_b200.state import LayerState
    w = synth.Workload("pf1", T=256, C=64, seed=61, **kw)
    perm = random_perm(w, seed=12)
    cfg = O.Config(B=w.B, H=w.H, Hk=w.hk, d=w.d, storage=O.STORE_DAMP, k_hi=w.k_hi, block=w.block,
                   hadamard=w.hadamard, decay_per_key=w.decay_per_key, low_bits=w.low_bits,
                   domain=O.DOMAIN_CANONICAL)
    L, wb = brs.layout_of(w), brs.writeback_of(w, C=64, mode=brs.MODES[mode])
    S0 = (np.random.default_rng(6).standard_normal((w.B, w.H, w.d, w.d)) * 0.05).astype(np.float32)
    packed0, _ = O.state_pack(cfg, S0, perm)
    inp = _seq_major(w, 0, w.T)
    d = {k: _dev(v) for k, v in inp.items()}
    runs = []
    for chunked in (False, True):
        st = LayerState(L, perm=perm)
        st.packed.copy_(torch.from_numpy(packed0))
        o = torch.zeros((w.B, w.T, w.H, w.d), device="cuda")
        dump = torch.zeros((w.B, w.H, w.d, w.d), device="cuda")
        spans = [(c * 64, 64) for c in range(w.T // 64)] if chunked else [(0, w.T)]
        for t0, T in spans:
            dc = {k: v[:, t0:t0 + T].contiguous() for k, v in d.items()}
            oc = torch.zeros((w.B, T, w.H, w.d), device="cuda")
            st.prefill(wb, t0, T, dc["q"], dc["k"], dc["v"], dc["beta"], dc["decay"], oc, state_dump=dump)
            o[:, t0:t0 + T] = oc
        assert st.errors() == 0
        runs.append((o.cpu().numpy(), st.packed.cpu().numpy(), st.aux.cpu().numpy(), dump.cpu().numpy()))
    for a, b in zip(runs[0], runs[1]):
        np.testing.assert_array_equal(a.view(np.uint8), b.view(np.uint8))


def test_handover_wait_runs_out():
    """With the hand-over withheld and the CTAs capped below the heads, every
    CTA that continues a cut head waits out its bound, the call reports
    BRS_ETIMEOUT through the flag word, and the next call (hand-over on) is
    correct again: it equals the same launch on a fresh state bit for bit."""
    import torch
    from bit_recurrent_state_b200 import brs
    from bit_recurrent_state_b200.state import LayerState
    w = synth.Workload("pfw", B=1, H=3, d=128, T=256, C=64, k_hi=16, block=128, seed=62)
    perm = random_perm(w, seed=13)
    L, wb = brs.layout_of(w), brs.writeback_of(w, C=64, mode=brs.ROUND_NEAREST)
    d = {k: _dev(v) for k, v in _seq_major(w, 0, w.T).items()}

    def run(withhold):
        st = LayerState(L, perm=perm)
        st.zero()
        o = torch.zeros((w.B, w.T, w.H, w.d), device="cuda")
        brs.test_prefill_ctas(2)                      # 3 heads of 4 chunks on 2 CTAs: head 1 is cut
        brs.test_prefill_withhold(withhold)
        try:
            st.prefill(wb, 0, w.T, d["q"], d["k"], d["v"], d["beta"], d["decay"], o)
            fl = st.errors()
        finally:
            brs.test_prefill_withhold(False)
            brs.test_prefill_ctas(0)
        return fl, o.cpu().numpy(), st.packed.cpu().numpy()

    fl, _, _ = run(True)
    assert fl & brs.FLAG_TIMEOUT
    fl1, o1, p1 = run(False)
    fl2, o2, p2 = run(False)
    assert fl1 == 0 and fl2 == 0
    np.testing.assert_array_equal(o1.view(np.uint32), o2.view(np.uint32))
    np.testing.assert_array_equal(p1, p2)
