"""GPU parity of the per-head variable-width decode step (one width per
head, FP16 steps per block of 32 key channels and column) against the
oracle, through the C ABI.  Teacher-forced: every step starts from the
oracle's stored state.  Widths, steps, codes, residuals and statistics must
be identical except for heads whose width sits on a rounding point of the
FP64 allocation (b* at a half-integer), where the two math libraries may
differ in the last bit (counted, must stay rare); outputs within 2e-3 x RMS
(expected identical)."""
import numpy as np
import pytest

from bit_recurrent_state_b200 import synth
from parity import MODE, oracle_cfg, to_dev
from ref64 import varbit_head_codes, varbit_head_sections

pytestmark = pytest.mark.gpu


def _vh_workload(**kw):
    base = dict(B=2, H=8, Hk=4, d=128, T=6, storage="varbit_head", hadamard=0, avg_bits=4.0, b_min=2,
                b_max=8, decay_per_key=0, seed=70)
    base.update(kw)
    return synth.Workload("vh", **base)


def _gpu_state(w, packed_np, aux_np, stats_np):
    import torch
    from bit_recurrent_state_b200 import brs
    from bit_recurrent_state_b200.state import LayerState
    st = LayerState(brs.layout_of(w))
    st.packed.copy_(torch.from_numpy(packed_np))
    st.aux.copy_(torch.from_numpy(np.pad(aux_np.view(np.uint8), (0, st.aux.numel() - aux_np.nbytes))))
    st.stats.copy_(torch.from_numpy(np.pad(stats_np.view(np.uint8), (0, st.stats.numel() - stats_np.nbytes))))
    return st


def _compare_step(w, pg, po, og, oo, tag, seqs=None):
    B, H, d = w.B, w.H, w.d
    payg, scg, wdg, ofg = varbit_head_sections(pg, B, H, d, w.avg_bits)
    payo, sco, wdo, ofo = varbit_head_sections(po, B, H, d, w.avg_bits)
    flips = 0
    for b in (range(B) if seqs is None else seqs):
        assert int(wdg[b].astype(int).sum()) == int(w.avg_bits * H)
        np.testing.assert_array_equal(ofg[b], np.concatenate([[0], np.cumsum(wdg[b].astype(np.int64))]) * (d * d // 8))
        for h in range(H):
            if wdg[b, h] != wdo[b, h]:
                flips += 1
                continue
            np.testing.assert_array_equal(scg[b, h], sco[b, h], err_msg=f"{tag} steps b={b} h={h}")
            cg = varbit_head_codes(payg[b], int(ofg[b, h]), int(wdg[b, h]), d)
            co = varbit_head_codes(payo[b], int(ofo[b, h]), int(wdo[b, h]), d)
            np.testing.assert_array_equal(cg, co, err_msg=f"{tag} codes b={b} h={h}")
        sel = slice(b * H, (b + 1) * H)
        og_b, oo_b = og.reshape(B * H, d)[sel], oo.reshape(B * H, d)[sel]
        tol = 2e-3 * float(np.sqrt(np.mean(oo_b.astype(np.float64) ** 2)))
        assert np.max(np.abs(og_b - oo_b)) <= tol, tag
    return flips


def _teacher_forced(w, T, seqs=None, inputs=None):
    import torch
    from bit_recurrent_state_b200 import brs
    from oracle import oracle as O
    cfg = oracle_cfg(w)
    packed_o, aux_o, stats_o = O.new_state(cfg)
    L = brs.layout_of(w)
    wb = brs.writeback_of(w)
    flips = 0
    o = torch.zeros((w.B, w.H, w.d), device="cuda")
    units = None if seqs is None else (seqs[0], seqs[-1] + 1)
    for t in range(T):
        inp = synth.token_inputs(w, t) if inputs is None else inputs(t)
        st = _gpu_state(w, packed_o, aux_o, stats_o)
        out = torch.zeros_like(st.packed)
        dev = to_dev(inp)
        brs.decode_step(L, wb, t, st.packed, out, st.aux, st.stats, st.workspace, None, dev["q"], dev["k"],
                        dev["v"], dev["beta"], dev["decay"], o)
        assert st.errors() == 0
        oo, fl, _ = O.run_parallel(cfg, MODE[w.mode], w.seed, 1, t, {k: v[None] for k, v in inp.items()},
                                   packed_o, aux=aux_o, stats=stats_o, units=units)
        assert fl == 0
        flips += _compare_step(w, out.cpu().numpy(), packed_o, o.cpu().numpy(), oo[0], f"{w.mode} t={t}", seqs)
        sg = st.stats.cpu().numpy()[: stats_o.nbytes].view(np.float64).reshape(w.B, -1)
        so = stats_o.reshape(w.B, -1)
        sl = slice(None) if seqs is None else slice(seqs[0], seqs[-1] + 1)
        np.testing.assert_array_equal(sg[sl], so[sl])
        if w.mode == "errfeedback" and flips == 0:
            ag = st.aux.cpu().numpy()[: aux_o.nbytes].view(np.uint16).reshape(w.B, -1)
            np.testing.assert_array_equal(ag[sl], aux_o.reshape(w.B, -1)[sl])
    return flips


@pytest.mark.parametrize("mode,b_min,b_max,avg,pers,per_key", [
    ("nearest", 2, 8, 4.0, 0, 0), ("stochastic", 2, 8, 4.0, 0, 0), ("errfeedback", 2, 8, 4.0, 0, 0),
    ("nearest", 2, 16, 6.0, 0, 0), ("stochastic", 2, 16, 6.0, 0, 0), ("nearest", 2, 8, 2.0, 0, 0),
    ("nearest", 2, 8, 3.0, 2, 0), ("errfeedback", 2, 8, 4.0, 1, 1)])
def test_varbit_head_teacher_forced(mode, b_min, b_max, avg, pers, per_key):
    """GDN heads (one decay per head) and, last, KDA heads (decay per key,
    the head's cost the mean of its rows' weights); widths up to 16 bits (a
    code spanning two words); the two-bit mean (every head at two bits)."""
    w = _vh_workload(mode=mode, b_min=b_min, b_max=b_max, avg_bits=avg, persistence=pers,
                     decay_per_key=per_key, Hk=4 if not per_key else 8)
    assert _teacher_forced(w, w.T) <= 2


def test_varbit_head_gdn_decode_size_sampled():
    """The GDN decode size (B=256, H=32, H_k=16, d=128, 4.0 bits, widths
    2..8) for 8 tokens; the oracle follows 4 of the 256 sequences (128 heads)
    whose stored bytes, statistics and outputs must match."""
    w = synth.WORKLOADS["gdn_varbit_decode"]
    assert _teacher_forced(w, 8, seqs=[100, 101, 102, 103]) <= 2


@pytest.mark.parametrize("b_max", [8, 16])
def test_varbit_head_pack_unpack_match_oracle(b_max):
    import torch
    from bit_recurrent_state_b200 import brs
    from bit_recurrent_state_b200.state import LayerState
    from oracle import oracle as O
    w = _vh_workload(b_max=b_max)
    cfg = oracle_cfg(w)
    rng = np.random.default_rng(4)
    S = (rng.standard_normal((w.B, w.H, w.d, w.d)) * rng.uniform(0.01, 2, (w.B, w.H, 1, w.d))).astype(np.float32)
    widths = np.full((w.B, w.H), 4, np.int64)
    for b in range(w.B):
        for _ in range(200):
            i, j = rng.integers(w.H, size=2)
            if widths[b, i] < b_max and widths[b, j] > 2 and i != j:
                widths[b, i] += 1
                widths[b, j] -= 1
    widths = widths.astype(np.uint8)
    st = LayerState(brs.layout_of(w))
    st.pack(torch.from_numpy(S).cuda(), widths=torch.from_numpy(widths).cuda())
    assert st.errors() == 0
    po, fl = O.state_pack(cfg, S, None, widths)
    assert fl == 0
    np.testing.assert_array_equal(st.packed.cpu().numpy(), po)
    Sg = st.unpack().cpu().numpy()
    So, _ = O.state_unpack(cfg, po)
    np.testing.assert_array_equal(Sg.view(np.uint32), So.view(np.uint32))


def test_varbit_head_pack_rejects_widths_off_budget():
    """A width map whose total is not avg_bits * H stores nothing for that
    sequence and raises the invalid-argument flag."""
    import torch
    from bit_recurrent_state_b200 import brs
    from bit_recurrent_state_b200.state import LayerState
    w = _vh_workload(B=1)
    st = LayerState(brs.layout_of(w))
    widths = torch.full((1, w.H), 4, dtype=torch.uint8, device="cuda")
    widths[0, 0] = 9
    st.pack(torch.zeros((1, w.H, w.d, w.d), device="cuda"), widths=widths)
    assert st.errors() & brs.FLAG_INVALID
    _, _, wd, _ = varbit_head_sections(st.packed.cpu().numpy(), 1, w.H, w.d, w.avg_bits)
    assert np.all(wd == 0)
