"""GPU parity of the variable-width (decay-aware allocation) decode step
against the oracle, through the C ABI.  Teacher-forced: every step starts
from the oracle's stored state.  Widths, FP16 steps, codes, residuals and
statistics must be identical except for rows whose width sits on a rounding
point of the FP64 allocation (b* within 1e-9 of a half-integer), where the
two math libraries may differ in the last bit (counted, must stay rare);
outputs within 2e-3 x RMS (expected identical)."""
import numpy as np
import pytest

from bit_recurrent_state_b200 import synth
from parity import MODE, oracle_cfg, to_dev
from ref64 import varbit_row_codes, varbit_sections

pytestmark = pytest.mark.gpu


def _vb_workload(**kw):
    base = dict(B=2, H=4, d=128, T=5, storage="varbit", hadamard=0, avg_bits=4.0, b_min=2, b_max=8, seed=50)
    base.update(kw)
    return synth.Workload("vb", **base)


def _gpu_state(w, scope, packed_np, aux_np, stats_np):
    import torch
    from bit_recurrent_state_b200 import brs
    from bit_recurrent_state_b200.state import LayerState
    L = brs.layout_of(w, budget_scope=scope)
    st = LayerState(L)
    st.packed.copy_(torch.from_numpy(packed_np))
    st.aux.copy_(torch.from_numpy(np.pad(aux_np.view(np.uint8), (0, st.aux.numel() - aux_np.nbytes))))
    st.stats.copy_(torch.from_numpy(np.pad(stats_np.view(np.uint8), (0, st.stats.numel() - stats_np.nbytes))))
    return st


def _compare_step(w, cfg, pg, po, og, oo, tag, seqs=None):
    B, H, d = w.B, w.H, w.d
    payg, scg, wdg, ofg = varbit_sections(pg, B, H, d, w.avg_bits)
    payo, sco, wdo, ofo = varbit_sections(po, B, H, d, w.avg_bits)
    seqs = range(B) if seqs is None else seqs
    flips = 0
    for b in seqs:
        assert int(wdg[b].astype(int).sum()) == int(w.avg_bits * H * d)
        np.testing.assert_array_equal(ofg[b][:-1], np.concatenate([[0], np.cumsum(wdg[b].astype(np.int64))[:-1]]) * (d // 8))
        for r in range(H * d):
            if wdg[b, r] != wdo[b, r]:
                flips += 1
                continue
            assert scg[b, r] == sco[b, r], (tag, b, r)
            cg = varbit_row_codes(payg[b], int(ofg[b, r]), int(wdg[b, r]), d)
            co = varbit_row_codes(payo[b], int(ofo[b, r]), int(wdo[b, r]), d)
            np.testing.assert_array_equal(cg, co, err_msg=f"{tag} b={b} row={r}")
        sel = slice(b * H, (b + 1) * H)
        og_b, oo_b = og.reshape(B * H, d)[sel], oo.reshape(B * H, d)[sel]
        tol = 2e-3 * float(np.sqrt(np.mean(oo_b.astype(np.float64) ** 2)))
        assert np.max(np.abs(og_b - oo_b)) <= tol
    return flips


@pytest.mark.parametrize("mode,scope,b_min,b_max,avg,pers", [
    ("nearest", 1, 2, 8, 4.0, 0), ("stochastic", 1, 2, 8, 4.0, 0), ("errfeedback", 1, 2, 8, 4.0, 0),
    ("nearest", 0, 2, 8, 4.0, 0), ("nearest", 1, 2, 16, 6.0, 0), ("errfeedback", 1, 2, 16, 6.0, 0),
    ("stochastic", 0, 2, 16, 6.0, 0), ("nearest", 1, 1, 8, 2.0, 0), ("stochastic", 1, 1, 8, 2.0, 0),
    ("errfeedback", 1, 1, 8, 2.0, 0), ("nearest", 0, 1, 16, 3.0, 0), ("nearest", 1, 2, 8, 4.0, 1),
    ("stochastic", 0, 2, 8, 4.0, 2)])
def test_varbit_teacher_forced(mode, scope, b_min, b_max, avg, pers):
    """b_max = 16 as at C = 1: widths up to 16 bits, a lane's four codes
    spanning up to three words of the row payload; b_min = 1: one-bit rows
    (the sign times the row's mean absolute value)."""
    import torch
    from bit_recurrent_state_b200 import brs
    from oracle import oracle as O
    w = _vb_workload(mode=mode, b_min=b_min, b_max=b_max, avg_bits=avg, persistence=pers)
    cfg = oracle_cfg(w)
    cfg.budget_scope = scope
    packed_o, aux_o, stats_o = O.new_state(cfg)
    L = brs.layout_of(w, budget_scope=scope)
    wb = brs.writeback_of(w)
    flips = 0
    o = torch.zeros((w.B, w.H, w.d), device="cuda")
    for t in range(w.T):
        inp = synth.token_inputs(w, t)
        st = _gpu_state(w, scope, packed_o, aux_o, stats_o)
        out = torch.zeros_like(st.packed)
        dev = to_dev(inp)
        brs.decode_step(L, wb, t, st.packed, out, st.aux, st.stats, st.workspace, None, dev["q"], dev["k"],
                        dev["v"], dev["beta"], dev["decay"], o)
        assert st.errors() == 0
        oo, fl, _ = O.run(cfg, MODE[mode], w.seed, 1, t, {k: v[None] for k, v in inp.items()}, packed_o,
                          aux=aux_o, stats=stats_o)
        assert fl == 0
        flips += _compare_step(w, cfg, out.cpu().numpy(), packed_o, o.cpu().numpy(), oo[0], f"{mode} t={t}")
        np.testing.assert_array_equal(st.stats.cpu().numpy()[: stats_o.nbytes].view(np.float64), stats_o)
        if mode == "errfeedback" and flips == 0:
            np.testing.assert_array_equal(st.aux.cpu().numpy()[: aux_o.nbytes], aux_o.view(np.uint8))
    assert flips <= 2


@pytest.mark.parametrize("b_min,b_max", [(2, 8), (2, 16), (1, 8)])
def test_varbit_pack_unpack_match_oracle(b_min, b_max):
    import torch
    from bit_recurrent_state_b200 import brs
    from bit_recurrent_state_b200.state import LayerState
    from oracle import oracle as O
    w = _vb_workload(b_min=b_min, b_max=b_max)
    cfg = oracle_cfg(w)
    rng = np.random.default_rng(3)
    S = (rng.standard_normal((w.B, w.H, w.d, w.d)) * rng.uniform(0.01, 2, (w.B, w.H, w.d, 1))).astype(np.float32)
    # widths 2..b_max that fill the budget exactly: move bits between random rows
    widths = np.full((w.B, w.H * w.d), 4, np.int64)
    for b in range(w.B):
        for _ in range(3000):
            i, j = rng.integers(w.H * w.d, size=2)
            if widths[b, i] < b_max and widths[b, j] > b_min and i != j:
                widths[b, i] += 1
                widths[b, j] -= 1
    widths = widths.astype(np.uint8)
    st = LayerState(brs.layout_of(w))
    st.pack(torch.from_numpy(S).cuda(), widths=torch.from_numpy(widths).cuda())
    po, fl = O.state_pack(cfg, S, None, widths)
    assert fl == 0
    np.testing.assert_array_equal(st.packed.cpu().numpy(), po)
    Sg = st.unpack().cpu().numpy()
    So, _ = O.state_unpack(cfg, po)
    np.testing.assert_array_equal(Sg.view(np.uint32), So.view(np.uint32))
