"""Pins of the variable-width write-back (decay-aware allocation): layer
budget, offsets, FP64 recomputation of the widths and of the update."""
import math

import numpy as np
import pytest

from bit_recurrent_state_b200 import synth
from ref64 import bf16_to_f64, dense_step, f16_bits_to_f64, varbit_row_codes, varbit_sections


def _levels(codes, bw):
    """Stored codes -> integer levels: offset binary, or +-1 for one-bit rows."""
    codes = codes.astype(int)
    return 2 * codes - 1 if bw == 1 else codes - (2 ** (bw - 1) - 1)


@pytest.mark.parametrize("mode,b_min,b_max,avg,pers", [(0, 2, 8, 4.0, 0), (1, 2, 8, 4.0, 0), (2, 2, 8, 4.0, 0),
                                                       (0, 2, 16, 4.0, 0), (2, 2, 16, 4.0, 0),
                                                       (0, 1, 8, 2.0, 0), (1, 1, 8, 2.0, 0), (2, 1, 8, 2.0, 0),
                                                       (0, 2, 8, 4.0, 1), (0, 2, 8, 4.0, 2)])
def test_varbit_teacher_forced_fp64(orc, mode, b_min, b_max, avg, pers):
    """b_max = 8, and 16 as at C = 1 (widths up to 16 bits, codes that span
    words of the row payload); b_min = 1 with one-bit rows (the sign times
    the row's mean absolute value)."""
    B, H, d, T = 2, 2, 32, 6
    w = synth.Workload("t", B=B, H=H, d=d, T=T, storage="varbit", hadamard=0, seed=20 + mode)
    cfg = orc.Config(B=B, H=H, d=d, storage=orc.STORE_VARBIT, hadamard=0, avg_bits=avg,
                     b_min=b_min, b_max=b_max, budget_scope=1, persistence=pers)
    inp_all = synth.run_inputs(w, 0, T)
    packed, aux, stats = orc.new_state(cfg)
    lam = (1 - 2 / 65)
    K64 = np.zeros((B, H * d))
    near_ties = 0
    for t in range(T):
        before = packed.copy()
        inp = {k: v[t:t + 1] for k, v in inp_all.items()}
        o, fl, _ = orc.run(cfg, mode, 99, 1, t, inp, packed, aux=aux, stats=stats)
        assert fl == 0
        pay0, sc0, wd0, of0 = varbit_sections(before, B, H, d, avg)
        pay, sc, wd, of = varbit_sections(packed, B, H, d, avg)
        for b in range(B):
            assert int(wd[b].astype(int).sum()) == int(avg * H * d)       # layer budget
            np.testing.assert_array_equal(of[b][:-1], np.concatenate([[0], np.cumsum(wd[b].astype(int))[:-1]]) * (d // 8))
            Rr = np.zeros(H * d)
            S_new = np.zeros((H, d, d))
            for h in range(H):
                S = np.zeros((d, d))
                for i in range(d):
                    r = h * d + i
                    bw = int(wd0[b, r])
                    S[i] = _levels(varbit_row_codes(pay0[b], int(of0[b, r]), bw, d), bw) * f16_bits_to_f64(sc0[b, r])
                k, q, v, a, beta = (bf16_to_f64(inp["k"][0, b, h]), bf16_to_f64(inp["q"][0, b, h]),
                                    bf16_to_f64(inp["v"][0, b, h]),
                                    inp["decay"][0, b, h].astype(np.float64), float(inp["beta"][0, b, h]))
                S, oo = dense_step(S, k, q, v, a, beta)
                assert np.max(np.abs(o[0, b, h] - oo)) <= 1e-5 * (np.max(np.abs(oo)) + 1e-30)
                S_new[h] = S
                Rr[h * d:(h + 1) * d] = np.max(np.abs(S), axis=1)
                kk = beta * (2 - beta) * k ** 2
                K64[b, h * d:(h + 1) * d] = kk if t == 0 else lam * K64[b, h * d:(h + 1) * d] + (1 - lam) * kk
            # widths from an FP64 recomputation of c = Gamma_hat * R~^2
            a2 = np.concatenate([inp["decay"][0, b, h].astype(np.float64) ** 2 for h in range(H)])
            s_hat = -0.5 * np.log(a2)
            if pers == 0:
                arg = np.maximum(2 * (s_hat + 0.5 * K64[b]), 1e-9)
                gam = 1.0 / np.expm1(arg)
            else:                                       # w^(1), and h^(C) at C = 1
                gam = 1.0 / (1.0 - a2)
            rms = np.sqrt(np.mean(Rr.reshape(H, d) ** 2, axis=1))
            Rt = (Rr.reshape(H, d) / rms[:, None]).ravel()
            c = gam * Rt ** 2
            bits64, _ = orc.allocate_bits(c, avg, b_min, b_max)
            bstar = avg + 0.5 * np.log2(c / np.exp(np.mean(np.log(c))))
            diff = bits64 != wd[b]
            if diff.any():
                # only where b* sits next to a half-integer
                assert np.all(np.abs(np.abs(bstar[diff] - np.floor(bstar[diff])) - 0.5) < 1e-6)
                near_ties += int(diff.sum())
            # each row holds its nearest levels (deterministic) / adjacent ones (stochastic)
            for r in range(H * d):
                bw = int(wd[b, r])
                if bw != 1:
                    continue
                # one-bit rows: scale = the mean absolute value (FP16), code = sign
                x = S_new[r // d, r % d]
                mu = f16_bits_to_f64(sc[b, r])
                if mode != 2:                     # (error feedback quantizes x + residual)
                    m64 = float(np.mean(np.abs(x)))
                    assert abs(mu - m64) <= 2.0 ** -10 * m64 + 1e-12, (mu, m64)
                if mode == 0:
                    lv = _levels(varbit_row_codes(pay[b], int(of[b, r]), bw, d), 1)
                    clear = np.abs(x) > 1e-6 * np.max(np.abs(x))
                    np.testing.assert_array_equal(lv[clear], np.where(x[clear] >= 0, 1, -1))
            if mode == 0:
                for r in range(H * d):
                    bw = int(wd[b, r]); nl = 2 ** (bw - 1) - 1
                    if bw == 1:
                        continue
                    D = f16_bits_to_f64(sc[b, r])
                    qv = varbit_row_codes(pay[b], int(of[b, r]), bw, d).astype(int) - nl
                    x = S_new[r // d, r % d]
                    if D == 0:
                        assert np.all(qv == 0)
                        continue
                    # the nearest level lies among the neighbours of round(x / D)
                    qn = np.clip(np.rint(x / D), -nl, nl).astype(int)
                    cand = np.clip(qn[:, None] + np.array([-1, 0, 1])[None, :], -nl, nl)
                    best = np.min(np.abs(x[:, None] - cand * D), axis=1)
                    got = np.abs(x - qv * D)
                    assert np.all(got - best <= 1e-4 * D)
    assert near_ties <= 2


def test_varbit_head_scope_budget(orc):
    B, H, d, T = 1, 3, 32, 4
    w = synth.Workload("t", B=B, H=H, d=d, T=T, storage="varbit", hadamard=0, seed=30)
    cfg = orc.Config(B=B, H=H, d=d, storage=orc.STORE_VARBIT, hadamard=0, avg_bits=3.0,
                     b_min=2, b_max=8, budget_scope=0)
    packed, aux, stats = orc.new_state(cfg)
    o, fl, _ = orc.run(cfg, 0, 0, 1, 0, synth.run_inputs(w, 0, T), packed, aux=aux, stats=stats)
    assert fl == 0
    _, _, wd, _ = varbit_sections(packed, B, H, d, 3.0)
    for h in range(H):
        assert int(wd[0, h * d:(h + 1) * d].astype(int).sum()) == 3 * d


def test_varbit_pack_rejects_widths_off_budget(orc):
    cfg = orc.Config(B=1, H=1, d=32, storage=orc.STORE_VARBIT, hadamard=0, avg_bits=4.0)
    S = np.zeros((1, 1, 32, 32), np.float32)
    w = np.full(32, 4, np.uint8)
    _, fl = orc.state_pack(cfg, S, None, w)
    assert fl == 0
    w[0] = 8
    _, fl = orc.state_pack(cfg, S, None, w)
    assert fl == orc.EINVAL


def test_persistence_weights_closed_forms(orc):
    """w^(1) = 1/(1 - A) and h^(C) = 1/(1 - A^C) for A = EMA(a^2) = e^(-2s),
    computed by the oracle through logarithms; the erasure rate with r = 0 is
    1/(C expm1(2s)) = 1/(C (1/A - 1))."""
    for A in (0.5, 0.81, 0.999):
        assert orc.persistence(1, A, 0.3, 7) == pytest.approx(1.0 / (1.0 - A), rel=1e-12)
        assert orc.persistence(2, A, 0.3, 4) == pytest.approx(1.0 / (1.0 - A ** 4), rel=1e-12)
        assert orc.persistence(2, A, 0.3, 1) == pytest.approx(orc.persistence(1, A, 0.0, 1), rel=1e-15)
        assert orc.persistence(0, A, 0.0, 4) == pytest.approx(1.0 / (4 * (1.0 / A - 1.0)), rel=1e-12)
    assert orc.persistence(1, 1.0, 0.0, 1) == pytest.approx(1e9, rel=1e-6)      # no decay: floored argument
