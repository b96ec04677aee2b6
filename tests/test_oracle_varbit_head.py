"""Pins of the per-head variable-width write-back ("Low-Bit Recurrent States
in Hybrid Language Models", Allocation units: per-head decay and
normalization give each head one width and one FP16 step per block of 32
key channels, R~ = 1 so only decay sets the widths, b_min = 2; State bit
allocation: one budget over the layer).  Checked against FP64
recomputations of the update, the head costs and the fitted steps, and
against the row quantizer for the stochastic-rounding element indices."""
import numpy as np
import pytest

from bit_recurrent_state_b200 import synth
from ref64 import bf16_to_f64, dense_step, f16_bits_to_f64, varbit_head_codes, varbit_head_sections


def f16(x):
    return np.float32(np.float16(x))


def _cfg(orc, B, H, Hk, d, avg=4.0, b_min=2, b_max=8, pers=0, per_key=0):
    return orc.Config(B=B, H=H, Hk=Hk, d=d, storage=orc.STORE_VARBIT_HEAD, hadamard=0,
                      decay_per_key=per_key, avg_bits=avg, b_min=b_min, b_max=b_max,
                      budget_scope=1, persistence=pers)


def _dequant64(pay, sc, wd, of, b, h, d):
    bw = int(wd[b, h])
    u = varbit_head_codes(pay[b], int(of[b, h]), bw, d).astype(int)
    steps = f16_bits_to_f64(sc[b, h])                       # [d/32][d]
    return (u - (2 ** (bw - 1) - 1)) * np.repeat(steps, 32, axis=0), u


@pytest.mark.parametrize("mode,d,pers,per_key", [(0, 32, 0, 0), (0, 64, 0, 0), (1, 64, 0, 0),
                                                 (2, 32, 0, 0), (0, 64, 2, 0), (0, 32, 0, 1)])
def test_head_units_teacher_forced_fp64(orc, mode, d, pers, per_key):
    """Every step from the oracle's own stored state: o and the updated state
    by an FP64 delta rule; widths by an FP64 recomputation of the head costs
    (mean of the rows' decay weights, no ranges) through the allocator; every
    (block, column) step is one of the 16 candidates built from that group's
    own range; levels are nearest (deterministic), adjacent (stochastic) or
    within a step of the target (error feedback)."""
    B, H, Hk, T, avg = 2, 6, 3, 6, 4.0
    w = synth.Workload("t", B=B, H=H, Hk=Hk, d=d, T=T, storage="varbit", hadamard=0,
                       decay_per_key=per_key, seed=40 + mode)
    cfg = _cfg(orc, B, H, Hk, d, avg=avg, pers=pers, per_key=per_key)
    inp_all = synth.run_inputs(w, 0, T)
    packed, aux, stats = orc.new_state(cfg)
    lam = 1 - 2 / 65
    A64 = np.zeros((B, H, d))
    K64 = np.zeros((B, H, d))
    near_ties = 0
    for t in range(T):
        before = packed.copy()
        inp = {k: v[t:t + 1] for k, v in inp_all.items()}
        o, fl, _ = orc.run(cfg, mode, 5, 1, t, inp, packed, aux=aux, stats=stats)
        assert fl == 0
        pay0, sc0, wd0, of0 = varbit_head_sections(before, B, H, d, avg)
        pay, sc, wd, of = varbit_head_sections(packed, B, H, d, avg)
        for b in range(B):
            assert int(wd[b].astype(int).sum()) == int(avg * H)                # layer budget
            assert wd[b].min() >= 2                                             # b_min = 2
            np.testing.assert_array_equal(
                of[b], np.concatenate([[0], np.cumsum(wd[b].astype(int))]) * (d * d // 8))
            S_new = np.zeros((H, d, d))
            for h in range(H):
                S, _ = _dequant64(pay0, sc0, wd0, of0, b, h, d)
                kh = h * Hk // H
                k, q, v = (bf16_to_f64(inp["k"][0, b, kh]), bf16_to_f64(inp["q"][0, b, kh]),
                           bf16_to_f64(inp["v"][0, b, h]))
                a = inp["decay"][0, b, h].astype(np.float64) * (np.ones(d) if not per_key else 1.0)
                beta = float(inp["beta"][0, b, h])
                S, oo = dense_step(S, k, q, v, a, beta)
                assert np.max(np.abs(o[0, b, h] - oo)) <= 1e-5 * (np.max(np.abs(oo)) + 1e-30)
                S_new[h] = S
                kk = beta * (2 - beta) * k ** 2
                A64[b, h] = a ** 2 if t == 0 else lam * A64[b, h] + (1 - lam) * a ** 2
                K64[b, h] = kk if t == 0 else lam * K64[b, h] + (1 - lam) * kk
            # head costs: mean over the head's rows of the decay weight, R~ = 1
            s_hat = -0.5 * np.log(A64[b])
            if pers == 0:
                gam = 1.0 / np.expm1(np.maximum(2 * (s_hat + 0.5 * K64[b]), 1e-9))
            else:                                    # h^(C) at C = 1
                gam = 1.0 / (1.0 - A64[b])
            c = gam.mean(axis=1)
            bits64, _ = orc.allocate_bits(c, avg, 2, 8)
            diff = bits64 != wd[b]
            if diff.any():
                bstar = avg + 0.5 * np.log2(c / np.exp(np.mean(np.log(c))))
                assert np.all(np.abs(np.abs(bstar[diff] - np.floor(bstar[diff])) - 0.5) < 1e-6)
                near_ties += int(diff.sum())
            for h in range(H):
                bw = int(wd[b, h])
                nl = 2 ** (bw - 1) - 1
                _, u = _dequant64(pay, sc, wd, of, b, h, d)
                qv = u - nl
                assert np.all(np.abs(qv) <= nl)
                D = np.repeat(f16_bits_to_f64(sc[b, h]), 32, axis=0)          # [d][d]
                x = S_new[h]
                for g in range(d // 32):
                    blk = slice(32 * g, 32 * g + 32)
                    R = np.max(np.abs(x[blk]), axis=0)                       # per column of the block
                    cand = np.array([[np.float64(f16(np.float32(np.float32((5 + m) / 20) * np.float32(r))
                                                     / np.float32(nl))) for m in range(16)] for r in R])
                    Dg = D[32 * g]
                    if mode != 2:                   # error feedback fits x + residual instead
                        rel = np.min(np.abs(cand - Dg[:, None]), axis=1) / np.maximum(Dg, 1e-30)
                        assert np.all(rel <= 2.0 ** -9), (t, b, h, g)
                if mode == 0:
                    qn = np.clip(np.rint(np.where(D > 0, x / np.where(D > 0, D, 1), 0)), -nl, nl)
                    got = np.abs(x - qv * D)
                    best = np.min(np.abs(x[..., None] - np.clip(qn[..., None] + np.array([-1, 0, 1]), -nl, nl) * D[..., None]), axis=-1)
                    assert np.all(got - best <= 1e-4 * D + 1e-30)
                elif mode == 1:
                    tq = x / np.where(D > 0, D, 1)
                    ok = (qv == np.clip(np.floor(tq), -nl, nl)) | (qv == np.clip(np.floor(tq) + 1, -nl, nl))
                    near = np.abs(tq - np.rint(tq)) < 1e-4                    # FP32 vs FP64 at a level
                    assert np.all(ok | near | (D == 0))
    assert near_ties <= 2


def test_two_bit_mean_is_uniform_block_quantization(orc):
    """At a two-bit mean with b_min = 2 every head has two bits: levels
    {-1, 0, 1} times the step of each (block, column) group."""
    B, H, Hk, d, T = 2, 4, 2, 64, 3
    w = synth.Workload("t", B=B, H=H, Hk=Hk, d=d, T=T, storage="varbit", hadamard=0,
                       decay_per_key=0, seed=50)
    cfg = _cfg(orc, B, H, Hk, d, avg=2.0, b_min=2, b_max=8)
    packed, aux, stats = orc.new_state(cfg)
    o, fl, _ = orc.run(cfg, 0, 0, 1, 0, synth.run_inputs(w, 0, T), packed, aux=aux, stats=stats)
    assert fl == 0
    pay, sc, wd, of = varbit_head_sections(packed, B, H, d, 2.0)
    assert np.all(wd == 2)
    for b in range(B):
        for h in range(H):
            u = varbit_head_codes(pay[b], int(of[b, h]), 2, d)
            assert set(np.unique(u)) <= {0, 1, 2}


def _gdn_decay_inputs(w, s_heads):
    """Inputs with a fixed decay rate per head (a = e^-s)."""
    inp = synth.run_inputs(w, 0, w.T)
    inp["decay"][:] = np.exp(-np.asarray(s_heads, np.float64)).astype(np.float32)[None, None, :]
    return inp


def test_widths_follow_decay_only(orc):
    """Widths fall as the decay rate rises (slower decay, longer memory, more
    bits), and do not change when the values (and so every range) are scaled
    by 64: R~ = 1."""
    B, H, Hk, d, T = 1, 8, 8, 32, 4
    w = synth.Workload("t", B=B, H=H, Hk=Hk, d=d, T=T, storage="varbit", hadamard=0,
                       decay_per_key=0, seed=60)
    s_heads = [0.002, 0.8, 0.01, 0.3, 0.05, 2.0, 0.1, 0.02]
    cfg = _cfg(orc, B, H, Hk, d, avg=4.0, b_min=2, b_max=8)
    widths = []
    for scale in (1.0, 64.0):
        inp = _gdn_decay_inputs(w, s_heads)
        vb = (inp["v"].view(np.uint16).astype(np.uint32) << 16).view(np.float32) * np.float32(scale)
        inp["v"] = synth.bf16_bits(vb)
        packed, aux, stats = orc.new_state(cfg)
        _, fl, _ = orc.run(cfg, 0, 0, 1, 0, inp, packed, aux=aux, stats=stats)
        assert fl == 0
        widths.append(varbit_head_sections(packed, B, H, d, 4.0)[2][0].astype(int))
    np.testing.assert_array_equal(widths[0], widths[1])
    order = np.argsort(s_heads)
    assert np.all(np.diff(widths[0][order]) <= 0), widths[0][order]
    assert widths[0].sum() == 4 * H and widths[0].min() >= 2


def test_group_stride_matches_row_indexing(orc):
    """A group whose elements sit d apart in the head draws the same
    stochastic-rounding words as those elements in a row: the group's values
    placed every d-th element of an otherwise zero row (zeros add nothing to
    a fit error and keep the range) round identically."""
    rng = np.random.default_rng(8)
    d = 64
    for trial in range(20):
        x = (rng.standard_normal(32) * rng.uniform(0.1, 3)).astype(np.float32)
        j, g, bw = int(rng.integers(d)), int(rng.integers(2)), int(rng.integers(2, 9))
        e0 = 32 * g * d + j
        gr = orc.varbit_group(x, bw, mode=orc.ROUND_STOCHASTIC, seed=3, step=trial, h=1, b=2,
                              elem0=e0, estride=d)
        row = np.zeros(32 * d, np.float32)
        row[::d] = x
        rw = orc.varbit_row(row, bw, mode=orc.ROUND_STOCHASTIC, seed=3, step=trial, h=1, b=2, elem0=e0)
        assert gr["delta"] == rw["delta"] and gr["m"] == rw["m"]
        np.testing.assert_array_equal(gr["q"], rw["q"][::d])


@pytest.mark.parametrize("bw", [2, 3, 5, 8])
def test_group_fit_matches_exhaustive_scan(orc, bw):
    """The 32-element group takes the row quantizer's fit: the chosen step has
    the least FP64 squared error over the 16 candidates, levels nearest."""
    rng = np.random.default_rng(30 + bw)
    n_l = 2 ** (bw - 1) - 1
    for trial in range(40):
        x = (rng.standard_normal(32) * rng.uniform(0.01, 5)).astype(np.float32)
        r = orc.varbit_group(x, bw, elem0=int(rng.integers(4096)), estride=128)
        R = np.max(np.abs(x)).astype(np.float64)
        errs = []
        for m in range(16):
            D = np.float64(f16(np.float32(np.float32((5 + m) / 20) * np.float32(R)) / np.float32(n_l)))
            lev = np.arange(-n_l, n_l + 1) * D
            errs.append(np.min((x[:, None].astype(np.float64) - lev[None, :]) ** 2, axis=1).sum())
        errs = np.array(errs)
        assert errs[r["m"]] <= errs.min() * (1 + 1e-5) + 1e-30
        D = f16_bits_to_f64(np.uint16(r["delta"]))
        dist = np.abs(x[:, None].astype(np.float64) - np.arange(-n_l, n_l + 1)[None, :] * D)
        assert np.all(dist[np.arange(32), r["q"] + n_l] - dist.min(axis=1) <= 1e-5 * D + 1e-30)


def test_storage_and_layout_rules(orc):
    gdn = _cfg(orc, 256, 32, 16, 128, avg=4.0)
    total, aux, stats = orc.state_bytes(gdn)
    P = 128 * 128 // 8 * 4 * 32
    assert total == P * 256 + 256 * 32 * 4 * 128 * 2 + 256 * 32 + ((256 * 33 * 4 + 255) // 256) * 256
    assert orc.bits_per_value(gdn) == 4.0 + 0.5 + 3.0 / (128 * 128)
    assert orc.bits_per_value(_cfg(orc, 1, 32, 16, 128, avg=4.0, b_max=16)) == 4.5 + 4.0 / (128 * 128)
    S = np.zeros((1, 3, 32, 32), np.float32)
    for bad in (dict(b_min=1), dict(avg=4.5), dict(avg=1.0)):
        cfg = _cfg(orc, 1, 3, 3, 32, **{"avg": 4.0, **bad})
        _, fl = orc.state_pack(cfg, S)
        assert fl == orc.EINVAL, bad
    cfg = _cfg(orc, 1, 3, 3, 32, avg=4.0)
    _, fl = orc.state_pack(cfg, S, None, np.array([4, 4, 5], np.uint8))      # off budget
    assert fl == orc.EINVAL
    packed, fl = orc.state_pack(cfg, S, None, np.array([2, 4, 6], np.uint8))
    assert fl == 0
    assert list(varbit_head_sections(packed, 1, 3, 32, 4.0)[2][0]) == [2, 4, 6]
