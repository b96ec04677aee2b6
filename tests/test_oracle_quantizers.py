"""Pins of the oracle's write-back quantizers: exhaustive level search,
tie-to-even, grid rails, unbiased stochastic rounding, error-feedback
bounds, the write dead zone, the variable-width fit against an exhaustive
FP64 scan."""
import numpy as np
import pytest

from conftest import golden


def f16(x):
    return np.float32(np.float16(np.float32(x)))


def test_int8_codes_are_nearest_level(orc):
    rng = np.random.default_rng(1)
    for trial in range(200):
        n = [32, 128][trial % 2]
        y = (rng.standard_normal(n) * 10.0 ** rng.uniform(-3, 2)).astype(np.float32)
        r = orc.int8_block(y)
        s = np.float64(np.uint16(r["scale"]).view(np.float16))
        z = np.float64(np.uint16(r["zero"]).view(np.float16))
        # the stored grid brackets the block (FP16 rounding of min and step)
        assert abs(z - y.min()) <= 2 ** -11 * abs(y.min()) + 2 ** -25
        assert abs(s * 255 - (y.max() - y.min())) <= 255 * 2 ** -11 * s + 2 ** -24 * 255
        levels = np.arange(256) * s + z
        dist = np.abs(y[:, None].astype(np.float64) - levels[None, :])
        best = dist.min(axis=1)
        got = dist[np.arange(n), r["codes"]]
        # nearest level up to the FP32 rounding of the grid coordinate
        assert np.all(got - best <= 1e-5 * s + 1e-30), trial


def test_int8_ties_to_even_and_rails(orc):
    # block spanning [0, 255] has step 1 and zero 0: t = y exactly
    y = np.zeros(32, np.float32)
    y[0], y[1] = 0.0, 255.0
    y[2:8] = [2.5, 3.5, 4.5, 0.5, 253.5, 254.5]
    r = orc.int8_block(y)
    assert r["scale"] == np.float16(1.0).view(np.uint16)
    assert list(r["codes"][2:8]) == [2, 4, 4, 0, 254, 254]
    # rails: a zero rounded above the minimum gives t < 0 -> clipped to 0
    y2 = np.linspace(1000.1, 1100.0, 32).astype(np.float32)
    r2 = orc.int8_block(y2)
    assert r2["codes"].min() == 0 and r2["codes"].max() <= 255


def test_int4_codes_are_nearest_level(orc):
    """The 4-bit low tier ([DAMP] per-block asymmetric affine, b = 4): 16
    levels, step fp16((max - min) / 15); every code is the nearest of the 16
    levels (exhaustive), up to the FP32 rounding of the grid coordinate."""
    rng = np.random.default_rng(11)
    for trial in range(200):
        n = [32, 128][trial % 2]
        y = (rng.standard_normal(n) * 10.0 ** rng.uniform(-3, 2)).astype(np.float32)
        r = orc.lowbit_block(y, 15)
        s = np.float64(np.uint16(r["scale"]).view(np.float16))
        z = np.float64(np.uint16(r["zero"]).view(np.float16))
        assert abs(s * 15 - (y.max() - y.min())) <= 15 * 2 ** -11 * s + 2 ** -24 * 15
        assert r["codes"].max() <= 15
        levels = np.arange(16) * s + z
        dist = np.abs(y[:, None].astype(np.float64) - levels[None, :])
        got = dist[np.arange(n), r["codes"]]
        assert np.all(got - dist.min(axis=1) <= 1e-5 * s + 1e-30), trial


def test_int4_ties_to_even_and_rails(orc):
    # a block spanning [0, 15] has step 1 and zero 0: the grid coordinate is y
    y = np.zeros(32, np.float32)
    y[0], y[1] = 0.0, 15.0
    y[2:8] = [2.5, 3.5, 4.5, 0.5, 13.5, 14.5]
    r = orc.lowbit_block(y, 15)
    assert r["scale"] == np.float16(1.0).view(np.uint16)
    assert list(r["codes"][2:8]) == [2, 4, 4, 0, 14, 14]
    # the INT8 quantizer is the same block with 255 levels
    np.testing.assert_array_equal(orc.lowbit_block(y * 17, 255)["codes"], orc.int8_block(y * 17)["codes"])


def test_int8_constant_block(orc):
    y = np.full(32, 3.25, np.float32)
    r = orc.int8_block(y)
    assert r["scale"] == 0 and np.all(r["codes"] == 0)
    assert np.float16(np.uint16(r["zero"]).view(np.float16)) == np.float16(3.25)


def test_stochastic_rounding_unbiased_and_reproducible(orc):
    rng = np.random.default_rng(2)
    y = (rng.standard_normal(32)).astype(np.float32)
    a = orc.int8_block(y, mode=orc.ROUND_STOCHASTIC, seed=7, step=3, h=1, b=2)
    b = orc.int8_block(y, mode=orc.ROUND_STOCHASTIC, seed=7, step=3, h=1, b=2)
    np.testing.assert_array_equal(a["codes"], b["codes"])
    s = np.float64(np.uint16(a["scale"]).view(np.float16))
    z = np.float64(np.uint16(a["zero"]).view(np.float16))
    N = 4000
    acc = np.zeros(32)
    for seed in range(N):
        acc += orc.int8_block(y, mode=orc.ROUND_STOCHASTIC, seed=seed)["codes"]
    mean_val = acc / N * s + z
    t = (y.astype(np.float64) - z) / s
    frac = t - np.floor(t)
    sigma = s * np.sqrt(frac * (1 - frac) / N) + 1e-12
    inside = (t >= 0) & (t <= 255)           # values past a rail are clipped, not unbiased
    assert inside.sum() >= 28
    assert np.all((np.abs(mean_val - y) <= 4 * sigma + 1e-5 * s)[inside])
    # each code is one of the two adjacent levels
    c = a["codes"].astype(np.float64)
    assert np.all((c == np.floor(t)) | (c == np.floor(t) + 1) | (c == 0) | (c == 255))


def test_error_feedback_residual_bounded(orc):
    rng = np.random.default_rng(3)
    e = np.zeros(32, np.uint16)
    for step in range(50):
        y = rng.standard_normal(32).astype(np.float32)
        r = orc.int8_block(y, mode=orc.ROUND_ERRFEEDBACK, e=e)
        s = np.float32(np.uint16(r["scale"]).view(np.float16))
        ev = np.uint16(r["e"]).view(np.float16).astype(np.float32)
        assert np.all(np.abs(ev) <= f16(s) + 1e-12)
        e = r["e"]


def _write_back_loop(orc, mode, delta, steps):
    """Persistent drift of one interior value; min/max pinned so the step
    stays 0.125 (the 4-bit grid spacing of the dead-zone fixture)."""
    g = golden("dead_zone.txt")
    D = float(g["delta_4"])
    y = np.zeros(32, np.float32)
    y[0], y[1] = 0.0, 255 * D            # step (max-min)/255 = 0.125 exactly
    y[2] = 100 * D                        # on a level
    e = np.zeros(32, np.uint16)
    moved_at = None
    cur = y.copy()
    code0 = None
    for t in range(steps):
        target = cur.copy()
        target[2] = cur[2] + np.float32(delta)
        r = orc.int8_block(target, mode=mode, e=e if mode == orc.ROUND_ERRFEEDBACK else None,
                           seed=11, step=t)
        s = np.float32(np.uint16(r["scale"]).view(np.float16))
        assert s == np.float32(D)
        z = np.float32(np.uint16(r["zero"]).view(np.float16))
        if code0 is None:
            code0 = int(round(100))
        if r["codes"][2] != code0 and moved_at is None:
            moved_at = t
        cur = (r["codes"].astype(np.float32) * s + z).astype(np.float32)
        if mode == orc.ROUND_ERRFEEDBACK:
            e = r["e"]
    return moved_at


def test_dead_zone_deterministic_never_moves(orc):
    g = golden("dead_zone.txt")
    half = float(g["half_step"])
    delta = 0.8 * half                       # write margin M = 2|delta|/Delta = 0.8 < 1
    assert 2 * delta / float(g["delta_4"]) < 1
    assert _write_back_loop(orc, orc.ROUND_NEAREST, delta, 200) is None


def test_dead_zone_error_feedback_moves(orc):
    g = golden("dead_zone.txt")
    delta = 0.1 * float(g["half_step"])      # far inside the dead zone
    t = _write_back_loop(orc, orc.ROUND_ERRFEEDBACK, delta, 200)
    # the residual crosses the half step after about half_step/delta steps
    assert t is not None and t <= int(np.ceil(1 / 0.1)) + 1


def test_dead_zone_stochastic_moves(orc):
    g = golden("dead_zone.txt")
    delta = 0.1 * float(g["half_step"])
    assert _write_back_loop(orc, orc.ROUND_STOCHASTIC, delta, 400) is not None


@pytest.mark.parametrize("bw", [2, 3, 4, 6, 8])
def test_varbit_fit_matches_exhaustive_scan(orc, bw):
    rng = np.random.default_rng(bw)
    n_l = 2 ** (bw - 1) - 1
    for trial in range(60):
        x = (rng.standard_normal(128) * rng.uniform(0.01, 5)).astype(np.float32)
        if trial % 3 == 0:
            x[rng.integers(128)] *= 8                         # an outlier
        r = orc.varbit_row(x, bw)
        R = np.max(np.abs(x)).astype(np.float64)
        # exhaustive FP64 scan of the 16 candidate steps, nearest level each
        errs = []
        for m in range(16):
            D = np.float64(f16(np.float32(np.float32((5 + m) / 20) * np.float32(R)) / np.float32(n_l)))
            lev = np.arange(-n_l, n_l + 1) * D
            err = np.min((x[:, None].astype(np.float64) - lev[None, :]) ** 2, axis=1).sum()
            errs.append(err)
        errs = np.array(errs)
        assert errs[r["m"]] <= errs.min() * (1 + 1e-5) + 1e-30, (trial, r["m"], errs)
        D = np.float64(np.uint16(r["delta"]).view(np.float16))
        lev = np.arange(-n_l, n_l + 1) * D
        dist = np.abs(x[:, None].astype(np.float64) - lev[None, :])
        got = dist[np.arange(128), r["q"] + n_l]
        assert np.all(got - dist.min(axis=1) <= 1e-5 * D + 1e-30)
        assert np.all(np.abs(r["q"]) <= n_l)


def test_varbit_zero_row(orc):
    r = orc.varbit_row(np.zeros(128, np.float32), 4)
    assert r["delta"] == 0 and np.all(r["q"] == 0)


# ---- direction memory ([WB] Post-training write-back interventions:
# signed sub-threshold votes, a trigger of one level, a reset counter,
# rails; Trajectory analysis: the voting region Delta/8 < |delta| < Delta/2;
# the Chinese summary's core method: threshold T_k = 2^(k-1), here k = 2)

def _dm_loop(orc, deltas, start_level=100):
    """One interior value drifting by deltas[t] per step on a fixed grid of
    spacing 0.125 (min and max pinned); returns its code after each step."""
    D = float(golden("dead_zone.txt")["delta_4"])
    cur = np.zeros(32, np.float32)
    cur[1] = 255 * D
    cur[2] = start_level * D
    m = np.zeros(32, np.int8)
    out = []
    for dl in deltas:
        tgt = cur.copy()
        tgt[2] = cur[2] + np.float32(dl)
        r = orc.int8_block_dm(tgt, cur, m)
        s = np.float32(np.uint16(r["scale"]).view(np.float16))
        assert s == np.float32(D)
        z = np.float32(np.uint16(r["zero"]).view(np.float16))
        m = r["m"]
        assert set(np.unique(m)) <= {-1, 0, 1}
        cur = (r["codes"].astype(np.float32) * s + z).astype(np.float32)
        out.append(int(r["codes"][2]))
    return out


def test_direction_memory_fixture_is_consistent():
    g = golden("direction_memory.txt")
    k = int(g["counter_bits"])
    assert int(g["threshold"]) == 2 ** (k - 1)          # T_k = 2^(k-1)
    assert int(g["active_states"]) == 2 ** k - 1        # counter values -(T-1) .. T-1
    assert float(g["vote_lo_frac"]) == 1 / 8 and float(g["vote_hi_frac"]) == 1 / 2


@pytest.mark.parametrize("frac", [0.2, 0.3, 0.45])
def test_direction_memory_moves_one_level_per_two_votes(orc, frac):
    """A constant drift inside the voting region (inside the dead zone, so
    nearest write-back never moves) moves the stored value by one level at
    every T-th step (T = 2 votes), then the counter restarts from 0."""
    g = golden("direction_memory.txt")
    lo, hi, T = float(g["vote_lo_frac"]), float(g["vote_hi_frac"]), int(g["threshold"])
    assert lo < frac < hi
    D = float(golden("dead_zone.txt")["delta_4"])
    codes = _dm_loop(orc, [frac * D] * 12)
    assert codes == [100 + (t + 1) // T for t in range(12)]
    down = _dm_loop(orc, [-frac * D] * 12)
    assert down == [100 - (t + 1) // T for t in range(12)]


def test_direction_memory_ignores_changes_outside_the_region(orc):
    D = float(golden("dead_zone.txt")["delta_4"])
    g = golden("direction_memory.txt")
    # below Delta/8 (and at it: the region is open): no vote, no move
    assert _dm_loop(orc, [0.1 * D] * 20) == [100] * 20
    assert _dm_loop(orc, [float(g["vote_lo_frac"]) * D] * 20) == [100] * 20
    # alternating directions cancel in the signed counter
    assert _dm_loop(orc, [0.3 * D, -0.3 * D] * 10) == [100] * 20
    # above Delta/2 the nearest level moves by itself and nothing votes
    assert _dm_loop(orc, [0.75 * D] * 6) == [101, 102, 103, 104, 105, 106]


def test_direction_memory_trigger_is_clipped_at_the_rail(orc):
    D = float(golden("dead_zone.txt")["delta_4"])
    y = np.zeros(32, np.float32)
    y[1] = 255 * D                                   # on the top rail
    xp = y.copy()
    xp[1] = y[1] - np.float32(0.3 * D)               # a vote up
    m = np.zeros(32, np.int8)
    m[1] = 1                                         # ... that completes the count
    r = orc.int8_block_dm(y, xp, m)
    assert r["codes"][1] == 255 and r["m"][1] == 0   # clipped, counter reset
    assert np.all(r["codes"][2:] == 0) and np.all(r["m"][2:] == 0)


def test_direction_memory_recurrence_keeps_a_still_state(orc):
    """beta = 0, a = 1 through the whole decode recurrence (no Hadamard): the
    proposals equal the stored values, nothing votes, and the stored state
    and counters stay as they are.  Reading the stored value the step started
    from anywhere else would give nonzero proposals of up to half a step."""
    from bit_recurrent_state_b200 import synth
    from parity import oracle_cfg, random_perm
    w = synth.Workload("dm_still", B=2, H=2, d=32, k_hi=4, block=32, hadamard=0, T=6, seed=3, mode="direction")
    cfg = oracle_cfg(w)
    S0 = (np.random.default_rng(5).standard_normal((w.B, w.H, w.d, w.d))).astype(np.float32)
    perm = random_perm(w, seed=2)
    packed, fl = orc.state_pack(cfg, S0, perm)
    assert fl == 0
    _, aux, stats = orc.new_state(cfg)
    before = packed.copy()
    inp = synth.run_inputs(w, 0, w.T)
    inp["beta"][:] = 0.0
    inp["decay"][:] = 1.0
    o, fl, _ = orc.run(cfg, orc.ROUND_DIRECTION, w.seed, 1, 0, inp, packed, aux=aux, stats=stats, perm=perm)
    assert fl == 0
    np.testing.assert_array_equal(packed, before)
    assert not np.any(aux)


def test_direction_memory_recurrence_counters_are_two_bit_fields(orc):
    """A decode run under direction memory: every stored counter field is
    one of -1, 0, 1 (the value -2 is never stored), some counters are
    nonzero, and the run only departs from nearest write-back after votes."""
    from bit_recurrent_state_b200 import synth
    from parity import oracle_cfg
    w = synth.Workload("dm_run", B=1, H=2, d=32, k_hi=4, block=32, T=12, seed=4, mode="direction")
    cfg = oracle_cfg(w)
    inp = synth.run_inputs(w, 0, w.T)
    pd, aux, stats = orc.new_state(cfg)
    o_d, fl, _ = orc.run(cfg, orc.ROUND_DIRECTION, w.seed, 1, 0, inp, pd, aux=aux, stats=stats)
    assert fl == 0
    fields = np.unpackbits(aux.view(np.uint8)[: w.B * w.H * (w.d - w.k_hi) * w.d // 4][:, None],
                           axis=1, bitorder="little").reshape(-1, 4, 2)
    vals = fields[..., 0] + 2 * fields[..., 1]
    assert not np.any(vals == 2)
    assert np.any(vals != 0)
    pn, auxn, statsn = orc.new_state(cfg)
    o_n, fl, _ = orc.run(cfg, orc.ROUND_NEAREST, w.seed, 1, 0, inp, pn, aux=auxn, stats=statsn)
    # the first token starts from the zero state on both sides: identical
    np.testing.assert_array_equal(o_d[0], o_n[0])
