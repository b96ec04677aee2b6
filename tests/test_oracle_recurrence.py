"""Pins of the oracle's recurrence against FP64 matrix-form references and
the invariants that the update rule fixes."""
import numpy as np
import pytest

from bit_recurrent_state_b200 import synth
from ref64 import (bf16_to_f64, damp_dequant64, damp_head_sections, dense_step, f16_bits_to_f64,
                   hadamard_n, int8_nearest64, token_vectors)


def _cfg(orc, w, **kw):
    st = {"fp32": orc.STORE_FP32, "damp": orc.STORE_DAMP, "varbit": orc.STORE_VARBIT}[w.storage]
    base = dict(B=w.B, H=w.H, Hk=w.hk, d=w.d, storage=st, k_hi=w.k_hi, block=w.block,
                hadamard=w.hadamard, decay_per_key=w.decay_per_key, avg_bits=w.avg_bits,
                b_min=w.b_min, b_max=w.b_max)
    base.update(kw)
    return orc.Config(**base)


def _rand_perm(rng, H, d):
    return np.stack([rng.permutation(d) for _ in range(H)]).astype(np.int16)


@pytest.mark.parametrize("d,H,Hk,per_key", [(16, 2, 2, 1), (32, 4, 2, 0), (64, 2, 2, 1)])
def test_fp32_storage_matches_fp64_dense(orc, d, H, Hk, per_key):
    w = synth.Workload("t", B=2, H=H, Hk=Hk, d=d, T=48, storage="fp32", decay_per_key=per_key,
                       seed=10 + d)
    cfg = _cfg(orc, w)
    rng = np.random.default_rng(d)
    perm = _rand_perm(rng, H, d)
    inp = synth.run_inputs(w, 0, w.T)
    packed, aux, stats = orc.new_state(cfg)
    o, fl, _ = orc.run(cfg, orc.ROUND_NEAREST, 0, 1, 0, inp, packed, perm=perm)
    assert fl == 0
    S_final = packed.view(np.float32).reshape(w.B, H, d, d)
    for b in range(w.B):
        for h in range(H):
            S = np.zeros((d, d))
            for t in range(w.T):
                k, q, v, a, beta = token_vectors(inp, t, b, h, H, Hk, perm[h], per_key)
                S, oo = dense_step(S, k, q, v, a, beta)
                scale = np.max(np.abs(oo)) + 1e-30
                assert np.max(np.abs(o[t, b, h] - oo)) <= 1e-5 * scale
            assert np.max(np.abs(S_final[b, h] - S)) <= 1e-5 * np.max(np.abs(S))


def test_beta_zero_decay_one_is_identity(orc):
    d, H = 32, 2
    cfg = orc.Config(B=1, H=H, d=d, storage=orc.STORE_FP32)
    rng = np.random.default_rng(1)
    S0 = rng.standard_normal((1, H, d, d)).astype(np.float32)
    packed, _ = orc.state_pack(cfg, S0)
    inp = synth.run_inputs(synth.Workload("t", B=1, H=H, d=d, T=5, seed=3), 0, 5)
    inp["beta"][:] = 0.0
    inp["decay"][:] = 1.0
    o, fl, _ = orc.run(cfg, orc.ROUND_NEAREST, 0, 1, 0, inp, packed)
    S1 = packed.view(np.float32).reshape(1, H, d, d)
    np.testing.assert_array_equal(S1.view(np.uint32), S0.view(np.uint32))
    for t in range(5):
        for h in range(H):
            q = bf16_to_f64(inp["q"][t, 0, h])
            np.testing.assert_allclose(o[t, 0, h], S0[0, h].astype(np.float64).T @ q,
                                       rtol=1e-5, atol=1e-6)


def test_unit_key_beta_one_writes_v(orc):
    """k = e_i, beta = 1, a = 1: after the write S^T k = v (exactly for a
    zero row; within the FP32 rounding of v - u otherwise)."""
    d, H = 32, 1
    cfg = orc.Config(B=1, H=H, d=d, storage=orc.STORE_FP32)
    rng = np.random.default_rng(2)
    w = synth.Workload("t", B=1, H=H, d=d, T=1, seed=4)
    for i, init in [(3, "zero"), (7, "rand")]:
        S0 = np.zeros((1, H, d, d), np.float32)
        if init == "rand":
            S0 = rng.standard_normal((1, H, d, d)).astype(np.float32)
        packed, _ = orc.state_pack(cfg, S0)
        inp = synth.run_inputs(w, 0, 1)
        key = np.zeros(d, np.float32)
        key[i] = 1.0
        inp["k"][0, 0, 0] = synth.bf16_bits(key)
        inp["beta"][:] = 1.0
        inp["decay"][:] = 1.0
        orc.run(cfg, orc.ROUND_NEAREST, 0, 1, 0, inp, packed)
        S1 = packed.view(np.float32).reshape(d, d)
        v = bf16_to_f64(inp["v"][0, 0, 0])
        if init == "zero":
            np.testing.assert_array_equal(S1[i].astype(np.float64), v)
        else:
            ulp = np.spacing(np.maximum(np.abs(v), np.abs(S0[0, 0, i])).astype(np.float32))
            assert np.all(np.abs(S1[i] - v) <= 2 * ulp)
        # rows other than i are untouched
        others = [r for r in range(d) if r != i]
        np.testing.assert_array_equal(S1[others], S0[0, 0][others])


@pytest.mark.parametrize("bits", [8, 4])
def test_damp_step_matches_fp64_brute_force(orc, bits):
    """Teacher-forced: each step starts from the oracle's stored state; the
    FP64 reference dequantizes, runs the matrix-form update, re-applies the
    Hadamard and picks every code by exhaustive search.  Codes may differ
    only where the FP64 grid coordinate lies within 1e-3 of a half step (the
    FP32/FP64 gap of the recurrence); a block whose FP16 step or zero flips
    must sit within 1e-5 (relative) of an FP16 rounding midpoint."""
    d, H, k_hi, block = 16, 2, 4, 16
    levels = (1 << bits) - 1
    w = synth.Workload("t", B=2, H=H, d=d, T=8, k_hi=k_hi, block=block, seed=5)
    cfg = _cfg(orc, w, low_bits=bits)
    rng = np.random.default_rng(3)
    perm = _rand_perm(rng, H, d)
    inp_all = synth.run_inputs(w, 0, w.T)
    S0 = (rng.standard_normal((w.B, H, d, d)) * 0.3).astype(np.float32)
    packed, _ = orc.state_pack(cfg, S0, perm)
    hb = packed.size // (w.B * H)
    Hn = hadamard_n(d)
    mism = 0
    for t in range(w.T):
        before = packed.copy()
        inp = {kk: vv[t:t + 1] for kk, vv in inp_all.items()}
        o, fl, tdump = orc.run(cfg, orc.ROUND_NEAREST, 1, t, 0, inp, packed, perm=perm) if False else \
            orc.run(cfg, orc.ROUND_NEAREST, 0, 1, t, inp, packed, perm=perm, dump_t=True)
        assert fl == 0
        for b in range(w.B):
            for h in range(H):
                u = b * H + h
                S = damp_dequant64(before[u * hb:(u + 1) * hb], d, k_hi, block, True, bits)
                k, q, v, a, beta = token_vectors(inp, 0, b, h, H, H, perm[h], True)
                S, oo = dense_step(S, k, q, v, a, beta)
                assert np.max(np.abs(o[0, b, h] - oo)) <= 1e-5 * (np.max(np.abs(oo)) + 1e-30)
                f16rows, codes, sz = damp_head_sections(packed[u * hb:(u + 1) * hb], d, k_hi, block, bits)
                ref16 = S[d - k_hi:].astype(np.float16).view(np.uint16)
                bad = f16rows != ref16
                if bad.any():
                    # only values within FP32 reach of an FP16 rounding midpoint
                    x = np.abs(S[d - k_hi:][bad])
                    ulp = np.spacing(x.astype(np.float16)).astype(np.float64)
                    frac = np.abs((x / ulp) % 1 - 0.5)
                    assert np.all(frac < 1e-3) and np.all(np.abs(f16rows[bad].astype(int) - ref16[bad]) == 1)
                    mism += int(bad.sum())
                R = S[:d - k_hi] @ Hn
                for r in range(d - k_hi):
                    c64, s64, z64, t64 = int8_nearest64(R[r], levels)
                    s_o = f16_bits_to_f64(sz[r, 0, 0])
                    z_o = f16_bits_to_f64(sz[r, 0, 1])
                    if s_o != s64 or z_o != z64:
                        mid = lambda x: abs(abs(x) / np.spacing(np.float16(abs(x)), dtype=np.float16).astype(float) % 1 - 0.5)
                        assert min(mid((R[r].max() - R[r].min()) / levels), mid(R[r].min())) < 1e-2
                        continue
                    diff = codes[r].astype(int) != c64
                    if diff.any():
                        frac = np.abs(t64[diff] - np.floor(t64[diff]) - 0.5)
                        assert np.all(frac < 1e-3), (t, b, h, r, t64[diff])
                        mism += int(diff.sum())
    assert mism <= 2


@pytest.mark.parametrize("name,dom", [("kda_tiny", 1), ("kda_tiny", 2), ("gdn", 2), ("nohad", 2),
                                      ("kda128", 2), ("kda128", 1), ("kda128_b32", 2), ("gdn128", 2)])
def test_reordered_modes_match_canonical(orc, name, dom):
    """The rotated mode (the whole update in the Hadamard basis) and the
    mixed-basis mode (each tier in its stored basis) compute the same update
    as the canonical mode in a different FP32 order.  Teacher-forced from the
    canonical trajectory, one step at a time: outputs agree to FP32 rounding
    and stored codes differ only next to a rounding boundary of the canonical
    grid coordinate.  The d = 128 cases are the measured layouts: 16 FP16 +
    112 INT8 Hadamard rows in blocks of 128 and of 32 (KDA decode and
    prefill), and all 128 rows INT8 with grouped key heads and one decay per
    head (GDN decode)."""
    w = {"kda_tiny": synth.WORKLOADS["kda_tiny"],
         "gdn": synth.Workload("g", B=2, H=4, Hk=2, d=32, T=32, k_hi=0, block=32, decay_per_key=0, seed=12),
         "nohad": synth.Workload("n", B=1, H=2, d=32, T=32, k_hi=8, block=16, hadamard=0, seed=13),
         "kda128": synth.Workload("k", B=2, H=3, d=128, T=16, k_hi=16, block=128, seed=14),
         "kda128_b32": synth.Workload("kb", B=2, H=3, d=128, T=16, k_hi=16, block=32, seed=15),
         "gdn128": synth.Workload("gg", B=2, H=4, Hk=2, d=128, T=16, k_hi=0, block=128, decay_per_key=0,
                                  seed=16)}[name]
    rng = np.random.default_rng(9)
    perm = _rand_perm(rng, w.H, w.d)
    inp_all = synth.run_inputs(w, 0, w.T)
    cc = _cfg(orc, w, domain=orc.DOMAIN_CANONICAL)
    cr = _cfg(orc, w, domain=dom)
    packed, _, _ = orc.new_state(cc)
    ncodes = ndiff = 0
    for t in range(w.T):
        inp = {kk: vv[t:t + 1] for kk, vv in inp_all.items()}
        pr = packed.copy()
        oc, fl, tc = orc.run(cc, orc.ROUND_NEAREST, 0, 1, t, inp, packed, perm=perm, dump_t=True)
        orr, fl2, _ = orc.run(cr, orc.ROUND_NEAREST, 0, 1, t, inp, pr, perm=perm)
        assert fl == 0 and fl2 == 0
        assert np.max(np.abs(oc - orr)) <= 2e-5 * (np.max(np.abs(oc)) + 1e-30)
        hb = packed.size // (w.B * w.H)
        for u in range(w.B * w.H):
            fc, cc_codes, szc = damp_head_sections(packed[u * hb:(u + 1) * hb], w.d, w.k_hi, w.block)
            fr, cr_codes, szr = damp_head_sections(pr[u * hb:(u + 1) * hb], w.d, w.k_hi, w.block)
            # FP16 rows: a value next to an FP16 rounding midpoint may land one unit apart
            assert np.all(np.abs(fc.astype(int) - fr.astype(int)) <= 1)
            ndiff += int(np.sum(fc != fr))
            tt = tc.reshape(w.B * w.H, w.d, w.d)[u, :w.d - w.k_hi]
            same_grid = np.all(szc == szr, axis=(1, 2))
            diff = (cc_codes != cr_codes) & same_grid[:, None]
            ncodes += cc_codes[same_grid].size
            ndiff += int(diff.sum())
            if diff.any():
                frac = np.abs(tt[diff] - np.floor(tt[diff]) - 0.5)
                assert np.all(frac < 1e-3)
    assert ndiff <= 1e-3 * ncodes


def test_dead_zone_through_the_recurrence(orc):
    """a = 1, unit key e_0, tiny beta, and v equal to the stored row except
    one interior element: that element drifts by beta (v_J - S_0J) per token,
    far under half a step, while the block's minimum and maximum stay put
    (step 1/128, zero -1, every stored value exact in bfloat16).
    Deterministic write-back never moves the stored code (the write dead
    zone); error feedback moves it once the carried residual passes half a
    step."""
    d, H, J = 32, 1, 17
    w = synth.Workload("t", B=1, H=H, d=d, T=1, seed=6)
    codes = np.random.default_rng(10).integers(1, 255, d)
    codes[0], codes[1] = 0, 255
    row = ((codes - 128) / 128.0).astype(np.float32)
    v = row.copy()
    v[J] += 0.5
    moved = {}
    for mode in (orc.ROUND_NEAREST, orc.ROUND_ERRFEEDBACK):
        cfg = orc.Config(B=1, H=H, d=d, storage=orc.STORE_DAMP, k_hi=0, block=32, hadamard=0)
        S0 = np.zeros((1, H, d, d), np.float32)
        S0[0, 0, 0] = row
        packed, _ = orc.state_pack(cfg, S0)
        _, aux, _ = orc.new_state(cfg)
        assert np.all(packed[:d] == codes)
        key = np.zeros(d, np.float32)
        key[0] = 1.0
        first = None
        for t in range(100):
            inp = synth.run_inputs(w, t, 1)
            inp["k"][0, 0, 0] = synth.bf16_bits(key)
            inp["v"][0, 0, 0] = synth.bf16_bits(v)
            inp["beta"][:] = 1e-3
            inp["decay"][:] = 1.0
            orc.run(cfg, mode, 0, 1, t, inp, packed, aux=aux)
            if first is None and np.any(packed[:d] != codes):
                first = t
                assert np.all(packed[:d][np.arange(d) != J] == codes[np.arange(d) != J])
                assert packed[J] == codes[J] + 1
        moved[mode] = first
    assert moved[orc.ROUND_NEAREST] is None
    # residual grows by beta*0.5 = 5e-4 per token; half a step is 1/256
    assert moved[orc.ROUND_ERRFEEDBACK] is not None and moved[orc.ROUND_ERRFEEDBACK] <= 9


def test_stochastic_rounding_reproducible(orc):
    w = synth.WORKLOADS["kda_tiny"]
    inp = synth.run_inputs(w, 0, 8)
    res = []
    for seed in (5, 5, 6):
        cfg = _cfg(orc, w)
        packed, aux, stats = orc.new_state(cfg)
        o, fl, _ = orc.run(cfg, orc.ROUND_STOCHASTIC, seed, 1, 0, inp, packed)
        res.append(packed.copy())
    np.testing.assert_array_equal(res[0], res[1])
    assert np.any(res[0] != res[2])


def test_checkpoint_resume_is_bitwise(orc):
    w = synth.WORKLOADS["kda_tiny"]
    inp = synth.run_inputs(w, 0, 16)
    cfg = _cfg(orc, w)
    p1, a1, s1 = orc.new_state(cfg)
    o1, _, _ = orc.run(cfg, orc.ROUND_ERRFEEDBACK, 0, 1, 0, inp, p1, aux=a1)
    p2, a2, s2 = orc.new_state(cfg)
    half = {k: v[:8] for k, v in inp.items()}
    rest = {k: v[8:] for k, v in inp.items()}
    orc.run(cfg, orc.ROUND_ERRFEEDBACK, 0, 1, 0, half, p2, aux=a2)
    p2, a2 = p2.copy(), a2.copy()          # "save and reload"
    o2, _, _ = orc.run(cfg, orc.ROUND_ERRFEEDBACK, 0, 1, 8, rest, p2, aux=a2)
    np.testing.assert_array_equal(p1, p2)
    np.testing.assert_array_equal(a1, a2)
    np.testing.assert_array_equal(o1[8:], o2)


def test_chunked_write_back_only_at_chunk_ends(orc):
    """C = 4: the stored state changes only after tokens 3, 7, ... and the
    outputs between write-backs come from the unquantized FP32 state."""
    w = synth.WORKLOADS["kda_tiny"]
    cfg = _cfg(orc, w)
    inp = synth.run_inputs(w, 0, 8)
    p, a, s = orc.new_state(cfg)
    o4, fl, _ = orc.run(cfg, orc.ROUND_NEAREST, 0, 4, 0, inp, p)
    assert fl == 0
    p1, _, _ = orc.new_state(cfg)
    o1, _, _ = orc.run(cfg, orc.ROUND_NEAREST, 0, 1, 0, inp, p1)
    # first token identical (same starting state), later tokens differ
    np.testing.assert_array_equal(o4[0], o1[0])
    assert np.any(o4[1] != o1[1])
    _, fl = orc.run(cfg, orc.ROUND_NEAREST, 0, 4, 0, {k: v[:3] for k, v in inp.items()}, p)[0:2]
    assert fl == orc.EINVAL


def test_pack_unpack_roundtrip(orc):
    rng = np.random.default_rng(8)
    d, H = 32, 2
    S = rng.standard_normal((2, H, d, d)).astype(np.float32)
    perm = _rand_perm(rng, H, d)
    cfg = orc.Config(B=2, H=H, d=d, storage=orc.STORE_FP32)
    p, _ = orc.state_pack(cfg, S, perm)
    S2, _ = orc.state_unpack(cfg, p, perm)
    np.testing.assert_array_equal(S, S2)
    cfg = orc.Config(B=2, H=H, d=d, storage=orc.STORE_DAMP, k_hi=4, block=32)
    p, _ = orc.state_pack(cfg, S, perm)
    S2, _ = orc.state_unpack(cfg, p, perm)
    for h in range(H):
        prot = perm[h, d - 4:]
        np.testing.assert_array_equal(S2[:, h, prot], S[:, h, prot].astype(np.float16).astype(np.float32))
    err = np.abs(S2 - S).max()
    assert err <= (S.max() - S.min()) / 255 * 2     # half a step per coordinate, spread by H


@pytest.mark.parametrize("mode,dom,low_bits", [(0, 0, 8), (1, 0, 8), (2, 0, 8), (3, 2, 8), (2, 2, 8),
                                                (4, 2, 8), (6, 2, 8), (0, 0, 4), (1, 0, 4), (2, 2, 4),
                                                (3, 2, 4), (5, 2, 4)])
def test_writeback_replay_equals_the_run(orc, mode, dom, low_bits):
    """The write-back entry (the quantizer alone, used to replay a state
    computed elsewhere) applied to the FP32 state the recurrence held just
    before its write-back reproduces the recurrence's stored bytes and
    residuals / counters / residual integers, in every rounding mode and for
    both low tiers."""
    w = synth.Workload("rp", B=2, H=3, d=32, T=4, k_hi=4, block=32, seed=21)
    cfg = _cfg(orc, w, domain=dom, low_bits=low_bits)
    rng = np.random.default_rng(22)
    perm = _rand_perm(rng, w.H, w.d)
    S0 = (rng.standard_normal((w.B, w.H, w.d, w.d)) * 0.1).astype(np.float32)
    packed, _ = orc.state_pack(cfg, S0, perm)
    _, aux, _ = orc.new_state(cfg)
    inp = synth.run_inputs(w, 0, w.T)
    for t in range(w.T):
        before_p, before_a = packed.copy(), aux.copy()
        _, fl, _, sd = orc.run(cfg, mode, 5, 1, t, {k: v[t:t + 1] for k, v in inp.items()}, packed,
                               aux=aux, perm=perm, dump_s=True)
        assert fl == 0
        fl = orc.damp_writeback(cfg, mode, 5, t, sd, before_p, before_a)
        assert fl == 0
        np.testing.assert_array_equal(before_p, packed)
        np.testing.assert_array_equal(before_a, aux)


def test_residual_memory_through_the_recurrence(orc):
    """k-bit residual memory on the dead-zone fixture of the test above
    (fixed grid, step 1/128, one element drifting by about 0.064 step per
    token).  The kept residual is at most (2^(k-1) - 1) step / 2^k: Delta/4
    for k = 2 and 3 Delta/8 for k = 3, so the target never reaches the half
    step and the code never moves, as under deterministic write-back; for
    k = 4 it reaches 7 Delta/16, which with the drift passes the half step:
    the code moves after 8 tokens (residual 1/16, 2/16, ..., 7/16 of a step),
    in the same token as error feedback (whose residual is kept in FP16)."""
    d, H, J = 32, 1, 17
    w = synth.Workload("t", B=1, H=H, d=d, T=1, seed=6)
    codes = np.random.default_rng(10).integers(1, 255, d)
    codes[0], codes[1] = 0, 255
    row = ((codes - 128) / 128.0).astype(np.float32)
    v = row.copy()
    v[J] += 0.5
    moved = {}
    for mode in (orc.ROUND_RESIDUAL2, orc.ROUND_RESIDUAL3, orc.ROUND_RESIDUAL4, orc.ROUND_ERRFEEDBACK):
        cfg = orc.Config(B=1, H=H, d=d, storage=orc.STORE_DAMP, k_hi=0, block=32, hadamard=0)
        S0 = np.zeros((1, H, d, d), np.float32)
        S0[0, 0, 0] = row
        packed, _ = orc.state_pack(cfg, S0)
        _, aux, _ = orc.new_state(cfg)
        key = np.zeros(d, np.float32)
        key[0] = 1.0
        first = None
        for t in range(100):
            inp = synth.run_inputs(w, t, 1)
            inp["k"][0, 0, 0] = synth.bf16_bits(key)
            inp["v"][0, 0, 0] = synth.bf16_bits(v)
            inp["beta"][:] = 1e-3
            inp["decay"][:] = 1.0
            _, fl, _ = orc.run(cfg, mode, 0, 1, t, inp, packed, aux=aux)
            assert fl == 0
            if first is None and np.any(packed[:d] != codes):
                first = t
                assert packed[J] == codes[J] + 1
        moved[mode] = first
    assert moved[orc.ROUND_RESIDUAL2] is None and moved[orc.ROUND_RESIDUAL3] is None
    assert moved[orc.ROUND_RESIDUAL4] == 7
    assert moved[orc.ROUND_ERRFEEDBACK] == moved[orc.ROUND_RESIDUAL4]


@pytest.mark.parametrize("kbits", [2, 3, 4])
def test_residual_memory_block_against_fp64(orc, kbits):
    """The residual-memory block against an FP64 restatement: the target
    y + m_prev sprev / 2^k, its nearest INT8 codes on the block's FP16 grid
    (exhaustive search over the 256 levels), and the new integer = the
    residual in units of step / 2^k rounded to nearest (ties to even) and
    clipped to +-(2^(k-1) - 1).  Values next to a rounding point of either
    rounding (FP32 against FP64) are skipped and counted."""
    from ref64 import int8_nearest64
    rng = np.random.default_rng(40 + kbits)
    mmax = 2 ** (kbits - 1) - 1
    skipped = total = 0
    for trial in range(300):
        n = 32
        y = (rng.standard_normal(n) * rng.uniform(0.01, 3.0)).astype(np.float32)
        sprev = float(np.float16(rng.uniform(0.0, 0.05)))
        mp = rng.integers(-mmax, mmax + 1, n).astype(np.int8)
        codes, sh, zh, m, fl = orc.int8_block_rm(y, kbits, sprev, mp)
        assert fl == 0
        tgt = y.astype(np.float64) + mp.astype(np.float64) * sprev / 2 ** kbits
        c64, s64, z64, t64 = int8_nearest64(tgt.astype(np.float32).astype(np.float64))
        for j in range(n):
            total += 1
            frac_t = abs(t64[j] - np.floor(t64[j]) - 0.5)
            if s64 == 0 or frac_t < 1e-3 or codes[j] != c64[j]:
                skipped += 1
                continue
            q = (tgt[j] - (c64[j] * s64 + z64)) / s64 * 2 ** kbits
            if abs(abs(q - np.floor(q)) - 0.5) < 1e-3:
                skipped += 1
                continue
            want = int(np.clip(np.rint(q), -mmax, mmax))
            assert m[j] == want, (trial, j, m[j], want, q)
    assert skipped <= 0.02 * total
