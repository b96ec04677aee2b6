"""GPU parity of the decode step (FP32 and DAMP storage) against the oracle,
through the C ABI.  Stored bytes (codes, FP16 rows, FP16 scale/zero,
residuals) must be identical; outputs within 2e-3 x RMS (expected identical
given the shared operation order)."""
import numpy as np
import pytest

from bit_recurrent_state_b200 import synth
from parity import MODE, o_tolerance, oracle_cfg, random_perm, to_dev

pytestmark = pytest.mark.gpu


def _run_both(w, T, perm=None, units=None, init_scale=0.0, seed_state=0):
    import torch
    from bit_recurrent_state_b200 import brs
    from bit_recurrent_state_b200.state import LayerState
    from oracle import oracle as O

    cfg = oracle_cfg(w)
    L = brs.layout_of(w)
    wb = brs.writeback_of(w)
    st = LayerState(L, perm=perm)
    S0 = (np.random.default_rng(seed_state).standard_normal((w.B, w.H, w.d, w.d)) * init_scale).astype(np.float32)
    st.pack(torch.from_numpy(S0).cuda())
    packed_o, _ = O.state_pack(cfg, S0, perm)
    _, aux_o, stats_o = O.new_state(cfg)
    gpu_packed0 = st.packed.cpu().numpy()
    np.testing.assert_array_equal(gpu_packed0, packed_o)      # pack parity
    o_gpu = torch.zeros((w.B, w.H, w.d), dtype=torch.float32, device="cuda")
    steps = []
    for t in range(T):
        inp = synth.token_inputs(w, t)
        dev = to_dev(inp)
        st.step(wb, t, dev["q"], dev["k"], dev["v"], dev["beta"], dev["decay"], o_gpu)
        og = o_gpu.cpu().numpy()
        oo, fl, _ = O.run_parallel(cfg, MODE[w.mode], w.seed, 1, t,
                                   {k: v[None] for k, v in inp.items()}, packed_o, aux=aux_o,
                                   stats=stats_o, perm=perm, units=units)
        assert fl == 0
        steps.append((og, oo[0], st.packed.cpu().numpy().copy(), packed_o.copy(),
                      st.aux.cpu().numpy()[: aux_o.nbytes].copy(), aux_o.view(np.uint8).copy()))
    assert st.errors() == 0
    return steps


def _compare(w, steps, units=None):
    hb = steps[0][2].size // (w.B * w.H)
    sel = np.arange(w.B * w.H) if units is None else np.arange(*units)
    for t, (og, oo, pg, po, ag, ao) in enumerate(steps):
        og_u = og.reshape(w.B * w.H, w.d)[sel]
        oo_u = oo.reshape(w.B * w.H, w.d)[sel]
        tol = o_tolerance(oo_u)
        assert np.max(np.abs(og_u - oo_u)) <= tol, (t, np.max(np.abs(og_u - oo_u)), tol)
        pg_u = pg.reshape(w.B * w.H, hb)[sel]
        po_u = po.reshape(w.B * w.H, hb)[sel]
        ndiff = int(np.sum(pg_u != po_u))
        assert ndiff == 0, f"step {t}: {ndiff} stored bytes differ"
        if w.mode == "errfeedback":
            per = ag.size // (w.B * w.H)
            np.testing.assert_array_equal(ag.reshape(w.B * w.H, per)[sel], ao.reshape(w.B * w.H, per)[sel])
        if (w.mode == "direction" or w.mode.startswith("residual")) and units is None:
            # 2-bit counters / k-bit residual integers of every head, then the
            # unused rest of the buffer
            np.testing.assert_array_equal(ag, ao, err_msg=f"{w.mode} auxiliary state after step {t}")


def test_kda_tiny_full_trajectory():
    w = synth.WORKLOADS["kda_tiny"]
    perm = random_perm(w)
    steps = _run_both(w, w.T, perm=perm)
    _compare(w, steps)
    # outputs bit-identical too (same operation order on both sides)
    for og, oo, *_ in steps:
        np.testing.assert_array_equal(og.view(np.uint32), oo.view(np.uint32))


@pytest.mark.parametrize("name,kw", [
    ("kda128_ragged", dict(B=3, H=5, d=128, k_hi=16, block=128)),
    ("kda128_block32", dict(B=2, H=3, d=128, k_hi=16, block=32)),
    ("kda128_khi8", dict(B=2, H=3, d=128, k_hi=8, block=128)),
    ("kda128_khi24_nohad_b32", dict(B=2, H=2, d=128, k_hi=24, block=32, hadamard=0)),
    ("kda128_all_fp16", dict(B=1, H=2, d=128, k_hi=128, block=128)),
    ("kda128_b32_sr", dict(B=2, H=2, d=128, k_hi=16, block=32, mode="stochastic")),
    ("kda64", dict(B=2, H=3, d=64, k_hi=8, block=64)),
    ("kda32_nohad", dict(B=2, H=2, d=32, k_hi=4, block=32, hadamard=0)),
    ("gdn128", dict(B=3, H=4, Hk=2, d=128, k_hi=0, block=128, decay_per_key=0)),
    ("kda128_sr", dict(B=2, H=3, d=128, k_hi=16, block=128, mode="stochastic")),
    ("kda128_ef", dict(B=2, H=3, d=128, k_hi=16, block=128, mode="errfeedback")),
    ("kda32_ef", dict(B=1, H=2, d=32, k_hi=4, block=32, mode="errfeedback")),
    ("kda128_dm", dict(B=2, H=3, d=128, k_hi=16, block=128, mode="direction")),
    ("kda128_b32_dm", dict(B=2, H=2, d=128, k_hi=16, block=32, mode="direction")),
    ("kda64_dm", dict(B=2, H=3, d=64, k_hi=8, block=64, mode="direction")),
    ("kda32_nohad_dm", dict(B=2, H=2, d=32, k_hi=4, block=32, hadamard=0, mode="direction")),
    ("gdn128_dm", dict(B=3, H=4, Hk=2, d=128, k_hi=0, block=128, decay_per_key=0, mode="direction")),
    ("kda128_rm2", dict(B=2, H=3, d=128, k_hi=16, block=128, mode="residual2")),
    ("kda128_b32_rm3", dict(B=2, H=2, d=128, k_hi=16, block=32, mode="residual3")),
    ("kda128_rm4", dict(B=2, H=3, d=128, k_hi=16, block=128, mode="residual4")),
    ("kda64_rm4", dict(B=2, H=3, d=64, k_hi=8, block=64, mode="residual4")),
    ("kda32_nohad_rm3", dict(B=2, H=2, d=32, k_hi=4, block=32, hadamard=0, mode="residual3")),
    ("gdn128_rm2", dict(B=3, H=4, Hk=2, d=128, k_hi=0, block=128, decay_per_key=0, mode="residual2")),
    ("fp32_64", dict(B=2, H=3, d=64, storage="fp32")),
    ("fp32_gdn128", dict(B=2, H=4, Hk=2, d=128, storage="fp32", decay_per_key=0)),
    # the 4-bit low tier (two codes per byte, 16 levels per block)
    ("kda128_int4_ragged", dict(B=3, H=5, d=128, k_hi=16, block=128, low_bits=4)),
    ("kda128_b32_int4_sr", dict(B=2, H=2, d=128, k_hi=16, block=32, mode="stochastic", low_bits=4)),
    ("kda128_int4_ef", dict(B=2, H=3, d=128, k_hi=16, block=128, mode="errfeedback", low_bits=4)),
    ("kda128_b32_int4_dm", dict(B=2, H=2, d=128, k_hi=16, block=32, mode="direction", low_bits=4)),
    ("kda128_int4_rm4", dict(B=2, H=3, d=128, k_hi=16, block=128, mode="residual4", low_bits=4)),
    ("kda64_int4_khi16", dict(B=2, H=3, d=64, k_hi=16, block=64, low_bits=4)),
    ("kda64_int4_ef", dict(B=2, H=3, d=64, k_hi=8, block=64, mode="errfeedback", low_bits=4)),
    ("kda32_int4", dict(B=2, H=2, d=32, k_hi=4, block=32, low_bits=4)),
    ("kda32_nohad_int4_sr", dict(B=2, H=2, d=32, k_hi=4, block=32, hadamard=0, mode="stochastic",
                                 low_bits=4)),
    ("kda32_int4_dm", dict(B=2, H=2, d=32, k_hi=8, block=32, mode="direction", low_bits=4)),
    ("kda32_nohad_int4_rm3", dict(B=2, H=2, d=32, k_hi=4, block=32, hadamard=0, mode="residual3",
                                  low_bits=4)),
    ("gdn128_int4", dict(B=3, H=4, Hk=2, d=128, k_hi=0, block=128, decay_per_key=0, low_bits=4)),
    ("gdn128_int4_rm2", dict(B=3, H=4, Hk=2, d=128, k_hi=0, block=128, decay_per_key=0, mode="residual2",
                             low_bits=4)),
])
def test_small_configs_bit_exact(name, kw):
    w = synth.Workload(name, T=12, seed=7, **kw)
    perm = random_perm(w, seed=3)
    steps = _run_both(w, w.T, perm=perm, init_scale=0.05)
    _compare(w, steps)


@pytest.mark.parametrize("mode", ["direction", "residual2", "residual4"])
def test_kda_decode_aux_memory_full_size_sampled(mode):
    """Direction-memory and residual-memory write-back at the KDA decode
    size (B=64, H=32, d=128; the general kernel) for 16 tokens from a
    nonzero state; the oracle runs 64 of the 2048 heads, whose codes, grids
    and auxiliary states (2-bit counters, k-bit residual integers) must
    match."""
    import dataclasses
    w = dataclasses.replace(synth.WORKLOADS["kda_decode"], mode=mode)
    perm = random_perm(w, seed=6)
    units = (500, 564)
    steps = _run_both(w, 16, perm=perm, units=units, init_scale=0.05)
    _compare(w, steps, units=units)
    nel = (w.d - w.k_hi) * w.d // (4 if mode == "direction" else 2)
    for *_, ag, ao in steps:
        np.testing.assert_array_equal(ag[units[0] * nel: units[1] * nel], ao[units[0] * nel: units[1] * nel])


def test_kda_decode_int4_full_size_sampled():
    """The 4-bit low tier at the KDA decode size (B=64, H=32, d=128, k_hi=16,
    block 128; the general kernel) for 16 tokens from a nonzero state: codes,
    FP16 rows and grids of 64 of the 2048 heads match the oracle."""
    import dataclasses
    w = dataclasses.replace(synth.WORKLOADS["kda_decode"], low_bits=4)
    perm = random_perm(w, seed=8)
    units = (1200, 1264)
    steps = _run_both(w, 16, perm=perm, units=units, init_scale=0.05)
    _compare(w, steps, units=units)


@pytest.mark.parametrize("low_bits", [8, 4])
def test_unpack_matches_oracle(low_bits):
    import torch
    from bit_recurrent_state_b200 import brs
    from bit_recurrent_state_b200.state import LayerState
    from oracle import oracle as O
    w = synth.Workload("u", B=2, H=3, d=128, T=1, k_hi=16, block=32, low_bits=low_bits)
    perm = random_perm(w, seed=9)
    cfg = oracle_cfg(w)
    S0 = np.random.default_rng(4).standard_normal((w.B, w.H, w.d, w.d)).astype(np.float32)
    st = LayerState(brs.layout_of(w), perm=perm)
    st.pack(torch.from_numpy(S0).cuda())
    Sg = st.unpack().cpu().numpy()
    So, _ = O.state_unpack(cfg, st.packed.cpu().numpy(), perm)
    np.testing.assert_array_equal(Sg.view(np.uint32), So.view(np.uint32))


def test_nonfinite_input_raises_flag():
    import torch
    from bit_recurrent_state_b200 import brs
    from bit_recurrent_state_b200.state import LayerState
    w = synth.Workload("nf", B=1, H=2, d=128, T=1, k_hi=16, block=128)
    st = LayerState(brs.layout_of(w))
    st.zero()
    dev = to_dev(synth.token_inputs(w, 0))
    dev["beta"][0, 1] = float("nan")
    o = torch.zeros((1, 2, 128), device="cuda")
    st.step(brs.writeback_of(w), 0, dev["q"], dev["k"], dev["v"], dev["beta"], dev["decay"], o)
    assert st.errors() & brs.FLAG_NONFINITE
    assert st.errors() == 0          # cleared by the first read


def test_argument_errors():
    import torch
    from bit_recurrent_state_b200 import brs
    w = synth.Workload("e", B=1, H=2, d=128, T=1, k_hi=16, block=128)
    L = brs.layout_of(w, d=96)
    with pytest.raises(brs.BrsError) as e:
        brs.state_bytes(L)
    assert "d must be" in str(e.value)
    L = brs.layout_of(w)
    buf = torch.zeros(1 << 20, dtype=torch.uint8, device="cuda")
    with pytest.raises(brs.BrsError) as e:
        brs.decode_step(L, brs.writeback_of(w), 0, buf[1:], buf, None, None, buf, None, buf, buf,
                        buf, buf, buf, buf)
    assert e.value.status == brs.EALIGN
    with pytest.raises(brs.BrsError) as e:
        brs.decode_step(L, brs.writeback_of(w, C=4), 0, buf, buf, None, None, buf, None, buf, buf,
                        buf, buf, buf, buf)
    assert e.value.status == brs.EUNSUPPORTED


def test_bounded_copy_wait_runs_out():
    """The decode kernel's waits on its shared-memory copies are bounded.
    With the test hook on, each head's copy barrier expects 16 bytes more
    than its copies deliver: the copies complete, the barrier never does,
    every wait runs out, the kernel raises the timeout flag and returns
    without writing the stored state or o.  The context stays usable: the
    next step, hook off, matches the oracle."""
    import torch
    from bit_recurrent_state_b200 import brs
    from bit_recurrent_state_b200.state import LayerState
    from oracle import oracle as O
    w = synth.Workload("to", B=1, H=4, d=128, T=1, k_hi=16, block=128, seed=41)
    perm = random_perm(w, seed=13)
    L, wb = brs.layout_of(w), brs.writeback_of(w)
    S0 = (np.random.default_rng(3).standard_normal((w.B, w.H, w.d, w.d)) * 0.1).astype(np.float32)
    st = LayerState(L, perm=perm)
    st.pack(torch.from_numpy(S0).cuda())
    before = st.packed.clone()
    dev = to_dev(synth.token_inputs(w, 0))
    o = torch.full((w.B, w.H, w.d), 7.0, device="cuda")
    brs.test_starve_copies(True)
    try:
        st.step(wb, 0, dev["q"], dev["k"], dev["v"], dev["beta"], dev["decay"], o)
    finally:
        brs.test_starve_copies(False)
    torch.cuda.synchronize()
    assert st.errors() & brs.FLAG_TIMEOUT
    assert torch.equal(st.packed, before)
    assert bool(torch.all(o == 7.0))
    # hook off: the same step now runs and matches the oracle
    cfg = oracle_cfg(w)
    packed_o, _ = O.state_pack(cfg, S0, perm)
    st.step(wb, 0, dev["q"], dev["k"], dev["v"], dev["beta"], dev["decay"], o)
    inp = synth.token_inputs(w, 0)
    oo, fl, _ = O.run(cfg, O.ROUND_NEAREST, w.seed, 1, 0, {k: v[None] for k, v in inp.items()}, packed_o,
                      perm=perm)
    assert fl == 0 and st.errors() == 0
    np.testing.assert_array_equal(st.packed.cpu().numpy(), packed_o)
    assert np.max(np.abs(o.cpu().numpy() - oo[0])) <= o_tolerance(oo[0])
