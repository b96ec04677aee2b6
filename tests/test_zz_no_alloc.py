"""The allocation-free decode entry point (brs_decode_step_noalloc), for
callers that cannot allocate device memory (a framework whose allocator owns
the device, a serving loop with a fixed memory budget): it takes no
workspace and uses a static scratch array inside the library.  Checked
against the regular entry point, which takes a caller-allocated workspace,
on two calls in a row, for a DAMP layout (the scratch holds only the flag
word) and a variable-width layout (the scratch also holds the per-row
allocation costs).  Its device flags are read back through
brs_fetch_errors_noalloc.  Collected last on purpose."""
import numpy as np
import pytest

from bit_recurrent_state_b200 import synth

pytestmark = pytest.mark.gpu


def _dev(inp):
    import torch
    return {k: torch.from_numpy(np.ascontiguousarray(v).view(np.int16) if v.dtype == np.uint16
                                else np.ascontiguousarray(v)).cuda() for k, v in inp.items()}


def _o_close(o_na, o_ref):
    import torch
    rms = float(torch.sqrt(torch.mean(o_ref.double() ** 2)))
    return float(torch.max(torch.abs(o_na - o_ref))) <= 2e-3 * rms


def test_noalloc_matches_regular_entry_two_calls():
    import torch
    from bit_recurrent_state_b200 import brs
    from bit_recurrent_state_b200.state import LayerState

    w = synth.Workload("na", B=3, H=5, d=128, T=2, k_hi=16, block=128, seed=31)
    rng = np.random.default_rng(7)
    perm = np.stack([rng.permutation(w.d) for _ in range(w.H)]).astype(np.int16)
    L, wb = brs.layout_of(w), brs.writeback_of(w)
    S0 = torch.from_numpy((rng.standard_normal((w.B, w.H, w.d, w.d)) * 0.1).astype(np.float32)).cuda()
    ref = LayerState(L, perm=perm)
    ref.pack(S0)
    na = LayerState(L, perm=perm)
    na.pack(S0)
    o_ref = torch.zeros((w.B, w.H, w.d), device="cuda")
    o_na = torch.full((w.B, w.H, w.d), float("nan"), device="cuda")
    for t in range(2):
        dev = _dev(synth.token_inputs(w, t))
        ref.step(wb, t, dev["q"], dev["k"], dev["v"], dev["beta"], dev["decay"], o_ref)
        brs.decode_step_noalloc(L, wb, t, na.packed, na.packed, na.aux, na.stats, na.perm, dev["q"],
                                dev["k"], dev["v"], dev["beta"], dev["decay"], o_na)
        torch.cuda.synchronize()
        assert _o_close(o_na, o_ref)
        assert torch.equal(na.packed, ref.packed), f"stored state differs after call {t + 1}"
    assert ref.errors() == 0
    assert brs.fetch_errors_noalloc() == 0


@pytest.mark.parametrize("mode", ["nearest", "stochastic"])
def test_noalloc_variable_width_matches_regular_entry_two_calls(mode):
    """B=1, H=2: the layout's scratch (flag word + one FP64 cost per row,
    2304 bytes) fits the static array, so the allocation costs go through
    it; packed_out is a second buffer as variable-width decode requires."""
    import torch
    from bit_recurrent_state_b200 import brs
    from bit_recurrent_state_b200.state import LayerState

    w = synth.Workload("nav", B=1, H=2, d=128, T=2, storage="varbit", hadamard=0, avg_bits=4.0,
                       b_min=2, b_max=8, mode=mode, seed=33)
    L, wb = brs.layout_of(w), brs.writeback_of(w)
    assert brs.state_bytes(L)[3] <= 4096
    rng = np.random.default_rng(8)
    S0 = torch.from_numpy((rng.standard_normal((w.B, w.H, w.d, w.d)) * 0.1).astype(np.float32)).cuda()
    ref = LayerState(L)
    ref.pack(S0)
    na = LayerState(L)
    na.pack(S0)
    ref_out, na_out = torch.zeros_like(ref.packed), torch.zeros_like(na.packed)
    o_ref = torch.zeros((w.B, w.H, w.d), device="cuda")
    o_na = torch.full((w.B, w.H, w.d), float("nan"), device="cuda")
    for t in range(2):
        dev = _dev(synth.token_inputs(w, t))
        brs.decode_step(L, wb, t, ref.packed, ref_out, ref.aux, ref.stats, ref.workspace, None, dev["q"],
                        dev["k"], dev["v"], dev["beta"], dev["decay"], o_ref)
        brs.decode_step_noalloc(L, wb, t, na.packed, na_out, na.aux, na.stats, None, dev["q"], dev["k"],
                                dev["v"], dev["beta"], dev["decay"], o_na)
        torch.cuda.synchronize()
        assert _o_close(o_na, o_ref)
        assert torch.equal(na_out, ref_out), f"stored state differs after call {t + 1}"
        assert torch.equal(na.stats, ref.stats)
        ref.packed, ref_out = ref_out, ref.packed
        na.packed, na_out = na_out, na.packed
    assert ref.errors() == 0
    assert brs.fetch_errors_noalloc() == 0


def test_noalloc_flags_reach_the_caller():
    """A non-finite beta makes the kernel raise the non-finite flag in the
    static scratch; brs_fetch_errors_noalloc reports it and clears it."""
    import torch
    from bit_recurrent_state_b200 import brs
    from bit_recurrent_state_b200.state import LayerState

    w = synth.Workload("naf", B=1, H=2, d=128, T=1, k_hi=16, block=128, seed=35)
    L, wb = brs.layout_of(w), brs.writeback_of(w)
    st = LayerState(L)
    st.zero()
    dev = _dev(synth.token_inputs(w, 0))
    dev["beta"][0, 1] = float("nan")
    o = torch.zeros((w.B, w.H, w.d), device="cuda")
    assert brs.fetch_errors_noalloc() == 0
    brs.decode_step_noalloc(L, wb, 0, st.packed, st.packed, st.aux, st.stats, None, dev["q"], dev["k"],
                            dev["v"], dev["beta"], dev["decay"], o)
    assert brs.fetch_errors_noalloc() & brs.FLAG_NONFINITE
    assert brs.fetch_errors_noalloc() == 0


def test_noalloc_rejects_layout_beyond_static_scratch():
    from bit_recurrent_state_b200 import brs
    w = synth.Workload("big", B=2, H=4, d=128, T=1, storage="varbit", hadamard=0)
    L = brs.layout_of(w)
    n, aux, st, ws = brs.state_bytes(L)
    assert ws > 4096
    with pytest.raises(brs.BrsError) as e:
        brs.decode_step_noalloc(L, brs.writeback_of(w), 0, 16, 16, 16, 16, None, 16, 16, 16, 16, 16, 16)
    assert "static array" in str(e.value)
