"""The allocation-free decode entry point (brs_decode_step_noalloc), for
callers that cannot allocate device memory (a framework whose allocator owns
the device, a serving loop with a fixed memory budget): it takes no
workspace and uses a static scratch array inside the library.  Checked
against the regular entry point, which takes a caller-allocated workspace,
on two calls in a row.  Collected last on purpose."""
import numpy as np
import pytest

from bit_recurrent_state_b200 import synth

pytestmark = pytest.mark.gpu


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
        inp = synth.token_inputs(w, t)
        dev = {k: torch.from_numpy(v.view(np.int16) if v.dtype == np.uint16 else v).cuda()
               for k, v in inp.items()}
        ref.step(wb, t, dev["q"], dev["k"], dev["v"], dev["beta"], dev["decay"], o_ref)
        brs.decode_step_noalloc(L, wb, t, na.packed, na.packed, na.aux, na.stats, na.perm, dev["q"],
                                dev["k"], dev["v"], dev["beta"], dev["decay"], o_na)
        torch.cuda.synchronize()
        rms = float(torch.sqrt(torch.mean(o_ref.double() ** 2)))
        assert float(torch.max(torch.abs(o_na - o_ref))) <= 2e-3 * rms
        assert torch.equal(na.packed, ref.packed), f"stored state differs after call {t + 1}"
    assert ref.errors() == 0


def test_noalloc_rejects_layout_beyond_static_scratch():
    from bit_recurrent_state_b200 import brs
    w = synth.Workload("big", B=2, H=4, d=128, T=1, storage="varbit", hadamard=0)
    L = brs.layout_of(w)
    n, aux, st, ws = brs.state_bytes(L)
    if ws <= 4096:
        pytest.skip("no layout with a workspace beyond the static scratch yet")
    with pytest.raises(brs.BrsError) as e:
        brs.decode_step_noalloc(L, brs.writeback_of(w), 0, 16, 16, 16, 16, None, 16, 16, 16, 16, 16, 16)
    assert "static array" in str(e.value)
