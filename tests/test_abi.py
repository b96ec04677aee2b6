"""The C-ABI library loads on a machine without a GPU and exports every
symbol include/brs.h declares (no compute calls)."""
import ctypes
import os
import re

import pytest

from conftest import ROOT


def _declared():
    src = open(os.path.join(ROOT, "include", "brs.h")).read()
    return sorted(set(re.findall(r"\b(brs_[a-z0-9_]+)\s*\(", src)))


def test_header_declarations_exported():
    from bit_recurrent_state_b200 import brs
    import __graft_entry__
    __graft_entry__.build()
    lib = ctypes.CDLL(brs.LIB_PATH)
    names = _declared()
    assert set(brs.SYMBOLS) <= set(names)
    for n in names:
        assert hasattr(lib, n), n


def test_host_only_calls_without_gpu():
    from bit_recurrent_state_b200 import brs, synth
    w = synth.WORKLOADS["kda_decode"]
    n, aux, st, ws = brs.state_bytes(brs.layout_of(w))
    assert n == 18880 * 64 * 32 and aux == 112 * 128 * 2 * 2048 and ws >= 4
    w = synth.WORKLOADS["gdn_decode"]
    assert brs.state_bytes(brs.layout_of(w))[0] == 16896 * 256 * 32
    with pytest.raises(brs.BrsError):
        brs.state_bytes(brs.layout_of(w, H_k=5))
    # the 4-bit low tier: 112 code rows of 64 bytes, the same FP16 rows and grid
    w4 = synth.WORKLOADS["kda_decode"].with_(low_bits=4)
    n4, aux4, _, _ = brs.state_bytes(brs.layout_of(w4))
    assert n4 == (112 * 64 + 16 * 128 * 2 + 112 * 4) * 64 * 32 and aux4 == aux
    assert brs.state_bytes(brs.layout_of(w4, low_bits=0))[0] == 18880 * 64 * 32   # 0 reads as 8
    # per-head widths: payload, steps per (block of 32 keys, column), widths, head offsets
    wh = synth.WORKLOADS["gdn_varbit_decode"]
    nh, auxh, sth, wsh = brs.state_bytes(brs.layout_of(wh))
    heads = 256 * 32
    assert nh == 2048 * 4 * heads + heads * 4 * 128 * 2 + heads + 256 * 33 * 4
    assert auxh == heads * 128 * 128 * 2 and sth == heads * 128 * 16 and wsh == 256 + heads * 8
    for bad, msg in ((dict(b_min=1), "b_min"), (dict(avg_bits=4.01), "integer"), (dict(d=64), "d = 128"),
                     (dict(hadamard=1), "Hadamard")):
        with pytest.raises(brs.BrsError) as e:               # state_bytes reports every layout error as EINVAL
            brs.state_bytes(brs.layout_of(wh.with_(**bad)))
        assert msg in str(e.value), bad
    with pytest.raises(brs.BrsError) as e:
        brs.state_bytes(brs.layout_of(wh, budget_scope=0))
    assert "budget" in str(e.value)


def test_prefill_workspace_size():
    """The prefill's workspace: the 256-byte flag word, the FP32 state
    carried between chunks (B*H*d*d floats), then one u32 hand-over counter
    per head (rounded to 256 bytes); layouts the prefill does not support
    have none."""
    from bit_recurrent_state_b200 import brs, synth
    w = synth.WORKLOADS["kda_prefill"]
    assert brs.prefill_workspace_bytes(brs.layout_of(w)) == 256 + 8 * 32 * 128 * 128 * 4 + 8 * 32 * 4
    with pytest.raises(brs.BrsError) as e:
        brs.prefill_workspace_bytes(brs.layout_of(synth.WORKLOADS["kda_tiny"]))
    assert e.value.status == brs.EUNSUPPORTED
    # the INT4 low tier: the same workspace (the FP32 scratch does not depend on the codes)
    assert brs.prefill_workspace_bytes(brs.layout_of(w, low_bits=4)) == brs.prefill_workspace_bytes(brs.layout_of(w))


def _param_counts():
    src = open(os.path.join(ROOT, "include", "brs.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    out = {}
    for m in re.finditer(r"\b(brs_[a-z0-9_]+)\s*\(([^)]*)\)\s*;", src):
        args = m.group(2).strip()
        out[m.group(1)] = 0 if args in ("", "void") else args.count(",") + 1
    return out


def test_binding_argument_counts_match_header():
    from bit_recurrent_state_b200 import brs
    lib = brs.lib()
    counts = _param_counts()
    assert counts, "no prototypes parsed"
    for name, n in counts.items():
        fn = getattr(lib, name)
        assert fn.argtypes is not None, name
        assert len(fn.argtypes) == n, (name, len(fn.argtypes), n)


def test_deferred_decode_host_checks():
    """Deferred write-back: the interval state's size, and the argument
    errors that return before any device work."""
    from bit_recurrent_state_b200 import brs, synth
    w = synth.WORKLOADS["kda_decode"]
    L = brs.layout_of(w)
    assert brs.decode_state32_bytes(L) == 64 * 32 * 128 * 128 * 4
    with pytest.raises(brs.BrsError) as e:
        brs.decode_state32_bytes(brs.layout_of(synth.WORKLOADS["varbit_decode"]))
    assert e.value.status == brs.EUNSUPPORTED
    p = 1 << 20                      # an aligned address that is never dereferenced on these paths
    args = dict(packed=p, aux=None, workspace=p, perm=None, q=p, k=p, v=p, beta=p, decay=p, o=p)

    def call(wb, step, state32):
        brs.decode_step_deferred(L, wb, step, args["packed"], args["aux"], args["workspace"], state32, args["perm"],
                                 args["q"], args["k"], args["v"], args["beta"], args["decay"], args["o"], stream=0)

    with pytest.raises(brs.BrsError) as e:              # C > 1 needs the interval state
        call(brs.writeback_of(w, C=4), 1, None)
    assert e.value.status == brs.EINVAL
    with pytest.raises(brs.BrsError) as e:              # C >= 1
        call(brs.writeback_of(w, C=0), 0, p)
    assert e.value.status == brs.EINVAL
    with pytest.raises(brs.BrsError) as e:              # 16-byte alignment
        call(brs.writeback_of(w, C=4), 1, p + 4)
    assert e.value.status == brs.EALIGN
    with pytest.raises(brs.BrsError) as e:              # DAMP storage only
        brs.decode_step_deferred(brs.layout_of(synth.WORKLOADS["gdn_decode_fp32"]), brs.writeback_of(w, C=4), 1,
                                 p, None, p, p, None, p, p, p, p, p, p, stream=0)
    assert e.value.status == brs.EUNSUPPORTED


def test_direction_memory_host_checks():
    """Direction memory: the argument errors that return before any device
    work (C = 1 only, DAMP only, the counter buffer required, no prefill)."""
    import dataclasses
    from bit_recurrent_state_b200 import brs, synth
    w = dataclasses.replace(synth.WORKLOADS["kda_decode"], mode="direction")
    L = brs.layout_of(w)
    p = 1 << 20                      # an aligned address that is never dereferenced on these paths
    with pytest.raises(brs.BrsError) as e:              # write-back every token only
        brs.decode_step_deferred(L, brs.writeback_of(w, C=4), 1, p, p, p, p, None, p, p, p, p, p, p, stream=0)
    assert e.value.status == brs.EUNSUPPORTED
    with pytest.raises(brs.BrsError) as e:              # the counters are required
        brs.decode_step(L, brs.writeback_of(w), 0, p, p, None, None, p, None, p, p, p, p, p, p, stream=0)
    assert e.value.status == brs.EINVAL
    wv = dataclasses.replace(synth.WORKLOADS["varbit_decode"], mode="direction")
    with pytest.raises(brs.BrsError) as e:              # DAMP storage only
        brs.decode_step(brs.layout_of(wv), brs.writeback_of(wv), 0, p, p + 16, p, p, p, None, p, p, p, p, p, p,
                        stream=0)
    assert e.value.status == brs.EUNSUPPORTED
    wp = dataclasses.replace(synth.WORKLOADS["kda_prefill"], mode="direction")
    with pytest.raises(brs.BrsError) as e:              # not built for the prefill
        brs.chunk_prefill(brs.layout_of(wp), brs.writeback_of(wp), 0, 64, p, p, p, None, p, p, p, p, p, p,
                          stream=0)
    assert e.value.status == brs.EUNSUPPORTED


def test_argument_errors_before_device_work():
    """Argument errors of the decode and prefill entries come back as a
    status before any device work: unknown rounding modes, the decode's
    write-back interval, required pointers, 16-byte alignment, the missing
    residual buffer of error feedback, unsupported DAMP shapes, and the
    variable-width storage's own rules."""
    import dataclasses
    from bit_recurrent_state_b200 import brs, synth
    p = 1 << 20                      # an aligned address that is never dereferenced on these paths
    w = synth.WORKLOADS["kda_decode"]
    L = brs.layout_of(w)

    def dec(wb, *, L=L, pin=p, pout=p, aux=p, stats=None, ws=p, perm=None, q=p):
        brs.decode_step(L, wb, 0, pin, pout, aux, stats, ws, perm, q, p, p, p, p, p, stream=0)

    def status(fn):
        with pytest.raises(brs.BrsError) as e:
            fn()
        return e.value.status

    for mode in (-1, 7):
        wb = brs.writeback_of(w, mode=mode)
        assert status(lambda: dec(wb)) == brs.EINVAL
        assert status(lambda: brs.decode_step_deferred(L, wb, 0, p, p, p, None, None, p, p, p, p, p, p,
                                                        stream=0)) == brs.EINVAL
    assert status(lambda: dec(brs.writeback_of(w, C=2))) == brs.EUNSUPPORTED          # decode writes back every token
    assert status(lambda: dec(brs.writeback_of(w), q=None)) == brs.EINVAL               # required pointer
    assert status(lambda: dec(brs.writeback_of(w), q=p + 8)) == brs.EALIGN              # 16-byte alignment
    assert status(lambda: dec(brs.writeback_of(w, mode=brs.ROUND_ERRFEEDBACK), aux=None)) == brs.EINVAL
    odd = brs.layout_of(dataclasses.replace(w, block=64))                                # (128, 64) not built
    assert status(lambda: dec(brs.writeback_of(w), L=odd)) == brs.EUNSUPPORTED
    # variable-width storage: packed_out distinct, no permutation, statistics required
    wv = synth.WORKLOADS["varbit_decode"]
    Lv = brs.layout_of(wv)
    assert status(lambda: dec(brs.writeback_of(wv), L=Lv, stats=p)) == brs.EINVAL      # packed_in == packed_out
    assert status(lambda: dec(brs.writeback_of(wv), L=Lv, pout=p + 16, stats=p, perm=p)) == brs.EINVAL
    assert status(lambda: dec(brs.writeback_of(wv), L=Lv, pout=p + 16, stats=None)) == brs.EINVAL
    # prefill: T and step0 multiples of C, known modes
    wp = synth.WORKLOADS["kda_prefill"]
    Lp = brs.layout_of(wp)

    def pre(wb, T=64, step0=0):
        brs.chunk_prefill(Lp, wb, step0, T, p, p, p, None, p, p, p, p, p, p, stream=0)

    assert status(lambda: pre(brs.writeback_of(wp), T=100)) == brs.EINVAL
    assert status(lambda: pre(brs.writeback_of(wp), step0=32)) == brs.EINVAL
    assert status(lambda: pre(brs.writeback_of(wp, mode=7))) == brs.EINVAL
    assert status(lambda: pre(brs.writeback_of(wp, C=32))) == brs.EUNSUPPORTED


def test_allocator_argument_errors():
    """brs_allocate_bits rejects, before any device work: rows not a
    multiple of the group, widths outside 1..16 or crossed, a budget that is
    not an integer number of bits or lies outside [b_min, b_max] per row,
    missing or misaligned device pointers."""
    from bit_recurrent_state_b200 import brs
    lib = brs.lib()
    p = 1 << 20

    def call(n, g, avg, bmin, bmax, cost=p, bits=p, offs=None):
        return lib.brs_allocate_bits(n, g, cost, avg, bmin, bmax, 1, bits, offs, None)

    assert call(100, 64, 4.0, 2, 8) == brs.EINVAL            # 100 rows, groups of 64
    assert call(0, 64, 4.0, 2, 8) == brs.EINVAL
    assert call(128, 64, 4.0, 0, 8) == brs.EINVAL            # b_min >= 1
    assert call(128, 64, 4.0, 2, 17) == brs.EINVAL           # b_max <= 16
    assert call(128, 64, 4.0, 8, 2) == brs.EINVAL            # crossed limits
    assert call(128, 64, 4.01, 2, 8) == brs.EINVAL           # 64 * 4.01 bits is not an integer
    assert call(128, 64, 9.0, 2, 8) == brs.EINVAL            # above b_max per row
    assert call(128, 64, 1.5, 2, 8) == brs.EINVAL            # below b_min per row
    assert call(128, 64, 4.0, 2, 8, cost=None) == brs.EINVAL
    assert call(128, 64, 4.0, 2, 8, bits=None) == brs.EINVAL
    assert call(128, 64, 4.0, 2, 8, cost=p + 8) == brs.EALIGN
    assert call(128, 64, 4.0, 2, 8, offs=p + 4) == brs.EALIGN


def test_layout_and_conversion_argument_errors():
    """Layout validation (shared by every entry) and the state conversion
    and calibration entries' own argument errors."""
    import dataclasses
    from bit_recurrent_state_b200 import brs, synth
    p = 1 << 20
    w = synth.WORKLOADS["kda_decode"]

    def size_status(**kw):
        with pytest.raises(brs.BrsError) as e:
            brs.state_bytes(brs.layout_of(dataclasses.replace(w, **kw)))
        return e.value.status

    assert size_status(d=96) == brs.EINVAL                 # d in {32, 64, 128}
    assert size_status(k_hi=6) == brs.EINVAL               # multiple of 4
    assert size_status(block=48) == brs.EINVAL             # power of two
    assert size_status(block=256) == brs.EINVAL            # at most d
    assert size_status(B=0) == brs.EINVAL
    assert size_status(low_bits=5) == brs.EINVAL           # 8 (or 0) or 4
    wv = synth.WORKLOADS["varbit_decode"]

    def vsize_status(**kw):
        with pytest.raises(brs.BrsError) as e:
            brs.state_bytes(brs.layout_of(dataclasses.replace(wv, **kw)))
        return e.value.status

    with pytest.raises(brs.BrsError) as e:                 # stored without the Hadamard (status from pack)
        brs.state_pack(brs.layout_of(dataclasses.replace(wv, hadamard=1)), p, None, p, p, stream=0)
    assert e.value.status == brs.EUNSUPPORTED and "Hadamard" in str(e.value)
    assert vsize_status(b_min=0) == brs.EINVAL
    assert vsize_status(avg_bits=9.0) == brs.EINVAL        # above b_max
    assert vsize_status(persistence=3) == brs.EINVAL
    L = brs.layout_of(w)
    Lv = brs.layout_of(wv)
    with pytest.raises(brs.BrsError) as e:                 # S required
        brs.state_pack(L, None, None, p, p, stream=0)
    assert e.value.status == brs.EINVAL
    with pytest.raises(brs.BrsError) as e:                 # variable-width rows stay in key-channel order
        brs.state_pack(Lv, p, p, p, p, stream=0)
    assert e.value.status == brs.EINVAL
    with pytest.raises(brs.BrsError) as e:
        brs.state_unpack(Lv, p, p, p, stream=0)
    assert e.value.status == brs.EINVAL
    with pytest.raises(brs.BrsError) as e:                 # 16-byte alignment
        brs.state_unpack(Lv, p + 4, None, p, stream=0)
    assert e.value.status == brs.EALIGN
    # calibration: DAMP layouts only, 0 < every <= T, tau > 0
    assert brs.calibrate_workspace_bytes(L, 4, 64, 8) > 0
    for args, st in [((Lv, 4, 64, 8, 1e-3), brs.EINVAL), ((L, 4, 64, 128, 1e-3), brs.EINVAL),
                     ((L, 4, 64, 8, 0.0), brs.EINVAL), ((L, 0, 64, 8, 1e-3), brs.EINVAL)]:
        with pytest.raises(brs.BrsError) as e:
            brs.calibrate(*args, p, p, p, p, p, p, p, stream=0)
        assert e.value.status == st, args
