"""Thin Python binding of the C ABI in include/brs.h (argument marshalling
only; every step of the update runs in the CUDA library libbrs.so).

Functions keep the C names without the ``brs_`` prefix and take torch CUDA
tensors (or raw integer device addresses) for the device pointers; the
stream defaults to torch's current stream.  There is no CPU fallback:
loading fails loudly when libbrs.so is missing.
"""
from __future__ import annotations

import ctypes as ct
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libbrs.so")

STORE_FP32, STORE_DAMP, STORE_VARBIT, STORE_VARBIT_HEAD = 0, 1, 2, 3
ROUND_NEAREST, ROUND_STOCHASTIC, ROUND_ERRFEEDBACK, ROUND_DIRECTION = 0, 1, 2, 3
ROUND_RESIDUAL2, ROUND_RESIDUAL3, ROUND_RESIDUAL4 = 4, 5, 6
OK, EINVAL, EUNSUPPORTED, EALIGN, ECUDA, ENONFINITE, EOVERFLOW, ETIMEOUT = range(8)
FLAG_NONFINITE, FLAG_OVERFLOW, FLAG_TIMEOUT, FLAG_INVALID = 1, 2, 4, 8
MODES = {"nearest": ROUND_NEAREST, "stochastic": ROUND_STOCHASTIC,
         "errfeedback": ROUND_ERRFEEDBACK, "direction": ROUND_DIRECTION,
         "residual2": ROUND_RESIDUAL2, "residual3": ROUND_RESIDUAL3, "residual4": ROUND_RESIDUAL4}
STORES = {"fp32": STORE_FP32, "damp": STORE_DAMP, "varbit": STORE_VARBIT, "varbit_head": STORE_VARBIT_HEAD}

# exported symbols declared in include/brs.h
SYMBOLS = ["brs_state_bytes", "brs_state_pack", "brs_state_unpack", "brs_decode_step",
           "brs_decode_step_noalloc", "brs_chunk_prefill", "brs_allocate_bits", "brs_fetch_errors",
           "brs_last_error", "brs_calibrate_workspace_bytes", "brs_calibrate", "brs_decode_state32_bytes",
           "brs_decode_step_deferred", "brs_prefill_workspace_bytes", "brs_fetch_errors_noalloc",
           "brs_test_starve_copies", "brs_test_prefill_ctas", "brs_test_prefill_withhold"]


class BrsError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"brs status {status}: {msg}")
        self.status = status


class Layout(ct.Structure):
    _fields_ = [("B", ct.c_int32), ("H", ct.c_int32), ("H_k", ct.c_int32), ("d", ct.c_int32),
                ("storage", ct.c_int32), ("k_hi", ct.c_int32), ("block", ct.c_int32),
                ("hadamard", ct.c_int32), ("decay_per_key", ct.c_int32),
                ("avg_bits", ct.c_double), ("b_min", ct.c_int32), ("b_max", ct.c_int32),
                ("budget_scope", ct.c_int32), ("persistence", ct.c_int32), ("low_bits", ct.c_int32)]


class WriteBack(ct.Structure):
    _fields_ = [("mode", ct.c_int32), ("seed", ct.c_uint64), ("C", ct.c_int32)]


def layout_of(w, **override) -> Layout:
    """brs_layout of a synth.Workload (fields may be overridden)."""
    f = dict(B=w.B, H=w.H, H_k=w.hk, d=w.d, storage=STORES[w.storage], k_hi=w.k_hi,
             block=w.block, hadamard=w.hadamard, decay_per_key=w.decay_per_key,
             avg_bits=w.avg_bits, b_min=w.b_min, b_max=w.b_max, budget_scope=1,
             persistence=w.persistence, low_bits=w.low_bits)
    f.update(override)
    return Layout(**f)


def writeback_of(w, **override) -> WriteBack:
    f = dict(mode=MODES[w.mode], seed=w.seed, C=w.C)
    f.update(override)
    return WriteBack(**f)


_lib = None


def lib():
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"CUDA library not built: {LIB_PATH} (run __graft_entry__.build())")
        L = ct.CDLL(LIB_PATH)
        P, S = ct.c_void_p, ct.c_int
        L.brs_state_bytes.restype = ct.c_size_t
        L.brs_state_bytes.argtypes = [P, P, P, P]
        L.brs_state_pack.restype = S
        L.brs_state_pack.argtypes = [P, P, P, P, P, P, P]
        L.brs_state_unpack.restype = S
        L.brs_state_unpack.argtypes = [P, P, P, P, P, P]
        L.brs_decode_step.restype = S
        L.brs_decode_step.argtypes = [P, P, ct.c_int64] + [P] * 13
        L.brs_decode_state32_bytes.restype = ct.c_size_t
        L.brs_decode_state32_bytes.argtypes = [P]
        L.brs_decode_step_deferred.restype = S
        L.brs_decode_step_deferred.argtypes = [P, P, ct.c_int64] + [P] * 12
        L.brs_decode_step_noalloc.restype = S
        L.brs_decode_step_noalloc.argtypes = [P, P, ct.c_int64] + [P] * 12
        L.brs_prefill_workspace_bytes.restype = ct.c_size_t
        L.brs_prefill_workspace_bytes.argtypes = [P]
        L.brs_chunk_prefill.restype = S
        L.brs_chunk_prefill.argtypes = [P, P, ct.c_int64, ct.c_int] + [P] * 12
        L.brs_allocate_bits.restype = S
        L.brs_allocate_bits.argtypes = [ct.c_int, ct.c_int, P, ct.c_double, ct.c_int, ct.c_int,
                                        ct.c_uint32, P, P, P]
        L.brs_calibrate_workspace_bytes.restype = ct.c_size_t
        L.brs_calibrate_workspace_bytes.argtypes = [P, ct.c_int, ct.c_int, ct.c_int]
        L.brs_calibrate.restype = S
        L.brs_calibrate.argtypes = [P, ct.c_int, ct.c_int, ct.c_int, ct.c_double] + [P] * 9
        L.brs_fetch_errors.restype = S
        L.brs_fetch_errors.argtypes = [P, P, P]
        L.brs_fetch_errors_noalloc.restype = S
        L.brs_fetch_errors_noalloc.argtypes = [P, P]
        L.brs_test_starve_copies.restype = None
        L.brs_test_starve_copies.argtypes = [ct.c_int]
        L.brs_test_prefill_ctas.restype = None
        L.brs_test_prefill_ctas.argtypes = [ct.c_int]
        L.brs_test_prefill_withhold.restype = None
        L.brs_test_prefill_withhold.argtypes = [ct.c_int]
        L.brs_last_error.restype = ct.c_char_p
        L.brs_last_error.argtypes = []
        _lib = L
    return _lib


def _ptr(x):
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def last_error() -> str:
    return lib().brs_last_error().decode()


def _check(status: int):
    if status != OK:
        raise BrsError(status, last_error())


def state_bytes(layout: Layout):
    """(state, aux, stats, workspace) byte counts."""
    aux, st, ws = ct.c_size_t(0), ct.c_size_t(0), ct.c_size_t(0)
    n = lib().brs_state_bytes(ct.byref(layout), ct.byref(aux), ct.byref(st), ct.byref(ws))
    if n == 0:
        raise BrsError(EINVAL, last_error())
    return int(n), int(aux.value), int(st.value), int(ws.value)


def state_pack(layout, S, perm, packed, workspace, widths=None, stream=None):
    _check(lib().brs_state_pack(ct.byref(layout), _ptr(S), _ptr(perm), _ptr(widths),
                                _ptr(packed), _ptr(workspace), _stream(stream)))


def state_unpack(layout, packed, perm, S, workspace=None, stream=None):
    _check(lib().brs_state_unpack(ct.byref(layout), _ptr(packed), _ptr(perm), _ptr(S),
                                  _ptr(workspace), _stream(stream)))


def decode_step(layout, wb, step, packed_in, packed_out, aux, stats, workspace, perm, q, k, v,
                beta, decay, o, stream=None):
    _check(lib().brs_decode_step(ct.byref(layout), ct.byref(wb), int(step), _ptr(packed_in),
                                 _ptr(packed_out), _ptr(aux), _ptr(stats), _ptr(workspace),
                                 _ptr(perm), _ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(decay),
                                 _ptr(o), _stream(stream)))


def decode_state32_bytes(layout) -> int:
    """brs_decode_state32_bytes: the FP32 interval state of deferred write-back."""
    n = int(lib().brs_decode_state32_bytes(ct.byref(layout)))
    if n == 0:
        _check(EUNSUPPORTED)
    return n


def decode_step_deferred(layout, wb, step, packed, aux, workspace, state32, perm, q, k, v, beta, decay, o,
                         stream=None):
    """brs_decode_step_deferred: one decode token with write-back every wb.C tokens."""
    _check(lib().brs_decode_step_deferred(ct.byref(layout), ct.byref(wb), int(step), _ptr(packed), _ptr(aux),
                                          _ptr(workspace), _ptr(state32), _ptr(perm), _ptr(q), _ptr(k), _ptr(v),
                                          _ptr(beta), _ptr(decay), _ptr(o), _stream(stream)))


def decode_step_noalloc(layout, wb, step, packed_in, packed_out, aux, stats, perm, q, k, v, beta,
                        decay, o, stream=None):
    """brs_decode_step without a workspace: the library's static scratch is
    used instead (for callers that cannot allocate device memory)."""
    _check(lib().brs_decode_step_noalloc(ct.byref(layout), ct.byref(wb), int(step), _ptr(packed_in),
                                         _ptr(packed_out), _ptr(aux), _ptr(stats), _ptr(perm), _ptr(q),
                                         _ptr(k), _ptr(v), _ptr(beta), _ptr(decay), _ptr(o),
                                         _stream(stream)))


def prefill_workspace_bytes(layout) -> int:
    """brs_prefill_workspace_bytes: flag word + the FP32 state between chunks."""
    n = int(lib().brs_prefill_workspace_bytes(ct.byref(layout)))
    if n == 0:
        raise BrsError(EUNSUPPORTED, last_error())
    return n


def chunk_prefill(layout, wb, step0, T, packed, aux, workspace, perm, q, k, v, beta, decay, o,
                  state_dump=None, stream=None):
    """brs_chunk_prefill: T tokens per sequence, write-back every wb.C tokens."""
    _check(lib().brs_chunk_prefill(ct.byref(layout), ct.byref(wb), int(step0), int(T), _ptr(packed),
                                   _ptr(aux), _ptr(workspace), _ptr(perm), _ptr(q), _ptr(k), _ptr(v),
                                   _ptr(beta), _ptr(decay), _ptr(o), _ptr(state_dump), _stream(stream)))


def allocate_bits(cost, rows_per_group, avg_bits, b_min, b_max, bits_out, offsets_out=None,
                  offset_unit=1, stream=None):
    """brs_allocate_bits on device f64 costs (torch tensor)."""
    _check(lib().brs_allocate_bits(int(cost.numel()), int(rows_per_group), _ptr(cost), float(avg_bits),
                                   int(b_min), int(b_max), int(offset_unit), _ptr(bits_out),
                                   _ptr(offsets_out), _stream(stream)))


def calibrate_workspace_bytes(layout, Bc: int, T: int, every: int) -> int:
    """brs_calibrate_workspace_bytes."""
    return int(lib().brs_calibrate_workspace_bytes(ct.byref(layout), int(Bc), int(T), int(every)))


def calibrate(layout, Bc, T, every, tau, q, k, v, beta, decay, workspace, perm_out, score_out=None,
              stream=None):
    """brs_calibrate: protected-row selection on a calibration batch (token-major inputs)."""
    _check(lib().brs_calibrate(ct.byref(layout), int(Bc), int(T), int(every), float(tau), _ptr(q), _ptr(k),
                               _ptr(v), _ptr(beta), _ptr(decay), _ptr(workspace), _ptr(score_out),
                               _ptr(perm_out), _stream(stream)))


def fetch_errors(workspace, stream=None) -> int:
    """Raw device flag bits (also raises BrsError if any is set)."""
    fl = ct.c_uint32(0)
    st = lib().brs_fetch_errors(_ptr(workspace), ct.byref(fl), _stream(stream))
    if st != OK and fl.value == 0:                 # a call error, not a device flag
        _check(st)
    return int(fl.value)


def fetch_errors_noalloc(stream=None) -> int:
    """Raw device flag bits collected by brs_decode_step_noalloc calls on the
    current device since the last read (also cleared)."""
    fl = ct.c_uint32(0)
    st = lib().brs_fetch_errors_noalloc(ct.byref(fl), _stream(stream))
    if st != OK and fl.value == 0:                 # a call error, not a device flag
        _check(st)
    return int(fl.value)


def test_prefill_ctas(n: int):
    """brs_test_prefill_ctas: cap the prefill's CTAs at n (0: the default),
    so that small batches exercise the hand-over of heads (test hook)."""
    lib().brs_test_prefill_ctas(int(n))


def test_prefill_withhold(on: bool):
    """brs_test_prefill_withhold: the prefill hands no head over, so that the
    bounded hand-over waits run out (test hook)."""
    lib().brs_test_prefill_withhold(1 if on else 0)


def test_starve_copies(on: bool):
    """brs_test_starve_copies: make the decode kernel's bounded copy waits run
    out (test hook)."""
    lib().brs_test_starve_copies(1 if on else 0)
