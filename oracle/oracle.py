"""Python access to the plain CPU oracle (``brs_oracle.c``).

TEST INFRASTRUCTURE ONLY: tests/, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may use this
module; the product path (``bit_recurrent_state_b200``) never imports it.

The oracle is compiled from source with gcc (``-O2 -ffp-contract=off``, no
fast-math) into ``oracle/liboracle.so``; ``build()`` does that and the module
rebuilds on import when the library is missing or older than its source.
Every wrapper takes and returns numpy arrays; the C functions release the GIL
(ctypes does), so ``run_parallel`` spreads independent units over threads.
"""
from __future__ import annotations

import ctypes as ct
import os
import subprocess
import threading
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "brs_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

STORE_FP32, STORE_DAMP, STORE_VARBIT, STORE_VARBIT_HEAD = 0, 1, 2, 3
ROUND_NEAREST, ROUND_STOCHASTIC, ROUND_ERRFEEDBACK, ROUND_DIRECTION = 0, 1, 2, 3
ROUND_RESIDUAL2, ROUND_RESIDUAL3, ROUND_RESIDUAL4 = 4, 5, 6
DOMAIN_CANONICAL, DOMAIN_ROTATED, DOMAIN_MIXED = 0, 1, 2
OK, EINVAL, ENONFINITE, EOVERFLOW = 0, 1, 2, 4


def build(force: bool = False) -> str:
    """Compile liboracle.so from brs_oracle.c (plain gcc, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < max(
        os.path.getmtime(_SRC), os.path.getmtime(os.path.join(_HERE, "brs_oracle.h"))
    ):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fPIC",
             "-shared", "-Wall", "-o", tmp, _SRC, "-lm"]
        )
        os.replace(tmp, _LIB)
    return _LIB


class Layout(ct.Structure):
    _fields_ = [
        ("B", ct.c_int), ("H", ct.c_int), ("Hk", ct.c_int), ("d", ct.c_int),
        ("storage", ct.c_int), ("k_hi", ct.c_int), ("block", ct.c_int),
        ("hadamard", ct.c_int), ("decay_per_key", ct.c_int),
        ("avg_bits", ct.c_double), ("b_min", ct.c_int), ("b_max", ct.c_int),
        ("budget_scope", ct.c_int), ("domain", ct.c_int), ("persistence", ct.c_int),
        ("low_bits", ct.c_int),
    ]


class WriteBack(ct.Structure):
    _fields_ = [("mode", ct.c_int), ("seed", ct.c_uint64), ("C", ct.c_int)]


_lib = None
_lock = threading.Lock()


def lib():
    global _lib
    with _lock:
        if _lib is None:
            build()
            L = ct.CDLL(_LIB)
            P = ct.c_void_p
            L.orc_f16_from_f32.restype = ct.c_uint16
            L.orc_f16_from_f32.argtypes = [ct.c_float]
            L.orc_f32_from_f16.restype = ct.c_float
            L.orc_f32_from_f16.argtypes = [ct.c_uint16]
            L.orc_philox4x32_10.argtypes = [P, P, P]
            L.orc_fwht.argtypes = [P, ct.c_int]
            L.orc_hadamard_scale.restype = ct.c_float
            L.orc_hadamard_scale.argtypes = [ct.c_int]
            L.orc_int8_block.restype = ct.c_int
            L.orc_int8_block.argtypes = [P, ct.c_int, ct.c_int, ct.c_uint64, ct.c_int64, ct.c_int,
                                         ct.c_int, ct.c_int, P, P, P, P, P]
            L.orc_lowbit_block.restype = ct.c_int
            L.orc_lowbit_block.argtypes = [P, ct.c_int, ct.c_int, ct.c_int, ct.c_uint64, ct.c_int64, ct.c_int,
                                           ct.c_int, ct.c_int, P, P, P, P, P]
            L.orc_int8_block_dm.restype = ct.c_int
            L.orc_int8_block_dm.argtypes = [P, P, ct.c_int, P, P, P, P, P]
            L.orc_int8_block_rm.restype = ct.c_int
            L.orc_int8_block_rm.argtypes = [P, ct.c_int, ct.c_int, ct.c_float, P, P, P, P, P]
            L.orc_persistence.restype = ct.c_double
            L.orc_persistence.argtypes = [ct.c_int, ct.c_double, ct.c_double, ct.c_int]
            L.orc_varbit_group.restype = ct.c_int
            L.orc_varbit_group.argtypes = [P, ct.c_int, ct.c_int, ct.c_int, ct.c_uint64, ct.c_int64,
                                           ct.c_int, ct.c_int, ct.c_int, ct.c_int, P, P, P, P, P]
            L.orc_varbit_row.restype = ct.c_int
            L.orc_varbit_row.argtypes = [P, ct.c_int, ct.c_int, ct.c_int, ct.c_uint64, ct.c_int64,
                                         ct.c_int, ct.c_int, ct.c_int, P, P, P, P, P]
            L.orc_gamma_hat.restype = ct.c_double
            L.orc_gamma_hat.argtypes = [ct.c_double, ct.c_double, ct.c_int]
            L.orc_allocate_bits.restype = ct.c_int
            L.orc_allocate_bits.argtypes = [ct.c_int, P, ct.c_double, ct.c_int, ct.c_int, P]
            L.orc_state_bytes.restype = ct.c_size_t
            L.orc_state_bytes.argtypes = [P, P, P]
            L.orc_bits_per_value.restype = ct.c_double
            L.orc_bits_per_value.argtypes = [P]
            L.orc_state_pack.restype = ct.c_int
            L.orc_state_pack.argtypes = [P, P, P, P, P]
            L.orc_state_unpack.restype = ct.c_int
            L.orc_state_unpack.argtypes = [P, P, P, P]
            L.orc_run.restype = ct.c_int
            L.orc_run.argtypes = [P, P, ct.c_int64, ct.c_int, ct.c_int, ct.c_int, P, P, P, P, P,
                                  P, P, P, P, P, P, P, P]
            L.orc_damp_writeback.restype = ct.c_int
            L.orc_damp_writeback.argtypes = [P, P, ct.c_int64, ct.c_int, ct.c_int, P, P, P]
            L.orc_calibrate.restype = ct.c_int
            L.orc_calibrate.argtypes = [P, ct.c_int, ct.c_int, ct.c_int, ct.c_double, P, P, P, P,
                                        P, P, P]
            _lib = L
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(ct.c_void_p)


def _c(a, dtype):
    return None if a is None else np.ascontiguousarray(a, dtype=dtype)


@dataclass
class Config:
    """A state layout in the oracle's own terms (mirrors the library's)."""
    B: int
    H: int
    d: int
    Hk: int = 0
    storage: int = STORE_DAMP
    k_hi: int = 0
    block: int = 128
    hadamard: int = 1
    decay_per_key: int = 1
    avg_bits: float = 4.0
    b_min: int = 2
    b_max: int = 8
    budget_scope: int = 1
    domain: int = DOMAIN_CANONICAL
    persistence: int = 0
    low_bits: int = 8

    def layout(self) -> Layout:
        return Layout(self.B, self.H, self.Hk or self.H, self.d, self.storage, self.k_hi,
                      self.block, self.hadamard, self.decay_per_key, self.avg_bits, self.b_min,
                      self.b_max, self.budget_scope, self.domain, self.persistence, self.low_bits)


# ---------------------------------------------------------------- scalars
def f16_from_f32(x: np.ndarray) -> np.ndarray:
    L = lib()
    x = np.asarray(x, dtype=np.float32).ravel()
    return np.array([L.orc_f16_from_f32(float(v)) for v in x], dtype=np.uint16)


def f32_from_f16(h: np.ndarray) -> np.ndarray:
    L = lib()
    h = np.asarray(h, dtype=np.uint16).ravel()
    return np.array([L.orc_f32_from_f16(int(v)) for v in h], dtype=np.float32)


def philox(ctr, key) -> np.ndarray:
    c = np.asarray(ctr, dtype=np.uint32).copy()
    k = np.asarray(key, dtype=np.uint32).copy()
    out = np.zeros(4, dtype=np.uint32)
    lib().orc_philox4x32_10(_p(c), _p(k), _p(out))
    return out


def fwht(x: np.ndarray) -> np.ndarray:
    y = np.array(x, dtype=np.float32).copy()
    lib().orc_fwht(_p(y), y.size)
    return y


def hadamard_scale(n: int) -> float:
    return lib().orc_hadamard_scale(n)


def int8_block(y, mode=ROUND_NEAREST, seed=0, step=0, h=0, b=0, elem0=0, e=None):
    y = _c(y, np.float32)
    n = y.size
    codes = np.zeros(n, np.uint8)
    sh = np.zeros(1, np.uint16)
    zh = np.zeros(1, np.uint16)
    t = np.zeros(n, np.float32)
    e = None if e is None else np.array(e, dtype=np.uint16)
    fl = lib().orc_int8_block(_p(y), n, mode, seed, step, h, b, elem0, _p(e), _p(codes), _p(sh),
                              _p(zh), _p(t))
    return dict(codes=codes, scale=sh[0], zero=zh[0], t=t, e=e, flags=fl)


def lowbit_block(y, levels, mode=ROUND_NEAREST, seed=0, step=0, h=0, b=0, elem0=0, e=None):
    """One asymmetric block with levels + 1 codes (255: INT8, 15: INT4)."""
    y = _c(y, np.float32)
    n = y.size
    codes = np.zeros(n, np.uint8)
    sh = np.zeros(1, np.uint16)
    zh = np.zeros(1, np.uint16)
    t = np.zeros(n, np.float32)
    e = None if e is None else np.array(e, dtype=np.uint16)
    fl = lib().orc_lowbit_block(_p(y), n, int(levels), mode, seed, step, h, b, elem0, _p(e), _p(codes), _p(sh),
                                _p(zh), _p(t))
    return dict(codes=codes, scale=sh[0], zero=zh[0], t=t, e=e, flags=fl)


def int8_block_dm(y, xprev, m):
    """One INT8 block under direction memory; m (int8 counters in -1..1) is
    returned updated."""
    y = _c(y, np.float32)
    xp = _c(xprev, np.float32)
    n = y.size
    codes = np.zeros(n, np.uint8)
    sh = np.zeros(1, np.uint16)
    zh = np.zeros(1, np.uint16)
    t = np.zeros(n, np.float32)
    m = np.array(m, dtype=np.int8)
    fl = lib().orc_int8_block_dm(_p(y), _p(xp), n, _p(m), _p(codes), _p(sh), _p(zh), _p(t))
    return dict(codes=codes, scale=sh[0], zero=zh[0], t=t, m=m, flags=fl)


def int8_block_rm(y, kbits, sprev, m):
    """One INT8 block under k-bit residual memory: (codes, scale_h, zero_h,
    m_new, flags) for targets y, previous integers m (int8) and the step
    sprev they were stored with."""
    y = _c(y, np.float32)
    m = np.array(m, dtype=np.int8)
    codes = np.zeros(len(y), np.uint8)
    sh, zh = ct.c_uint16(0), ct.c_uint16(0)
    fl = lib().orc_int8_block_rm(_p(y), len(y), int(kbits), float(sprev), _p(m), _p(codes), ct.byref(sh),
                                 ct.byref(zh), None)
    return codes, sh.value, zh.value, m, fl


def varbit_row(x, bw, mode=ROUND_NEAREST, seed=0, step=0, h=0, b=0, elem0=0, e=None):
    x = _c(x, np.float32)
    n = x.size
    q = np.zeros(n, np.int32)
    dh = np.zeros(1, np.uint16)
    ms = np.zeros(1, np.int32)
    t = np.zeros(n, np.float32)
    e = None if e is None else np.array(e, dtype=np.uint16)
    fl = lib().orc_varbit_row(_p(x), n, bw, mode, seed, step, h, b, elem0, _p(e), _p(q), _p(dh),
                              _p(ms), _p(t))
    return dict(q=q, delta=dh[0], m=int(ms[0]), t=t, e=e, flags=fl)


def varbit_group(x, bw, mode=ROUND_NEAREST, seed=0, step=0, h=0, b=0, elem0=0, estride=1, e=None):
    x = _c(x, np.float32)
    n = x.size
    q = np.zeros(n, np.int32)
    dh = np.zeros(1, np.uint16)
    ms = np.zeros(1, np.int32)
    t = np.zeros(n, np.float32)
    e = None if e is None else np.array(e, dtype=np.uint16)
    fl = lib().orc_varbit_group(_p(x), n, bw, mode, seed, step, h, b, elem0, estride, _p(e), _p(q),
                                _p(dh), _p(ms), _p(t))
    return dict(q=q, delta=dh[0], m=int(ms[0]), t=t, e=e, flags=fl)


def gamma_hat(A: float, K: float, C: int) -> float:
    return lib().orc_gamma_hat(A, K, C)


def allocate_bits(c, avg_bits, b_min, b_max):
    c = _c(c, np.float64)
    bits = np.zeros(c.size, np.uint8)
    fl = lib().orc_allocate_bits(c.size, _p(c), avg_bits, b_min, b_max, _p(bits))
    return bits, fl


# ---------------------------------------------------------------- layout
def state_bytes(cfg: Config):
    aux = ct.c_size_t(0)
    st = ct.c_size_t(0)
    L = cfg.layout()
    total = lib().orc_state_bytes(ct.byref(L), ct.byref(aux), ct.byref(st))
    return int(total), int(aux.value), int(st.value)


def bits_per_value(cfg: Config) -> float:
    L = cfg.layout()
    return lib().orc_bits_per_value(ct.byref(L))


def state_pack(cfg: Config, S, perm=None, widths=None):
    L = cfg.layout()
    total, _, _ = state_bytes(cfg)
    packed = np.zeros(total, np.uint8)
    S = _c(S, np.float32)
    perm = _c(perm, np.int16)
    widths = _c(widths, np.uint8)
    fl = lib().orc_state_pack(ct.byref(L), _p(S), _p(perm), _p(widths), _p(packed))
    return packed, fl


def state_unpack(cfg: Config, packed, perm=None):
    L = cfg.layout()
    S = np.zeros((cfg.B, cfg.H, cfg.d, cfg.d), np.float32)
    packed = _c(packed, np.uint8)
    perm = _c(perm, np.int16)
    fl = lib().orc_state_unpack(ct.byref(L), _p(packed), _p(perm), _p(S))
    return S, fl


def new_state(cfg: Config):
    """Zero initial state in the stored format, with zero residuals and stats."""
    total, aux, st = state_bytes(cfg)
    S = np.zeros((cfg.B, cfg.H, cfg.d, cfg.d), np.float32)
    packed, fl = state_pack(cfg, S)
    assert fl == OK
    return packed, np.zeros(aux // 2, np.uint16), np.zeros(max(st // 8, 1), np.float64)


def run(cfg: Config, wb_mode: int, seed: int, C: int, step0: int, inputs: dict, packed, aux=None,
        stats=None, perm=None, units=None, dump_t=False, dump_s=False):
    """Run T tokens (T = inputs['q'].shape[0]) over the given units.

    ``packed``/``aux``/``stats`` are updated in place.  Returns (o, flags,
    t_dump).  ``o`` is [T][B][H][d] and only the rows of the requested units
    are written (the rest stay zero)."""
    L = cfg.layout()
    wb = WriteBack(wb_mode, seed, C)
    q = _c(inputs["q"], np.uint16)
    k = _c(inputs["k"], np.uint16)
    v = _c(inputs["v"], np.uint16)
    beta = _c(inputs["beta"], np.float32)
    decay = _c(inputs["decay"], np.float32)
    T = q.shape[0]
    o = np.zeros((T, cfg.B, cfg.H, cfg.d), np.float32)
    nunits = cfg.B if cfg.storage in (STORE_VARBIT, STORE_VARBIT_HEAD) else cfg.B * cfg.H
    u0, u1 = (0, nunits) if units is None else units
    t = np.zeros(cfg.B * cfg.H * cfg.d * cfg.d, np.float32) if dump_t else None
    sd = np.zeros((cfg.B, cfg.H, cfg.d, cfg.d), np.float32) if dump_s else None
    assert packed.flags["C_CONTIGUOUS"]
    perm = _c(perm, np.int16)
    fl = lib().orc_run(ct.byref(L), ct.byref(wb), step0, T, u0, u1, _p(packed), _p(packed),
                       _p(aux), _p(stats), _p(perm), _p(q), _p(k), _p(v), _p(beta), _p(decay),
                       _p(o), _p(t), _p(sd))
    if dump_s:
        return o, fl, t, sd
    return o, fl, t


def damp_writeback(cfg: Config, wb_mode: int, seed: int, step: int, S, packed, aux=None, units=None):
    """One write-back (the quantizer alone) of the FP32 states S [B][H][d][d]
    (stored row order, the domain's working basis) of the given units into
    ``packed`` (updated in place, as are the residuals / counters ``aux``).
    Returns the flags."""
    L = cfg.layout()
    wb = WriteBack(wb_mode, seed, 1)
    S = _c(S, np.float32)
    u0, u1 = (0, cfg.B * cfg.H) if units is None else units
    assert packed.flags["C_CONTIGUOUS"] and (aux is None or aux.flags["C_CONTIGUOUS"])
    return lib().orc_damp_writeback(ct.byref(L), ct.byref(wb), step, u0, u1, _p(S), _p(packed), _p(aux))


def run_parallel(cfg: Config, wb_mode: int, seed: int, C: int, step0: int, inputs: dict, packed,
                 aux=None, stats=None, perm=None, units=None, threads=None, dump_s=False):
    """``run`` with the units split over threads (units are independent).

    Returns (o, flags, threads_used), and the state dump of ``run`` last when
    ``dump_s`` is set."""
    nunits = cfg.B if cfg.storage in (STORE_VARBIT, STORE_VARBIT_HEAD) else cfg.B * cfg.H
    u0, u1 = (0, nunits) if units is None else units
    nthr = max(1, min(threads or os.cpu_count() or 1, u1 - u0))
    L = cfg.layout()
    wb = WriteBack(wb_mode, seed, C)
    q = _c(inputs["q"], np.uint16)
    k = _c(inputs["k"], np.uint16)
    v = _c(inputs["v"], np.uint16)
    beta = _c(inputs["beta"], np.float32)
    decay = _c(inputs["decay"], np.float32)
    T = q.shape[0]
    o = np.zeros((T, cfg.B, cfg.H, cfg.d), np.float32)
    perm = _c(perm, np.int16)
    bounds = np.linspace(u0, u1, nthr + 1).astype(int)
    sd = np.zeros((cfg.B, cfg.H, cfg.d, cfg.d), np.float32) if dump_s else None

    def work(i):
        return lib().orc_run(ct.byref(L), ct.byref(wb), step0, T, int(bounds[i]),
                             int(bounds[i + 1]), _p(packed), _p(packed), _p(aux), _p(stats),
                             _p(perm), _p(q), _p(k), _p(v), _p(beta), _p(decay), _p(o), None,
                             _p(sd))

    with ThreadPoolExecutor(nthr) as ex:
        flags = list(ex.map(work, range(nthr)))
    fl = 0
    for f in flags:
        fl |= f
    if dump_s:
        return o, fl, nthr, sd
    return o, fl, nthr


def calibrate(cfg: Config, inputs: dict, every: int = 8, tau: float = 1e-3):
    """DAMP protected-row selection on a calibration run; returns (perm, score)."""
    L = cfg.layout()
    q = _c(inputs["q"], np.uint16)
    T, Bc = q.shape[0], q.shape[1]
    perm = np.zeros((cfg.H, cfg.d), np.int16)
    score = np.zeros((cfg.H, cfg.d), np.float64)
    fl = lib().orc_calibrate(ct.byref(L), Bc, T, every, tau, _p(q),
                             _p(_c(inputs["k"], np.uint16)), _p(_c(inputs["v"], np.uint16)),
                             _p(_c(inputs["beta"], np.float32)),
                             _p(_c(inputs["decay"], np.float32)), _p(score), _p(perm))
    assert fl == OK, fl
    return perm, score


def persistence(kind: int, A: float, K: float, C: int) -> float:
    """The allocation cost's row weight (orc_persistence)."""
    return float(lib().orc_persistence(int(kind), float(A), float(K), int(C)))
