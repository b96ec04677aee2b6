"""Synthetic studies of write-back error ("Low-Bit Recurrent States in Hybrid
Language Models", Correlated rounding errors and Approximate erasure rate),
computed from the oracle: plain FP64 numpy over the oracle's own runs.

Test infrastructure, like the rest of oracle/: only tests/, the package's
smoke check and bench.py's CPU baselines may import it.

Study A, correlated rounding errors.  A layer runs T tokens twice from the
same zero state on the same inputs: once with FP32 storage (the reference)
and once with variable-width storage at a fixed width b for every row
(write-back every token, nearest rounding).  At token t the write-back
error is e_t = Q(y_t) - y_t, with y_t the FP32 state the quantized run held
before its write-back (the stored state of t - 1, dequantized, advanced by
one FP32 token).  Reported:
  - the lag-one autocorrelation of e_t of every element (centred on the
    element's mean over the run), averaged per row, and the row decay s_i;
  - the readout error: the mean over tokens of ||o_q(t) - o_ref(t)||^2,
    against the prediction of the independent-noise model, in which every
    write-back adds to row i an independent error of variance
    sigma_i^2 = Delta_i^2 / 12 (Delta_i the row's stored step at that
    write-back) that propagates through F_t = (I - beta_t k_t k_t^T) D_t:
    P_t = F_t P_{t-1} F_t^T + diag(sigma_t^2), and the readout of token t
    sees d_v q_t^T F_t P_{t-1} F_t^T q_t (outputs precede quantization).

Study B, approximate versus exact erasure rates.  For a head whose rows
have decays s_i and whose keys are either fresh every token or one fixed
key, the exact erasure rate of row i is the diagonal of the observability
Gramian, sum over lags l >= 1 of ||F_{t+l} ... F_{t+1} e_i||^2, averaged
over start tokens t; the approximate rate is Gamma_hat = 1 / (C expm1(2 (s
+ r))) with r = E[beta (2 - beta) k_i^2] / 2.  Both are allocated at the
same budget; the allocation distortion sum Gamma_i 4^(-b_i) is evaluated
under the exact rates, and the excess of the approximate allocation over
the exact one is reported.
"""
from __future__ import annotations

import numpy as np

from . import oracle as O


# ---------------------------------------------------------------- helpers
def _bf16(bits):
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def transitions(inp: dict, b: int, h: int, H: int, Hk: int) -> np.ndarray:
    """F_t = (I - beta_t k_t k_t^T) D_t of head (b, h) for every token of a
    token-major input stack: [T][d][d] in FP64."""
    k = _bf16(inp["k"][:, b, h * Hk // H])                      # [T][d]
    beta = inp["beta"][:, b, h].astype(np.float64)
    dec = inp["decay"][:, b, h].astype(np.float64)
    T, d = k.shape
    a = dec if dec.ndim == 2 else np.repeat(dec[:, None], d, axis=1)
    eye = np.eye(d)
    return (eye[None] - beta[:, None, None] * k[:, :, None] * k[:, None, :]) * a[:, None, :]


def lag1_autocorrelation(sum1, sum2, cross, first, last, n):
    """Centred lag-one autocorrelation of series of n values from their
    running sums: sum1 = sum e_t, sum2 = sum e_t^2 (t < n), cross = sum
    e_t e_(t+1) (t < n - 1), first = e_0, last = e_(n-1); elementwise."""
    m = sum1 / n
    num = cross - m * (sum1 - last) - m * (sum1 - first) + (n - 1) * m * m
    den = sum2 - n * m * m
    with np.errstate(invalid="ignore", divide="ignore"):
        return np.where(den > 0, num / np.where(den > 0, den, 1.0), 0.0)


def readout_model(F: np.ndarray, q: np.ndarray, sigma2: np.ndarray, d_v: int) -> np.ndarray:
    """Independent-noise readout error of one head: F [T][d][d], q [T][d]
    (FP64), sigma2 [T][d] (row variances added by the write-back after token
    t).  Returns [T]: the expected ||o error||^2 of each token's readout."""
    T, d, _ = F.shape
    P = np.zeros((d, d))
    out = np.zeros(T)
    for t in range(T):
        G = F[t] @ P @ F[t].T
        out[t] = d_v * float(q[t] @ G @ q[t])
        P = G + np.diag(sigma2[t])
    return out


def gramian_diag(F: np.ndarray, starts, lags: int) -> np.ndarray:
    """Diagonal of the observability Gramian: for each start token t the sum
    over l = 1..lags of the squared column norms of F_(t+l) ... F_(t+1),
    averaged over the starts.  F [T][d][d]."""
    d = F.shape[1]
    acc = np.zeros(d)
    for t0 in starts:
        M = np.eye(d)
        for l in range(1, lags + 1):
            M = F[t0 + l] @ M
            acc += np.sum(M * M, axis=0)
    return acc / len(starts)


def approx_gamma(inp: dict, b: int, h: int, H: int, Hk: int, C: int = 1) -> np.ndarray:
    """Gamma_hat of every row of head (b, h) from the run's means of a^2 and
    beta (2 - beta) k^2 (the expectations of the pages' formula)."""
    k = _bf16(inp["k"][:, b, h * Hk // H])
    beta = inp["beta"][:, b, h].astype(np.float64)
    dec = inp["decay"][:, b, h].astype(np.float64)
    a2 = dec ** 2 if dec.ndim == 2 else np.repeat(dec[:, None] ** 2, k.shape[1], axis=1)
    A = a2.mean(axis=0)
    K = ((beta * (2.0 - beta))[:, None] * k * k).mean(axis=0)
    return np.array([O.gamma_hat(float(A[i]), float(K[i]), C) for i in range(k.shape[1])])


def allocation_excess(gamma_exact, gamma_approx, avg_bits, b_min, b_max, allocate=None):
    """(widths from the exact rates, widths from the approximate rates, the
    approximate allocation's distortion over the exact one's minus 1), the
    distortion sum Gamma_exact 4^(-b) in both cases."""
    allocate = allocate or (lambda c: O.allocate_bits(c, avg_bits, b_min, b_max)[0])
    be = np.asarray(allocate(np.asarray(gamma_exact, np.float64)), np.int64)
    ba = np.asarray(allocate(np.asarray(gamma_approx, np.float64)), np.int64)
    g = np.asarray(gamma_exact, np.float64)
    de = float(np.sum(g * 4.0 ** (-be)))
    da = float(np.sum(g * 4.0 ** (-ba)))
    return be, ba, da / de - 1.0


# ---------------------------------------------------------------- study A
def rounding_study(w, T: int, bits: int, burn_in: int = 0) -> dict:
    """Study A on the oracle.  w: a synth.Workload (d, B, H, Hk, decays,
    keys, seed); the quantized run stores every row at `bits` bits.
    Returns per-head arrays: corr [B][H][d] (row means of the elements'
    lag-one autocorrelations), s [B][H][d] (row decay rates), readout
    [B][H] (measured mean squared readout error), model [B][H]."""
    from bit_recurrent_state_b200 import synth
    B, H, Hk, d = w.B, w.H, w.hk, w.d
    cq = O.Config(B=B, H=H, Hk=Hk, d=d, storage=O.STORE_VARBIT, hadamard=0, decay_per_key=w.decay_per_key,
                  avg_bits=float(bits), b_min=bits, b_max=bits, budget_scope=1)
    cf = O.Config(B=B, H=H, Hk=Hk, d=d, storage=O.STORE_FP32, hadamard=0, decay_per_key=w.decay_per_key)
    inp = synth.run_inputs(w, 0, T)
    pq, aux, stats = O.new_state(cq)
    pref, _, _ = O.new_state(cf)
    n = T - burn_in
    s1 = np.zeros((B, H, d, d)); s2 = np.zeros_like(s1); cr = np.zeros_like(s1)
    first = np.zeros_like(s1); prev = np.zeros_like(s1)
    sig2 = np.zeros((T, B, H, d))
    err = np.zeros((T, B, H))
    for t in range(T):
        tok = {k: v[t:t + 1] for k, v in inp.items()}
        o_ref, fl, _ = O.run(cf, O.ROUND_NEAREST, 0, 1, t, tok, pref)
        assert fl == 0
        # y_t: the quantized run's stored state, dequantized, advanced one FP32 token
        Sq, _ = O.state_unpack(cq, pq)
        py, _ = O.state_pack(cf, Sq)
        o_q, fl, _ = O.run(cf, O.ROUND_NEAREST, 0, 1, t, tok, py)
        assert fl == 0
        y, _ = O.state_unpack(cf, py)
        o_q2, fl, _ = O.run(cq, O.ROUND_NEAREST, 0, 1, t, tok, pq, aux=aux, stats=stats)
        assert fl == 0
        assert np.array_equal(o_q, o_q2)           # outputs precede quantization
        Sq, _ = O.state_unpack(cq, pq)
        e = Sq.astype(np.float64) - y.astype(np.float64)
        steps = _row_steps(pq, B, H, d, bits)
        sig2[t] = steps ** 2 / 12.0
        err[t] = np.sum((o_q2[0].astype(np.float64) - o_ref[0].astype(np.float64)) ** 2, axis=-1)
        if t >= burn_in:
            s1 += e; s2 += e * e
            if t == burn_in:
                first = e.copy()
            else:
                cr += prev * e
            prev = e
    corr = lag1_autocorrelation(s1, s2, cr, first, prev, n).mean(axis=-1)
    model = np.zeros((B, H))
    for b in range(B):
        for h in range(H):
            F = transitions(inp, b, h, H, Hk)
            q = _bf16(inp["q"][:, b, h * Hk // H])
            model[b, h] = readout_model(F, q, sig2[:, b, h], d).mean()
    dec0 = inp["decay"][0].astype(np.float64)                  # [B][H][d] (KDA) or [B][H] (GDN)
    if dec0.ndim == 2:
        dec0 = np.repeat(dec0[..., None], d, axis=2)
    return dict(corr=corr, s=-np.log(dec0), readout=err.mean(axis=0), model=model)


def _row_steps(packed, B, H, d, bits):
    """Stored FP16 step of every row of a uniform-width variable-width state."""
    rows = H * d
    P = d // 8 * bits * rows
    off = (P * B + 255) // 256 * 256
    st = np.frombuffer(packed[off: off + rows * B * 2].tobytes(), np.float16).astype(np.float64)
    return st.reshape(B, H, d)
