"""FP64 brute-force references used to pin the oracle (test-side only).

Written from the matrix form of the update, S <- (I - beta k k^T) Diag(a) S
+ beta k v^T and o = S^T q, and from exhaustive level search, rather than
from the oracle's loop form."""
import numpy as np
from scipy.linalg import hadamard


def bf16_to_f64(bits):
    return (np.asarray(bits, dtype=np.uint32) << 16).view(np.float32).astype(np.float64)


def f16_bits_to_f64(bits):
    return np.asarray(bits, dtype=np.uint16).view(np.float16).astype(np.float64)


def dense_step(S, k, q, v, a, beta):
    """One token on one head in FP64 matrix form.  S is d x d in stored row
    order; k, q, a gathered in the same order."""
    d = S.shape[0]
    A = (np.eye(d) - beta * np.outer(k, k)) @ np.diag(a)
    S = A @ S + beta * np.outer(k, v)
    return S, S.T @ q


def token_vectors(inputs, t, b, h, H, Hk, perm_h, per_key):
    kh = h * Hk // H
    k = bf16_to_f64(inputs["k"][t, b, kh])[perm_h]
    q = bf16_to_f64(inputs["q"][t, b, kh])[perm_h]
    v = bf16_to_f64(inputs["v"][t, b, h])
    a = (inputs["decay"][t, b, h].astype(np.float64)[perm_h] if per_key
         else np.full(len(perm_h), float(inputs["decay"][t, b, h])))
    beta = float(inputs["beta"][t, b, h])
    return k, q, v, a, beta


def hadamard_n(n):
    return hadamard(n).astype(np.float64) / np.sqrt(n)


def damp_head_sections(packed_head, d, k_hi, block, bits=8):
    """Stored head -> (FP16 rows [k_hi][d], codes [d-k_hi][d], (scale, zero)
    [d-k_hi][d/block][2]); low-tier rows come first in stored order, their
    codes one per byte (bits = 8) or two per byte, code j in the low nibble
    for even j (bits = 4)."""
    nb = d // block
    nlo = d - k_hi
    cb = nlo * d * bits // 8
    raw = np.asarray(packed_head[:cb], dtype=np.uint8)
    if bits == 8:
        codes = raw.reshape(nlo, d)
    else:
        codes = np.stack([raw & 15, raw >> 4], axis=-1).reshape(nlo, d)
    f16rows = np.frombuffer(packed_head[cb: cb + k_hi * d * 2].tobytes(), np.uint16).reshape(k_hi, d)
    sz = np.frombuffer(packed_head[cb + k_hi * d * 2:].tobytes(), np.uint16)
    sz = sz.reshape(nlo, nb, 2)
    return f16rows, codes, sz


def damp_dequant64(packed_head, d, k_hi, block, had, bits=8):
    """Stored head -> FP64 canonical state (stored row order)."""
    f16rows, codes, sz = damp_head_sections(packed_head, d, k_hi, block, bits)
    nlo = d - k_hi
    S = np.zeros((d, d))
    S[nlo:] = f16_bits_to_f64(f16rows)
    s = np.repeat(f16_bits_to_f64(sz[:, :, 0]), block, axis=1)
    z = np.repeat(f16_bits_to_f64(sz[:, :, 1]), block, axis=1)
    r = codes.astype(np.float64) * s + z
    S[:nlo] = r @ hadamard_n(d) if had else r
    return S


def int8_nearest64(y, levels=255):
    """FP64 reference of one asymmetric block (levels = 255: INT8, 15: INT4):
    the FP16 step and zero from the block's range, then the nearest of the
    levels + 1 grid points (exhaustive)."""
    mn, mx = y.min(), y.max()
    s = float(np.float16((mx - mn) / levels))
    z = float(np.float16(mn))
    if s == 0:
        return np.zeros(len(y), int), s, z, np.zeros(len(y))
    lev = np.arange(levels + 1) * s + z
    dist = np.abs(y[:, None] - lev[None, :])
    return np.argmin(dist, axis=1), s, z, (y - z) / s


def r256(x):
    return (x + 255) // 256 * 256


def varbit_sections(packed, B, H, d, avg_bits):
    """Split a variable-width state into its documented sections."""
    rows = H * d
    P = int(d // 8 * avg_bits * rows)
    off_scale = r256(P * B)
    off_width = off_scale + r256(rows * B * 2)
    off_offs = off_width + r256(rows * B)
    pay = packed[: P * B].reshape(B, P)
    sc = np.frombuffer(packed[off_scale: off_scale + rows * B * 2].tobytes(), np.uint16).reshape(B, rows)
    wd = packed[off_width: off_width + rows * B].reshape(B, rows)
    of = np.frombuffer(packed[off_offs: off_offs + (rows + 1) * B * 4].tobytes(), np.uint32)
    return pay, sc, wd, of.reshape(B, rows + 1)


def varbit_row_codes(pay_seq, off, bw, d):
    """Unsigned codes of one row from its little-endian bitstream."""
    nbytes = d * bw // 8
    raw = np.unpackbits(pay_seq[off: off + nbytes], bitorder="little")
    return raw.reshape(d, bw) @ (1 << np.arange(bw))


def varbit_head_sections(packed, B, H, d, avg_bits):
    """Split a per-head variable-width state into its documented sections:
    payload [B][P], FP16 steps [B][H][d/32][d], widths [B][H], head offsets
    [B][H+1]."""
    nbk = d // 32
    P = int(d * d // 8 * avg_bits * H)
    off_scale = r256(P * B)
    off_width = off_scale + r256(B * H * nbk * d * 2)
    off_offs = off_width + r256(B * H)
    pay = packed[: P * B].reshape(B, P)
    sc = np.frombuffer(packed[off_scale: off_scale + B * H * nbk * d * 2].tobytes(), np.uint16)
    wd = packed[off_width: off_width + B * H].reshape(B, H)
    of = np.frombuffer(packed[off_offs: off_offs + B * (H + 1) * 4].tobytes(), np.uint32)
    return pay, sc.reshape(B, H, nbk, d), wd, of.reshape(B, H + 1)


def varbit_head_codes(pay_seq, off, bw, d):
    """Unsigned codes [d][d] of one head: element (i, j) at bit (i d + j) bw."""
    nbytes = d * d * bw // 8
    raw = np.unpackbits(pay_seq[off: off + nbytes], bitorder="little")
    return (raw.reshape(d * d, bw) @ (1 << np.arange(bw))).reshape(d, d)
