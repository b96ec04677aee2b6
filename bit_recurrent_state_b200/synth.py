"""Seeded synthetic inputs and the workload table.

This module holds no arithmetic of the method: it only draws inputs with
the shapes and distributions the pages describe and names the workloads.
Both the CUDA path and the oracle consume exactly these arrays.

Distributions (per workload, one seed each):
  q, k   ~ N(0, 1) per element, L2-normalised over the key axis in FP64,
           rounded to bfloat16 (nearest, ties to even);
  v      ~ N(0, 1), rounded to bfloat16;
  beta   = sigmoid(N(0, 1)), FP32;
  s      log-uniform in [1e-3, 1], drawn once per (head, key channel) for
         KDA and once per head for GDN, shared by every sequence and every
         token (the decay ordering is a stable property of the head); the
         decay input is a = exp(-s) in FP32.
Token t's inputs come from a generator seeded with (seed, 1, t), so any
token can be regenerated alone, whatever the run length.
"""
from __future__ import annotations

from dataclasses import dataclass, replace

import numpy as np


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """float -> bfloat16 bit patterns, round to nearest, ties to even (finite
    inputs: the sum below stays under 2^32 for every finite float)."""
    f = np.ascontiguousarray(x, dtype=np.float32)
    u = f.view(np.uint32)
    r = ((u + (np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1)))) >> np.uint32(16)).astype(np.uint16)
    return r


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    d: int
    T: int
    Hk: int = 0
    storage: str = "damp"          # "fp32" | "damp" | "varbit" | "varbit_head"
    k_hi: int = 0
    block: int = 128
    hadamard: int = 1
    decay_per_key: int = 1
    avg_bits: float = 4.0
    b_min: int = 2
    b_max: int = 8
    C: int = 1
    persistence: int = 0              # variable-width cost weight (0 Gamma_hat, 1 w^(1), 2 h^(C))
    low_bits: int = 8                 # DAMP low tier: 8 (INT8) or 4 (two codes per byte)
    s_min: float = 1e-3               # decay rates s log-uniform in [s_min, 1]
    persistent_keys: int = 0          # 1: one fixed key per (sequence, key head) for every token
    mode: str = "nearest"          # "nearest" | "stochastic" | "errfeedback" | "direction"
    seed: int = 0

    @property
    def hk(self) -> int:
        return self.Hk or self.H

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


# The five measured configurations (shapes of the pages' KDA and GDN heads).
WORKLOADS = {
    "kda_tiny": Workload("kda_tiny", B=1, H=2, d=32, T=64, k_hi=4, block=32, seed=0),
    "kda_decode": Workload("kda_decode", B=64, H=32, d=128, T=1024, k_hi=16, block=128, seed=1),
    "gdn_decode": Workload("gdn_decode", B=256, H=32, Hk=16, d=128, T=512, k_hi=0, block=128,
                           decay_per_key=0, seed=2),
    "gdn_decode_fp32": Workload("gdn_decode_fp32", B=256, H=32, Hk=16, d=128, T=512, storage="fp32",
                                hadamard=0, decay_per_key=0, seed=2),
    "varbit_decode": Workload("varbit_decode", B=128, H=32, d=128, T=1024, storage="varbit",
                              hadamard=0, avg_bits=4.0, b_min=2, b_max=8, seed=3),
    "kda_prefill": Workload("kda_prefill", B=8, H=32, d=128, T=8192, k_hi=16, block=128, C=64,
                            seed=4),
    # decode with deferred write-back every 8 tokens (a NEXT configuration)
    "kda_decode_c8": Workload("kda_decode_c8", B=64, H=32, d=128, T=1024, k_hi=16, block=128, C=8, seed=1),
    # GDN heads with one width per head (a NEXT configuration): the GDN decode
    # shape and inputs, 4.0 bits per value on average, widths 2..8
    "gdn_varbit_decode": Workload("gdn_varbit_decode", B=256, H=32, Hk=16, d=128, T=512,
                                  storage="varbit_head", hadamard=0, avg_bits=4.0, b_min=2, b_max=8,
                                  decay_per_key=0, seed=2),
}


def decay_table(w: Workload) -> np.ndarray:
    """a = exp(-s), s log-uniform in [s_min, 1] (s_min = 1e-3 unless the
    workload says otherwise): [H][d] (KDA) or [H] (GDN)."""
    rng = np.random.default_rng([w.seed, 0])
    shape = (w.H, w.d) if w.decay_per_key else (w.H,)
    s = np.exp(rng.uniform(np.log(w.s_min), np.log(1.0), size=shape))
    return np.exp(-s).astype(np.float32)


def token_inputs(w: Workload, t: int, batch: slice | None = None) -> dict:
    """Inputs of token t for the whole batch (or a slice of sequences).

    Shapes: q,k [B][Hk][d] bf16 bits; v [B][H][d] bf16 bits; beta [B][H];
    decay [B][H][d] (KDA) or [B][H] (GDN)."""
    rng = np.random.default_rng([w.seed, 1, t])
    B, H, Hk, d = w.B, w.H, w.hk, w.d
    q = rng.standard_normal((B, Hk, d))
    k = rng.standard_normal((B, Hk, d))
    v = rng.standard_normal((B, H, d))
    beta = 1.0 / (1.0 + np.exp(-rng.standard_normal((B, H))))
    if w.persistent_keys:
        k = np.random.default_rng([w.seed, 2]).standard_normal((B, Hk, d))
    q /= np.linalg.norm(q, axis=-1, keepdims=True)
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    a = decay_table(w)
    decay = np.broadcast_to(a, (B,) + a.shape)
    out = dict(q=bf16_bits(q), k=bf16_bits(k), v=bf16_bits(v), beta=beta.astype(np.float32),
               decay=np.ascontiguousarray(decay, dtype=np.float32))
    if batch is not None:
        out = {key: np.ascontiguousarray(val[batch]) for key, val in out.items()}
    return out


def run_inputs(w: Workload, t0: int, T: int, batch: slice | None = None) -> dict:
    """Tokens [t0, t0+T) stacked token-major: q [T][B][Hk][d] and so on."""
    toks = [token_inputs(w, t0 + t, batch) for t in range(T)]
    return {key: np.stack([tk[key] for tk in toks]) for key in toks[0]}


def calibration_inputs(w: Workload, batch: int = 32, tokens: int = 256) -> dict:
    """Calibration run inputs: fresh q/k/v/beta (seed + 1), the head's own
    decays (seed of the measured workload)."""
    cw = w.with_(B=batch, seed=w.seed + 1)
    out = run_inputs(cw, 0, tokens)
    a = decay_table(w)
    out["decay"] = np.ascontiguousarray(
        np.broadcast_to(a, (tokens, batch) + a.shape), dtype=np.float32)
    return out
