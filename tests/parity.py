"""Shared helpers of the GPU parity tests: the same seeded inputs go to the
CUDA library (through the C ABI) and to the oracle."""
import numpy as np

from bit_recurrent_state_b200 import synth
from oracle import oracle as O

MODE = {"nearest": O.ROUND_NEAREST, "stochastic": O.ROUND_STOCHASTIC,
        "errfeedback": O.ROUND_ERRFEEDBACK, "direction": O.ROUND_DIRECTION,
        "residual2": O.ROUND_RESIDUAL2, "residual3": O.ROUND_RESIDUAL3, "residual4": O.ROUND_RESIDUAL4}
STORE = {"fp32": O.STORE_FP32, "damp": O.STORE_DAMP, "varbit": O.STORE_VARBIT,
         "varbit_head": O.STORE_VARBIT_HEAD}


def oracle_cfg(w: synth.Workload) -> O.Config:
    """The oracle mode the CUDA path follows: DAMP heads are updated in the
    mixed basis (each tier in the basis it is stored in)."""
    return O.Config(B=w.B, H=w.H, Hk=w.hk, d=w.d, storage=STORE[w.storage], k_hi=w.k_hi,
                    block=w.block, hadamard=w.hadamard, decay_per_key=w.decay_per_key,
                    avg_bits=w.avg_bits, b_min=w.b_min, b_max=w.b_max, persistence=w.persistence,
                    low_bits=w.low_bits,
                    domain=O.DOMAIN_MIXED if w.storage == "damp" else O.DOMAIN_CANONICAL)


def random_perm(w: synth.Workload, seed=0):
    rng = np.random.default_rng(1000 + seed)
    return np.stack([rng.permutation(w.d) for _ in range(w.H)]).astype(np.int16)


def to_dev(inp: dict, device="cuda"):
    import torch
    out = {}
    for k, v in inp.items():
        a = np.ascontiguousarray(v)
        if a.dtype == np.uint16:
            a = a.view(np.int16)
        out[k] = torch.from_numpy(a).to(device)
    return out


def o_tolerance(o_ref: np.ndarray) -> float:
    """max |o_gpu - o_oracle| allowed: 2e-3 of the run's output RMS."""
    return 2e-3 * float(np.sqrt(np.mean(o_ref.astype(np.float64) ** 2)))
