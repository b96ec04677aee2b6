"""Synthetic studies of write-back error on the GPU ("Low-Bit Recurrent
States in Hybrid Language Models", Correlated rounding errors; Approximate
erasure rate).  The trajectories come from the library's kernels through
the C ABI; the statistics are FP64 reductions in torch.

    python -m bit_recurrent_state_b200.simulate [--tokens T] [--out file.json]

Study A, correlated rounding errors: a layer of KDA heads (decay rates log-
uniform in [s_min, 1], rank-one delta-rule writes) runs T tokens from a
zero state twice on the same inputs, with FP32 storage (reference) and with
variable-width storage at one width b for every row (write-back every
token, nearest rounding).  The write-back error of token t is e_t = Q(y_t) -
y_t, y_t the FP32 state the quantized run holds before writing back (its
stored state of t - 1, dequantized, advanced one token by the FP32 decode
kernel).  Reported: the lag-one autocorrelation of e_t per element (centred
on the element's mean), averaged per row and binned by the row's decay
rate; the measured readout error, mean over tokens of ||o_q - o_ref||^2, over
the prediction of independent write-back noise of variance Delta^2 / 12 per
element propagated by F_t = (I - beta_t k_t k_t^T) D_t.

Study B, approximate against exact erasure rates: the exact rate of row i is
the diagonal of the observability Gramian, sum over lags of ||F_(t+l) ...
F_(t+1) e_i||^2 averaged over start tokens; the approximate one is
Gamma_hat = 1 / (C expm1(2 (s + r))), r = E[beta (2 - beta) k_i^2] / 2.
Both are allocated by the library's allocator at one layer budget, and the
approximate allocation's distortion sum Gamma_i 4^(-b_i), under the exact
rates, is reported relative to the exact allocation's, for fresh keys every
token and for one persistent key.
"""
from __future__ import annotations

import argparse
import json

import numpy as np
import torch

from . import brs, synth
from .state import LayerState


def _dev_inputs(inp: dict, device) -> dict:
    out = {}
    for k, v in inp.items():
        a = np.ascontiguousarray(v)
        if a.dtype == np.uint16:
            a = a.view(np.int16)
        out[k] = torch.from_numpy(a).to(device)
    return out


def _bf16_to_f64(t: torch.Tensor) -> torch.Tensor:
    """bfloat16 bit patterns (int16 tensor) -> float64."""
    return (t.to(torch.int32) << 16).view(torch.float32).to(torch.float64)


def _head_vectors(x: dict, w) -> tuple:
    """k [B][H][d], beta [B][H], a [B][H][d] in FP64 for one token."""
    B, H, Hk, d = w.B, w.H, w.hk, w.d
    kh = torch.arange(H, device=x["k"].device) * Hk // H
    k = _bf16_to_f64(x["k"])[:, kh]                            # [B][H][d]
    beta = x["beta"].to(torch.float64)
    a = x["decay"].to(torch.float64)
    if a.dim() == 2:
        a = a[..., None].expand(B, H, d)
    return k, beta, a


def _transition(k, beta, a) -> torch.Tensor:
    """F = (I - beta k k^T) diag(a), batched over heads: [..][d][d]."""
    d = k.shape[-1]
    eye = torch.eye(d, dtype=torch.float64, device=k.device)
    return (eye - beta[..., None, None] * k[..., :, None] * k[..., None, :]) * a[..., None, :]


def _row_steps(packed: torch.Tensor, w, bits: int) -> torch.Tensor:
    """FP16 step of every row of a uniform-width variable-width state (the
    step section follows the payload, on a 256-byte boundary)."""
    rows = w.H * w.d
    P = w.d // 8 * bits * rows
    off = (P * w.B + 255) // 256 * 256
    return packed[off: off + rows * w.B * 2].view(torch.float16).to(torch.float64).view(w.B, w.H, w.d)


def rounding_study(w, T: int, bits: int, burn_in: int = 0, device="cuda") -> dict:
    """Study A for workload w (B, H, H_k, d = 128, decays, keys, seed) at
    width `bits`.  Returns numpy arrays: corr [B][H][d], s [B][H][d],
    readout [B][H], model [B][H]."""
    dev = torch.device(device)
    Lq = brs.layout_of(w, storage=brs.STORE_VARBIT, hadamard=0, avg_bits=float(bits), b_min=bits,
                       b_max=bits, budget_scope=1, persistence=0)
    Lf = brs.layout_of(w, storage=brs.STORE_FP32, hadamard=0)
    wb = brs.WriteBack(brs.ROUND_NEAREST, 0, 1)
    stq, stf, sty = LayerState(Lq, device=dev), LayerState(Lf, device=dev), LayerState(Lf, device=dev)
    for st in (stq, stf, sty):
        st.zero()
    spare = torch.empty_like(stq.packed)
    B, H, d = w.B, w.H, w.d
    o_ref = torch.zeros((B, H, d), device=dev)
    o_y = torch.zeros_like(o_ref)
    o_q = torch.zeros_like(o_ref)
    shape = (B, H, d, d)
    f64 = dict(dtype=torch.float64, device=dev)
    s1, s2, cr = torch.zeros(shape, **f64), torch.zeros(shape, **f64), torch.zeros(shape, **f64)
    first, prev = torch.zeros(shape, **f64), torch.zeros(shape, **f64)
    P = torch.zeros((B, H, d, d), **f64)
    err = torch.zeros((B, H), **f64)
    model = torch.zeros((B, H), **f64)
    yv = sty.packed.view(torch.float32)
    for t in range(T):
        x = _dev_inputs(synth.token_inputs(w, t), dev)
        args = (x["q"], x["k"], x["v"], x["beta"], x["decay"])
        stf.step(wb, t, *args, o_ref)
        yv.copy_(stq.unpack().reshape(-1))
        sty.step(wb, t, *args, o_y)
        y = yv.view(shape).to(torch.float64)
        spare = stq.step(wb, t, *args, o_q, packed_out=spare)
        e = stq.unpack().to(torch.float64) - y
        if not torch.equal(o_q, o_y):
            raise RuntimeError("the quantized step's readout differs from the FP32 step from the same state")
        err += ((o_q.to(torch.float64) - o_ref.to(torch.float64)) ** 2).sum(-1)
        # independent-noise model: readout through F_t, then this token's noise
        k, beta, a = _head_vectors(x, w)
        F = _transition(k, beta, a)
        q = _bf16_to_f64(x["q"])[:, torch.arange(H, device=dev) * w.hk // H]
        G = F @ P @ F.transpose(-1, -2)
        model += d * torch.einsum("bhi,bhij,bhj->bh", q, G, q)
        P = G + torch.diag_embed(_row_steps(stq.packed, w, bits) ** 2 / 12.0)
        if t >= burn_in:
            s1 += e
            s2 += e * e
            if t == burn_in:
                first = e.clone()
            else:
                cr += prev * e
            prev = e
    n = T - burn_in
    m = s1 / n
    num = cr - m * (s1 - prev) - m * (s1 - first) + (n - 1) * m * m
    den = s2 - n * m * m
    corr = torch.where(den > 0, num / torch.where(den > 0, den, torch.ones_like(den)), torch.zeros_like(den))
    for st in (stq, stf, sty):
        if st.errors():
            raise RuntimeError("device flags raised during the study")
    a0 = _head_vectors(_dev_inputs(synth.token_inputs(w, 0), dev), w)[2]
    return dict(corr=corr.mean(-1).cpu().numpy(), s=(-torch.log(a0)).cpu().numpy(),
                readout=(err / T).cpu().numpy(), model=(model / T).cpu().numpy())


def gamma_hat(A: torch.Tensor, K: torch.Tensor, C: int = 1) -> torch.Tensor:
    """Approximate erasure rate 1 / (C expm1(2 (s + r))), s = -ln(A) / 2,
    r = K / 2, the argument floored at 1e-9."""
    arg = torch.clamp(2.0 * (-0.5 * torch.log(A) + 0.5 * K), min=1e-9)
    return 1.0 / (C * torch.expm1(arg))


def erasure_study(w, T: int, starts, lags: int, avg_bits: float, b_min: int, b_max: int,
                  device="cuda") -> dict:
    """Study B for sequence 0 of workload w: exact rates (Gramian diagonal)
    and approximate rates of every row of its H heads, the allocator's
    widths for each at one layer budget, and the distortion excess."""
    dev = torch.device(device)
    H, d = w.H, w.d
    toks = [_head_vectors(_dev_inputs(synth.token_inputs(w.with_(B=1), t), dev), w.with_(B=1))
            for t in range(T)]
    ks = torch.stack([t[0][0] for t in toks])                # [T][H][d]
    betas = torch.stack([t[1][0] for t in toks])             # [T][H]
    as_ = torch.stack([t[2][0] for t in toks])               # [T][H][d]
    gam = torch.zeros((H, d), dtype=torch.float64, device=dev)
    st = torch.as_tensor(list(starts), device=dev)
    M = torch.eye(d, dtype=torch.float64, device=dev).expand(len(starts), H, d, d).clone()
    for l in range(1, lags + 1):
        idx = st + l
        F = _transition(ks[idx], betas[idx], as_[idx])      # [S][H][d][d]
        M = F @ M
        gam += (M * M).sum(-2).sum(0)                        # squared column norms
    gam /= len(starts)
    A = (as_ ** 2).mean(0)
    K = ((betas * (2.0 - betas))[..., None] * ks * ks).mean(0)
    ghat = gamma_hat(A, K, 1)

    def alloc(c):
        bits = torch.zeros(c.numel(), dtype=torch.uint8, device=dev)
        brs.allocate_bits(c.reshape(-1).contiguous(), c.numel(), avg_bits, b_min, b_max, bits)
        return bits.to(torch.int64)

    be, ba = alloc(gam), alloc(ghat)
    g = gam.reshape(-1)
    de = (g * 4.0 ** (-be.to(torch.float64))).sum()
    da = (g * 4.0 ** (-ba.to(torch.float64))).sum()
    torch.cuda.synchronize(dev)
    return dict(gamma=gam.cpu().numpy(), gamma_hat=ghat.cpu().numpy(), bits_exact=be.cpu().numpy(),
                bits_approx=ba.cpu().numpy(), excess=float(da / de - 1.0))


def summary(tokens: int = 2048, device="cuda") -> dict:
    """Both studies at their reporting sizes: 4 sequences x 4 KDA heads of
    d = 128, s log-uniform in [1e-4, 1], widths 3..6 and 8 bits; the
    erasure study on 4 heads with lags up to 4096 tokens."""
    out = {"rounding": {}, "erasure": {}}
    w = synth.Workload("sim", B=4, H=4, d=128, T=tokens, s_min=1e-4, seed=11)
    for bits in (3, 4, 5, 6, 8):
        r = rounding_study(w, tokens, bits, burn_in=tokens // 8, device=device)
        s, c = r["s"].ravel(), r["corr"].ravel()
        bins = {}
        for lo, hi in ((1e-4, 1e-3), (1e-3, 1e-2), (1e-2, 1e-1), (1e-1, 1.0)):
            m = (s >= lo) & (s < hi)
            bins[f"s in [{lo:g}, {hi:g})"] = dict(rows=int(m.sum()), mean=float(c[m].mean()),
                                                  max=float(c[m].max()))
        ratio = (r["readout"] / r["model"]).ravel()
        out["rounding"][f"{bits} bits"] = dict(lag1=bins, readout_over_model=[float(ratio.min()),
                                                                             float(ratio.max())])
    for name, pk in (("fresh keys", 0), ("persistent key", 1)):
        we = synth.Workload("sim_erasure", B=1, H=4, d=128, T=8192, s_min=1e-3, persistent_keys=pk, seed=12)
        r = erasure_study(we, T=8192, starts=range(0, 2048, 512), lags=4096, avg_bits=4.0, b_min=1, b_max=8,
                          device=device)
        out["erasure"][name] = dict(excess=r["excess"])
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--tokens", type=int, default=2048)
    ap.add_argument("--out", default=None)
    args = ap.parse_args()
    res = summary(args.tokens)
    txt = json.dumps(res, indent=1)
    print(txt)
    if args.out:
        with open(args.out, "w") as f:
            f.write(txt + "\n")


if __name__ == "__main__":
    main()
