"""GPU parity at the measured sizes, over whole runs, through the C ABI.

Every configuration runs in the benchmark's launch configuration (the whole
batch on the GPU); the oracle follows a subset of the units (64 heads, or 8
sequences for variable-width storage, whose width budget spans a sequence)
for every step of the run, the subset rule that keeps the plain CPU oracle
within minutes:

  KDA decode   B=64 H=32, 16 FP16 + 112 INT8-Hadamard rows, block 128,
               all 1024 tokens, free-running;
  GDN decode   B=256, 16 key / 32 value heads, all rows INT8, all 512
               tokens, free-running, and the FP32-state run of the same
               inputs;
  var-width    B=128 H=32, 4.0-bit mean, widths 2..8, layer budget, all 1024
               tokens in each write-back mode (nearest, Philox stochastic,
               error feedback), teacher-forced per token (each token starts
               from the oracle's stored state, so a width flip at an FP64
               rounding point of the allocation cannot end the run);
  prefill      B=8 H=32 T=8192, write-back every 64 tokens, all 128 chunks in
               each write-back mode, teacher-forced per chunk; stored codes
               and residuals equal the oracle's write-back replayed on the
               GPU's own pre-write-back state.

Stored bytes (codes, FP16 rows, FP16 scale/zero, residuals, widths, steps,
offsets) must be identical; outputs within 2e-3 x RMS of the oracle's.

Inputs: the followed sequences draw fresh seeded inputs every token (a
workload of just those sequences, same seed and decay table); the other
sequences of the batch keep the benchmark workload's token-0 inputs, which
keeps the host-side input generation of a 1024-token run short."""
import numpy as np
import pytest

from bit_recurrent_state_b200 import synth
from parity import MODE, o_tolerance, oracle_cfg, random_perm, to_dev
from ref64 import varbit_row_codes

pytestmark = pytest.mark.gpu


class Inputs:
    """Full-batch token inputs whose followed sequences [b0, b1) are
    regenerated per token."""

    def __init__(self, w, b0, b1):
        self.w, self.b0, self.b1 = w, b0, b1
        self.sub = w.with_(B=b1 - b0)
        self.base = synth.token_inputs(w, 0)

    def token(self, t):
        sub = synth.token_inputs(self.sub, t)
        out = {}
        for k, v in self.base.items():
            a = v.copy()
            a[self.b0:self.b1] = sub[k]
            out[k] = a
        return out


def _decode_free_running(w, units, perm=None):
    import torch
    from bit_recurrent_state_b200 import brs
    from bit_recurrent_state_b200.state import LayerState
    from oracle import oracle as O

    cfg = oracle_cfg(w)
    L, wb = brs.layout_of(w), brs.writeback_of(w)
    st = LayerState(L, perm=perm)
    st.zero()
    packed_o, aux_o, stats_o = O.new_state(cfg)
    heads = w.B * w.H
    hb = packed_o.size // heads
    u0, u1 = units
    assert np.array_equal(st.packed.view(heads, hb)[u0:u1].cpu().numpy(), packed_o.reshape(heads, hb)[u0:u1])
    nel = aux_o.size // heads
    src = Inputs(w, u0 // w.H, (u1 - 1) // w.H + 1)
    o = torch.zeros((w.B, w.H, w.d), dtype=torch.float32, device="cuda")
    worst = 0.0
    for t in range(w.T):
        inp = src.token(t)
        dev = to_dev(inp)
        st.step(wb, t, dev["q"], dev["k"], dev["v"], dev["beta"], dev["decay"], o)
        oo, fl, _ = O.run_parallel(cfg, MODE[w.mode], w.seed, 1, t, {k: v[None] for k, v in inp.items()},
                                   packed_o, aux=aux_o, stats=stats_o, perm=perm, units=units)
        assert fl == 0
        og = o.view(heads, w.d)[u0:u1].cpu().numpy()
        oo_u = oo[0].reshape(heads, w.d)[u0:u1]
        err = float(np.max(np.abs(og - oo_u)))
        tol = o_tolerance(oo_u)
        assert err <= tol, (t, err, tol)
        worst = max(worst, err / max(tol, 1e-30))
        pg = st.packed.view(heads, hb)[u0:u1].cpu().numpy()
        ndiff = int(np.sum(pg != packed_o.reshape(heads, hb)[u0:u1]))
        assert ndiff == 0, f"token {t}: {ndiff} stored bytes differ"
        if w.mode == "errfeedback":
            ag = st.aux[: aux_o.nbytes].view(torch.int16).view(heads, nel)[u0:u1].cpu().numpy().view(np.uint16)
            np.testing.assert_array_equal(ag, aux_o.reshape(heads, nel)[u0:u1], err_msg=f"residuals, token {t}")
    assert st.errors() == 0
    return worst


def test_kda_decode_full_length():
    """All 1024 tokens of the KDA decode configuration; heads 1000..1063."""
    w = synth.WORKLOADS["kda_decode"]
    _decode_free_running(w, (1000, 1064), perm=random_perm(w, seed=5))


@pytest.mark.parametrize("mode", ["stochastic", "errfeedback"])
def test_kda_decode_full_size_other_modes(mode):
    """The KDA decode launch in the stochastic and error-feedback write-back
    modes, 128 tokens; heads 700..763."""
    w = synth.WORKLOADS["kda_decode"].with_(mode=mode, T=128)
    _decode_free_running(w, (700, 764), perm=random_perm(w, seed=6))


@pytest.mark.parametrize("name", ["gdn_decode", "gdn_decode_fp32"])
def test_gdn_decode_full_length(name):
    """All 512 tokens of the GDN decode configuration (INT8 state, and the
    FP32-state run of the same inputs); heads 4000..4063."""
    w = synth.WORKLOADS[name]
    _decode_free_running(w, (4000, 4064))


# ---- variable-width storage, teacher-forced per token --------------------

def _vb_ranges(w, b):
    """Byte ranges of sequence b in the stored state's sections (payload,
    FP16 steps, widths, offsets), as the header lays them out."""
    from ref64 import r256
    B, rows = w.B, w.H * w.d
    P = int(w.d // 8 * w.avg_bits * rows)
    off_scale = r256(P * B)
    off_width = off_scale + r256(rows * B * 2)
    off_offs = off_width + r256(rows * B)
    return [(b * P, (b + 1) * P), (off_scale + b * rows * 2, off_scale + (b + 1) * rows * 2),
            (off_width + b * rows, off_width + (b + 1) * rows),
            (off_offs + b * (rows + 1) * 4, off_offs + (b + 1) * (rows + 1) * 4)]


def _vb_seq(buf, w, b):
    """(payload, steps, widths, offsets) of sequence b from a stored state
    (numpy array, or a torch tensor copied range by range)."""
    parts = []
    for lo, hi in _vb_ranges(w, b):
        x = buf[lo:hi]
        parts.append(x.cpu().numpy() if hasattr(x, "cpu") else x)
    pay, sc, wd, of = parts
    return pay, sc.view(np.uint16), wd, of.view(np.uint32)


def _vb_put(st, w, packed_o, aux_o, stats_o, seqs):
    """Copy the oracle's stored state, residuals and statistics of the
    followed sequences into the GPU buffers."""
    import torch
    per_aux, per_st = aux_o.nbytes // w.B, stats_o.nbytes // w.B
    for b in seqs:
        for lo, hi in _vb_ranges(w, b):
            st.packed[lo:hi].copy_(torch.from_numpy(packed_o[lo:hi]))
        st.aux[b * per_aux:(b + 1) * per_aux].copy_(torch.from_numpy(aux_o.view(np.uint8)[b * per_aux:(b + 1) * per_aux]))
        st.stats[b * per_st:(b + 1) * per_st].copy_(
            torch.from_numpy(stats_o.view(np.uint8)[b * per_st:(b + 1) * per_st]))


def _vb_compare(w, pg, po, og, oo, seqs, tag):
    """Byte comparison of the followed sequences (pg: GPU state tensor, po:
    oracle state); a row whose width differs (an FP64 rounding point of the
    allocation) is counted, and the other rows of that sequence are compared
    code by code."""
    H, d = w.H, w.d
    flips = 0
    for b in seqs:
        payg, scg, wdg, ofg = _vb_seq(pg, w, b)
        payo, sco, wdo, ofo = _vb_seq(po, w, b)
        assert int(wdg.astype(int).sum()) == int(w.avg_bits * H * d)
        if np.array_equal(wdg, wdo):
            np.testing.assert_array_equal(ofg, ofo)
            np.testing.assert_array_equal(scg, sco, err_msg=f"{tag} steps b={b}")
            np.testing.assert_array_equal(payg, payo, err_msg=f"{tag} payload b={b}")
        else:
            for r in np.nonzero(wdg == wdo)[0]:
                assert scg[r] == sco[r], (tag, b, r)
                np.testing.assert_array_equal(varbit_row_codes(payg, int(ofg[r]), int(wdg[r]), d),
                                              varbit_row_codes(payo, int(ofo[r]), int(wdo[r]), d))
            flips += int(np.sum(wdg != wdo))
        og_b, oo_b = og[b], oo[b]
        assert np.max(np.abs(og_b - oo_b)) <= o_tolerance(oo_b), (tag, b)
    return flips


def test_varbit_decode_full_length_all_modes():
    """The variable-width configuration in its three write-back modes over
    all 1024 tokens, 8 followed sequences per mode (the modes' oracle runs
    share the host's cores)."""
    import os
    import torch
    from concurrent.futures import ThreadPoolExecutor
    from bit_recurrent_state_b200 import brs
    from bit_recurrent_state_b200.state import LayerState
    from oracle import oracle as O

    base = synth.WORKLOADS["varbit_decode"]
    seqs = tuple(range(3, 11))
    modes = ["nearest", "stochastic", "errfeedback"]
    runs = []
    for m in modes:
        w = base.with_(mode=m)
        cfg = oracle_cfg(w)
        st = LayerState(brs.layout_of(w))
        st.zero()
        packed_o, aux_o, stats_o = O.new_state(cfg)
        runs.append(dict(w=w, cfg=cfg, st=st, other=torch.zeros_like(st.packed), po=packed_o, ao=aux_o,
                         so=stats_o, wb=brs.writeback_of(w), flips=0))
    src = Inputs(base, seqs[0], seqs[-1] + 1)
    o = torch.zeros((base.B, base.H, base.d), dtype=torch.float32, device="cuda")
    threads = max(1, (os.cpu_count() or 3) // len(modes))
    B = base.B
    sl = slice(seqs[0], seqs[-1] + 1)

    def oracle_step(r, t, inp):
        out, fl, _ = O.run_parallel(r["cfg"], MODE[r["w"].mode], r["w"].seed, 1, t,
                                    {k: v[None] for k, v in inp.items()}, r["po"], aux=r["ao"], stats=r["so"],
                                    units=(seqs[0], seqs[-1] + 1), threads=threads)
        assert fl == 0
        return out[0]

    with ThreadPoolExecutor(len(modes)) as ex:
        for t in range(base.T):
            inp = src.token(t)
            dev = to_dev(inp)
            gpu = []
            for r in runs:
                st = r["st"]
                _vb_put(st, r["w"], r["po"], r["ao"], r["so"], seqs)
                brs.decode_step(brs.layout_of(r["w"]), r["wb"], t, st.packed, r["other"], st.aux, st.stats,
                                st.workspace, None, dev["q"], dev["k"], dev["v"], dev["beta"], dev["decay"], o)
                per_aux, per_st = r["ao"].nbytes // B, r["so"].nbytes // B
                gpu.append((o.cpu().numpy(),
                            st.stats[seqs[0] * per_st:(seqs[-1] + 1) * per_st].cpu().numpy(),
                            st.aux[seqs[0] * per_aux:(seqs[-1] + 1) * per_aux].cpu().numpy()))
            outs = list(ex.map(lambda r: oracle_step(r, t, inp), runs))
            for r, (og, sg, ag), oo in zip(runs, gpu, outs):
                r["flips"] += _vb_compare(r["w"], r["other"], r["po"], og, oo, seqs, f"{r['w'].mode} t={t}")
                np.testing.assert_array_equal(sg.view(np.float64), r["so"].reshape(B, -1)[sl].reshape(-1))
                if r["w"].mode == "errfeedback" and r["flips"] == 0:
                    np.testing.assert_array_equal(ag.view(np.uint16), r["ao"].reshape(B, -1)[sl].reshape(-1))
    for r in runs:
        assert r["st"].errors() == 0
        # widths on an FP64 rounding point of the allocation: rare
        assert r["flips"] <= 8, (r["w"].mode, r["flips"])


# ---- chunked prefill, teacher-forced per chunk ----------------------------

@pytest.mark.parametrize("mode", ["nearest", "stochastic", "errfeedback"])
def test_prefill_full_length(mode):
    """The prefill configuration over all 128 chunks of 64 tokens; heads
    96..159 (sequences 3 and 4).  Every chunk starts from the oracle's stored
    state and residuals; the GPU's outputs and pre-write-back state are within
    2e-3 x RMS of the oracle's token-by-token run, and its stored codes and
    residuals equal the oracle's write-back of the GPU's own state."""
    import torch
    from bit_recurrent_state_b200 import brs
    from bit_recurrent_state_b200.state import LayerState
    from oracle import oracle as O

    w = synth.WORKLOADS["kda_prefill"].with_(mode=mode)
    perm = random_perm(w, seed=11)
    cfg = O.Config(B=w.B, H=w.H, Hk=w.hk, d=w.d, storage=O.STORE_DAMP, k_hi=w.k_hi, block=w.block,
                   hadamard=w.hadamard, decay_per_key=w.decay_per_key, domain=O.DOMAIN_CANONICAL)
    L, wb = brs.layout_of(w), brs.writeback_of(w)
    st = LayerState(L, perm=perm)
    st.zero()
    packed_o, aux_o, _ = O.new_state(cfg)
    heads = w.B * w.H
    hb = packed_o.size // heads
    nel = aux_o.size // heads
    u0, u1 = 96, 160
    b0, b1 = u0 // w.H, u1 // w.H
    sub = w.with_(B=b1 - b0)
    o = torch.zeros((w.B, 64, w.H, w.d), device="cuda")
    dump = torch.zeros((w.B, w.H, w.d, w.d), device="cuda")
    base = {k: np.ascontiguousarray(np.swapaxes(v, 0, 1)) for k, v in synth.run_inputs(w, 0, 64).items()}
    for c in range(w.T // 64):
        t0 = 64 * c
        fresh = synth.run_inputs(sub, t0, 64)                      # token-major, followed sequences
        inp = {}
        for k, v in base.items():
            a = v.copy()
            a[b0:b1] = np.swapaxes(fresh[k], 0, 1)
            inp[k] = a
        st.packed.copy_(torch.from_numpy(packed_o))
        st.aux[: aux_o.nbytes].copy_(torch.from_numpy(aux_o.view(np.uint8)))
        before_p, before_a = packed_o.copy(), aux_o.copy()
        d = {k: torch.from_numpy(np.ascontiguousarray(v).view(np.int16) if v.dtype == np.uint16 else v).cuda()
             for k, v in inp.items()}
        st.prefill(wb, t0, 64, d["q"], d["k"], d["v"], d["beta"], d["decay"], o, state_dump=dump)
        tok = {k: np.ascontiguousarray(np.swapaxes(v, 0, 1)) for k, v in inp.items()}
        oo, fl, _, so = O.run_parallel(cfg, MODE[mode], w.seed, 64, t0, tok, packed_o, aux=aux_o, perm=perm,
                                       units=(u0, u1), dump_s=True)
        assert fl == 0
        og = np.swapaxes(o.cpu().numpy(), 1, 2).reshape(heads, 64, w.d)[u0:u1]
        oo_u = np.swapaxes(oo, 0, 1).swapaxes(1, 2).reshape(heads, 64, w.d)[u0:u1]
        rms_o = np.sqrt(np.mean(oo_u.astype(np.float64) ** 2))
        assert np.max(np.abs(og - oo_u)) <= 2e-3 * rms_o, (c, np.max(np.abs(og - oo_u)) / rms_o)
        sg = dump.cpu().numpy()
        sg_u = sg.reshape(heads, w.d, w.d)[u0:u1]
        so_u = so.reshape(heads, w.d, w.d)[u0:u1]
        rms_s = np.sqrt(np.mean(so_u.astype(np.float64) ** 2))
        assert np.max(np.abs(sg_u - so_u)) <= 2e-3 * rms_s, (c, np.max(np.abs(sg_u - so_u)) / rms_s)
        # replay: the oracle's write-back of the GPU's own state gives its stored bytes
        fl = O.damp_writeback(cfg, MODE[mode], w.seed, t0 + 63, sg, before_p, before_a, units=(u0, u1))
        assert fl == 0
        pg = st.packed.view(heads, hb)[u0:u1].cpu().numpy()
        np.testing.assert_array_equal(pg, before_p.reshape(heads, hb)[u0:u1], err_msg=f"codes, chunk {c}")
        if mode == "errfeedback":
            ag = st.aux[: aux_o.nbytes].view(torch.int16).view(heads, nel)[u0:u1].cpu().numpy().view(np.uint16)
            np.testing.assert_array_equal(ag, before_a.reshape(heads, nel)[u0:u1], err_msg=f"residuals, chunk {c}")
    assert st.errors() == 0
