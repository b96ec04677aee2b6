"""Benchmark of the decode step (state-update tokens*heads/s and state HBM
GB/s against the measured B200 copy bandwidth).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload kda_decode|gdn_decode|gdn_decode_fp32|varbit_decode|
                                gdn_varbit_decode|kda_decode_c8|kda_prefill|kda_tiny]

A step is one decode token for every (sequence, head) of the workload: one
launch of the fused decode kernel (dequantize, decay, delta-rule write, read
o, requantize, write back).  Consecutive steps rotate over 8 independent
layer states (each with its own seeded inputs), so a step never finds its
state in L2 (8 x 38.7 MB > 126 MB).  With N GPUs (torchrun) every rank runs
its own batch of the same size (weak scaling, no collective on the data
path); the time is the maximum over ranks.

With `--workload kda_prefill` a step is instead one chunked-prefill launch
over the whole batch (B x T tokens x H heads, write-back every 64 tokens).
`--workload kda_decode_c8` decodes with write-back every 8 tokens (the FP32
state carried in HBM between write-backs; state bytes averaged over the
interval).

`--workload gdn_varbit_decode` runs GDN heads with one width per head (steps
per block of 32 key channels), three launches per step as for varbit_decode.

`--impl reference` times the plain CPU oracle on this host's cores on the
same workload and metric (bounded samples), which is the only other place
the oracle runs besides the cpu_baseline leg.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "state-update tokens·heads/s and state HBM GB/s (% of B200 peak), decode"
UNIT = "tokens·heads/s"
FALLBACK_HBM_GBS = 6650.0
NLAYERS = 8
# the sources of each decode kernel (a DRAM record stays valid while they hash the same)
KERNEL_SOURCES = {
    "cta": ["bit_recurrent_state_b200/csrc/decode_cta.cu", "bit_recurrent_state_b200/csrc/brs_device.cuh"],
    "warp": ["bit_recurrent_state_b200/csrc/decode.cu", "bit_recurrent_state_b200/csrc/brs_device.cuh"],
    "varbit": ["bit_recurrent_state_b200/csrc/varbit.cu", "bit_recurrent_state_b200/csrc/allocate.cu",
               "bit_recurrent_state_b200/csrc/brs_device.cuh"],
    "varbit_head": ["bit_recurrent_state_b200/csrc/varbit_head.cu", "bit_recurrent_state_b200/csrc/allocate.cu",
                    "bit_recurrent_state_b200/csrc/brs_device.cuh"],
}

VARBIT_STORES = ("varbit", "varbit_head")


def kernel_family(w) -> str:
    if w.storage in VARBIT_STORES:
        return w.storage
    cta = (w.storage == "damp" and w.d == 128 and w.k_hi % 16 == 0 and
           (w.C == 1 or w.mode in ("nearest", "stochastic", "errfeedback")))
    return "cta" if cta else "warp"


def kernel_hash(family: str = "cta") -> str:
    h = hashlib.sha256()
    for p in KERNEL_SOURCES[family]:
        with open(os.path.join(ROOT, p), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def algorithmic_bytes(w) -> dict:
    """Bytes one decode launch must move: the stored state read and written
    once, the token's inputs read, o written."""
    from bit_recurrent_state_b200 import brs
    n, aux, stats, _ = brs.state_bytes(brs.layout_of(w))
    heads = w.B * w.H
    inputs = (2 * w.B * w.hk * w.d * 2 + heads * w.d * 2 + heads * 4 +
              (heads * w.d * 4 if w.decay_per_key else heads * 4) +
              (w.H * w.d * 2 if w.storage not in VARBIT_STORES else 0))
    out = heads * w.d * 4
    ef = 2 * aux if w.mode == "errfeedback" else 0
    if w.mode == "direction":
        # 2-bit counters of the INT8 rows, read and written
        ef = 2 * (heads * (w.d - w.k_hi) * w.d // 4)
    if w.mode.startswith("residual"):
        # k-bit residual integers of the INT8 rows (kept in 4 bits), read and written
        ef = 2 * (heads * (w.d - w.k_hi) * w.d // 2)
    st = 2 * stats
    state = 2 * n
    if w.C > 1 and w.storage == "damp":
        # deferred write-back, averaged over an interval of C tokens: the
        # stored state is read at its first token and written at its last,
        # the FP32 interval state written at the other C - 1 and read at the
        # other C - 1 (residuals touched at the write-back only)
        f32 = heads * w.d * w.d * 4
        state = (2 * n + 2 * (w.C - 1) * f32) / w.C
        ef = ef / w.C
    return dict(state=state, inputs=inputs, output=out, aux=ef, stats=st,
                total=state + inputs + out + ef + st)


def rank_workload(w, rank: int):
    """A rank's own batch: the same shape, its own sequences (seed offset by
    rank).  Units are independent, so ranks exchange nothing on the data path."""
    return w.with_(seed=w.seed + 1000 * rank)


def max_over_ranks(x: float, world: int, device) -> float:
    """The job's time for a per-rank time: its maximum over the ranks."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def kernel_name(w) -> str:
    """The kernel a decode step of workload w launches (the dominant one)."""
    if w.storage == "varbit":
        return "brs::varbit_kernel (update pass + fit pass) and brs::allocate_kernel"
    if w.storage == "varbit_head":
        return "brs::varbit_head_kernel (update pass + fit pass) and brs::allocate_kernel"
    if kernel_family(w) == "cta":
        return "brs::decode_cta_kernel"
    return "brs::decode_warp_kernel"


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


# FP32 lanes per SM (4 sub-partitions x 32) and the B200's maximum SM clock
FP32_LANES_PER_SM, SM_COUNT, SM_MAX_MHZ = 128, 148, 1965.0


def fp32_issue_peak():
    """Peak FP32 lane operations per second (one operation per lane per
    cycle; a paired f32x2 instruction counts as two): 148 SMs x 128 lanes x
    the maximum SM clock, in Gop/s."""
    return SM_COUNT * FP32_LANES_PER_SM * SM_MAX_MHZ * 1e6 / 1e9


def fit_ops(w) -> float:
    """Algorithmic FP32 operations of one variable-width write-back's step
    fit: every stored value is scored against 16 clip-factor candidates,
    7 operations each (scale, round = add + subtract of the magic constant,
    clip, step times level, residual, square-accumulate)."""
    return float(w.B * w.H * w.d * w.d) * 16 * 7


def tf32_peak():
    """Dense TF32 tensor peak: the measured bf16 GEMM rate times the nominal
    TF32/BF16 ratio (1.1 / 2.25 PFLOP/s)."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["bf16_tflops"]) * 1.1 / 2.25, "measured bf16 burst x nominal TF32/BF16 (1.1/2.25)"
    return 1590.0 * 1.1 / 2.25, "fallback bf16 1.59 PFLOP/s x nominal TF32/BF16 (1.1/2.25)"


def prefill_traffic():
    """DRAM bytes per prefill launch from the committed ncu record, while the
    kernel source still hashes to the profiled version."""
    p = os.path.join(ROOT, "profiles", "prefill_kda_prefill_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        rec = json.load(f)
    h = hashlib.sha256()
    with open(os.path.join(ROOT, "bit_recurrent_state_b200/csrc/prefill_tc.cu"), "rb") as f:
        h.update(f.read())
    if rec.get("kernel_hash") != h.hexdigest()[:16]:
        return None
    return rec.get("dram_bytes_per_launch")


def traffic_record(w):
    """DRAM bytes per launch from a committed ncu summary, only while the
    sources of the workload's kernel still hash to the profiled version."""
    p = os.path.join(ROOT, "profiles", f"decode_{w.name}_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        rec = json.load(f)
    if rec.get("kernel_hash") != kernel_hash(kernel_family(w)):
        return None
    if w.mode != rec.get("mode", "nearest"):           # the records are captured in nearest mode
        return None
    return rec.get("dram_bytes_per_launch")


class ClockSampler:
    def __init__(self, index: int):
        self.index = index
        self.proc = None
        fd, self.path = tempfile.mkstemp(prefix="brs_clocks_", suffix=".csv")
        os.close(fd)

    def __enter__(self):
        os.makedirs(os.path.dirname(self.path), exist_ok=True)
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index),
                 "--query-gpu=index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
                 "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                 "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap",
                 "--format=csv,noheader,nounits", "-lms", "100"], stdout=self.f,
                stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
            return self
        # nvidia-smi takes a moment to start: the timed region begins once
        # the first sample is written (at most 10 s)
        t0 = time.time()
        while time.time() - t0 < 10.0 and self.proc.poll() is None:
            self.f.flush()
            if os.path.getsize(self.path) > 0:
                break
            time.sleep(0.05)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            self.proc.wait()
            self.f.close()

    def summary(self):
        if self.proc is None or not os.path.exists(self.path):
            return None
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    mx = float(parts[2])
                except ValueError:
                    continue
                for n, v in zip(names, parts[5:9]):
                    if v.lower() == "active":
                        reasons.add(n)
        try:
            os.remove(self.path)
        except OSError:
            pass
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def _oracle_cfg(w):
    from oracle import oracle as O
    st = {"fp32": O.STORE_FP32, "damp": O.STORE_DAMP, "varbit": O.STORE_VARBIT,
          "varbit_head": O.STORE_VARBIT_HEAD}[w.storage]
    return O.Config(B=w.B, H=w.H, Hk=w.hk, d=w.d, storage=st, k_hi=w.k_hi, block=w.block,
                    hadamard=w.hadamard, decay_per_key=w.decay_per_key, avg_bits=w.avg_bits,
                    b_min=w.b_min, b_max=w.b_max, low_bits=w.low_bits,
                    domain=O.DOMAIN_MIXED if w.storage == "damp" else O.DOMAIN_CANONICAL)


def is_prefill(w) -> bool:
    """Workloads whose step is one chunked-prefill launch (decode workloads
    may still write back every C > 1 tokens)."""
    return w.name == "kda_prefill" or w.name.startswith("kda_prefill_")


def workload_config(w, world: int) -> dict:
    """The `config` object of both arms: the workload by name and sizes."""
    cfg = {"workload": w.name if w.mode == "nearest" else f"{w.name}_{w.mode}",
           "B": w.B, "H": w.H, "H_k": w.hk, "d": w.d, "storage": w.storage, "k_hi": w.k_hi,
           "block": w.block, "mode": w.mode, "per_rank_batch": w.B, "parallelism": f"dp{world}"}
    if w.C > 1:
        cfg.update(T=w.T, C=w.C)
    if w.storage in VARBIT_STORES:
        cfg.update(avg_bits=w.avg_bits, b_min=w.b_min, b_max=w.b_max)
    if w.storage == "damp" and w.low_bits != 8:
        cfg.update(low_bits=w.low_bits)
    cfg["l2"] = l2_policy(w)
    return cfg


def l2_policy(w) -> str:
    """How the GPU arm keeps a timed step out of L2 (part of the workload's
    definition, so both arms name it the same way)."""
    from bit_recurrent_state_b200 import brs
    if is_prefill(w):
        inputs = w.B * w.T * (2 * w.hk * w.d * 2 + w.H * w.d * 2 + w.H * 4 +
                              (w.H * w.d * 4 if w.decay_per_key else w.H * 4))
        return f"inputs {inputs / 1e9:.1f} GB per step (> 126 MB L2)"
    n = brs.state_bytes(brs.layout_of(w))[0]
    return f"{NLAYERS} rotating layer states of {n / 1e6:.1f} MB (> 126 MB L2)"


class OracleRunner:
    """The oracle, as it stands, over a bounded sample of the workload: the
    first `units` units (heads, or whole sequences for variable-width
    storage, whose width budget spans a sequence) for `ntok` consecutive
    tokens per call, split over the host's cores (units are independent)."""

    def __init__(self, w):
        from bit_recurrent_state_b200 import synth
        from oracle import oracle as O
        self.O, self.synth, self.w = O, synth, w
        self.cfg = _oracle_cfg(w)
        self.packed, self.aux, self.stats = O.new_state(self.cfg)
        self.cores = os.cpu_count() or 1
        self.t = 0
        self.cache = {}
        self.varbit = w.storage in VARBIT_STORES
        self.units_total = w.B if self.varbit else w.B * w.H
        self.heads_per_unit = w.H if self.varbit else 1
        self.mode = {"nearest": O.ROUND_NEAREST, "stochastic": O.ROUND_STOCHASTIC,
                     "errfeedback": O.ROUND_ERRFEEDBACK, "direction": O.ROUND_DIRECTION,
                     "residual2": O.ROUND_RESIDUAL2, "residual3": O.ROUND_RESIDUAL3,
                     "residual4": O.ROUND_RESIDUAL4}[w.mode]

    def inputs(self, ntok):
        key = (self.t, ntok)
        if key not in self.cache:
            self.cache = {key: self.synth.run_inputs(self.w, self.t, ntok)}
        return self.cache[key]

    def run(self, units, ntok):
        """Returns (seconds, threads used, token*heads processed)."""
        inp = self.inputs(ntok)
        t0 = time.perf_counter()
        _, fl, used = self.O.run_parallel(self.cfg, self.mode, self.w.seed, self.w.C, self.t, inp,
                                          self.packed, aux=self.aux, stats=self.stats,
                                          units=(0, units), threads=self.cores)
        dt = time.perf_counter() - t0
        if fl & self.O.EINVAL:
            raise RuntimeError("oracle run rejected its arguments")
        self.t += ntok
        return dt, used, units * self.heads_per_unit * ntok

    def rate(self):
        """token*heads per second, from a short calibration run (one
        write-back interval, so later runs start on an interval boundary)."""
        units = max(1, min(self.units_total, 4 * self.cores // self.heads_per_unit))
        dt, _, th = self.run(units, self.w.C)
        return th / max(dt, 1e-6)


def cpu_oracle_sample(w, target_s: float = 12.0):
    """cpu_baseline: the oracle on host cores, about target_s seconds of work
    on the workload's units (all of them when that fits, else a prefix)."""
    R = OracleRunner(w)
    r = R.rate()
    want = r * target_s / R.heads_per_unit            # unit-tokens in the budget
    if w.C > 1:                      # whole write-back chunks, up to the sequence length
        ntok = w.C * int(max(1, min(w.T // w.C, want // (R.units_total * w.C))))
    else:
        ntok = int(max(1, min(64, want // R.units_total)))
    units = int(max(1, min(R.units_total, want // ntok)))
    dt, used, th = R.run(units, ntok)
    what = "sequences" if R.varbit else "heads"
    return {"value": th / dt, "unit": UNIT, "cores": used, "kind": "oracle",
            "sample": f"{units} of {R.units_total} {what} x {ntok} tokens of {w.name} "
                      f"({dt:.1f} s wall on {used} threads)"}


def time_steps(args, step, first: int, stream, barrier):
    """Device time of args.steps consecutive steps (first, first+1, ...),
    bracketed by a barrier and a synchronize on both sides, CUDA events on
    the launching stream.  The steps are captured once into a CUDA graph and
    replayed (no host launch overhead between the timed kernels) unless
    --eager is given."""
    import torch
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if args.eager:
        barrier()
        ev0.record(stream)
        for i in range(args.steps):
            step(first + i)
        ev1.record(stream)
        barrier()
        return ev0.elapsed_time(ev1)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):              # captured on torch's side stream (the library launches on
        for i in range(args.steps):        # the current stream, which is the capture stream here)
            step(first + i)
    barrier()
    ev0.record(stream)
    with torch.cuda.stream(stream):
        g.replay()
    ev1.record(stream)
    barrier()
    t = ev0.elapsed_time(ev1)
    del g
    return t


def run_reference(args, w):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    R = OracleRunner(w)
    prefill = is_prefill(w)
    total = w.B * w.H * (w.T if prefill else 1)      # token*heads of one step of our arm
    per_step_s = max(0.005, min(4.0, args.ref_budget / (args.warmup + args.steps)))
    units = int(max(1, min(R.units_total, R.rate() * per_step_s / (R.heads_per_unit * w.C))))
    vals, used = [], 1
    for i in range(args.warmup + args.steps):
        dt, used, th = R.run(units, w.C)
        if i >= args.warmup:
            vals.append(th / dt)
    value = statistics.median(vals)
    what = "sequences" if R.varbit else "heads"
    metric = METRIC.replace("decode", "chunked prefill") if prefill else METRIC
    line = {"impl": "reference", "metric": metric, "value": value, "unit": UNIT,
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * total / value, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": workload_config(w, args.gpus),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": used, "kind": "oracle",
                             "sample": f"each step: {units} of {R.units_total} {what} x {w.C} "
                                       f"token(s) of {w.name} on {used} threads"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_prefill(args, w):
    """A step = the chunked prefill of the whole batch (B sequences x T
    tokens x H heads, write-back every 64 tokens); value = tokens*heads/s."""
    import torch
    import torch.distributed as dist

    from bit_recurrent_state_b200 import brs, synth
    from bit_recurrent_state_b200.state import LayerState

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream()
    wr = rank_workload(w, rank)
    L, wb = brs.layout_of(wr), brs.writeback_of(wr)
    rng = np.random.default_rng(wr.seed)
    perm = np.stack([rng.permutation(w.d) for _ in range(w.H)]).astype(np.int16)
    st = LayerState(L, device=dev, perm=perm)
    st.zero()
    inp = synth.run_inputs(wr, 0, w.T)
    host = {k: torch.from_numpy(np.ascontiguousarray(np.swapaxes(v, 0, 1)).view(np.int16)
                                if v.dtype == np.uint16 else np.ascontiguousarray(np.swapaxes(v, 0, 1)))
            for k, v in inp.items()}
    x = {k: v.to(dev) for k, v in host.items()}
    o = torch.empty((w.B, w.T, w.H, w.d), dtype=torch.float32, device=dev)

    def step(i, xs=None, out=None):
        xs = x if xs is None else xs
        out = o if out is None else out
        st.prefill(wb, i * w.T, w.T, xs["q"], xs["k"], xs["v"], xs["beta"], xs["decay"], out)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        ms_run = time_steps(args, step, 0, stream, barrier)
    ms_step = max_over_ranks(ms_run, world, dev) / args.steps
    flags = st.errors()
    # end to end: every step's inputs copied from pinned host memory and its o
    # read back inside the timed region, on copy streams that overlap the
    # neighbouring steps' kernels (two device input sets and two o buffers,
    # reuse ordered by events)
    pinned = {k: v.pin_memory() for k, v in host.items()}
    xs2 = [x, {k: torch.empty_like(v) for k, v in x.items()}]
    outs = [o, torch.empty_like(o)]
    outs_h = [torch.empty_like(o, device="cpu").pin_memory() for _ in range(2)]
    h2d_s, d2h_s = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    in_ready = [torch.cuda.Event() for _ in range(2)]
    k_done = [torch.cuda.Event() for _ in range(2)]
    out_done = [torch.cuda.Event() for _ in range(2)]

    def issue_h2d(i):
        if i >= 2:
            h2d_s.wait_event(k_done[i % 2])          # the kernel of step i-2 read this set
        with torch.cuda.stream(h2d_s):
            for k, v in pinned.items():
                xs2[i % 2][k].copy_(v, non_blocking=True)
        in_ready[i % 2].record(h2d_s)

    barrier()
    ev0.record(stream)
    h2d_s.wait_event(ev0)
    d2h_s.wait_event(ev0)
    issue_h2d(0)
    for i in range(args.steps):
        if i + 1 < args.steps:
            issue_h2d(i + 1)
        stream.wait_event(in_ready[i % 2])
        if i >= 2:
            stream.wait_event(out_done[i % 2])       # o buffer read back
        step(args.warmup + i, xs2[i % 2], outs[i % 2])
        k_done[i % 2].record(stream)
        d2h_s.wait_event(k_done[i % 2])
        with torch.cuda.stream(d2h_s):
            outs_h[i % 2].copy_(outs[i % 2], non_blocking=True)
        out_done[i % 2].record(d2h_s)
    stream.wait_event(out_done[(args.steps - 1) % 2])
    ev1.record(stream)
    barrier()
    ms_e2e = max_over_ranks(ev0.elapsed_time(ev1), world, dev) / args.steps
    units = w.B * w.H * w.T * world
    n, aux, _, _ = brs.state_bytes(L)
    chunks = w.T // 64
    inputs_b = sum(v.numel() * v.element_size() for v in host.values())
    out_b = o.numel() * o.element_size()
    total = 2 * n * chunks + inputs_b + out_b
    peak, src = peaks()
    achieved = total / (ms_step * 1e-3) / 1e9
    # the chunk contractions: [K~;Q~] K^T (128x64x128), S_0^T [K~;Q~]^T (128x128x128),
    # lower(Q~ K^T) W (64x128x64), K^T W (128x128x64), forward substitution 64*63/2*128
    flops_chunk = 2 * (128 * 64 * 128 + 128 * 128 * 128 + 64 * 128 * 64 + 128 * 128 * 64) + 64 * 63 * 128
    flops = flops_chunk * w.B * w.H * (w.T // 64)                 # one launch on this GPU
    tflops = flops / (ms_step * 1e-3) / 1e12
    tpeak, tsrc = tf32_peak()
    line = {
        "metric": METRIC.replace("decode", "chunked prefill"), "value": units / (ms_step * 1e-3),
        "unit": UNIT, "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f32", "data": "synthetic",
        "config": workload_config(w, world),
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "peak_source": src, "algorithmic_bytes_per_launch": total,
                     "traffic": prefill_traffic(), "kernel": "brs::prefill_tc_kernel",
                     "tensor": {"achieved": tflops, "peak": tpeak, "unit": "TFLOP/s", "frac": tflops / tpeak,
                                "peak_source": tsrc, "flops_per_launch": flops}},
        "e2e": {"value": units / (ms_e2e * 1e-3), "unit": UNIT, "h2d_bytes_per_step": inputs_b,
                "d2h_bytes_per_step": out_b},
        "gpu_launches": args.steps, "device_flags": flags,
        "launch": "eager" if args.eager else "cuda_graph (the timed steps captured once, replayed)",
    }
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_oracle_sample(w)
    if rank == 0:
        line["clocks"] = clk.summary()
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def staged_inputs(inp: dict, dev):
    """One token's inputs in one pinned host buffer and one device buffer
    (each tensor a view at a 256-byte aligned offset), so that a token's
    host-to-device transfer is a single copy.  Returns (host buffer, device
    buffer, device views by name)."""
    import torch
    offs, total = {}, 0
    for k, v in inp.items():
        offs[k] = total
        total += (v.nbytes + 255) // 256 * 256
    host = torch.empty(total, dtype=torch.uint8).pin_memory()
    hv = host.numpy()
    for k, v in inp.items():
        a = np.ascontiguousarray(v)
        hv[offs[k]: offs[k] + a.nbytes] = a.view(np.uint8).ravel()
    devbuf = host.to(dev)
    views = {}
    for k, v in inp.items():
        dt = torch.int16 if v.dtype == np.uint16 else torch.float32
        n = int(np.prod(v.shape))
        views[k] = devbuf[offs[k]: offs[k] + n * (2 if dt == torch.int16 else 4)].view(dt).view(v.shape)
    return host, devbuf, views


def run_ours(args, w):
    import torch
    import torch.distributed as dist

    from bit_recurrent_state_b200 import brs, synth
    from bit_recurrent_state_b200.state import LayerState

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream()

    # per-rank workload: same shape, own sequences (seed offset by rank)
    wr = rank_workload(w, rank)
    L = brs.layout_of(wr)
    wb = brs.writeback_of(wr)
    rng = np.random.default_rng(wr.seed)
    perm = np.stack([rng.permutation(w.d) for _ in range(w.H)]).astype(np.int16)
    varbit = w.storage in VARBIT_STORES
    if varbit:
        perm = None                    # variable-width rows stay in key-channel order
    layers, spares, inputs, host_inputs = [], [], [], []
    for l in range(NLAYERS):
        st = LayerState(L, device=dev, perm=perm)
        st.zero()
        layers.append(st)
        spares.append(torch.empty_like(st.packed) if varbit else None)
        inp = synth.token_inputs(wr.with_(seed=wr.seed + 17 * l), 0)
        host, devbuf, views = staged_inputs(inp, dev)
        host_inputs.append((host, devbuf))
        inputs.append(views)
    o = torch.zeros((w.B, w.H, w.d), dtype=torch.float32, device=dev)
    o_host = torch.zeros_like(o, device="cpu").pin_memory()

    def step(i, out=None):
        l = i % NLAYERS
        st = layers[l]
        x = inputs[l]
        out = o if out is None else out
        if varbit:
            # variable-width states change their row offsets: write to the other buffer
            spares[l] = st.step(wb, i, x["q"], x["k"], x["v"], x["beta"], x["decay"], out,
                                packed_out=spares[l])
        else:
            # with deferred write-back a layer's calls must cover consecutive
            # steps: its own token counter
            st.step(wb, i // NLAYERS if w.C > 1 else i, x["q"], x["k"], x["v"], x["beta"], x["decay"], out)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    flags = layers[0].errors()

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    # ---- device-resident throughput (kernel per step)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        ms_run = time_steps(args, step, args.warmup, stream, barrier)
    ms_max = max_over_ranks(ms_run, world, dev)
    ms_step = ms_max / args.steps

    # ---- end to end through the public API with host buffers: every token's
    # inputs are copied from pinned host memory and its o read back inside the
    # timed region.  Copies run on their own streams (host to device on two,
    # alternating by token, so that two transfers overlap their fixed costs;
    # device to host on a third) so that the next tokens' inputs and token
    # i-1's output move while token i's kernel runs; events order each
    # buffer's reuse (an input set is rewritten only after the kernel that read
    # it, an o buffer only after its read-back).
    h2d = host_inputs[0][0].numel()                  # the one buffer copied per token
    d2h = o.numel() * o.element_size()
    h2d_ss = [torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)]
    d2h_s = torch.cuda.Stream(device=dev)
    outs = [o, torch.zeros_like(o)]
    outs_h = [o_host, torch.zeros_like(o_host).pin_memory()]
    R = 2 * NLAYERS                                  # event ring (slots reused after R tokens)
    in_ready = [torch.cuda.Event() for _ in range(R)]
    k_done = [torch.cuda.Event() for _ in range(R)]
    out_done = [torch.cuda.Event() for _ in range(R)]
    n = args.steps
    base = args.warmup + args.steps

    def issue_h2d(i):
        l = (base + i) % NLAYERS                     # the input set token base + i reads
        h2d_s = h2d_ss[i % 2]
        if i >= NLAYERS:
            h2d_s.wait_event(k_done[(i - NLAYERS) % R])
        with torch.cuda.stream(h2d_s):
            host, devbuf = host_inputs[l]
            devbuf.copy_(host, non_blocking=True)          # the token's inputs, one copy
        in_ready[i % R].record(h2d_s)

    barrier()
    ev0.record(stream)
    for hs in h2d_ss:
        hs.wait_event(ev0)
    d2h_s.wait_event(ev0)
    issue_h2d(0)
    for i in range(n):
        if i + 1 < n:
            issue_h2d(i + 1)
        stream.wait_event(in_ready[i % R])
        if i >= 2:
            stream.wait_event(out_done[(i - 2) % R])
        step(base + i, outs[i % 2])
        k_done[i % R].record(stream)
        d2h_s.wait_event(k_done[i % R])
        with torch.cuda.stream(d2h_s):
            outs_h[i % 2].copy_(outs[i % 2], non_blocking=True)
        out_done[i % R].record(d2h_s)
    stream.wait_event(out_done[(n - 1) % R])
    ev1.record(stream)
    barrier()
    ms_e2e = max_over_ranks(ev0.elapsed_time(ev1), world, dev)
    flags |= layers[0].errors()

    units = w.B * w.H * world
    value = units * args.steps / (ms_max * 1e-3)
    e2e_value = units * args.steps / (ms_e2e * 1e-3)
    ab = algorithmic_bytes(w)
    peak, src = peaks()
    achieved = ab["total"] / (ms_step * 1e-3) / 1e9
    traffic = traffic_record(w)
    roof = {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
            "frac": achieved / peak, "peak_source": src + " (MEASURED_PEAKS.json hbm_gbs)"
            if src == "measured" else "fallback 6.65 TB/s",
            "algorithmic_bytes_per_launch": ab["total"],
            "traffic": traffic,
            "kernel": kernel_name(w), "state_gbs": ab["state"] / (ms_step * 1e-3) / 1e9}
    if varbit:
        # the step is bound by the FP32 issue of the step fit, not by HBM: its
        # algorithmic operations over the whole step's time (the update pass
        # and the allocator included), the HBM figures beside it
        fa = fit_ops(w) / (ms_step * 1e-3) / 1e9
        fp = fp32_issue_peak()
        roof = {"bound": "alu", "achieved": fa, "peak": fp, "unit": "Gop/s", "frac": fa / fp,
                "peak_source": "derived: 148 SMs x 128 FP32 lanes x 1965 MHz (one op per lane per cycle)",
                "algorithmic_ops_per_step": fit_ops(w), "traffic": traffic, "kernel": kernel_name(w),
                "hbm": {"achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                        "algorithmic_bytes_per_launch": ab["total"]}}
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": workload_config(w, world),
        "roofline": roof,
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": args.steps * (3 if varbit else 1),
        "device_flags": flags,
        "launch": "eager" if args.eager else "cuda_graph (the timed steps captured once, replayed)",
    }
    if rank == 0:
        line["clocks"] = clk.summary()
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_oracle_sample(w)
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None,
                    help="timed steps (default: 20000 decode steps, 5 prefill steps)")
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="kda_decode")
    ap.add_argument("--mode", default=None,
                    help="write-back rounding: nearest | stochastic | errfeedback | direction")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--eager", action="store_true",
                    help="launch the timed steps one by one instead of replaying them as a CUDA graph")
    ap.add_argument("--batch", type=int, default=None, help="override the workload's batch (small profiling cases)")
    ap.add_argument("--low-bits", type=int, default=None, choices=[4, 8],
                    help="DAMP low-tier width (4: the INT4 tier; the workload is then named *_int4)")
    ap.add_argument("--tokens", type=int, default=None, help="override the prefill length (small profiling cases)")
    ap.add_argument("--ref-budget", type=float, default=120.0,
                    help="seconds of oracle work for the whole --impl reference run")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    from bit_recurrent_state_b200 import synth
    w = synth.WORKLOADS[args.workload]
    if args.mode:
        w = w.with_(mode=args.mode)
    if args.batch:
        # another batch is another workload (no committed DRAM record applies)
        w = w.with_(B=args.batch, name=f"{w.name}_b{args.batch}")
    if args.low_bits == 4:
        w = w.with_(low_bits=4, name=w.name + "_int4")
    if args.tokens:
        w = w.with_(T=args.tokens)
    if args.steps is None:
        # long enough a timed region for the clock sampler (>= ~0.5 s on
        # the GPU); the oracle arm times a few bounded samples
        args.steps = 10 if args.impl == "reference" else (40 if is_prefill(w) else 20000)
    if args.impl == "reference":
        run_reference(args, w)
    else:
        from bit_recurrent_state_b200 import brs
        brs.lib()          # the in-tree CUDA library; fails loudly when it is missing
        if is_prefill(w):
            run_prefill(args, w)
        else:
            run_ours(args, w)


if __name__ == "__main__":
    main()
