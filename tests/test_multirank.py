"""The N > 1 benchmark path on CPU: two gloo ranks (spawned processes,
rendezvous on 127.0.0.1).  Units are independent (sequence, head) pairs, so
the only cross-rank step is the timing reduction: every rank runs its own
batch of the same shape (weak scaling) and the job's time is the maximum
over ranks.  The oracle stands in for the GPU step so the test needs no GPU:
each rank's result must equal the single-process result for that rank's
inputs (nothing leaks between ranks), the reduction must return the maximum,
and only rank 0 of the reference arm prints."""
import json
import os
import socket
import subprocess
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

WORKER = r'''
import os, sys, json
sys.path.insert(0, os.environ["BRS_ROOT"])
sys.path.insert(0, os.path.join(os.environ["BRS_ROOT"], "tests"))
import datetime
import numpy as np
import torch
import torch.distributed as dist
import bench
from bit_recurrent_state_b200 import synth
from parity import MODE, oracle_cfg
from oracle import oracle as O

rank, world = int(os.environ["RANK"]), int(os.environ["WORLD_SIZE"])
dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
w = bench.rank_workload(synth.WORKLOADS["kda_tiny"], rank)
cfg = oracle_cfg(w)
packed, aux, stats = O.new_state(cfg)
inp = synth.run_inputs(w, 0, 4)
o, fl, _ = O.run(cfg, MODE[w.mode], w.seed, 1, 0, inp, packed, aux=aux, stats=stats)
t_rank = 1.5 + rank                       # a per-rank "time"
t_job = bench.max_over_ranks(t_rank, world, "cpu")
res = {"rank": rank, "seed": w.seed, "o_sum": float(np.sum(o.astype(np.float64))),
       "packed_crc": int(np.sum(packed.astype(np.uint64) * np.arange(packed.size, dtype=np.uint64) % 1000003)),
       "flags": int(fl), "t_job": t_job}
with open(os.path.join(os.environ["BRS_OUT"], f"rank{rank}.json"), "w") as f:
    json.dump(res, f)
dist.barrier()
dist.destroy_process_group()
'''


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _launch(tmp_path, world=2):
    script = tmp_path / "worker.py"
    script.write_text(WORKER)
    port = _free_port()
    procs = []
    for r in range(world):
        env = dict(os.environ, RANK=str(r), LOCAL_RANK=str(r), WORLD_SIZE=str(world), MASTER_ADDR="127.0.0.1",
                   MASTER_PORT=str(port), BRS_ROOT=ROOT, BRS_OUT=str(tmp_path), CUDA_VISIBLE_DEVICES="")
        procs.append(subprocess.Popen([sys.executable, str(script)], env=env, stdout=subprocess.PIPE,
                                      stderr=subprocess.STDOUT))
    outs = [p.communicate(timeout=240)[0].decode() for p in procs]
    for p, out in zip(procs, outs):
        assert p.returncode == 0, out
    return [json.loads((tmp_path / f"rank{r}.json").read_text()) for r in range(world)]


def test_two_gloo_ranks_independent_batches_and_max_time(tmp_path, orc):
    res = _launch(tmp_path)
    assert [r["rank"] for r in res] == [0, 1]
    assert res[0]["seed"] != res[1]["seed"]                 # each rank its own sequences
    assert res[0]["o_sum"] != res[1]["o_sum"]
    assert all(r["flags"] == 0 for r in res)
    assert all(r["t_job"] == 2.5 for r in res)               # max over ranks, on every rank
    # each rank's result equals a single-process run on that rank's inputs
    import bench
    from bit_recurrent_state_b200 import synth
    from parity import MODE, oracle_cfg
    for r in res:
        w = bench.rank_workload(synth.WORKLOADS["kda_tiny"], r["rank"])
        cfg = oracle_cfg(w)
        packed, aux, stats = orc.new_state(cfg)
        o, fl, _ = orc.run(cfg, MODE[w.mode], w.seed, 1, 0, synth.run_inputs(w, 0, 4), packed, aux=aux,
                           stats=stats)
        assert float(np.sum(o.astype(np.float64))) == r["o_sum"]
        crc = int(np.sum(packed.astype(np.uint64) * np.arange(packed.size, dtype=np.uint64) % 1000003))
        assert crc == r["packed_crc"]


def test_reference_arm_prints_on_rank0_only(tmp_path):
    base = [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload", "kda_tiny",
            "--steps", "3", "--warmup", "3", "--ref-budget", "2"]
    outs = {}
    for r in (0, 1):
        env = dict(os.environ, RANK=str(r), WORLD_SIZE="2", LOCAL_RANK=str(r), CUDA_VISIBLE_DEVICES="")
        p = subprocess.run(base, env=env, capture_output=True, text=True, timeout=300)
        assert p.returncode == 0, p.stderr
        outs[r] = p.stdout.strip()
    assert outs[1] == ""
    line = json.loads(outs[0].splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "tokens·heads/s" and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"
