"""Host-side pieces of the benchmark that need no GPU: which kernel a
workload's decode step runs (and so which DRAM record may describe it), the
algorithmic bytes per launch, and the reference arm (the oracle) under a
non-default write-back mode."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def test_kernel_family_and_bytes():
    import bench
    from bit_recurrent_state_b200 import synth
    w = synth.WORKLOADS["kda_decode"]
    assert bench.kernel_family(w) == "cta"
    assert bench.kernel_family(w.with_(mode="direction")) == "cta"       # every write-back mode at C = 1
    assert bench.kernel_family(w.with_(mode="residual3", low_bits=4)) == "cta"
    assert bench.kernel_family(w.with_(d=64, k_hi=8, block=64)) == "warp"
    assert bench.kernel_family(synth.WORKLOADS["kda_decode_c8"]) == "cta"    # deferred instantiations
    assert bench.kernel_family(synth.WORKLOADS["kda_decode_c8"].with_(d=64, k_hi=8, block=64)) == "warp"
    assert bench.kernel_family(synth.WORKLOADS["varbit_decode"]) == "varbit"
    base = bench.algorithmic_bytes(w)
    assert base["state"] == 2 * 64 * 32 * 18880                           # stored state read + written
    dm = bench.algorithmic_bytes(w.with_(mode="direction"))
    assert dm["aux"] == 2 * 64 * 32 * (112 * 128 // 4)                    # 2-bit counters read + written
    assert dm["total"] - base["total"] == dm["aux"]
    # a DRAM record keyed to the CTA kernel does not describe the general kernel
    assert bench.traffic_record(w.with_(mode="direction")) is None


def test_reference_arm_direction_mode():
    p = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload",
                        "kda_tiny", "--mode", "direction", "--steps", "3", "--warmup", "3", "--ref-budget", "2"],
                       env=dict(os.environ, CUDA_VISIBLE_DEVICES=""), capture_output=True, text=True, timeout=300)
    assert p.returncode == 0, p.stderr
    line = json.loads(p.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["value"] > 0
    # both arms print the same config object (the GPU arm prints workload_config too)
    import bench
    from bit_recurrent_state_b200 import synth
    w = synth.WORKLOADS["kda_tiny"].with_(mode="direction")
    assert line["config"] == bench.workload_config(w, 1)
    assert "l2" in line["config"]


def test_fit_roofline_arithmetic():
    """The variable-width decodes report the step fit against the FP32 issue
    peak: 16 candidates x 7 operations per stored value, 148 x 128 lanes at
    1965 MHz."""
    import bench
    from bit_recurrent_state_b200 import synth
    w = synth.WORKLOADS["varbit_decode"]
    assert bench.fit_ops(w) == 128 * 32 * 128 * 128 * 112
    assert bench.fp32_issue_peak() == 148 * 128 * 1965e6 / 1e9
    assert bench.kernel_family(synth.WORKLOADS["gdn_varbit_decode"]) == "varbit_head"


def test_staged_inputs_layout(monkeypatch):
    """A token's inputs staged in one buffer for a single host-to-device
    copy: each tensor a view at a 256-byte aligned offset holding exactly the
    input's values (checked on the host with a CPU 'device')."""
    import numpy as np
    import torch
    import bench
    from bit_recurrent_state_b200 import synth
    monkeypatch.setattr(torch.Tensor, "pin_memory", lambda self: self)     # no CUDA here
    for name in ("kda_decode", "gdn_decode"):
        inp = synth.token_inputs(synth.WORKLOADS[name], 3)
        host, dev, views = bench.staged_inputs(inp, "cpu")
        assert host.numel() == dev.numel() >= sum(v.nbytes for v in inp.values())
        for k, v in inp.items():
            a = views[k].numpy()
            assert a.shape == v.shape
            assert (views[k].data_ptr() - dev.data_ptr()) % 256 == 0
            np.testing.assert_array_equal(a.view(np.uint16) if v.dtype == np.uint16 else a, v)
