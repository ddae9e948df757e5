"""The benchmark's one-line JSON output: the fields and units a reader of the
line relies on, for the reference arm (CPU) and the product arm (GPU)."""
import json
import math
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(args, timeout):
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py")] + args, cwd=ROOT,
                         capture_output=True, text=True, timeout=timeout)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, out.stdout[-2000:]
    return json.loads(lines[0])


COMMON = ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
          "scaling", "vs_baseline", "dtype", "data", "config", "e2e", "cpu_baseline")


def test_reference_arm_line():
    d = _run(["--impl", "reference", "--workload", "n4096", "--steps", "1", "--warmup", "0"], 600)
    for k in COMMON:
        assert k in d, k
    assert d["impl"] == "reference" and d["dtype"] == "f64" and d["higher_is_better"] is True
    assert d["value"] > 0 and d["unit"] == "causal logits/s"
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"] and cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    assert d["config"]["workload"].startswith("qkv-self-relation") and d["config"]["n"] == 4096


@pytest.mark.gpu
@pytest.mark.parametrize("grads", [None, "partials", "dq"])
def test_product_arm_line(grads):
    """The default step (bf16 fused self-relation gradients) and the fp32 forms."""
    import torch
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    K = 4
    d = _run(["--workload", "n4096", "--steps", str(K), "--warmup", "3", "--cpu-seconds", "1"] +
             ([] if grads is None else ["--grads", grads]), 900)
    for k in COMMON + ("roofline", "clocks", "gpu_launches", "extra_hbm", "tflops", "kernel_ms"):
        assert k in d, k
    assert d["n_gpus"] == 1 and d["steps"] == K and d["warmup"] == 3 and d["scaling"] == "weak"
    assert d["dtype"] == "bf16" and d["vs_baseline"] is None and d["value"] > 0
    r = d["roofline"]
    for k in ("bound", "achieved", "peak", "unit", "frac", "traffic"):
        assert k in r, k
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    assert 0 < r["frac"] < 1.5 and math.isclose(r["frac"], r["achieved"] / r["peak"], rel_tol=1e-9)
    assert r["cycles_per_tile"] > r["tensor_cycles_per_tile"] > 0
    p1 = d["phase1_roofline"]
    assert p1["bound"] == "alu" and p1["measured_ex2_per_clk_per_sm"] > 0 and 0 < p1["frac"] < 1.5
    e = d["e2e"]
    grads_bytes = {None: 2, "dq": 4, "partials": 8}[grads] * 3 * 32 * 4096 * 128
    assert e["value"] > 0 and e["unit"] == d["unit"] and e["d2h_bytes_per_step"] == grads_bytes + 4
    assert e["h2d_bytes_per_step"] == 6 * 32 * 4096 * 128 * 2  # six bf16 input tensors per step
    assert d["gpu_launches"] == (5 if grads is None else 4) * K  # + the rounding pass of bf16 outputs
    x = d["extra_hbm"]
    assert x["state_bytes_expected"] == 12 * 3 * 32 * 4096 + 4 * 3 * 32
    # the allocator rounds each of the 4 state buffers of a relation up to its 512-byte granule
    assert x["state_bytes_expected"] <= x["state_bytes"] <= x["state_bytes_expected"] + 3 * 4 * 512
    assert x["allocated_per_step_bytes"] == 0 and x["torch_peak_above_buffers_bytes"] == 0
    assert set(d["clocks"]) >= {"sm_mhz", "sm_max_mhz", "reasons"}
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] > 0 and cb["unit"] == d["unit"]


@pytest.mark.gpu
def test_product_arm_job_split_one_rank():
    """--scaling strong on one GPU: the one rank's slice is the whole job."""
    import torch
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    d = _run(["--workload", "gqa-n8000", "--steps", "3", "--warmup", "3", "--no-cpu-baseline",
              "--scaling", "strong", "--no-probe"], 900)
    assert d["scaling"] == "strong" and d["n_gpus"] == 1 and d["value"] > 0
    assert d["config"]["parallelism"].startswith("units1")
    assert d["extra_hbm"]["rows"] == 2 * (32 + 8 + 8) * 8000


def test_reference_arm_other_ranks_exit_quietly():
    """Under torchrun only rank 0 runs the reference arm and prints its line."""
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--workload", "n4096", "--steps", "1", "--warmup", "0", "--gpus", "2"],
                         cwd=ROOT, env=env, capture_output=True, text=True, timeout=300)
    assert out.returncode == 0, out.stderr[-2000:]
    assert not [ln for ln in out.stdout.splitlines() if ln.startswith("{")]
