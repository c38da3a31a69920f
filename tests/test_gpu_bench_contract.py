"""bench.py on the GPU prints one JSON line carrying the whole contract:
the metric and workload, the kernel's roofline (with the DRAM traffic of the
committed ncu summary, or null), the end-to-end figure through the public
API with the bytes it moved, the clocks seen and the launches counted."""
import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def run_bench(*args):
    proc = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], cwd=ROOT,
                          capture_output=True, text=True, timeout=900)
    assert proc.returncode == 0, proc.stderr[-2000:]
    lines = [l for l in proc.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    return json.loads(lines[0])


def test_default_decode_line(cuda_device):
    d = run_bench("--steps", "8", "--warmup", "3", "--no-cpu-baseline")
    assert d["metric"].startswith("paged decode attention effective KV GB/s")
    assert d["unit"] == "GB/s" and d["higher_is_better"] is True and d["scaling"] == "weak"
    assert d["n_gpus"] == 1 and d["steps"] == 8 and d["warmup"] == 3
    assert d["value"] > 0 and d["ms_per_step"] > 0 and d["dtype"] == "bf16"
    assert d["config"]["workload"] == "7b_s256_h32_d128_bs16_bf16"
    r = d["roofline"]
    assert r["bound"] == "hbm" and r["unit"] == "GB/s" and r["peak"] > 0
    assert abs(r["frac"] - r["achieved"] / r["peak"]) < 1e-3
    assert r["traffic"] is None or r["traffic"] > 0
    e = d["e2e"]
    assert e["value"] > 0 and e["unit"] == "GB/s"
    assert e["h2d_bytes_per_step"] > 0 and e["d2h_bytes_per_step"] > 0
    assert d["gpu_launches"] >= 2 * d["steps"]  # slot write + attention per step
    m = d["memory"]  # the host pool's KV memory after the steps
    assert 0 < m["blocks_in_use"] <= d["config"]["pool_blocks"]
    assert m["slots_in_use"] == 16 * m["blocks_in_use"]
    assert 0.9 < m["utilization"] <= 1.0  # no sharing: at most 15 empty slots a sequence
    assert m["empty_slots_per_sequence_max"] <= 15
    assert m["contiguous_prealloc_utilization"] < m["utilization"]
    c = d["clocks"]
    assert c is None or (c["sm_max_mhz"] > 0 and isinstance(c["reasons"], list))


def test_prefill_line(cuda_device):
    d = run_bench("--workload", "prefill_s8_l2048_hq32_hkv8_d128_bs16_bf16", "--steps", "4",
                  "--warmup", "3", "--no-cpu-baseline")
    assert d["unit"] == "TFLOP/s" and d["value"] > 0
    r = d["roofline"]
    assert r["bound"] == "tensor" and r["kernel"] == "paged_prefill_kernel"
    assert 0 < r["frac"] < 2
    assert d["gpu_launches"] == 2 * d["steps"]
