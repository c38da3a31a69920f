"""bench.py's roofline `traffic`: the DRAM bytes come from a committed ncu
summary only for the workload that summary covers, and only while the
kernel source digest it records matches the sources."""
import importlib.util
import os

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def recorded(path):
    vals = {}
    with open(path) as f:
        for line in f:
            line = line.strip().strip("`").strip("-").strip()
            if ":" in line:
                k, v = line.split(":", 1)
                vals[k.strip()] = v.strip()
    return vals


def test_every_summary_exists_and_records_a_digest_and_bytes(bench):
    for workload, path in bench.PROFILE_TRAFFIC.items():
        vals = recorded(path)
        assert len(vals.get("kernel_source_sha256", "")) == 16, workload
        assert float(vals["dram_bytes_per_launch_full_size"]) > 0, workload


def test_traffic_only_with_the_recorded_digest(bench):
    for workload, path in bench.PROFILE_TRAFFIC.items():
        vals = recorded(path)
        got = bench.profiled_traffic(vals["kernel_source_sha256"], workload)
        assert got == float(vals["dram_bytes_per_launch_full_size"])
        assert bench.profiled_traffic("0" * 16, workload) is None


def test_no_traffic_for_a_workload_without_a_summary(bench):
    digest = bench.kernel_source_digest()
    assert bench.profiled_traffic(digest, "shared_prefix_p16x8_pre1024_h32_d128_bs16_bf16") is None
    assert bench.profiled_traffic(digest, "no_such_workload") is None


def test_digests_cover_each_kernels_own_sources(bench):
    assert bench.kernel_source_digest("decode") != bench.kernel_source_digest("prefill")
    for names in bench.KERNEL_SOURCES.values():
        for n in names:
            assert os.path.exists(os.path.join(ROOT, "paged_kv_cache_337_b200", "csrc", n))
