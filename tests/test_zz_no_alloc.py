"""pkv_decode_attention_noalloc: decode attention for callers that cannot
allocate device memory (a host framework that owns the whole device and
forbids plug-ins from calling cudaMalloc, or a loop that must not pay for an
allocation).  Its split-K scratch is a device array built into the library.

Checked through the C ABI against the fp64 oracle and against
pkv_decode_attention given a workspace allocated by the caller, on two calls
in a row with different inputs (the second call reuses the array the first
one left behind), and for the property the entry point exists for: a call
leaves the device's free memory unchanged.  This file is collected last on
purpose.
"""
import numpy as np
import pytest
import torch

from oracle import reference as ref
from paged_kv_cache_337_b200 import _abi, build
from tests.helpers import paged_problem, tolerance_violation

pytestmark = pytest.mark.gpu

ATOL, RTOL = 2e-3, 1e-2


def _device_args(p, dev):
    return (p["q"].to(dev), p["kc"].to(dev), p["vc"].to(dev),
            torch.as_tensor(p["tables"]).to(dev), torch.as_tensor(p["lens"]).to(dev))


def _with_workspace(p, dev, scale, P):
    q, kc, vc, tables, lens = _device_args(p, dev)
    max_len = int(max(p["lens"]))
    n = _abi.pkv_decode_workspace_bytes(q.shape[0], q.shape[1], max_len, P, q.shape[2])
    ws = torch.empty(n, dtype=torch.uint8, device=dev) if n else None
    out = torch.empty_like(q)
    _abi.pkv_decode_attention(out, q, kc, vc, tables, lens, max_len, scale, P, ws)
    torch.cuda.synchronize()
    return out.cpu()


def _without_allocation(p, dev, scale, P):
    q, kc, vc, tables, lens = _device_args(p, dev)
    out = torch.full_like(q, float("nan"))
    err = torch.zeros(2, dtype=torch.int32, device=dev)
    _abi.pkv_decode_attention_noalloc(out, q, kc, vc, tables, lens, int(max(p["lens"])), scale,
                                      P, dev_error=err)
    torch.cuda.synchronize()
    assert err.tolist() == [0, 0]
    return out.cpu()


def test_noalloc_matches_the_oracle_and_the_workspace_entry_point_on_two_calls(cuda_device):
    build.build()
    _abi.lib()
    scale = 1.0 / np.sqrt(128)
    # two different problems, both split into partitions (scratch in use)
    first = paged_problem(31, 32, 8, 128, 32, [3000, 1, 511, 512, 513, 2048, 77], "bf16")
    second = paged_problem(32, 64, 8, 128, 16, [700, 4096, 33, 1500], "bf16")
    for p, P, bs in ((first, 128, 32), (second, 256, 16)):
        need = _abi.pkv_decode_workspace_bytes(len(p["lens"]), p["q"].shape[1],
                                               int(max(p["lens"])), P, 128)
        assert 0 < need <= _abi.PKV_NOALLOC_WORKSPACE_BYTES
        want = _with_workspace(p, cuda_device, scale, P)
        got = _without_allocation(p, cuda_device, scale, P)
        oracle = ref.decode_attention(p["q"], p["kc"], p["vc"], p["tables"], p["lens"], scale,
                                      "bf16", 8, bs)
        assert torch.isfinite(got).all()
        assert tolerance_violation(got, oracle, ATOL, RTOL) <= 0
        assert tolerance_violation(got, want.double().numpy(), ATOL, RTOL) <= 0


def test_noalloc_call_leaves_free_device_memory_unchanged(cuda_device):
    """After a first call (which loads the kernel and finds the array), a
    split-K call takes no device memory: the driver's free-memory count is
    the same before and after it.  Tensors from torch's caching allocator
    are made before the count is read."""
    build.build()
    _abi.lib()
    p = paged_problem(34, 16, 4, 128, 16, [900, 64, 2000], "bf16")
    q, kc, vc, tables, lens = _device_args(p, cuda_device)
    out = torch.empty_like(q)
    err = torch.zeros(2, dtype=torch.int32, device=cuda_device)
    for _ in range(2):
        _abi.pkv_decode_attention_noalloc(out, q, kc, vc, tables, lens, 2000, 0.1, 128,
                                          dev_error=err)
        torch.cuda.synchronize()
    free_before = torch.cuda.mem_get_info(cuda_device)[0]
    _abi.pkv_decode_attention_noalloc(out, q, kc, vc, tables, lens, 2000, 0.1, 128,
                                      dev_error=err)
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info(cuda_device)[0] == free_before
    assert err.tolist() == [0, 0]
    oracle = ref.decode_attention(p["q"], p["kc"], p["vc"], p["tables"], p["lens"], 0.1, "bf16",
                                  4, 16)
    assert tolerance_violation(out.cpu(), oracle, ATOL, RTOL) <= 0


def test_noalloc_rejects_sizes_beyond_its_scratch(cuda_device):
    build.build()
    p = paged_problem(33, 8, 8, 128, 16, [40], "bf16")
    q, kc, vc, tables, lens = _device_args(p, cuda_device)
    # 1024 sequences x 64 heads x 2048 partitions of 16 tokens: far above 64 MiB
    big_s = 1024
    need = _abi.pkv_decode_workspace_bytes(big_s, 64, 32768, 16, 128)
    assert need > _abi.PKV_NOALLOC_WORKSPACE_BYTES
    lib = _abi.lib()
    st = lib.pkv_decode_attention_noalloc(
        q.data_ptr(), q.data_ptr(), kc.data_ptr(), vc.data_ptr(), tables.data_ptr(), 2048,
        lens.data_ptr(), big_s, 32768, 64, 8, 128, p["NB"], 16, 16 * 8 * 128, 0.1, 16,
        _abi.PKV_BF16, None, None)
    assert st == _abi.PKV_ERR_WORKSPACE
    assert b"built into the library" in lib.pkv_last_error()
