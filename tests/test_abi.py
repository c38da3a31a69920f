"""The C-ABI library loads and exports every entry point include/pkv.h
declares, with a binding of the same name; host-only entry points answer
without a GPU.  (No kernel is launched here.)"""
import os
import re

import pytest

from paged_kv_cache_337_b200 import _abi, build

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include")


def declared_functions():
    names = []
    for fn in sorted(os.listdir(HEADER)):
        if fn.endswith(".h"):
            text = open(os.path.join(HEADER, fn), encoding="utf-8").read()
            names += re.findall(r"^PKV_API\s+[\w\s\*]+?\b(pkv_\w+)\s*\(", text, re.M)
    return names


@pytest.fixture(scope="module")
def lib():
    build.build()
    return _abi.lib()


def test_header_declares_the_entry_points():
    names = declared_functions()
    for must in ("pkv_write_slots", "pkv_decode_attention", "pkv_copy_blocks",
                 "pkv_decode_workspace_bytes", "pkv_pool_create", "pkv_seq_append"):
        assert must in names
    assert len(names) == len(set(names))


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
        assert name in _abi.SIGNATURES, "binding lacks " + name


def test_host_only_calls(lib):
    assert _abi.pkv_block_bytes(16, 32, 128, 1, 2) == 262144
    assert lib.pkv_status_string(_abi.PKV_ERR_OOM) == b"block pool exhausted"
    assert lib.pkv_version() >= 100
    # no partitions -> no workspace
    assert _abi.pkv_decode_workspace_bytes(4, 8, 100, 0, 64) == 0
    assert _abi.pkv_decode_workspace_bytes(4, 8, 100, 128, 64) == 0
    # 8 seqs x 32 heads x 64 partitions: counters (room for 8 x 32), m and l
    # (each 256-byte aligned) + o
    n = 8 * 32 * 64
    assert _abi.pkv_decode_workspace_bytes(8, 32, 32768, 512, 128) == \
        1024 + 2 * n * 4 + n * 128 * 4


def test_argument_errors_are_reported_before_any_launch(lib):
    import ctypes as C

    st = lib.pkv_decode_attention(None, None, None, None, None, 0, None, 1, 0, 8, 8, 96, 1, 16,
                                  16 * 8 * 96, 1.0, 0, None, 0, 1, None, None)
    assert st == _abi.PKV_ERR_UNSUPPORTED  # head_dim 96 is not built
    assert b"head_dim" in lib.pkv_last_error()
    st = lib.pkv_decode_attention(None, None, None, None, None, 0, None, 1, 0, 8, 3, 128, 1,
                                  16, 16 * 3 * 128, 1.0, 0, None, 0, 1, None, None)
    assert st == _abi.PKV_ERR_INVALID  # 8 query heads over 3 KV heads
    st = lib.pkv_write_slots(None, None, None, None, None, 4, 8, 16, 2, 6, 16 * 12, 1, None, None)
    assert st == _abi.PKV_ERR_INVALID  # row of 12 elements is not a multiple of 8
    st = lib.pkv_copy_blocks(None, None, None, 0, 8, 16, 2, 64, 16 * 2 * 64, 1, None, None)
    assert st == _abi.PKV_OK  # nothing to copy
    st = lib.pkv_decode_attention(None, None, None, None, None, 4, None, 2, 16, 8, 8, 64, 4, 16,
                                  16 * 8 * 64, 1.0, 24, None, 0, 1, None, None)
    assert st == _abi.PKV_ERR_INVALID  # partition of 24 tokens is not a multiple of 16
    assert C.sizeof(C.c_void_p) == 8


def test_prefill_rejects_a_non_positive_scale_before_any_device_work():
    # the check precedes every pointer or device access, so it runs on CPU
    L = _abi.lib()
    st = L.pkv_prefill_attention(None, None, None, None, None, 1, None, None, 1, 1, 4, 4, 128,
                                 8, 16, 16 * 4 * 128, 0.0, _abi.PKV_BF16, None, None)
    assert st == _abi.PKV_ERR_INVALID
    assert b"scale" in L.pkv_last_error()


def test_ex2_selftest_checks_its_count_before_any_device_work(lib):
    # a count outside 0 .. 2^28 is refused, and a count of zero is a no-op,
    # both before any pointer or device access
    for n in (-1, (1 << 28) + 1):
        assert lib.pkv_selftest_ex2_poly(None, None, n, None) == _abi.PKV_ERR_INVALID
        assert b"pkv_selftest_ex2_poly" in lib.pkv_last_error()
    assert lib.pkv_selftest_ex2_poly(None, None, 0, None) == _abi.PKV_OK
