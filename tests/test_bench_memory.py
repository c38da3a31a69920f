"""bench.py's `memory` record of the host pool (the pages' GPU memory
utilisation): blocks and slots in use, logical tokens, the empty slots of
each sequence's last block, and a contiguous reservation for comparison,
checked against a hand count on a small pool with a fork and a
copy-on-write append."""
import importlib.util
import os

import pytest

from paged_kv_cache_337_b200 import _abi

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_pool_memory_hand_count(bench):
    pool = _abi.BlockPool(64, 16)
    pool.add(0, 20)    # 2 blocks, 12 empty slots in the last
    pool.add(1, 33)    # 3 blocks, 15 empty
    pool.fork(1, 2)    # shares sequence 1's 3 blocks
    pool.append(2)     # 34 tokens: its shared partial block is copied, 14 empty
    m = bench.pool_memory(pool, [0, 1, 2], 16, 64, 100)
    assert m["blocks_in_use"] == 6 and m["blocks_free"] == 58
    assert m["slots_in_use"] == 96
    assert m["tokens"] == 20 + 33 + 34
    assert m["utilization"] == round(87 / 96, 4)
    assert m["empty_slots_per_sequence_max"] == 15
    assert m["empty_slots_per_sequence_mean"] == round((12 + 15 + 14) / 3, 2)
    assert m["contiguous_prealloc_slots"] == 300
    assert m["contiguous_prealloc_utilization"] == round(87 / 300, 4)


def test_pool_memory_sharing_passes_one(bench):
    """Eight samples sharing a 64-token prompt: 4 physical blocks hold 512
    logical tokens."""
    pool = _abi.BlockPool(16, 16)
    pool.add(0, 64)
    for c in range(1, 8):
        pool.fork(0, c)
    m = bench.pool_memory(pool, list(range(8)), 16, 16, 64)
    assert m["blocks_in_use"] == 4
    assert m["tokens"] == 512
    assert m["utilization"] == 8.0
    assert m["empty_slots_per_sequence_max"] == 0
