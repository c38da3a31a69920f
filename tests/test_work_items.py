"""The decode work list (pkv_decode_work_items), host side.

The planner must list exactly the (sequence, KV head, partition) triples of
pkv_decode_attention's grid that hold tokens — partition p of sequence s
exists for p < max(1, ceil(L_s / P)), so an empty context keeps one item,
whose CTA writes its zeros — as flat grid indices, ordered by the number of
16-token tiles they hold, largest first, grid order among equals.  The
expected list here is built by enumerating every grid slot and sorting with
Python's sort, independently of the planner's counting sort.
"""
import numpy as np
import pytest
import torch

from paged_kv_cache_337_b200 import _abi, build


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    _abi.lib()


def grid(max_len, P):
    """Partition length and count of pkv_decode_attention's grid: one pass
    (the longest context rounded up to a tile) when P is 0 or covers it."""
    if P <= 0 or P >= max_len:
        return -(-max(max_len, 1) // 16) * 16, 1
    return P, -(-max_len // P)


def expected(lens, hkv, max_len, P, grid_order=False):
    Pe, NP = grid(max_len, P)
    slots = []
    for s in range(len(lens)):
        for h in range(hkv):
            for p in range(NP):
                L = int(lens[s])
                tokens = min(Pe, L - p * Pe)
                if p == 0 or tokens > 0:  # partition 0 always, later ones if they hold tokens
                    slots.append(((s * hkv + h) * NP + p, tokens))

    def tiles(tokens):
        return -(-tokens // 16)

    if not grid_order:
        slots.sort(key=lambda it: (-tiles(it[1]), it[0]))
    return [f for f, _ in slots]


@pytest.mark.parametrize("P", [0, 16, 64, 512, 1024, 4096])
@pytest.mark.parametrize("hkv", [1, 3, 8])
def test_items_are_the_grid_slots_holding_tokens_longest_first(P, hkv):
    g = np.random.default_rng(P * 31 + hkv)
    for trial in range(6):
        S = int(g.integers(1, 40))
        lens = g.integers(0, 3000, S).astype(np.int32)
        lens[g.integers(0, S)] = 0
        max_len = int(lens.max()) + int(g.integers(0, 50))
        got = _abi.pkv_decode_work_items(lens, hkv, max_len, P).tolist()
        assert got == expected(lens, hkv, max_len, P)
        got = _abi.pkv_decode_work_items(lens, hkv, max_len, P, order=_abi.PKV_ITEMS_GRID)
        assert got.tolist() == expected(lens, hkv, max_len, P, grid_order=True)


def test_order_and_counts_of_a_hand_worked_batch():
    # lengths 5, 40, 17, 0, 1024, 1025, 3000 over 2 KV heads, P = 1024:
    # the grid has 3 partitions per (sequence, KV head)
    lens = [5, 40, 17, 0, 1024, 1025, 3000]
    got = _abi.pkv_decode_work_items(lens, 2, 3000, 1024).tolist()
    assert got == [24, 27, 30, 33, 36, 37, 39, 40,  # 64 tiles: full partitions
                   38, 41,                          # 60 tiles: 3000 - 2048 = 952 tokens
                   6, 9,                            # 40 tokens
                   12, 15,                          # 17 tokens
                   0, 3, 31, 34,                    # 5 tokens; 1025's second partition
                   18, 21]                          # the empty context


def test_grid_order_keeps_the_grid_and_drops_empty_slots():
    lens = [5, 40, 17, 0, 1024, 1025, 3000]
    got = _abi.pkv_decode_work_items(lens, 2, 3000, 1024, order=_abi.PKV_ITEMS_GRID).tolist()
    assert got == [0, 3, 6, 9, 12, 15, 18, 21, 24, 27, 30, 31, 33, 34, 36, 37, 38, 39, 40, 41]


def test_unknown_order_is_refused():
    with pytest.raises(_abi.PkvError):
        _abi.pkv_decode_work_items([3, 4], 1, 4, 0, order=2)


def test_single_pass_orders_sequences_by_length():
    lens = [100, 2048, 7, 900]
    got = _abi.pkv_decode_work_items(lens, 1, 2048, 0).tolist()
    assert got == [1, 3, 0, 2]


def test_item_count_and_capacity():
    lens = [33, 0, 500]
    n = 4 * (1 + 1 + 4)  # P = 128: 1, 1 and 4 partitions, 4 KV heads
    assert _abi.pkv_decode_work_items(lens, 4, 500, 128).numel() == n
    out = torch.full((n,), -7, dtype=torch.int32)
    got = _abi.pkv_decode_work_items(lens, 4, 500, 128, out=out)
    assert got.data_ptr() == out.data_ptr() and (out >= 0).all()
    small = torch.full((n - 1,), -7, dtype=torch.int32)
    with pytest.raises(_abi.PkvError):
        _abi.pkv_decode_work_items(lens, 4, 500, 128, out=small)
    assert (small == -7).all()  # nothing written


@pytest.mark.parametrize("lens,max_len,P", [([5, -1], 10, 0), ([5, 11], 10, 0),
                                             ([5, 6], 10, 24 + 1)])
def test_bad_lengths_or_partition_size_are_refused(lens, max_len, P):
    with pytest.raises(_abi.PkvError):
        _abi.pkv_decode_work_items(lens, 2, max_len, P)


def test_empty_batch_has_no_items():
    assert _abi.pkv_decode_work_items([], 4, 0, 0).numel() == 0
