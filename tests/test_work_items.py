"""The decode work list (pkv_decode_work_items), host side.

The planner must list exactly the (sequence, KV head, partition) triples of
pkv_decode_attention's grid that hold tokens — partition p of sequence s
exists for p < max(1, ceil(L_s / P)), so an empty context keeps one item,
whose CTA writes its zeros — as flat grid indices (s * Hkv + h) * NP + p.
Within a sequence the items go partition by partition with the KV heads
side by side; the orders then sort by the 16-token tiles an item holds
(longest first), by sequence length (sequences longest first) or not at all
(batch order).  The expected lists here are built by enumerating every grid
slot and sorting with Python's sort, independently of the planner's
counting sort.
"""
import numpy as np
import pytest
import torch

from paged_kv_cache_337_b200 import _abi, build

ORDERS = (_abi.PKV_ITEMS_LONGEST_FIRST, _abi.PKV_ITEMS_SEQUENCES_LONGEST_FIRST,
          _abi.PKV_ITEMS_BATCH_ORDER)


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


def expected(lens, hkv, max_len, P, order):
    Pe, NP = grid(max_len, P)
    slots = []
    for s in range(len(lens)):
        L = int(lens[s])
        for h in range(hkv):
            for p in range(NP):
                tokens = min(Pe, L - p * Pe)
                if p == 0 or tokens > 0:  # partition 0 always, later ones if they hold tokens
                    slots.append(dict(flat=(s * hkv + h) * NP + p, s=s, h=h, p=p, L=L,
                                      tiles=-(-tokens // 16)))
    if order == _abi.PKV_ITEMS_LONGEST_FIRST:
        key = lambda it: (-it["tiles"], it["s"], it["p"], it["h"])  # noqa: E731
    elif order == _abi.PKV_ITEMS_SEQUENCES_LONGEST_FIRST:
        key = lambda it: (-it["L"], it["s"], it["p"], it["h"])  # noqa: E731
    else:
        key = lambda it: (it["s"], it["p"], it["h"])  # noqa: E731
    return [it["flat"] for it in sorted(slots, key=key)]


@pytest.mark.parametrize("P", [0, 16, 64, 512, 1024, 4096])
@pytest.mark.parametrize("hkv", [1, 3, 8])
def test_items_are_the_grid_slots_holding_tokens_in_each_order(P, hkv):
    g = np.random.default_rng(P * 31 + hkv)
    for trial in range(6):
        S = int(g.integers(1, 40))
        lens = g.integers(0, 3000, S).astype(np.int32)
        lens[g.integers(0, S)] = 0
        lens[g.integers(0, S)] = lens[g.integers(0, S)]  # a tie
        max_len = int(lens.max()) + int(g.integers(0, 50))
        for order in ORDERS:
            got = _abi.pkv_decode_work_items(lens, hkv, max_len, P, order=order).tolist()
            assert got == expected(lens, hkv, max_len, P, order), order


# lengths 5, 40, 17, 0, 1024, 1025, 3000 over 2 KV heads, P = 1024: the grid
# has 3 partitions per (sequence, KV head); flat = (s * 2 + h) * 3 + p
HAND = [5, 40, 17, 0, 1024, 1025, 3000]


def test_longest_first_on_a_hand_worked_batch():
    got = _abi.pkv_decode_work_items(HAND, 2, 3000, 1024).tolist()
    assert got == [24, 27, 30, 33, 36, 39, 37, 40,  # 64 tiles: full partitions
                   38, 41,                          # 60 tiles: 3000 - 2048 = 952 tokens
                   6, 9,                            # 40 tokens
                   12, 15,                          # 17 tokens
                   0, 3, 31, 34,                    # 5 tokens; 1025's second partition
                   18, 21]                          # the empty context


def test_sequences_longest_first_on_a_hand_worked_batch():
    got = _abi.pkv_decode_work_items(HAND, 2, 3000, 1024,
                                     order=_abi.PKV_ITEMS_SEQUENCES_LONGEST_FIRST).tolist()
    assert got == [36, 39, 37, 40, 38, 41,  # 3000 tokens: partitions 0, 1, 2
                   30, 33, 31, 34,          # 1025
                   24, 27,                  # 1024
                   6, 9, 12, 15, 0, 3,      # 40, 17, 5
                   18, 21]                  # 0


def test_batch_order_on_a_hand_worked_batch():
    got = _abi.pkv_decode_work_items(HAND, 2, 3000, 1024,
                                     order=_abi.PKV_ITEMS_BATCH_ORDER).tolist()
    assert got == [0, 3, 6, 9, 12, 15, 18, 21, 24, 27, 30, 33, 31, 34, 36, 39, 37, 40, 38, 41]


def test_unknown_order_is_refused():
    with pytest.raises(_abi.PkvError):
        _abi.pkv_decode_work_items([3, 4], 1, 4, 0, order=3)


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
