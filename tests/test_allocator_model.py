"""Pins of the Python block-pool model (the allocator oracle).

The model is pinned by a hand-worked trace, by the pages' worked
fragmentation example, and by invariants the pages state: waste of at most
block_size - 1 slots per sequence, conservation of blocks, refcount equal to
the number of holders, and copy-on-write only for a shared block.
"""
import random

import pytest

from oracle.allocator_model import ERR_INVALID, ERR_OOM, OK, PoolModel
from tests.conftest import golden_lines


def run_trace(pool, rows):
    for r in rows:
        op = r[0]
        if op in ("pool", "expect_free", "expect_refcount", "expect_seq"):
            continue
        arrow = r.index("->")
        args = [int(x) for x in r[1:arrow]]
        want = [int(x) for x in r[arrow + 1:]]
        if op == "add":
            got = [pool.seq_add(*args)]
        elif op == "fork":
            got = [pool.seq_fork(*args)]
        elif op == "free":
            got = [pool.seq_free(*args)]
        elif op == "append":
            got = list(pool.seq_append(*args))
            if want[0] != 0:
                got = got[:1]
        else:
            raise AssertionError(op)
        assert got == want, (r, got)


def test_hand_worked_trace():
    rows = golden_lines("allocator_trace.txt")
    nb, bs = int(rows[0][1]), int(rows[0][2])
    pool = PoolModel(nb, bs)
    run_trace(pool, rows)
    exp = {r[0]: r[1:] for r in rows if r[0].startswith("expect")}
    assert pool.free == [int(x) for x in exp["expect_free"]]
    assert pool.refcount == [int(x) for x in exp["expect_refcount"]]
    sid, table, ntok = exp["expect_seq"]
    assert pool.tables == {int(sid): [int(x) for x in table.split(",")]}
    assert pool.tokens == {int(sid): int(ntok)}


def test_pages_worked_fragmentation_example():
    g = {r[0]: int(r[1]) for r in golden_lines("waste_worked_example.txt")}
    assert g["reserved_tokens"] - g["used_tokens"] == g["contiguous_waste"]
    pool = PoolModel(64, g["block_size"])
    assert pool.seq_add(0, g["used_tokens"]) == OK
    assert len(pool.tables[0]) == g["paged_blocks"]
    assert len(pool.tables[0]) * pool.block_size == g["paged_slots"]
    assert pool.waste(0) == g["paged_waste"]
    assert g["paged_waste"] <= g["max_waste_per_sequence"] == g["block_size"] - 1


def test_first_allocations_are_in_order_and_lifo_reuse():
    pool = PoolModel(8, 4)
    assert pool.seq_add(0, 9) == OK
    assert pool.tables[0] == [0, 1, 2]
    assert pool.seq_free(0) == OK
    assert pool.free[-3:] == [0, 1, 2]  # pushed in table order
    assert pool.seq_add(1, 4) == OK
    assert pool.tables[1] == [2]  # last freed, first reused


def test_oom_changes_nothing():
    pool = PoolModel(3, 4)
    assert pool.seq_add(0, 8) == OK
    before = pool.state()
    assert pool.seq_add(1, 5) == ERR_OOM
    assert pool.state() == before
    assert pool.seq_add(1, 3) == OK
    mid = pool.state()
    st, slot, src, dst = pool.seq_append(1)  # fills offset 3: no new block
    assert (st, src, dst) == (OK, -1, -1) and slot == pool.tables[1][0] * 4 + 3
    assert pool.state() != mid
    before = pool.state()
    assert pool.seq_append(1)[0] == ERR_OOM  # would need a 4th block
    assert pool.state() == before


def test_invalid_operations():
    pool = PoolModel(4, 4)
    assert pool.seq_add(0, 1) == OK
    assert pool.seq_add(0, 1) == ERR_INVALID
    assert pool.seq_fork(5, 6) == ERR_INVALID
    assert pool.seq_fork(0, 0) == ERR_INVALID
    assert pool.seq_free(9) == ERR_INVALID
    assert pool.seq_append(9)[0] == ERR_INVALID


def test_eight_siblings_share_a_partial_block_seven_copy():
    """Parallel sampling: 8 sequences share a prompt whose last block is
    partial.  Appending in ascending id order, the first 7 copy the block,
    the last holder writes in place."""
    bs = 16
    pool = PoolModel(200, bs)
    assert pool.seq_add(0, 1024 + 5) == OK
    for c in range(1, 8):
        assert pool.seq_fork(0, c) == OK
    shared_last = pool.tables[0][-1]
    assert pool.refcount[shared_last] == 8
    cows = []
    for s in range(8):
        st, slot, src, dst = pool.seq_append(s)
        assert st == OK
        assert slot == pool.tables[s][-1] * bs + 5
        if src >= 0:
            cows.append((s, src, dst))
    assert [c[0] for c in cows] == list(range(7))
    assert all(src == shared_last for _, src, _ in cows)
    assert pool.tables[7][-1] == shared_last and pool.refcount[shared_last] == 1
    # the prefix's full blocks stay shared by all 8
    for b in pool.tables[0][:-1]:
        assert pool.refcount[b] == 8


def random_ops(pool, rng, n_ops, max_seqs=12):
    live = []
    next_id = 0
    for _ in range(n_ops):
        r = rng.random()
        if r < 0.2 or not live:
            st = pool.seq_add(next_id, rng.randint(0, 3 * pool.block_size))
            if st == OK:
                live.append(next_id)
            next_id += 1
        elif r < 0.35 and len(live) < max_seqs:
            parent = rng.choice(live)
            assert pool.seq_fork(parent, next_id) == OK
            live.append(next_id)
            next_id += 1
        elif r < 0.85:
            pool.seq_append(rng.choice(live))
        else:
            s = rng.choice(live)
            assert pool.seq_free(s) == OK
            live.remove(s)
        yield


def check_invariants(pool):
    holders = [0] * pool.num_blocks
    for s, table in pool.tables.items():
        for b in table:
            holders[b] += 1
        # waste bound of the pages: at most block_size - 1 unused slots
        assert 0 <= pool.waste(s) <= pool.block_size - 1
        assert len(table) == -(-pool.tokens[s] // pool.block_size)
    assert holders == pool.refcount
    used = sum(1 for h in holders if h > 0)
    assert used + len(pool.free) == pool.num_blocks
    assert len(set(pool.free)) == len(pool.free)
    assert all(holders[b] == 0 for b in pool.free)


@pytest.mark.parametrize("seed", range(6))
def test_invariants_under_random_operations(seed):
    rng = random.Random(seed)
    pool = PoolModel(rng.choice([8, 16, 40]), rng.choice([1, 2, 4, 16]))
    for _ in random_ops(pool, rng, 400):
        check_invariants(pool)


def test_initial_order_is_taken_front_first():
    pool = PoolModel(5, 2, free_order=[3, 0, 4, 1, 2])
    assert pool.seq_add(0, 3) == OK
    assert pool.tables[0] == [3, 0]
    assert pool.seq_append(0)[1] == 0 * 2 + 1
    assert pool.seq_append(0)[1] == 4 * 2 + 0
    with pytest.raises(ValueError):
        PoolModel(3, 2, free_order=[0, 0, 1])


# ---------------------------------------------------------------------------
# block swapping ("PagedAttention 动态内存分页" page, 动态块分配与回收)
# ---------------------------------------------------------------------------
def test_swap_hand_worked_trace():
    # GPU pool of 4 blocks (first taken 0, 1, ...), host pool of 3, bs 4
    pool = PoolModel(4, 4)
    assert pool.seq_swap_out(1) == (ERR_INVALID, [])  # no host pool yet
    assert pool.set_host_blocks(3) == OK
    assert pool.set_host_blocks(3) == ERR_INVALID  # made once
    assert pool.seq_add(1, 6) == OK  # blocks 0, 1
    assert pool.seq_fork(1, 2) == OK  # both shared
    # seq 1 out: host blocks 0, 1; the GPU blocks stay with seq 2
    assert pool.seq_swap_out(1) == (OK, [(0, 0), (1, 1)])
    assert pool.refcount == [1, 1, 0, 0] and pool.free == [3, 2]
    assert pool.host_free == [2] and pool.tables[1] == [0, 1]
    assert pool.seq_append(1)[0] == ERR_INVALID
    assert pool.seq_fork(1, 3) == ERR_INVALID
    assert pool.seq_swap_out(1) == (ERR_INVALID, [])
    # seq 1 back in: GPU blocks 2, 3; host blocks return in table order
    assert pool.seq_swap_in(1) == (OK, [(0, 2), (1, 3)])
    assert pool.free == [] and pool.host_free == [2, 0, 1]
    assert pool.tables[1] == [2, 3] and pool.tokens[1] == 6
    assert pool.seq_swap_in(1) == (ERR_INVALID, [])
    # seq 2 out: host 1 then 0; its GPU blocks are freed in table order
    assert pool.seq_swap_out(2) == (OK, [(0, 1), (1, 0)])
    assert pool.free == [0, 1] and pool.refcount == [0, 0, 1, 1]
    # a third sequence of 3 blocks cannot go out: one host block is left
    assert pool.seq_free(1) == OK  # pushes 2, 3: free [0, 1, 2, 3]
    assert pool.seq_add(3, 12) == OK  # takes 3, 2, 1 (LIFO)
    assert pool.tables[3] == [3, 2, 1]
    before = (pool.state(), pool.host_state())
    assert pool.seq_swap_out(3) == (ERR_OOM, [])
    assert (pool.state(), pool.host_state()) == before
    # swapped-out seq 2 (2 blocks) cannot come back while only block 0 is free
    assert pool.free == [0]
    assert pool.seq_swap_in(2) == (ERR_OOM, [])
    assert (pool.state(), pool.host_state()) == before
    # freeing a swapped sequence returns its host blocks
    assert pool.seq_free(2) == OK
    assert pool.host_free == [2, 1, 0] and pool.host_refcount == [0, 0, 0]


def _check_swap_invariants(pool):
    resident = {s: t for s, t in pool.tables.items() if s not in pool.swapped}
    swapped = {s: t for s, t in pool.tables.items() if s in pool.swapped}
    for b in range(pool.num_blocks):
        holders = sum(t.count(b) for t in resident.values())
        assert pool.refcount[b] == holders
        assert (b in pool.free) == (holders == 0)
    for h in range(len(pool.host_refcount)):
        holders = sum(t.count(h) for t in swapped.values())
        assert pool.host_refcount[h] == holders <= 1
        assert (h in pool.host_free) == (holders == 0)
    assert len(pool.free) == len(set(pool.free))
    assert len(pool.host_free) == len(set(pool.host_free))


@pytest.mark.parametrize("seed", range(6))
def test_swap_invariants_under_random_operations(seed):
    rnd = random.Random(seed)
    pool = PoolModel(40, 4)
    pool.set_host_blocks(30)
    tokens_before = {}
    for _ in range(600):
        op = rnd.random()
        ids = list(pool.tables)
        if op < 0.2 or not ids:
            pool.seq_add(rnd.randrange(100), rnd.randrange(0, 30))
        elif op < 0.3:
            pool.seq_fork(rnd.choice(ids), rnd.randrange(100))
        elif op < 0.55:
            pool.seq_append(rnd.choice(ids))
        elif op < 0.7:
            s = rnd.choice(ids)
            tokens_before[s] = pool.tokens[s]
            st, pairs = pool.seq_swap_out(s)
            if st == OK:
                assert [h for _, h in pairs] == pool.tables[s]
        elif op < 0.85:
            s = rnd.choice(ids)
            table = list(pool.tables[s])
            st, pairs = pool.seq_swap_in(s)
            if st == OK:
                assert [h for h, _ in pairs] == table
                assert pool.tokens[s] == tokens_before[s]
        else:
            pool.seq_free(rnd.choice(ids))
        _check_swap_invariants(pool)
