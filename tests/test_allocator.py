"""The native block pool agrees bit for bit with the Python allocator model
(the allocator oracle) after every operation: free stack, refcounts, tables,
token counts, slots and copy-on-write pairs."""
import random

import pytest

from oracle.allocator_model import ERR_INVALID, ERR_OOM, OK, PoolModel
from paged_kv_cache_337_b200 import _abi, build
from tests.conftest import golden_lines


@pytest.fixture(scope="module", autouse=True)
def _built():
    build.build()


def native_state(pool, seq_ids):
    tables = []
    for s in sorted(seq_ids):
        tables.append((s, tuple(pool.block_table(s)), pool.num_tokens(s)))
    return tuple(pool.free_list()), tuple(pool.refcounts()), tuple(tables)


def status_of(fn, *args):
    try:
        r = fn(*args)
        return OK, r
    except _abi.PkvError as e:
        return e.status, None


def test_native_follows_hand_worked_trace():
    rows = golden_lines("allocator_trace.txt")
    nb, bs = int(rows[0][1]), int(rows[0][2])
    pool = _abi.BlockPool(nb, bs)
    live = set()
    for r in rows[1:]:
        if r[0].startswith("expect"):
            continue
        arrow = r.index("->")
        args = [int(x) for x in r[1:arrow]]
        want = [int(x) for x in r[arrow + 1:]]
        op = r[0]
        if op == "add":
            st, _ = status_of(pool.add, *args)
            got = [st]
            if st == OK:
                live.add(args[0])
        elif op == "fork":
            st, _ = status_of(pool.fork, *args)
            got = [st]
            live.add(args[1])
        elif op == "free":
            st, _ = status_of(pool.free, *args)
            got = [st]
            live.discard(args[0])
        else:
            st, res = status_of(pool.append, *args)
            got = [st] + (list(res) if st == OK else [])
        assert got == want, (r, got)
    exp = {r[0]: r[1:] for r in rows if r[0].startswith("expect")}
    assert pool.free_list() == [int(x) for x in exp["expect_free"]]
    assert pool.refcounts() == [int(x) for x in exp["expect_refcount"]]
    sid, table, ntok = exp["expect_seq"]
    assert pool.block_table(int(sid)) == [int(x) for x in table.split(",")]
    assert pool.num_tokens(int(sid)) == int(ntok)


@pytest.mark.parametrize("seed", range(8))
def test_native_matches_model_under_random_operations(seed):
    rng = random.Random(100 + seed)
    nb = rng.choice([6, 16, 40, 97])
    bs = rng.choice([1, 4, 16, 32])
    order = list(range(nb))
    if seed % 2:
        rng.shuffle(order)
    model = PoolModel(nb, bs, free_order=order)
    native = _abi.BlockPool(nb, bs, free_order=order)
    live, next_id = [], 0
    for step in range(500):
        r = rng.random()
        if r < 0.2 or not live:
            n = rng.randint(0, 3 * bs)
            a = model.seq_add(next_id, n)
            b, _ = status_of(native.add, next_id, n)
            assert a == b
            if a == OK:
                live.append(next_id)
            next_id += 1
        elif r < 0.35:
            parent = rng.choice(live)
            assert model.seq_fork(parent, next_id) == OK
            assert status_of(native.fork, parent, next_id)[0] == OK
            live.append(next_id)
            next_id += 1
        elif r < 0.85:
            s = rng.choice(live)
            st, slot, src, dst = model.seq_append(s)
            nst, res = status_of(native.append, s)
            assert nst == st
            if st == OK:
                assert res == (slot, src, dst)
        else:
            s = rng.choice(live)
            assert model.seq_free(s) == OK
            assert status_of(native.free, s)[0] == OK
            live.remove(s)
        assert native_state(native, live) == model.state(), step


def test_batch_append_matches_single_appends():
    bs = 16
    model = PoolModel(400, bs)
    native = _abi.BlockPool(400, bs)
    for pool_add, pool_fork in ((model.seq_add, model.seq_fork), (native.add, native.fork)):
        pool_add(0, 1024 + 5)
        for c in range(1, 8):
            pool_fork(0, c)
        pool_add(100, 17)
    ids = list(range(8)) + [100]
    slots, pairs = native.append_batch(ids)
    want_slots, want_pairs = [], []
    for s in ids:
        st, slot, src, dst = model.seq_append(s)
        want_slots.append(slot)
        if src >= 0:
            want_pairs.append([src, dst])
    assert slots.tolist() == want_slots
    assert pairs.tolist() == want_pairs
    assert len(want_pairs) == 7
    assert native_state(native, ids) == model.state()


def test_dense_tables_and_lengths():
    native = _abi.BlockPool(10, 4, free_order=[9, 8, 7, 6, 5, 4, 3, 2, 1, 0])
    native.add(5, 6)
    native.add(7, 1)
    tables, lens = native.block_tables([7, 5], 3, fill=-1)
    assert tables.tolist() == [[7, -1, -1], [9, 8, -1]]
    assert lens.tolist() == [1, 6]
    with pytest.raises(_abi.PkvError):
        native.block_tables([5], 1)


def test_oom_and_invalid_statuses():
    native = _abi.BlockPool(2, 4)
    assert status_of(native.add, 0, 9)[0] == ERR_OOM
    assert native.num_free() == 2
    native.add(0, 8)
    assert status_of(native.append, 0)[0] == ERR_OOM
    assert native.num_tokens(0) == 8
    assert status_of(native.add, 0, 1)[0] == ERR_INVALID
    assert status_of(native.free, 3)[0] == ERR_INVALID
    with pytest.raises(_abi.PkvError):
        _abi.BlockPool(3, 4, free_order=[0, 0, 1])


# ---------------------------------------------------------------------------
# block swapping: the native pool follows the model's host pool too
# ---------------------------------------------------------------------------
def native_host_state(pool, seq_ids):
    swapped = tuple(sorted(s for s in seq_ids if pool.is_swapped(s)))
    return tuple(pool.host_free_list()), tuple(pool.host_refcounts()), swapped


@pytest.mark.parametrize("seed", range(8))
def test_native_matches_model_with_swaps(seed):
    rng = random.Random(300 + seed)
    nb = rng.choice([8, 24, 60])
    nh = rng.choice([4, 16, 50])
    bs = rng.choice([1, 4, 16])
    order = list(range(nb))
    rng.shuffle(order)
    model = PoolModel(nb, bs, free_order=order)
    native = _abi.BlockPool(nb, bs, free_order=order)
    assert model.set_host_blocks(nh) == OK
    native.set_host_blocks(nh)
    assert status_of(native.set_host_blocks, nh)[0] == model.set_host_blocks(nh) == ERR_INVALID
    live, next_id = [], 0
    for step in range(600):
        r = rng.random()
        if r < 0.15 or not live:
            n = rng.randint(0, 3 * bs)
            a = model.seq_add(next_id, n)
            assert status_of(native.add, next_id, n)[0] == a
            if a == OK:
                live.append(next_id)
            next_id += 1
        elif r < 0.25:
            parent = rng.choice(live)
            a = model.seq_fork(parent, next_id)
            assert status_of(native.fork, parent, next_id)[0] == a
            if a == OK:
                live.append(next_id)
            next_id += 1
        elif r < 0.55:
            s = rng.choice(live)
            st, slot, src, dst = model.seq_append(s)
            nst, res = status_of(native.append, s)
            assert nst == st
            if st == OK:
                assert res == (slot, src, dst)
        elif r < 0.7:
            s = rng.choice(live)
            st, pairs = model.seq_swap_out(s)
            nst, res = status_of(native.swap_out, s)
            assert nst == st
            if st == OK:
                assert res.tolist() == [list(p) for p in pairs]
        elif r < 0.85:
            s = rng.choice(live)
            st, pairs = model.seq_swap_in(s)
            nst, res = status_of(native.swap_in, s)
            assert nst == st
            if st == OK:
                assert res.tolist() == [list(p) for p in pairs]
        else:
            s = rng.choice(live)
            assert model.seq_free(s) == OK
            assert status_of(native.free, s)[0] == OK
            live.remove(s)
        assert native_state(native, live) == model.state(), step
        assert native_host_state(native, live) == model.host_state(), step


def test_swapped_sequences_leave_the_decode_tables():
    native = _abi.BlockPool(8, 4)
    native.set_host_blocks(8)
    native.add(1, 5)
    native.add(2, 3)
    native.swap_out(1)
    with pytest.raises(_abi.PkvError):
        native.block_tables([1, 2], 4)
    with pytest.raises(_abi.PkvError):
        native.slot_mapping(1, 0, 5)
    tables, lens = native.block_tables([2], 4)
    assert lens.tolist() == [3]
    native.swap_in(1)
    tables, lens = native.block_tables([1, 2], 4)
    assert lens.tolist() == [5, 3]
