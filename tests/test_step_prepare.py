"""pkv_step_prepare (the host part of a decode step in one call) against the
three calls it composes — pkv_seq_append_batch, pkv_pool_block_tables and
pkv_decode_work_items — on two pools driven through the same operations,
and the layout of pkv_decode_step_args as the binding declares it against a
C compiler's."""
import ctypes as C
import os
import subprocess
import tempfile

import numpy as np
import pytest
import torch

from paged_kv_cache_337_b200 import _abi, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    _abi.lib()


def _separate(pool, ids, mb, hkv, P, order_split, order_one):
    slots, pairs = pool.append_batch(ids)
    tables, lens, longest = pool.block_tables(ids, mb, -1, with_max=True)
    split = 0 < P < longest
    order = order_split if split else order_one
    items = None
    if order >= 0 and len(ids):
        items = _abi.pkv_decode_work_items(lens, hkv, longest, P, order=order)
    return slots, pairs, tables, lens, longest, items


def _combined(pool, ids, mb, hkv, P, order_split, order_one, cap):
    n = len(ids)
    ids_t = torch.as_tensor(ids, dtype=torch.int64)
    slots = torch.empty(n, dtype=torch.int64)
    pairs = torch.empty((n, 2), dtype=torch.int32)
    tables = torch.empty((n, mb), dtype=torch.int32)
    lens = torch.empty(n, dtype=torch.int32)
    items = torch.full((cap,), -7, dtype=torch.int32)
    npairs, longest, nitems = C.c_int(), C.c_int(), C.c_int()
    st = _abi.lib().pkv_step_prepare(
        pool._h, n, _abi._ptr(ids_t), _abi._ptr(slots), _abi._ptr(pairs), C.byref(npairs),
        _abi._ptr(tables), mb, _abi._ptr(lens), C.byref(longest), hkv, P, order_split,
        order_one, _abi._ptr(items), cap, C.byref(nitems))
    _abi._check(st, "pkv_step_prepare")
    it = items[:nitems.value] if nitems.value >= 0 else None
    return slots, pairs[:npairs.value], tables, lens, longest.value, it


@pytest.mark.parametrize("orders", [(-1, -1), (0, -1), (1, -1), (2, 2), (0, 0)])
@pytest.mark.parametrize("P", [0, 32, 256])
def test_one_call_equals_the_three_it_composes(orders, P):
    g = np.random.default_rng(P + 7 * orders[0] + 13)
    nb, bs, hkv, mb = 400, 16, 4, 64
    order0 = torch.randperm(nb, generator=torch.Generator().manual_seed(P)).tolist()
    pools = [_abi.BlockPool(nb, bs, order0) for _ in range(2)]
    lens = g.integers(0, 300, 12).tolist()
    lens[3], lens[5] = 37, 50  # partial last blocks, shared by the forks below
    for pool in pools:
        for s, L in enumerate(lens):
            pool.add(s, L)
        pool.fork(3, 100)  # a shared partial block: the next appends copy it
        pool.fork(5, 101)
    ids = list(range(12)) + [100, 101]
    cap = len(ids) * hkv * mb
    for step in range(20):
        a = _separate(pools[0], ids, mb, hkv, P, *orders)
        b = _combined(pools[1], ids, mb, hkv, P, *orders, cap)
        assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])
        assert torch.equal(a[2], b[2]) and torch.equal(a[3], b[3]) and a[4] == b[4]
        assert (a[5] is None) == (b[5] is None)
        if a[5] is not None:
            assert torch.equal(a[5], b[5])
        if step == 0:
            assert a[1].shape[0] == 2  # the two forked sequences' copies
    assert pools[0].free_list() == pools[1].free_list()


def test_no_sequences_and_an_unknown_sequence():
    pool = _abi.BlockPool(8, 16)
    out = _combined(pool, [], 4, 2, 0, 0, 0, 1)
    assert out[4] == 0 and out[5] is None
    with pytest.raises(_abi.PkvError):
        _combined(pool, [5], 4, 2, 0, 0, 0, 8)


def test_step_args_layout_matches_the_header():
    fields = [f for f, _ in _abi.DecodeStepArgs._fields_]
    src = ['#include <stdio.h>', '#include <stddef.h>', '#include "pkv.h"', 'int main(void) {']
    src += ['printf("%%s %%zu\\n", "%s", offsetof(pkv_decode_step_args, %s));' % (f, f)
            for f in fields]
    src += ['printf("size %zu\\n", sizeof(pkv_decode_step_args));', 'return 0;', '}']
    with tempfile.TemporaryDirectory() as d:
        c_file, exe = os.path.join(d, "layout.c"), os.path.join(d, "layout")
        with open(c_file, "w") as f:
            f.write("\n".join(src))
        subprocess.check_call(["gcc", "-I", os.path.join(ROOT, "include"), "-I",
                               "/usr/local/cuda/include", c_file, "-o", exe])
        out = subprocess.check_output([exe]).decode().split()
    got = dict(zip(out[0::2], map(int, out[1::2])))
    assert got.pop("size") == C.sizeof(_abi.DecodeStepArgs)
    assert got == {f: getattr(_abi.DecodeStepArgs, f).offset for f in fields}


def test_decode_step_rejects_an_upload_stream_without_its_event():
    """pkv_decode_step returns PKV_ERR_INVALID before any device work when
    the uploads go on meta_stream but no meta_event is given, or when an
    input upload has no buffers.  (The stream value is never used: the
    check comes first.)"""
    a = _abi.DecodeStepArgs()
    host = (C.c_uint8 * 64)()
    a.meta_host, a.meta_device, a.meta_bytes = C.addressof(host), C.addressof(host), 64
    a.meta_stream, a.meta_event = 0x1, None
    assert _abi.lib().pkv_decode_step(C.byref(a), None) == _abi.PKV_ERR_INVALID
    b = _abi.DecodeStepArgs()
    b.in_bytes, b.in_host, b.in_device = 64, None, None
    assert _abi.lib().pkv_decode_step(C.byref(b), None) == _abi.PKV_ERR_INVALID
