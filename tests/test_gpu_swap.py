"""Block swap between the GPU pool and pinned host memory ("PagedAttention
动态内存分页" page, 动态块分配与回收), through the C ABI.

The copies are compared bit for bit with the oracle's swap copy in both
directions; the decode step driver's swap-out / swap-in round trip leaves
every swapped sequence's attention output bit-identical (its blocks come
back elsewhere, and decode is bit-exact under block permutation) and equal
to the oracle within the attention tolerance.
"""
import ctypes as C

import numpy as np
import pytest
import torch

from oracle import reference as ref
from paged_kv_cache_337_b200 import _abi, build
from paged_kv_cache_337_b200.cache import PagedKVCache
from tests.helpers import tolerance_violation

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib(cuda_device):
    build.build()
    _abi.lib()


def _pairs(gen, n_src, n_dst, n):
    src = torch.randperm(n_src, generator=gen)[:n]
    dst = torch.randperm(n_dst, generator=gen)[:n]
    return torch.stack([src, dst], dim=1).to(torch.int32)


@pytest.mark.parametrize("shape,dtype", [((16, 32, 128), torch.bfloat16),
                                         ((16, 8, 64), torch.float16),
                                         ((3, 1, 8), torch.bfloat16),
                                         ((16, 32, 128), torch.uint8)])
def test_swap_out_and_in_bit_exact(shape, dtype, cuda_device):
    g = torch.Generator().manual_seed(61)
    nb, nh = 37, 23
    if dtype == torch.uint8:
        mk = lambda n: torch.randint(0, 256, (n,) + shape, generator=g, dtype=torch.uint8)
    else:
        mk = lambda n: torch.randn((n,) + shape, generator=g).to(dtype)
    gk, gv = mk(nb), mk(nb)
    hk, hv = mk(nh).pin_memory(), mk(nh).pin_memory()
    dk, dv = gk.to(cuda_device), gv.to(cuda_device)
    err = torch.zeros(2, dtype=torch.int32, device=cuda_device)
    out_pairs = _pairs(g, nb, nh, 19)
    want_hk = ref.swap_blocks(hk, gk, out_pairs)
    want_hv = ref.swap_blocks(hv, gv, out_pairs)
    _abi.pkv_swap_blocks(dk, dv, hk, hv, out_pairs.to(cuda_device), dev_error=err)
    torch.cuda.synchronize()
    assert np.array_equal(ref._u8(hk), want_hk)
    assert np.array_equal(ref._u8(hv), want_hv)
    in_pairs = _pairs(g, nh, nb, 17)
    want_gk = ref.swap_blocks(gk, hk, in_pairs)
    want_gv = ref.swap_blocks(gv, hv, in_pairs)
    _abi.pkv_swap_blocks(hk, hv, dk, dv, in_pairs.to(cuda_device), dev_error=err)
    torch.cuda.synchronize()
    assert np.array_equal(ref._u8(dk.cpu()), want_gk)
    assert np.array_equal(ref._u8(dv.cpu()), want_gv)
    assert err.tolist() == [0, 0]


def test_swap_one_pool_with_4_byte_words(cuda_device):
    # fp32 scales of 2 KV heads: 8-byte blocks, the 4-byte path
    g = torch.Generator().manual_seed(62)
    ks = torch.rand(40, 2, generator=g)
    host = torch.zeros(30, 2).pin_memory()
    pairs = _pairs(g, 40, 30, 25)
    want = ref.swap_blocks(host, ks, pairs)
    _abi.pkv_swap_blocks(ks.to(cuda_device), None, host, None, pairs.to(cuda_device))
    torch.cuda.synchronize()
    assert np.array_equal(ref._u8(host), want)


def test_swap_pairs_in_pinned_memory_and_bad_pairs_reported(cuda_device):
    g = torch.Generator().manual_seed(63)
    gk = torch.randn(8, 16, 4, 8).to(torch.float16).to(cuda_device)
    hk = torch.zeros(4, 16, 4, 8, dtype=torch.float16).pin_memory()
    pairs = torch.tensor([[1, 0], [7, 3], [2, 4]], dtype=torch.int32).pin_memory()
    err = torch.zeros(2, dtype=torch.int32, device=cuda_device)
    _abi.pkv_swap_blocks(gk, None, hk, None, pairs, dev_error=err)
    torch.cuda.synchronize()
    assert err.tolist() == [_abi.PKV_DEVERR_PAIR, 2]  # host block 4 of 4
    assert torch.equal(hk[0], gk[1].cpu()) and torch.equal(hk[3], gk[7].cpu())


def test_pageable_host_memory_is_rejected_before_launch(cuda_device):
    gk = torch.zeros(4, 256, dtype=torch.uint8, device=cuda_device)
    pageable = np.zeros((4, 256), np.uint8)
    pairs = torch.tensor([[0, 0]], dtype=torch.int32, device=cuda_device)
    L = _abi.lib()
    st = L.pkv_swap_blocks(gk.data_ptr(), None, pageable.ctypes.data_as(C.c_void_p), None,
                           pairs.data_ptr(), 1, 4, 4, 256, 256, 256, None, None)
    assert st == _abi.PKV_ERR_INVALID
    assert b"pageable" in L.pkv_last_error()
    with pytest.raises(ValueError):
        _abi.pkv_swap_blocks(gk, None, torch.zeros(4, 256, dtype=torch.uint8), None, pairs)
    torch.cuda.synchronize()
    assert not pageable.any()


@pytest.mark.parametrize("fp8", [False, True])
def test_cache_swap_round_trip_keeps_outputs(fp8, cuda_device):
    dev = cuda_device
    g = torch.Generator().manual_seed(64 + fp8)
    bs, Hq, Hkv, D = 16, 8, 2, 128
    lens = [40, 300, 17, 129, 64, 200]
    nb = sum(-(-(L + 40) // bs) for L in lens) + 4
    cache = PagedKVCache(nb, bs, Hq, Hkv, D, torch.bfloat16, dev, 64,
                         free_order=torch.randperm(nb, generator=g).tolist(),
                         kv_dtype=torch.uint8 if fp8 else None, kv_scale=0.02)
    cache.enable_swap(nb)
    if fp8:
        # distinct scales per (block, KV head), set before any write
        cache.k_scale.copy_((0.01 + 0.02 * torch.rand(nb, Hkv, generator=g)).to(dev))
        cache.v_scale.copy_((0.01 + 0.02 * torch.rand(nb, Hkv, generator=g)).to(dev))
    for s, L in enumerate(lens):
        k = torch.randn(L, Hkv, D, generator=g).to(torch.bfloat16).to(dev)
        v = torch.randn(L, Hkv, D, generator=g).to(torch.bfloat16).to(dev)
        cache.add_sequence(s, L, k, v)
    ids = list(range(len(lens)))
    qs = torch.randn(len(lens), Hq, D, generator=g).to(torch.bfloat16)

    def attend(seq_ids):
        tables, tl = cache.pool.block_tables(seq_ids, cache.max_blocks_per_seq)
        q = qs[seq_ids].to(dev)
        out = torch.empty_like(q)
        cache._attend(out, q, tables.to(dev), tl.to(dev), int(tl.max()), cache.workspace(
            len(seq_ids), int(tl.max())), None)
        torch.cuda.synchronize()
        return out.cpu()

    before = attend(ids)
    gone = [1, 3, 4]
    moved = cache.swap_out(gone)
    assert moved == sum(-(-lens[s] // bs) for s in gone)
    stay = [0, 2, 5]
    # the other sequences keep decoding into the freed blocks
    for _ in range(40):
        S = len(stay)
        q = torch.randn(S, Hq, D, generator=g).to(torch.bfloat16).to(dev)
        k = torch.randn(S, Hkv, D, generator=g).to(torch.bfloat16).to(dev)
        v = torch.randn(S, Hkv, D, generator=g).to(torch.bfloat16).to(dev)
        cache.decode_step(stay, q, k, v)
    assert cache.swap_in(gone) == moved
    after = attend(gone)
    cache.check_errors()
    assert torch.equal(after, before[gone])
    # and against the oracle on the swapped-in blocks
    tables, tl = cache.pool.block_tables(gone, cache.max_blocks_per_seq)
    q = qs[gone]
    if fp8:
        want = ref.decode_attention_fp8(q, cache.key_cache.cpu(), cache.value_cache.cpu(),
                                        cache.k_scale.cpu(), cache.v_scale.cpu(), tables, tl,
                                        cache.scale, "bf16", Hkv, bs)
    else:
        want = ref.decode_attention(q, cache.key_cache.cpu(), cache.value_cache.cpu(), tables,
                                    tl, cache.scale, "bf16", Hkv, bs)
    assert tolerance_violation(after, want) <= 0
