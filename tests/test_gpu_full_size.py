"""Parity at the workloads' full sizes, in the launch configuration the
benchmark times (same partition size, same pool, same step driver).

The caches are drawn on the CPU (seeded) so the oracle sees the same bits.
The oracle recomputes a seeded sample of whole output rows (every head of
the sampled sequences); the slot write is checked bit for bit at every
written slot and on a sample of untouched blocks.  The shared-prefix
workload is small enough to check whole caches bit for bit.
"""
import numpy as np
import pytest
import torch

from oracle import reference as ref
from oracle.allocator_model import PoolModel
from paged_kv_cache_337_b200 import _abi, build
from paged_kv_cache_337_b200 import workloads as W
from paged_kv_cache_337_b200.cache import PagedKVCache
from tests.helpers import tolerance_violation

pytestmark = pytest.mark.gpu

ATOL, RTOL = 2e-3, 1e-2


@pytest.fixture(scope="module", autouse=True)
def _lib(cuda_device):
    build.build()
    _abi.lib()


def full_step(spec, dev, n_sample=16):
    inp = W.make_decode_inputs(spec)
    S, bs, Hkv = spec.num_seqs, spec.block_size, spec.num_kv_heads
    lens = inp.context_lens.tolist()
    order = inp.free_order.tolist()
    model = PoolModel(inp.num_blocks, bs, free_order=order)
    cache = PagedKVCache(inp.num_blocks, bs, spec.num_q_heads, Hkv, spec.head_dim,
                         spec.torch_dtype, dev, spec.max_blocks_per_seq, spec.partition_size,
                         free_order=order, key_cache=inp.key_cache.to(dev),
                         value_cache=inp.value_cache.to(dev), scale=spec.scale)
    for s in range(S):
        cache.add_sequence(s, lens[s] - 1)
        assert model.seq_add(s, lens[s] - 1) == 0
    out = cache.decode_step(list(range(S)), inp.query.to(dev), inp.new_key.to(dev),
                            inp.new_value.to(dev)).cpu()
    cache.check_errors()
    slots = []
    for s in range(S):
        st, slot, src, dst = model.seq_append(s)
        assert st == 0 and src < 0
        slots.append(slot)
        assert cache.pool.block_table(s) == model.tables[s]

    # slot write: every written row, bit for bit
    blk = torch.tensor([x // bs for x in slots])
    off = torch.tensor([x % bs for x in slots])
    got_k = cache.key_cache[blk.to(dev), off.to(dev)].cpu()
    got_v = cache.value_cache[blk.to(dev), off.to(dev)].cpu()
    assert torch.equal(got_k.view(torch.int16), inp.new_key.view(torch.int16))
    assert torch.equal(got_v.view(torch.int16), inp.new_value.view(torch.int16))
    # untouched blocks stay as drawn
    g = torch.Generator().manual_seed(spec.seed + 7)
    written = set(blk.tolist())
    probe = [b for b in torch.randperm(inp.num_blocks, generator=g)[:64].tolist()
             if b not in written]
    pb = torch.tensor(probe)
    assert torch.equal(cache.key_cache[pb.to(dev)].cpu().view(torch.int16),
                       inp.key_cache[pb].view(torch.int16))

    # attention: whole rows of a seeded sample of sequences
    kc = inp.key_cache
    vc = inp.value_cache
    kc[blk, off] = inp.new_key
    vc[blk, off] = inp.new_value
    rows = sorted(torch.randperm(S, generator=g)[:n_sample].tolist())
    tables = np.full((len(rows), spec.max_blocks_per_seq), -1, np.int32)
    for i, s in enumerate(rows):
        tables[i, :len(model.tables[s])] = model.tables[s]
    want = ref.decode_attention(inp.query[rows], kc, vc, tables,
                                np.array([lens[s] for s in rows], np.int32), spec.scale,
                                spec.dtype, Hkv, bs)
    assert tolerance_violation(out[rows], want, ATOL, RTOL) <= 0
    assert torch.isfinite(out.float()).all()
    return out


def test_full_size_7b_decode_step(cuda_device):
    full_step(W.DECODE_7B, cuda_device)


def test_full_size_70b_gqa_decode_step(cuda_device):
    full_step(W.GQA_70B, cuda_device)


@pytest.mark.parametrize("spec", [W.LONG_BS32, W.LONG_BS64], ids=["bs32", "bs64"])
def test_full_size_long_context_split_k(spec, cuda_device):
    full_step(spec, cuda_device, n_sample=8)


def test_full_size_shared_prefix_workload(cuda_device):
    """16 prompts x 8 samples sharing a 1024-token prefix: fork step with
    112 copy-on-write copies, divergence, steady step; whole caches bit-exact,
    every output row within tolerance, outputs bit-identical to physically
    duplicated prefixes."""
    from tests.shared_prefix import run_shared_prefix

    run_shared_prefix(W.SHARED_PREFIX, cuda_device, partition_size=0, check_all=True)
