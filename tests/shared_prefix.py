"""Shared-prefix parallel sampling scenario, run on the GPU path and on the
oracle side step by step (used by the GPU parity tests).

Scenario ("PagedAttention 动态内存分页" page, 写时复制与内存共享: samples of one
prompt share its blocks; a shared block is copied when one of them writes):
each prompt's first sample takes the prompt's blocks (prefix plus a few
already-decoded tokens, so its last block is partial), the other samples
fork from it, then
  (i)   fork step: every sample appends one token -> copy-on-write of the
        shared partial block for all but the last holder, write, decode;
  (ii)  every sample advances by its own number of private tokens;
  (iii) steady step: one more token each -> write, decode.
"""
import numpy as np
import torch

from oracle import reference as ref
from oracle.allocator_model import PoolModel
from paged_kv_cache_337_b200.cache import PagedKVCache
from paged_kv_cache_337_b200 import workloads as W
from tests.helpers import tolerance_violation

ATOL, RTOL = 2e-3, 1e-2


def _tables(model, ids, mb):
    t = np.full((len(ids), mb), -1, np.int32)
    lens = np.zeros(len(ids), np.int32)
    for i, s in enumerate(ids):
        row = model.tables[s]
        t[i, :len(row)] = row
        lens[i] = model.tokens[s]
    return t, lens


def _native_state(cache, ids):
    pool = cache.pool
    return (tuple(pool.free_list()), tuple(pool.refcounts()),
            tuple(sorted((s, tuple(pool.block_table(s)), pool.num_tokens(s)) for s in ids)))


def run_shared_prefix(spec, dev, partition_size=0, check_all=True, sample_seqs=None):
    inp = W.make_shared_prefix_inputs(spec)
    P, N, bs = spec.num_prompts, spec.samples_per_prompt, spec.block_size
    Hq, Hkv, D, dt = spec.num_q_heads, spec.num_kv_heads, spec.head_dim, spec.torch_dtype
    S = P * N
    ids = list(range(S))
    order = inp.free_order.tolist()
    nb = inp.num_blocks
    max_tokens = int(inp.prompt_lens.max()) + int(inp.diverge.max()) + 2
    mb = -(-max_tokens // bs)
    g = torch.Generator().manual_seed(inp.seed_values)

    model = PoolModel(nb, bs, free_order=order)
    kc0 = torch.zeros((nb, bs, Hkv, D), dtype=dt)
    cache = PagedKVCache(nb, bs, Hq, Hkv, D, dt, dev, mb, partition_size, free_order=order,
                         key_cache=kc0.to(dev), value_cache=kc0.to(dev), scale=spec.scale)
    okc = ref.bits(kc0).copy()
    ovc = okc.copy()

    # prompts: the first sample of each prompt takes and fills the blocks
    for p in range(P):
        n = int(inp.prompt_lens[p])
        k = torch.randn(n, Hkv, D, generator=g).to(dt)
        v = torch.randn(n, Hkv, D, generator=g).to(dt)
        s0 = p * N
        assert model.seq_add(s0, n) == 0
        cache.add_sequence(s0, n, k.to(dev), v.to(dev))
        slots = [model.tables[s0][t // bs] * bs + t % bs for t in range(n)]
        okc, ovc = ref.write_slots(okc, ovc, k, v, slots, bs, Hkv)
        for c in range(1, N):
            assert model.seq_fork(s0, s0 + c) == 0
            cache.fork(s0, s0 + c)
    assert _native_state(cache, ids) == model.state()

    def step(tag):
        nonlocal okc, ovc
        q = torch.randn(S, Hq, D, generator=g).to(dt)
        k = torch.randn(S, Hkv, D, generator=g).to(dt)
        v = torch.randn(S, Hkv, D, generator=g).to(dt)
        out = cache.decode_step(ids, q.to(dev), k.to(dev), v.to(dev)).cpu()
        cache.check_errors()
        slots, pairs = [], []
        for s in ids:
            st, slot, src, dst = model.seq_append(s)
            assert st == 0
            slots.append(slot)
            if src >= 0:
                pairs.append((src, dst))
        assert _native_state(cache, ids) == model.state(), tag
        if pairs:
            okc, ovc = ref.copy_blocks(okc, ovc, pairs, bs, Hkv, D)
        okc, ovc = ref.write_slots(okc, ovc, k, v, slots, bs, Hkv)
        tables, lens = _tables(model, ids, mb)
        if check_all:
            assert np.array_equal(ref.bits(cache.key_cache.cpu()).reshape(-1), okc.reshape(-1))
            assert np.array_equal(ref.bits(cache.value_cache.cpu()).reshape(-1), ovc.reshape(-1))
            rows = ids
        else:
            rows = sample_seqs
        want = ref.decode_attention(q[rows], okc, ovc, tables[rows], lens[rows], spec.scale,
                                    spec.dtype, Hkv, bs)
        assert tolerance_violation(out[rows], want, ATOL, RTOL) <= 0, tag
        return out, q, tables, lens, pairs

    # (i) fork step: every sample but the last holder copies the shared block
    out1, q1, tables1, lens1, pairs1 = step("fork step")
    assert len(pairs1) == P * (N - 1)

    # (ii) each sample advances by its private tokens, one append at a time
    remaining = {s: int(inp.diverge[s]) for s in ids}
    slots, owners = [], []
    while any(remaining.values()):
        for s in ids:
            if remaining[s]:
                st, slot, src, dst = model.seq_append(s)
                nslot, nsrc, ndst = cache.pool.append(s)
                assert st == 0 and (slot, src, dst) == (nslot, nsrc, ndst)
                assert src < 0  # private last blocks: no more copies
                slots.append(slot)
                owners.append(s)
                remaining[s] -= 1
    if slots:
        k = torch.randn(len(slots), Hkv, D, generator=g).to(dt)
        v = torch.randn(len(slots), Hkv, D, generator=g).to(dt)
        from paged_kv_cache_337_b200 import _abi

        _abi.pkv_write_slots(k.to(dev), v.to(dev), cache.key_cache, cache.value_cache,
                             torch.tensor(slots, dtype=torch.int64, device=dev))
        okc, ovc = ref.write_slots(okc, ovc, k, v, slots, bs, Hkv)

    # (iii) steady step
    out3, q3, tables3, lens3, pairs3 = step("steady step")
    assert pairs3 == []

    # copy-on-write equivalence: the same attention with every shared block
    # physically duplicated gives bit-identical outputs
    from paged_kv_cache_337_b200 import _abi

    counts = {}
    for row in tables3:
        for b in row[row >= 0]:
            counts[int(b)] = counts.get(int(b), 0) + 1
    shared = sorted(b for b, c in counts.items() if c > 1)
    assert shared, "the scenario must leave shared prefix blocks"
    extra = sum(counts[b] - 1 for b in shared)
    kbig = torch.cat([cache.key_cache, torch.empty((extra, bs, Hkv, D), dtype=dt, device=dev)])
    vbig = torch.cat([cache.value_cache, torch.empty((extra, bs, Hkv, D), dtype=dt, device=dev)])
    dup = tables3.copy()
    nxt = nb
    seen = {}
    for i in range(S):
        for j in range(mb):
            b = int(dup[i, j])
            if b >= 0 and counts[b] > 1:
                if seen.get(b, 0) > 0:  # first holder keeps the original
                    kbig[nxt] = kbig[b]
                    vbig[nxt] = vbig[b]
                    dup[i, j] = nxt
                    nxt += 1
                seen[b] = seen.get(b, 0) + 1
    out_dup = torch.empty_like(q3).to(dev)
    maxlen = int(lens3.max())
    ws_bytes = _abi.pkv_decode_workspace_bytes(S, Hq, maxlen, partition_size, D)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev) if ws_bytes else None
    _abi.pkv_decode_attention(out_dup, q3.to(dev), kbig, vbig, torch.from_numpy(dup).to(dev),
                              torch.from_numpy(lens3).to(dev), maxlen, spec.scale,
                              partition_size, ws)
    assert torch.equal(out_dup.cpu(), out3)
    return cache
