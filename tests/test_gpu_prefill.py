"""Paged prefill attention on the GPU against the fp64 oracle ("Paged KV"
wiki page, 实现原理 / 运行阶段), elementwise within |gpu - oracle| <= 2e-3 +
1e-2 |oracle|: whole prompts and later chunks, ragged lengths across row
and key tiles, every built GQA group, f16 and bf16, block sizes 16-64,
plus the prompt write through the pool's slot mapping."""
import zlib

import numpy as np
import pytest
import torch

from oracle import reference as ref
from paged_kv_cache_337_b200 import _abi, build
from paged_kv_cache_337_b200.cache import PagedKVCache
from tests.helpers import DT, paged_problem, tolerance_violation

pytestmark = pytest.mark.gpu

ATOL, RTOL = 2e-3, 1e-2


@pytest.fixture(scope="module", autouse=True)
def _lib(cuda_device):
    build.build()
    _abi.lib()


def run_prefill(p, q, qs, scale, dev, dev_error=None):
    out = torch.full_like(q, float("nan")).to(dev)
    n = np.diff(qs)
    _abi.pkv_prefill_attention(out, q.to(dev), p["kc"].to(dev), p["vc"].to(dev),
                               torch.as_tensor(p["tables"]).to(dev),
                               torch.as_tensor(p["lens"]).to(dev),
                               torch.as_tensor(qs, dtype=torch.int32).to(dev),
                               int(n.max()) if n.size else 0, scale, dev_error=dev_error)
    torch.cuda.synchronize()
    return out.cpu()


def case(seed, Hq, Hkv, bs, lens, chunks, dtype):
    p = paged_problem(seed, Hq, Hkv, 128, bs, lens, dtype)
    g = torch.Generator().manual_seed(seed + 7)
    n = [min(c, L) for c, L in zip(chunks, lens)]
    qs = np.concatenate([[0], np.cumsum(n)]).astype(np.int32)
    q = torch.randn(int(qs[-1]), Hq, 128, generator=g).to(DT[dtype])
    return p, q, qs


WHOLE = ([1, 16, 17, 65, 130, 257], [1, 16, 17, 65, 130, 257])
CHUNKED = ([40, 129, 300, 64, 77, 5], [8, 64, 100, 1, 77, 0])


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
@pytest.mark.parametrize("Hq,Hkv", [(4, 4), (8, 2), (16, 2), (12, 4), (32, 8), (6, 6)])
@pytest.mark.parametrize("bs", [16, 32, 64])
@pytest.mark.parametrize("lens,chunks", [WHOLE, CHUNKED], ids=["whole", "chunked"])
def test_prefill_matches_oracle(dtype, Hq, Hkv, bs, lens, chunks, cuda_device):
    seed = zlib.crc32(repr((dtype, Hq, Hkv, bs, lens)).encode()) % 10000
    p, q, qs = case(seed, Hq, Hkv, bs, lens, chunks, dtype)
    scale = 1.0 / np.sqrt(128)
    err = torch.zeros(2, dtype=torch.int32, device=cuda_device)
    got = run_prefill(p, q, qs, scale, cuda_device, err)
    want = ref.prefill_attention(q, p["kc"], p["vc"], p["tables"], p["lens"], qs, scale, dtype,
                                 Hkv, bs)
    assert err.tolist() == [0, 0]
    assert torch.isfinite(got).all()
    assert tolerance_violation(got, want, ATOL, RTOL) <= 0


def test_prefill_large_scores_stay_finite(cuda_device):
    p, q, qs = case(5, 8, 8, 16, [200], [200], "bf16")
    got = run_prefill(p, q * 8, qs, 1.0, cuda_device)
    want = ref.prefill_attention(q * 8, p["kc"], p["vc"], p["tables"], p["lens"], qs, 1.0,
                                 "bf16", 8, 16)
    assert torch.isfinite(got).all()
    assert tolerance_violation(got, want, ATOL, RTOL) <= 0


def test_prefill_bf16_values_beyond_f16_range(cuda_device):
    """A bf16 cache's P V runs in f16 where its values allow (the V tile
    converted in shared memory); a 16-key group holding a value of
    magnitude 65536 or more keeps bf16 and the two-part P.  Such values sit
    in a few late groups (the middle of tile 3, the last partial tile, a
    group of the second sequence), beside plain groups of the same tiles.
    Rows that cannot see them are held to the usual bound.  The rows that
    do see them get 2^-15 max|V| w_big more, w_big being the weight those
    tokens carry in the row (the oracle's output over an indicator V): the
    two-part P holds a weight to about 2^-17 of itself, and that rounding
    times a 1e5 value can exceed 2e-3 on its own, in any 16-bit P."""
    p, q, qs = case(11, 8, 2, 16, [300, 70], [300, 70], "bf16")
    g = torch.Generator().manual_seed(12)
    vc = p["vc"].float()
    big = ((0, 243), (0, 250), (0, 299), (1, 66))
    for s, tok in big:
        blk = int(p["tables"][s][tok // 16])
        vc[blk, tok % 16] = torch.randn(vc.shape[2:], generator=g) * 1e5
    p["vc"] = vc.to(torch.bfloat16)
    vmax = float(p["vc"].float().abs().max())
    assert vmax > 65536
    scale = 1.0 / np.sqrt(128)
    err = torch.zeros(2, dtype=torch.int32, device=cuda_device)
    got = run_prefill(p, q, qs, scale, cuda_device, err)
    want = ref.prefill_attention(q, p["kc"], p["vc"], p["tables"], p["lens"], qs, scale, "bf16",
                                 2, 16)
    assert err.tolist() == [0, 0]
    assert torch.isfinite(got).all()
    # a row sees a big token when its position is at or past it
    sees = np.zeros(int(qs[-1]), bool)
    for s, tok in big:
        L, n = int(p["lens"][s]), int(qs[s + 1] - qs[s])
        pos = L - n + np.arange(n)
        sees[qs[s]:qs[s + 1]] |= pos >= tok
    assert (~sees).sum() > 300 and sees.sum() > 50
    assert tolerance_violation(got[~sees], want[~sees], ATOL, RTOL) <= 0
    ind = torch.zeros(p["vc"].shape)
    for s, tok in big:
        ind[int(p["tables"][s][tok // 16]), tok % 16] = 1.0
    w_big = ref.prefill_attention(q, p["kc"], ind.to(torch.bfloat16), p["tables"], p["lens"], qs,
                                  scale, "bf16", 2, 16)[..., :1]
    excess = (np.abs(got.double().numpy() - want)
              - (ATOL + vmax * 2.0 ** -15 * w_big + RTOL * np.abs(want)))
    assert excess[sees].max() <= 0


def test_prefill_bf16_all_values_beyond_f16_range(cuda_device):
    """Every V group of a bf16 cache beyond f16's range: the whole P V takes
    the two-part bf16 path.  V scaled by 2^17 scales the exact output by
    2^17 and changes no weight, so got / 2^17 must meet the usual bound
    against the oracle of the unscaled cache."""
    p, q, qs = case(13, 8, 2, 16, [300, 70], [300, 70], "bf16")
    scale = 1.0 / np.sqrt(128)
    want = ref.prefill_attention(q, p["kc"], p["vc"], p["tables"], p["lens"], qs, scale, "bf16",
                                 2, 16)
    big = dict(p)
    big["vc"] = (p["vc"].float() * 2.0 ** 17).to(torch.bfloat16)  # exact: a power of two
    err = torch.zeros(2, dtype=torch.int32, device=cuda_device)
    got = run_prefill(big, q, qs, scale, cuda_device, err)
    assert err.tolist() == [0, 0]
    assert torch.isfinite(got).all()
    assert tolerance_violation(got.double() / 2.0 ** 17, want, ATOL, RTOL) <= 0


def test_prefill_bad_lengths_are_reported(cuda_device):
    p, q, qs = case(6, 4, 4, 16, [10, 20], [10, 20], "f16")
    lens = torch.tensor([10, 5], dtype=torch.int32)  # sequence 1: 20 rows but 5 tokens
    out = torch.zeros(q.shape, dtype=q.dtype, device=cuda_device)
    err = torch.zeros(2, dtype=torch.int32, device=cuda_device)
    _abi.pkv_prefill_attention(out, q.to(cuda_device), p["kc"].to(cuda_device),
                               p["vc"].to(cuda_device), torch.as_tensor(p["tables"]).to(cuda_device),
                               lens.to(cuda_device), torch.as_tensor(qs).to(cuda_device), 20, 0.1,
                               dev_error=err)
    torch.cuda.synchronize()
    assert err.tolist() == [_abi.PKV_DEVERR_CONTEXT_LEN, 1]
    assert not out[10:].any()  # its rows are left unwritten
    want = ref.prefill_attention(q[:10], p["kc"], p["vc"], p["tables"][:1], [10], [0, 10], 0.1,
                                 "f16", 4, 16)
    assert tolerance_violation(out[:10].cpu(), want, ATOL, RTOL) <= 0


def test_prompt_write_then_prefill_through_the_pool(cuda_device):
    """The prefill step as the driver runs it: the pool takes each prompt's
    blocks, pkv_write_slots fills them through the slot mapping, and prefill
    attention reads them back through the Block Tables."""
    dev = cuda_device
    g = torch.Generator().manual_seed(9)
    bs, Hq, Hkv, D = 16, 16, 4, 128
    prompts = [37, 160, 1, 96]
    nb = sum(-(-L // bs) for L in prompts) + 5
    cache = PagedKVCache(nb, bs, Hq, Hkv, D, torch.float16, dev, 16,
                         free_order=torch.randperm(nb, generator=g).tolist())
    qs = np.concatenate([[0], np.cumsum(prompts)]).astype(np.int32)
    T = int(qs[-1])
    q = torch.randn(T, Hq, D, generator=g).to(torch.float16)
    k = torch.randn(T, Hkv, D, generator=g).to(torch.float16)
    v = torch.randn(T, Hkv, D, generator=g).to(torch.float16)
    for s, L in enumerate(prompts):
        cache.add_sequence(s, L, k[qs[s]:qs[s + 1]].to(dev), v[qs[s]:qs[s + 1]].to(dev))
    tables, lens = cache.pool.block_tables(list(range(len(prompts))), 16)
    out = torch.empty(T, Hq, D, dtype=torch.float16, device=dev)
    _abi.pkv_prefill_attention(out, q.to(dev), cache.key_cache, cache.value_cache, tables.to(dev),
                               lens.to(dev), torch.as_tensor(qs).to(dev), max(prompts),
                               cache.scale)
    torch.cuda.synchronize()
    # the oracle reads its own write of the same prompts (into zeroed
    # caches) through the same Block Tables
    kc0 = np.zeros((nb, bs, Hkv, D), np.uint16)
    slots = np.concatenate([cache.pool.slot_mapping(s, 0, L).numpy()
                            for s, L in enumerate(prompts)])
    wk, wv = ref.write_slots(kc0, kc0, k, v, slots, bs, Hkv)
    want = ref.prefill_attention(q, wk, wv, tables, lens, qs, cache.scale, "f16", Hkv, bs)
    assert tolerance_violation(out.cpu(), want, ATOL, RTOL) <= 0
    # and the prompt write itself is bit-exact at every slot it filled
    got_k = ref.bits(cache.key_cache.cpu()).reshape(nb * bs, Hkv, D)[slots]
    got_v = ref.bits(cache.value_cache.cpu()).reshape(nb * bs, Hkv, D)[slots]
    assert np.array_equal(got_k, wk.reshape(nb * bs, Hkv, D)[slots])
    assert np.array_equal(got_v, wv.reshape(nb * bs, Hkv, D)[slots])


def row_tiles(chunks, group):
    """The kernel's work items: 256-row tiles x sequences x KV heads."""
    return -(-max(chunks) * group // 256)


@pytest.mark.parametrize("kind", ["whole", "chunked"])
def test_prefill_many_row_tiles_per_cta(kind, cuda_device):
    """More 256-row tiles than SMs, of uneven weight, with the tiles past
    short sequences' rows skipped: each persistent CTA walks several items,
    so its ring stages, S buffers and barrier phases carry across items."""
    lens = [600, 3, 450, 257, 64, 1, 520, 333, 130, 47, 40, 300]
    chunks = lens if kind == "whole" else [600, 3, 100, 257, 17, 1, 520, 64, 130, 47, 1, 299]
    Hq, Hkv = 32, 8
    items = row_tiles(chunks, Hq // Hkv) * len(lens) * Hkv
    assert items > 2 * torch.cuda.get_device_properties(cuda_device).multi_processor_count
    p, q, qs = case(31 if kind == "whole" else 32, Hq, Hkv, 16, lens, chunks, "bf16")
    scale = 1.0 / np.sqrt(128)
    err = torch.zeros(2, dtype=torch.int32, device=cuda_device)
    got = run_prefill(p, q, qs, scale, cuda_device, err)
    want = ref.prefill_attention(q, p["kc"], p["vc"], p["tables"], p["lens"], qs, scale, "bf16",
                                 Hkv, 16)
    assert err.tolist() == [0, 0]
    assert torch.isfinite(got).all()
    assert tolerance_violation(got, want, ATOL, RTOL) <= 0


def test_prefill_full_size_sampled_rows(cuda_device):
    """The benchmark's launch: 8 prompts of 2048 tokens, 32 query / 8 KV
    heads, block size 16, bf16: 2048 row tiles, about 14 per persistent CTA.
    Checked on sampled rows: row p of a prompt is attention over its tokens
    0 .. p, which the oracle computes as a one-row sequence of context p + 1."""
    S, L, Hq, Hkv, D, bs = 8, 2048, 32, 8, 128, 16
    p = paged_problem(77, Hq, Hkv, D, bs, [L] * S, "bf16")
    g = torch.Generator().manual_seed(78)
    q = torch.randn(S * L, Hq, D, generator=g).to(torch.bfloat16)
    qs = np.arange(0, S * L + 1, L, dtype=np.int32)
    scale = 1.0 / np.sqrt(D)
    err = torch.zeros(2, dtype=torch.int32, device=cuda_device)
    got = run_prefill(p, q, qs, scale, cuda_device, err)
    assert err.tolist() == [0, 0]
    assert torch.isfinite(got).all()
    rng = np.random.default_rng(79)
    edges = [0, 1, 15, 16, 63, 64, 255, 256, 1023, 1024, 2046, 2047]
    seqs, pos = [], []
    for s in range(S):
        for t in edges + list(rng.integers(0, L, 4)):
            seqs.append(s)
            pos.append(int(t))
    rows = np.asarray(seqs) * L + np.asarray(pos)
    want = ref.prefill_attention(q[rows], p["kc"], p["vc"], p["tables"][seqs],
                                 np.asarray(pos, np.int32) + 1,
                                 np.arange(len(rows) + 1, dtype=np.int32), scale, "bf16", Hkv, bs)
    assert tolerance_violation(got[rows], want, ATOL, RTOL) <= 0


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_prefill_repeated_launches_agree_bit_for_bit(dtype, cuda_device):
    """Short items (one to three key tiles), where an item's end follows its
    last P hand-over closely, launched 300 times back to back: no bounded
    wait runs out, and every launch gives the first launch's output bit for
    bit (the work split and every accumulation order are fixed)."""
    lens, chunks = [40, 129, 300, 64, 77, 5, 190, 33], [8, 64, 100, 1, 77, 5, 190, 33]
    p, q, qs = case(91, 8, 2, 16, lens, chunks, dtype)
    dev = cuda_device
    n = np.diff(qs)
    args = (q.to(dev), p["kc"].to(dev), p["vc"].to(dev), torch.as_tensor(p["tables"]).to(dev),
            torch.as_tensor(p["lens"]).to(dev), torch.as_tensor(qs, dtype=torch.int32).to(dev),
            int(n.max()), 1.0 / np.sqrt(128))
    err = torch.zeros(2, dtype=torch.int32, device=dev)
    first = torch.full_like(args[0], float("nan"))
    _abi.pkv_prefill_attention(first, *args, dev_error=err)
    out = torch.empty_like(first)
    mismatches = torch.zeros((), dtype=torch.int64, device=dev)
    for _ in range(300):
        out.fill_(float("nan"))
        _abi.pkv_prefill_attention(out, *args, dev_error=err)
        mismatches += (out.view(torch.int16) != first.view(torch.int16)).sum()
    torch.cuda.synchronize()
    assert err.tolist() == [0, 0]
    assert int(mismatches) == 0
    assert torch.isfinite(first).all()
    want = ref.prefill_attention(q, p["kc"], p["vc"], p["tables"], p["lens"], qs, 1.0 / np.sqrt(128),
                                 dtype, 2, 16)
    assert tolerance_violation(first.cpu(), want, ATOL, RTOL) <= 0
