"""Parity of the CUDA path (through the C ABI) with the fp64 CPU oracle.

Slot writes, block copies and allocator state are compared bit for bit over
whole tensors; attention elementwise within |gpu - oracle| <= 2e-3 +
1e-2 |oracle| (16-bit outputs, fp32 accumulation).  Sizes span several
tiles, ragged tails, partition boundaries, every built group size, head_dim,
block size and dtype.
"""
import zlib

import numpy as np
import pytest
import torch

from oracle import reference as ref
from oracle.allocator_model import PoolModel
from paged_kv_cache_337_b200 import _abi, build
from paged_kv_cache_337_b200.cache import PagedKVCache
from paged_kv_cache_337_b200 import workloads as W
from tests.helpers import DT, paged_problem, tolerance_violation

pytestmark = pytest.mark.gpu

ATOL, RTOL = 2e-3, 1e-2


@pytest.fixture(scope="module", autouse=True)
def _lib(cuda_device):
    build.build()
    _abi.lib()


def to_dev(t, dev):
    return torch.as_tensor(t).to(dev)


def gpu_decode(p, Hkv, bs, scale, partition_size, dev, dev_error=None, max_len=None):
    q = p["q"].to(dev)
    kc = p["kc"].to(dev)
    vc = p["vc"].to(dev)
    tables = to_dev(p["tables"], dev)
    lens = to_dev(p["lens"], dev)
    max_len = int(max(p["lens"])) if max_len is None else max_len
    out = torch.full_like(q, float("nan"))
    ws_bytes = _abi.pkv_decode_workspace_bytes(q.shape[0], q.shape[1], max_len,
                                               partition_size, q.shape[2])
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev) if ws_bytes else None
    _abi.pkv_decode_attention(out, q, kc, vc, tables, lens, max_len, scale, partition_size,
                              ws, dev_error=dev_error)
    torch.cuda.synchronize()
    return out.cpu()


def oracle_decode(p, Hkv, bs, scale, dtype):
    return ref.decode_attention(p["q"], p["kc"], p["vc"], p["tables"], p["lens"], scale, dtype,
                                Hkv, bs)


LENS = [1, 2, 15, 16, 17, 63, 64, 65, 129, 200, 257]


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("Hq,Hkv", [(4, 4), (6, 3), (8, 2), (16, 2), (32, 2), (12, 4)])
@pytest.mark.parametrize("bs,P", [(16, 0), (16, 32), (32, 64), (64, 0), (64, 128), (48, 16)])
def test_decode_matches_oracle(dtype, D, Hq, Hkv, bs, P, cuda_device):
    seed = zlib.crc32(repr((dtype, D, Hq, Hkv, bs, P)).encode()) % 10000
    p = paged_problem(seed, Hq, Hkv, D, bs, LENS, dtype)
    scale = 1.0 / np.sqrt(D)
    got = gpu_decode(p, Hkv, bs, scale, P, cuda_device)
    want = oracle_decode(p, Hkv, bs, scale, dtype)
    assert torch.isfinite(got).all()
    assert tolerance_violation(got, want, ATOL, RTOL) <= 0


def test_decode_with_large_scores_stays_finite_and_close(cuda_device):
    """Scores of several hundred (large scale) exercise the running max."""
    p = paged_problem(5, 8, 8, 128, 16, [5, 40, 300, 999], "bf16")
    got = gpu_decode(p, 8, 16, 3.0, 64, cuda_device)
    want = oracle_decode(p, 8, 16, 3.0, "bf16")
    assert tolerance_violation(got, want, ATOL, RTOL) <= 0


def test_empty_context_gives_zeros(cuda_device):
    p = paged_problem(6, 8, 2, 64, 16, [0, 17, 0, 40], "f16")
    got = gpu_decode(p, 2, 16, 0.125, 16, cuda_device)
    assert torch.all(got[0] == 0) and torch.all(got[2] == 0)
    want = oracle_decode(p, 2, 16, 0.125, "f16")
    assert tolerance_violation(got, want, ATOL, RTOL) <= 0


@pytest.mark.parametrize("Hq,Hkv", [(8, 8), (16, 2)])
def test_context_of_one_returns_v_bit_exactly(Hq, Hkv, cuda_device):
    p = paged_problem(7, Hq, Hkv, 128, 16, [1, 1, 1], "bf16")
    got = gpu_decode(p, Hkv, 16, 0.088, 0, cuda_device)
    G = Hq // Hkv
    for s in range(3):
        b = int(p["tables"][s, 0])
        for h in range(Hq):
            assert torch.equal(got[s, h], p["vc"][b, 0, h // G])


@pytest.mark.parametrize("Hq,Hkv,P", [(32, 32, 0), (64, 8, 64)])
def test_physical_permutation_invariance_bit_exact(Hq, Hkv, P, cuda_device):
    bs = 16
    p = paged_problem(8, Hq, Hkv, 128, bs, [33, 100, 250], "bf16", extra_blocks=9)
    base = gpu_decode(p, Hkv, bs, 0.1, P, cuda_device)
    g = torch.Generator().manual_seed(9)
    perm = torch.randperm(p["NB"], generator=g)
    p2 = dict(p)
    p2["kc"] = torch.empty_like(p["kc"])
    p2["vc"] = torch.empty_like(p["vc"])
    p2["kc"][perm] = p["kc"]
    p2["vc"][perm] = p["vc"]
    p2["tables"] = np.where(p["tables"] >= 0, perm.numpy()[np.maximum(p["tables"], 0)],
                            -1).astype(np.int32)
    again = gpu_decode(p2, Hkv, bs, 0.1, P, cuda_device)
    assert torch.equal(base, again)


def test_split_k_agrees_with_single_pass(cuda_device):
    p = paged_problem(10, 32, 8, 128, 32, [3000, 1, 511, 512, 513, 2048], "bf16")
    want = oracle_decode(p, 8, 32, 0.08838834764831845, "bf16")
    outs = {}
    for P in (0, 16, 128, 512, 1024, 4096):
        outs[P] = gpu_decode(p, 8, 32, 0.08838834764831845, P, cuda_device)
        assert tolerance_violation(outs[P], want, ATOL, RTOL) <= 0, P
    for P in outs:
        assert tolerance_violation(outs[P], outs[0].double().numpy(), ATOL, RTOL) <= 0


@pytest.mark.parametrize("Hq,Hkv", [(8, 8), (32, 4)])
def test_split_k_repeated_launches_agree_bit_for_bit(Hq, Hkv, cuda_device):
    """The split-K merge over 200 back-to-back launches on one workspace:
    the partition counters start from zero each time (cleared before the
    launch and reset by the merging CTA), no device error is recorded, and
    every launch gives the first one's output bit for bit (the partials are
    merged in partition order, whichever CTA arrives last)."""
    p = paged_problem(12, Hq, Hkv, 128, 16, [1500, 3, 700, 2048, 64, 1025], "bf16")
    dev = cuda_device
    q, kc, vc = p["q"].to(dev), p["kc"].to(dev), p["vc"].to(dev)
    tables, lens = to_dev(p["tables"], dev), to_dev(p["lens"], dev)
    max_len, P, scale = int(max(p["lens"])), 256, 1.0 / np.sqrt(128)
    ws = torch.empty(_abi.pkv_decode_workspace_bytes(q.shape[0], Hq, max_len, P, 128),
                     dtype=torch.uint8, device=dev)
    err = torch.zeros(2, dtype=torch.int32, device=dev)
    first = torch.full_like(q, float("nan"))
    _abi.pkv_decode_attention(first, q, kc, vc, tables, lens, max_len, scale, P, ws,
                              dev_error=err)
    out = torch.empty_like(first)
    mismatches = torch.zeros((), dtype=torch.int64, device=dev)
    for _ in range(200):
        out.fill_(float("nan"))
        _abi.pkv_decode_attention(out, q, kc, vc, tables, lens, max_len, scale, P, ws,
                                  dev_error=err)
        mismatches += (out.view(torch.int16) != first.view(torch.int16)).sum()
    torch.cuda.synchronize()
    assert err.tolist() == [0, 0]
    assert int(mismatches) == 0
    assert torch.isfinite(first).all()
    want = oracle_decode(p, Hkv, 16, scale, "bf16")
    assert tolerance_violation(first.cpu(), want, ATOL, RTOL) <= 0


def test_combined_kv_layout_via_block_stride(cuda_device):
    """One [NB, 2, bs, Hkv, D] tensor: K and V views with block stride
    2 * bs * Hkv * D."""
    bs, Hkv, Hq, D = 16, 4, 8, 128
    p = paged_problem(11, Hq, Hkv, D, bs, [20, 77], "bf16")
    comb = torch.stack([p["kc"], p["vc"]], dim=1).to(cuda_device)
    kview, vview = comb[:, 0], comb[:, 1]
    q = p["q"].to(cuda_device)
    out = torch.empty_like(q)
    _abi.pkv_decode_attention(out, q, kview, vview, to_dev(p["tables"], cuda_device),
                              to_dev(p["lens"], cuda_device), 77, 0.1, 0, None)
    flat = ref.bits(comb.cpu()).reshape(-1)
    be = bs * Hkv * D
    want = ref.decode_attention(p["q"], flat, flat[be:], p["tables"], p["lens"], 0.1, "bf16",
                                Hkv, bs, block_stride=2 * be)
    assert tolerance_violation(out.cpu(), want, ATOL, RTOL) <= 0
    # slot write through the same views, bit-exact against the oracle
    k = torch.randn(2, Hkv, D).to(torch.bfloat16)
    v = torch.randn(2, Hkv, D).to(torch.bfloat16)
    slots = torch.tensor([5, 3 * bs + 2], dtype=torch.int64)
    _abi.pkv_write_slots(k.to(cuda_device), v.to(cuda_device), kview, vview,
                         slots.to(cuda_device))
    kc2, vc2 = ref.write_slots(flat, flat[be:].copy(), k, v, slots, bs, Hkv,
                               block_stride=2 * be)
    nb = p["NB"]
    got = ref.bits(comb.cpu()).reshape(nb, 2, be)
    want_k = kc2.reshape(nb, 2, be)[:, 0]
    want_v = np.concatenate([vc2, np.zeros(be, np.uint16)]).reshape(nb, 2, be)[:, 0]
    assert np.array_equal(got[:, 0], want_k)
    assert np.array_equal(got[:, 1], want_v)


# ---------------------------------------------------------------------------
# slot write and block copy: bit-exact on whole tensors
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("dtype,Hkv,D,bs", [("bf16", 32, 128, 16), ("f16", 8, 64, 32),
                                            ("bf16", 2, 8, 5)])
def test_write_slots_bit_exact(dtype, Hkv, D, bs, cuda_device):
    g = torch.Generator().manual_seed(12)
    nb, T = 23, 40
    dt = DT[dtype]
    kc = torch.randn(nb, bs, Hkv, D, generator=g).to(dt)
    vc = torch.randn(nb, bs, Hkv, D, generator=g).to(dt)
    k = torch.randn(T, Hkv, D, generator=g).to(dt)
    v = torch.randn(T, Hkv, D, generator=g).to(dt)
    slots = torch.randperm(nb * bs, generator=g)[:T].to(torch.int64)
    slots[::7] = -1  # padding tokens
    dk, dv = kc.to(cuda_device), vc.to(cuda_device)
    err = torch.zeros(2, dtype=torch.int32, device=cuda_device)
    _abi.pkv_write_slots(k.to(cuda_device), v.to(cuda_device), dk, dv, slots.to(cuda_device),
                         dev_error=err)
    wk, wv = ref.write_slots(kc, vc, k, v, slots, bs, Hkv)
    assert np.array_equal(ref.bits(dk.cpu()).reshape(-1), wk.reshape(-1))
    assert np.array_equal(ref.bits(dv.cpu()).reshape(-1), wv.reshape(-1))
    assert err.tolist() == [0, 0]


@pytest.mark.parametrize("dtype,Hkv,D,bs", [("bf16", 32, 128, 16), ("f16", 4, 64, 64),
                                            ("bf16", 1, 8, 3)])
def test_copy_blocks_bit_exact(dtype, Hkv, D, bs, cuda_device):
    g = torch.Generator().manual_seed(13)
    nb = 64
    dt = DT[dtype]
    kc = torch.randn(nb, bs, Hkv, D, generator=g).to(dt)
    vc = torch.randn(nb, bs, Hkv, D, generator=g).to(dt)
    perm = torch.randperm(nb, generator=g)
    pairs = torch.stack([perm[:20], perm[20:40]], dim=1).to(torch.int32)  # disjoint
    dk, dv = kc.to(cuda_device), vc.to(cuda_device)
    _abi.pkv_copy_blocks(dk, dv, pairs.to(cuda_device))
    wk, wv = ref.copy_blocks(kc, vc, pairs, bs, Hkv, D)
    assert np.array_equal(ref.bits(dk.cpu()).reshape(-1), wk.reshape(-1))
    assert np.array_equal(ref.bits(dv.cpu()).reshape(-1), wv.reshape(-1))


# ---------------------------------------------------------------------------
# metadata errors are reported, never trapped
# ---------------------------------------------------------------------------
def test_device_errors_are_reported(cuda_device):
    dev = cuda_device
    p = paged_problem(14, 8, 8, 64, 16, [10, 40], "bf16")
    err = torch.zeros(2, dtype=torch.int32, device=dev)
    bad = dict(p)
    bad["lens"] = np.array([10, 41], np.int32)  # longer than max_context_len below
    gpu_decode(bad, 8, 16, 0.1, 0, dev, dev_error=err, max_len=40)
    assert err.tolist() == [_abi.PKV_DEVERR_CONTEXT_LEN, 1]
    err.zero_()
    bad = dict(p)
    t = p["tables"].copy()
    t[1, 2] = p["NB"] + 100  # outside the pool: reported, read as zeros
    bad["tables"] = t
    gpu_decode(bad, 8, 16, 0.1, 0, dev, dev_error=err)
    assert err.tolist() == [_abi.PKV_DEVERR_BLOCK_ID, 1]
    err.zero_()
    kc = torch.zeros(4, 16, 8, 64, dtype=torch.bfloat16, device=dev)
    vc = torch.zeros_like(kc)
    k = torch.ones(3, 8, 64, dtype=torch.bfloat16, device=dev)
    _abi.pkv_write_slots(k, k, kc, vc, torch.tensor([0, 64, 5], device=dev), dev_error=err)
    torch.cuda.synchronize()
    assert err.tolist() == [_abi.PKV_DEVERR_SLOT, 1]
    assert kc[0, 0].eq(1).all() and kc[0, 5].eq(1).all()
    err.zero_()
    pairs = torch.tensor([[0, 1], [2, 9]], dtype=torch.int32, device=dev)
    _abi.pkv_copy_blocks(kc, vc, pairs, dev_error=err)
    torch.cuda.synchronize()
    assert err.tolist() == [_abi.PKV_DEVERR_PAIR, 1]
    assert torch.equal(kc[1], kc[0])


def test_host_side_argument_errors_raise(cuda_device):
    dev = cuda_device
    p = paged_problem(15, 8, 8, 64, 16, [10, 700], "bf16")
    with pytest.raises(_abi.PkvError) as e:  # split-K without a workspace
        q = p["q"].to(dev)
        _abi.pkv_decode_attention(torch.empty_like(q), q, p["kc"].to(dev), p["vc"].to(dev),
                                  to_dev(p["tables"], dev), to_dev(p["lens"], dev), 700, 0.1,
                                  64, None)
    assert e.value.status == _abi.PKV_ERR_WORKSPACE
    with pytest.raises(ValueError):  # host tensor handed to a kernel
        _abi.pkv_decode_attention(p["q"], p["q"], p["kc"], p["vc"],
                                  torch.as_tensor(p["tables"]), torch.as_tensor(p["lens"]),
                                  700, 0.1)


# ---------------------------------------------------------------------------
# whole decode steps through the allocator
# ---------------------------------------------------------------------------
def decode_step_both_sides(spec, inp, dev, partition_size):
    """Run one decode step of a DecodeSpec workload on the GPU (native pool)
    and on the oracle side (pool model); check allocator parity; return the
    GPU output, the oracle output and both final caches."""
    S, bs = spec.num_seqs, spec.block_size
    lens = inp.context_lens.tolist()
    order = inp.free_order.tolist()
    model = PoolModel(inp.num_blocks, bs, free_order=order)
    cache = PagedKVCache(inp.num_blocks, bs, spec.num_q_heads, spec.num_kv_heads,
                         spec.head_dim, spec.torch_dtype, dev, spec.max_blocks_per_seq,
                         partition_size, free_order=order,
                         key_cache=inp.key_cache.to(dev), value_cache=inp.value_cache.to(dev),
                         scale=spec.scale)
    for s in range(S):
        model.seq_add(s, lens[s] - 1)
        cache.add_sequence(s, lens[s] - 1)
    out = cache.decode_step(list(range(S)), inp.query.to(dev), inp.new_key.to(dev),
                            inp.new_value.to(dev))
    torch.cuda.synchronize()
    cache.check_errors()
    # allocator parity
    slots, pairs = [], []
    for s in range(S):
        st, slot, src, dst = model.seq_append(s)
        assert st == 0
        slots.append(slot)
        if src >= 0:
            pairs.append((src, dst))
    assert pairs == []
    tables = np.full((S, spec.max_blocks_per_seq), -1, np.int32)
    for s in range(S):
        t = model.tables[s]
        tables[s, :len(t)] = t
        assert cache.pool.block_table(s) == t
    kc, vc = ref.write_slots(inp.key_cache, inp.value_cache, inp.new_key, inp.new_value,
                             slots, bs, spec.num_kv_heads)
    return cache, out.cpu(), (kc, vc), tables, np.array(lens, np.int32)


def test_tiny_workload_full_step(cuda_device):
    spec = W.TINY
    inp = W.make_decode_inputs(spec)
    cache, got, (kc, vc), tables, lens = decode_step_both_sides(spec, inp, cuda_device, 0)
    assert np.array_equal(ref.bits(cache.key_cache.cpu()).reshape(-1), kc.reshape(-1))
    assert np.array_equal(ref.bits(cache.value_cache.cpu()).reshape(-1), vc.reshape(-1))
    want = ref.decode_attention(inp.query, kc, vc, tables, lens, spec.scale, spec.dtype,
                                spec.num_kv_heads, spec.block_size)
    assert tolerance_violation(got, want, ATOL, RTOL) <= 0


def test_shared_prefix_small_workload(cuda_device):
    """Parallel sampling with copy-on-write on a small shared-prefix case:
    allocator parity with the model, bit-exact caches after the copies and
    writes, attention within tolerance, and outputs bit-identical to the same
    step with every shared block physically duplicated."""
    from tests.shared_prefix import run_shared_prefix

    run_shared_prefix(W.SHARED_PREFIX_SMALL, cuda_device, partition_size=32, check_all=True)


def test_bounded_wait_expires_and_reports(cuda_device):
    """The failure path of every mbarrier wait: a wait on a barrier nothing
    completes gives up after its limit and reports a timeout; the context
    stays usable afterwards."""
    import time

    err = torch.zeros(2, dtype=torch.int32, device=cuda_device)
    t0 = time.perf_counter()
    _abi.pkv_selftest_bounded_wait(err, 20000)  # 20 ms
    torch.cuda.synchronize()
    assert time.perf_counter() - t0 >= 0.019
    assert err.tolist() == [_abi.PKV_DEVERR_TIMEOUT, 0]
    # the context still runs kernels correctly
    p = paged_problem(40, 8, 2, 64, 16, [33, 70], "bf16")
    got = gpu_decode(p, 2, 16, 0.125, 0, cuda_device)
    want = oracle_decode(p, 2, 16, 0.125, "bf16")
    assert tolerance_violation(got, want, ATOL, RTOL) <= 0


def test_fma_pipe_exp2_within_its_bound(cuda_device):
    """The 2^x the prefill softmax takes from the FMA pipe for part of its
    exponentials, held to the exact power of two: within 3.0e-6 relative on
    [-126, 8] (the softmax's range is (-inf, 8]), exact at integers, +0 at
    and below -127 (masked scores, -inf, NaN), and between 0 and 2^-126 in
    (-127, -126)."""
    rng = np.random.default_rng(5)
    dense = np.linspace(-126.0, 8.0, 1_000_003, dtype=np.float32)
    near = (np.arange(-126, 8)[:, None] + np.float32(1) - rng.random((134, 64)) * 1e-5)
    x = np.concatenate([dense, near.astype(np.float32).ravel(),
                        rng.uniform(-126, 8, 200_000).astype(np.float32)])
    xt = torch.from_numpy(x).to(cuda_device)
    y = torch.empty_like(xt)
    _abi.pkv_selftest_ex2_poly(xt, y)
    got = y.cpu().double().numpy()
    rel = np.abs(got / np.exp2(x.astype(np.float64)) - 1.0)
    assert rel.max() <= 3.0e-6, rel.max()
    ints = np.arange(-126, 9, dtype=np.float32)
    edges = np.array([-127.0, -128.0, -1e30, -np.inf, np.nan], np.float32)
    sub = np.array([-126.999, -126.5, -126.001], np.float32)
    xt = torch.from_numpy(np.concatenate([ints, edges, sub])).to(cuda_device)
    y = torch.full_like(xt, 7.0)
    _abi.pkv_selftest_ex2_poly(xt, y)
    got = y.cpu().double().numpy()
    assert (got[:len(ints)] == np.exp2(ints.astype(np.float64))).all()
    assert (got[len(ints):len(ints) + len(edges)] == 0.0).all()
    tail = got[len(ints) + len(edges):]
    assert ((tail >= 0.0) & (tail <= 2.0 ** -126)).all()
    # an odd count: the last element has no partner
    xt = torch.tensor([1.5, -0.25, 3.0], device=cuda_device)
    y = torch.zeros_like(xt)
    _abi.pkv_selftest_ex2_poly(xt, y)
    assert np.allclose(y.cpu().double().numpy(), np.exp2([1.5, -0.25, 3.0]), rtol=3.0e-6, atol=0)
