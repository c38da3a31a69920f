"""Parity of the e4m3 (FP8) cache path with the fp64 oracle ("Paged KV" wiki
page, 局限性: a quantised KV cache with a scale per block).

The quantising slot write and the block copy (bytes and scales) are compared
bit for bit; attention over the dequantised caches elementwise within
|gpu - oracle| <= 2e-3 + 1e-2 |oracle|, the bound of the 16-bit path (the
dequantised values are exact in fp32, so only the accumulation differs).
"""
import zlib

import numpy as np
import pytest
import torch

from oracle import reference as ref
from paged_kv_cache_337_b200 import _abi, build
from tests.helpers import DT, random_tables, tolerance_violation

pytestmark = pytest.mark.gpu

ATOL, RTOL = 2e-3, 1e-2
LENS = [1, 2, 15, 16, 17, 63, 64, 65, 129, 200, 257]


@pytest.fixture(scope="module", autouse=True)
def _lib(cuda_device):
    build.build()
    _abi.lib()


def padded_scales(values, dev):
    """Device copy of a [NB, Hkv] float32 scale table with padded storage."""
    nb, hkv = values.shape
    t = _abi.fp8_scales(nb, hkv, dev)
    t.copy_(torch.as_tensor(values, dtype=torch.float32))
    return t


def fp8_problem(seed, Hq, Hkv, D, bs, lens, dtype):
    """Seeded e4m3 caches for the given lengths.  Each (block, KV head) gets
    the scale max|x| / 448 of N(0, 1) rows drawn for it, times a factor in
    [0.5, 2] (so some rows saturate); the valid slots hold those rows
    quantised by the oracle's write; every other slot keeps random bytes,
    NaN codes included."""
    g = torch.Generator().manual_seed(seed)
    dt = DT[dtype]
    tables, nb = random_tables(g, lens, bs)
    q = torch.randn(len(lens), Hq, D, generator=g).to(dt)
    k = torch.randn(nb * bs, Hkv, D, generator=g).to(dt)
    v = torch.randn(nb * bs, Hkv, D, generator=g).to(dt)

    def scales(x):
        amax = x.float().abs().view(nb, bs, Hkv, D).amax(dim=(1, 3))
        f = 0.5 + 1.5 * torch.rand(nb, Hkv, generator=g)
        return (amax / 448.0 * f).numpy().astype(np.float32)

    ks, vs = scales(k), scales(v)
    kc = torch.randint(0, 256, (nb, bs, Hkv, D), generator=g, dtype=torch.uint8)
    vc = torch.randint(0, 256, (nb, bs, Hkv, D), generator=g, dtype=torch.uint8)
    slots = np.full(nb * bs, -1, np.int64)  # only the slots sequences own
    for s, L in enumerate(lens):
        for t in range(L):
            phys = int(tables[s, t // bs])
            slots[phys * bs + t % bs] = phys * bs + t % bs
    kc, vc = ref.write_slots_fp8(kc, vc, k, v, slots, bs, Hkv, ks, vs, dtype)
    return dict(q=q, kc=torch.from_numpy(kc.reshape(nb, bs, Hkv, D)),
                vc=torch.from_numpy(vc.reshape(nb, bs, Hkv, D)), ks=ks, vs=vs,
                tables=tables, lens=np.asarray(lens, np.int32), NB=nb)


def gpu_decode_fp8(p, scale, partition_size, dev, dev_error=None):
    q = p["q"].to(dev)
    kc, vc = p["kc"].to(dev), p["vc"].to(dev)
    ks, vs = padded_scales(p["ks"], dev), padded_scales(p["vs"], dev)
    tables = torch.as_tensor(p["tables"]).to(dev)
    lens = torch.as_tensor(p["lens"]).to(dev)
    max_len = int(max(p["lens"]))
    out = torch.full_like(q, float("nan"))
    ws_bytes = _abi.pkv_decode_workspace_bytes(q.shape[0], q.shape[1], max_len,
                                               partition_size, q.shape[2])
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev) if ws_bytes else None
    _abi.pkv_decode_attention_fp8(out, q, kc, vc, ks, vs, tables, lens, max_len, scale,
                                  partition_size, ws, dev_error=dev_error)
    torch.cuda.synchronize()
    return out.cpu()


def oracle_decode_fp8(p, Hkv, bs, scale, dtype):
    return ref.decode_attention_fp8(p["q"], p["kc"], p["vc"], p["ks"], p["vs"], p["tables"],
                                    p["lens"], scale, dtype, Hkv, bs)


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
@pytest.mark.parametrize("Hq,Hkv", [(4, 4), (6, 3), (8, 2), (16, 2), (32, 2), (12, 4)])
@pytest.mark.parametrize("bs,P", [(16, 0), (16, 32), (32, 64), (64, 0), (64, 128), (48, 16)])
def test_decode_fp8_matches_oracle(dtype, Hq, Hkv, bs, P, cuda_device):
    seed = zlib.crc32(repr(("fp8", dtype, Hq, Hkv, bs, P)).encode()) % 10000
    p = fp8_problem(seed, Hq, Hkv, 128, bs, LENS, dtype)
    scale = 1.0 / np.sqrt(128)
    err = torch.zeros(2, dtype=torch.int32, device=cuda_device)
    got = gpu_decode_fp8(p, scale, P, cuda_device, dev_error=err)
    want = oracle_decode_fp8(p, Hkv, bs, scale, dtype)
    assert err.tolist() == [0, 0]
    assert torch.isfinite(got).all()
    assert tolerance_violation(got, want, ATOL, RTOL) <= 0


def test_decode_fp8_split_agrees_with_single_pass(cuda_device):
    p = fp8_problem(31, 16, 2, 128, 16, [1000, 37, 513], "bf16")
    scale = 1.0 / np.sqrt(128)
    one = gpu_decode_fp8(p, scale, 0, cuda_device)
    split = gpu_decode_fp8(p, scale, 64, cuda_device)
    want = oracle_decode_fp8(p, 2, 16, scale, "bf16")
    assert tolerance_violation(one, want, ATOL, RTOL) <= 0
    assert tolerance_violation(split, want, ATOL, RTOL) <= 0


def test_decode_fp8_empty_and_single_token(cuda_device):
    # L = 0 gives zeros; L = 1 gives the dequantised V row (weight 1)
    p = fp8_problem(32, 8, 8, 128, 16, [0, 1, 1], "f16")
    got = gpu_decode_fp8(p, 0.1, 0, cuda_device)
    want = oracle_decode_fp8(p, 8, 16, 0.1, "f16")
    assert torch.equal(got[0], torch.zeros_like(got[0]))
    assert tolerance_violation(got, want, ATOL, RTOL) <= 0


@pytest.mark.parametrize("dtype,Hkv,D,bs", [("bf16", 8, 128, 16), ("f16", 2, 64, 32),
                                            ("bf16", 3, 16, 4)])
def test_write_slots_fp8_bit_exact(dtype, Hkv, D, bs, cuda_device):
    g = torch.Generator().manual_seed(41)
    nb, T = 29, 60
    dt = DT[dtype]
    kc = torch.randint(0, 256, (nb, bs, Hkv, D), generator=g, dtype=torch.uint8)
    vc = torch.randint(0, 256, (nb, bs, Hkv, D), generator=g, dtype=torch.uint8)
    # magnitudes over several decades: subnormal codes, ties and saturation
    k = (torch.randn(T, Hkv, D, generator=g) * torch.exp(4 * torch.randn(T, 1, 1, generator=g)))
    v = (torch.randn(T, Hkv, D, generator=g) * torch.exp(4 * torch.randn(T, 1, 1, generator=g)))
    k, v = k.to(dt), v.to(dt)
    ks = torch.exp(2 * torch.randn(nb, Hkv, generator=g)).numpy().astype(np.float32)
    vs = torch.exp(2 * torch.randn(nb, Hkv, generator=g)).numpy().astype(np.float32)
    slots = torch.randperm(nb * bs, generator=g)[:T].to(torch.int64)
    slots[::9] = -1  # padding tokens
    dev = cuda_device
    dk, dv = kc.to(dev), vc.to(dev)
    err = torch.zeros(2, dtype=torch.int32, device=dev)
    _abi.pkv_write_slots_fp8(k.to(dev), v.to(dev), dk, dv, padded_scales(ks, dev),
                             padded_scales(vs, dev), slots.to(dev), dev_error=err)
    wk, wv = ref.write_slots_fp8(kc, vc, k, v, slots, bs, Hkv, ks, vs, dtype)
    assert np.array_equal(dk.cpu().numpy().reshape(-1), wk.reshape(-1))
    assert np.array_equal(dv.cpu().numpy().reshape(-1), wv.reshape(-1))
    assert err.tolist() == [0, 0]


def test_write_slots_fp8_accepts_float8_tensors(cuda_device):
    g = torch.Generator().manual_seed(42)
    nb, bs, Hkv, D, T = 5, 16, 2, 128, 7
    dev = cuda_device
    k = torch.randn(T, Hkv, D, generator=g).to(torch.bfloat16)
    v = torch.randn(T, Hkv, D, generator=g).to(torch.bfloat16)
    ks = np.full((nb, Hkv), 0.02, np.float32)
    slots = torch.arange(T, dtype=torch.int64) * 3
    kc = torch.zeros(nb, bs, Hkv, D, dtype=torch.float8_e4m3fn, device=dev)
    vc = torch.zeros(nb, bs, Hkv, D, dtype=torch.float8_e4m3fn, device=dev)
    _abi.pkv_write_slots_fp8(k.to(dev), v.to(dev), kc, vc, padded_scales(ks, dev),
                             padded_scales(ks, dev), slots.to(dev))
    z = np.zeros((nb, bs, Hkv, D), np.uint8)
    wk, wv = ref.write_slots_fp8(z, z, k, v, slots, bs, Hkv, ks, ks, "bf16")
    assert np.array_equal(kc.view(torch.uint8).cpu().numpy().reshape(-1), wk.reshape(-1))
    assert np.array_equal(vc.view(torch.uint8).cpu().numpy().reshape(-1), wv.reshape(-1))


@pytest.mark.parametrize("Hkv,D,bs", [(8, 128, 16), (4, 64, 64), (1, 16, 3)])
def test_copy_blocks_fp8_bit_exact(Hkv, D, bs, cuda_device):
    g = torch.Generator().manual_seed(43)
    nb = 64
    kc = torch.randint(0, 256, (nb, bs, Hkv, D), generator=g, dtype=torch.uint8)
    vc = torch.randint(0, 256, (nb, bs, Hkv, D), generator=g, dtype=torch.uint8)
    ks = torch.rand(nb, Hkv, generator=g).numpy().astype(np.float32)
    vs = torch.rand(nb, Hkv, generator=g).numpy().astype(np.float32)
    perm = torch.randperm(nb, generator=g)
    pairs = torch.stack([perm[:20], perm[20:40]], dim=1).to(torch.int32)  # disjoint
    dev = cuda_device
    dk, dv = kc.to(dev), vc.to(dev)
    dks, dvs = padded_scales(ks, dev), padded_scales(vs, dev)
    _abi.pkv_copy_blocks_fp8(dk, dv, dks, dvs, pairs.to(dev))
    # the oracle's block copy on 16-bit words: a block of bytes is a block of
    # byte pairs, and a block's scale row is Hkv pairs of 16-bit halves
    wk, wv = ref.copy_blocks(kc.numpy().view(np.uint16), vc.numpy().view(np.uint16), pairs, bs,
                             Hkv, D // 2)
    wks, wvs = ref.copy_blocks(ks.view(np.uint16), vs.view(np.uint16), pairs, 1, Hkv, 2)
    assert np.array_equal(dk.cpu().numpy().view(np.uint16).reshape(-1), wk.reshape(-1))
    assert np.array_equal(dv.cpu().numpy().view(np.uint16).reshape(-1), wv.reshape(-1))
    assert np.array_equal(dks.cpu().numpy().view(np.uint16).reshape(-1), wks.reshape(-1))
    assert np.array_equal(dvs.cpu().numpy().view(np.uint16).reshape(-1), wvs.reshape(-1))


def test_fp8_argument_errors_raise(cuda_device):
    dev = cuda_device
    kc = torch.zeros(4, 16, 2, 128, dtype=torch.uint8, device=dev)
    q = torch.zeros(1, 2, 128, dtype=torch.bfloat16, device=dev)
    tables = torch.zeros(1, 1, dtype=torch.int32, device=dev)
    lens = torch.ones(1, dtype=torch.int32, device=dev)
    good = _abi.fp8_scales(4, 2, dev)
    unpadded = torch.ones(4 * 2 + 1, device=dev)[1:].view(4, 2)  # misaligned start
    with pytest.raises(_abi.PkvError):
        _abi.pkv_decode_attention_fp8(q.clone(), q, kc, kc, unpadded, good, tables, lens, 1,
                                      0.1)
    # head_dim 64 is not built for e4m3 caches
    kc64 = torch.zeros(4, 16, 2, 64, dtype=torch.uint8, device=dev)
    q64 = torch.zeros(1, 2, 64, dtype=torch.bfloat16, device=dev)
    with pytest.raises(_abi.PkvError):
        _abi.pkv_decode_attention_fp8(q64.clone(), q64, kc64, kc64, good, good, tables, lens, 1,
                                      0.1)
    # a 16-bit cache is not an e4m3 cache
    with pytest.raises(ValueError):
        _abi.pkv_decode_attention_fp8(q.clone(), q, kc.to(torch.bfloat16), kc, good, good,
                                      tables, lens, 1, 0.1)


@pytest.mark.parametrize("work_list", [False, True], ids=["grid", "work_list"])
def test_decode_fp8_gqa_shape_at_its_partition_size(work_list, cuda_device):
    """The 70B-shaped GQA layout (64 query / 8 KV heads, block size 16) over
    an e4m3 cache at the partition size that workload uses for e4m3 caches
    (3584 tokens), lengths on and around the partition boundaries, on the
    full grid and on the work list (items longest first)."""
    from paged_kv_cache_337_b200 import workloads as W
    P = W.GQA_70B.partition_for(True)
    assert P == 3584
    lens = [512, 3583, 3584, 3585, 7168, 6000, 1, 7167, 17, 4200, 8192, 7169]
    p = fp8_problem(2024, 64, 8, 128, 16, lens, "bf16")
    scale = 1.0 / np.sqrt(128)
    dev = cuda_device
    q = p["q"].to(dev)
    kc, vc = p["kc"].to(dev), p["vc"].to(dev)
    ks, vs = padded_scales(p["ks"], dev), padded_scales(p["vs"], dev)
    tables = torch.as_tensor(p["tables"]).to(dev)
    tl = torch.as_tensor(p["lens"]).to(dev)
    max_len = int(max(lens))
    out = torch.full_like(q, float("nan"))
    ws = torch.empty(_abi.pkv_decode_workspace_bytes(len(lens), 64, max_len, P, 128),
                     dtype=torch.uint8, device=dev)
    err = torch.zeros(2, dtype=torch.int32, device=dev)
    items = None
    if work_list:
        items = _abi.pkv_decode_work_items(lens, 8, max_len, P).to(dev)
    _abi.pkv_decode_attention_fp8(out, q, kc, vc, ks, vs, tables, tl, max_len, scale, P, ws,
                                  dev_error=err, work_items=items)
    torch.cuda.synchronize()
    want = oracle_decode_fp8(p, 8, 16, scale, "bf16")
    assert err.tolist() == [0, 0]
    assert tolerance_violation(out.cpu(), want, ATOL, RTOL) <= 0
