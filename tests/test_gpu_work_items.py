"""Decode over the planner's work list (pkv_decode_attention_items and its
e4m3 form), in each of its orders, against the fp64 oracle and against the
full grid.

Each CTA computes the same (sequence, KV head, partition) whatever order
the CTAs run in, and the merging CTA combines the partials in partition
order, so the work-list launch must give the full grid's output bit for
bit, and the oracle's within |gpu - oracle| <= 2e-3 + 1e-2 |oracle|.
"""
import zlib

import numpy as np
import pytest
import torch

from oracle import reference as ref
from paged_kv_cache_337_b200 import _abi, build
from paged_kv_cache_337_b200.cache import PagedKVCache
from tests.helpers import paged_problem, tolerance_violation
from tests.test_gpu_fp8 import fp8_problem, padded_scales

pytestmark = pytest.mark.gpu

ATOL, RTOL = 2e-3, 1e-2
LENS = [0, 1, 15, 16, 17, 64, 65, 129, 200, 257, 1000, 3]


@pytest.fixture(scope="module", autouse=True)
def _lib(cuda_device):
    build.build()
    _abi.lib()


def decode(p, scale, P, dev, items=None, fp8=False, dev_error=None, fill=float("nan")):
    q = p["q"].to(dev)
    kc, vc = p["kc"].to(dev), p["vc"].to(dev)
    tables = torch.as_tensor(p["tables"]).to(dev)
    lens = torch.as_tensor(p["lens"]).to(dev)
    max_len = int(max(p["lens"]))
    out = torch.full_like(q, fill)
    ws_bytes = _abi.pkv_decode_workspace_bytes(q.shape[0], q.shape[1], max_len, P, q.shape[2])
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev) if ws_bytes else None
    wl = torch.as_tensor(items, dtype=torch.int32).to(dev) if items is not None else None
    if fp8:
        ks, vs = padded_scales(p["ks"], dev), padded_scales(p["vs"], dev)
        _abi.pkv_decode_attention_fp8(out, q, kc, vc, ks, vs, tables, lens, max_len, scale, P,
                                      ws, dev_error=dev_error, work_items=wl)
    else:
        _abi.pkv_decode_attention(out, q, kc, vc, tables, lens, max_len, scale, P, ws,
                                  dev_error=dev_error, work_items=wl)
    torch.cuda.synchronize()
    return out.cpu()


def plan(p, Hkv, P, order=_abi.PKV_ITEMS_LONGEST_FIRST):
    return _abi.pkv_decode_work_items(p["lens"], Hkv, int(max(p["lens"])), P, order=order)


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
@pytest.mark.parametrize("D,Hq,Hkv", [(128, 8, 8), (128, 16, 4), (128, 16, 2), (128, 32, 2),
                                      (64, 12, 4), (64, 4, 4)])
@pytest.mark.parametrize("bs,P", [(16, 0), (16, 32), (32, 64), (64, 128), (48, 16)])
def test_work_list_matches_oracle_and_full_grid(dtype, D, Hq, Hkv, bs, P, cuda_device):
    seed = zlib.crc32(repr(("wl", dtype, D, Hq, Hkv, bs, P)).encode()) % 10000
    p = paged_problem(seed, Hq, Hkv, D, bs, LENS, dtype)
    scale = 1.0 / np.sqrt(D)
    order = (_abi.PKV_ITEMS_LONGEST_FIRST, _abi.PKV_ITEMS_SEQUENCES_LONGEST_FIRST,
             _abi.PKV_ITEMS_BATCH_ORDER)[seed % 3]
    got = decode(p, scale, P, cuda_device, items=plan(p, Hkv, P, order))
    full = decode(p, scale, P, cuda_device)
    want = ref.decode_attention(p["q"], p["kc"], p["vc"], p["tables"], p["lens"], scale, dtype,
                                Hkv, bs)
    assert torch.equal(got.view(torch.int16), full.view(torch.int16))
    assert tolerance_violation(got, want, ATOL, RTOL) <= 0


@pytest.mark.parametrize("Hq,Hkv,bs,P", [(8, 8, 16, 0), (16, 2, 16, 32), (32, 2, 64, 128),
                                         (8, 1, 32, 64)])
@pytest.mark.parametrize("order", [_abi.PKV_ITEMS_LONGEST_FIRST,
                                   _abi.PKV_ITEMS_SEQUENCES_LONGEST_FIRST])
def test_work_list_e4m3_matches_oracle_and_full_grid(Hq, Hkv, bs, P, order, cuda_device):
    p = fp8_problem(zlib.crc32(repr((Hq, Hkv, bs, P)).encode()) % 10000, Hq, Hkv, 128, bs,
                    LENS, "bf16")
    got = decode(p, 0.09, P, cuda_device, items=plan(p, Hkv, P, order), fp8=True)
    full = decode(p, 0.09, P, cuda_device, fp8=True)
    want = ref.decode_attention_fp8(p["q"], p["kc"], p["vc"], p["ks"], p["vs"], p["tables"],
                                    p["lens"], 0.09, "bf16", Hkv, bs)
    assert torch.equal(got.view(torch.int16), full.view(torch.int16))
    assert tolerance_violation(got, want, ATOL, RTOL) <= 0


def test_item_outside_the_grid_is_reported_and_skipped(cuda_device):
    p = paged_problem(3, 8, 2, 128, 16, [40, 300, 7], "bf16")
    items = plan(p, 2, 64).tolist()
    grid_size = 3 * 2 * (300 // 64 + 1)
    bad = items[:4] + [grid_size] + items[4:]
    err = torch.zeros(2, dtype=torch.int32, device=cuda_device)
    got = decode(p, 0.1, 64, cuda_device, items=bad, dev_error=err)
    assert err.tolist() == [_abi.PKV_DEVERR_WORK_ITEM, 4]
    want = ref.decode_attention(p["q"], p["kc"], p["vc"], p["tables"], p["lens"], 0.1, "bf16",
                                2, 16)
    assert tolerance_violation(got, want, ATOL, RTOL) <= 0


def test_missing_item_leaves_only_its_sequence_unwritten(cuda_device):
    # sequence 1 (300 tokens) is split into 5 partitions of 64; drop one of
    # its KV head 0 items: that (sequence, KV head) never completes its
    # merge, every other output is written
    p = paged_problem(4, 8, 2, 128, 16, [40, 300, 7], "bf16")
    NP = 300 // 64 + 1
    items = [f for f in plan(p, 2, 64).tolist() if f != (1 * 2 + 0) * NP + 2]
    got = decode(p, 0.1, 64, cuda_device, items=items, fill=-5.0)
    want = ref.decode_attention(p["q"], p["kc"], p["vc"], p["tables"], p["lens"], 0.1, "bf16",
                                2, 16)
    assert (got[1, :4] == -5.0).all()  # query heads 0-3 share KV head 0
    keep = torch.ones(got.shape[:2], dtype=torch.bool)
    keep[1, :4] = False
    assert tolerance_violation(got[keep], want[keep.numpy()], ATOL, RTOL) <= 0


def test_empty_work_list_launches_nothing(cuda_device):
    p = paged_problem(5, 4, 4, 64, 16, [10, 20], "f16")
    got = decode(p, 0.1, 0, cuda_device, items=[], fill=-3.0)
    assert (got == -3.0).all()


@pytest.mark.parametrize("work_list", ["auto", "longest_first", "sequences_longest_first",
                                       "batch_order"])
def test_cache_driver_runs_the_work_list(work_list, cuda_device):
    """PagedKVCache plans the work list on the host for each step; its steps
    give the full grid's output bit for bit, in every order."""
    dev = cuda_device
    g = torch.Generator().manual_seed(9)
    S, Hq, Hkv, D, bs, P = 6, 16, 4, 128, 16, 64
    lens = [1, 70, 300, 15, 129, 0]
    nb = 64
    order = torch.randperm(nb, generator=g).tolist()
    kc = torch.randn(nb, bs, Hkv, D, generator=g).to(torch.bfloat16).to(dev)
    vc = torch.randn(nb, bs, Hkv, D, generator=g).to(torch.bfloat16).to(dev)
    outs = []
    for wl in (work_list, False):
        c = PagedKVCache(nb, bs, Hq, Hkv, D, torch.bfloat16, dev, 32, P, free_order=order,
                         key_cache=kc.clone(), value_cache=vc.clone(), scale=0.1, work_list=wl)
        for s in range(S):
            c.add_sequence(s, lens[s])
        gq = torch.Generator().manual_seed(10)
        step = []
        for _ in range(3):
            q = torch.randn(S, Hq, D, generator=gq).to(torch.bfloat16).to(dev)
            k = torch.randn(S, Hkv, D, generator=gq).to(torch.bfloat16).to(dev)
            v = torch.randn(S, Hkv, D, generator=gq).to(torch.bfloat16).to(dev)
            step.append(c.decode_step(list(range(S)), q, k, v).cpu())
        torch.cuda.synchronize()
        c.check_errors()
        outs.append(step)
    for a, b in zip(*outs):
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))


@pytest.mark.parametrize("fp8,readback", [(False, False), (True, False), (False, True)],
                         ids=["bf16", "e4m3", "bf16_readback_and_upload_streams"])
def test_run_step_in_one_call_matches_the_separate_calls(fp8, readback, cuda_device):
    """PagedKVCache.run_step (pkv_decode_step: upload, copies, write, attention
    and the output's copy to pinned host memory in one native call) gives
    bit for bit the output of upload_step + launch_step on an identical
    cache, through copy-on-write steps, and its host copy equals the
    device output, also when that copy runs on a readback stream (waited
    for through an event recorded there) and the step's inputs and metadata
    go up on an upload stream inside the call."""
    dev = cuda_device
    g = torch.Generator().manual_seed(12)
    S, Hq, Hkv, D, bs, P = 5, 16, 4, 128, 16, 64
    lens = [37, 70, 300, 1, 129]
    nb = 80
    order = torch.randperm(nb, generator=g).tolist()
    kv = torch.uint8 if fp8 else None
    init = (torch.randint(0, 120, (nb, bs, Hkv, D), generator=g, dtype=torch.uint8) if fp8 else
            torch.randn(nb, bs, Hkv, D, generator=g).to(torch.bfloat16))
    caches = []
    for _ in range(2):
        c = PagedKVCache(nb, bs, Hq, Hkv, D, torch.bfloat16, dev, 32, P, free_order=order,
                         key_cache=init.clone().to(dev), value_cache=init.clone().to(dev),
                         scale=0.1, kv_dtype=kv, kv_scale=0.02)
        for s in range(S):
            c.add_sequence(s, lens[s])
        c.fork(0, 5)  # sequence 0's partial last block is shared: a copy-on-write step
        caches.append(c)
    ids = list(range(S + 1))
    host = torch.empty(S + 1, Hq, D, dtype=torch.bfloat16).pin_memory()
    gq = torch.Generator().manual_seed(13)
    for step in range(4):
        q = torch.randn(S + 1, Hq, D, generator=gq).to(torch.bfloat16).to(dev)
        k = torch.randn(S + 1, Hkv, D, generator=gq).to(torch.bfloat16).to(dev)
        v = torch.randn(S + 1, Hkv, D, generator=gq).to(torch.bfloat16).to(dev)
        a, b = caches
        pa, pb = a.prepare_step(ids), b.prepare_step(ids)
        assert pa["num_pairs"] == pb["num_pairs"] == (1 if step == 0 else 0)
        out_a = torch.empty_like(q)
        host.fill_(float("nan"))
        if readback:
            # q, k and v go up from one pinned buffer inside the call
            rs, us = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
            h_in = torch.cat([q.flatten(), k.flatten(), v.flatten()]).cpu().pin_memory()
            d_in = torch.empty_like(h_in, device=dev)
            nq, nk = q.numel(), k.numel()
            dq, dk = d_in[:nq].view(q.shape), d_in[nq:nq + nk].view(k.shape)
            dv = d_in[nq + nk:].view(v.shape)
            a.run_step(pa, dq, dk, dv, out_a, out_host=host, readback_stream=rs,
                       upload_stream=us, inputs=(h_in, d_in))
            done = torch.cuda.Event()
            done.record(rs)
            done.synchronize()
        else:
            a.run_step(pa, q, k, v, out_a, out_host=host)
        b.upload_step(pb)
        out_b = b.launch_step(pb, q, k, v, torch.empty_like(q))
        torch.cuda.synchronize()
        assert torch.equal(out_a.view(torch.int16), out_b.view(torch.int16))
        assert torch.equal(host.view(torch.int16), out_a.cpu().view(torch.int16))
    for c in caches:
        c.check_errors()
    assert torch.equal(caches[0].key_cache, caches[1].key_cache)
    assert torch.equal(caches[0].value_cache, caches[1].value_cache)
