"""Host logic of the multi-GPU path, on CPU with two gloo ranks.

Sequences are independent, so each rank owns its own block pool and batch
and the data path has no collective; the only cross-rank steps are the
barrier around the timed region and the max (time) / sum (bytes) reductions
that turn per-rank measurements into one whole-job number.
"""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    import bench
    from paged_kv_cache_337_b200 import _abi
    from paged_kv_cache_337_b200 import workloads as W

    w, r, _ = bench.dist_setup(backend="gloo")
    try:
        assert (w, r) == (world, rank)
        dev = torch.device("cpu")
        bench.barrier(w)
        t = bench.max_over_ranks(10.0 + rank, w, dev)
        b = bench.sum_over_ranks(100.0 * (rank + 1), w, dev)
        # each rank drives its own pool over its own shard of sequences
        spec = W.TINY
        gen = torch.Generator().manual_seed(spec.seed + rank)
        lens = W.draw_lens(spec, gen).tolist()
        pool = _abi.BlockPool(spec.pool_blocks, spec.block_size)
        for s, L in enumerate(lens):
            pool.add(s, L - 1)
        slots, pairs = pool.append_batch(list(range(len(lens))))
        local_bytes = bench.decode_bytes(spec, lens, 0)
        total = bench.sum_over_ranks(local_bytes, w, dev)
        out[rank] = (t, b, local_bytes, total, slots.tolist(), pairs.shape[0])
    finally:
        torch.distributed.destroy_process_group()


@pytest.mark.timeout(120)
def test_two_gloo_ranks_reduce_time_and_bytes():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world,
                       start_method="spawn", join=True)
    assert sorted(out.keys()) == [0, 1]
    for r in range(world):
        t, b, local, total, slots, npairs = out[r]
        assert t == 11.0  # max over ranks of 10 + rank
        assert b == 300.0  # 100 + 200
        assert npairs == 0
        assert len(slots) == 4 and len(set(slots)) == 4
    assert out[0][3] == out[1][3] == out[0][2] + out[1][2]
