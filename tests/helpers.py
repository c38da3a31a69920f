"""Test-side builders of paged problems (layouts and seeded values only)."""
import numpy as np
import torch

DT = {"f16": torch.float16, "bf16": torch.bfloat16}


def scatter_to_pages(k_seqs, v_seqs, tables, num_blocks, bs):
    """Place each sequence's contiguous [L, Hkv, D] K/V into a paged cache
    [NB, bs, Hkv, D] following its block table."""
    Hkv, D = k_seqs[0].shape[1:]
    dt = k_seqs[0].dtype
    kc = torch.zeros((num_blocks, bs, Hkv, D), dtype=dt)
    vc = torch.zeros((num_blocks, bs, Hkv, D), dtype=dt)
    for s, (k, v) in enumerate(zip(k_seqs, v_seqs)):
        for t in range(k.shape[0]):
            b = int(tables[s][t // bs])
            kc[b, t % bs] = k[t]
            vc[b, t % bs] = v[t]
    return kc, vc


def random_tables(gen, lens, bs, extra_blocks=3, mb=None):
    """Block tables drawing distinct physical blocks from a seeded
    permutation of a pool with a few spare blocks; -1 past each sequence."""
    need = sum(-(-int(L) // bs) for L in lens)
    nb = need + extra_blocks
    perm = torch.randperm(nb, generator=gen).tolist()
    mb = mb or max(1, max(-(-int(L) // bs) for L in lens))
    tables = np.full((len(lens), mb), -1, dtype=np.int32)
    i = 0
    for s, L in enumerate(lens):
        for j in range(-(-int(L) // bs)):
            tables[s, j] = perm[i]
            i += 1
    return tables, nb


def paged_problem(seed, Hq, Hkv, D, bs, lens, dtype, extra_blocks=3):
    """Random N(0,1) caches, queries and tables for the given lengths."""
    g = torch.Generator().manual_seed(seed)
    dt = DT[dtype]
    tables, nb = random_tables(g, lens, bs, extra_blocks)
    q = torch.randn(len(lens), Hq, D, generator=g).to(dt)
    kc = torch.randn(nb, bs, Hkv, D, generator=g).to(dt)
    vc = torch.randn(nb, bs, Hkv, D, generator=g).to(dt)
    return dict(q=q, kc=kc, vc=vc, tables=tables, lens=np.asarray(lens, np.int32), NB=nb)


def tolerance_violation(gpu, ref, atol=2e-3, rtol=1e-2):
    """Largest excess of |gpu - ref| over atol + rtol * |ref| (<= 0 passes)."""
    g = gpu.double().cpu().numpy() if hasattr(gpu, "double") else np.asarray(gpu, np.float64)
    err = np.abs(g - ref) - (atol + rtol * np.abs(ref))
    return float(err.max()) if err.size else 0.0
