"""Copy-on-write over a multi-layer cache in one launch
(pkv_copy_blocks_layers), bit for bit against the oracle's per-layer copy
("Paged KV" wiki page, 初始化阶段: one physical block id spans every
layer)."""
import numpy as np
import pytest
import torch

from oracle import reference as ref
from paged_kv_cache_337_b200 import _abi, build

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib(cuda_device):
    build.build()
    _abi.lib()


@pytest.mark.parametrize("layers,Hkv,D,bs,dtype", [(4, 8, 128, 16, torch.bfloat16),
                                                   (3, 2, 64, 32, torch.float16),
                                                   (5, 4, 128, 16, torch.uint8)])
def test_copy_blocks_layers_bit_exact(layers, Hkv, D, bs, dtype, cuda_device):
    g = torch.Generator().manual_seed(71)
    nb = 50

    def mk():
        if dtype == torch.uint8:
            return torch.randint(0, 256, (nb, bs, Hkv, D), generator=g, dtype=torch.uint8)
        return torch.randn(nb, bs, Hkv, D, generator=g).to(dtype)

    ks = [mk() for _ in range(layers)]
    vs = [mk() for _ in range(layers)]
    perm = torch.randperm(nb, generator=g)
    pairs = torch.stack([perm[:15], perm[15:30]], dim=1).to(torch.int32)
    dks = [k.to(cuda_device) for k in ks]
    dvs = [v.to(cuda_device) for v in vs]
    err = torch.zeros(2, dtype=torch.int32, device=cuda_device)
    _abi.pkv_copy_blocks_layers(dks, dvs, pairs.to(cuda_device), dev_error=err)
    torch.cuda.synchronize()
    # the oracle copies 16-bit words: an e4m3 block is a block of byte pairs
    as16 = (lambda t: t.numpy().view(np.uint16)) if dtype == torch.uint8 else (lambda t: t)
    want = ref.copy_blocks_layers([as16(k) for k in ks], [as16(v) for v in vs], pairs, bs, Hkv,
                                  D // 2 if dtype == torch.uint8 else D)
    for l in range(layers):
        got_k = dks[l].cpu().contiguous().view(torch.int16).numpy().view(np.uint16) \
            if dtype != torch.uint8 else dks[l].cpu().numpy().view(np.uint16)
        got_v = dvs[l].cpu().contiguous().view(torch.int16).numpy().view(np.uint16) \
            if dtype != torch.uint8 else dvs[l].cpu().numpy().view(np.uint16)
        assert np.array_equal(got_k.reshape(-1), want[l][0].reshape(-1))
        assert np.array_equal(got_v.reshape(-1), want[l][1].reshape(-1))
    assert err.tolist() == [0, 0]


def test_copy_blocks_layers_reports_bad_pairs(cuda_device):
    ks = [torch.zeros(4, 16, 2, 8, dtype=torch.float16, device=cuda_device) for _ in range(2)]
    vs = [torch.zeros_like(k) for k in ks]
    err = torch.zeros(2, dtype=torch.int32, device=cuda_device)
    pairs = torch.tensor([[0, 1], [2, 9]], dtype=torch.int32, device=cuda_device)
    _abi.pkv_copy_blocks_layers(ks, vs, pairs, dev_error=err)
    torch.cuda.synchronize()
    assert err.tolist() == [_abi.PKV_DEVERR_PAIR, 1]
