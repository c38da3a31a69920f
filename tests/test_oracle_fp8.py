"""Pins of the oracle's FP8 (e4m3) cache: decoding of every code against
torch's float8_e4m3fn, quantisation against torch's rounding inside the
range where both round to nearest-even (and saturation at 448 by
definition), the quantising slot write against the division-then-round
definition, and attention over e4m3 caches against library softmax
attention on the dequantised values."""
import numpy as np
import pytest
import scipy.special
import torch

from oracle import reference as ref
from tests.helpers import DT, random_tables


def test_e4m3_decode_every_code_matches_torch():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    want = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = np.array([ref.e4m3_to_f64(c) for c in range(256)])
    nan = np.isnan(want)
    assert np.array_equal(np.isnan(got), nan) and nan.sum() == 2  # S.1111.111
    assert np.array_equal(got[~nan], want[~nan])
    assert got[0x7e] == 448.0 and got[1] == 2.0 ** -9


def test_e4m3_quantisation_matches_torch_in_range():
    g = torch.Generator().manual_seed(3)
    vals = [torch.randn(4000, generator=g) * s for s in (0.001, 0.05, 1.0, 30.0, 150.0)]
    # every midpoint between neighbouring codes: the ties
    finite = np.array([ref.e4m3_to_f64(c) for c in range(0x7f)])
    mids = (finite[:-1] + finite[1:]) / 2
    vals.append(torch.tensor(np.concatenate([mids, -mids, finite, -finite]), dtype=torch.float32))
    x = torch.cat(vals).float()
    x = x[x.abs() < 464.0]  # torch turns |x| >= 480 into NaN; below 464 both round alike
    want = x.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([ref.f32_to_e4m3(v) for v in x.tolist()], dtype=np.uint8)
    assert np.array_equal(got, want)


def test_e4m3_quantisation_saturates_at_448():
    for v in (464.0, 480.0, 1e6, float("inf")):
        assert ref.f32_to_e4m3(v) == 0x7e
        assert ref.f32_to_e4m3(-v) == 0xfe
    assert ref.f32_to_e4m3(float("nan")) == 0x7f
    assert ref.f32_to_e4m3(2.0 ** -10) == 0x00  # half the smallest subnormal: ties to 0
    assert ref.f32_to_e4m3(3 * 2.0 ** -10) == 0x02  # 1.5 x smallest: ties to the even code


def fp8_problem(seed, Hq, Hkv, D, bs, lens, dtype="bf16"):
    g = torch.Generator().manual_seed(seed)
    tables, nb = random_tables(g, lens, bs, extra_blocks=2)
    q = torch.randn(len(lens), Hq, D, generator=g).to(DT[dtype])
    kc = torch.randint(0, 256, (nb, bs, Hkv, D), generator=g, dtype=torch.int32).to(torch.uint8)
    vc = torch.randint(0, 256, (nb, bs, Hkv, D), generator=g, dtype=torch.int32).to(torch.uint8)
    for c in (kc, vc):  # no NaN codes in a cache
        c[(c & 0x7f) == 0x7f] = 0x7e
    ks = (torch.rand(nb, Hkv, generator=g) * 0.02 + 0.005).float()
    vs = (torch.rand(nb, Hkv, generator=g) * 0.02 + 0.005).float()
    return dict(q=q, kc=kc, vc=vc, ks=ks, vs=vs, tables=tables,
                lens=np.asarray(lens, np.int32), NB=nb)


def test_write_slots_fp8_is_division_then_rounding():
    bs, Hkv, D = 16, 2, 8
    p = fp8_problem(5, 2, Hkv, D, bs, [40, 9])
    g = torch.Generator().manual_seed(6)
    k = torch.randn(5, Hkv, D, generator=g).to(torch.bfloat16)
    v = (torch.randn(5, Hkv, D, generator=g) * 3).to(torch.bfloat16)
    slots = torch.tensor([3, -1, 17, 16 * 2 + 5, 40], dtype=torch.int64)
    kc, vc = ref.write_slots_fp8(p["kc"], p["vc"], k, v, slots, bs, Hkv, p["ks"], p["vs"],
                                 "bf16")
    kc = kc.reshape(p["NB"], bs, Hkv, D)
    vc = vc.reshape(p["NB"], bs, Hkv, D)
    touched = set()
    for t, st in enumerate(slots.tolist()):
        if st < 0:
            continue
        b, o = divmod(st, bs)
        touched.add((b, o))
        for h in range(Hkv):
            kq = (k[t, h].float() / p["ks"][b, h]).to(torch.float8_e4m3fn).view(torch.uint8)
            vq = (v[t, h].float() / p["vs"][b, h]).to(torch.float8_e4m3fn).view(torch.uint8)
            assert np.array_equal(kc[b, o, h], kq.numpy())
            assert np.array_equal(vc[b, o, h], vq.numpy())
    for b in range(p["NB"]):
        for o in range(bs):
            if (b, o) not in touched:
                assert np.array_equal(kc[b, o], p["kc"][b, o].numpy())


@pytest.mark.parametrize("Hq,Hkv", [(4, 4), (8, 2)])
def test_fp8_attention_matches_library_on_dequantised_values(Hq, Hkv):
    bs, D = 16, 16
    lens = [1, 15, 17, 40]
    p = fp8_problem(7 + Hq, Hq, Hkv, D, bs, lens)
    scale = 0.3
    out = ref.decode_attention_fp8(p["q"], p["kc"], p["vc"], p["ks"], p["vs"], p["tables"],
                                   p["lens"], scale, "bf16", Hkv, bs)
    kd = p["kc"].view(torch.float8_e4m3fn).to(torch.float64) * p["ks"].double()[:, None, :, None]
    vd = p["vc"].view(torch.float8_e4m3fn).to(torch.float64) * p["vs"].double()[:, None, :, None]
    G = Hq // Hkv
    for s, L in enumerate(lens):
        blocks = [int(b) for b in p["tables"][s][: -(-L // bs)]]
        k = torch.cat([kd[b] for b in blocks])[:L].numpy()
        v = torch.cat([vd[b] for b in blocks])[:L].numpy()
        for h in range(Hq):
            w = scipy.special.softmax(scale * (k[:, h // G] @ p["q"][s, h].double().numpy()))
            np.testing.assert_allclose(out[s, h], w @ v[:, h // G], rtol=1e-12, atol=1e-14)


def test_fp8_context_of_one_returns_the_dequantised_v():
    p = fp8_problem(9, 4, 4, 32, 16, [1, 1])
    out = ref.decode_attention_fp8(p["q"], p["kc"], p["vc"], p["ks"], p["vs"], p["tables"],
                                   p["lens"], 0.1, "bf16", 4, 16)
    for s in range(2):
        b = int(p["tables"][s, 0])
        want = p["vc"][b, 0].view(torch.float8_e4m3fn).double() * p["vs"][b].double()[:, None]
        assert np.array_equal(out[s], want.numpy())
