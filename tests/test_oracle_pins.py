"""Pins of the CPU oracle against things other than itself.

Each test ties one part of the oracle to what the pages or the mathematics
fix: exhaustive checks of the 16-bit widening against numpy/torch, library
softmax attention on contiguous K/V (the special case an identity block
table reduces to), closed forms, invariants the pages state (logical order
only; physical placement is free), brute force over block placements, and
hand-worked golden fixtures.  A plausible slip in the oracle (wrong GQA head,
wrong offset inside a block, a missing scale, a max of the wrong sign, a
transposed operand) fails at least one of them.
"""
import itertools
import math

import numpy as np
import pytest
import scipy.special
import torch

from oracle import reference as ref
from tests.conftest import golden_lines
from tests.helpers import DT, scatter_to_pages


def library_attention(q, k, v, scale):
    """softmax(scale * K q) V for one head, fp64, via numpy + scipy."""
    q64 = q.to(torch.float64).numpy()
    k64 = k.to(torch.float64).numpy()
    v64 = v.to(torch.float64).numpy()
    w = scipy.special.softmax(scale * (k64 @ q64))
    return w @ v64


def random_problem(seed, S, Hq, Hkv, D, bs, lens, dtype="bf16", extra_blocks=3):
    g = torch.Generator().manual_seed(seed)
    dt = DT[dtype]
    MB = max(1, max(-(-L // bs) for L in lens))
    need = sum(-(-L // bs) for L in lens)
    NB = need + extra_blocks
    perm = torch.randperm(NB, generator=g).tolist()
    tables = np.full((S, MB), -1, dtype=np.int32)
    i = 0
    for s, L in enumerate(lens):
        for j in range(-(-L // bs)):
            tables[s, j] = perm[i]
            i += 1
    k_seqs = [torch.randn(L, Hkv, D, generator=g).to(dt) for L in lens]
    v_seqs = [torch.randn(L, Hkv, D, generator=g).to(dt) for L in lens]
    q = torch.randn(S, Hq, D, generator=g).to(dt)
    kc, vc = scatter_to_pages(k_seqs, v_seqs, tables, NB, bs)
    return dict(q=q, kc=kc, vc=vc, tables=tables, lens=np.array(lens, np.int32),
                k_seqs=k_seqs, v_seqs=v_seqs, NB=NB, MB=MB)


def run_oracle(p, scale, dtype, Hkv, bs, **kw):
    return ref.decode_attention(p["q"], p["kc"], p["vc"], p["tables"], p["lens"],
                                scale, dtype, Hkv, bs, **kw)


# ---------------------------------------------------------------------------
# exact widening of 16-bit storage
# ---------------------------------------------------------------------------
def test_widen_bf16_exhaustive_matches_torch():
    pats = np.arange(65536, dtype=np.uint16)
    want = torch.from_numpy(pats.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    got = np.array([ref.bf16_to_f64(b) for b in pats])
    nan = np.isnan(want)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], want[~nan])


def test_widen_f16_exhaustive_matches_numpy():
    pats = np.arange(65536, dtype=np.uint16)
    want = pats.view(np.float16).astype(np.float64)
    got = np.array([ref.f16_to_f64(b) for b in pats])
    nan = np.isnan(want)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], want[~nan])
    # signed zeros keep their sign
    assert math.copysign(1.0, ref.f16_to_f64(0x8000)) == -1.0


# ---------------------------------------------------------------------------
# attention: reduction to library softmax attention on contiguous K/V
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("dtype", ["f16", "bf16"])
@pytest.mark.parametrize("Hq,Hkv", [(4, 4), (8, 2), (8, 1)])
def test_attention_matches_library_softmax(dtype, Hq, Hkv):
    bs, D = 4, 16
    lens = [1, 3, 4, 5, 11, 17]
    p = random_problem(7 + Hq + Hkv, len(lens), Hq, Hkv, D, bs, lens, dtype)
    scale = 0.37
    out = run_oracle(p, scale, dtype, Hkv, bs)
    G = Hq // Hkv
    for s, L in enumerate(lens):
        for h in range(Hq):
            want = library_attention(p["q"][s, h], p["k_seqs"][s][:, h // G],
                                     p["v_seqs"][s][:, h // G], scale)
            np.testing.assert_allclose(out[s, h], want, rtol=1e-12, atol=1e-13)


def test_attention_combined_kv_layout_with_block_stride():
    """K and V interleaved per block ([NB, 2, bs, Hkv, D]); blocks are
    2*bs*Hkv*D elements apart."""
    bs, Hkv, Hq, D = 4, 2, 4, 8
    lens = [6, 9]
    p = random_problem(3, 2, Hq, Hkv, D, bs, lens, "bf16")
    NB = p["NB"]
    comb = torch.zeros((NB, 2, bs, Hkv, D), dtype=torch.bfloat16)
    comb[:, 0] = p["kc"]
    comb[:, 1] = p["vc"]
    flat = ref.bits(comb).reshape(-1)
    be = bs * Hkv * D
    out = ref.decode_attention(p["q"], flat, flat[be:], p["tables"], p["lens"], 0.5,
                               "bf16", Hkv, bs, block_stride=2 * be)
    want = run_oracle(p, 0.5, "bf16", Hkv, bs)
    assert np.array_equal(out, want)


# ---------------------------------------------------------------------------
# closed forms
# ---------------------------------------------------------------------------
def test_context_of_one_returns_v_exactly():
    p = random_problem(11, 3, 4, 2, 32, 16, [1, 1, 1], "bf16")
    out = run_oracle(p, 0.125, "bf16", 2, 16)
    for s in range(3):
        for h in range(4):
            assert np.array_equal(out[s, h], p["v_seqs"][s][0, h // 2].double().numpy())


def test_zero_scale_gives_mean_of_v():
    p = random_problem(12, 2, 2, 2, 16, 4, [7, 13], "f16")
    out = run_oracle(p, 0.0, "f16", 2, 4)
    for s, L in enumerate([7, 13]):
        for h in range(2):
            want = p["v_seqs"][s][:, h].double().numpy().mean(axis=0)
            np.testing.assert_allclose(out[s, h], want, rtol=1e-13, atol=1e-15)


def test_identical_keys_give_mean_of_v():
    p = random_problem(13, 1, 2, 1, 8, 4, [10], "bf16")
    k = p["k_seqs"][0]
    k[:] = k[0:1]  # every key equal
    p["kc"], p["vc"] = scatter_to_pages(p["k_seqs"], p["v_seqs"], p["tables"], p["NB"], 4)
    out = run_oracle(p, 0.9, "bf16", 1, 4)
    want = p["v_seqs"][0][:, 0].double().numpy().mean(axis=0)
    for h in range(2):
        np.testing.assert_allclose(out[0, h], want, rtol=1e-13, atol=1e-15)


def test_constant_v_gives_the_constant():
    p = random_problem(14, 2, 4, 4, 8, 4, [5, 9], "bf16")
    for s in range(2):
        p["v_seqs"][s][:] = 1.5
    p["kc"], p["vc"] = scatter_to_pages(p["k_seqs"], p["v_seqs"], p["tables"], p["NB"], 4)
    out = run_oracle(p, 0.3, "bf16", 4, 4)
    np.testing.assert_allclose(out, 1.5, rtol=1e-14)


def test_two_tokens_sigmoid_form():
    """softmax over two scores a, b: v0 + (v1 - v0) * sigmoid(b - a)."""
    p = random_problem(15, 1, 1, 1, 16, 4, [2], "bf16")
    q = p["q"][0, 0].double().numpy()
    k = p["k_seqs"][0][:, 0].double().numpy()
    v = p["v_seqs"][0][:, 0].double().numpy()
    scale = 0.25
    a, b = scale * np.dot(k[0], q), scale * np.dot(k[1], q)
    want = v[0] + (v[1] - v[0]) * scipy.special.expit(b - a)
    out = run_oracle(p, scale, "bf16", 1, 4)
    np.testing.assert_allclose(out[0, 0], want, rtol=1e-12, atol=1e-14)


def test_one_hot_limit_picks_the_dominant_key():
    """With one key aligned with q and a huge scale, every other weight
    underflows to exactly zero, so the output is that token's V."""
    bs, D, L = 4, 8, 9
    p = random_problem(16, 1, 1, 1, D, bs, [L], "bf16")
    k = p["k_seqs"][0]
    k[:] = 0
    k[:, 0, 0] = -1.0
    k[5, 0, 0] = 1.0
    p["q"][:] = 0
    p["q"][0, 0, 0] = 1.0
    p["kc"], p["vc"] = scatter_to_pages(p["k_seqs"], p["v_seqs"], p["tables"], p["NB"], bs)
    out = run_oracle(p, 1000.0, "bf16", 1, bs)
    assert np.array_equal(out[0, 0], p["v_seqs"][0][5, 0].double().numpy())


def test_empty_context_gives_zeros():
    p = random_problem(17, 2, 2, 2, 8, 4, [0, 5], "bf16")
    out = run_oracle(p, 0.5, "bf16", 2, 4)
    assert np.all(out[0] == 0.0)
    assert np.any(out[1] != 0.0)


# ---------------------------------------------------------------------------
# indirection: logical order only, physical placement free
# ---------------------------------------------------------------------------
def test_gqa_head_mapping_contiguous_groups():
    """KV head j holds V = j everywhere, so query head h must output h // G."""
    Hq, Hkv, D, bs = 8, 2, 4, 4
    p = random_problem(18, 1, Hq, Hkv, D, bs, [6], "f16")
    for j in range(Hkv):
        p["v_seqs"][0][:, j] = float(j)
    p["kc"], p["vc"] = scatter_to_pages(p["k_seqs"], p["v_seqs"], p["tables"], p["NB"], bs)
    out = run_oracle(p, 0.5, "f16", Hkv, bs)
    for h in range(Hq):
        assert np.all(out[0, h] == float(h // (Hq // Hkv)))


def test_block_table_addressing_golden():
    """Each logical token reads the physical slot the hand-worked table says."""
    rows = golden_lines("block_table_example.txt")
    bs = int(rows[0][1])
    table = [int(x) for x in rows[1][1:]]
    cases = [tuple(int(x) for x in r) for r in rows[2:]]
    NB, D = max(table) + 1, 2
    kc = torch.zeros((NB, bs, 1, D), dtype=torch.float16)
    vc = torch.zeros((NB, bs, 1, D), dtype=torch.float16)
    for b in range(NB):
        for o in range(bs):
            vc[b, o, 0, 0] = float(b)
            vc[b, o, 0, 1] = float(o)
            kc[b, o, 0, 0] = -1.0
    L = len(table) * bs
    tables = np.array([table], dtype=np.int32)
    for t, b, o, slot in cases:
        assert slot == b * bs + o
        k2 = kc.clone()
        k2[b, o, 0, 0] = 1.0  # the only key aligned with q
        q = torch.tensor([[[1.0, 0.0]]], dtype=torch.float16)
        out = ref.decode_attention(q, k2, vc, tables, np.array([L], np.int32), 1000.0,
                                   "f16", 1, bs)
        assert out[0, 0, 0] == b and out[0, 0, 1] == o
        # the token sits at logical position t: with the context cut just
        # before t the aligned key is out of reach and the output changes
        if t > 0:
            short = ref.decode_attention(q, k2, vc, tables, np.array([t], np.int32),
                                         1000.0, "f16", 1, bs)
            assert not (short[0, 0, 0] == b and short[0, 0, 1] == o)


def test_physical_permutation_invariance_bit_exact():
    bs, Hq, Hkv, D = 4, 4, 2, 16
    lens = [3, 8, 13, 16, 21]
    p = random_problem(19, len(lens), Hq, Hkv, D, bs, lens, "bf16", extra_blocks=5)
    base = run_oracle(p, 0.3, "bf16", Hkv, bs)
    g = torch.Generator().manual_seed(5)
    for _ in range(4):
        perm = torch.randperm(p["NB"], generator=g)  # new physical id of block b
        kc2 = torch.empty_like(p["kc"])
        vc2 = torch.empty_like(p["vc"])
        kc2[perm] = p["kc"]
        vc2[perm] = p["vc"]
        t2 = np.where(p["tables"] >= 0, perm.numpy()[np.maximum(p["tables"], 0)], -1)
        out = ref.decode_attention(p["q"], kc2, vc2, t2.astype(np.int32), p["lens"], 0.3,
                                   "bf16", Hkv, bs)
        assert np.array_equal(out, base)


def test_brute_force_every_placement_in_a_tiny_pool():
    """A 3-block sequence in a 4-block pool: all 24 placements agree bit for
    bit, and agree with contiguous library attention."""
    bs, D, L = 2, 4, 5
    g = torch.Generator().manual_seed(20)
    k = torch.randn(L, 1, D, generator=g).to(torch.bfloat16)
    v = torch.randn(L, 1, D, generator=g).to(torch.bfloat16)
    q = torch.randn(1, 1, D, generator=g).to(torch.bfloat16)
    want = library_attention(q[0, 0], k[:, 0], v[:, 0], 0.7)
    outs = []
    for place in itertools.permutations(range(4), 3):
        tables = np.array([place], dtype=np.int32)
        kc, vc = scatter_to_pages([k], [v], tables, 4, bs)
        outs.append(ref.decode_attention(q, kc, vc, tables, np.array([L], np.int32), 0.7,
                                         "bf16", 1, bs))
    assert len(outs) == 24
    for o in outs:
        assert np.array_equal(o, outs[0])
    np.testing.assert_allclose(outs[0][0, 0], want, rtol=1e-12, atol=1e-14)


def test_memory_outside_the_context_is_never_read():
    bs, Hkv, D = 4, 2, 8
    lens = [6, 9]
    p = random_problem(21, 2, 2, Hkv, D, bs, lens, "bf16", extra_blocks=4)
    base = run_oracle(p, 0.4, "bf16", Hkv, bs)
    used = {int(b) for b in p["tables"].reshape(-1) if b >= 0}
    kc, vc = p["kc"].clone(), p["vc"].clone()
    for b in range(p["NB"]):
        if b not in used:
            kc[b] = 99.0
            vc[b] = -99.0
    # tail slots of each sequence's last block
    for s, L in enumerate(lens):
        last = int(p["tables"][s][(L - 1) // bs])
        kc[last, L % bs or bs:] = 77.0
        vc[last, L % bs or bs:] = 77.0
    tables = p["tables"].copy()
    tables[tables < 0] = 12345  # entries past ceil(L/bs) must not be followed
    out = ref.decode_attention(p["q"], kc, vc, tables, p["lens"], 0.4, "bf16", Hkv, bs)
    assert np.array_equal(out, base)


def test_oracle_rejects_bad_metadata():
    p = random_problem(22, 1, 1, 1, 4, 4, [5], "bf16")
    bad = p["tables"].copy()
    bad[0, 1] = p["NB"]  # physical id out of range
    with pytest.raises(ref.OracleError):
        ref.decode_attention(p["q"], p["kc"], p["vc"], bad, p["lens"], 1.0, "bf16", 1, 4)
    with pytest.raises(ref.OracleError):  # context longer than the table
        ref.decode_attention(p["q"], p["kc"], p["vc"], p["tables"], np.array([9], np.int32),
                             1.0, "bf16", 1, 4)


# ---------------------------------------------------------------------------
# split-K partials and merge: the algebraic identity
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("P", [1, 3, 4, 7, 16, 40])
def test_merge_of_partials_equals_plain_attention(P):
    bs, Hq, Hkv, D = 4, 4, 2, 8
    lens = [1, 6, 17, 33, 40]
    p = random_problem(23, len(lens), Hq, Hkv, D, bs, lens, "bf16")
    NP = -(-max(lens) // P)
    m, l, o = ref.decode_partials(p["q"], p["kc"], p["vc"], p["tables"], p["lens"], 0.3,
                                  "bf16", Hkv, bs, P, NP)
    merged = ref.merge_partials(m, l, o, p["lens"], P)
    plain = run_oracle(p, 0.3, "bf16", Hkv, bs)
    np.testing.assert_allclose(merged, plain, rtol=1e-12, atol=1e-14)
    # partitions past the end of a sequence are empty: m=-inf, l=0, o=0
    for s, L in enumerate(lens):
        for pp in range(-(-L // P), NP):
            assert np.all(np.isneginf(m[s, :, pp])) and np.all(l[s, :, pp] == 0)


def test_single_partition_merge_is_plain_normalisation():
    bs, D = 4, 8
    lens = [7, 12]
    p = random_problem(24, 2, 2, 2, D, bs, lens, "f16")
    m, l, o = ref.decode_partials(p["q"], p["kc"], p["vc"], p["tables"], p["lens"], 0.5,
                                  "f16", 2, bs, 64, 1)
    merged = ref.merge_partials(m, l, o, p["lens"], 64)
    assert np.array_equal(merged, o[:, :, 0, :] / l[:, :, 0, None])


# ---------------------------------------------------------------------------
# slot write and block copy: hand-worked fixtures
# ---------------------------------------------------------------------------
def _hex(x):
    return int(x, 16)


def test_write_slots_golden():
    rows = golden_lines("write_slots_tiny.txt")
    kv = {r[0]: int(r[1]) for r in rows if len(r) == 2}
    NB, bs, Hkv, D = kv["num_blocks"], kv["block_size"], kv["num_kv_heads"], kv["head_dim"]
    toks = [r for r in rows if r[0] == "token"]
    slots = np.array([int(r[2]) for r in toks], np.int64)
    key = np.array([[_hex(r[3]), _hex(r[4])] for r in toks], np.uint16).reshape(-1, Hkv, D)
    val = np.array([[_hex(r[5]), _hex(r[6])] for r in toks], np.uint16).reshape(-1, Hkv, D)
    kc = np.full((NB, bs, Hkv, D), 0xAAAA, np.uint16)
    vc = kc.copy()
    k2, v2 = ref.write_slots(kc, vc, key, val, slots, bs, Hkv)
    k2 = k2.reshape(NB, -1)
    v2 = v2.reshape(NB, -1)
    for r in rows:
        if r[0] in ("key_block", "value_block"):
            arr = k2 if r[0] == "key_block" else v2
            assert list(arr[int(r[1])]) == [_hex(x) for x in r[2:]], r


def test_write_slots_rejects_duplicates_and_out_of_range():
    kc = np.zeros((2, 4, 1, 2), np.uint16)
    key = np.ones((2, 1, 2), np.uint16)
    with pytest.raises(ref.OracleError):
        ref.write_slots(kc, kc, key, key, [3, 3], 4, 1)
    with pytest.raises(ref.OracleError):
        ref.write_slots(kc, kc, key, key, [0, 8], 4, 1)


def test_copy_blocks_golden():
    rows = golden_lines("copy_blocks_tiny.txt")
    kv = {r[0]: int(r[1]) for r in rows if len(r) == 2}
    NB, bs = kv["num_blocks"], kv["block_size"]
    pairs = [(int(r[1]), int(r[2])) for r in rows if r[0] == "pair"]
    kc = np.array([0x1000 + 16 * b + o for b in range(NB) for o in range(bs)], np.uint16)
    vc = np.array([0x2000 + 16 * b + o for b in range(NB) for o in range(bs)], np.uint16)
    k2, v2 = ref.copy_blocks(kc, vc, pairs, bs, 1, 1)
    want = {r[0]: [_hex(x) for x in r[1:]] for r in rows if r[0] in ("key", "value")}
    assert list(k2) == want["key"]
    assert list(v2) == want["value"]


def test_block_bytes_golden():
    for r in golden_lines("block_bytes.txt"):
        bs, hkv, d, layers, dtb, want = map(int, r)
        assert ref.block_bytes(bs, hkv, d, layers, dtb) == want


# ---------------------------------------------------------------------------
# block swap copy ("PagedAttention 动态内存分页" page, 动态块分配与回收)
# ---------------------------------------------------------------------------
def test_swap_blocks_matches_fancy_indexing_and_round_trips():
    rng = np.random.default_rng(5)
    gpu = rng.integers(0, 2**16, size=(12, 4, 2, 8), dtype=np.uint16)
    host = rng.integers(0, 2**16, size=(9, 4, 2, 8), dtype=np.uint16)
    src = rng.permutation(12)[:6]
    dst = rng.permutation(9)[:6]
    pairs = np.stack([src, dst], axis=1).astype(np.int32)
    out = ref.swap_blocks(host, gpu, pairs).view(np.uint16).reshape(host.shape)
    want = host.copy()
    want[dst] = gpu[src]  # the library's gather/scatter
    assert np.array_equal(out, want)
    # and back: the inverse pairs restore the original blocks elsewhere
    fresh = np.zeros_like(gpu)
    back = ref.swap_blocks(fresh, out, pairs[:, ::-1]).view(np.uint16).reshape(gpu.shape)
    assert np.array_equal(back[src], gpu[src])
    assert not back[np.setdiff1d(np.arange(12), src)].any()


def test_swap_blocks_rejects_pairs_outside_either_pool():
    gpu = np.zeros((4, 16), np.uint8)
    host = np.zeros((2, 16), np.uint8)
    with pytest.raises(Exception):
        ref.swap_blocks(host, gpu, [[3, 2]])  # host block 2 of 2
    with pytest.raises(Exception):
        ref.swap_blocks(host, gpu, [[4, 0]])  # gpu block 4 of 4


def test_copy_blocks_layers_copies_each_layer_and_nothing_else():
    import torch

    g = torch.Generator().manual_seed(8)
    L, nb, bs, H, D = 3, 10, 4, 2, 8
    ks = [torch.randn(nb, bs, H, D, generator=g).to(torch.bfloat16) for _ in range(L)]
    vs = [torch.randn(nb, bs, H, D, generator=g).to(torch.bfloat16) for _ in range(L)]
    pairs = np.array([[2, 7], [5, 0], [9, 3]], np.int32)
    out = ref.copy_blocks_layers(ks, vs, pairs, bs, H, D)
    for l in range(L):
        for c, (k_or_v) in enumerate((ks[l], vs[l])):
            want = ref.bits(k_or_v).copy()
            want[pairs[:, 1]] = want[pairs[:, 0]]  # the library's gather/scatter
            assert np.array_equal(out[l][c].reshape(want.shape), want)


# ---------------------------------------------------------------------------
# paged prefill attention ("Paged KV" wiki page, 实现原理 / 运行阶段)
# ---------------------------------------------------------------------------
def _prefill_case(seed, lens, chunk, Hq, Hkv, D, bs, dtype="bf16"):
    import torch

    from tests.helpers import paged_problem

    p = paged_problem(seed, Hq, Hkv, D, bs, lens, dtype)
    g = torch.Generator().manual_seed(seed + 1)
    n = [min(c, L) for c, L in zip(chunk, lens)]
    qs = np.concatenate([[0], np.cumsum(n)]).astype(np.int32)
    q = torch.randn(int(qs[-1]), Hq, D, generator=g).to(p["q"].dtype)
    return p, q, qs, n


def _dense_causal(p, q, qs, n, lens, Hq, Hkv, D, bs, scale):
    """The definition on gathered dense K/V with numpy and scipy's softmax."""
    from scipy.special import softmax

    kc = p["kc"].double().numpy()
    vc = p["vc"].double().numpy()
    qd = q.double().numpy()
    out = np.zeros_like(qd)
    G = Hq // Hkv
    for s, L in enumerate(lens):
        idx = [(p["tables"][s][t // bs], t % bs) for t in range(L)]
        K = np.stack([kc[b, o] for b, o in idx]) if L else np.zeros((0, Hkv, D))
        V = np.stack([vc[b, o] for b, o in idx]) if L else np.zeros((0, Hkv, D))
        for i in range(n[s]):
            pos = L - n[s] + i
            for h in range(Hq):
                sc = scale * K[:pos + 1, h // G] @ qd[qs[s] + i, h]
                out[qs[s] + i, h] = softmax(sc) @ V[:pos + 1, h // G]
    return out


@pytest.mark.parametrize("lens,chunk", [([5, 17, 33], [5, 17, 33]),  # whole prompts
                                        ([40, 9, 70], [8, 9, 31]),   # later chunks
                                        ([1, 16, 0], [1, 3, 0])])    # tiny and empty
def test_prefill_matches_dense_causal_softmax(lens, chunk):
    Hq, Hkv, D, bs, scale = 6, 2, 16, 8, 0.3
    p, q, qs, n = _prefill_case(11, lens, chunk, Hq, Hkv, D, bs)
    got = ref.prefill_attention(q, p["kc"], p["vc"], p["tables"], p["lens"], qs, scale, "bf16",
                                Hkv, bs)
    want = _dense_causal(p, q, qs, n, lens, Hq, Hkv, D, bs, scale)
    assert np.allclose(got, want, rtol=1e-12, atol=1e-12)


def test_prefill_with_one_row_per_sequence_is_decode():
    Hq, Hkv, D, bs, scale = 8, 2, 32, 16, 0.2
    lens = [3, 16, 47, 100]
    p, q, qs, n = _prefill_case(12, lens, [1] * 4, Hq, Hkv, D, bs)
    got = ref.prefill_attention(q, p["kc"], p["vc"], p["tables"], p["lens"], qs, scale, "bf16",
                                Hkv, bs)
    want = ref.decode_attention(q, p["kc"], p["vc"], p["tables"], p["lens"], scale, "bf16",
                                Hkv, bs)
    assert np.array_equal(got, want)


def test_prefill_first_prompt_row_is_v0_and_chunks_compose():
    Hq, Hkv, D, bs, scale = 4, 4, 16, 8, 0.25
    L = 29
    p, q, qs, n = _prefill_case(13, [L], [L], Hq, Hkv, D, bs)
    full = ref.prefill_attention(q, p["kc"], p["vc"], p["tables"], p["lens"], qs, scale, "bf16",
                                 Hkv, bs)
    b0 = p["tables"][0][0]
    assert np.array_equal(full[0], p["vc"][b0, 0].double().numpy())  # one token: weight 1
    # the same prompt in two chunks: 12 tokens, then 17 more
    a = ref.prefill_attention(q[:12], p["kc"], p["vc"], p["tables"], [12], [0, 12], scale,
                              "bf16", Hkv, bs)
    b = ref.prefill_attention(q[12:], p["kc"], p["vc"], p["tables"], [L], [0, 17], scale,
                              "bf16", Hkv, bs)
    assert np.array_equal(np.concatenate([a, b]), full)
