"""Seeded synthetic inputs for the paged decode workloads.

This module only draws random numbers and fixes shapes; it holds none of the
method's arithmetic (no slot or table computation, no attention).  Both the
CUDA path and the CPU oracle receive the inputs it makes, so the two sides
see identical bits.

Distributions: context lengths are integer-uniform with both ends inclusive;
queries and cache values are N(0, 1) drawn in fp32 and rounded to the 16-bit
storage type; the initial free-block order of the pool is a seeded random
permutation, so sequences land on scattered physical blocks.  Workload k is
seeded with ``1000 + k``.

The named workloads follow the shapes the pages' deployments imply (a
7B-class model with 32 query = 32 KV heads; a 70B-class model with 64 query
heads over 8 KV heads; long 32K contexts at block sizes 32 and 64; parallel
sampling from a shared 1024-token prompt) and the block size 16 the
"PagedAttention 动态内存分页" page names as typical.
"""
import dataclasses
import math

import torch

_DT = {"f16": torch.float16, "bf16": torch.bfloat16}


@dataclasses.dataclass
class DecodeSpec:
    """Shape and distribution of one decode workload."""

    name: str
    seed: int
    num_seqs: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    len_lo: int  # context lengths ~ U[len_lo, len_hi], new token included
    len_hi: int
    dtype: str  # "f16" | "bf16"
    pool_blocks: int = 0  # 0: ceil(pool_factor * blocks the sequences need)
    pool_factor: float = 1.1
    partition_size: int = 0  # 0: single pass
    partition_size_e4m3: int = -1  # over an e4m3 cache (-1: partition_size)
    shared_prefix: bool = False

    @property
    def torch_dtype(self):
        return _DT[self.dtype]

    @property
    def scale(self):
        return 1.0 / math.sqrt(self.head_dim)

    @property
    def max_blocks_per_seq(self):
        return -(-self.len_hi // self.block_size)

    def partition_for(self, fp8):
        """Tokens per split-K partition over a 16-bit (fp8 False) or an e4m3
        cache."""
        if fp8 and self.partition_size_e4m3 >= 0:
            return self.partition_size_e4m3
        return self.partition_size


# The five workloads (sizes as the benchmark configurations state them).
TINY = DecodeSpec("tiny_s4_h8_d64_bs16_f16", 1001, 4, 8, 8, 64, 16, 1, 128, "f16",
                  pool_blocks=64)
DECODE_7B = DecodeSpec("7b_s256_h32_d128_bs16_bf16", 1002, 256, 32, 32, 128, 16,
                       128, 2048, "bf16")
# The GQA configuration fixes no partition size.  Over a 16-bit cache 2048
# tokens (about three waves of CTAs for this batch on 148 SMs) measured
# fastest among 512-4096; an e4m3 token is half the bytes, and 3584 tokens
# with sequences longest first measured fastest there (2048: 4892 GB/s,
# 3072: 4943, 4096: 5277 with items longest first; 3584: 5358-5368 with
# sequences longest first, against 5271-5277 for 4096 in the same runs).
# The long-context configuration fixes 512.
GQA_70B = DecodeSpec("70b_gqa_s64_hq64_hkv8_d128_bs16_bf16", 1003, 64, 64, 8, 128,
                     16, 512, 8192, "bf16", partition_size=2048, partition_size_e4m3=3584)
LONG_BS32 = DecodeSpec("long_s8_l32768_hq32_hkv8_d128_bs32_bf16", 1004, 8, 32, 8,
                       128, 32, 32768, 32768, "bf16", partition_size=512)
LONG_BS64 = DecodeSpec("long_s8_l32768_hq32_hkv8_d128_bs64_bf16", 1004, 8, 32, 8,
                       128, 64, 32768, 32768, "bf16", partition_size=512)

SPECS = {s.name: s for s in (TINY, DECODE_7B, GQA_70B, LONG_BS32, LONG_BS64)}


@dataclasses.dataclass
class DecodeInputs:
    """Host (CPU) tensors of one decode step, before any allocation."""

    spec: DecodeSpec
    context_lens: torch.Tensor  # int32 [S]: tokens after this step's write
    free_order: torch.Tensor  # int32 [NB]: initial pool order, first taken first
    query: torch.Tensor  # [S, Hq, D]
    key_cache: torch.Tensor  # [NB, bs, Hkv, D]
    value_cache: torch.Tensor  # [NB, bs, Hkv, D]
    new_key: torch.Tensor  # [S, Hkv, D]: K of the token written this step
    new_value: torch.Tensor  # [S, Hkv, D]

    @property
    def num_blocks(self):
        return int(self.free_order.numel())


def randn16(shape, gen, dtype, chunk=1 << 24):
    """N(0,1) in fp32, rounded to ``dtype``; drawn in chunks so a multi-GB
    tensor never needs its fp32 image in memory at once."""
    out = torch.empty(shape, dtype=dtype)
    flat = out.view(-1)
    for i in range(0, flat.numel(), chunk):
        n = min(chunk, flat.numel() - i)
        flat[i:i + n] = torch.randn(n, generator=gen, dtype=torch.float32).to(dtype)
    return out


def draw_lens(spec, gen):
    return torch.randint(spec.len_lo, spec.len_hi + 1, (spec.num_seqs,),
                         generator=gen, dtype=torch.int64).to(torch.int32)


def pool_size(spec, lens):
    if spec.pool_blocks:
        return spec.pool_blocks
    need = sum(-(-int(L) // spec.block_size) for L in lens)
    return int(math.ceil(spec.pool_factor * need))


def make_decode_inputs(spec, cache_values=True):
    """Draw every input of ``spec`` on the CPU from its seed.

    With ``cache_values=False`` the cache tensors are left empty (shape and
    dtype only), for callers that fill them on the device themselves.
    """
    gen = torch.Generator("cpu").manual_seed(spec.seed)
    lens = draw_lens(spec, gen)
    nb = pool_size(spec, lens)
    order = torch.randperm(nb, generator=gen, dtype=torch.int64).to(torch.int32)
    S, Hq, Hkv, D, bs = (spec.num_seqs, spec.num_q_heads, spec.num_kv_heads,
                         spec.head_dim, spec.block_size)
    dt = spec.torch_dtype
    q = randn16((S, Hq, D), gen, dt)
    k_new = randn16((S, Hkv, D), gen, dt)
    v_new = randn16((S, Hkv, D), gen, dt)
    if cache_values:
        kc = randn16((nb, bs, Hkv, D), gen, dt)
        vc = randn16((nb, bs, Hkv, D), gen, dt)
    else:
        kc = torch.empty((nb, bs, Hkv, D), dtype=dt)
        vc = torch.empty((nb, bs, Hkv, D), dtype=dt)
    return DecodeInputs(spec, lens, order, q, kc, vc, k_new, v_new)


def fill_device_cache_(tensor, seed):
    """Fill a device cache tensor with N(0,1) values from a seeded device
    generator (used by the benchmark, whose multi-GB caches are not checked
    element by element against the CPU oracle)."""
    gen = torch.Generator(tensor.device).manual_seed(seed)
    flat = tensor.view(-1)
    chunk = 1 << 28
    for i in range(0, flat.numel(), chunk):
        n = min(chunk, flat.numel() - i)
        flat[i:i + n] = torch.randn(n, generator=gen, device=tensor.device,
                                    dtype=torch.float32).to(tensor.dtype)
    return tensor


def fill_device_scales_(scales, seed, amax=4.0):
    """Seeded per-(block, KV head) e4m3 scales: amax / 448 (amax about the
    largest |x| of the 2048 N(0,1) values a block of 16 slots x 128 dims
    holds per head) times U[0.75, 1.25], so blocks differ."""
    gen = torch.Generator(scales.device).manual_seed(seed)
    u = torch.rand(scales.shape, generator=gen, device=scales.device, dtype=torch.float32)
    scales.copy_((0.75 + 0.5 * u) * (amax / 448.0))
    return scales


def fill_device_cache_fp8_(cache, scales, seed):
    """Fill an e4m3 cache ([NB, bs, Hkv, D] uint8) with N(0,1) values
    quantised (by torch's float8 conversion, setup only; the benchmark's
    caches are not compared with the oracle) with the block's scale for each
    KV head."""
    gen = torch.Generator(cache.device).manual_seed(seed)
    nb, bs, hkv, d = cache.shape
    step = max(1, (1 << 26) // (bs * hkv * d))
    for b0 in range(0, nb, step):
        b1 = min(nb, b0 + step)
        x = torch.randn((b1 - b0, bs, hkv, d), generator=gen, device=cache.device,
                        dtype=torch.float32)
        x /= scales[b0:b1, None, :, None]
        x.clamp_(-448.0, 448.0)  # saturate: the cast would give NaN beyond 448
        cache[b0:b1].copy_(x.to(torch.float8_e4m3fn).view(torch.uint8))
    return cache


# ---------------------------------------------------------------------------
# Shared-prefix parallel sampling (copy-on-write workload)
# ---------------------------------------------------------------------------
@dataclasses.dataclass
class SharedPrefixSpec:
    name: str = "shared_prefix_p16x8_pre1024_h32_d128_bs16_bf16"
    seed: int = 1005
    num_prompts: int = 16
    samples_per_prompt: int = 8
    prefix_len: int = 1024
    extra_lo: int = 1  # decoded tokens already in the shared prompt: U[1, 15]
    extra_hi: int = 15
    diverge_lo: int = 0  # private tokens per sample: U[0, 256]
    diverge_hi: int = 256
    num_q_heads: int = 32
    num_kv_heads: int = 32
    head_dim: int = 128
    block_size: int = 16
    dtype: str = "bf16"
    pool_factor: float = 1.1

    @property
    def torch_dtype(self):
        return _DT[self.dtype]

    @property
    def scale(self):
        return 1.0 / math.sqrt(self.head_dim)

    @property
    def num_seqs(self):
        return self.num_prompts * self.samples_per_prompt


SHARED_PREFIX = SharedPrefixSpec()
SHARED_PREFIX_SMALL = SharedPrefixSpec(
    name="shared_prefix_small_p3x4_pre40_h4_d64_bs16_f16", seed=1006, num_prompts=3,
    samples_per_prompt=4, prefix_len=40, extra_lo=1, extra_hi=7, diverge_lo=0,
    diverge_hi=40, num_q_heads=4, num_kv_heads=4, head_dim=64, dtype="f16")


@dataclasses.dataclass
class SharedPrefixInputs:
    spec: SharedPrefixSpec
    prompt_lens: torch.Tensor  # int32 [num_prompts]: prefix + already decoded
    diverge: torch.Tensor  # int32 [num_seqs]: private tokens before the steady step
    num_blocks: int
    free_order: torch.Tensor  # int32 [NB]
    seed_values: int  # seed for the K/V values written along the way


def make_shared_prefix_inputs(spec):
    gen = torch.Generator("cpu").manual_seed(spec.seed)
    P, N = spec.num_prompts, spec.samples_per_prompt
    extra = torch.randint(spec.extra_lo, spec.extra_hi + 1, (P,), generator=gen)
    prompt_lens = (spec.prefix_len + extra).to(torch.int32)
    diverge = torch.randint(spec.diverge_lo, spec.diverge_hi + 1, (P * N,),
                            generator=gen).to(torch.int32)
    bs = spec.block_size
    # worst case: every prompt's blocks, plus per sample one copied block and
    # the blocks of its private tokens and of two more steps
    need = sum(-(-int(L) // bs) for L in prompt_lens)
    need += sum(2 + -(-(int(d) + 2) // bs) for d in diverge)
    nb = int(math.ceil(spec.pool_factor * need))
    order = torch.randperm(nb, generator=gen, dtype=torch.int64).to(torch.int32)
    seed_values = int(torch.randint(0, 2**31 - 1, (1,), generator=gen))
    return SharedPrefixInputs(spec, prompt_lens, diverge, nb, order, seed_values)
