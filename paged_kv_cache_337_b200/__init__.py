"""B200-native paged KV cache: the data-parallel hot path of PagedAttention.

The work runs in ``libpkv.so`` (CUDA kernels for sm_100a and a C++ block
pool) behind a C ABI declared in ``include/pkv.h``.  This package holds the
thin ctypes binding (:mod:`._abi`, same names as the C entry points), the
decode-step driver built on it (:mod:`.cache`), the library build
(:mod:`.build`) and the seeded workload generators (:mod:`.workloads`).
Importing the package loads nothing; the first call loads the library and
raises if it has not been built.
"""
from ._abi import (  # noqa: F401
    BlockPool,
    PkvError,
    fp8_scales,
    pkv_block_bytes,
    pkv_copy_blocks,
    pkv_copy_blocks_fp8,
    pkv_decode_attention,
    pkv_decode_attention_fp8,
    pkv_decode_attention_noalloc,
    pkv_decode_workspace_bytes,
    pkv_write_slots,
    pkv_write_slots_fp8,
)
