"""ctypes wrapper over the fp64 C oracle (``pkv_oracle.c``).

TEST INFRASTRUCTURE ONLY (tests, smoke check, CPU-baseline leg of the
benchmark).  Inputs are CPU arrays: 16-bit caches and queries are passed as
their raw bit patterns (numpy ``uint16``, or a CPU torch ``float16`` /
``bfloat16`` tensor which is reinterpreted without conversion).  Outputs of
the attention functions are numpy ``float64``.

Every function follows the C oracle's definition; see the comments there for
the passages of the pages each one restates.
"""
import ctypes as C

import numpy as np

from . import build_oracle

F16, BF16 = 0, 1
_DTYPES = {"f16": F16, "float16": F16, "fp16": F16, "bf16": BF16, "bfloat16": BF16}

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = build_oracle.build()
        L = C.CDLL(path)
        p = C.c_void_p
        i = C.c_int
        i64 = C.c_int64
        d = C.c_double
        L.pkv_oracle_bf16_to_f64.argtypes = [C.c_uint16]
        L.pkv_oracle_bf16_to_f64.restype = d
        L.pkv_oracle_f16_to_f64.argtypes = [C.c_uint16]
        L.pkv_oracle_f16_to_f64.restype = d
        L.pkv_oracle_decode_attention.argtypes = [p, p, p, p, p, i, p, i, i, i, i, i, i, i64, d, i, i]
        L.pkv_oracle_decode_partials.argtypes = [p, p, p, p, p, p, p, i, p, i, i, i, i, i, i, i64, d, i, i, i]
        L.pkv_oracle_merge_partials.argtypes = [p, p, p, p, p, i, i, i, i, i]
        L.pkv_oracle_write_slots.argtypes = [p, p, p, p, p, i, i, i, i, i, i64]
        L.pkv_oracle_copy_blocks.argtypes = [p, p, p, i, i, i, i, i, i64]
        L.pkv_oracle_swap_blocks.argtypes = [p, p, p, i, i, i, i64, i64, i64]
        L.pkv_oracle_prefill_attention.argtypes = [p, p, p, p, p, i, p, p, i, i, i, i, i, i,
                                                   i64, d, i, i]
        L.pkv_oracle_block_bytes.argtypes = [i, i, i, i, i]
        L.pkv_oracle_block_bytes.restype = i64
        L.pkv_oracle_max_threads.argtypes = []
        L.pkv_oracle_e4m3_to_f64.argtypes = [C.c_uint8]
        L.pkv_oracle_e4m3_to_f64.restype = d
        L.pkv_oracle_f32_to_e4m3_sat.argtypes = [C.c_float]
        L.pkv_oracle_f32_to_e4m3_sat.restype = C.c_uint8
        L.pkv_oracle_write_slots_fp8.argtypes = [p, p, p, p, p, i, i, i, i, i, i64, p, p, i]
        L.pkv_oracle_write_slots_fp8.restype = i
        L.pkv_oracle_decode_attention_fp8.argtypes = [p, p, p, p, p, p, p, i, p, i, i, i, i, i,
                                                      i, i64, d, i, i]
        L.pkv_oracle_decode_attention_fp8.restype = i
        for name in ("pkv_oracle_decode_attention", "pkv_oracle_decode_partials",
                     "pkv_oracle_merge_partials", "pkv_oracle_write_slots",
                     "pkv_oracle_copy_blocks", "pkv_oracle_max_threads"):
            getattr(L, name).restype = i
        _lib = L
    return _lib


class OracleError(RuntimeError):
    pass


def _dtype_code(dtype):
    if isinstance(dtype, int):
        return dtype
    name = str(dtype).replace("torch.", "")
    return _DTYPES[name]


def bits(x):
    """Raw 16-bit patterns of ``x`` as a C-contiguous numpy uint16 array."""
    if isinstance(x, np.ndarray):
        if x.dtype == np.uint16:
            return np.ascontiguousarray(x)
        if x.dtype == np.float16:
            return np.ascontiguousarray(x).view(np.uint16)
        raise TypeError("expected uint16 bits or float16, got %s" % x.dtype)
    # torch tensor (kept duck-typed so this module does not need torch)
    t = x.detach().cpu().contiguous()
    import torch

    return t.view(torch.int16).numpy().view(np.uint16)


def _ptr(a):
    return a.ctypes.data_as(C.c_void_p)


def _i32(a):
    a = np.ascontiguousarray(np.asarray(a), dtype=np.int32)
    return a


def _i64(a):
    return np.ascontiguousarray(np.asarray(a), dtype=np.int64)


def _num_blocks(size, block_stride, block_elems):
    """Blocks that fit in a flat buffer of ``size`` elements whose blocks of
    ``block_elems`` elements start ``block_stride`` elements apart."""
    if size < block_elems:
        return 0
    return (size - block_elems) // block_stride + 1


def _check(rc, what):
    if rc != 0:
        raise OracleError("%s: oracle rejected the input (status %d)" % (what, rc))


def bf16_to_f64(b):
    return lib().pkv_oracle_bf16_to_f64(int(b))


def f16_to_f64(b):
    return lib().pkv_oracle_f16_to_f64(int(b))


def decode_attention(query, key_cache, value_cache, block_tables, context_lens,
                     scale, dtype, num_kv_heads, block_size, block_stride=None,
                     num_threads=0):
    """Paged decode attention in fp64.

    query ``[S, Hq, D]``; caches hold ``NB`` blocks of ``[bs, Hkv, D]`` at
    ``block_stride`` elements apart (default: contiguous blocks);
    block_tables ``int32 [S, MB]``; context_lens ``int32 [S]``.
    Returns ``float64 [S, Hq, D]``.
    """
    q = bits(query)
    kc = bits(key_cache)
    vc = bits(value_cache)
    S, Hq, D = q.shape
    tables = _i32(block_tables)
    lens = _i32(context_lens)
    MB = tables.shape[1] if tables.ndim == 2 else 0
    if block_stride is None:
        block_stride = block_size * num_kv_heads * D
    NB = _num_blocks(kc.size, block_stride, block_size * num_kv_heads * D)
    out = np.zeros((S, Hq, D), dtype=np.float64)
    rc = lib().pkv_oracle_decode_attention(
        _ptr(out), _ptr(q), _ptr(kc), _ptr(vc), _ptr(tables), MB, _ptr(lens), S,
        Hq, num_kv_heads, D, NB, block_size, block_stride, float(scale),
        _dtype_code(dtype), int(num_threads))
    _check(rc, "decode_attention")
    return out


def decode_partials(query, key_cache, value_cache, block_tables, context_lens,
                    scale, dtype, num_kv_heads, block_size, partition_size,
                    num_partitions, block_stride=None):
    """Per-partition (m, l, o) in fp64: token ranges [pP, min((p+1)P, L))."""
    q = bits(query)
    kc = bits(key_cache)
    vc = bits(value_cache)
    S, Hq, D = q.shape
    tables = _i32(block_tables)
    lens = _i32(context_lens)
    MB = tables.shape[1]
    if block_stride is None:
        block_stride = block_size * num_kv_heads * D
    NB = _num_blocks(kc.size, block_stride, block_size * num_kv_heads * D)
    NP = int(num_partitions)
    m = np.zeros((S, Hq, NP), dtype=np.float64)
    l = np.zeros((S, Hq, NP), dtype=np.float64)
    o = np.zeros((S, Hq, NP, D), dtype=np.float64)
    rc = lib().pkv_oracle_decode_partials(
        _ptr(m), _ptr(l), _ptr(o), _ptr(q), _ptr(kc), _ptr(vc), _ptr(tables), MB,
        _ptr(lens), S, Hq, num_kv_heads, D, NB, block_size, block_stride,
        float(scale), _dtype_code(dtype), int(partition_size), NP)
    _check(rc, "decode_partials")
    return m, l, o


def merge_partials(m, l, o, context_lens, partition_size):
    m = np.ascontiguousarray(m, dtype=np.float64)
    l = np.ascontiguousarray(l, dtype=np.float64)
    o = np.ascontiguousarray(o, dtype=np.float64)
    lens = _i32(context_lens)
    S, Hq, NP, D = o.shape
    out = np.zeros((S, Hq, D), dtype=np.float64)
    rc = lib().pkv_oracle_merge_partials(_ptr(out), _ptr(m), _ptr(l), _ptr(o),
                                         _ptr(lens), S, Hq, D, int(partition_size), NP)
    _check(rc, "merge_partials")
    return out


def write_slots(key_cache, value_cache, key, value, slot_mapping, block_size,
                num_kv_heads, block_stride=None):
    """Returns new (key_cache, value_cache) bit arrays with the tokens written."""
    kc = bits(key_cache).copy()
    vc = bits(value_cache).copy()
    k = bits(key)
    v = bits(value)
    slots = _i64(slot_mapping)
    T = slots.shape[0]
    D = k.shape[-1]
    if block_stride is None:
        block_stride = block_size * num_kv_heads * D
    NB = _num_blocks(kc.size, block_stride, block_size * num_kv_heads * D)
    rc = lib().pkv_oracle_write_slots(_ptr(kc), _ptr(vc), _ptr(k), _ptr(v), _ptr(slots),
                                      T, NB, block_size, num_kv_heads, D, block_stride)
    _check(rc, "write_slots")
    return kc, vc


def prefill_attention(query, key_cache, value_cache, block_tables, context_lens, query_start,
                      scale, dtype, num_kv_heads, block_size, block_stride=None, num_threads=0):
    """Causal paged attention of each sequence's last n_s tokens (query rows
    query_start[s] .. query_start[s+1]-1 of query [T, Hq, D]) over its
    cached K/V, in fp64.  Returns [T, Hq, D]."""
    q = bits(query)
    kc = bits(key_cache)
    vc = bits(value_cache)
    T, Hq, D = q.shape
    tables = _i32(block_tables)
    lens = _i32(context_lens)
    qs = _i32(query_start)
    S = lens.shape[0]
    if qs.shape[0] != S + 1 or qs[-1] != T:
        raise ValueError("query_start must be [num_seqs + 1] ending at the number of rows")
    MB = tables.shape[1] if tables.ndim == 2 else 0
    if block_stride is None:
        block_stride = block_size * num_kv_heads * D
    NB = _num_blocks(kc.size, block_stride, block_size * num_kv_heads * D)
    out = np.zeros((T, Hq, D), dtype=np.float64)
    rc = lib().pkv_oracle_prefill_attention(
        _ptr(out), _ptr(q), _ptr(kc), _ptr(vc), _ptr(tables), MB, _ptr(lens), _ptr(qs), S, Hq,
        num_kv_heads, D, NB, block_size, block_stride, float(scale), _dtype_code(dtype),
        int(num_threads))
    _check(rc, "prefill_attention")
    return out


def copy_blocks_layers(key_caches, value_caches, block_pairs, block_size, num_kv_heads,
                       head_dim):
    """Copy-on-write over a multi-layer cache: one physical block id names
    the block in every layer ("Paged KV" wiki page, 初始化阶段: a block holds
    K and V of all layers), so each pair is copied in each layer.  Returns
    the new per-layer (key, value) bit arrays."""
    return [copy_blocks(k, v, block_pairs, block_size, num_kv_heads, head_dim)
            for k, v in zip(key_caches, value_caches)]


def swap_blocks(dst_pool, src_pool, block_pairs):
    """Returns a copy of dst_pool ([NB_dst, ...], any dtype) whose block
    pairs[i][1] holds block pairs[i][0] of src_pool; one block is one row of
    the leading dimension."""
    dst = _u8(dst_pool).copy()
    src = _u8(src_pool)
    nd, ns = int(dst_pool.shape[0]), int(src_pool.shape[0])
    dst = dst.reshape(nd, -1)
    src = np.ascontiguousarray(src).reshape(ns, -1)
    if dst.shape[1] != src.shape[1]:
        raise ValueError("the pools' blocks differ in size")
    pairs = _i32(block_pairs).reshape(-1, 2)
    nbytes = dst.shape[1]
    rc = lib().pkv_oracle_swap_blocks(_ptr(dst), _ptr(src), _ptr(pairs), pairs.shape[0], ns, nd,
                                      nbytes, nbytes, nbytes)
    _check(rc, "swap_blocks")
    return dst.reshape(_u8(dst_pool).shape)


def copy_blocks(key_cache, value_cache, block_pairs, block_size, num_kv_heads,
                head_dim, block_stride=None):
    """Returns new (key_cache, value_cache) bit arrays after the copies."""
    kc = bits(key_cache).copy()
    vc = bits(value_cache).copy()
    pairs = _i32(block_pairs).reshape(-1, 2)
    if block_stride is None:
        block_stride = block_size * num_kv_heads * head_dim
    NB = _num_blocks(kc.size, block_stride, block_size * num_kv_heads * head_dim)
    rc = lib().pkv_oracle_copy_blocks(_ptr(kc), _ptr(vc), _ptr(pairs), pairs.shape[0],
                                      NB, block_size, num_kv_heads, head_dim, block_stride)
    _check(rc, "copy_blocks")
    return kc, vc


def block_bytes(block_size, num_kv_heads, head_dim, num_layers, dtype_bytes):
    return int(lib().pkv_oracle_block_bytes(block_size, num_kv_heads, head_dim,
                                            num_layers, dtype_bytes))


def max_threads():
    return int(lib().pkv_oracle_max_threads())


# ---------------------------------------------------------------------------
# FP8 (e4m3) caches with a float32 scale per (block, KV head)
# ---------------------------------------------------------------------------
def _u8(x):
    if isinstance(x, np.ndarray):
        return np.ascontiguousarray(x, dtype=np.uint8) if x.dtype == np.uint8 else \
            np.ascontiguousarray(x).view(np.uint8)
    import torch

    return x.detach().cpu().contiguous().view(torch.uint8).numpy()


def _f32(x):
    if isinstance(x, np.ndarray):
        return np.ascontiguousarray(x, dtype=np.float32)
    return x.detach().cpu().contiguous().float().numpy()


def e4m3_to_f64(code):
    return lib().pkv_oracle_e4m3_to_f64(int(code))


def f32_to_e4m3(x):
    return int(lib().pkv_oracle_f32_to_e4m3_sat(float(x)))


def write_slots_fp8(key_cache, value_cache, key, value, slot_mapping, block_size,
                    num_kv_heads, k_scale, v_scale, dtype, block_stride=None):
    """e4m3 caches (uint8) after writing 16-bit K/V rows quantised with the
    scale of their (block, KV head)."""
    kc = _u8(key_cache).copy()
    vc = _u8(value_cache).copy()
    k = bits(key)
    v = bits(value)
    slots = _i64(slot_mapping)
    ks, vs = _f32(k_scale), _f32(v_scale)
    D = k.shape[-1]
    if block_stride is None:
        block_stride = block_size * num_kv_heads * D
    NB = _num_blocks(kc.size, block_stride, block_size * num_kv_heads * D)
    rc = lib().pkv_oracle_write_slots_fp8(_ptr(kc), _ptr(vc), _ptr(k), _ptr(v), _ptr(slots),
                                          slots.shape[0], NB, block_size, num_kv_heads, D,
                                          block_stride, _ptr(ks), _ptr(vs), _dtype_code(dtype))
    _check(rc, "write_slots_fp8")
    return kc, vc


def decode_attention_fp8(query, key_cache, value_cache, k_scale, v_scale, block_tables,
                         context_lens, scale, dtype, num_kv_heads, block_size,
                         block_stride=None, num_threads=0):
    """Paged decode attention in fp64 over e4m3 caches with per-(block, KV
    head) scales; query is 16-bit ([S, Hq, D])."""
    q = bits(query)
    kc = _u8(key_cache)
    vc = _u8(value_cache)
    ks, vs = _f32(k_scale), _f32(v_scale)
    S, Hq, D = q.shape
    tables = _i32(block_tables)
    lens = _i32(context_lens)
    MB = tables.shape[1] if tables.ndim == 2 else 0
    if block_stride is None:
        block_stride = block_size * num_kv_heads * D
    NB = _num_blocks(kc.size, block_stride, block_size * num_kv_heads * D)
    out = np.zeros((S, Hq, D), dtype=np.float64)
    rc = lib().pkv_oracle_decode_attention_fp8(
        _ptr(out), _ptr(q), _ptr(kc), _ptr(vc), _ptr(ks), _ptr(vs), _ptr(tables), MB,
        _ptr(lens), S, Hq, num_kv_heads, D, NB, block_size, block_stride, float(scale),
        _dtype_code(dtype), int(num_threads))
    _check(rc, "decode_attention_fp8")
    return out
