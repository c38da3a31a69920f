"""ctypes binding of ``libpkv.so`` (argument marshalling only).

Every function here has the name of the C entry point it calls and does no
work of its own beyond reading shapes, strides and pointers off torch tensors:
the computation runs in the library's CUDA kernels and C++ allocator.  There
is no fallback: if the library is missing, every call raises.
"""
import ctypes as C
import os

import torch

from . import build as _build

PKV_OK = 0
PKV_ERR_INVALID = -1
PKV_ERR_UNSUPPORTED = -2
PKV_ERR_CUDA = -3
PKV_ERR_OOM = -4
PKV_ERR_WORKSPACE = -5

PKV_F16 = 0
PKV_BF16 = 1

PKV_DEVERR_NONE = 0
PKV_DEVERR_CONTEXT_LEN = 1
PKV_DEVERR_BLOCK_ID = 2
PKV_DEVERR_SLOT = 3
PKV_DEVERR_PAIR = 4
PKV_DEVERR_TIMEOUT = 5
PKV_DEVERR_WORK_ITEM = 6

PKV_ITEMS_LONGEST_FIRST = 0
PKV_ITEMS_SEQUENCES_LONGEST_FIRST = 1
PKV_ITEMS_BATCH_ORDER = 2

PKV_NOALLOC_WORKSPACE_BYTES = 64 << 20

_DTYPE = {torch.float16: PKV_F16, torch.bfloat16: PKV_BF16}

# name -> (restype, argtypes)
_p, _i, _i64, _sz, _f = C.c_void_p, C.c_int, C.c_int64, C.c_size_t, C.c_float
SIGNATURES = {
    "pkv_write_slots": (_i, [_p, _p, _p, _p, _p, _i, _i, _i, _i, _i, _i64, _i, _p, _p]),
    "pkv_copy_blocks": (_i, [_p, _p, _p, _i, _i, _i, _i, _i, _i64, _i, _p, _p]),
    "pkv_copy_blocks_layers": (_i, [_p, _p, _i, _p, _i, _i, _i64, _i64, _p, _p]),
    "pkv_decode_workspace_bytes": (_sz, [_i, _i, _i, _i, _i]),
    "pkv_decode_attention": (_i, [_p, _p, _p, _p, _p, _i, _p, _i, _i, _i, _i, _i, _i, _i,
                                  _i64, _f, _i, _p, _sz, _i, _p, _p]),
    "pkv_decode_attention_items": (_i, [_p, _p, _p, _p, _p, _i, _p, _i, _i, _i, _i, _i, _i,
                                        _i, _i64, _f, _i, _p, _sz, _p, _i, _i, _p, _p]),
    "pkv_decode_work_items": (_i, [_p, _i, _i, _i, _i, _i, _p, _i, _p]),
    "pkv_decode_attention_noalloc": (_i, [_p, _p, _p, _p, _p, _i, _p, _i, _i, _i, _i, _i, _i,
                                          _i, _i64, _f, _i, _i, _p, _p]),
    "pkv_prefill_attention": (_i, [_p, _p, _p, _p, _p, _i, _p, _p, _i, _i, _i, _i, _i, _i, _i,
                                   _i64, _f, _i, _p, _p]),
    "pkv_write_slots_fp8": (_i, [_p, _p, _p, _p, _p, _p, _p, _i, _i, _i, _i, _i, _i64, _i, _p,
                                 _p]),
    "pkv_copy_blocks_fp8": (_i, [_p, _p, _p, _p, _p, _i, _i, _i, _i, _i, _i64, _p, _p]),
    "pkv_decode_attention_fp8": (_i, [_p, _p, _p, _p, _p, _p, _p, _i, _p, _i, _i, _i, _i, _i,
                                      _i, _i, _i64, _f, _i, _p, _sz, _i, _p, _p]),
    "pkv_decode_attention_fp8_items": (_i, [_p, _p, _p, _p, _p, _p, _p, _i, _p, _i, _i, _i,
                                            _i, _i, _i, _i, _i64, _f, _i, _p, _sz, _p, _i, _i,
                                            _p, _p]),
    "pkv_step_prepare": (_i, [_p, _i, _p, _p, _p, _p, _p, _i, _p, _p, _i, _i, _i, _i, _p, _i,
                              _p]),
    "pkv_decode_step": (_i, [_p, _p]),
    "pkv_pool_create": (_i, [_i, _i, _p, C.POINTER(_p)]),
    "pkv_pool_destroy": (None, [_p]),
    "pkv_seq_add": (_i, [_p, _i64, _i]),
    "pkv_seq_fork": (_i, [_p, _i64, _i64]),
    "pkv_seq_append": (_i, [_p, _i64, _p, _p, _p]),
    "pkv_seq_append_batch": (_i, [_p, _i, _p, _p, _p, _p, _p]),
    "pkv_seq_free": (_i, [_p, _i64]),
    "pkv_seq_num_tokens": (_i, [_p, _i64, _p]),
    "pkv_seq_block_table": (_i, [_p, _i64, _p, _i, _p]),
    "pkv_seq_slot_mapping": (_i, [_p, _i64, _i, _i, _p]),
    "pkv_pool_block_tables": (_i, [_p, _i, _p, _p, _i, C.c_int32, _p, _p]),
    "pkv_pool_num_free": (_i, [_p]),
    "pkv_pool_num_blocks": (_i, [_p]),
    "pkv_pool_block_size": (_i, [_p]),
    "pkv_pool_free_list": (_i, [_p, _p, _i, _p]),
    "pkv_block_refcount": (_i, [_p, _i]),
    "pkv_pool_set_host_blocks": (_i, [_p, _i]),
    "pkv_seq_swap_out": (_i, [_p, _i64, _p, _i, _p]),
    "pkv_seq_swap_in": (_i, [_p, _i64, _p, _i, _p]),
    "pkv_seq_is_swapped": (_i, [_p, _i64, _p]),
    "pkv_pool_num_free_host": (_i, [_p]),
    "pkv_pool_host_free_list": (_i, [_p, _p, _i, _p]),
    "pkv_host_block_refcount": (_i, [_p, _i]),
    "pkv_swap_blocks": (_i, [_p, _p, _p, _p, _p, _i, _i, _i, _i64, _i64, _i64, _p, _p]),
    "pkv_block_bytes": (_i64, [_i, _i, _i, _i, _i]),
    "pkv_selftest_bounded_wait": (_i, [_p, _i, _p]),
    "pkv_selftest_ex2_poly": (_i, [_p, _p, _i, _p]),
    "pkv_status_string": (C.c_char_p, [_i]),
    "pkv_last_error": (C.c_char_p, []),
    "pkv_version": (_i, []),
}

_lib = None


class DecodeStepArgs(C.Structure):
    """pkv_decode_step_args (include/pkv.h): one decode step's device work."""

    _fields_ = [("meta_host", _p), ("meta_device", _p), ("meta_bytes", _sz),
                ("cow_pairs", _p), ("num_pairs", _i),
                ("key", _p), ("value", _p), ("slot_mapping", _p), ("num_tokens", _i),
                ("key_cache", _p), ("value_cache", _p), ("k_scale", _p), ("v_scale", _p),
                ("num_blocks", _i), ("block_size", _i), ("num_kv_heads", _i), ("head_dim", _i),
                ("block_stride", _i64),
                ("out", _p), ("query", _p), ("block_tables", _p), ("max_blocks_per_seq", _i),
                ("context_lens", _p), ("num_seqs", _i), ("max_context_len", _i),
                ("num_q_heads", _i), ("scale", _f), ("partition_size", _i),
                ("workspace", _p), ("workspace_bytes", _sz),
                ("work_items", _p), ("num_items", _i),
                ("out_host", _p), ("out_bytes", _sz),
                ("dtype", _i), ("dev_error", _p), ("out_stream", _p), ("out_event", _p),
                ("meta_stream", _p), ("meta_event", _p), ("meta_after", _p),
                ("in_host", _p), ("in_device", _p), ("in_bytes", _sz)]


class PkvError(RuntimeError):
    def __init__(self, status, what):
        self.status = status
        super().__init__(what)


def library_path():
    return _build.LIB


def lib():
    """The loaded library; raises if it has not been built."""
    global _lib
    if _lib is None:
        path = library_path()
        if not os.path.exists(path):
            raise RuntimeError(
                "libpkv.so is not built (%s); run `python -m paged_kv_cache_337_b200.build`" % path)
        L = C.CDLL(path)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _check(status, name):
    if status != PKV_OK:
        msg = lib().pkv_last_error().decode(errors="replace")
        raise PkvError(status, "%s: %s (%s)" % (name, lib().pkv_status_string(status).decode(), msg))


def _ptr(t):
    return C.c_void_p(t.data_ptr()) if t is not None else C.c_void_p(0)


def _stream(stream, device):
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return C.c_void_p(stream.cuda_stream)


def _cache_geometry(cache):
    """(num_blocks, block_size, num_kv_heads, head_dim, block_stride) of a
    [NB, bs, Hkv, D] cache view whose last three dims are contiguous."""
    if cache.dim() != 4:
        raise ValueError("cache must be [num_blocks, block_size, num_kv_heads, head_dim]")
    nb, bs, hkv, d = cache.shape
    st = cache.stride()
    if st[3] != 1 or st[2] != d or st[1] != hkv * d:
        raise ValueError("a cache block must be contiguous")
    stride0 = st[0] if nb > 1 else bs * hkv * d
    return nb, bs, hkv, d, stride0


def _dtype(t):
    try:
        return _DTYPE[t.dtype]
    except KeyError:
        raise PkvError(PKV_ERR_UNSUPPORTED, "unsupported dtype %s" % t.dtype) from None


def _on_device(name, *tensors):
    """Kernel arguments must live on one CUDA device (a host pointer handed
    to a kernel would fault)."""
    dev = None
    for t in tensors:
        if t is None:
            continue
        if not t.is_cuda:
            raise ValueError("%s: every tensor argument must be a CUDA tensor" % name)
        if dev is None:
            dev = t.device
        elif t.device != dev:
            raise ValueError("%s: tensors on different devices" % name)
    return dev


def _need(t, dtype, name, device=None):
    if t.dtype != dtype:
        raise ValueError("%s must be %s, got %s" % (name, dtype, t.dtype))
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)


# ---------------------------------------------------------------------------
# kernels
# ---------------------------------------------------------------------------
def pkv_write_slots(key, value, key_cache, value_cache, slot_mapping, dev_error=None,
                    stream=None):
    """Write token rows key/value [T, Hkv, D] into their slots (int64 [T])."""
    _on_device("pkv_write_slots", key, value, key_cache, value_cache, slot_mapping, dev_error)
    nb, bs, hkv, d, bstride = _cache_geometry(key_cache)
    if _cache_geometry(value_cache) != (nb, bs, hkv, d, bstride):
        raise ValueError("key_cache and value_cache differ in geometry")
    _need(slot_mapping, torch.int64, "slot_mapping")
    _need(key, key_cache.dtype, "key")
    _need(value, key_cache.dtype, "value")
    T = slot_mapping.numel()
    if key.shape != (T, hkv, d) or value.shape != (T, hkv, d):
        raise ValueError("key/value must be [num_tokens, num_kv_heads, head_dim]")
    st = lib().pkv_write_slots(_ptr(key), _ptr(value), _ptr(key_cache), _ptr(value_cache),
                               _ptr(slot_mapping), T, nb, bs, hkv, d, bstride,
                               _dtype(key_cache), _ptr(dev_error),
                               _stream(stream, key_cache.device))
    _check(st, "pkv_write_slots")


def pkv_copy_blocks(key_cache, value_cache, block_pairs, dev_error=None, stream=None):
    """Copy whole blocks for each (src, dst) row of int32 block_pairs [n, 2]."""
    _on_device("pkv_copy_blocks", key_cache, value_cache, block_pairs, dev_error)
    nb, bs, hkv, d, bstride = _cache_geometry(key_cache)
    if _cache_geometry(value_cache) != (nb, bs, hkv, d, bstride):
        raise ValueError("key_cache and value_cache differ in geometry")
    _need(block_pairs, torch.int32, "block_pairs")
    n = block_pairs.numel() // 2
    st = lib().pkv_copy_blocks(_ptr(key_cache), _ptr(value_cache), _ptr(block_pairs), n, nb,
                               bs, hkv, d, bstride, _dtype(key_cache), _ptr(dev_error),
                               _stream(stream, key_cache.device))
    _check(st, "pkv_copy_blocks")


def layer_pointers(caches, device):
    """A device int64 array of the caches' data pointers (one per layer),
    for pkv_copy_blocks_layers."""
    return torch.tensor([c.data_ptr() for c in caches], dtype=torch.int64, device=device)


def pkv_copy_blocks_layers(key_caches, value_caches, block_pairs, dev_error=None, stream=None,
                           key_ptrs=None, value_ptrs=None):
    """Copy whole blocks in every layer for each (src, dst) row of int32
    block_pairs [n, 2]; key_caches / value_caches are per-layer
    [NB, bs, Hkv, D] caches of one geometry.  key_ptrs / value_ptrs may pass
    prebuilt layer_pointers arrays."""
    if len(key_caches) != len(value_caches) or not key_caches:
        raise ValueError("one K and one V cache per layer")
    _on_device("pkv_copy_blocks_layers", *key_caches, *value_caches, block_pairs, dev_error)
    geom = _cache_geometry(key_caches[0])
    for c in list(key_caches) + list(value_caches):
        if _cache_geometry(c) != geom or c.dtype != key_caches[0].dtype:
            raise ValueError("pkv_copy_blocks_layers: every layer's caches must match")
    _need(block_pairs, torch.int32, "block_pairs")
    nb, bs, hkv, d, stride = geom
    es = key_caches[0].element_size()
    dev = key_caches[0].device
    kp = key_ptrs if key_ptrs is not None else layer_pointers(key_caches, dev)
    vp = value_ptrs if value_ptrs is not None else layer_pointers(value_caches, dev)
    st = lib().pkv_copy_blocks_layers(_ptr(kp), _ptr(vp), len(key_caches), _ptr(block_pairs),
                                      block_pairs.numel() // 2, nb, bs * hkv * d * es,
                                      stride * es, _ptr(dev_error), _stream(stream, dev))
    _check(st, "pkv_copy_blocks_layers")


def pkv_decode_workspace_bytes(num_seqs, num_q_heads, max_context_len, partition_size,
                               head_dim):
    return int(lib().pkv_decode_workspace_bytes(num_seqs, num_q_heads, max_context_len,
                                                partition_size, head_dim))


def pkv_decode_work_items(context_lens, num_kv_heads, max_context_len, partition_size,
                          out=None, order=PKV_ITEMS_LONGEST_FIRST):
    """The decode work list for these lengths (a host int32 tensor or
    sequence): every (sequence, KV head, partition) that holds tokens, as
    flat grid indices, in one of the PKV_ITEMS_* orders.  Returns an int32
    CPU tensor (a view of `out` when given, e.g. pinned staging)."""
    lens = torch.as_tensor(context_lens, dtype=torch.int32)
    if lens.device.type != "cpu":
        raise ValueError("pkv_decode_work_items: context_lens must be on the host")
    lens = lens.contiguous()
    S = lens.numel()
    n = C.c_int()
    cap = out.numel() if out is not None else 0
    if out is None:
        lib().pkv_decode_work_items(_ptr(lens), S, num_kv_heads, int(max_context_len),
                                    int(partition_size), int(order), None, 0, C.byref(n))
        if n.value == 0 and S > 0:  # a size error: report it
            _check(lib().pkv_decode_work_items(_ptr(lens), S, num_kv_heads,
                                               int(max_context_len), int(partition_size),
                                               int(order), None, 0, C.byref(n)),
                   "pkv_decode_work_items")
        out = torch.empty(max(n.value, 1), dtype=torch.int32)
        cap = out.numel()
    elif out.dtype != torch.int32 or out.device.type != "cpu" or not out.is_contiguous():
        raise ValueError("pkv_decode_work_items: out must be a contiguous host int32 tensor")
    _check(lib().pkv_decode_work_items(_ptr(lens), S, num_kv_heads, int(max_context_len),
                                       int(partition_size), int(order), _ptr(out), cap,
                                       C.byref(n)), "pkv_decode_work_items")
    return out[:n.value]


def pkv_decode_attention(out, query, key_cache, value_cache, block_tables, context_lens,
                         max_context_len, scale, partition_size=0, workspace=None,
                         dev_error=None, stream=None, work_items=None):
    """Paged decode attention: out/query [S, Hq, D]; block_tables int32
    [S, MB]; context_lens int32 [S]; workspace a uint8 device tensor of at
    least pkv_decode_workspace_bytes(...) bytes when partitions are used.
    work_items: a device int32 list from pkv_decode_work_items for the same
    lengths (pkv_decode_attention_items), or None for the full grid."""
    _on_device("pkv_decode_attention", out, query, key_cache, value_cache, block_tables,
               context_lens, workspace, dev_error, work_items)
    nb, bs, hkv, d, bstride = _cache_geometry(key_cache)
    if _cache_geometry(value_cache) != (nb, bs, hkv, d, bstride):
        raise ValueError("key_cache and value_cache differ in geometry")
    S, hq, dq = query.shape
    if dq != d or out.shape != query.shape:
        raise ValueError("query/out must be [num_seqs, num_q_heads, head_dim]")
    _need(query, key_cache.dtype, "query")
    _need(out, key_cache.dtype, "out")
    _need(block_tables, torch.int32, "block_tables")
    _need(context_lens, torch.int32, "context_lens")
    if block_tables.dim() != 2 or block_tables.shape[0] != S or context_lens.numel() != S:
        raise ValueError("block_tables must be [num_seqs, max_blocks] and context_lens [num_seqs]")
    if dev_error is not None:
        _need(dev_error, torch.int32, "dev_error")
    mb = block_tables.shape[1]
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    if work_items is not None:
        _need(work_items, torch.int32, "work_items")
        st = lib().pkv_decode_attention_items(
            _ptr(out), _ptr(query), _ptr(key_cache), _ptr(value_cache), _ptr(block_tables), mb,
            _ptr(context_lens), S, int(max_context_len), hq, hkv, d, nb, bs, bstride,
            float(scale), int(partition_size), _ptr(workspace), ws_bytes, _ptr(work_items),
            work_items.numel(), _dtype(query), _ptr(dev_error), _stream(stream, query.device))
        _check(st, "pkv_decode_attention_items")
        return
    st = lib().pkv_decode_attention(
        _ptr(out), _ptr(query), _ptr(key_cache), _ptr(value_cache), _ptr(block_tables), mb,
        _ptr(context_lens), S, int(max_context_len), hq, hkv, d, nb, bs, bstride,
        float(scale), int(partition_size), _ptr(workspace), ws_bytes, _dtype(query),
        _ptr(dev_error), _stream(stream, query.device))
    _check(st, "pkv_decode_attention")


def pkv_prefill_attention(out, query, key_cache, value_cache, block_tables, context_lens,
                          query_start, max_query_len, scale, dev_error=None, stream=None):
    """Causal paged attention of each sequence's last n_s tokens: query/out
    [T, Hq, D] (rows query_start[s] .. query_start[s+1]-1 for sequence s),
    int32 block_tables [S, MB], context_lens [S], query_start [S + 1]."""
    _on_device("pkv_prefill_attention", out, query, key_cache, value_cache, block_tables,
               context_lens, query_start, dev_error)
    nb, bs, hkv, d, bstride = _cache_geometry(key_cache)
    if _cache_geometry(value_cache) != (nb, bs, hkv, d, bstride):
        raise ValueError("key_cache and value_cache differ in geometry")
    T, hq, dq = query.shape
    if dq != d or out.shape != query.shape:
        raise ValueError("query/out must be [rows, num_q_heads, head_dim]")
    _need(query, key_cache.dtype, "query")
    _need(out, key_cache.dtype, "out")
    _need(block_tables, torch.int32, "block_tables")
    _need(context_lens, torch.int32, "context_lens")
    _need(query_start, torch.int32, "query_start")
    S = context_lens.numel()
    if block_tables.dim() != 2 or block_tables.shape[0] != S or query_start.numel() != S + 1:
        raise ValueError("block_tables [S, MB], context_lens [S], query_start [S + 1]")
    st = lib().pkv_prefill_attention(
        _ptr(out), _ptr(query), _ptr(key_cache), _ptr(value_cache), _ptr(block_tables),
        block_tables.shape[1], _ptr(context_lens), _ptr(query_start), S, int(max_query_len), hq,
        hkv, d, nb, bs, bstride, float(scale), _dtype(query), _ptr(dev_error),
        _stream(stream, query.device))
    _check(st, "pkv_prefill_attention")


def pkv_decode_attention_noalloc(out, query, key_cache, value_cache, block_tables,
                                 context_lens, max_context_len, scale, partition_size=0,
                                 dev_error=None, stream=None):
    """pkv_decode_attention for callers that cannot allocate device memory:
    the split-K scratch is the library's built-in device array (at most
    PKV_NOALLOC_WORKSPACE_BYTES), shared by every call on the device, so
    calls must not overlap on the GPU."""
    _on_device("pkv_decode_attention_noalloc", out, query, key_cache, value_cache,
               block_tables, context_lens, dev_error)
    nb, bs, hkv, d, bstride = _cache_geometry(key_cache)
    if _cache_geometry(value_cache) != (nb, bs, hkv, d, bstride):
        raise ValueError("key_cache and value_cache differ in geometry")
    S, hq, dq = query.shape
    if dq != d or out.shape != query.shape:
        raise ValueError("query/out must be [num_seqs, num_q_heads, head_dim]")
    _need(query, key_cache.dtype, "query")
    _need(out, key_cache.dtype, "out")
    _need(block_tables, torch.int32, "block_tables")
    _need(context_lens, torch.int32, "context_lens")
    if block_tables.dim() != 2 or block_tables.shape[0] != S or context_lens.numel() != S:
        raise ValueError("block_tables must be [num_seqs, max_blocks] and context_lens [num_seqs]")
    st = lib().pkv_decode_attention_noalloc(
        _ptr(out), _ptr(query), _ptr(key_cache), _ptr(value_cache), _ptr(block_tables),
        block_tables.shape[1], _ptr(context_lens), S, int(max_context_len), hq, hkv, d, nb, bs,
        bstride, float(scale), int(partition_size), _dtype(query), _ptr(dev_error),
        _stream(stream, query.device))
    _check(st, "pkv_decode_attention_noalloc")


# ---------------------------------------------------------------------------
# FP8 (e4m3) caches with a scale per (block, KV head)
# ---------------------------------------------------------------------------
_FP8_CACHE_DTYPES = (torch.uint8, torch.float8_e4m3fn)


def fp8_scales(num_blocks, num_kv_heads, device, fill=1.0):
    """A [num_blocks, num_kv_heads] fp32 scale table whose storage is padded
    to a multiple of 4 floats (the kernels fetch scales 16 bytes at a time)."""
    n = num_blocks * num_kv_heads
    buf = torch.full(((n + 3) // 4 * 4,), fill, dtype=torch.float32, device=device)
    return buf[:n].view(num_blocks, num_kv_heads)


def _fp8_geometry(name, key_cache, value_cache, k_scale, v_scale):
    for c in (key_cache, value_cache):
        if c.dtype not in _FP8_CACHE_DTYPES:
            raise ValueError("%s: caches must be uint8 or float8_e4m3fn, got %s" % (name, c.dtype))
    geom = _cache_geometry(key_cache)
    if _cache_geometry(value_cache) != geom:
        raise ValueError("key_cache and value_cache differ in geometry")
    nb, _, hkv, _, _ = geom
    need = (nb * hkv + 3) // 4 * 4
    for sc in (k_scale, v_scale):
        _need(sc, torch.float32, "scales")
        if sc.numel() != nb * hkv:
            raise ValueError("%s: scales must hold num_blocks * num_kv_heads floats" % name)
        if sc.untyped_storage().nbytes() < (sc.storage_offset() + need) * 4:
            raise ValueError("%s: scale storage must be padded to a multiple of 4 floats "
                             "(use fp8_scales)" % name)
    return geom


def pkv_write_slots_fp8(key, value, key_cache, value_cache, k_scale, v_scale, slot_mapping,
                        dev_error=None, stream=None):
    """Quantise token rows key/value [T, Hkv, D] (f16/bf16) to e4m3 with the
    destination block's scale and write them into their slots."""
    _on_device("pkv_write_slots_fp8", key, value, key_cache, value_cache, k_scale, v_scale,
               slot_mapping, dev_error)
    nb, bs, hkv, d, bstride = _fp8_geometry("pkv_write_slots_fp8", key_cache, value_cache,
                                            k_scale, v_scale)
    _need(slot_mapping, torch.int64, "slot_mapping")
    _need(key, key.dtype, "key")
    _need(value, key.dtype, "value")
    T = slot_mapping.numel()
    if key.shape != (T, hkv, d) or value.shape != (T, hkv, d):
        raise ValueError("key/value must be [num_tokens, num_kv_heads, head_dim]")
    st = lib().pkv_write_slots_fp8(_ptr(key), _ptr(value), _ptr(key_cache), _ptr(value_cache),
                                   _ptr(k_scale), _ptr(v_scale), _ptr(slot_mapping), T, nb, bs,
                                   hkv, d, bstride, _dtype(key), _ptr(dev_error),
                                   _stream(stream, key_cache.device))
    _check(st, "pkv_write_slots_fp8")


def pkv_copy_blocks_fp8(key_cache, value_cache, k_scale, v_scale, block_pairs, dev_error=None,
                        stream=None):
    """Copy whole e4m3 blocks and their scales for each (src, dst) row of
    int32 block_pairs [n, 2]."""
    _on_device("pkv_copy_blocks_fp8", key_cache, value_cache, k_scale, v_scale, block_pairs,
               dev_error)
    nb, bs, hkv, d, bstride = _fp8_geometry("pkv_copy_blocks_fp8", key_cache, value_cache,
                                            k_scale, v_scale)
    _need(block_pairs, torch.int32, "block_pairs")
    n = block_pairs.numel() // 2
    st = lib().pkv_copy_blocks_fp8(_ptr(key_cache), _ptr(value_cache), _ptr(k_scale),
                                   _ptr(v_scale), _ptr(block_pairs), n, nb, bs, hkv, d, bstride,
                                   _ptr(dev_error), _stream(stream, key_cache.device))
    _check(st, "pkv_copy_blocks_fp8")


def pkv_decode_attention_fp8(out, query, key_cache, value_cache, k_scale, v_scale,
                             block_tables, context_lens, max_context_len, scale,
                             partition_size=0, workspace=None, dev_error=None, stream=None,
                             work_items=None):
    """pkv_decode_attention over e4m3 caches with per-(block, KV head)
    scales; query/out stay f16 or bf16.  work_items as in
    pkv_decode_attention (pkv_decode_attention_fp8_items)."""
    _on_device("pkv_decode_attention_fp8", out, query, key_cache, value_cache, k_scale, v_scale,
               block_tables, context_lens, workspace, dev_error, work_items)
    nb, bs, hkv, d, bstride = _fp8_geometry("pkv_decode_attention_fp8", key_cache, value_cache,
                                            k_scale, v_scale)
    S, hq, dq = query.shape
    if dq != d or out.shape != query.shape:
        raise ValueError("query/out must be [num_seqs, num_q_heads, head_dim]")
    _need(query, query.dtype, "query")
    _need(out, query.dtype, "out")
    _need(block_tables, torch.int32, "block_tables")
    _need(context_lens, torch.int32, "context_lens")
    if block_tables.dim() != 2 or block_tables.shape[0] != S or context_lens.numel() != S:
        raise ValueError("block_tables must be [num_seqs, max_blocks] and context_lens [num_seqs]")
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    if work_items is not None:
        _need(work_items, torch.int32, "work_items")
        st = lib().pkv_decode_attention_fp8_items(
            _ptr(out), _ptr(query), _ptr(key_cache), _ptr(value_cache), _ptr(k_scale),
            _ptr(v_scale), _ptr(block_tables), block_tables.shape[1], _ptr(context_lens), S,
            int(max_context_len), hq, hkv, d, nb, bs, bstride, float(scale),
            int(partition_size), _ptr(workspace), ws_bytes, _ptr(work_items),
            work_items.numel(), _dtype(query), _ptr(dev_error), _stream(stream, query.device))
        _check(st, "pkv_decode_attention_fp8_items")
        return
    st = lib().pkv_decode_attention_fp8(
        _ptr(out), _ptr(query), _ptr(key_cache), _ptr(value_cache), _ptr(k_scale),
        _ptr(v_scale), _ptr(block_tables), block_tables.shape[1], _ptr(context_lens), S,
        int(max_context_len), hq, hkv, d, nb, bs, bstride, float(scale), int(partition_size),
        _ptr(workspace), ws_bytes, _dtype(query), _ptr(dev_error), _stream(stream, query.device))
    _check(st, "pkv_decode_attention_fp8")


def pkv_selftest_bounded_wait(dev_error, limit_us, stream=None):
    """Run one bounded mbarrier wait that can never complete; the kernel
    records PKV_DEVERR_TIMEOUT in dev_error (int32[2] on the device)."""
    _on_device("pkv_selftest_bounded_wait", dev_error)
    _need(dev_error, torch.int32, "dev_error")
    _check(lib().pkv_selftest_bounded_wait(_ptr(dev_error), int(limit_us),
                                           _stream(stream, dev_error.device)),
           "pkv_selftest_bounded_wait")


def pkv_selftest_ex2_poly(x, y, stream=None):
    """y = 2^x elementwise by the prefill softmax's FMA-pipe exponential
    (float32 device tensors of one size)."""
    _on_device("pkv_selftest_ex2_poly", x, y)
    _need(x, torch.float32, "x")
    _need(y, torch.float32, "y")
    if x.numel() != y.numel():
        raise ValueError("x and y differ in size")
    _check(lib().pkv_selftest_ex2_poly(_ptr(x), _ptr(y), x.numel(), _stream(stream, x.device)),
           "pkv_selftest_ex2_poly")


def pkv_block_bytes(block_size, num_kv_heads, head_dim, num_layers, dtype_bytes):
    v = int(lib().pkv_block_bytes(block_size, num_kv_heads, head_dim, num_layers, dtype_bytes))
    if v < 0:
        _check(v, "pkv_block_bytes")
    return v


# ---------------------------------------------------------------------------
# host block pool
# ---------------------------------------------------------------------------
class BlockPool:
    """The library's host block pool (pkv_pool_* / pkv_seq_*)."""

    def __init__(self, num_blocks, block_size, free_order=None):
        handle = C.c_void_p()
        order = None
        if free_order is not None:
            order = torch.as_tensor(free_order, dtype=torch.int32).contiguous()
            if order.numel() != num_blocks:
                raise ValueError("free_order must have num_blocks entries")
        st = lib().pkv_pool_create(num_blocks, block_size, _ptr(order) if order is not None
                                   else C.c_void_p(0), C.byref(handle))
        _check(st, "pkv_pool_create")
        self._h = handle
        self.num_blocks = num_blocks
        self.block_size = block_size

    def close(self):
        if getattr(self, "_h", None):
            lib().pkv_pool_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def add(self, seq_id, num_tokens):
        _check(lib().pkv_seq_add(self._h, seq_id, num_tokens), "pkv_seq_add")

    def fork(self, parent, child):
        _check(lib().pkv_seq_fork(self._h, parent, child), "pkv_seq_fork")

    def append(self, seq_id):
        """Returns (slot, cow_src, cow_dst)."""
        slot = C.c_int64()
        src = C.c_int32()
        dst = C.c_int32()
        _check(lib().pkv_seq_append(self._h, seq_id, C.byref(slot), C.byref(src),
                                    C.byref(dst)), "pkv_seq_append")
        return slot.value, src.value, dst.value

    def append_batch(self, seq_ids, slots_out=None, pairs_out=None):
        """Append one token to each sequence in order.  Returns (slots int64
        [n], cow_pairs int32 [n_cow, 2]) as CPU tensors (views of the given
        output buffers, which may be pinned)."""
        ids = torch.as_tensor(seq_ids, dtype=torch.int64).contiguous()
        n = ids.numel()
        slots = slots_out if slots_out is not None else torch.empty(n, dtype=torch.int64)
        pairs = pairs_out if pairs_out is not None else torch.empty((n, 2), dtype=torch.int32)
        ncow = C.c_int()
        done = C.c_int()
        st = lib().pkv_seq_append_batch(self._h, n, _ptr(ids), _ptr(slots), _ptr(pairs),
                                        C.byref(ncow), C.byref(done))
        _check(st, "pkv_seq_append_batch")
        return slots[:n], pairs[:ncow.value]

    def free(self, seq_id):
        _check(lib().pkv_seq_free(self._h, seq_id), "pkv_seq_free")

    def num_tokens(self, seq_id):
        n = C.c_int()
        _check(lib().pkv_seq_num_tokens(self._h, seq_id, C.byref(n)), "pkv_seq_num_tokens")
        return n.value

    def slot_mapping(self, seq_id, first_token, num_tokens, out=None):
        """int64 [num_tokens] slots of the sequence's tokens from first_token."""
        slots = out if out is not None else torch.empty(num_tokens, dtype=torch.int64)
        _check(lib().pkv_seq_slot_mapping(self._h, seq_id, first_token, num_tokens,
                                          _ptr(slots)), "pkv_seq_slot_mapping")
        return slots[:num_tokens]

    def block_table(self, seq_id):
        n = C.c_int()
        cap = self.num_blocks
        buf = (C.c_int32 * max(cap, 1))()
        _check(lib().pkv_seq_block_table(self._h, seq_id, buf, cap, C.byref(n)),
               "pkv_seq_block_table")
        return list(buf[:n.value])

    def block_tables(self, seq_ids, max_blocks_per_seq, fill=-1, out=None, lens_out=None,
                     with_max=False):
        """Dense int32 [n, max_blocks_per_seq] tables and int32 [n] lengths
        (and, with with_max, the largest length)."""
        ids = torch.as_tensor(seq_ids, dtype=torch.int64).contiguous()
        n = ids.numel()
        tables = out if out is not None else torch.empty((n, max_blocks_per_seq),
                                                         dtype=torch.int32)
        lens = lens_out if lens_out is not None else torch.empty(n, dtype=torch.int32)
        longest = C.c_int32(0)
        st = lib().pkv_pool_block_tables(self._h, n, _ptr(ids), _ptr(tables),
                                         max_blocks_per_seq, fill, _ptr(lens),
                                         C.byref(longest))
        _check(st, "pkv_pool_block_tables")
        return (tables, lens, longest.value) if with_max else (tables, lens)

    def num_free(self):
        v = lib().pkv_pool_num_free(self._h)
        if v < 0:
            _check(v, "pkv_pool_num_free")
        return v

    def free_list(self):
        n = C.c_int()
        buf = (C.c_int32 * max(self.num_blocks, 1))()
        _check(lib().pkv_pool_free_list(self._h, buf, self.num_blocks, C.byref(n)),
               "pkv_pool_free_list")
        return list(buf[:n.value])

    def refcount(self, block):
        v = lib().pkv_block_refcount(self._h, block)
        if v < 0:
            _check(v, "pkv_block_refcount")
        return v

    def refcounts(self):
        return [self.refcount(b) for b in range(self.num_blocks)]

    # -- swapping to host blocks ------------------------------------------
    def set_host_blocks(self, num_host_blocks):
        _check(lib().pkv_pool_set_host_blocks(self._h, num_host_blocks),
               "pkv_pool_set_host_blocks")
        self.num_host_blocks = num_host_blocks

    def _swap(self, fn, name, seq_id):
        n = C.c_int()
        cap = max(self.num_blocks, 1)
        pairs = torch.empty((cap, 2), dtype=torch.int32)
        _check(fn(self._h, seq_id, _ptr(pairs), cap, C.byref(n)), name)
        return pairs[:n.value]

    def swap_out(self, seq_id):
        """int32 [n, 2] (gpu block, host block) pairs, in table order."""
        return self._swap(lib().pkv_seq_swap_out, "pkv_seq_swap_out", seq_id)

    def swap_in(self, seq_id):
        """int32 [n, 2] (host block, gpu block) pairs, in table order."""
        return self._swap(lib().pkv_seq_swap_in, "pkv_seq_swap_in", seq_id)

    def is_swapped(self, seq_id):
        v = C.c_int()
        _check(lib().pkv_seq_is_swapped(self._h, seq_id, C.byref(v)), "pkv_seq_is_swapped")
        return bool(v.value)

    def num_free_host(self):
        v = lib().pkv_pool_num_free_host(self._h)
        if v < 0:
            _check(v, "pkv_pool_num_free_host")
        return v

    def host_free_list(self):
        cap = max(getattr(self, "num_host_blocks", 0), 1)
        n = C.c_int()
        buf = (C.c_int32 * cap)()
        _check(lib().pkv_pool_host_free_list(self._h, buf, cap, C.byref(n)),
               "pkv_pool_host_free_list")
        return list(buf[:n.value])

    def host_refcounts(self):
        out = []
        for h in range(getattr(self, "num_host_blocks", 0)):
            v = lib().pkv_host_block_refcount(self._h, h)
            if v < 0:
                _check(v, "pkv_host_block_refcount")
            out.append(v)
        return out


def _pool_geometry(name, t):
    """(num_blocks, block_bytes, block_stride_bytes) of a [NB, ...] pool
    whose blocks are contiguous."""
    if t.dim() < 1:
        raise ValueError("%s must be [num_blocks, ...]" % name)
    nb = t.shape[0]
    inner = t[0] if nb else t
    if nb and not inner.is_contiguous():
        raise ValueError("%s: each block must be contiguous" % name)
    es = t.element_size()
    block_bytes = (t.numel() // nb if nb else 0) * es
    stride = t.stride(0) * es if nb > 1 else block_bytes
    return nb, block_bytes, stride


def pkv_swap_blocks(src_key, src_value, dst_key, dst_value, block_pairs, dev_error=None,
                    stream=None):
    """Copy blocks src -> dst for each (src, dst) row of int32 block_pairs
    [n, 2] between a device pool and a pinned host pool ([NB, ...] tensors
    of one block layout; src_value / dst_value may both be None)."""
    if (src_value is None) != (dst_value is None):
        raise ValueError("src_value and dst_value must both be given or both be None")
    dev = next(t.device for t in (src_key, dst_key) if t.is_cuda)
    for name, t in (("src_key", src_key), ("dst_key", dst_key), ("src_value", src_value),
                    ("dst_value", dst_value)):
        if t is not None and not t.is_cuda and not t.is_pinned():
            raise ValueError("pkv_swap_blocks: %s must be a CUDA tensor or pinned" % name)
    _need(block_pairs, torch.int32, "block_pairs")
    snb, sbytes, sstride = _pool_geometry("src_key", src_key)
    dnb, dbytes, dstride = _pool_geometry("dst_key", dst_key)
    if sbytes != dbytes:
        raise ValueError("pkv_swap_blocks: the pools' blocks differ in size")
    if src_value is not None:
        if (_pool_geometry("src_value", src_value) != (snb, sbytes, sstride)
                or _pool_geometry("dst_value", dst_value) != (dnb, dbytes, dstride)):
            raise ValueError("pkv_swap_blocks: K and V pools differ in geometry")
    n = block_pairs.numel() // 2
    st = lib().pkv_swap_blocks(_ptr(src_key), _ptr(src_value), _ptr(dst_key), _ptr(dst_value),
                               _ptr(block_pairs), n, snb, dnb, sbytes, sstride, dstride,
                               _ptr(dev_error), _stream(stream, dev))
    _check(st, "pkv_swap_blocks")
