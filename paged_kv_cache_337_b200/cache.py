"""Decode-step driver over the C ABI: one paged KV cache (one layer) with its
block pool, and the per-step sequence of calls the pages describe.

A decode step for a batch of sequences ("Paged KV" wiki page, 实现原理 /
运行阶段; "PagedAttention 动态内存分页" page, 写时复制与内存共享):

1. the host pool reserves each sequence's next slot, taking a new block when
   the current one is full and copying a shared current block first
   (``pkv_seq_append_batch``);
2. the copy-on-write pairs are applied on the GPU (``pkv_copy_blocks``);
3. the new tokens' K/V are written into their slots (``pkv_write_slots``);
4. decode attention runs over every sequence's blocks through its Block
   Table (``pkv_decode_attention``; split-K with a merge for long contexts).

With an e4m3 cache ("Paged KV" wiki page, 局限性: KV FP8 with a scale per
block) the three device calls are their ``_fp8`` forms, which also copy and
read the per-(block, KV head) scales.

Steps 2-4 are launched on one stream; the metadata of step 1 travels to the
device through pinned host staging buffers.  When the step splits
sequences into partitions, step 1 also asks the library for the decode work
list (``pkv_decode_work_items``: every (sequence, KV head, partition)
holding tokens, in the order ``work_list`` picks) and step 4 runs over it
(``pkv_decode_attention_items``) instead of the full grid, whose slots past
the shorter sequences' ends would launch and exit.  All arithmetic is in
the library; this module only moves arguments.

``upload_step`` and ``launch_step`` may run on different streams: the
launch waits for the upload's event, and the next upload into the same
staging bank waits for the last launch that read it.
"""
import torch

from . import _abi


class PagedKVCache:
    def __init__(self, num_blocks, block_size, num_q_heads, num_kv_heads, head_dim, dtype,
                 device, max_blocks_per_seq, partition_size=0, free_order=None,
                 key_cache=None, value_cache=None, scale=None, kv_dtype=None, kv_scale=1.0,
                 work_list="auto"):
        """dtype is the type of queries, new K/V rows and outputs (f16 or
        bf16).  kv_dtype torch.uint8 (or torch.float8_e4m3fn) stores the
        cache as e4m3 codes with a scale per (block, KV head) in k_scale /
        v_scale ([num_blocks, num_kv_heads] fp32, every entry kv_scale until
        the caller sets them); None stores it in dtype.

        work_list: the decode grid.  "auto" (or True): the full grid when
        every sequence fits one partition, else the library's work list,
        items longest first for an e4m3 cache and sequences longest first
        for a 16-bit cache (the orders measured fastest on B200 for the
        GQA and long-context batches); "longest_first",
        "sequences_longest_first", "batch_order": the work list in that
        order on every step; False or "none": the full grid."""
        self.num_blocks = num_blocks
        self.block_size = block_size
        self.num_q_heads = num_q_heads
        self.num_kv_heads = num_kv_heads
        self.head_dim = head_dim
        self.dtype = dtype
        self.device = torch.device(device)
        self.max_blocks_per_seq = max_blocks_per_seq
        self.partition_size = partition_size
        orders = {"longest_first": _abi.PKV_ITEMS_LONGEST_FIRST,
                  "sequences_longest_first": _abi.PKV_ITEMS_SEQUENCES_LONGEST_FIRST,
                  "batch_order": _abi.PKV_ITEMS_BATCH_ORDER}
        if work_list is True:
            work_list = "auto"
        if work_list in (False, "none"):
            work_list = None
        if work_list is not None and work_list != "auto" and work_list not in orders:
            raise ValueError("work_list must be 'auto', 'longest_first', "
                             "'sequences_longest_first', 'batch_order' or False")
        self.work_list = work_list is not None
        self._item_order = orders.get(work_list)  # None: "auto"
        self.scale = scale if scale is not None else 1.0 / (head_dim ** 0.5)
        shape = (num_blocks, block_size, num_kv_heads, head_dim)
        kv_dtype = dtype if kv_dtype is None else kv_dtype
        self.fp8 = kv_dtype in (torch.uint8, torch.float8_e4m3fn)
        self.key_cache = key_cache if key_cache is not None else torch.empty(
            shape, dtype=kv_dtype, device=self.device)
        self.value_cache = value_cache if value_cache is not None else torch.empty(
            shape, dtype=kv_dtype, device=self.device)
        self.k_scale = self.v_scale = None
        if self.fp8:
            self.k_scale = _abi.fp8_scales(num_blocks, num_kv_heads, self.device, kv_scale)
            self.v_scale = _abi.fp8_scales(num_blocks, num_kv_heads, self.device, kv_scale)
        self.pool = _abi.BlockPool(num_blocks, block_size, free_order)
        self.dev_error = torch.zeros(2, dtype=torch.int32, device=self.device)
        self._workspace = torch.empty(0, dtype=torch.uint8, device=self.device)
        self._staging = {}
        self._seen = set()  # tensor signatures the binding has checked
        self._geom = _abi._cache_geometry(self.key_cache)
        self._dtype_code = _abi._DTYPE[dtype]

    # -- sequence management (host) ---------------------------------------
    def add_sequence(self, seq_id, num_tokens, key=None, value=None, stream=None):
        """Prefill allocation of num_tokens tokens; with key/value
        ([num_tokens, Hkv, D] device tensors) their rows are written into the
        blocks taken, in order."""
        self.pool.add(seq_id, num_tokens)
        if key is not None and num_tokens > 0:
            slots = self.pool.slot_mapping(seq_id, 0, num_tokens).to(self.device)
            self._write(key, value, slots, stream)

    def fork(self, parent, child):
        self.pool.fork(parent, child)

    def free(self, seq_id):
        self.pool.free(seq_id)

    # -- one decode step --------------------------------------------------
    def _item_capacity(self, n):
        """Work items a batch of n sequences can need: every (sequence, KV
        head, partition) of the longest context the tables can hold."""
        if not self.work_list:
            return 0
        longest = self.max_blocks_per_seq * self.block_size
        P = self.partition_size
        parts = 1 if P <= 0 or P >= longest else -(-longest // P)
        return n * self.num_kv_heads * parts

    def _stage(self, n):
        """Staging for a batch of n sequences: two banks, each one pinned host
        buffer and one device buffer holding slots | lengths | copy pairs |
        Block Tables | work items, so a step's metadata travels in one copy
        (of the used prefix) and the next step can be prepared while the
        previous upload is in flight."""
        banks = self._staging.get(n)
        if banks is None:
            pin = torch.cuda.is_available()
            mb = self.max_blocks_per_seq
            cap = self._item_capacity(n)
            t0 = 5 * n
            i0 = t0 + n * mb
            words = i0 + cap  # int32 words

            def views(buf):
                return dict(slots=buf[:2 * n].view(torch.int64), lens=buf[2 * n:3 * n],
                            pairs=buf[3 * n:5 * n].view(n, 2),
                            tables=buf[t0:i0].view(n, mb), items=buf[i0:])

            banks = []
            for _ in range(2):
                h = torch.empty(max(words, 1), dtype=torch.int32, pin_memory=pin)
                d = torch.empty(max(words, 1), dtype=torch.int32, device=self.device)
                hv, dv = views(h), views(d)
                banks.append(dict(ids=torch.empty(n, dtype=torch.int64), h=h, d=d,
                                  h_slots=hv["slots"], h_lens=hv["lens"], h_pairs=hv["pairs"],
                                  h_tables=hv["tables"], h_items=hv["items"],
                                  d_slots=dv["slots"], d_lens=dv["lens"], d_pairs=dv["pairs"],
                                  d_tables=dv["tables"], d_items=dv["items"], items_off=i0,
                                  uploaded=None, consumed=None))
            self._staging[n] = banks = [banks, 0]
        banks[1] ^= 1
        return banks[0][banks[1]]

    def prepare_step(self, seq_ids):
        """Host part of a decode step: reserve one slot per sequence (new
        blocks and copy-on-write pairs as needed) and gather the Block Tables
        and lengths into pinned memory.  Returns the prepared step."""
        st = self._stage(len(seq_ids))
        if st["uploaded"] is not None:
            st["uploaded"].synchronize()  # this bank's last upload has left
        if st.get("ids_src") is not seq_ids:  # a new id list: convert it once
            st["ids"].copy_(torch.as_tensor(seq_ids, dtype=torch.int64))
            st["ids_src"] = seq_ids
        slots, pairs = self.pool.append_batch(st["ids"], st["h_slots"], st["h_pairs"])
        tables, lens, longest = self.pool.block_tables(
            st["ids"], self.max_blocks_per_seq, -1, st["h_tables"], st["h_lens"], with_max=True)
        n_items = -1  # the full grid
        order = self._item_order
        split = 0 < self.partition_size < longest
        if self.work_list and order is None and split:
            order = (_abi.PKV_ITEMS_LONGEST_FIRST if self.fp8 else
                     _abi.PKV_ITEMS_SEQUENCES_LONGEST_FIRST)
        if self.work_list and order is not None:
            n_items = _abi.pkv_decode_work_items(lens, self.num_kv_heads, longest,
                                                 self.partition_size, st["h_items"],
                                                 order).numel()
        return dict(st=st, num_pairs=pairs.shape[0], max_len=longest, num_items=n_items)

    def upload_step(self, prep, stream=None):
        """One host-to-device copy of a prepared step's metadata (the work
        items the step uses, not the whole capacity)."""
        st = prep["st"]
        s = stream if stream is not None else torch.cuda.current_stream(self.device)
        used = st["items_off"] + max(prep.get("num_items", 0), 0)
        with torch.cuda.stream(s):
            if st["consumed"] is not None:
                s.wait_event(st["consumed"])  # the last launch that read this bank
            st["d"][:used].copy_(st["h"][:used], non_blocking=True)
            if st["uploaded"] is None:
                st["uploaded"] = torch.cuda.Event()
            st["uploaded"].record(s)

    def workspace(self, num_seqs, max_len):
        need = _abi.pkv_decode_workspace_bytes(num_seqs, self.num_q_heads, max_len,
                                               self.partition_size, self.head_dim)
        if self._workspace.numel() < need:
            self._workspace = torch.empty(need, dtype=torch.uint8, device=self.device)
        return self._workspace if need else None

    def launch_step(self, prep, query, key, value, out, max_len=None, stream=None):
        """Device part of a decode step (copy, write, attention) with the
        prepared metadata uploaded by upload_step (on this or another
        stream: the launch waits for it)."""
        st = prep["st"]
        n = prep["num_pairs"]
        items = prep.get("num_items", -1)
        if max_len is not None and max_len != prep["max_len"]:
            items = -1  # the work list was planned for the prepared bound
        max_len = prep["max_len"] if max_len is None else max_len
        s_ = stream if stream is not None else torch.cuda.current_stream(self.device)
        if st["uploaded"] is not None:
            s_.wait_event(st["uploaded"])
        try:
            return self._launch(st, n, items, max_len, query, key, value, out, stream)
        finally:
            if st["consumed"] is None:
                st["consumed"] = torch.cuda.Event()
            st["consumed"].record(s_)

    def _launch(self, st, n, items, max_len, query, key, value, out, stream):
        if n:
            self._copy(st["d_pairs"][:n], stream)
        ws = self.workspace(len(st["ids"]), max_len)
        wl = st["d_items"][:items] if items >= 0 else None
        if not self._checked(query, key, value, out):
            # first use of these tensor shapes: the binding's full checks
            self._write(key, value, st["d_slots"], stream)
            self._attend(out, query, st["d_tables"], st["d_lens"], max_len, ws, stream, wl)
            self._seen.add(self._signature(query, key, value, out))
            return out
        # same shapes, dtypes and device as a call already checked: pass the
        # pointers straight to the C entry points
        L = _abi.lib()
        sp = _abi._stream(stream, self.device)
        kc, vc = self.key_cache, self.value_cache
        nb, bs, hkv, d, bstride = self._geom
        S = query.shape[0]
        err = self.dev_error.data_ptr()
        wsp, wsn = (ws.data_ptr(), ws.numel()) if ws is not None else (None, 0)
        args = (st["d_tables"].data_ptr(), self.max_blocks_per_seq, st["d_lens"].data_ptr(), S,
                int(max_len), self.num_q_heads, hkv, d, nb, bs, bstride, float(self.scale),
                int(self.partition_size), wsp, wsn)
        tail = (self._dtype_code, err, sp)
        if wl is not None:
            tail = (wl.data_ptr(), wl.numel()) + tail
        if self.fp8:
            ks, vs = self.k_scale.data_ptr(), self.v_scale.data_ptr()
            _abi._check(L.pkv_write_slots_fp8(
                key.data_ptr(), value.data_ptr(), kc.data_ptr(), vc.data_ptr(), ks, vs,
                st["d_slots"].data_ptr(), S, nb, bs, hkv, d, bstride, self._dtype_code, err, sp),
                "pkv_write_slots_fp8")
            fn = L.pkv_decode_attention_fp8_items if wl is not None else L.pkv_decode_attention_fp8
            _abi._check(fn(out.data_ptr(), query.data_ptr(), kc.data_ptr(), vc.data_ptr(), ks, vs,
                           *args, *tail), "pkv_decode_attention_fp8")
            return out
        _abi._check(L.pkv_write_slots(key.data_ptr(), value.data_ptr(), kc.data_ptr(),
                                      vc.data_ptr(), st["d_slots"].data_ptr(), S, nb, bs, hkv,
                                      d, bstride, self._dtype_code, err, sp), "pkv_write_slots")
        fn = L.pkv_decode_attention_items if wl is not None else L.pkv_decode_attention
        _abi._check(fn(out.data_ptr(), query.data_ptr(), kc.data_ptr(), vc.data_ptr(), *args,
                       *tail), "pkv_decode_attention")
        return out

    # -- the three device calls, for either cache type ---------------------
    def _copy(self, pairs, stream):
        if self.fp8:
            _abi.pkv_copy_blocks_fp8(self.key_cache, self.value_cache, self.k_scale,
                                     self.v_scale, pairs, dev_error=self.dev_error,
                                     stream=stream)
        else:
            _abi.pkv_copy_blocks(self.key_cache, self.value_cache, pairs,
                                 dev_error=self.dev_error, stream=stream)

    def _write(self, key, value, slots, stream):
        if self.fp8:
            _abi.pkv_write_slots_fp8(key, value, self.key_cache, self.value_cache, self.k_scale,
                                     self.v_scale, slots, dev_error=self.dev_error,
                                     stream=stream)
        else:
            _abi.pkv_write_slots(key, value, self.key_cache, self.value_cache, slots,
                                 dev_error=self.dev_error, stream=stream)

    def _attend(self, out, query, tables, lens, max_len, ws, stream, work_items=None):
        if self.fp8:
            _abi.pkv_decode_attention_fp8(out, query, self.key_cache, self.value_cache,
                                          self.k_scale, self.v_scale, tables, lens, max_len,
                                          self.scale, self.partition_size, ws,
                                          dev_error=self.dev_error, stream=stream,
                                          work_items=work_items)
        else:
            _abi.pkv_decode_attention(out, query, self.key_cache, self.value_cache, tables,
                                      lens, max_len, self.scale, self.partition_size, ws,
                                      dev_error=self.dev_error, stream=stream,
                                      work_items=work_items)

    def _signature(self, query, key, value, out):
        return tuple((tuple(t.shape), t.dtype, t.device, t.is_contiguous())
                     for t in (query, key, value, out))

    def _checked(self, query, key, value, out):
        return self._signature(query, key, value, out) in self._seen

    def decode_step(self, seq_ids, query, key, value, out=None, stream=None):
        """One full decode step for seq_ids (query [S, Hq, D], key/value
        [S, Hkv, D] on the device).  Returns out [S, Hq, D]."""
        prep = self.prepare_step(seq_ids)
        self.upload_step(prep, stream)
        if out is None:
            out = torch.empty_like(query)
        return self.launch_step(prep, query, key, value, out, stream=stream)

    # -- swapping to pinned host memory -------------------------------------
    def enable_swap(self, num_host_blocks):
        """Host caches of num_host_blocks blocks in pinned memory (and the
        pool's host block stack), for swap_out / swap_in."""
        self.pool.set_host_blocks(num_host_blocks)
        shape = (num_host_blocks,) + tuple(self.key_cache.shape[1:])
        pin = dict(dtype=self.key_cache.dtype, pin_memory=True)
        self.host_key_cache = torch.empty(shape, **pin)
        self.host_value_cache = torch.empty(shape, **pin)
        if self.fp8:
            hs = dict(dtype=torch.float32, pin_memory=True)
            self.host_k_scale = torch.empty((num_host_blocks, self.num_kv_heads), **hs)
            self.host_v_scale = torch.empty((num_host_blocks, self.num_kv_heads), **hs)

    def _swap(self, seq_ids, out, stream):
        fn = self.pool.swap_out if out else self.pool.swap_in
        pairs = [fn(s) for s in seq_ids]
        pairs = torch.cat(pairs) if pairs else torch.empty((0, 2), dtype=torch.int32)
        if pairs.numel() == 0:
            return 0
        s = stream if stream is not None else torch.cuda.current_stream(self.device)
        with torch.cuda.stream(s):
            d_pairs = pairs.pin_memory().to(self.device, non_blocking=True)
        dev = (self.key_cache, self.value_cache)
        host = (self.host_key_cache, self.host_value_cache)
        src, dst = (dev, host) if out else (host, dev)
        _abi.pkv_swap_blocks(src[0], src[1], dst[0], dst[1], d_pairs, dev_error=self.dev_error,
                             stream=s)
        if self.fp8:
            dev = (self.k_scale, self.v_scale)
            host = (self.host_k_scale, self.host_v_scale)
            src, dst = (dev, host) if out else (host, dev)
            _abi.pkv_swap_blocks(src[0], src[1], dst[0], dst[1], d_pairs,
                                 dev_error=self.dev_error, stream=s)
        return int(pairs.shape[0])

    def swap_out(self, seq_ids, stream=None):
        """Moves the sequences' blocks to the host caches ("PagedAttention 动态
        内存分页" page, 动态块分配与回收); their GPU blocks return to the pool.
        Returns the number of blocks moved."""
        return self._swap(seq_ids, True, stream)

    def swap_in(self, seq_ids, stream=None):
        """Brings swapped-out sequences back into (new) GPU blocks.  Returns
        the number of blocks moved."""
        return self._swap(seq_ids, False, stream)

    def check_errors(self):
        """Raises if a kernel recorded bad metadata since the last check."""
        err = self.dev_error.tolist()
        if err[0] != _abi.PKV_DEVERR_NONE:
            self.dev_error.zero_()
            raise _abi.PkvError(_abi.PKV_ERR_INVALID,
                                "device error code %d at index %d" % (err[0], err[1]))
