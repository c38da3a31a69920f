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
import ctypes as C

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
        sequences longest first (the order measured fastest on B200 for the
        GQA batches, 16-bit and e4m3, and level with the others on the
        long-context batches); "longest_first",
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
            s = stream if stream is not None else torch.cuda.current_stream(self.device)
            with torch.cuda.stream(s):  # the slots go up on the stream that writes them
                slots = self.pool.slot_mapping(seq_id, 0, num_tokens).to(self.device)
            self._write(key, value, slots, s)

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
        previous upload is in flight.  Each bank keeps the step arguments
        (pkv_decode_step_args) whose pointers into it do not change."""
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
                ids = torch.empty(n, dtype=torch.int64)
                hv, dv = views(h), views(d)
                bank = dict(ids=ids, h=h, d=d, h_slots=hv["slots"], h_lens=hv["lens"],
                            h_pairs=hv["pairs"], h_tables=hv["tables"], h_items=hv["items"],
                            d_slots=dv["slots"], d_lens=dv["lens"], d_pairs=dv["pairs"],
                            d_tables=dv["tables"], d_items=dv["items"], items_off=i0,
                            items_cap=cap, uploaded=None, consumed=None, stream=None)
                # host pointers of the bank for pkv_step_prepare
                bank["prep_ptrs"] = (ids.data_ptr(), hv["slots"].data_ptr(),
                                     hv["pairs"].data_ptr(), hv["tables"].data_ptr(),
                                     hv["lens"].data_ptr(), hv["items"].data_ptr())
                bank["args"] = self._step_args(bank, n)
                banks.append(bank)
            self._staging[n] = banks = [banks, 0]
        banks[1] ^= 1
        return banks[0][banks[1]]

    def _step_args(self, bank, n):
        """pkv_decode_step_args with every field that stays fixed for a bank."""
        a = _abi.DecodeStepArgs()
        nb, bs, hkv, d, bstride = self._geom
        a.meta_host, a.meta_device = bank["h"].data_ptr(), bank["d"].data_ptr()
        a.cow_pairs, a.slot_mapping = bank["d_pairs"].data_ptr(), bank["d_slots"].data_ptr()
        a.key_cache, a.value_cache = self.key_cache.data_ptr(), self.value_cache.data_ptr()
        if self.fp8:
            a.k_scale, a.v_scale = self.k_scale.data_ptr(), self.v_scale.data_ptr()
        a.num_blocks, a.block_size, a.num_kv_heads, a.head_dim = nb, bs, hkv, d
        a.block_stride = bstride
        a.block_tables, a.max_blocks_per_seq = bank["d_tables"].data_ptr(), self.max_blocks_per_seq
        a.context_lens, a.num_seqs, a.num_tokens = bank["d_lens"].data_ptr(), n, n
        a.num_q_heads, a.scale, a.partition_size = (self.num_q_heads, float(self.scale),
                                                    int(self.partition_size))
        a.dtype, a.dev_error = self._dtype_code, self.dev_error.data_ptr()
        return a

    def _orders(self):
        """(order when the step splits sequences, order when it does not) for
        pkv_step_prepare; -1: no work list."""
        if not self.work_list:
            return -1, -1
        if self._item_order is None:  # "auto"
            return _abi.PKV_ITEMS_SEQUENCES_LONGEST_FIRST, -1
        return self._item_order, self._item_order

    def prepare_step(self, seq_ids):
        """Host part of a decode step (pkv_step_prepare): reserve one slot per
        sequence (new blocks and copy-on-write pairs as needed), gather the
        Block Tables and lengths into pinned memory and plan the work list.
        Returns the prepared step."""
        st = self._stage(len(seq_ids))
        if st["uploaded"] is not None:
            st["uploaded"].synchronize()  # this bank's last upload has left
        if st.get("ids_src") is not seq_ids:  # a new id list: convert it once
            st["ids"].copy_(torch.as_tensor(seq_ids, dtype=torch.int64))
            st["ids_src"] = seq_ids
        ids, slots, pairs, tables, lens, items = st["prep_ptrs"]
        npairs, longest, nitems = C.c_int(), C.c_int(), C.c_int()
        split, one = self._orders()
        _abi._check(_abi.lib().pkv_step_prepare(
            self.pool._h, len(seq_ids), ids, slots, pairs, C.byref(npairs), tables,
            self.max_blocks_per_seq, lens, C.byref(longest), self.num_kv_heads,
            int(self.partition_size), split, one, items, st["items_cap"], C.byref(nitems)),
            "pkv_step_prepare")
        return dict(st=st, num_pairs=npairs.value, max_len=longest.value,
                    num_items=nitems.value)

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

    def _check_step_tensors(self, query, key, value, out, out_host):
        """The binding's checks, once per set of shapes, dtypes and devices."""
        sig = self._signature(query, key, value, out) + (
            None if out_host is None else (tuple(out_host.shape), out_host.dtype,
                                           out_host.is_pinned()),)
        if sig in self._seen:
            return
        S = query.shape[0]
        _abi._on_device("decode step", query, key, value, out)
        if query.device != self.device:
            raise ValueError("decode step: tensors must be on the cache's device")
        want = {"query": (query, (S, self.num_q_heads, self.head_dim)),
                "key": (key, (S, self.num_kv_heads, self.head_dim)),
                "value": (value, (S, self.num_kv_heads, self.head_dim)),
                "out": (out, (S, self.num_q_heads, self.head_dim))}
        for name, (t, shape) in want.items():
            if tuple(t.shape) != shape or t.dtype != self.dtype or not t.is_contiguous():
                raise ValueError("decode step: %s must be a contiguous %s tensor of shape %s"
                                 % (name, self.dtype, shape))
        if out_host is not None and (out_host.device.type != "cpu" or
                                     out_host.shape != out.shape or
                                     out_host.dtype != out.dtype or
                                     not out_host.is_contiguous()):
            raise ValueError("decode step: out_host must be a host copy of out's shape")
        self._seen.add(sig)

    def run_step(self, prep, query, key, value, out, out_host=None, stream=None,
                 readback_stream=None, upload_stream=None, inputs=None):
        """Device part of a prepared decode step in one native call
        (pkv_decode_step): the metadata upload, the copy-on-write copies, the
        slot write, decode attention and, with out_host (pinned host memory
        for an asynchronous copy), the output's copy to the host.  All on
        `stream` (the current stream by default), except the output's copy
        when readback_stream is given: it then runs there once the attention
        is done, overlapping what comes next on `stream`.  The caller reads
        out_host, and writes `out` again, only after that copy (an event
        recorded on readback_stream after this call).  With upload_stream,
        the metadata upload goes there (after the last launch that read this
        staging bank) and `stream` waits for it: on the compute stream it
        would wait in the copy engine behind the previous step's readback,
        on a stream of its own it lands while the previous step computes.
        inputs=(host, device): a pinned host tensor copied into a device
        tensor of the same size first (on upload_stream when given), e.g.
        the step's query, key and value rows, which query, key and value
        then view; the copy waits, like the metadata's, for the last launch
        that read this staging bank, so the caller alternates its input
        buffers as the banks alternate (one per step, two of them)."""
        st = prep["st"]
        S = len(st["ids"])
        self._check_step_tensors(query, key, value, out, out_host)
        s_ = stream if stream is not None else torch.cuda.current_stream(self.device)
        if st["consumed"] is not None and st["stream"] is not s_:
            s_.wait_event(st["consumed"])  # a launch on another stream read this bank
        a = st["args"]
        items = prep.get("num_items", -1)
        a.meta_bytes = 4 * (st["items_off"] + max(items, 0))
        a.num_pairs = prep["num_pairs"]
        a.key, a.value, a.query, a.out = (key.data_ptr(), value.data_ptr(), query.data_ptr(),
                                          out.data_ptr())
        a.max_context_len = prep["max_len"]
        ws = self.workspace(S, prep["max_len"])
        a.workspace, a.workspace_bytes = (ws.data_ptr(), ws.numel()) if ws is not None else (
            None, 0)
        a.work_items = st["d_items"].data_ptr() if items >= 0 else None
        a.num_items = max(items, 0)
        if out_host is not None:
            a.out_host, a.out_bytes = out_host.data_ptr(), out.numel() * out.element_size()
        else:
            a.out_host, a.out_bytes = None, 0
        a.out_stream, a.out_event = None, None
        a.meta_stream, a.meta_event, a.meta_after = None, None, None
        a.in_host, a.in_device, a.in_bytes = None, None, 0
        if inputs is not None:
            h, d = inputs
            nbytes = d.numel() * d.element_size()
            key_ = ("inputs", h.data_ptr(), d.data_ptr(), nbytes)
            if key_ not in self._seen:  # checked once per pair of buffers
                if (h.device.type != "cpu" or not h.is_pinned() or not h.is_contiguous() or
                        d.device != self.device or not d.is_contiguous() or
                        h.numel() * h.element_size() != nbytes):
                    raise ValueError("decode step: inputs must be a pinned host tensor and a "
                                     "contiguous device tensor of the same size")
                self._seen.add(key_)
            a.in_host, a.in_device, a.in_bytes = h.data_ptr(), d.data_ptr(), nbytes
        if upload_stream is not None and (a.meta_bytes > 0 or a.in_bytes > 0):
            if st.get("meta_up") is None:
                st["meta_up"] = torch.cuda.Event()
                st["meta_up"].record(upload_stream)  # the handle exists once recorded
            a.meta_stream = upload_stream.cuda_stream
            a.meta_event = st["meta_up"].cuda_event
            if st["consumed"] is not None:
                a.meta_after = st["consumed"].cuda_event
        if out_host is not None and readback_stream is not None:
            if st.get("attended") is None:
                st["attended"] = torch.cuda.Event()
                st["attended"].record(s_)  # the handle exists once recorded
            a.out_stream = readback_stream.cuda_stream
            a.out_event = st["attended"].cuda_event
        _abi._check(_abi.lib().pkv_decode_step(C.byref(a), C.c_void_p(s_.cuda_stream)),
                    "pkv_decode_step")
        for ev in ("uploaded", "consumed"):
            if st[ev] is None:
                st[ev] = torch.cuda.Event()
            st[ev].record(s_)
        st["stream"] = s_
        return out

    def launch_step(self, prep, query, key, value, out, max_len=None, stream=None):
        """Device part of a decode step (copy, write, attention) with the
        prepared metadata uploaded by upload_step (on this or another
        stream: the launch waits for it)."""
        st = prep["st"]
        s_ = stream if stream is not None else torch.cuda.current_stream(self.device)
        if st["uploaded"] is not None:
            s_.wait_event(st["uploaded"])
        if max_len is not None and max_len != prep["max_len"]:
            # the work list was planned for the prepared bound: the full grid
            prep = dict(prep, max_len=max_len, num_items=-1)
        self._check_step_tensors(query, key, value, out, None)
        a = st["args"]
        items = prep.get("num_items", -1)
        a.meta_bytes = 0
        a.num_pairs = prep["num_pairs"]
        a.key, a.value, a.query, a.out = (key.data_ptr(), value.data_ptr(), query.data_ptr(),
                                          out.data_ptr())
        a.max_context_len = prep["max_len"]
        ws = self.workspace(len(st["ids"]), prep["max_len"])
        a.workspace, a.workspace_bytes = (ws.data_ptr(), ws.numel()) if ws is not None else (
            None, 0)
        a.work_items = st["d_items"].data_ptr() if items >= 0 else None
        a.num_items = max(items, 0)
        a.out_host, a.out_bytes = None, 0
        a.out_stream, a.out_event = None, None
        a.meta_stream, a.meta_event, a.meta_after = None, None, None
        a.in_host, a.in_device, a.in_bytes = None, None, 0
        _abi._check(_abi.lib().pkv_decode_step(C.byref(a), C.c_void_p(s_.cuda_stream)),
                    "pkv_decode_step")
        if st["consumed"] is None:
            st["consumed"] = torch.cuda.Event()
        st["consumed"].record(s_)
        st["stream"] = s_
        return out

    # -- single device calls, for either cache type ---------------------------
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

    def decode_step(self, seq_ids, query, key, value, out=None, stream=None):
        """One full decode step for seq_ids (query [S, Hq, D], key/value
        [S, Hkv, D] on the device).  Returns out [S, Hq, D]."""
        prep = self.prepare_step(seq_ids)
        if out is None:
            out = torch.empty_like(query)
        return self.run_step(prep, query, key, value, out, stream=stream)

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
