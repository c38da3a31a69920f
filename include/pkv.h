/*
 * pkv.h — C ABI of the B200 paged KV cache library (libpkv.so).
 *
 * The library implements the data-parallel hot path of PagedAttention as the
 * pages describe it:
 *   - a physical block pool with per-sequence Block Tables, refcounts and
 *     copy-on-write ("Paged KV" wiki page, sections 实现原理 / 初始化阶段 and
 *     运行阶段; "PagedAttention 动态内存分页" page, sections 块粒度与块表,
 *     写时复制与内存共享, 动态块分配与回收);
 *   - the slot-mapped write of each new token's K/V (运行阶段);
 *   - decode attention that reads K/V block by block through the Block Table
 *     ("Paged KV" wiki page, section Attention Kernel 的适配);
 *   - the copy of a shared block before a sequence writes into it.
 *
 * Conventions shared by every entry point
 *   - Every function returns a pkv_status (0 on success) and never throws.
 *     pkv_last_error() gives a message for the calling thread's last failure.
 *   - Device memory is owned by the caller: the library allocates none, and
 *     every pointer it is given stays the caller's.  Kernels run
 *     asynchronously on the caller's stream; a host-side argument error is
 *     reported before anything is launched.
 *   - Cache layout: K and V are separate caches, each a sequence of physical
 *     blocks of shape [block_size, num_kv_heads, head_dim] (contiguous inside
 *     a block), block b starting block_stride ELEMENTS after block 0.  A plain
 *     [num_blocks, block_size, num_kv_heads, head_dim] tensor has
 *     block_stride = block_size * num_kv_heads * head_dim; a combined or
 *     multi-layer tensor passes a larger stride (a multiple of 8 elements).
 *   - A slot is physical_block * block_size + offset.
 *   - dev_error, where taken, is NULL or a device int32[2] that the caller
 *     zeroes; a kernel that meets bad metadata records the first problem as
 *     {code, index} (PKV_DEVERR_*), skips that piece of work and carries on.
 *     No kernel traps.
 *   - Supported: fp16 and bf16 storage; head_dim 64 or 128 for attention
 *     (any multiple of 8 for the write and the copy); block_size a multiple
 *     of 16 up to 256 for attention (any positive size for the write and the
 *     copy); num_q_heads / num_kv_heads from 1 to 16.
 */
#ifndef PKV_H
#define PKV_H

#include <stddef.h>
#include <stdint.h>

#include <cuda_runtime_api.h>

#if defined(__GNUC__)
#define PKV_API __attribute__((visibility("default")))
#else
#define PKV_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    PKV_OK = 0,
    PKV_ERR_INVALID = -1,     /* bad argument: shape, pointer, alignment, id */
    PKV_ERR_UNSUPPORTED = -2, /* valid but not built: dtype, head_dim, ... */
    PKV_ERR_CUDA = -3,        /* a CUDA runtime call or launch failed */
    PKV_ERR_OOM = -4,         /* the block pool has too few free blocks */
    PKV_ERR_WORKSPACE = -5    /* workspace missing or too small */
} pkv_status;

typedef enum { PKV_F16 = 0, PKV_BF16 = 1 } pkv_dtype;

/* The host block pool (opaque; see "Host block pool" below). */
typedef struct pkv_pool pkv_pool;

/* Codes a kernel writes into dev_error[0]; dev_error[1] gets the index. */
#define PKV_DEVERR_NONE 0
#define PKV_DEVERR_CONTEXT_LEN 1 /* index: seq; len < 0, > max_context_len or > table */
#define PKV_DEVERR_BLOCK_ID 2    /* index: seq; a table entry outside [0, num_blocks) */
#define PKV_DEVERR_SLOT 3        /* index: token; slot >= num_blocks * block_size */
#define PKV_DEVERR_PAIR 4        /* index: pair; a block id outside [0, num_blocks) */
#define PKV_DEVERR_TIMEOUT 5     /* index: 0; a bounded wait on a copy ran out */
#define PKV_DEVERR_WORK_ITEM 6   /* index: CTA; a work-list entry outside the grid */

/* ---------------------------------------------------------------------- */
/* Slot write                                                              */
/* ---------------------------------------------------------------------- */
/*
 * Writes the K and V rows of num_tokens new tokens into their slots
 * ("Paged KV" wiki page, 实现原理 / 运行阶段: each decoded token goes to the
 * next slot of the sequence's current block; prefill fills blocks in order).
 *
 *   key, value     device, [num_tokens, num_kv_heads, head_dim], contiguous
 *   key_cache,     device caches in the layout above (num_blocks blocks)
 *   value_cache
 *   slot_mapping   device int64 [num_tokens]; token t goes to block
 *                  slot / block_size, offset slot % block_size; a negative
 *                  slot writes nothing.  Slots must be distinct (else which
 *                  token lands is unspecified).  A slot >= num_blocks *
 *                  block_size is skipped and reported (PKV_DEVERR_SLOT).
 *   All pointers 16-byte aligned; num_kv_heads * head_dim a multiple of 8.
 */
PKV_API int pkv_write_slots(const void* key, const void* value, void* key_cache,
                    void* value_cache, const int64_t* slot_mapping,
                    int num_tokens, int num_blocks, int block_size,
                    int num_kv_heads, int head_dim, int64_t block_stride,
                    pkv_dtype dtype, int32_t* dev_error, cudaStream_t stream);

/* ---------------------------------------------------------------------- */
/* Copy-on-write block copy                                                */
/* ---------------------------------------------------------------------- */
/*
 * For every pair (src, dst), block dst of both caches becomes a copy of
 * block src: all block_size slots of all heads ("PagedAttention 动态内存
 * 分页" page, 写时复制与内存共享: a block shared by several sequences is copied
 * when one of them needs to write into it).
 *
 *   block_pairs  device int32 [num_pairs, 2] = (src, dst).  Pairs run
 *                concurrently: destinations must be distinct and no
 *                destination may be another pair's source.  A pair naming a
 *                block outside [0, num_blocks) is skipped and reported
 *                (PKV_DEVERR_PAIR).
 *   Cache pointers 16-byte aligned, block_stride a multiple of 8 elements.
 */
PKV_API int pkv_copy_blocks(void* key_cache, void* value_cache,
                    const int32_t* block_pairs, int num_pairs, int num_blocks,
                    int block_size, int num_kv_heads, int head_dim,
                    int64_t block_stride, pkv_dtype dtype, int32_t* dev_error,
                    cudaStream_t stream);

/*
 * pkv_copy_blocks over every layer of a multi-layer cache in one launch.  A
 * physical block id names the block in all layers ("Paged KV" wiki page,
 * 初始化阶段: a block holds K and V of every layer), so one copy-on-write
 * pair from the pool is copied in each layer.
 *
 *   key_caches, value_caches  device arrays of num_layers device pointers
 *                (layer l's K and V caches, each 16-byte aligned, all with
 *                the same geometry)
 *   block_pairs  device int32 [num_pairs, 2]; rules and errors as for
 *                pkv_copy_blocks
 *   block_bytes, block_stride_bytes
 *                one block of one cache and the distance between blocks,
 *                in bytes (multiples of 16; any element type, e4m3 too)
 */
PKV_API int pkv_copy_blocks_layers(void* const* key_caches, void* const* value_caches,
                                   int num_layers, const int32_t* block_pairs, int num_pairs,
                                   int num_blocks, int64_t block_bytes,
                                   int64_t block_stride_bytes, int32_t* dev_error,
                                   cudaStream_t stream);

/* ---------------------------------------------------------------------- */
/* Paged decode attention                                                  */
/* ---------------------------------------------------------------------- */
/*
 * Bytes of workspace pkv_decode_attention needs for these sizes (0 when every
 * sequence fits one partition, i.e. partition_size == 0 or
 * partition_size >= max_context_len).  The workspace holds an int32 counter
 * per (sequence, KV head) — cleared by the library on the caller's stream
 * before each launch — and, per (seq, query head, partition), the fp32
 * running maximum, sum and unnormalised output.
 */
PKV_API size_t pkv_decode_workspace_bytes(int num_seqs, int num_q_heads,
                                  int max_context_len, int partition_size,
                                  int head_dim);

/*
 * One decode step of attention for num_seqs sequences, one query token each
 * ("Paged KV" wiki page, Attention Kernel 的适配: besides the usual inputs the
 * kernel takes the Block Table and block_size and reads K/V block by block
 * through that indirection).  For sequence s and query head h, with
 * kv = h / (num_q_heads / num_kv_heads) and L = context_lens[s]:
 *     out[s, h] = sum_t softmax_t(scale * <query[s, h], K_t>) V_t,  t < L,
 * where token t is slot t % block_size of physical block
 * block_tables[s, t / block_size].  L counts every cached token, the one
 * written this step included.  L == 0 gives zeros.
 *
 *   out, query       device [num_seqs, num_q_heads, head_dim], dtype
 *   key_cache,       device caches (layout above); 16-byte aligned
 *   value_cache
 *   block_tables     device int32 [num_seqs, max_blocks_per_seq]; only the
 *                    first ceil(L / block_size) entries of a row are read
 *   context_lens     device int32 [num_seqs]
 *   max_context_len  host copy of max(context_lens) (or any bound on it):
 *                    it sizes the grid; a longer sequence is reported
 *                    (PKV_DEVERR_CONTEXT_LEN) and gets zeros
 *   scale            multiplies the dot product before the softmax
 *   partition_size   0: one pass per sequence.  Otherwise a multiple of 16:
 *                    each sequence is split into partitions of that many
 *                    tokens that run in parallel; the last partition of a
 *                    (sequence, KV head) to finish merges their fp32 partial
 *                    results (split-K for long contexts).  PKV_ERR_UNSUPPORTED
 *                    when a CTA cannot hold the merge of that many
 *                    partitions (group * partitions above ~8000).
 *   workspace        device scratch of pkv_decode_workspace_bytes() bytes,
 *                    16-byte aligned (may be NULL when that is 0); its
 *                    contents on entry and exit are unspecified
 * Returns PKV_ERR_UNSUPPORTED for a head_dim, block_size or group size that
 * is not built, PKV_ERR_WORKSPACE when the workspace is too small.
 */
PKV_API int pkv_decode_attention(void* out, const void* query, const void* key_cache,
                         const void* value_cache, const int32_t* block_tables,
                         int max_blocks_per_seq, const int32_t* context_lens,
                         int num_seqs, int max_context_len, int num_q_heads,
                         int num_kv_heads, int head_dim, int num_blocks,
                         int block_size, int64_t block_stride, float scale,
                         int partition_size, void* workspace,
                         size_t workspace_bytes, pkv_dtype dtype,
                         int32_t* dev_error, cudaStream_t stream);

/* ---------------------------------------------------------------------- */
/* Decode work list: per-sequence partitions, longest first                */
/* ---------------------------------------------------------------------- */
/*
 * The pages note that sequences of very different lengths are what makes a
 * batch costly to schedule ("PagedAttention 动态内存分页" page, 技术边界与取舍).
 * pkv_decode_attention's grid has num_seqs * num_kv_heads * NP slots (NP =
 * partitions of the longest sequence), and slots past a shorter sequence's
 * end exit at once, in grid order.  This host-side planner lists instead
 * the work items that hold tokens: one per (sequence s, KV head, partition
 * p) with p < max(1, ceil(L_s / P)), so a short sequence runs one pass and
 * a long one is split.  Within a sequence the items go partition by
 * partition, the KV heads of a partition side by side (their slices of a
 * block share its memory rows).  order:
 *   PKV_ITEMS_LONGEST_FIRST  by the 16-token tiles each item holds, most
 *                            first (ties as above, sequences in batch
 *                            order): the long items start first and the
 *                            short ones fill the end of the launch
 *   PKV_ITEMS_SEQUENCES_LONGEST_FIRST
 *                            sequences by context length, longest first
 *                            (ties in batch order), each sequence's items
 *                            together
 *   PKV_ITEMS_BATCH_ORDER    sequences in batch order, each sequence's
 *                            items together (sequences next to each other
 *                            in the batch, such as samples sharing a
 *                            prefix, run side by side)
 *
 *   context_lens     HOST int32 [num_seqs]: the same lengths the device
 *                    copy passed to the attention call holds
 *   max_context_len, partition_size
 *                    exactly as they will be passed to the attention call
 *                    (they fix P and NP as pkv_decode_attention does)
 *   items            HOST int32 [capacity]: receives the items, each the
 *                    flat index (s * num_kv_heads + kv_head) * NP + p
 *   num_items        receives the number of items.  When it exceeds
 *                    capacity, nothing is written to items and
 *                    PKV_ERR_INVALID is returned (num_items still set);
 *                    num_kv_heads * sum_s max(1, ceil(L_s / P)) is the count
 *                    and num_seqs * num_kv_heads * NP always suffices.
 * A length outside [0, max_context_len] or an unknown order returns
 * PKV_ERR_INVALID.  Host work only: O(items + P / 16), plus a sort of the
 * sequences for PKV_ITEMS_SEQUENCES_LONGEST_FIRST.
 */
#define PKV_ITEMS_LONGEST_FIRST 0
#define PKV_ITEMS_SEQUENCES_LONGEST_FIRST 1
#define PKV_ITEMS_BATCH_ORDER 2
PKV_API int pkv_decode_work_items(const int32_t* context_lens, int num_seqs, int num_kv_heads,
                                  int max_context_len, int partition_size, int order,
                                  int32_t* items, int capacity, int* num_items);

/*
 * pkv_decode_attention over a work list from pkv_decode_work_items: one
 * CTA per item, in list order.  Every other argument, the result and the
 * errors are those of pkv_decode_attention.
 *   work_items       DEVICE int32 [num_items]: the planner's list for the
 *                    same context lengths, max_context_len and
 *                    partition_size.  An entry outside the grid is reported
 *                    (PKV_DEVERR_WORK_ITEM) and skipped; a list that misses
 *                    an item of a sequence leaves that sequence's output
 *                    unwritten, and one that repeats an item gives an
 *                    unspecified result for that sequence (no access leaves
 *                    the buffers either way).
 *   num_items        0 launches nothing
 */
PKV_API int pkv_decode_attention_items(void* out, const void* query, const void* key_cache,
                                       const void* value_cache, const int32_t* block_tables,
                                       int max_blocks_per_seq, const int32_t* context_lens,
                                       int num_seqs, int max_context_len, int num_q_heads,
                                       int num_kv_heads, int head_dim, int num_blocks,
                                       int block_size, int64_t block_stride, float scale,
                                       int partition_size, void* workspace,
                                       size_t workspace_bytes, const int32_t* work_items,
                                       int num_items, pkv_dtype dtype, int32_t* dev_error,
                                       cudaStream_t stream);

/* ---------------------------------------------------------------------- */
/* One decode step in two calls                                            */
/* ---------------------------------------------------------------------- */
/*
 * The per-step sequence the pages describe ("Paged KV" wiki page, 实现原理 /
 * 运行阶段: take a slot, write the new K/V, attend through the Block Table;
 * "PagedAttention 动态内存分页" page, 写时复制与内存共享: copy a shared block
 * before writing into it), as one host call and one device call.  They
 * compose the entry points above and add no arithmetic: a caller saves the
 * per-call overhead of driving the steps one by one.
 */

/*
 * Host part: pkv_seq_append_batch for the n sequences (slots, cow_pairs,
 * *num_pairs), then pkv_pool_block_tables (block_tables [n,
 * max_blocks_per_seq] padded with -1, context_lens [n], *max_context_len),
 * then, when a work list is wanted, pkv_decode_work_items into work_items
 * (*num_items; -1 when none was made).  order_split is the list's order
 * (PKV_ITEMS_*) when the step splits a sequence into partitions
 * (0 < partition_size < *max_context_len), order_one_pass when it does not;
 * -1 makes no list for that case.  All pointers are host memory.  Errors
 * are those of the three calls; an error in the first leaves the sequences
 * before the failing one appended (as pkv_seq_append_batch does).
 */
PKV_API int pkv_step_prepare(pkv_pool* pool, int n, const int64_t* seq_ids, int64_t* slots,
                             int32_t* cow_pairs, int* num_pairs, int32_t* block_tables,
                             int max_blocks_per_seq, int32_t* context_lens,
                             int* max_context_len, int num_kv_heads, int partition_size,
                             int order_split, int order_one_pass, int32_t* work_items,
                             int items_capacity, int* num_items);

/*
 * Device part, enqueued on `stream` in this order:
 *   0. in_bytes from in_host to in_device (cudaMemcpyAsync; 0 bytes:
 *      none) — typically the step's queries and new key/value rows, which
 *      query, key and value then point into; on meta_stream when that is
 *      set, like step 1;
 *   1. meta_bytes from meta_host to meta_device (cudaMemcpyAsync; pinned
 *      host memory keeps it asynchronous; 0 bytes: none) — typically the
 *      step's slots, pairs, tables, lengths and work list in one buffer,
 *      which the pointers below then point into.  With meta_stream not
 *      NULL the copy goes on meta_stream instead, after meta_stream waits
 *      for meta_after (when not NULL: an event the caller recorded after
 *      the last launch that read meta_device), and `stream` waits for
 *      meta_event, which the call records on meta_stream after the copy.
 *      A copy on the compute stream waits, in the copy engine, behind the
 *      previous step's output copy; on a stream of its own it is done
 *      while the previous step computes;
 *   2. pkv_copy_blocks (or _fp8) of the num_pairs cow_pairs (0: none);
 *   3. pkv_write_slots (or _fp8) of the num_tokens new rows (0: none);
 *   4. pkv_decode_attention (or _fp8), over work_items when that is not
 *      NULL (pkv_decode_attention_items);
 *   5. out_bytes of out to out_host (cudaMemcpyAsync; 0: none).  With
 *      out_stream not NULL the copy goes on out_stream instead: the call
 *      records out_event on `stream` after step 4 and makes out_stream
 *      wait for it, so that the copy overlaps whatever the caller enqueues
 *      next on `stream`.  Both handles are the caller's (out_event an
 *      event it created; PKV_ERR_INVALID when it is NULL); the caller must
 *      not overwrite `out` before the copy has run (wait on an event it
 *      records on out_stream).
 * The cache is e4m3 (the _fp8 calls, block_stride in bytes) when k_scale
 * or v_scale is not NULL.  Every field means what the argument of the same
 * name means in those calls; the key/value rows and queries are
 * [num_tokens | num_seqs, heads, head_dim] in dtype.  A failing part
 * returns its status with the parts before it already enqueued.
 */
typedef struct pkv_decode_step_args {
    const void* meta_host;
    void* meta_device;
    size_t meta_bytes;
    const int32_t* cow_pairs;
    int num_pairs;
    const void* key;
    const void* value;
    const int64_t* slot_mapping;
    int num_tokens;
    void* key_cache;
    void* value_cache;
    float* k_scale;
    float* v_scale;
    int num_blocks;
    int block_size;
    int num_kv_heads;
    int head_dim;
    int64_t block_stride;
    void* out;
    const void* query;
    const int32_t* block_tables;
    int max_blocks_per_seq;
    const int32_t* context_lens;
    int num_seqs;
    int max_context_len;
    int num_q_heads;
    float scale;
    int partition_size;
    void* workspace;
    size_t workspace_bytes;
    const int32_t* work_items;
    int num_items;
    void* out_host;
    size_t out_bytes;
    pkv_dtype dtype;
    int32_t* dev_error;
    cudaStream_t out_stream; /* NULL: the readback goes on `stream` */
    cudaEvent_t out_event;   /* used with out_stream */
    cudaStream_t meta_stream; /* NULL: the uploads go on `stream` */
    cudaEvent_t meta_event;   /* used with meta_stream (PKV_ERR_INVALID when NULL) */
    cudaEvent_t meta_after;   /* optional, with meta_stream */
    const void* in_host;      /* step 0: pinned host source */
    void* in_device;          /* step 0: device destination */
    size_t in_bytes;          /* 0: no input upload */
} pkv_decode_step_args;

PKV_API int pkv_decode_step(const pkv_decode_step_args* args, cudaStream_t stream);

/* ---------------------------------------------------------------------- */
/* Paged prefill attention                                                 */
/* ---------------------------------------------------------------------- */
/*
 * Causal attention of a prompt (or a later chunk of one) over the paged
 * cache ("Paged KV" wiki page, 实现原理 / 运行阶段: prefill takes blocks in
 * order and fills them with the prompt's K/V — pkv_write_slots with the
 * prompt's slots — and its tokens then attend through the same Block
 * Table).  Sequence s owns query rows query_start[s] .. query_start[s+1]-1,
 * n_s of them: the last n_s of its L = context_lens[s] cached tokens.  Row
 * query_start[s] + i is token p = L - n_s + i, and for each query head h
 * (KV head h / (num_q_heads / num_kv_heads)):
 *     out[row, h] = sum_{t <= p} softmax_t(scale * <query[row, h], K_t>) V_t.
 *
 *   out, query       device [total rows, num_q_heads, head_dim], dtype
 *   block_tables     device int32 [num_seqs, max_blocks_per_seq]
 *   context_lens     device int32 [num_seqs]: L, the chunk's tokens included
 *   query_start      device int32 [num_seqs + 1], non-decreasing from 0
 *   max_query_len    host bound on every n_s: it sizes the list of 256-row
 *                    tiles that the kernel's persistent CTAs (one per SM) walk
 *   scale            > 0 (PKV_ERR_INVALID otherwise)
 * A sequence with n_s > L, n_s > max_query_len or L > max_blocks_per_seq *
 * block_size is reported (PKV_DEVERR_CONTEXT_LEN) and its rows are left
 * unwritten.  Built for head_dim 128 and block_size a multiple of 16;
 * f16 or bf16.  Caches 16-byte aligned, block_stride in elements.
 */
PKV_API int pkv_prefill_attention(void* out, const void* query, const void* key_cache,
                                  const void* value_cache, const int32_t* block_tables,
                                  int max_blocks_per_seq, const int32_t* context_lens,
                                  const int32_t* query_start, int num_seqs, int max_query_len,
                                  int num_q_heads, int num_kv_heads, int head_dim,
                                  int num_blocks, int block_size, int64_t block_stride,
                                  float scale, pkv_dtype dtype, int32_t* dev_error,
                                  cudaStream_t stream);

/*
 * Scratch built into the library for pkv_decode_attention_noalloc: the
 * largest workspace (as pkv_decode_workspace_bytes counts it) that entry
 * point accepts.
 */
#define PKV_NOALLOC_WORKSPACE_BYTES (64u << 20) /* 64 MiB */

/*
 * pkv_decode_attention for callers that cannot allocate device memory.
 * The pages have no counterpart to this entry point: it exists for callers
 * that are not allowed to call cudaMalloc, or that have no spare memory to
 * give — for example a host framework whose allocator reserves the whole
 * device and forbids plug-ins from allocating, or a latency-bound loop that
 * must not pay for an allocation.  Arguments, results and errors are those
 * of pkv_decode_attention without `workspace` / `workspace_bytes`: the
 * caller still passes every input and output, and the split-K scratch comes
 * from a device array built into the library.
 *
 *   - The array is PKV_NOALLOC_WORKSPACE_BYTES long and lives on every GPU
 *     where this entry point has been called, until the process exits.
 *     With CUDA_MODULE_LOADING=EAGER it lives on every GPU whose context
 *     loads the library, called or not.  A call whose sizes need more (see
 *     pkv_decode_workspace_bytes) returns PKV_ERR_WORKSPACE and launches
 *     nothing.
 *   - The first call on a device with num_seqs > 0 (split-K or not) looks
 *     up that device's copy of the array (cudaGetSymbolAddress) and keeps
 *     the address, keyed by the device's CUDA context; make that first
 *     call before any stream capture.  A context made anew on the device
 *     (after cudaDeviceReset, say) is looked up again at its first call.
 *   - Nothing here allocates: no cudaMalloc, no cudaFree, no allocating
 *     library routine.
 *   - Every call on a device shares the one array, which keeps whatever the
 *     last call left in it (the kernels write every entry they read, so no
 *     clearing is needed).  Calls that overlap on the GPU — on different
 *     streams, or from different host threads — race on it: serialise them.
 */
PKV_API int pkv_decode_attention_noalloc(void* out, const void* query, const void* key_cache,
                                         const void* value_cache, const int32_t* block_tables,
                                         int max_blocks_per_seq, const int32_t* context_lens,
                                         int num_seqs, int max_context_len, int num_q_heads,
                                         int num_kv_heads, int head_dim, int num_blocks,
                                         int block_size, int64_t block_stride, float scale,
                                         int partition_size, pkv_dtype dtype,
                                         int32_t* dev_error, cudaStream_t stream);

/* ---------------------------------------------------------------------- */
/* FP8 (e4m3) caches with a scale per (block, KV head)                     */
/* ---------------------------------------------------------------------- */
/*
 * A quantised cache ("Paged KV" wiki page, 局限性: KV FP8 with a scale per
 * block).  Each cache holds one byte per value, an OCP e4m3 code (bias 7,
 * finite up to 448, no infinities, 0x7f/0xff are NaN), in the layout above
 * with block_stride counted in BYTES (a multiple of 16).  Block b, KV head h
 * has one scale per cache, k_scale[b * num_kv_heads + h] and
 * v_scale[b * num_kv_heads + h] (device fp32, 16-byte aligned, at least
 * num_blocks * num_kv_heads floats rounded up to a multiple of 4).  A code c
 * stands for the value e4m3(c) * scale.  Scales are positive and finite.
 * The caller sets a block's scales before the block's first write and keeps
 * them while the block holds tokens; the library reads them and copies them
 * with the block.
 */

/*
 * pkv_write_slots into an e4m3 cache: value x of token t (f16 or bf16 per
 * dtype, the type of key/value) is stored as the e4m3 code nearest to the
 * fp32 quotient x / scale (round to nearest, ties to the even code; beyond
 * 448 in magnitude it saturates to +-448; NaN stays NaN), scale being the
 * destination block's scale for that KV head.  Slot rules, alignment and
 * errors are those of pkv_write_slots; num_kv_heads * head_dim a multiple
 * of 8.
 */
PKV_API int pkv_write_slots_fp8(const void* key, const void* value, void* key_cache,
                                void* value_cache, const float* k_scale, const float* v_scale,
                                const int64_t* slot_mapping, int num_tokens, int num_blocks,
                                int block_size, int num_kv_heads, int head_dim,
                                int64_t block_stride, pkv_dtype dtype, int32_t* dev_error,
                                cudaStream_t stream);

/*
 * pkv_copy_blocks for e4m3 caches: block dst of both caches becomes a copy of
 * block src, bytes and scales (k_scale and v_scale rows of dst take src's).
 * Pair rules and errors are those of pkv_copy_blocks; the block's bytes
 * (block_size * num_kv_heads * head_dim) a multiple of 16.
 */
PKV_API int pkv_copy_blocks_fp8(void* key_cache, void* value_cache, float* k_scale,
                                float* v_scale, const int32_t* block_pairs, int num_pairs,
                                int num_blocks, int block_size, int num_kv_heads, int head_dim,
                                int64_t block_stride, int32_t* dev_error, cudaStream_t stream);

/*
 * pkv_decode_attention over e4m3 caches: K_t and V_t are the dequantised
 * rows (code * scale of the token's block and KV head); query and out keep
 * dtype (f16 or bf16).  Built for head_dim 128 and block_size a multiple of
 * 16 (the kernel's tile is 16 slots of one block); the other arguments,
 * the workspace (pkv_decode_workspace_bytes) and errors are those of
 * pkv_decode_attention.
 */
PKV_API int pkv_decode_attention_fp8(void* out, const void* query, const void* key_cache,
                                     const void* value_cache, const float* k_scale,
                                     const float* v_scale, const int32_t* block_tables,
                                     int max_blocks_per_seq, const int32_t* context_lens,
                                     int num_seqs, int max_context_len, int num_q_heads,
                                     int num_kv_heads, int head_dim, int num_blocks,
                                     int block_size, int64_t block_stride, float scale,
                                     int partition_size, void* workspace,
                                     size_t workspace_bytes, pkv_dtype dtype,
                                     int32_t* dev_error, cudaStream_t stream);

/*
 * pkv_decode_attention_fp8 over a work list from pkv_decode_work_items
 * (work_items and num_items as in pkv_decode_attention_items).
 */
PKV_API int pkv_decode_attention_fp8_items(void* out, const void* query, const void* key_cache,
                                           const void* value_cache, const float* k_scale,
                                           const float* v_scale, const int32_t* block_tables,
                                           int max_blocks_per_seq, const int32_t* context_lens,
                                           int num_seqs, int max_context_len, int num_q_heads,
                                           int num_kv_heads, int head_dim, int num_blocks,
                                           int block_size, int64_t block_stride, float scale,
                                           int partition_size, void* workspace,
                                           size_t workspace_bytes, const int32_t* work_items,
                                           int num_items, pkv_dtype dtype, int32_t* dev_error,
                                           cudaStream_t stream);

/* ---------------------------------------------------------------------- */
/* Host block pool (allocator)                                             */
/* ---------------------------------------------------------------------- */
/*
 * One global pool of num_blocks physical blocks, from which sequences take
 * blocks on demand and to which they return them ("一文读懂vLLM的…
 * PagedAttention" page, 运行模式的根本转变; "Paged KV" wiki page, 初始化阶段
 * and 运行阶段; "PagedAttention 动态内存分页" page, 块粒度与块表, 写时复制与内存
 * 共享, 动态块分配与回收).  Policy where the pages are silent: the free pool is a
 * LIFO stack; a fresh pool hands out free_order[0], free_order[1], ... (or
 * 0, 1, ... when free_order is NULL); freed blocks are pushed in table order;
 * an operation that runs out of blocks returns PKV_ERR_OOM and changes
 * nothing.  Not thread-safe: the caller serialises calls on one pool.
 * All pointers here are host pointers.  (pkv_pool is declared at the top.)
 */

/* free_order: NULL or a permutation of 0..num_blocks-1 (host int32). */
PKV_API int pkv_pool_create(int num_blocks, int block_size, const int32_t* free_order,
                    pkv_pool** out);
PKV_API void pkv_pool_destroy(pkv_pool* pool);

/* Prefill: a new sequence of num_tokens tokens takes ceil(num_tokens /
 * block_size) blocks in pool order.  PKV_ERR_INVALID if seq_id exists. */
PKV_API int pkv_seq_add(pkv_pool* pool, int64_t seq_id, int num_tokens);

/* The child shares every block of the parent (refcount + 1 each). */
PKV_API int pkv_seq_fork(pkv_pool* pool, int64_t parent, int64_t child);

/* Reserves the slot of one new token of seq_id.  When the current block is
 * full a new block is appended to the table.  When the current block is
 * shared (refcount > 1) it is replaced by a fresh block, *cow_src / *cow_dst
 * receive the pair to copy with pkv_copy_blocks before the write, and the
 * old block loses one reference; otherwise both are set to -1. */
PKV_API int pkv_seq_append(pkv_pool* pool, int64_t seq_id, int64_t* slot,
                   int32_t* cow_src, int32_t* cow_dst);

/* pkv_seq_append for n sequences in order.  slots[i] receives the slot of
 * seq_ids[i]; the copy pairs are packed into cow_pairs (capacity n pairs,
 * int32 [n, 2]) and counted in *num_cow.  Stops at the first failure, with
 * *num_done (may be NULL) appends completed. */
PKV_API int pkv_seq_append_batch(pkv_pool* pool, int n, const int64_t* seq_ids,
                         int64_t* slots, int32_t* cow_pairs, int* num_cow,
                         int* num_done);

/* Drops the sequence's reference to each of its blocks; blocks that reach
 * refcount 0 return to the pool. */
PKV_API int pkv_seq_free(pkv_pool* pool, int64_t seq_id);

PKV_API int pkv_seq_num_tokens(const pkv_pool* pool, int64_t seq_id, int* num_tokens);

/* Slots of tokens [first_token, first_token + num_tokens) of the sequence, in
 * order, into out (host int64): slot = table[t / block_size] * block_size +
 * t % block_size.  The range must lie inside the sequence.  Used to write a
 * prompt's K/V after pkv_seq_add ("Paged KV" wiki page, 运行阶段: prefill
 * fills the blocks it took, in order). */
PKV_API int pkv_seq_slot_mapping(const pkv_pool* pool, int64_t seq_id, int first_token,
                                 int num_tokens, int64_t* out);

/* Copies the sequence's Block Table (physical ids in logical order) into
 * out[0..cap); *n receives its length (PKV_ERR_INVALID if cap < length). */
PKV_API int pkv_seq_block_table(const pkv_pool* pool, int64_t seq_id, int32_t* out,
                        int cap, int* n);

/* Fills a dense [n, max_blocks_per_seq] table for seq_ids (rows padded with
 * `fill`), and, where the pointers are not NULL, their token counts and the
 * largest of them. */
PKV_API int pkv_pool_block_tables(const pkv_pool* pool, int n, const int64_t* seq_ids,
                          int32_t* out, int max_blocks_per_seq, int32_t fill,
                          int32_t* context_lens, int32_t* max_context_len);

/* Free blocks, total blocks and block size of the pool (negative status on
 * a NULL pool). */
PKV_API int pkv_pool_num_free(const pkv_pool* pool);
PKV_API int pkv_pool_num_blocks(const pkv_pool* pool);
PKV_API int pkv_pool_block_size(const pkv_pool* pool);

/* The free stack from bottom to top (the next block taken is the last). */
PKV_API int pkv_pool_free_list(const pkv_pool* pool, int32_t* out, int cap, int* n);

/* Refcount of a block (number of tables holding it), or a negative status. */
PKV_API int pkv_block_refcount(const pkv_pool* pool, int block);

/* ---------------------------------------------------------------------- */
/* Block swapping to pinned host memory                                    */
/* ---------------------------------------------------------------------- */
/*
 * When GPU memory runs short, a sequence's KV blocks can move to CPU memory
 * and come back when it runs again ("PagedAttention 动态内存分页" page,
 * 动态块分配与回收; 性能监控要点 names the swap bandwidth as a figure to
 * watch).  The pool keeps a second stack of host block ids; the caller owns
 * the host caches those ids index (pinned, e.g. cudaHostAlloc) and moves the
 * bytes with pkv_swap_blocks.
 *
 * Rules: a swap moves one whole sequence, in table order.  Swap-out gives
 * each block a host block (pair (gpu, host)) and then drops the sequence's
 * reference to the GPU block, which returns to the pool at refcount 0 (a
 * block still shared with a resident sequence stays for it).  Swap-in gives
 * each host block a GPU block (pair (host, gpu)) and returns the host block.
 * Either one that runs out of blocks changes nothing (PKV_ERR_OOM).  While
 * swapped out, a sequence cannot be appended to, forked, or listed by
 * pkv_pool_block_tables / pkv_seq_slot_mapping (PKV_ERR_INVALID);
 * pkv_seq_block_table lists its host blocks; pkv_seq_free returns them.
 */

/* Makes the host pool (once): host blocks 0 .. num_host_blocks-1, handed out
 * 0, 1, ... first, freed blocks reused last-in first-out. */
PKV_API int pkv_pool_set_host_blocks(pkv_pool* pool, int num_host_blocks);

/* Swap-out of a resident sequence.  pairs (host int32, capacity cap pairs)
 * receives (gpu block, host block) per block in table order, *num_pairs
 * their count (PKV_ERR_INVALID, nothing changed, if cap is too small). */
PKV_API int pkv_seq_swap_out(pkv_pool* pool, int64_t seq_id, int32_t* pairs, int cap,
                             int* num_pairs);

/* Swap-in of a swapped-out sequence: pairs receives (host block, gpu block). */
PKV_API int pkv_seq_swap_in(pkv_pool* pool, int64_t seq_id, int32_t* pairs, int cap,
                            int* num_pairs);

/* *swapped = 1 while the sequence's blocks are on the host, else 0. */
PKV_API int pkv_seq_is_swapped(const pkv_pool* pool, int64_t seq_id, int* swapped);

/* Free host blocks (negative status on a NULL pool; 0 without a host pool). */
PKV_API int pkv_pool_num_free_host(const pkv_pool* pool);

/* The host free stack from bottom to top (the next block taken is the last). */
PKV_API int pkv_pool_host_free_list(const pkv_pool* pool, int32_t* out, int cap, int* n);

/* Refcount of a host block (1 while a swapped sequence holds it, else 0). */
PKV_API int pkv_host_block_refcount(const pkv_pool* pool, int block);

/*
 * Copies whole blocks from one pool to another: for each pair (src, dst),
 * block dst of dst_key (and dst_value) becomes block src of src_key (and
 * src_value).  One side is the GPU cache, the other a host cache in pinned
 * memory mapped for the device (cudaHostAlloc; the library passes the
 * kernel the mapping cudaPointerGetAttributes reports).  Swap-out copies
 * GPU -> host with the pairs of pkv_seq_swap_out, swap-in host -> GPU with
 * those of pkv_seq_swap_in.  The kernel reads or writes host memory over
 * the host link directly, one launch for all pairs.
 *
 *   src_value, dst_value  both NULL to copy one pool (e.g. the fp32 scales
 *                  of an e4m3 cache: block_bytes = num_kv_heads * 4)
 *   block_pairs    int32 [num_pairs, 2] in device memory or mapped pinned
 *                  host memory.  Pairs run concurrently: destinations
 *                  distinct.  A pair outside [0, src_num_blocks) x
 *                  [0, dst_num_blocks) is skipped and reported
 *                  (PKV_DEVERR_PAIR).
 *   block_bytes, src_block_stride, dst_block_stride
 *                  in bytes, multiples of 4 (16-byte vectors are used when
 *                  every pointer, size and stride allows)
 * Pageable host memory, or host memory without a device mapping, is
 * rejected (PKV_ERR_INVALID) before anything is launched.
 */
PKV_API int pkv_swap_blocks(const void* src_key, const void* src_value, void* dst_key,
                            void* dst_value, const int32_t* block_pairs, int num_pairs,
                            int src_num_blocks, int dst_num_blocks, int64_t block_bytes,
                            int64_t src_block_stride, int64_t dst_block_stride,
                            int32_t* dev_error, cudaStream_t stream);

/* ---------------------------------------------------------------------- */
/* Sizing and diagnostics                                                  */
/* ---------------------------------------------------------------------- */
/* Bytes of one physical block over all layers ("Paged KV" wiki page,
 * 初始化阶段): block_size * num_kv_heads * head_dim * 2 (K and V) *
 * num_layers * dtype_bytes.  Negative on bad arguments. */
PKV_API int64_t pkv_block_bytes(int block_size, int num_kv_heads, int head_dim,
                        int num_layers, int dtype_bytes);

/* Self-test of the kernels' failure path: launches one CTA that waits, with
 * the same bounded wait the attention kernel uses, on an mbarrier that never
 * completes.  After limit_us microseconds (1 .. 10^6) the wait gives up and
 * records {PKV_DEVERR_TIMEOUT, 0} in dev_error (device int32[2], zeroed by
 * the caller); the context stays usable.  No other kernel waits are
 * affected. */
PKV_API int pkv_selftest_bounded_wait(int32_t* dev_error, int limit_us, cudaStream_t stream);

/* Self-test of the 2^x that the prefill softmax takes from the FMA pipe for
 * part of its exponentials (its own arithmetic; the pages give no
 * exponential): y[i] = 2^x[i] for n fp32 values, x and y device arrays of n
 * floats (0 <= n <= 2^28), launched on stream.  Within 3.0e-6 relative for
 * x in [-126, 8]; +0 for x <= -127, -inf and NaN; subnormal below 2^-126
 * for x in (-127, -126). */
PKV_API int pkv_selftest_ex2_poly(const float* x, float* y, int n, cudaStream_t stream);

PKV_API const char* pkv_status_string(int status);
/* Message of the calling thread's last failed call ("" if none). */
PKV_API const char* pkv_last_error(void);
/* Library version as major * 10000 + minor * 100 + patch. */
PKV_API int pkv_version(void);

#ifdef __cplusplus
}
#endif
#endif /* PKV_H */
