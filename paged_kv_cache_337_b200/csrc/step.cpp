// step.cpp — one decode step in two calls: the host part (the pool's slot
// appends, the Block Tables and lengths, the work list) and the device part
// (metadata upload, copy-on-write copies, slot write, decode attention, the
// output's copy to the host), each one pass over the library's own entry
// points ("Paged KV" wiki page, 实现原理 / 运行阶段: append, write, attend;
// "PagedAttention 动态内存分页" page, 写时复制与内存共享).  They hold no
// arithmetic of their own; they save a caller the per-call overhead of
// driving the steps one by one.
#include <cuda_runtime.h>

#include "internal.h"

extern "C" int pkv_step_prepare(pkv_pool* pool, int n, const int64_t* seq_ids, int64_t* slots,
                                int32_t* cow_pairs, int* num_pairs, int32_t* block_tables,
                                int max_blocks_per_seq, int32_t* context_lens,
                                int* max_context_len, int num_kv_heads, int partition_size,
                                int order_split, int order_one_pass, int32_t* work_items,
                                int items_capacity, int* num_items) {
    PKV_NVTX_RANGE("pkv_step_prepare");
    PKV_REQUIRE(num_pairs && max_context_len && num_items, PKV_ERR_INVALID,
                "pkv_step_prepare: NULL count");
    *num_pairs = 0;
    *max_context_len = 0;
    *num_items = -1;
    int done = 0;
    int st = pkv_seq_append_batch(pool, n, seq_ids, slots, cow_pairs, num_pairs, &done);
    if (st != PKV_OK) return st;
    int32_t longest = 0;
    st = pkv_pool_block_tables(pool, n, seq_ids, block_tables, max_blocks_per_seq, -1,
                               context_lens, &longest);
    if (st != PKV_OK) return st;
    *max_context_len = longest;
    const bool split = partition_size > 0 && partition_size < longest;
    const int order = split ? order_split : order_one_pass;
    if (order < 0 || n == 0) return PKV_OK;  // the full grid
    return pkv_decode_work_items(context_lens, n, num_kv_heads, longest, partition_size, order,
                                 work_items, items_capacity, num_items);
}

extern "C" int pkv_decode_step(const pkv_decode_step_args* a, cudaStream_t stream) {
    PKV_NVTX_RANGE("pkv_decode_step");
    PKV_REQUIRE(a != nullptr, PKV_ERR_INVALID, "pkv_decode_step: NULL arguments");
    const bool fp8 = a->k_scale != nullptr || a->v_scale != nullptr;
    cudaError_t e;
    // steps 0 and 1: the uploads, on meta_stream when the caller gives one
    const bool uploads = a->in_bytes > 0 || a->meta_bytes > 0;
    cudaStream_t us = stream;
    if (uploads && a->meta_stream != nullptr) {
        PKV_REQUIRE(a->meta_event != nullptr, PKV_ERR_INVALID,
                    "pkv_decode_step: meta_stream without meta_event");
        us = a->meta_stream;
        e = a->meta_after != nullptr ? cudaStreamWaitEvent(us, a->meta_after, 0) : cudaSuccess;
        if (e != cudaSuccess)
            return pkv::fail(PKV_ERR_CUDA, "pkv_decode_step: upload stream: %s",
                             cudaGetErrorString(e));
    }
    if (a->in_bytes > 0) {
        PKV_REQUIRE(a->in_host && a->in_device, PKV_ERR_INVALID,
                    "pkv_decode_step: NULL input buffer");
        e = cudaMemcpyAsync(a->in_device, a->in_host, a->in_bytes, cudaMemcpyHostToDevice, us);
        if (e != cudaSuccess)
            return pkv::fail(PKV_ERR_CUDA, "pkv_decode_step: input upload: %s",
                             cudaGetErrorString(e));
    }
    if (a->meta_bytes > 0) {
        PKV_REQUIRE(a->meta_host && a->meta_device, PKV_ERR_INVALID,
                    "pkv_decode_step: NULL metadata buffer");
        e = cudaMemcpyAsync(a->meta_device, a->meta_host, a->meta_bytes, cudaMemcpyHostToDevice,
                            us);
        if (e != cudaSuccess)
            return pkv::fail(PKV_ERR_CUDA, "pkv_decode_step: metadata upload: %s",
                             cudaGetErrorString(e));
    }
    if (uploads && a->meta_stream != nullptr) {
        e = cudaEventRecord(a->meta_event, us);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(stream, a->meta_event, 0);
        if (e != cudaSuccess)
            return pkv::fail(PKV_ERR_CUDA, "pkv_decode_step: upload event: %s",
                             cudaGetErrorString(e));
    }
    int st = PKV_OK;
    if (a->num_pairs > 0) {
        st = fp8 ? pkv_copy_blocks_fp8(a->key_cache, a->value_cache, a->k_scale, a->v_scale,
                                       a->cow_pairs, a->num_pairs, a->num_blocks, a->block_size,
                                       a->num_kv_heads, a->head_dim, a->block_stride,
                                       a->dev_error, stream)
                 : pkv_copy_blocks(a->key_cache, a->value_cache, a->cow_pairs, a->num_pairs,
                                   a->num_blocks, a->block_size, a->num_kv_heads, a->head_dim,
                                   a->block_stride, a->dtype, a->dev_error, stream);
        if (st != PKV_OK) return st;
    }
    if (a->num_tokens > 0) {
        st = fp8 ? pkv_write_slots_fp8(a->key, a->value, a->key_cache, a->value_cache,
                                       a->k_scale, a->v_scale, a->slot_mapping, a->num_tokens,
                                       a->num_blocks, a->block_size, a->num_kv_heads,
                                       a->head_dim, a->block_stride, a->dtype, a->dev_error,
                                       stream)
                 : pkv_write_slots(a->key, a->value, a->key_cache, a->value_cache,
                                   a->slot_mapping, a->num_tokens, a->num_blocks, a->block_size,
                                   a->num_kv_heads, a->head_dim, a->block_stride, a->dtype,
                                   a->dev_error, stream);
        if (st != PKV_OK) return st;
    }
    if (a->work_items != nullptr) {
        st = fp8 ? pkv_decode_attention_fp8_items(
                       a->out, a->query, a->key_cache, a->value_cache, a->k_scale, a->v_scale,
                       a->block_tables, a->max_blocks_per_seq, a->context_lens, a->num_seqs,
                       a->max_context_len, a->num_q_heads, a->num_kv_heads, a->head_dim,
                       a->num_blocks, a->block_size, a->block_stride, a->scale,
                       a->partition_size, a->workspace, a->workspace_bytes, a->work_items,
                       a->num_items, a->dtype, a->dev_error, stream)
                 : pkv_decode_attention_items(
                       a->out, a->query, a->key_cache, a->value_cache, a->block_tables,
                       a->max_blocks_per_seq, a->context_lens, a->num_seqs, a->max_context_len,
                       a->num_q_heads, a->num_kv_heads, a->head_dim, a->num_blocks,
                       a->block_size, a->block_stride, a->scale, a->partition_size,
                       a->workspace, a->workspace_bytes, a->work_items, a->num_items, a->dtype,
                       a->dev_error, stream);
    } else {
        st = fp8 ? pkv_decode_attention_fp8(
                       a->out, a->query, a->key_cache, a->value_cache, a->k_scale, a->v_scale,
                       a->block_tables, a->max_blocks_per_seq, a->context_lens, a->num_seqs,
                       a->max_context_len, a->num_q_heads, a->num_kv_heads, a->head_dim,
                       a->num_blocks, a->block_size, a->block_stride, a->scale,
                       a->partition_size, a->workspace, a->workspace_bytes, a->dtype,
                       a->dev_error, stream)
                 : pkv_decode_attention(
                       a->out, a->query, a->key_cache, a->value_cache, a->block_tables,
                       a->max_blocks_per_seq, a->context_lens, a->num_seqs, a->max_context_len,
                       a->num_q_heads, a->num_kv_heads, a->head_dim, a->num_blocks,
                       a->block_size, a->block_stride, a->scale, a->partition_size,
                       a->workspace, a->workspace_bytes, a->dtype, a->dev_error, stream);
    }
    if (st != PKV_OK) return st;
    if (a->out_bytes > 0) {
        PKV_REQUIRE(a->out_host && a->out, PKV_ERR_INVALID, "pkv_decode_step: NULL output");
        cudaStream_t rs = stream;
        if (a->out_stream != nullptr) {
            PKV_REQUIRE(a->out_event != nullptr, PKV_ERR_INVALID,
                        "pkv_decode_step: out_stream without out_event");
            e = cudaEventRecord(a->out_event, stream);
            if (e == cudaSuccess) e = cudaStreamWaitEvent(a->out_stream, a->out_event, 0);
            if (e != cudaSuccess)
                return pkv::fail(PKV_ERR_CUDA, "pkv_decode_step: readback stream: %s",
                                 cudaGetErrorString(e));
            rs = a->out_stream;
        }
        e = cudaMemcpyAsync(a->out_host, a->out, a->out_bytes, cudaMemcpyDeviceToHost, rs);
        if (e != cudaSuccess)
            return pkv::fail(PKV_ERR_CUDA, "pkv_decode_step: output readback: %s",
                             cudaGetErrorString(e));
    }
    return PKV_OK;
}
