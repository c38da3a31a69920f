// pool.cpp — the host block pool: free stack, refcounts, per-sequence Block
// Tables and copy-on-write on append.
//
// The pages fix the behaviour: one global pool of equal physical blocks made
// at start-up, blocks taken and returned on demand ("一文读懂vLLM的…
// PagedAttention" page, 运行模式的根本转变); prefill takes blocks in order and
// decode writes the next slot of the current block, taking a new block when
// it is full ("Paged KV" wiki page, 实现原理 / 运行阶段); new blocks are
// appended to the table's tail lazily and a finished sequence's blocks go
// back at once ("PagedAttention 动态内存分页" page, 块粒度与块表 and 动态块分配与
// 回收); sequences may share blocks, and a shared block is copied before a
// write (same page, 写时复制与内存共享).
//
// Readings where they are silent: the free pool is a LIFO stack (the most
// recently freed block is reused first, which keeps hot blocks in L2); a
// fresh pool hands blocks out in a caller-given order (default 0, 1, ...);
// an operation that would run out of blocks changes nothing.
//
// Block swapping (same page, 动态块分配与回收: when GPU memory runs short, a
// sequence's KV blocks move to CPU memory and come back when needed): a
// second LIFO stack of host block ids, made once.  A swap moves one whole
// sequence, in table order, and returns the (src, dst) pairs to copy; a GPU
// block still shared with a resident sequence stays on the GPU for it.  A
// swapped-out sequence cannot be appended to or forked.
#include <algorithm>
#include <new>
#include <unordered_map>
#include <vector>

#include "internal.h"

namespace {

struct Seq {
    std::vector<int32_t> table;  // physical block ids in logical order (host ids if swapped)
    int64_t tokens = 0;
    bool swapped = false;
};

}  // namespace

struct pkv_pool {
    int num_blocks = 0;
    int block_size = 0;
    std::vector<int32_t> free_stack;  // top = back()
    std::vector<int32_t> refcount;
    std::unordered_map<int64_t, Seq> seqs;
    bool has_host = false;
    std::vector<int32_t> host_free;  // top = back()
    std::vector<int32_t> host_refcount;

    int32_t take() {
        int32_t b = free_stack.back();
        free_stack.pop_back();
        refcount[b] = 1;
        return b;
    }
};

extern "C" int pkv_pool_create(int num_blocks, int block_size,
                               const int32_t* free_order, pkv_pool** out) {
    PKV_REQUIRE(out != nullptr, PKV_ERR_INVALID, "pkv_pool_create: out is NULL");
    *out = nullptr;
    PKV_REQUIRE(num_blocks >= 0 && block_size > 0, PKV_ERR_INVALID,
                "pkv_pool_create: num_blocks %d, block_size %d", num_blocks,
                block_size);
    pkv_pool* p = new (std::nothrow) pkv_pool;
    PKV_REQUIRE(p != nullptr, PKV_ERR_INVALID, "pkv_pool_create: out of host memory");
    p->num_blocks = num_blocks;
    p->block_size = block_size;
    p->refcount.assign(num_blocks, 0);
    p->free_stack.resize(num_blocks);
    if (free_order) {
        std::vector<char> seen(num_blocks, 0);
        for (int i = 0; i < num_blocks; ++i) {
            int32_t b = free_order[i];
            if (b < 0 || b >= num_blocks || seen[b]) {
                delete p;
                return pkv::fail(PKV_ERR_INVALID,
                                 "pkv_pool_create: free_order is not a permutation "
                                 "(entry %d = %d)", i, b);
            }
            seen[b] = 1;
            p->free_stack[num_blocks - 1 - i] = b;  // first entry on top
        }
    } else {
        for (int i = 0; i < num_blocks; ++i) p->free_stack[i] = num_blocks - 1 - i;
    }
    *out = p;
    return PKV_OK;
}

extern "C" void pkv_pool_destroy(pkv_pool* pool) { delete pool; }

extern "C" int pkv_seq_add(pkv_pool* pool, int64_t seq_id, int num_tokens) {
    PKV_REQUIRE(pool, PKV_ERR_INVALID, "pkv_seq_add: pool is NULL");
    PKV_REQUIRE(num_tokens >= 0, PKV_ERR_INVALID, "pkv_seq_add: num_tokens %d", num_tokens);
    PKV_REQUIRE(!pool->seqs.count(seq_id), PKV_ERR_INVALID,
                "pkv_seq_add: sequence %lld exists", (long long)seq_id);
    int64_t need = ((int64_t)num_tokens + pool->block_size - 1) / pool->block_size;
    PKV_REQUIRE(need <= (int64_t)pool->free_stack.size(), PKV_ERR_OOM,
                "pkv_seq_add: needs %lld blocks, %zu free", (long long)need,
                pool->free_stack.size());
    Seq s;
    s.table.reserve(need);
    for (int64_t i = 0; i < need; ++i) s.table.push_back(pool->take());
    s.tokens = num_tokens;
    pool->seqs.emplace(seq_id, std::move(s));
    return PKV_OK;
}

extern "C" int pkv_seq_fork(pkv_pool* pool, int64_t parent, int64_t child) {
    PKV_REQUIRE(pool, PKV_ERR_INVALID, "pkv_seq_fork: pool is NULL");
    auto it = pool->seqs.find(parent);
    PKV_REQUIRE(it != pool->seqs.end(), PKV_ERR_INVALID,
                "pkv_seq_fork: no sequence %lld", (long long)parent);
    PKV_REQUIRE(!it->second.swapped, PKV_ERR_INVALID,
                "pkv_seq_fork: sequence %lld is swapped out", (long long)parent);
    PKV_REQUIRE(!pool->seqs.count(child), PKV_ERR_INVALID,
                "pkv_seq_fork: sequence %lld exists", (long long)child);
    Seq c = it->second;  // copy before emplace: emplace may rehash
    for (int32_t b : c.table) ++pool->refcount[b];
    pool->seqs.emplace(child, std::move(c));
    return PKV_OK;
}

extern "C" int pkv_seq_append(pkv_pool* pool, int64_t seq_id, int64_t* slot,
                              int32_t* cow_src, int32_t* cow_dst) {
    PKV_REQUIRE(pool && slot && cow_src && cow_dst, PKV_ERR_INVALID,
                "pkv_seq_append: NULL argument");
    auto it = pool->seqs.find(seq_id);
    PKV_REQUIRE(it != pool->seqs.end(), PKV_ERR_INVALID,
                "pkv_seq_append: no sequence %lld", (long long)seq_id);
    Seq& s = it->second;
    PKV_REQUIRE(!s.swapped, PKV_ERR_INVALID, "pkv_seq_append: sequence %lld is swapped out",
                (long long)seq_id);
    const int bs = pool->block_size;
    const int off = (int)(s.tokens % bs);
    int32_t src = -1, dst = -1;
    if (off == 0) {
        // the current block is full (or there is none): take a new one
        PKV_REQUIRE(!pool->free_stack.empty(), PKV_ERR_OOM,
                    "pkv_seq_append: pool exhausted");
        s.table.push_back(pool->take());
    } else {
        int32_t last = s.table.back();
        if (pool->refcount[last] > 1) {
            // shared partial block: copy before writing into it
            PKV_REQUIRE(!pool->free_stack.empty(), PKV_ERR_OOM,
                        "pkv_seq_append: pool exhausted (copy-on-write)");
            int32_t fresh = pool->take();
            --pool->refcount[last];
            s.table.back() = fresh;
            src = last;
            dst = fresh;
        }
    }
    ++s.tokens;
    *slot = (int64_t)s.table.back() * bs + off;
    *cow_src = src;
    *cow_dst = dst;
    return PKV_OK;
}

extern "C" int pkv_seq_append_batch(pkv_pool* pool, int n, const int64_t* seq_ids,
                                    int64_t* slots, int32_t* cow_pairs,
                                    int* num_cow, int* num_done) {
    PKV_NVTX_RANGE("pkv_seq_append_batch");
    PKV_REQUIRE(pool && n >= 0 && (n == 0 || (seq_ids && slots && cow_pairs)) && num_cow,
                PKV_ERR_INVALID, "pkv_seq_append_batch: bad argument");
    *num_cow = 0;
    if (num_done) *num_done = 0;
    for (int i = 0; i < n; ++i) {
        int32_t src, dst;
        int st = pkv_seq_append(pool, seq_ids[i], &slots[i], &src, &dst);
        if (st != PKV_OK) return st;
        if (src >= 0) {
            cow_pairs[2 * *num_cow] = src;
            cow_pairs[2 * *num_cow + 1] = dst;
            ++*num_cow;
        }
        if (num_done) *num_done = i + 1;
    }
    return PKV_OK;
}

extern "C" int pkv_seq_free(pkv_pool* pool, int64_t seq_id) {
    PKV_REQUIRE(pool, PKV_ERR_INVALID, "pkv_seq_free: pool is NULL");
    auto it = pool->seqs.find(seq_id);
    PKV_REQUIRE(it != pool->seqs.end(), PKV_ERR_INVALID,
                "pkv_seq_free: no sequence %lld", (long long)seq_id);
    if (it->second.swapped) {
        for (int32_t h : it->second.table)
            if (--pool->host_refcount[h] == 0) pool->host_free.push_back(h);
    } else {
        for (int32_t b : it->second.table)
            if (--pool->refcount[b] == 0) pool->free_stack.push_back(b);
    }
    pool->seqs.erase(it);
    return PKV_OK;
}

extern "C" int pkv_seq_num_tokens(const pkv_pool* pool, int64_t seq_id, int* num_tokens) {
    PKV_REQUIRE(pool && num_tokens, PKV_ERR_INVALID, "pkv_seq_num_tokens: NULL argument");
    auto it = pool->seqs.find(seq_id);
    PKV_REQUIRE(it != pool->seqs.end(), PKV_ERR_INVALID,
                "pkv_seq_num_tokens: no sequence %lld", (long long)seq_id);
    *num_tokens = (int)it->second.tokens;
    return PKV_OK;
}

extern "C" int pkv_seq_slot_mapping(const pkv_pool* pool, int64_t seq_id, int first_token,
                                    int num_tokens, int64_t* out) {
    PKV_REQUIRE(pool && (out || num_tokens == 0), PKV_ERR_INVALID,
                "pkv_seq_slot_mapping: NULL argument");
    auto it = pool->seqs.find(seq_id);
    PKV_REQUIRE(it != pool->seqs.end(), PKV_ERR_INVALID,
                "pkv_seq_slot_mapping: no sequence %lld", (long long)seq_id);
    const Seq& s = it->second;
    PKV_REQUIRE(!s.swapped, PKV_ERR_INVALID, "pkv_seq_slot_mapping: sequence %lld is swapped out",
                (long long)seq_id);
    PKV_REQUIRE(first_token >= 0 && num_tokens >= 0 &&
                    (int64_t)first_token + num_tokens <= s.tokens,
                PKV_ERR_INVALID, "pkv_seq_slot_mapping: tokens [%d, %d) outside 0..%lld",
                first_token, first_token + num_tokens, (long long)s.tokens);
    const int bs = pool->block_size;
    for (int i = 0; i < num_tokens; ++i) {
        const int64_t t = (int64_t)first_token + i;
        out[i] = (int64_t)s.table[t / bs] * bs + t % bs;
    }
    return PKV_OK;
}

extern "C" int pkv_seq_block_table(const pkv_pool* pool, int64_t seq_id, int32_t* out,
                                   int cap, int* n) {
    PKV_REQUIRE(pool && n, PKV_ERR_INVALID, "pkv_seq_block_table: NULL argument");
    auto it = pool->seqs.find(seq_id);
    PKV_REQUIRE(it != pool->seqs.end(), PKV_ERR_INVALID,
                "pkv_seq_block_table: no sequence %lld", (long long)seq_id);
    const auto& t = it->second.table;
    *n = (int)t.size();
    PKV_REQUIRE((int64_t)cap >= (int64_t)t.size() && (t.empty() || out), PKV_ERR_INVALID,
                "pkv_seq_block_table: capacity %d < %zu", cap, t.size());
    std::copy(t.begin(), t.end(), out);
    return PKV_OK;
}

extern "C" int pkv_pool_block_tables(const pkv_pool* pool, int n, const int64_t* seq_ids,
                                     int32_t* out, int max_blocks_per_seq, int32_t fill,
                                     int32_t* context_lens, int32_t* max_context_len) {
    PKV_REQUIRE(pool && n >= 0 && max_blocks_per_seq >= 0 &&
                    (n == 0 || (seq_ids && (out || max_blocks_per_seq == 0))),
                PKV_ERR_INVALID, "pkv_pool_block_tables: bad argument");
    int64_t longest = 0;
    for (int i = 0; i < n; ++i) {
        auto it = pool->seqs.find(seq_ids[i]);
        PKV_REQUIRE(it != pool->seqs.end(), PKV_ERR_INVALID,
                    "pkv_pool_block_tables: no sequence %lld", (long long)seq_ids[i]);
        PKV_REQUIRE(!it->second.swapped, PKV_ERR_INVALID,
                    "pkv_pool_block_tables: sequence %lld is swapped out",
                    (long long)seq_ids[i]);
        const auto& t = it->second.table;
        PKV_REQUIRE((int64_t)t.size() <= max_blocks_per_seq, PKV_ERR_INVALID,
                    "pkv_pool_block_tables: sequence %lld has %zu blocks > %d",
                    (long long)seq_ids[i], t.size(), max_blocks_per_seq);
        int32_t* row = out + (int64_t)i * max_blocks_per_seq;
        std::copy(t.begin(), t.end(), row);
        std::fill(row + t.size(), row + max_blocks_per_seq, fill);
        if (context_lens) context_lens[i] = (int32_t)it->second.tokens;
        longest = std::max<int64_t>(longest, it->second.tokens);
    }
    if (max_context_len) *max_context_len = (int32_t)longest;
    return PKV_OK;
}

extern "C" int pkv_pool_num_free(const pkv_pool* pool) {
    PKV_REQUIRE(pool, PKV_ERR_INVALID, "pkv_pool_num_free: pool is NULL");
    return (int)pool->free_stack.size();
}

extern "C" int pkv_pool_num_blocks(const pkv_pool* pool) {
    PKV_REQUIRE(pool, PKV_ERR_INVALID, "pkv_pool_num_blocks: pool is NULL");
    return pool->num_blocks;
}

extern "C" int pkv_pool_block_size(const pkv_pool* pool) {
    PKV_REQUIRE(pool, PKV_ERR_INVALID, "pkv_pool_block_size: pool is NULL");
    return pool->block_size;
}

extern "C" int pkv_pool_free_list(const pkv_pool* pool, int32_t* out, int cap, int* n) {
    PKV_REQUIRE(pool && n, PKV_ERR_INVALID, "pkv_pool_free_list: NULL argument");
    *n = (int)pool->free_stack.size();
    PKV_REQUIRE((int64_t)cap >= (int64_t)pool->free_stack.size() &&
                    (pool->free_stack.empty() || out),
                PKV_ERR_INVALID, "pkv_pool_free_list: capacity %d < %zu", cap,
                pool->free_stack.size());
    std::copy(pool->free_stack.begin(), pool->free_stack.end(), out);
    return PKV_OK;
}

extern "C" int pkv_block_refcount(const pkv_pool* pool, int block) {
    PKV_REQUIRE(pool && block >= 0 && block < pool->num_blocks, PKV_ERR_INVALID,
                "pkv_block_refcount: bad block %d", block);
    return pool->refcount[block];
}

// ---------------------------------------------------------------------------
// block swapping
// ---------------------------------------------------------------------------
extern "C" int pkv_pool_set_host_blocks(pkv_pool* pool, int num_host_blocks) {
    PKV_REQUIRE(pool && num_host_blocks >= 0, PKV_ERR_INVALID,
                "pkv_pool_set_host_blocks: bad argument");
    PKV_REQUIRE(!pool->has_host, PKV_ERR_INVALID,
                "pkv_pool_set_host_blocks: the host pool exists");
    pool->has_host = true;
    pool->host_refcount.assign(num_host_blocks, 0);
    pool->host_free.resize(num_host_blocks);
    for (int i = 0; i < num_host_blocks; ++i) pool->host_free[i] = num_host_blocks - 1 - i;
    return PKV_OK;
}

extern "C" int pkv_seq_swap_out(pkv_pool* pool, int64_t seq_id, int32_t* pairs, int cap,
                                int* num_pairs) {
    PKV_REQUIRE(pool && num_pairs, PKV_ERR_INVALID, "pkv_seq_swap_out: NULL argument");
    *num_pairs = 0;
    PKV_REQUIRE(pool->has_host, PKV_ERR_INVALID, "pkv_seq_swap_out: no host pool");
    auto it = pool->seqs.find(seq_id);
    PKV_REQUIRE(it != pool->seqs.end(), PKV_ERR_INVALID,
                "pkv_seq_swap_out: no sequence %lld", (long long)seq_id);
    Seq& s = it->second;
    PKV_REQUIRE(!s.swapped, PKV_ERR_INVALID, "pkv_seq_swap_out: sequence %lld is swapped out",
                (long long)seq_id);
    const size_t n = s.table.size();
    PKV_REQUIRE((int64_t)cap >= (int64_t)n && (n == 0 || pairs), PKV_ERR_INVALID,
                "pkv_seq_swap_out: capacity %d < %zu pairs", cap, n);
    PKV_REQUIRE(n <= pool->host_free.size(), PKV_ERR_OOM,
                "pkv_seq_swap_out: needs %zu host blocks, %zu free", n, pool->host_free.size());
    for (size_t i = 0; i < n; ++i) {
        const int32_t h = pool->host_free.back();
        pool->host_free.pop_back();
        pool->host_refcount[h] = 1;
        pairs[2 * i] = s.table[i];
        pairs[2 * i + 1] = h;
    }
    for (size_t i = 0; i < n; ++i) {
        const int32_t b = s.table[i];
        if (--pool->refcount[b] == 0) pool->free_stack.push_back(b);
        s.table[i] = pairs[2 * i + 1];
    }
    s.swapped = true;
    *num_pairs = (int)n;
    return PKV_OK;
}

extern "C" int pkv_seq_swap_in(pkv_pool* pool, int64_t seq_id, int32_t* pairs, int cap,
                               int* num_pairs) {
    PKV_REQUIRE(pool && num_pairs, PKV_ERR_INVALID, "pkv_seq_swap_in: NULL argument");
    *num_pairs = 0;
    auto it = pool->seqs.find(seq_id);
    PKV_REQUIRE(it != pool->seqs.end(), PKV_ERR_INVALID,
                "pkv_seq_swap_in: no sequence %lld", (long long)seq_id);
    Seq& s = it->second;
    PKV_REQUIRE(s.swapped, PKV_ERR_INVALID, "pkv_seq_swap_in: sequence %lld is resident",
                (long long)seq_id);
    const size_t n = s.table.size();
    PKV_REQUIRE((int64_t)cap >= (int64_t)n && (n == 0 || pairs), PKV_ERR_INVALID,
                "pkv_seq_swap_in: capacity %d < %zu pairs", cap, n);
    PKV_REQUIRE(n <= pool->free_stack.size(), PKV_ERR_OOM,
                "pkv_seq_swap_in: needs %zu blocks, %zu free", n, pool->free_stack.size());
    for (size_t i = 0; i < n; ++i) {
        pairs[2 * i] = s.table[i];
        pairs[2 * i + 1] = pool->take();
    }
    for (size_t i = 0; i < n; ++i) {
        const int32_t h = s.table[i];
        if (--pool->host_refcount[h] == 0) pool->host_free.push_back(h);
        s.table[i] = pairs[2 * i + 1];
    }
    s.swapped = false;
    *num_pairs = (int)n;
    return PKV_OK;
}

extern "C" int pkv_seq_is_swapped(const pkv_pool* pool, int64_t seq_id, int* swapped) {
    PKV_REQUIRE(pool && swapped, PKV_ERR_INVALID, "pkv_seq_is_swapped: NULL argument");
    auto it = pool->seqs.find(seq_id);
    PKV_REQUIRE(it != pool->seqs.end(), PKV_ERR_INVALID,
                "pkv_seq_is_swapped: no sequence %lld", (long long)seq_id);
    *swapped = it->second.swapped ? 1 : 0;
    return PKV_OK;
}

extern "C" int pkv_pool_num_free_host(const pkv_pool* pool) {
    PKV_REQUIRE(pool, PKV_ERR_INVALID, "pkv_pool_num_free_host: pool is NULL");
    return (int)pool->host_free.size();
}

extern "C" int pkv_pool_host_free_list(const pkv_pool* pool, int32_t* out, int cap, int* n) {
    PKV_REQUIRE(pool && n, PKV_ERR_INVALID, "pkv_pool_host_free_list: NULL argument");
    *n = (int)pool->host_free.size();
    PKV_REQUIRE((int64_t)cap >= (int64_t)pool->host_free.size() &&
                    (pool->host_free.empty() || out),
                PKV_ERR_INVALID, "pkv_pool_host_free_list: capacity %d < %zu", cap,
                pool->host_free.size());
    std::copy(pool->host_free.begin(), pool->host_free.end(), out);
    return PKV_OK;
}

extern "C" int pkv_host_block_refcount(const pkv_pool* pool, int block) {
    PKV_REQUIRE(pool && block >= 0 && block < (int)pool->host_refcount.size(), PKV_ERR_INVALID,
                "pkv_host_block_refcount: bad host block %d", block);
    return pool->host_refcount[block];
}
