// decode_plan.cpp — host-side planning of a decode launch: the work list of
// (sequence, KV head, partition) items that pkv_decode_attention_items runs
// over.  Host code only; the kernels live in decode_attention.cu.
#include <algorithm>
#include <vector>

#include "internal.h"

// The decode work list ("PagedAttention 动态内存分页" page, 技术边界与取舍: a
// batch of very uneven lengths is what costs).  Items are the (sequence, KV
// head, partition) triples that hold tokens.  Within a sequence they go
// partition by partition with the KV heads of a partition side by side: the
// heads' slices of one block share its memory rows.  Longest first, a
// counting sort on the number of 16-token tiles each item holds orders them
// largest first, keeping that order among equals, in O(items + P / 16).
extern "C" int pkv_decode_work_items(const int32_t* context_lens, int num_seqs,
                                     int num_kv_heads, int max_context_len, int partition_size,
                                     int order, int32_t* items, int capacity, int* num_items) {
    PKV_NVTX_RANGE("pkv_decode_work_items");
    using pkv::plan_partitions;
    constexpr int kTile = 16;
    PKV_REQUIRE(num_items != nullptr, PKV_ERR_INVALID, "pkv_decode_work_items: NULL count");
    *num_items = 0;
    PKV_REQUIRE(num_seqs >= 0 && num_kv_heads > 0 && max_context_len >= 0 && capacity >= 0,
                PKV_ERR_INVALID, "pkv_decode_work_items: bad sizes");
    PKV_REQUIRE(partition_size >= 0 && partition_size % kTile == 0, PKV_ERR_INVALID,
                "pkv_decode_work_items: partition_size %d is not a multiple of 16",
                partition_size);
    PKV_REQUIRE(order == PKV_ITEMS_LONGEST_FIRST || order == PKV_ITEMS_SEQUENCES_LONGEST_FIRST ||
                    order == PKV_ITEMS_BATCH_ORDER,
                PKV_ERR_INVALID, "pkv_decode_work_items: order %d", order);
    if (num_seqs == 0) return PKV_OK;
    PKV_REQUIRE(context_lens != nullptr, PKV_ERR_INVALID, "pkv_decode_work_items: NULL lengths");
    int P, NP;
    plan_partitions(max_context_len, partition_size, &P, &NP);
    PKV_REQUIRE((int64_t)num_seqs * num_kv_heads * NP < (1ll << 31), PKV_ERR_UNSUPPORTED,
                "pkv_decode_work_items: grid too large");
    int64_t total = 0;
    for (int s = 0; s < num_seqs; ++s) {
        const int L = context_lens[s];
        PKV_REQUIRE(L >= 0 && L <= max_context_len, PKV_ERR_INVALID,
                    "pkv_decode_work_items: context_lens[%d] = %d outside [0, %d]", s, L,
                    max_context_len);
        total += (int64_t)(L > 0 ? (L + P - 1) / P : 1) * num_kv_heads;
    }
    *num_items = (int)total;
    PKV_REQUIRE(total <= capacity, PKV_ERR_INVALID,
                "pkv_decode_work_items: %lld items, capacity %d", (long long)total, capacity);
    PKV_REQUIRE(items != nullptr, PKV_ERR_INVALID, "pkv_decode_work_items: NULL items");
    // the sequences in the order their items are emitted
    std::vector<int> seqs(num_seqs);
    for (int s = 0; s < num_seqs; ++s) seqs[s] = s;
    if (order == PKV_ITEMS_SEQUENCES_LONGEST_FIRST)
        std::stable_sort(seqs.begin(), seqs.end(),
                         [&](int a, int b) { return context_lens[a] > context_lens[b]; });
    // bucket of an item: its tiles (largest first) for longest first, one
    // bucket otherwise
    const bool by_tiles = order == PKV_ITEMS_LONGEST_FIRST;
    const int nbuckets = by_tiles ? P / kTile + 1 : 1;  // tiles per item: 0 .. P / 16
    auto bucket = [&](int tokens) { return by_tiles ? (tokens + kTile - 1) / kTile : 0; };
    std::vector<int64_t> start(nbuckets + 1, 0);
    for (int s = 0; s < num_seqs; ++s) {
        const int L = context_lens[s];
        const int np = L > 0 ? (L + P - 1) / P : 1;
        for (int part = 0; part < np; ++part)
            start[bucket(std::min(P, L - part * P))] += num_kv_heads;
    }
    int64_t at = 0;  // counts to start offsets, the largest bucket first
    for (int b = nbuckets - 1; b >= 0; --b) {
        const int64_t c = start[b];
        start[b] = at;
        at += c;
    }
    for (int s : seqs) {
        const int L = context_lens[s];
        const int np = L > 0 ? (L + P - 1) / P : 1;
        for (int part = 0; part < np; ++part) {
            int64_t& pos = start[bucket(std::min(P, L - part * P))];
            for (int h = 0; h < num_kv_heads; ++h)
                items[pos++] = (int32_t)(((int64_t)s * num_kv_heads + h) * NP + part);
        }
    }
    return PKV_OK;
}
