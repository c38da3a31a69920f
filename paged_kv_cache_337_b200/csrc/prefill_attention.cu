// prefill_attention.cu — paged prefill attention ("Paged KV" wiki page,
// 实现原理 / 运行阶段: prefill takes blocks in order and fills them with the
// prompt's K/V; the prompt's tokens then attend over the sequence through
// the same Block Table, as decode does with one token).
//
// Sequence s has n_s query rows (query_start[s] .. query_start[s+1]-1), the
// last n_s of its L_s cached tokens: row i is token p = L_s - n_s + i and
// attends causally to tokens 0 .. p.
//
// A work item is 256 rows of one (sequence, KV head) as two 128-row Q
// tiles: (query token, head of the GQA group) pairs, so each K/V tile is
// streamed once for the group and both tiles.  The CTAs are persistent, one
// per SM: each walks a fixed list of items, heaviest first, and every role
// keeps running counters across items, so that one item's startup (Q
// staging, the first K/V tiles and S) overlaps the previous item's last key
// tiles and output.
// The work runs on the 5th-generation tensor cores with the accumulators in
// tensor memory:
//   - two producer warps, one for K and one for V, bring 64-key tiles
//     through a 4-stage ring (one TMA box per 16 slots of a block and per
//     64-dim half);
//   - two MMA warps, one per Q tile, issue per key tile S = Q K^T (M 128,
//     N 64, K 16 steps; Q and K from shared memory) into tensor memory,
//     then O += P V as the tile's P is ready (P read from tensor memory, V
//     from shared memory as an MN-major B operand), so that the tensor
//     cores work on one tile while the other tile's softmax runs, and
//     neither tile's issue waits behind the other's P;
//   - eight softmax warps, four per Q tile (one tensor-memory lane quarter
//     each, one row per thread), read S, apply the causal mask, keep the
//     running max and sum, take a quarter of the exponentials from an
//     FMA-pipe polynomial and the rest from the exponential unit, write P
//     over S (one f16 rounding; a bf16 high
//     part and its remainder, two MMAs, for a bf16 V group beyond f16's
//     range) and rescale O when the running max grows by more than 2^8,
//     then write the normalised output;
//   - four Q warps stage each item's Q tiles once the previous item's last
//     S has read them, and convert each landed bf16 V tile to f16 in
//     shared memory, so that P V runs as one f16 MMA per 16 keys.
#include <cudaTypedefs.h>

#include <algorithm>

#include "common.cuh"
#include "packed_f32.cuh"
#include "tcgen05.cuh"
#include "tensor_maps.h"

namespace pkv {
namespace {

constexpr int kD = 128;                 // head_dim (built)
constexpr int kRows = 128;              // rows per Q tile = UMMA M
constexpr int kQTiles = 2;              // Q tiles per CTA
constexpr int kKeys = 64;               // keys per tile = UMMA N of S, K of P V
constexpr int kStages = 4;
constexpr int kHalfBytes = kKeys * 128; // one 64-dim half of a K (or V) tile: 8 KiB
constexpr int kTileBytes = 2 * kHalfBytes;          // 32 KiB
constexpr int kStageBytes = 2 * kTileBytes;         // K + V
constexpr int kQHalfBytes = kRows * 128;            // 16 KiB
constexpr int kQTileBytes = 2 * kQHalfBytes;      // one Q tile, both halves
constexpr int kQBytes = kQTiles * kQTileBytes;
constexpr int kBoxKeys = 16;                        // slots per TMA box
constexpr int kProducerWarp = 0, kMmaWarp = 1, kSoftmaxWarp0 = 2, kSoftmaxWarps = 4 * kQTiles;
constexpr int kQWarp0 = kSoftmaxWarp0 + kSoftmaxWarps, kQWarps = 4;
constexpr int kVProducerWarp = kQWarp0 + kQWarps, kMmaWarpB = kVProducerWarp + 1;
constexpr int kThreads = (kMmaWarpB + 1) * 32;
// tensor-memory columns per Q tile t: two S buffers (64 columns each; P
// high | P low, 32 each, written over S once it is read) at 256 t and
// 256 t + 64, O at 256 t + 128; key tile j uses S buffer j % 2
constexpr uint32_t kTileCols = 256, kColO = 128, kColPl = kKeys / 2, kTmemCols = 512;
// kv_full/kv_empty/v_ready per stage; s_full/p_full per (Q tile, S
// buffer); o_done and o_free per Q tile; drain, q_ready, q_free; item_done
// per Q tile
constexpr int kNumBars = 3 * kStages + 7 * kQTiles + 3;
// after the barriers: the tensor-memory address (16 bytes) and, per stage,
// one byte per 16-key group of V: 1 = converted to f16, 0 = left in bf16
constexpr size_t kSmemBytes = 1024 + kQBytes + kStages * kStageBytes + kNumBars * 8 + 16 + 16;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleLog2 = 8.f;  // rescale O when the max grows by more than 2^8

struct PrefillParams {
    void* out;
    const void* query;
    const int32_t* block_tables;
    const int32_t* context_lens;
    const int32_t* query_start;
    int32_t* dev_error;
    int num_seqs, max_blocks_per_seq, num_q_heads, num_kv_heads, group;
    int num_blocks, block_size, max_query_len, tiles_per_seq;
    int num_items;  // tiles_per_seq x num_seqs x num_kv_heads
    float scale_log2;
};

// swizzled byte offset of (row, 16-byte chunk) inside one 64-dim half laid
// out as rows of 128 bytes (the TMA 128-byte swizzle and the UMMA canonical
// K-major / MN-major 128-byte swizzle agree on it)
__device__ __forceinline__ uint32_t swz(int r, int chunk) {
    return r * 128 + (((chunk & 7) ^ (r & 7)) << 4);
}

__device__ __forceinline__ uint8_t* align_1024(uint8_t* p) {
    const uint32_t a = smem_addr(p);
    return p + ((1024u - (a & 1023u)) & 1023u);
}

__device__ __forceinline__ void mbar_arrive_one(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

// Cache policy of the L2: the streaming Q reads and output writes are
// evicted first, so that the K/V of the sequences in flight, which every
// row tile of a sequence re-reads, stay in L2 (PKV_PREFILL_L2_HINTS 0: no
// hints).
#ifndef PKV_PREFILL_L2_HINTS
#define PKV_PREFILL_L2_HINTS 1
#endif
constexpr bool kL2Hints = PKV_PREFILL_L2_HINTS != 0;

// Of every eight key pairs of a softmax pass, how many take 2^x from the
// FMA-pipe polynomial (ex2_poly2) instead of the exponential unit.  The
// softmax is bound by instruction issue more than by the exponential unit:
// two of eight measured fastest, each pair moved beyond that slower.
#ifndef PKV_PREFILL_POLY_EXP
#define PKV_PREFILL_POLY_EXP 2
#endif
constexpr int kPolyPairsPer8 = PKV_PREFILL_POLY_EXP;
static_assert(kPolyPairsPer8 >= 0 && kPolyPairsPer8 <= 8, "pairs of eight");

// 16-byte copy global -> shared that does not wait (cp.async, L2 only);
// when copy is false, the destination is zero-filled and nothing is read
__device__ __forceinline__ void cp_async_16(void* dst, const void* src, bool copy,
                                            uint64_t policy) {
    if constexpr (kL2Hints)
        asm volatile("cp.async.cg.shared.global.L2::cache_hint [%0], [%1], 16, %2, %3;"
                     ::"r"(smem_addr(dst)), "l"(src), "r"(copy ? 16 : 0), "l"(policy)
                     : "memory");
    else
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_addr(dst)),
                     "l"(src), "r"(copy ? 16 : 0)
                     : "memory");
}

// waits for every cp.async this thread issued
__device__ __forceinline__ void cp_async_wait_all() {
    asm volatile("cp.async.wait_all;" ::: "memory");
}


struct Bars {
    uint64_t* kv_full;   // [kStages]: TMA bytes landed
    uint64_t* kv_empty;  // [kStages]: the P V MMAs reading the stage completed
    uint64_t* v_ready;   // [kStages]: a bf16 V tile converted (the four Q warps)
    uint64_t* s_full;    // [kQTiles][2]: S of the buffer in tensor memory
    uint64_t* p_full;    // [kQTiles][2]: P of the buffer written (and O rescaled)
    uint64_t* o_done;    // [kQTiles]: the P V MMAs of the Q tile completed
    uint64_t* o_free;    // [kQTiles]: the Q tile's softmax warps have read O (item end)
    uint64_t* drain;     // every MMA issued completed (exit)
    uint64_t* q_ready;   // the Q tiles of the next item are staged
    uint64_t* q_free;    // every S MMA of the item completed: Q may be restaged
    uint64_t* item_done; // [kQTiles]: the item's last P V of the Q tile completed
};

// One work item: 256 rows of one (sequence, KV head).
struct Item {
    int s, kvh, q0, n, L, r0, nrows, ntiles;
    bool run;  // false: past the sequence's rows, or an invalid sequence
};

// Index of this CTA's k-th item.  Items are numbered heaviest first (the
// last row tile of every (sequence, KV head), then the tile before, ...)
// and dealt one per CTA per round, in alternate directions, so that every
// CTA gets a similar share of heavy and light items.
__device__ __forceinline__ int item_index(int k) {
    const int g = (int)gridDim.x;
    return k * g + ((k & 1) ? g - 1 - (int)blockIdx.x : (int)blockIdx.x);
}

// Every role decodes the same items in the same order, so the running
// counters that pick ring stages, S buffers and barrier phases agree.
__device__ Item decode_item(const PrefillParams& p, int idx, bool report) {
    Item it;
    const int pairs = p.num_seqs * p.num_kv_heads;
    const int tile = p.tiles_per_seq - 1 - idx / pairs;
    const int rest = idx % pairs;
    it.kvh = rest % p.num_kv_heads;
    it.s = rest / p.num_kv_heads;
    it.q0 = __ldg(p.query_start + it.s);
    it.n = __ldg(p.query_start + it.s + 1) - it.q0;
    it.L = __ldg(p.context_lens + it.s);
    it.nrows = it.n * p.group;
    it.r0 = tile * kRows * kQTiles;
    it.ntiles = 0;
    it.run = false;
    if (it.n < 0 || it.n > it.L || it.n > p.max_query_len ||
        (int64_t)it.L > (int64_t)p.max_blocks_per_seq * p.block_size) {
        if (report && tile == p.tiles_per_seq - 1 && it.kvh == 0)
            report_error(p.dev_error, PKV_DEVERR_CONTEXT_LEN, it.s);
        return it;
    }
    if (it.r0 >= it.nrows) return it;  // a row tile past this sequence's rows
    const int last_row = min(it.nrows, it.r0 + kRows * kQTiles) - 1;
    const int kv_end = it.L - it.n + last_row / p.group + 1;
    it.ntiles = (kv_end + kKeys - 1) / kKeys;
    it.run = true;
    return it;
}

// Producers: warp 0 loads the K tiles, warp 14 the V tiles, into the
// same ring stages (each stage's full barrier takes one arrival per
// producer with its byte count).  A box past the context still loads a
// block (the last one) so that every stage receives its full byte count;
// those rows are masked (K) or zeroed (V) downstream.  The block ids come
// from the Block Table one warp-wide load per eight key tiles (lane i: the
// id of box i of the window), handed by shuffles to the lanes that issue
// the loads: eight lanes, one box each (a TMA box costs its issuing lane
// less when several lanes of the warp issue one each).  The ring position
// runs on across items, so the next item's tiles load while the current
// one finishes.
__device__ void produce(const CUtensorMap& kmap, const CUtensorMap& vmap, const PrefillParams& p,
                        uint8_t* stages, const Bars& b, int lane, bool is_v, bool* failed) {
    constexpr int kBoxes = kKeys / kBoxKeys;       // TMA boxes per key tile and 64-dim half
    constexpr int kWindowTiles = 32 / kBoxes;      // key tiles per warp-wide block-id load
    const int bs = p.block_size;
    const uint64_t keep = l2_policy_evict_last();  // K/V: re-read by later row tiles
    int gk = 0;  // key tiles issued over all items
    for (int k = 0; !*failed; ++k) {
        const int idx = item_index(k);
        if (idx >= p.num_items) break;
        const Item it = decode_item(p, idx, lane == 0);
        if (!it.run) continue;
        const int32_t* row = p.block_tables + (int64_t)it.s * p.max_blocks_per_seq;
        const int last_block = it.L > 0 ? (it.L - 1) / bs : 0;
        int phys_lane = 0;
        for (int j = 0; j < it.ntiles; ++j) {
            if (j % kWindowTiles == 0) {
                const int box = j * kBoxes + lane;  // box of this lane in the window
                phys_lane = __ldg(row + min(box * kBoxKeys / bs, last_block));
                if (box < it.ntiles * kBoxes && (phys_lane < 0 || phys_lane >= p.num_blocks))
                    report_error(p.dev_error, PKV_DEVERR_BLOCK_ID, it.s);
            }
            const int st = gk % kStages;
            if (gk >= kStages &&
                !__all_sync(0xffffffffu,
                            mbar_wait_bounded(&b.kv_empty[st], ((gk / kStages) - 1) & 1))) {
                *failed = true;
                break;
            }
            const int phys_box =
                __shfl_sync(0xffffffffu, phys_lane, (j % kWindowTiles) * kBoxes + ((lane >> 1) & 3));
            // one lane per box of this warp's operand (box lane / 2 of the
            // tile, 64-dim half lane % 2)
            if (lane == 0) mbar_arrive_expect_tx(&b.kv_full[st], kTileBytes);
            __syncwarp();
            if (lane < 2 * kBoxes) {
                const int bx = lane >> 1, h = lane & 1;
                const int key0 = j * kKeys + bx * kBoxKeys;
                const int off = key0 < it.L ? key0 % bs : 0;
                uint8_t* dst = stages + st * kStageBytes + (is_v ? kTileBytes : 0) +
                               h * kHalfBytes + bx * kBoxKeys * 128;
                const CUtensorMap* map = is_v ? &vmap : &kmap;
                if constexpr (kL2Hints)
                    tma_load_5d_hint(dst, map, &b.kv_full[st], 0, it.kvh, off, h, phys_box, keep);
                else
                    tma_load_5d(dst, map, &b.kv_full[st], 0, it.kvh, off, h, phys_box);
            }
            __syncwarp();
            ++gk;
        }
    }
    // before leaving, every issued load has landed (bounded)
    if (lane == 0)
        for (int q = max(0, gk - kStages); q < gk; ++q)
            mbar_wait_bounded(&b.kv_full[q % kStages], (q / kStages) & 1);
}

// MMA issuers: warp 1 for Q tile 0 and warp 15 for Q tile 1, each in
// step; one elected lane issues each MMA and commit, the descriptors stay
// warp-uniform.  A commit tracks the MMAs of the thread that executes it,
// so the barriers both tiles release (a stage's kv_empty, q_free, drain)
// take one commit from each warp.  g counts key tiles over all items: it
// picks the ring stage (g mod kStages) and the S buffer (g mod 2).
template <bool BF16>
__device__ void issue_mmas(const PrefillParams& p, const Bars& b, uint32_t tmem, uint32_t qaddr,
                           uint8_t* stages, const uint32_t* vflags, int t, bool* failed) {
    // one lane issues every MMA and every commit (a commit tracks the MMAs
    // of the thread that executes it)
    const bool leader = tc::elect_one();
    constexpr uint32_t kIdS = tc::f16_idesc(BF16, false, kRows, kKeys);  // K: K-major B
    constexpr uint32_t kIdPV = tc::f16_idesc(BF16, true, kRows, kD);     // V: MN-major B
    constexpr uint32_t kIdPVh = tc::f16_idesc(false, true, kRows, kD);   // V converted to f16
    // descriptor bases; a step's byte offset enters the start-address
    // field (16-byte units, no carry: shared addresses stay below 256 KiB)
    const uint64_t qd0 = tc::sw128_desc(qaddr, 16, 1024);
    const uint64_t sd0 = tc::sw128_desc(smem_addr(stages), 16, 1024);
    const uint64_t vd0 = tc::sw128_desc(smem_addr(stages) + kTileBytes, kHalfBytes, 1024);
    // S = Q K^T of Q tile t for key tile g into S buffer g % 2: 8 steps of
    // 16 dims (4 per 128-byte swizzle atom).  In issue order it follows P V
    // of tile t for key tile g - 2, which reads the P written over that
    // buffer.
    auto issue_s = [&](int t, int g) {
        const uint64_t kd = sd0 + (uint64_t)(((g % kStages) * kStageBytes) >> 4);
        const uint64_t qd = qd0 + (uint64_t)((t * kQTileBytes) >> 4);
        const uint32_t dst = tmem + kTileCols * t + kKeys * (g & 1);
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) {
            const uint32_t off = ((kk >> 2) * kQHalfBytes + (kk & 3) * 32) >> 4;
            const uint32_t koff = ((kk >> 2) * kHalfBytes + (kk & 3) * 32) >> 4;
            if (leader) tc::mma_ss(dst, qd + off, kd + koff, kIdS, kk > 0 ? 1u : 0u);
        }
        if (leader) tc::commit(smem_addr(&b.s_full[2 * t + (g & 1)]));
    };
    // O += P V of Q tile t for key tile g (O = P V for an item's first):
    // 8 steps of 16 keys; V's 8-key groups 1 KiB apart (SBO), its 64-dim
    // halves 16 KiB apart (LBO)
    // A bf16 V tile's 16-key groups are in f16 (flag byte 1: one MMA with
    // the f16 P) or still in bf16 (two MMAs: P's high part and remainder).
    auto issue_pv = [&](int t, int g, bool first, uint32_t flags) {
        const uint64_t vd = vd0 + (uint64_t)(((g % kStages) * kStageBytes) >> 4);
        const uint32_t cs = kTileCols * t, cp = cs + kKeys * (g & 1);
#pragma unroll
        for (int kk = 0; kk < kKeys / 16; ++kk) {
            if (leader) {
                const uint64_t v = vd + kk * (2048 >> 4);
                const uint32_t acc = (!first || kk > 0) ? 1u : 0u;
                if (!BF16 || ((flags >> (8 * kk)) & 1u)) {
                    tc::mma_ts(tmem + cs + kColO, tmem + cp + kk * 8, v, BF16 ? kIdPVh : kIdPV,
                               acc);
                } else {
                    tc::mma_ts(tmem + cs + kColO, tmem + cp + kk * 8, v, kIdPV, acc);
                    tc::mma_ts(tmem + cs + kColO, tmem + cp + kColPl + kk * 8, v, kIdPV, 1u);
                }
            }
        }
        if (leader) tc::commit(smem_addr(&b.o_done[t]));
    };
    auto wait = [&](uint64_t* bar, uint32_t parity) {
        if (!__all_sync(0xffffffffu, mbar_wait_bounded(bar, parity))) {
            *failed = true;
            return false;
        }
        tc::fence_after_sync();
        return true;
    };
    // Per item, S runs two key tiles ahead of P V, so that the tile's
    // softmax finds its next S ready, and the tensor cores take this tile's
    // P V and S while the other tile's softmax runs:
    //   S(0) S(1) | P(j): PV(j) S(j+2)
    // After both tiles' last S, q_free lets the Q warps stage the next item;
    // before an item's first P V overwrites O, o_free says the previous
    // item's output has been read.
    int g0 = 0;  // first key tile of the item, counted over all items
    int nk = 0;  // items run so far
    for (int k = 0; !*failed; ++k) {
        const int idx = item_index(k);
        if (idx >= p.num_items) break;
        const Item it = decode_item(p, idx, false);
        if (!it.run) continue;
        const int nt = it.ntiles;
        if (!wait(b.q_ready, nk & 1)) break;
        for (int j = 0; j < min(nt, 2); ++j) {
            const int g = g0 + j;
            if (!wait(&b.kv_full[g % kStages], (g / kStages) & 1)) break;
            issue_s(t, g);
        }
        if (*failed) break;
        if (nt <= 2 && leader) tc::commit(smem_addr(b.q_free));  // the tile's last S issued
        for (int j = 0; j < nt; ++j) {
            const int g = g0 + j, buf = g & 1;
            if (!wait(&b.p_full[2 * t + buf], (g >> 1) & 1)) break;
            if (j == 0 && nk > 0 && !wait(&b.o_free[t], (nk - 1) & 1)) break;
            // a bf16 V tile converted (it landed before its S)
            if (BF16 && !wait(&b.v_ready[g % kStages], (g / kStages) & 1)) break;
            const uint32_t vf =
                BF16 ? *reinterpret_cast<const volatile uint32_t*>(vflags + g % kStages) : 0u;
            issue_pv(t, g, j == 0, vf);
            if (leader) tc::commit(smem_addr(&b.kv_empty[g % kStages]));  // this tile's P V
            if (j + 2 < nt) {
                if (!wait(&b.kv_full[(g + 2) % kStages], ((g + 2) / kStages) & 1)) break;
                issue_s(t, g + 2);
                if (j + 3 == nt && leader) tc::commit(smem_addr(b.q_free));  // the tile's last S
            }
        }
        // one phase per item: every MMA of this tile so far, its last P V
        // included, completed
        if (!*failed && leader) tc::commit(smem_addr(&b.item_done[t]));
        g0 += nt;
        ++nk;
    }
    // every MMA issued has completed before the tensor memory is freed
    if (nk > 0) {
        if (leader) tc::commit(smem_addr(b.drain));
        mbar_wait_bounded(b.drain, 0);
    }
}

// A bounded wait whose outcome is the same for the whole warp (the
// tensor-memory loads and stores that follow are warp-collective).
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity) {
    const bool ok = mbar_wait_bounded(bar, parity);
    return __all_sync(0xffffffffu, ok);
}

// bf16 V tile -> f16, in place, by the four Q warps (bf16 caches only).
// P V then runs as one f16 MMA per 16 keys: P rounded once to f16 carries
// at most 2^-11 relative error per weight (P <= 2^8, row sum >= 1), where a
// bf16 P alone would need a second MMA for its remainder.  The conversion
// is exact for every bf16 value of magnitude 2^-14 .. 65504 and within
// 2^-25 absolute below.  A 16-key group holding a value of magnitude
// 65536 or more (or an infinity or NaN) stays in bf16 and its P V takes the
// two-part bf16 path, so no input changes the result's accuracy.  Q warp qw
// owns keys 16 qw .. 16 qw + 15 of the tile (2 KiB of each 64-dim half;
// the swizzle permutes 16-byte chunks within a row, so the rows stay put);
// rows at or past `valid` (keys past the context) are zeroed.  Returns the
// group's flag: 1 converted, 0 left in bf16.
__device__ __forceinline__ uint32_t convert_v_group(uint8_t* vt, int qw, int lane, int valid) {
    constexpr int kChunks = 8;  // 16-byte chunks per lane: 4 per 64-dim half
    uint4 v[kChunks];
    uint32_t mx = 0;  // largest magnitude (bf16 bits) of each 16-bit lane, valid rows
#pragma unroll
    for (int i = 0; i < kChunks; ++i) {
        const int row = 16 * qw + (lane >> 3) + 4 * (i & 3);
        v[i] = *reinterpret_cast<const uint4*>(vt + (i >> 2) * kHalfBytes + qw * 2048 +
                                               (lane + 32 * (i & 3)) * 16);
        if (row < valid) {
            const uint32_t w[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
#pragma unroll
            for (int e = 0; e < 4; ++e)
                asm("max.u16x2 %0, %0, %1;" : "+r"(mx) : "r"(w[e] & 0x7fff7fffu));
        }
    }
    // 0x4780 is bf16 65536, the first magnitude beyond f16's 65504
    const bool wide = __any_sync(0xffffffffu, (mx >> 16) >= 0x4780u || (mx & 0xffffu) >= 0x4780u);
#pragma unroll
    for (int i = 0; i < kChunks; ++i) {
        const int row = 16 * qw + (lane >> 3) + 4 * (i & 3);
        uint4 o = make_uint4(0, 0, 0, 0);
        if (row < valid) {
            if (wide) {
                o = v[i];
            } else {
                uint32_t w[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    w[e] = Storage<__half>::from_float2(__uint_as_float(w[e] << 16),
                                                        __uint_as_float(w[e] & 0xffff0000u));
                o = make_uint4(w[0], w[1], w[2], w[3]);
            }
        }
        *reinterpret_cast<uint4*>(vt + (i >> 2) * kHalfBytes + qw * 2048 +
                                  (lane + 32 * (i & 3)) * 16) = o;
    }
    return wide ? 0u : 1u;
}

// Q warps (warps 10-13): per item, once every S MMA of the previous item
// has completed (q_free), Q rows (token r / G, head kvh * G + r % G) are
// copied into shared memory swizzled as the MMA reads them.  Q warp w takes
// rows 64 w .. 64 w + 63; its lane i copies 16-byte chunk i % 16 of rows
// 64 w + i / 16, + 2, ...; all copies are in flight before one wait, and
// rows past the sequence's are zero-filled.
template <typename T>
__device__ void stage_q(const PrefillParams& p, const Bars& b, uint8_t* qsm, uint8_t* stages,
                        uint32_t* vflags, int qw, int lane, bool* failed) {
    constexpr int kRowsPerWarp = kQTiles * kRows / kQWarps;
    const T* qbase = static_cast<const T*>(p.query);
    const int G = p.group, Hq = p.num_q_heads;
    const int ch = lane & 15;
    const uint64_t stream_once = l2_policy_evict_first();  // Q is read once
    int nk = 0;
    int gv = 0;  // V tiles converted over all items
    for (int k = 0; !*failed; ++k) {
        const int idx = item_index(k);
        if (idx >= p.num_items) break;
        const Item it = decode_item(p, idx, false);
        if (!it.run) continue;
        if (nk > 0 && !warp_wait(b.q_free, (nk - 1) & 1)) {
            *failed = true;
            break;
        }
        tc::fence_after_sync();
        int r = kRowsPerWarp * qw + (lane >> 4);  // row of the item's 256
        int tok = (it.r0 + r) / G, g = (it.r0 + r) - tok * G;
        for (; r < kRowsPerWarp * (qw + 1); r += 2) {
            const bool in = it.r0 + r < it.nrows;
            const T* src = qbase + ((int64_t)(it.q0 + (in ? tok : 0)) * Hq + it.kvh * G +
                                    (in ? g : 0)) * kD + ch * 8;
            cp_async_16(qsm + (r / kRows) * kQTileBytes + (ch >> 3) * kQHalfBytes +
                            swz(r % kRows, ch),
                        src, in, stream_once);
            g += 2;  // next row of this lane: two rows on
            while (g >= G) {
                g -= G;
                ++tok;
            }
        }
        cp_async_wait_all();
        tc::fence_proxy_async_smem();  // the tensor cores read Q through the async proxy
        __syncwarp();
        if (lane == 0) mbar_arrive_one(b.q_ready);
        ++nk;
        if constexpr (std::is_same<T, __nv_bfloat16>::value) {
            // the item's V tiles, as they land
            for (int j = 0; j < it.ntiles; ++j, ++gv) {
                const int st = gv % kStages;
                if (!warp_wait(&b.kv_full[st], (gv / kStages) & 1)) {
                    *failed = true;
                    break;
                }
                const uint32_t f = convert_v_group(stages + st * kStageBytes + kTileBytes, qw,
                                                   lane, it.L - j * kKeys);
                tc::fence_proxy_async_smem();  // the tensor cores read V through the async proxy
                if (lane == 0) reinterpret_cast<uint8_t*>(vflags + st)[qw] = (uint8_t)f;
                __syncwarp();
                if (lane == 0) mbar_arrive_one(&b.v_ready[st]);
            }
        }
    }
}

template <typename T>
__device__ void softmax_rows(const PrefillParams& p, const Bars& b, uint32_t tmem,
                             uint8_t* stages, const uint32_t* vflags, int warp, int lane,
                             bool* failed) {
    const int t = (warp - kSoftmaxWarp0) >> 2;  // Q tile of this warp
    const int quarter = warp & 3;              // tensor-memory lanes 32 * quarter .. + 31
    const uint32_t trow = tmem + ((uint32_t)(32 * quarter) << 16) + kTileCols * t;
    const int r = 32 * quarter + lane;
    const float sl = p.scale_log2;
    int g0 = 0;  // first key tile of the item, counted over all items
    int ni = 0;  // items run so far (the phase of item_done)
    for (int k = 0; !*failed; ++k) {
        const int idx = item_index(k);
        if (idx >= p.num_items) break;
        const Item it = decode_item(p, idx, false);
        if (!it.run) continue;
        const int R = it.r0 + kRows * t + r;
        const bool ok = R < it.nrows;
        const int pos = it.L - it.n + (ok ? R / p.group : 0);
        float m = -INFINITY, l = 0.f;
        int j = 0;
        for (; j < it.ntiles; ++j) {
            const int g = g0 + j, buf = g & 1;
            const uint32_t srow = trow + kKeys * buf;  // this key tile's S buffer
            if (!warp_wait(&b.s_full[2 * t + buf], (g >> 1) & 1)) break;
            tc::fence_after_sync();
            // raw scores; the scale (positive) is applied with the max subtraction
            float sv[kKeys];
            {
                uint32_t u[kKeys / 32][32];
#pragma unroll
                for (int c = 0; c < kKeys / 32; ++c) tc::ld32(srow + 32 * c, u[c]);
                tc::wait_ld();
                const int key0 = j * kKeys;
                // the causal mask only where some row of the warp stops inside
                // this tile (or a row is past the sequence's rows)
                if (__all_sync(0xffffffffu, ok && key0 + kKeys - 1 <= pos)) {
#pragma unroll
                    for (int c = 0; c < kKeys / 32; ++c)
#pragma unroll
                        for (int e = 0; e < 32; ++e) sv[32 * c + e] = __uint_as_float(u[c][e]);
                } else {
#pragma unroll
                    for (int c = 0; c < kKeys / 32; ++c)
#pragma unroll
                        for (int e = 0; e < 32; ++e) {
                            const int key = key0 + 32 * c + e;
                            sv[32 * c + e] =
                                (ok && key <= pos) ? __uint_as_float(u[c][e]) : -INFINITY;
                        }
                }
            }
            const float mt = max_tree<kKeys>(sv) * sl;  // the tile's max in base-2 units
            const bool resc = mt > m + kRescaleLog2;    // also the first finite max
            const float alpha = resc ? ex2_approx(m - mt) : 1.f;
            if (resc) m = mt;
            l *= alpha;
            const float mu = m == -INFINITY ? 0.f : m;
            // O changes only after the P V of the previous key tile is done
            // (S of this tile was issued after the P V of tile g - 2, so at
            // most that one P V is outstanding)
            if (j > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
                if (!warp_wait(&b.o_done[t], (g - 1) & 1)) break;
                tc::fence_after_sync();
#pragma unroll 1
                for (int c = 0; c < 4; ++c) {
                    uint32_t o[32];
                    tc::ld32(trow + kColO + 32 * c, o);
                    tc::wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; ++e)
                        o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
                    tc::st32(trow + kColO + 32 * c, o);
                }
            }
            // P = 2^(s - m) on key pairs (packed fp32 FMA, add and subtract);
            // the row sum in four independent packed partial sums.  P enters
            // P V as one f16 rounding (2^-11 relative error per weight, P <=
            // 2^8, row sum >= 1): f16 caches, and bf16 caches whose V group
            // the Q warps converted to f16.  A bf16 group left in bf16 takes
            // P as a bf16 high part and its bf16 remainder (two MMAs): one
            // bf16 rounding alone carries up to 2^-9 per weight.
            constexpr bool kBf16 = std::is_same<T, __nv_bfloat16>::value;
            const float2 sl2 = make_float2(sl, sl), nmu2 = make_float2(-mu, -mu);
            float2 ls[4] = {};
            float2 w[kKeys / 2];
#pragma unroll
            for (int e = 0; e < kKeys / 2; ++e) {
                const float2 x = ffma2(make_float2(sv[2 * e], sv[2 * e + 1]), sl2, nmu2);
                if ((e & 7) < kPolyPairsPer8)
                    w[e] = ex2_poly2(x);
                else
                    w[e] = make_float2(ex2_approx(x.x), ex2_approx(x.y));
                ls[e & 3] = fadd2(ls[e & 3], w[e]);
            }
            // the V groups' format, once the exponentials are done
            uint32_t fl = 0x01010101u;  // one byte per 16-key group: 1 = f16
            if constexpr (kBf16) {
                const int st = g % kStages;
                if (!warp_wait(&b.v_ready[st], (g / kStages) & 1)) break;
                fl = *reinterpret_cast<const volatile uint32_t*>(vflags + st);
            }
#pragma unroll
            for (int c = 0; c < kKeys / 32; ++c) {
                uint32_t hi[16], lo[16];
                const uint32_t pair = (fl >> (16 * c)) & 0x0101u;  // groups 2c, 2c + 1
                if (pair == 0x0101u) {
#pragma unroll
                    for (int e = 0; e < 16; ++e)
                        hi[e] = Storage<__half>::from_float2(w[16 * c + e].x, w[16 * c + e].y);
                    tc::st16(srow + 16 * c, hi);  // over S, already read
                } else {
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        const float2 we = w[16 * c + e];
                        if ((pair >> (8 * (e >> 3))) & 1u) {
                            hi[e] = Storage<__half>::from_float2(we.x, we.y);
                            lo[e] = 0u;
                        } else {
                            hi[e] = Storage<T>::from_float2(we.x, we.y);
                            const float2 rem = fsub2(we, Storage<T>::to_float2(hi[e]));
                            lo[e] = Storage<T>::from_float2(rem.x, rem.y);
                        }
                    }
                    tc::st16(srow + 16 * c, hi);
                    tc::st16(srow + kColPl + 16 * c, lo);
                }
            }
            ls[0] = fadd2(fadd2(ls[0], ls[1]), fadd2(ls[2], ls[3]));
            l += ls[0].x + ls[0].y;
            // keys past the context in the item's last tile: zero their V
            // rows (NaN bit patterns there must not meet their zero weights);
            // the Q warps do it for bf16 caches while converting
            const int key0 = j * kKeys;
            if (!kBf16 && t == 0 && key0 + kKeys > it.L) {
                const int st = g % kStages;
                if (!warp_wait(&b.kv_full[st], (g / kStages) & 1)) break;
                uint8_t* vt = stages + st * kStageBytes + kTileBytes;
                const int first = max(it.L - key0, 0);
                const int tid = (warp - kSoftmaxWarp0) * 32 + lane;  // tile 0's 128 threads
                for (int c = tid; c < (kKeys - first) * 16; c += 4 * 32) {
                    const int kr = first + (c >> 4), cc = c & 15;
                    *reinterpret_cast<uint4*>(vt + (cc >> 3) * kHalfBytes + swz(kr, cc)) =
                        make_uint4(0, 0, 0, 0);
                }
                tc::fence_proxy_async_smem();
            }
            tc::wait_st();
            tc::fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive_one(&b.p_full[2 * t + buf]);
        }
        // The item's last P V, through item_done (phase ni, one per item;
        // the next needs this item's o_free, so the wait cannot alias).  A
        // parity wait is sound only while its barrier is at most one phase
        // past the phase waited for; o_done, one phase per key tile, can
        // here be one or two phases past P V ge - 2.
        const int ge = g0 + it.ntiles;
        if (j < it.ntiles || !warp_wait(&b.item_done[t], ni & 1)) {
            *failed = true;
            break;
        }
        tc::fence_after_sync();
        // every lane takes part in the (warp-collective) tensor-memory loads;
        // only rows of this sequence are stored
        const int tok = ok ? R / p.group : 0, gh = ok ? R - tok * p.group : 0;
        T* dst = static_cast<T*>(p.out) +
                 ((int64_t)(it.q0 + tok) * p.num_q_heads + it.kvh * p.group + gh) * kD;
        const float inv = l > 0.f ? 1.f / l : 0.f;
        const uint64_t write_once = l2_policy_evict_first();
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
            uint32_t o[32];
            tc::ld32(trow + kColO + 32 * c, o);
            tc::wait_ld();
            uint32_t pk[16];
#pragma unroll
            for (int e = 0; e < 16; ++e)
                pk[e] = Storage<T>::from_float2(__uint_as_float(o[2 * e]) * inv,
                                                __uint_as_float(o[2 * e + 1]) * inv);
            if (ok) {
#pragma unroll
                for (int v = 0; v < 4; ++v) {
                    const uint4 w = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2],
                                               pk[4 * v + 3]);
                    if constexpr (kL2Hints)
                        st_global_v4_hint(reinterpret_cast<uint4*>(dst + 32 * c) + v, w,
                                          write_once);
                    else
                        reinterpret_cast<uint4*>(dst + 32 * c)[v] = w;
                }
            }
        }
        // O has been read: the next item's first P V may overwrite it
        tc::fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive_one(&b.o_free[t]);
        g0 = ge;
        ++ni;
    }
}

template <typename T>
__global__ void __launch_bounds__(kThreads, 1)
paged_prefill_kernel(const __grid_constant__ CUtensorMap kmap,
                     const __grid_constant__ CUtensorMap vmap, const PrefillParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align_1024(smem_raw);
    uint8_t* qsm = smem;
    uint8_t* stages = smem + kQBytes;
    uint64_t* bars = reinterpret_cast<uint64_t*>(stages + kStages * kStageBytes);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + kNumBars);
    uint32_t* vflags = tmem_slot + 4;  // [kStages]: four group bytes each
    uint64_t* sp = bars + 3 * kStages;
    uint64_t* tail = sp + 6 * kQTiles;
    Bars b{bars,
           bars + kStages,
           bars + 2 * kStages,
           sp,
           sp + 2 * kQTiles,
           sp + 4 * kQTiles,
           sp + 5 * kQTiles,
           tail,
           tail + 1,
           tail + 2,
           tail + 3};
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (warp == kProducerWarp) {
        tc::tmem_alloc(smem_addr(tmem_slot), kTmemCols);
        tc::tmem_relinquish();
    }
    if (threadIdx.x == 32 * kMmaWarp) {
        for (int i = 0; i < kStages; ++i) {
            mbar_init(&b.kv_full[i], 2);  // the K and the V producer
            mbar_init(&b.kv_empty[i], 2);  // the P V of each Q tile
            mbar_init(&b.v_ready[i], kQWarps);
        }
        for (int t = 0; t < kQTiles; ++t) {
            for (int u = 0; u < 2; ++u) {
                mbar_init(&b.s_full[2 * t + u], 1);
                mbar_init(&b.p_full[2 * t + u], 4);  // the tile's four softmax warps
            }
            mbar_init(&b.o_done[t], 1);
            mbar_init(&b.o_free[t], 4);  // the tile's four softmax warps
            mbar_init(&b.item_done[t], 1);
        }
        mbar_init(b.drain, 2);     // both MMA warps
        mbar_init(b.q_ready, kQWarps);  // the Q warps
        mbar_init(b.q_free, 2);   // a commit after each Q tile's last S
        fence_barrier_init();
        prefetch_tensormap(&kmap);
        prefetch_tensormap(&vmap);
    }
    tc::fence_before_sync();
    __syncthreads();  // barriers initialised, tensor memory allocated
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_slot;

    bool failed = false;
    if (warp == kProducerWarp || warp == kVProducerWarp)
        produce(kmap, vmap, p, stages, b, lane, warp == kVProducerWarp, &failed);
    else if (warp == kMmaWarp || warp == kMmaWarpB)
        issue_mmas<std::is_same<T, __nv_bfloat16>::value>(p, b, tmem, smem_addr(qsm), stages,
                                                          vflags, warp == kMmaWarpB, &failed);
    else if (warp >= kQWarp0 && warp < kQWarp0 + kQWarps)
        stage_q<T>(p, b, qsm, stages, vflags, warp - kQWarp0, lane, &failed);
    else
        softmax_rows<T>(p, b, tmem, stages, vflags, warp, lane, &failed);
    if (failed) report_error(p.dev_error, PKV_DEVERR_TIMEOUT, 0);
    tc::fence_before_sync();
    __syncthreads();
    if (warp == kProducerWarp) {
        __syncwarp();
        tc::fence_after_sync();
        tc::tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace
}  // namespace pkv

extern "C" int pkv_prefill_attention(void* out, const void* query, const void* key_cache,
                                     const void* value_cache, const int32_t* block_tables,
                                     int max_blocks_per_seq, const int32_t* context_lens,
                                     const int32_t* query_start, int num_seqs,
                                     int max_query_len, int num_q_heads, int num_kv_heads,
                                     int head_dim, int num_blocks, int block_size,
                                     int64_t block_stride, float scale, pkv_dtype dtype,
                                     int32_t* dev_error, cudaStream_t stream) {
    PKV_NVTX_RANGE("pkv_prefill_attention");
    using namespace pkv;
    PKV_REQUIRE(dtype == PKV_F16 || dtype == PKV_BF16, PKV_ERR_UNSUPPORTED,
                "pkv_prefill_attention: dtype %d", (int)dtype);
    PKV_REQUIRE(head_dim == kD, PKV_ERR_UNSUPPORTED,
                "pkv_prefill_attention: head_dim %d (built: 128)", head_dim);
    PKV_REQUIRE(scale > 0.f, PKV_ERR_INVALID, "pkv_prefill_attention: scale %g (must be > 0)",
                (double)scale);
    PKV_REQUIRE(num_seqs >= 0 && max_query_len >= 0 && num_q_heads > 0 && num_kv_heads > 0 &&
                    num_q_heads % num_kv_heads == 0 && max_blocks_per_seq >= 0,
                PKV_ERR_INVALID, "pkv_prefill_attention: bad sizes");
    PKV_REQUIRE(block_size > 0 && block_size % kBoxKeys == 0, PKV_ERR_UNSUPPORTED,
                "pkv_prefill_attention: block_size %d (a multiple of 16)", block_size);
    const int64_t block_elems = (int64_t)block_size * num_kv_heads * head_dim;
    PKV_REQUIRE(block_stride >= block_elems && block_stride % 8 == 0, PKV_ERR_INVALID,
                "pkv_prefill_attention: block_stride %lld", (long long)block_stride);
    if (num_seqs == 0 || max_query_len == 0) return PKV_OK;
    PKV_REQUIRE(out && query && key_cache && value_cache && block_tables && context_lens &&
                    query_start && num_blocks > 0,
                PKV_ERR_INVALID, "pkv_prefill_attention: NULL pointer or empty pool");
    PKV_REQUIRE(aligned16(out) && aligned16(query) && aligned16(key_cache) &&
                    aligned16(value_cache),
                PKV_ERR_INVALID, "pkv_prefill_attention: pointers must be 16-byte aligned");
    PrefillParams p;
    p.out = out;
    p.query = query;
    p.block_tables = block_tables;
    p.context_lens = context_lens;
    p.query_start = query_start;
    p.dev_error = dev_error;
    p.num_seqs = num_seqs;
    p.max_blocks_per_seq = max_blocks_per_seq;
    p.num_q_heads = num_q_heads;
    p.num_kv_heads = num_kv_heads;
    p.group = num_q_heads / num_kv_heads;
    p.num_blocks = num_blocks;
    p.block_size = block_size;
    p.max_query_len = max_query_len;
    p.tiles_per_seq =
        (int)(((int64_t)max_query_len * p.group + kRows * kQTiles - 1) / (kRows * kQTiles));
    p.scale_log2 = scale * kLog2e;
    const int64_t items = (int64_t)p.tiles_per_seq * num_seqs * num_kv_heads;
    PKV_REQUIRE(items < (1ll << 31), PKV_ERR_UNSUPPORTED, "pkv_prefill_attention: %lld row tiles",
                (long long)items);
    p.num_items = (int)items;
    CUtensorMap kmap, vmap;
    int st = encode_paged_map_16bit(&kmap, key_cache, dtype, head_dim, num_kv_heads, block_size,
                                    num_blocks, block_stride, 1);
    if (st != PKV_OK) return st;
    st = encode_paged_map_16bit(&vmap, value_cache, dtype, head_dim, num_kv_heads, block_size,
                                num_blocks, block_stride, 1);
    if (st != PKV_OK) return st;
    DeviceGuard guard(stream, key_cache);
    auto kern = dtype == PKV_BF16 ? paged_prefill_kernel<__nv_bfloat16>
                                  : paged_prefill_kernel<__half>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kSmemBytes);
    if (e != cudaSuccess)
        return fail(PKV_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
    // persistent CTAs: one per SM, at most one per row tile
    int dev = 0, sms = 0;
    e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess || sms <= 0)
        return fail(PKV_ERR_CUDA, "pkv_prefill_attention: SM count: %s", cudaGetErrorString(e));
    const int ctas = (int)std::min<int64_t>(items, sms);
    kern<<<(unsigned)ctas, kThreads, kSmemBytes, stream>>>(kmap, vmap, p);
    return launch_status("pkv_prefill_attention");
}
