// prefill_attention.cu — paged prefill attention ("Paged KV" wiki page,
// 实现原理 / 运行阶段: prefill takes blocks in order and fills them with the
// prompt's K/V; the prompt's tokens then attend over the sequence through
// the same Block Table, as decode does with one token).
//
// Sequence s has n_s query rows (query_start[s] .. query_start[s+1]-1), the
// last n_s of its L_s cached tokens: row i is token p = L_s - n_s + i and
// attends causally to tokens 0 .. p.
//
// One CTA takes 256 rows of one (sequence, KV head) as two 128-row Q tiles:
// (query token, head of the GQA group) pairs, so each K/V tile is streamed
// once for the group and both tiles.
// The work runs on the 5th-generation tensor cores with the accumulators in
// tensor memory:
//   - a producer warp brings 64-key K and V tiles through a 4-stage ring
//     (one TMA box per 16 slots of a block and per 64-dim half);
//   - an MMA warp issues, per key tile, S = Q K^T for both Q tiles (M 128,
//     N 64, K 16 steps; Q and K from shared memory) into tensor memory,
//     then O += P V for each tile as its P is ready (P read from tensor
//     memory, V from shared memory as an MN-major B operand), so that the
//     tensor cores work on one tile while the other tile's softmax runs;
//   - eight softmax warps, four per Q tile (one tensor-memory lane quarter
//     each, one row per thread), read S, apply the causal mask, keep the
//     running max and sum, write P over S (a 16-bit high part and its
//     16-bit remainder, two MMAs) and rescale O when the running max grows
//     by more than 2^8, then write the normalised output.
#include <cudaTypedefs.h>

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
constexpr int kThreads = (kSoftmaxWarp0 + kSoftmaxWarps) * 32;
// tensor-memory columns per Q tile t: two S buffers (64 columns each; P
// high | P low, 32 each, written over S once it is read) at 256 t and
// 256 t + 64, O at 256 t + 128; key tile j uses S buffer j % 2
constexpr uint32_t kTileCols = 256, kColO = 128, kColPl = kKeys / 2, kTmemCols = 512;
constexpr int kNumBars = 2 * kStages + 5 * kQTiles + 2;  // kv_full/empty, s_full/p_full per (tile, buffer), o_done per tile, drain, q_ready
constexpr size_t kSmemBytes = 1024 + kQBytes + kStages * kStageBytes + kNumBars * 8 + 16;
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

// 16-byte copy global -> shared that does not wait (cp.async, L2 only);
// when copy is false, the destination is zero-filled and nothing is read
__device__ __forceinline__ void cp_async_16(void* dst, const void* src, bool copy) {
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
    uint64_t* s_full;    // [kQTiles][2]: S of the buffer in tensor memory
    uint64_t* p_full;    // [kQTiles][2]: P of the buffer written (and O rescaled)
    uint64_t* o_done;    // [kQTiles]: the P V MMAs of the tile completed
    uint64_t* drain;     // every MMA issued completed (exit)
    uint64_t* q_ready;   // the Q tiles are staged (every staging warp arrived)
};

// Producer: warp 0.  A box past the context still loads a block (the last
// one) so that every stage receives its full byte count; those rows are
// masked (K) or zeroed (V) downstream.  The block ids come from the Block
// Table one warp-wide load per eight key tiles (lane i: the id of box i of
// the window), handed to lane 0, which issues the TMA loads, by shuffles.
__device__ void produce(const CUtensorMap& kmap, const CUtensorMap& vmap, const PrefillParams& p,
                        int s, int kvh, int L, int ntiles, uint8_t* stages, const Bars& b,
                        int lane, bool* failed) {
    constexpr int kBoxes = kKeys / kBoxKeys;       // TMA boxes per key tile and 64-dim half
    constexpr int kWindowTiles = 32 / kBoxes;      // key tiles per warp-wide block-id load
    const int bs = p.block_size;
    const int32_t* row = p.block_tables + (int64_t)s * p.max_blocks_per_seq;
    const int last_block = L > 0 ? (L - 1) / bs : 0;
    int phys_lane = 0;
    int issued = 0;
    for (int j = 0; j < ntiles; ++j) {
        if (j % kWindowTiles == 0) {
            const int box = j * kBoxes + lane;  // box of this lane in the window
            phys_lane = __ldg(row + min(box * kBoxKeys / bs, last_block));
            if (box < ntiles * kBoxes && (phys_lane < 0 || phys_lane >= p.num_blocks))
                report_error(p.dev_error, PKV_DEVERR_BLOCK_ID, s);
        }
        const int st = j % kStages;
        if (j >= kStages &&
            !__all_sync(0xffffffffu,
                        mbar_wait_bounded(&b.kv_empty[st], ((j / kStages) - 1) & 1))) {
            *failed = true;
            break;
        }
        int phys[kBoxes];
#pragma unroll
        for (int bx = 0; bx < kBoxes; ++bx)
            phys[bx] = __shfl_sync(0xffffffffu, phys_lane, (j % kWindowTiles) * kBoxes + bx);
        if (lane == 0) {
            uint8_t* kdst = stages + st * kStageBytes;
            uint8_t* vdst = kdst + kTileBytes;
            mbar_arrive_expect_tx(&b.kv_full[st], kStageBytes);
#pragma unroll
            for (int bx = 0; bx < kBoxes; ++bx) {
                const int key0 = j * kKeys + bx * kBoxKeys;
                const int off = key0 < L ? key0 % bs : 0;
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    tma_load_5d(kdst + h * kHalfBytes + bx * kBoxKeys * 128, &kmap,
                                &b.kv_full[st], 0, kvh, off, h, phys[bx]);
                    tma_load_5d(vdst + h * kHalfBytes + bx * kBoxKeys * 128, &vmap,
                                &b.kv_full[st], 0, kvh, off, h, phys[bx]);
                }
            }
        }
        __syncwarp();
        ++issued;
    }
    // before leaving, every issued load has landed (bounded)
    if (lane == 0)
        for (int j = max(0, issued - kStages); j < issued; ++j)
            mbar_wait_bounded(&b.kv_full[j % kStages], (j / kStages) & 1);
}

// MMA issuer: warp 1, in step; one elected lane issues each MMA and commit,
// the descriptors stay warp-uniform.
template <bool BF16>
__device__ void issue_mmas(const Bars& b, uint32_t tmem, uint32_t qaddr, uint8_t* stages,
                           int ntiles, bool* failed) {
    // one lane issues every MMA and every commit (a commit tracks the MMAs
    // of the thread that executes it)
    const bool leader = tc::elect_one();
    constexpr uint32_t kIdS = tc::f16_idesc(BF16, false, kRows, kKeys);  // K: K-major B
    constexpr uint32_t kIdPV = tc::f16_idesc(BF16, true, kRows, kD);     // V: MN-major B
    // S = Q K^T of Q tile t for key tile j into S buffer j % 2: 8 steps of
    // 16 dims (4 per 128-byte swizzle atom).  In issue order it follows P V
    // of tile t for key tile j - 2, which reads the P written over that
    // buffer.
    // descriptor bases; a step's byte offset enters the start-address
    // field (16-byte units, no carry: shared addresses stay below 256 KiB)
    const uint64_t qd0 = tc::sw128_desc(qaddr, 16, 1024);
    const uint64_t sd0 = tc::sw128_desc(smem_addr(stages), 16, 1024);
    const uint64_t vd0 = tc::sw128_desc(smem_addr(stages) + kTileBytes, kHalfBytes, 1024);
    auto issue_s = [&](int t, int j) {
        const uint64_t kd = sd0 + (uint64_t)(((j % kStages) * kStageBytes) >> 4);
        const uint64_t qd = qd0 + (uint64_t)((t * kQTileBytes) >> 4);
        const uint32_t dst = tmem + kTileCols * t + kKeys * (j & 1);
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) {
            const uint32_t off = ((kk >> 2) * kQHalfBytes + (kk & 3) * 32) >> 4;
            const uint32_t koff = ((kk >> 2) * kHalfBytes + (kk & 3) * 32) >> 4;
            if (leader) tc::mma_ss(dst, qd + off, kd + koff, kIdS, kk > 0 ? 1u : 0u);
        }
        if (leader) tc::commit(smem_addr(&b.s_full[2 * t + (j & 1)]));
    };
    // O += P V of Q tile t for key tile j: 8 steps of 16 keys; V's 8-key
    // groups 1 KiB apart (SBO), its 64-dim halves 16 KiB apart (LBO)
    auto issue_pv = [&](int t, int j) {
        const uint64_t vd = vd0 + (uint64_t)(((j % kStages) * kStageBytes) >> 4);
        const uint32_t cs = kTileCols * t, cp = cs + kKeys * (j & 1);
#pragma unroll
        for (int kk = 0; kk < kKeys / 16; ++kk) {
            if (leader) {
                tc::mma_ts(tmem + cs + kColO, tmem + cp + kk * 8, vd + kk * (2048 >> 4),
                               kIdPV, (j > 0 || kk > 0) ? 1u : 0u);
                tc::mma_ts(tmem + cs + kColO, tmem + cp + kColPl + kk * 8,
                               vd + kk * (2048 >> 4), kIdPV, 1u);
            }
        }
        if (leader) tc::commit(smem_addr(&b.o_done[t]));
    };
    // S runs two key tiles ahead of P V, so that a tile's softmax finds its
    // next S ready, and the tensor cores take one tile's P V and S while the
    // other tile's softmax runs:
    //   S_A(0) S_B(0) S_A(1) S_B(1) | P_A(j): PV_A(j) S_A(j+2) | P_B(j): PV_B(j) S_B(j+2)
    for (int j = 0; j < min(ntiles, 2) && !*failed; ++j) {
        if (!__all_sync(0xffffffffu, mbar_wait_bounded(&b.kv_full[j], 0))) {
            *failed = true;
            break;
        }
        tc::fence_after_sync();
        issue_s(0, j);
        issue_s(1, j);
    }
    for (int j = 0; j < ntiles && !*failed; ++j) {
        const int st = j % kStages, buf = j & 1;
        const uint32_t ph = (j >> 1) & 1;
        const bool more = j + 2 < ntiles;
        // tile A
        if (!__all_sync(0xffffffffu, mbar_wait_bounded(&b.p_full[buf], ph))) {
            *failed = true;
            break;
        }
        tc::fence_after_sync();
        issue_pv(0, j);
        if (more) {
            if (!__all_sync(0xffffffffu, mbar_wait_bounded(&b.kv_full[(j + 2) % kStages],
                                                           ((j + 2) / kStages) & 1))) {
                *failed = true;
                break;
            }
            tc::fence_after_sync();
            issue_s(0, j + 2);
        }
        // tile B
        if (!__all_sync(0xffffffffu, mbar_wait_bounded(&b.p_full[2 + buf], ph))) {
            *failed = true;
            break;
        }
        tc::fence_after_sync();
        issue_pv(1, j);
        if (leader) tc::commit(smem_addr(&b.kv_empty[st]));  // both tiles' P V of this stage
        if (more) issue_s(1, j + 2);
    }
    // every MMA issued has completed before the tensor memory is freed
    if (leader) tc::commit(smem_addr(b.drain));
    mbar_wait_bounded(b.drain, 0);
}

// A bounded wait whose outcome is the same for the whole warp (the
// tensor-memory loads and stores that follow are warp-collective).
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity) {
    const bool ok = mbar_wait_bounded(bar, parity);
    return __all_sync(0xffffffffu, ok);
}

template <typename T>
__device__ void softmax_rows(const PrefillParams& p, const Bars& b, uint32_t tmem,
                             uint8_t* stages, int L, int n, int q0, int kvh, int r0, int nrows,
                             int ntiles, int warp, int lane, bool* failed) {
    const int t = (warp - kSoftmaxWarp0) >> 2;  // Q tile of this warp
    const int quarter = warp & 3;              // tensor-memory lanes 32 * quarter .. + 31
    const uint32_t trow = tmem + ((uint32_t)(32 * quarter) << 16) + kTileCols * t;
    const int r = 32 * quarter + lane;
    const int R = r0 + kRows * t + r;
    const bool ok = R < nrows;
    const int pos = L - n + (ok ? R / p.group : 0);
    const float sl = p.scale_log2;
    float m = -INFINITY, l = 0.f;
    int j = 0;
    for (; j < ntiles; ++j) {
        const int buf = j & 1;
        const uint32_t srow = trow + kKeys * buf;  // this key tile's S buffer
        if (!warp_wait(&b.s_full[2 * t + buf], (j >> 1) & 1)) break;
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
                        sv[32 * c + e] = (ok && key <= pos) ? __uint_as_float(u[c][e]) : -INFINITY;
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
        // (S of this tile was issued after the P V of tile j - 2, so at
        // most that one P V is outstanding)
        if (j > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
            if (!warp_wait(&b.o_done[t], (j - 1) & 1)) break;
            tc::fence_after_sync();
            {
#pragma unroll 1
                for (int c = 0; c < 4; ++c) {
                    uint32_t o[32];
                    tc::ld32(trow + kColO + 32 * c, o);
                    tc::wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
                    tc::st32(trow + kColO + 32 * c, o);
                }
            }
        }
        // P = 2^(s - m) as a 16-bit high part and the 16-bit remainder, on
        // key pairs (packed fp32 FMA, add and subtract); the row sum in four
        // independent packed partial sums
        const float2 sl2 = make_float2(sl, sl), nmu2 = make_float2(-mu, -mu);
        float2 ls[4] = {};
#pragma unroll
        for (int c = 0; c < kKeys / 32; ++c) {
            uint32_t hi[16], lo[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) {
                const float2 x =
                    ffma2(make_float2(sv[32 * c + 2 * e], sv[32 * c + 2 * e + 1]), sl2, nmu2);
                const float2 w = make_float2(ex2_approx(x.x), ex2_approx(x.y));
                ls[e & 3] = fadd2(ls[e & 3], w);
                hi[e] = Storage<T>::from_float2(w.x, w.y);
                const float2 rem = fsub2(w, Storage<T>::to_float2(hi[e]));
                lo[e] = Storage<T>::from_float2(rem.x, rem.y);
            }
            tc::st16(srow + 16 * c, hi);  // over S, already read
            tc::st16(srow + kColPl + 16 * c, lo);
        }
        ls[0] = fadd2(fadd2(ls[0], ls[1]), fadd2(ls[2], ls[3]));
        l += ls[0].x + ls[0].y;
        // keys past the context in the last tile: zero their V rows (NaN
        // bit patterns there must not meet their zero weights)
        const int key0 = j * kKeys;
        if (t == 0 && key0 + kKeys > L) {
            const int st = j % kStages;
            if (!warp_wait(&b.kv_full[st], (j / kStages) & 1)) break;
            uint8_t* vt = stages + st * kStageBytes + kTileBytes;
            const int first = max(L - key0, 0);
            const int tid = (warp - kSoftmaxWarp0) * 32 + lane;  // tile 0's 128 threads
            for (int c = tid; c < (kKeys - first) * 16; c += 4 * 32) {
                const int k = first + (c >> 4), ch = c & 15;
                *reinterpret_cast<uint4*>(vt + (ch >> 3) * kHalfBytes + swz(k, ch)) =
                    make_uint4(0, 0, 0, 0);
            }
            tc::fence_proxy_async_smem();
        }
        tc::wait_st();
        tc::fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive_one(&b.p_full[2 * t + buf]);
    }
    // the last two P V (phases ntiles - 2 and ntiles - 1 of o_done), in order
    if (j < ntiles || (ntiles >= 2 && !warp_wait(&b.o_done[t], (ntiles - 2) & 1)) ||
        !warp_wait(&b.o_done[t], (ntiles - 1) & 1)) {
        *failed = true;
        return;
    }
    tc::fence_after_sync();
    // every lane takes part in the (warp-collective) tensor-memory loads;
    // only rows of this sequence are stored
    const int tok = ok ? R / p.group : 0, g = ok ? R - tok * p.group : 0;
    T* dst = static_cast<T*>(p.out) + ((int64_t)(q0 + tok) * p.num_q_heads + kvh * p.group + g) * kD;
    const float inv = l > 0.f ? 1.f / l : 0.f;
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
            for (int v = 0; v < 4; ++v)
                reinterpret_cast<uint4*>(dst + 32 * c)[v] =
                    make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
        }
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
    Bars b{bars, bars + kStages, bars + 2 * kStages, bars + 2 * kStages + 2 * kQTiles,
           bars + 2 * kStages + 4 * kQTiles, bars + 2 * kStages + 5 * kQTiles,
           bars + 2 * kStages + 5 * kQTiles + 1};

    // flat grid: the heaviest row tile of every (sequence, KV head) first
    const int pairs = p.num_seqs * p.num_kv_heads;
    const int tile = p.tiles_per_seq - 1 - (int)(blockIdx.x / (unsigned)pairs);
    const int rest = (int)(blockIdx.x % (unsigned)pairs);
    const int kvh = rest % p.num_kv_heads, s = rest / p.num_kv_heads;
    const int G = p.group;
    const int q0 = __ldg(p.query_start + s);
    const int n = __ldg(p.query_start + s + 1) - q0;
    const int L = __ldg(p.context_lens + s);
    const int nrows = n * G;
    const int r0 = tile * kRows * kQTiles;
    if (n < 0 || n > L || n > p.max_query_len ||
        (int64_t)L > (int64_t)p.max_blocks_per_seq * p.block_size) {
        if (tile == p.tiles_per_seq - 1 && kvh == 0 && threadIdx.x == 0)
            report_error(p.dev_error, PKV_DEVERR_CONTEXT_LEN, s);
        return;
    }
    if (r0 >= nrows) return;  // a row tile past this sequence's rows
    const int last_row = min(nrows, r0 + kRows * kQTiles) - 1;
    const int kv_end = L - n + last_row / G + 1;
    const int ntiles = (kv_end + kKeys - 1) / kKeys;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (warp == kProducerWarp) {
        tc::tmem_alloc(smem_addr(tmem_slot), kTmemCols);
        tc::tmem_relinquish();
    }
    if (threadIdx.x == 32 * kMmaWarp) {
        for (int i = 0; i < kStages; ++i) {
            mbar_init(&b.kv_full[i], 1);
            mbar_init(&b.kv_empty[i], 1);
        }
        for (int t = 0; t < kQTiles; ++t) {
            for (int u = 0; u < 2; ++u) {
                mbar_init(&b.s_full[2 * t + u], 1);
                mbar_init(&b.p_full[2 * t + u], 4);  // the tile's four softmax warps
            }
            mbar_init(&b.o_done[t], 1);
        }
        mbar_init(b.drain, 1);
        mbar_init(b.q_ready, kThreads / 32 - 1);  // every warp but the producer
        fence_barrier_init();
        prefetch_tensormap(&kmap);
        prefetch_tensormap(&vmap);
    }
    tc::fence_before_sync();
    __syncthreads();  // barriers initialised, tensor memory allocated
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_slot;

    bool failed = false;
    if (warp == kProducerWarp) {
        // K/V do not depend on Q: stream them while the other warps stage it
        produce(kmap, vmap, p, s, kvh, L, ntiles, stages, b, lane, &failed);
    } else {
        // Q rows (token r / G, head kvh * G + r % G), swizzled as the MMA
        // reads them, staged by every warp but the producer: each thread
        // issues all its 16-byte copies (zero-filled past the sequence's
        // rows) before waiting, so the CTA pays one memory latency
        const int Hq = p.num_q_heads;
        const T* qbase = static_cast<const T*>(p.query);
        for (int c = threadIdx.x - 32; c < kQTiles * kRows * (kD / 8); c += kThreads - 32) {
            const int r = c >> 4, ch = c & 15;  // r: row of the CTA's 256
            const int row = r0 + r;
            const bool in = row < nrows;
            const int tok = in ? row / G : 0, g = in ? row - tok * G : 0;
            const T* src = qbase + ((int64_t)(q0 + tok) * Hq + kvh * G + g) * kD + ch * 8;
            cp_async_16(qsm + (r / kRows) * kQTileBytes + (ch >> 3) * kQHalfBytes +
                            swz(r % kRows, ch),
                        src, in);
        }
        cp_async_wait_all();
        tc::fence_proxy_async_smem();  // the tensor cores read Q through the async proxy
        __syncwarp();
        if (lane == 0) mbar_arrive_one(b.q_ready);
        if (warp == kMmaWarp) {
            if (!__all_sync(0xffffffffu, mbar_wait_bounded(b.q_ready, 0))) {
                failed = true;
            } else {
                tc::fence_after_sync();
                issue_mmas<std::is_same<T, __nv_bfloat16>::value>(b, tmem, smem_addr(qsm), stages,
                                                                  ntiles, &failed);
            }
        } else {
            softmax_rows<T>(p, b, tmem, stages, L, n, q0, kvh, r0, nrows, ntiles, warp, lane,
                            &failed);
        }
    }
    if (failed) report_error(p.dev_error, PKV_DEVERR_TIMEOUT, s);
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
    const int64_t ctas = (int64_t)p.tiles_per_seq * num_seqs * num_kv_heads;
    PKV_REQUIRE(ctas < (1ll << 31), PKV_ERR_UNSUPPORTED, "pkv_prefill_attention: %lld CTAs",
                (long long)ctas);
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
    kern<<<(unsigned)ctas, kThreads, kSmemBytes, stream>>>(kmap, vmap, p);
    return launch_status("pkv_prefill_attention");
}
