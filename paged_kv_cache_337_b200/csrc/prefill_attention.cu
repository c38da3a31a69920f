// prefill_attention.cu — paged prefill attention ("Paged KV" wiki page,
// 实现原理 / 运行阶段: prefill takes blocks in order and fills them with the
// prompt's K/V; the prompt's tokens then attend over the sequence through
// the same Block Table, as decode does with one token).
//
// Sequence s has n_s query rows (query_start[s] .. query_start[s+1]-1), the
// last n_s of its L_s cached tokens: row i is token p = L_s - n_s + i and
// attends causally to tokens 0 .. p.  A whole prompt has n_s = L_s; a later
// chunk of a long prompt has n_s < L_s.
//
// One CTA takes 64 rows of one (sequence, KV head): the rows are (query
// token, head of the GQA group) pairs, so the K/V tile the CTA streams is
// shared by the group's heads.  A producer warp brings 64-key K and V tiles
// through a 2-stage ring (one 5-D TMA box per 16 slots of a block; block
// size a multiple of 16), and four consumer warps each own 16 rows:
// S = Q K^T and O += P V on mma.sync m16n8k16 with fp32 accumulators, the
// online softmax in base 2, and the causal mask as a per-row select.  The
// grid is flat and dispatches every sequence's last (heaviest) row tile
// first.  Bound: the tensor pipe for long prompts.
#include <cudaTypedefs.h>

#include "common.cuh"
#include "tensor_maps.h"

namespace pkv {
namespace {

constexpr int kD = 128;                          // head_dim (built)
constexpr int kRows = 64;                        // (token, head) rows per CTA
constexpr int kKeys = 64;                        // keys per tile
constexpr int kConsumers = 4;                    // warps of 16 rows
constexpr int kThreads = (kConsumers + 1) * 32;  // + the producer warp
constexpr int kStages = 2;
constexpr int kBoxKeys = 16;                          // slots per TMA box
constexpr int kBoxBytes = kBoxKeys * kD * 2;          // 4 KiB: two 16 x 128 B sub-tiles
constexpr int kTileBytes = kKeys * kD * 2;            // 16 KiB of K (or V)
constexpr int kStageBytes = 2 * kTileBytes;           // K + V
constexpr int kQBytes = kRows * kD * 2;               // 16 KiB
constexpr size_t kSmemBytes = 1024 + kQBytes + kStages * kStageBytes + (2 * kStages + 1) * 8;
constexpr float kLog2e = 1.4426950408889634f;
constexpr unsigned kFull = 0xffffffffu;

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

// byte offset of (row, 16-byte chunk) in a swizzled tile of 16-row x 128-B
// sub-tiles (the layout one TMA box lands in; chunk >> 3 picks the 64-dim half)
__device__ __forceinline__ uint32_t swz16(int r, int chunk) {
    return (chunk >> 3) * (kBoxKeys * 128) + r * 128 + (((chunk & 7) ^ (r & 7)) << 4);
}

// the Q tile: two 64-row x 128-B halves, swizzled the same way
__device__ __forceinline__ uint32_t swz_q(int r, int chunk) {
    return (chunk >> 3) * (kRows * 128) + r * 128 + (((chunk & 7) ^ (r & 7)) << 4);
}

__device__ __forceinline__ uint8_t* align_1024(uint8_t* p) {
    const uint32_t a = smem_addr(p);
    return p + ((1024u - (a & 1023u)) & 1023u);
}

__device__ __forceinline__ void mbar_arrive_one(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

// The producer: lane 0 of the last warp streams the K and V tiles of keys
// [0, kv_end) into the ring.  A box past the context still loads a block
// (the last one) so that every stage receives its full byte count; its rows
// are masked (K) or zeroed (V) by the consumers.
__device__ void produce(const CUtensorMap& kmap, const CUtensorMap& vmap, const PrefillParams& p,
                        int s, int kvh, int L, int ntiles, uint8_t* stages, uint64_t* full,
                        uint64_t* empty) {
    const int bs = p.block_size;
    const int32_t* row = p.block_tables + (int64_t)s * p.max_blocks_per_seq;
    const int last_block = L > 0 ? (L - 1) / bs : 0;
    for (int j = 0; j < ntiles; ++j) {
        const int st = j % kStages;
        if (j >= kStages && !mbar_wait_bounded(&empty[st], ((j / kStages) - 1) & 1)) {
            report_error(p.dev_error, PKV_DEVERR_TIMEOUT, s);
            return;
        }
        uint8_t* kdst = stages + st * kStageBytes;
        uint8_t* vdst = kdst + kTileBytes;
        mbar_arrive_expect_tx(&full[st], kStageBytes);
#pragma unroll
        for (int b = 0; b < kKeys / kBoxKeys; ++b) {
            const int key0 = j * kKeys + b * kBoxKeys;
            const int lb = min(key0 / bs, last_block);
            const int off = key0 < L ? key0 % bs : 0;
            const int32_t phys = __ldg(row + lb);
            if (phys < 0 || phys >= p.num_blocks) report_error(p.dev_error, PKV_DEVERR_BLOCK_ID, s);
            // an out-of-range block id reads as zeros (TMA fill), never out of the cache
            tma_load_5d(kdst + b * kBoxBytes, &kmap, &full[st], 0, kvh, off, 0, phys);
            tma_load_5d(vdst + b * kBoxBytes, &vmap, &full[st], 0, kvh, off, 0, phys);
        }
    }
}

template <typename T>
__device__ __forceinline__ uint32_t pack2(float a, float b) {
    return Storage<T>::from_float2(a, b);
}

template <typename T>
__global__ void __launch_bounds__(kThreads, 2)
paged_prefill_kernel(const __grid_constant__ CUtensorMap kmap,
                     const __grid_constant__ CUtensorMap vmap, const PrefillParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align_1024(smem_raw);
    uint8_t* qsm = smem;
    uint8_t* stages = smem + kQBytes;
    uint64_t* full = reinterpret_cast<uint64_t*>(stages + kStages * kStageBytes);
    uint64_t* empty = full + kStages;
    uint64_t* zeroed = empty + kStages;  // the last tile's V rows are zeroed

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
    const int r0 = tile * kRows;
    if (n < 0 || n > L || n > p.max_query_len ||
        (int64_t)L > (int64_t)p.max_blocks_per_seq * p.block_size) {
        if (tile == p.tiles_per_seq - 1 && kvh == 0 && threadIdx.x == 0)
            report_error(p.dev_error, PKV_DEVERR_CONTEXT_LEN, s);
        return;
    }
    if (r0 >= nrows) return;  // a row tile past this sequence's rows
    const int last_row = min(nrows, r0 + kRows) - 1;
    const int kv_end = L - n + last_row / G + 1;  // keys the tile's last row sees
    const int ntiles = (kv_end + kKeys - 1) / kKeys;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int i = 0; i < kStages; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], kConsumers);
        }
        mbar_init(zeroed, kConsumers);
        fence_barrier_init();
        prefetch_tensormap(&kmap);
        prefetch_tensormap(&vmap);
    }
    const int Hq = p.num_q_heads;
    if (warp < kConsumers) {
        // Q rows (token r / G, head kvh * G + r % G) into the swizzled tile
        for (int c = threadIdx.x; c < kRows * (kD / 8); c += kConsumers * 32) {
            const int r = c >> 4, ch = c & 15;
            const int row = r0 + r;
            uint4 v = make_uint4(0, 0, 0, 0);
            if (row < nrows) {
                const int tok = row / G, g = row - tok * G;
                v = *reinterpret_cast<const uint4*>(
                    static_cast<const T*>(p.query) +
                    ((int64_t)(q0 + tok) * Hq + kvh * G + g) * kD + ch * 8);
            }
            *reinterpret_cast<uint4*>(qsm + swz_q(r, ch)) = v;
        }
    }
    __syncthreads();
    if (warp == kConsumers) {
        if (lane == 0) produce(kmap, vmap, p, s, kvh, L, ntiles, stages, full, empty);
        return;
    }

    // ---- consumer warp: rows 16 * warp + (lane >> 2) and that + 8 ----
    const uint32_t qbase = smem_addr(qsm);
    uint32_t qf[kD / 16][4];
#pragma unroll
    for (int kk = 0; kk < kD / 16; ++kk)
        ldmatrix_x4(qf[kk], qbase + swz_q(16 * warp + (lane & 15), 2 * kk + (lane >> 4)));
    int pos[2];
    bool ok[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int row = r0 + 16 * warp + (lane >> 2) + 8 * h;
        ok[h] = row < nrows;
        pos[h] = L - n + (ok[h] ? row / G : 0);
    }
    float o[kD / 8][4];
#pragma unroll
    for (int i = 0; i < kD / 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
    float m[2] = {-INFINITY, -INFINITY}, l[2] = {0.f, 0.f};
    const float sl = p.scale_log2;
    bool failed = false;
    int j = 0;
    for (; j < ntiles; ++j) {
        const int st = j % kStages;
        if (!mbar_wait_bounded(&full[st], (j / kStages) & 1)) {
            failed = true;
            break;
        }
        uint8_t* kt = stages + st * kStageBytes;
        uint8_t* vt = kt + kTileBytes;
        const int key0 = j * kKeys;
        if (key0 + kKeys > L) {
            // rows past the context may hold anything (NaN included): zero V
            // there so that their zero weights contribute exactly 0
            // (only the last tile can reach past L: one use of `zeroed`)
            const int first = max(L - key0, 0);
            for (int c = threadIdx.x; c < (kKeys - first) * 16; c += kConsumers * 32) {
                const int k = first + (c >> 4), ch = c & 15;
                *reinterpret_cast<uint4*>(vt + (k >> 4) * kBoxBytes + swz16(k & 15, ch)) =
                    make_uint4(0, 0, 0, 0);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive_one(zeroed);
            if (!mbar_wait_bounded(zeroed, 0)) {
                failed = true;
                ++j;  // this tile's loads have landed
                break;
            }
        }
        const uint32_t kb = smem_addr(kt), vb = smem_addr(vt);
        // S = Q K^T for 64 keys: 8 n-tiles of 8 keys
        float sacc[kKeys / 8][4];
#pragma unroll
        for (int i = 0; i < kKeys / 8; ++i) sacc[i][0] = sacc[i][1] = sacc[i][2] = sacc[i][3] = 0.f;
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) {
#pragma unroll
            for (int np = 0; np < kKeys / 16; ++np) {
                uint32_t b[4];
                const int mtx = lane >> 3;
                const int r = (mtx >> 1) * 8 + (lane & 7);
                ldmatrix_x4(b, kb + np * kBoxBytes + swz16(r, 2 * kk + (mtx & 1)));
                Mma<T>::m16n8k16(sacc[2 * np], qf[kk], b[0], b[1]);
                Mma<T>::m16n8k16(sacc[2 * np + 1], qf[kk], b[2], b[3]);
            }
        }
        // causal mask, online softmax (base 2)
        float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
        for (int nt = 0; nt < kKeys / 8; ++nt)
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int h = i >> 1;
                const int key = key0 + nt * 8 + 2 * (lane & 3) + (i & 1);
                const float v = (ok[h] && key <= pos[h]) ? sacc[nt][i] * sl : -INFINITY;
                sacc[nt][i] = v;
                mx[h] = fmaxf(mx[h], v);
            }
        float alpha[2], mu[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            mx[h] = fmaxf(mx[h], __shfl_xor_sync(kFull, mx[h], 1));
            mx[h] = fmaxf(mx[h], __shfl_xor_sync(kFull, mx[h], 2));
            const float mn = fmaxf(m[h], mx[h]);
            mu[h] = mn == -INFINITY ? 0.f : mn;  // a row with no key yet stays at zero
            alpha[h] = exp2f(m[h] - mu[h]);
            m[h] = mn;
            l[h] *= alpha[h];
        }
#pragma unroll
        for (int i = 0; i < kD / 8; ++i) {
            o[i][0] *= alpha[0];
            o[i][1] *= alpha[0];
            o[i][2] *= alpha[1];
            o[i][3] *= alpha[1];
        }
        // P as A fragments: the C fragments of n-tiles 2k, 2k + 1 are the A
        // fragment of key step k.  P goes in as a 16-bit high part plus the
        // 16-bit remainder (two products into one accumulator).
#pragma unroll
        for (int k = 0; k < kKeys / 16; ++k) {
            float pv[2][4];
#pragma unroll
            for (int t = 0; t < 2; ++t)
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    pv[t][i] = exp2f(sacc[2 * k + t][i] - mu[i >> 1]);
                    l[i >> 1] += pv[t][i];
                }
            uint32_t hi[4], lo[4];
#pragma unroll
            for (int t = 0; t < 2; ++t)
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const float a = pv[t][2 * h], c = pv[t][2 * h + 1];
                    const uint32_t w = pack2<T>(a, c);
                    const float2 back = Storage<T>::to_float2(w);
                    hi[2 * t + h] = w;
                    lo[2 * t + h] = pack2<T>(a - back.x, c - back.y);
                }
            const int mtx = lane >> 3;
            const int r = (mtx & 1) * 8 + (lane & 7);
#pragma unroll
            for (int dp = 0; dp < kD / 16; ++dp) {
                uint32_t b[4];
                ldmatrix_x4_trans(b, vb + k * kBoxBytes + swz16(r, 2 * dp + (mtx >> 1)));
                Mma<T>::m16n8k16(o[2 * dp], hi, b[0], b[1]);
                Mma<T>::m16n8k16(o[2 * dp], lo, b[0], b[1]);
                Mma<T>::m16n8k16(o[2 * dp + 1], hi, b[2], b[3]);
                Mma<T>::m16n8k16(o[2 * dp + 1], lo, b[2], b[3]);
            }
        }
        // every read of this stage has fed an instruction above: release it
        __syncwarp();
        if (lane == 0) mbar_arrive_one(&empty[st]);
    }
    if (failed) {
        // wait (bounded) for this CTA's loads still in flight, then leave
        for (int k = j; k < ntiles && k < j + kStages; ++k)
            mbar_wait_bounded(&full[k % kStages], (k / kStages) & 1);
        if (lane == 0) report_error(p.dev_error, PKV_DEVERR_TIMEOUT, s);
        return;
    }
    // rows' sums over the quad, then normalised 16-bit output
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        l[h] += __shfl_xor_sync(kFull, l[h], 1);
        l[h] += __shfl_xor_sync(kFull, l[h], 2);
    }
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        if (!ok[h]) continue;
        const int row = r0 + 16 * warp + (lane >> 2) + 8 * h;
        const int tok = row / G, g = row - tok * G;
        T* dst = static_cast<T*>(p.out) + ((int64_t)(q0 + tok) * Hq + kvh * G + g) * kD;
        const float inv = l[h] > 0.f ? 1.f / l[h] : 0.f;
#pragma unroll
        for (int nt = 0; nt < kD / 8; ++nt)
            *reinterpret_cast<uint32_t*>(dst + nt * 8 + 2 * (lane & 3)) =
                pack2<T>(o[nt][2 * h] * inv, o[nt][2 * h + 1] * inv);
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
    p.tiles_per_seq = (int)(((int64_t)max_query_len * p.group + kRows - 1) / kRows);
    p.scale_log2 = scale * kLog2e;
    const int64_t ctas = (int64_t)p.tiles_per_seq * num_seqs * num_kv_heads;
    PKV_REQUIRE(ctas < (1ll << 31), PKV_ERR_UNSUPPORTED, "pkv_prefill_attention: %lld CTAs",
                (long long)ctas);
    CUtensorMap kmap, vmap;
    int st = encode_paged_map_16bit(&kmap, key_cache, dtype, head_dim, num_kv_heads, block_size,
                                    num_blocks, block_stride);
    if (st != PKV_OK) return st;
    st = encode_paged_map_16bit(&vmap, value_cache, dtype, head_dim, num_kv_heads, block_size,
                                num_blocks, block_stride);
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
