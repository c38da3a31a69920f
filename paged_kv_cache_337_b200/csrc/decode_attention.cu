// decode_attention.cu — single-token decode attention over the paged KV cache
// ("Paged KV" wiki page, Attention Kernel 的适配: the kernel takes the Block
// Table and block_size and reads K/V block by block through the table; the
// result is ordinary softmax attention over the sequence's tokens in logical
// order, since PagedAttention changes the storage, not the algorithm —
// "一文读懂vLLM的…PagedAttention" page, opening section).
//
// Work decomposition
//   One CTA per (sequence, KV head, partition).  A partition is a run of
//   partition_size tokens (the whole context in single-pass mode).  The G
//   query heads that share the KV head are packed into the CTA, so each K/V
//   byte is read from HBM once per step.  Each of the CTA's warps owns every
//   NW-th 16-token tile of the partition and runs its own TMA pipeline:
//   lane 0 resolves the tile's physical block from the partition's slice of
//   the Block Table (staged in shared memory once per CTA) and issues one
//   5-D tiled TMA load for the K tile and one for the V tile into a
//   STAGES-deep ring of 128B-swizzled shared-memory buffers, completing on
//   per-stage mbarriers.
//   Softmax is online (running max and sum in fp32, base-2 exponentials with
//   scale * log2(e) folded into the scores).  The warps' partial results are
//   merged through shared memory at the end; with several partitions the CTA
//   writes fp32 (max, sum, unnormalised output) to the workspace, and the
//   last CTA of each (sequence, KV head) to finish merges them (a counter
//   per pair, cleared by a memset on the stream before the launch).  The
//   flat grid runs a pair's partitions side by side, so merges overlap the
//   streaming of later pairs.
//
// Arithmetic paths
//   G == 1 (no grouping): a GEMV; FFMA with warp shuffles.  Lane l owns
//   head_dim / 32 dimensions; the 16 partial dot products of a tile are
//   reduce-scattered across the warp (16 shuffles) so lane l ends with token
//   l / 2's score.
//   G >= 2: the G query heads form a real dense contraction.  S^T = K Q^T is
//   an m16n8k16 tensor-core product with the 16 tokens as M and up to 8
//   heads as N (K tiles through ldmatrix, Q^T fragments in registers);
//   O^T += V^T P^T takes V^T tiles through ldmatrix.trans and P^T from the
//   score fragments by movmatrix, with head_dim as M.  Over 16-bit caches P
//   enters as a 16-bit high part plus a 16-bit remainder (two products into
//   one accumulator), so rounding the softmax weights costs no accuracy;
//   over e4m3 caches, whose products all run in f16, P is one f16 rounding.
//
// Every wait on an mbarrier is bounded (1 s); on expiry the kernel records
// PKV_DEVERR_TIMEOUT, waits (bounded) for its loads in flight and skips its
// output.  Table entries outside [0, num_blocks) are reported; the TMA unit
// fills such a tile with zeros, so no access leaves the cache.
#include <cudaTypedefs.h>

#include <cmath>
#include <type_traits>
#include <mutex>

#include "common.cuh"

namespace pkv {
namespace {

constexpr int kTile = 16;                          // tokens per tile
constexpr int kBoxD = 64;                          // head_dim per TMA box (128 B)
constexpr int kSubTileBytes = kTile * kBoxD * 2;   // one swizzled box: 2 KiB
// Compile-time shape of the attention CTA: warps per CTA and TMA stages per
// warp (one stage holds the K and V tiles of 16 tokens).
#ifndef PKV_DECODE_WARPS
#define PKV_DECODE_WARPS 4
#endif
#ifndef PKV_DECODE_STAGES_D128
#define PKV_DECODE_STAGES_D128 2
#endif
#ifndef PKV_DECODE_STAGES_D64
#define PKV_DECODE_STAGES_D64 4
#endif
constexpr int kWarps = PKV_DECODE_WARPS;
constexpr float kLog2e = 1.4426950408889634f;
constexpr unsigned kFull = 0xffffffffu;

template <int D>
struct Geom {
    static constexpr int kBoxes = D / kBoxD;             // boxes per K (or V) tile
    static constexpr int kKBytes = kBoxes * kSubTileBytes;
    static constexpr int kStages = D == 128 ? PKV_DECODE_STAGES_D128 : PKV_DECODE_STAGES_D64;
};

struct DecodeParams {
    void* out;
    const void* query;
    const int32_t* block_tables;
    const int32_t* context_lens;
    float* ws_m;
    float* ws_l;
    float* ws_o;
    int32_t* ws_count;  // [S, Hkv]: partitions finished (zeroed before the launch)
    const float* k_scale;  // e4m3 caches: [num_blocks, Hkv] dequantisation scales
    const float* v_scale;
    int32_t* dev_error;
    // Optional work list: CTA i handles item work_items[i], a flat index
    // (s * num_kv_heads + kvh) * num_partitions + part; null means CTA i
    // handles item i of the full grid.
    const int32_t* work_items;
    int num_seqs;
    int num_kv_heads;
    int max_blocks_per_seq;
    int max_context_len;
    int num_q_heads;
    int group;  // query heads per KV head
    int num_blocks;
    int block_size;
    int partition_size;  // tokens per partition
    int num_partitions;  // grid.z and the workspace's partition extent
    float scale_log2;    // scale * log2(e)
};

// Byte offset of 16-byte chunk `chunk` (0 .. D/8-1) of row `r` inside a tile
// written by TMA with 128-byte swizzling: each 64-element box is 16 rows of
// 128 bytes whose chunks are XOR-permuted by the row index.
__device__ __forceinline__ uint32_t swz(int r, int chunk) {
    return (chunk >> 3) * kSubTileBytes + r * 128 + (((chunk & 7) ^ (r & 7)) << 4);
}

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
    const uint32_t a = smem_addr(p);
    return p + ((1024u - (a & 1023u)) & 1023u);
}

// Context length of sequence s as the kernels use it: a value outside
// [0, max_context_len] or beyond the table row is treated as 0 (reported by
// the attention kernel).
__device__ __forceinline__ int checked_len(const DecodeParams& p, int s, bool* bad) {
    int L = __ldg(p.context_lens + s);
    *bad = L < 0 || L > p.max_context_len ||
           (int64_t)L > (int64_t)p.max_blocks_per_seq * p.block_size;
    return *bad ? 0 : L;
}

// ---------------------------------------------------------------------------
// Per-warp arithmetic, G == 1: FFMA + shuffles
// ---------------------------------------------------------------------------
// (16-bit caches; e4m3 caches take the tensor-core path for every group)
template <typename T, int D>
struct GemvWarp {
    static constexpr int DV = D / 32;  // dims per lane
    static constexpr int GP = 1;       // heads held (padded)
    static constexpr bool kMma = false;
    float q[DV], o[DV], m, l;

    __device__ __forceinline__ void init(const DecodeParams& p, int s, int kvh, int lane) {
        const T* qrow = static_cast<const T*>(p.query) + ((int64_t)s * p.num_q_heads + kvh) * D;
        load(reinterpret_cast<const uint8_t*>(qrow + lane * DV), q);
#pragma unroll
        for (int j = 0; j < DV; ++j) o[j] = 0.f;
        m = -INFINITY;
        l = 0.f;
    }

    __device__ __forceinline__ static void load(const uint8_t* src, float (&v)[DV]) {
        if constexpr (DV == 4) {
            const uint2 w = *reinterpret_cast<const uint2*>(src);
            const float2 a = Storage<T>::to_float2(w.x), b = Storage<T>::to_float2(w.y);
            v[0] = a.x; v[1] = a.y; v[2] = b.x; v[3] = b.y;
        } else {
            const uint32_t w = *reinterpret_cast<const uint32_t*>(src);
            const float2 a = Storage<T>::to_float2(w);
            v[0] = a.x; v[1] = a.y;
        }
    }

    // lane's DV elements of row r of a swizzled tile
    __device__ __forceinline__ static const uint8_t* at(const uint8_t* tile, int r, int lane) {
        const int d0 = lane * DV;
        return tile + swz(r, d0 >> 3) + (d0 & 7) * 2;
    }

    // One tile.  scale_log2 multiplies q.k; vscale multiplies the V rows.
    __device__ __forceinline__ void tile(const uint8_t* kt, const uint8_t* vt, int valid,
                                         float scale_log2, int lane, float vscale = 1.f) {
        float part[16];
#pragma unroll
        for (int r = 0; r < 16; ++r) {
            float k[DV];
            load(at(kt, r, lane), k);
            float acc = 0.f;
#pragma unroll
            for (int j = 0; j < DV; ++j) acc = fmaf(q[j], k[j], acc);
            part[r] = acc;
        }
        // reduce-scatter the 16 partial sums over the 32 lanes: after the
        // rounds with masks 16, 8, 4, 2 and a final pairwise add, lane l
        // holds the full dot product of token l / 2
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const bool up = lane & 16;
            const float send = up ? part[i] : part[i + 8];
            const float keep = up ? part[i + 8] : part[i];
            part[i] = keep + __shfl_xor_sync(kFull, send, 16);
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const bool up = lane & 8;
            const float send = up ? part[i] : part[i + 4];
            const float keep = up ? part[i + 4] : part[i];
            part[i] = keep + __shfl_xor_sync(kFull, send, 8);
        }
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const bool up = lane & 4;
            const float send = up ? part[i] : part[i + 2];
            const float keep = up ? part[i + 2] : part[i];
            part[i] = keep + __shfl_xor_sync(kFull, send, 4);
        }
        {
            const bool up = lane & 2;
            const float send = up ? part[0] : part[1];
            const float keep = up ? part[1] : part[0];
            part[0] = keep + __shfl_xor_sync(kFull, send, 2);
        }
        const float dot = part[0] + __shfl_xor_sync(kFull, part[0], 1);
        const int r = lane >> 1;
        const float sc = r < valid ? dot * scale_log2 : -INFINITY;
        float mx = sc;
        mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 2));
        mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 4));
        mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 8));
        mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 16));
        const float m_new = fmaxf(m, mx);
        const float alpha = exp2f(m - m_new);
        const float pr = exp2f(sc - m_new);
        l = l * alpha + ((lane & 1) ? 0.f : pr);  // each token is held by 2 lanes
        m = m_new;
#pragma unroll
        for (int j = 0; j < DV; ++j) o[j] *= alpha;
        const float prv = pr * vscale;
#pragma unroll
        for (int rr = 0; rr < 16; ++rr) {
            const float pb = __shfl_sync(kFull, prv, rr * 2);
            float v[DV];
            load(at(vt, rr, lane), v);
#pragma unroll
            for (int j = 0; j < DV; ++j) o[j] = fmaf(pb, v[j], o[j]);
        }
    }

    // warp-level totals: m is already uniform; l is summed over the lanes
    __device__ __forceinline__ void finish() {
#pragma unroll
        for (int x = 1; x < 32; x <<= 1) l += __shfl_xor_sync(kFull, l, x);
    }

    __device__ __forceinline__ void store_ml(float* sm_m, float* sm_l, int warp, int lane,
                                             int G) {
        if (lane == 0) {
            sm_m[warp * GP] = m;
            sm_l[warp * GP] = l;
        }
    }

    // scaled output into sm_o[warp][head][d]
    __device__ __forceinline__ void store_o(float* sm_o, const float* M, int warp, int lane,
                                            int G) {
        const float f = M[0] == -INFINITY ? 0.f : exp2f(m - M[0]);
#pragma unroll
        for (int j = 0; j < DV; ++j) sm_o[warp * D + lane * DV + j] = o[j] * f;
    }
};

// ---------------------------------------------------------------------------
// Per-warp arithmetic, G >= 2: mma.sync m16n8k16 on the head group
// ---------------------------------------------------------------------------
// Token held by row r of the e4m3 path's S^T fragments: rows 2j, 2j+1 are
// tokens 4j, 4j+1 and rows 8+2j, 9+2j are tokens 4j+2, 4j+3, the order in
// which the transposing byte load delivers V (so P's fragments line up).
__device__ __forceinline__ int token_of_row(int r) {
    return r < 8 ? 4 * (r >> 1) + (r & 1) : 4 * ((r - 8) >> 1) + 2 + (r & 1);
}

// E4 (e4m3 caches): K comes straight from the e4m3 tile and every product
// runs on f16 (e4m3 values are exact in f16), whatever T is; the queries
// are scaled by a power of two into f16 range and the scale is undone on
// the scores.
template <typename T, int D, int NT, bool E4 = false>
struct MmaWarp {
    using MT = typename std::conditional<E4, __half, T>::type;  // MMA operand type
    static constexpr int KS = D / 16;  // k-steps of S^T, m-tiles of O^T
    static constexpr int GP = NT * 8;  // heads held (padded)
    static constexpr bool kMma = true;
    // Over e4m3 caches P enters the P V product as one f16 rounding
    // (relative error <= 2^-11 per weight, so the output moves by at most
    // 2^-11 * sum_t p_t |v_t| / l); over 16-bit caches it adds its rounded
    // remainder as a second product (a bf16 P alone is off by up to 2^-8)
    static constexpr bool kPRem = !E4;
    uint32_t qf[KS][NT][2];            // Q^T B-fragments
    float acc[KS][NT][4];              // O^T[d][head]
    float m[NT][2], l[NT][2];          // per lane: heads nt*8 + (lane&3)*2 + {0,1}
    float vs;                          // acc is in units of this V scale (e4m3 caches)
    float qinv;                        // undoes the queries' power-of-two scale

    __device__ __forceinline__ void init(const DecodeParams& p, int s, int kvh, int lane) {
        const int G = p.group;
        const T* qbase = static_cast<const T*>(p.query) +
                         ((int64_t)s * p.num_q_heads + (int64_t)kvh * G) * D;
        if constexpr (E4) {
            // k-step kk of head h holds dims 16kk + 4j .. 16kk + 4j + 3 in
            // the lane with j = lane & 3: the order the e4m3 K fragments
            // arrive in (see tile)
            float qv[KS][NT][4];
            float mx = 0.f;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                const int h = nt * 8 + (lane >> 2);
#pragma unroll
                for (int kk = 0; kk < KS; ++kk) {
                    if (h < G) {
                        const uint2 w = *reinterpret_cast<const uint2*>(
                            qbase + (int64_t)h * D + kk * 16 + (lane & 3) * 4);
                        const float2 a = Storage<T>::to_float2(w.x), b = Storage<T>::to_float2(w.y);
                        qv[kk][nt][0] = a.x;
                        qv[kk][nt][1] = a.y;
                        qv[kk][nt][2] = b.x;
                        qv[kk][nt][3] = b.y;
                    } else {
                        qv[kk][nt][0] = qv[kk][nt][1] = qv[kk][nt][2] = qv[kk][nt][3] = 0.f;
                    }
#pragma unroll
                    for (int i = 0; i < 4; ++i) mx = fmaxf(mx, fabsf(qv[kk][nt][i]));
                }
            }
#pragma unroll
            for (int x = 1; x < 32; x <<= 1) mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, x));
            // largest |q| into [2^14, 2^15): below f16's maximum, and every
            // value within 2^29 of it keeps its bits
            int ex = 0;
            frexpf(mx, &ex);
            const int sh = mx > 0.f ? max(-120, min(120, 15 - ex)) : 0;
            const float qs = ldexpf(1.f, sh);
            qinv = ldexpf(1.f, -sh);
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int kk = 0; kk < KS; ++kk) {
                    qf[kk][nt][0] = Storage<__half>::from_float2(qv[kk][nt][0] * qs,
                                                                 qv[kk][nt][1] * qs);
                    qf[kk][nt][1] = Storage<__half>::from_float2(qv[kk][nt][2] * qs,
                                                                 qv[kk][nt][3] * qs);
                }
        } else {
            qinv = 1.f;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                const int h = nt * 8 + (lane >> 2);
#pragma unroll
                for (int kk = 0; kk < KS; ++kk) {
                    if (h < G) {
                        const T* qrow = qbase + (int64_t)h * D + kk * 16 + (lane & 3) * 2;
                        qf[kk][nt][0] = *reinterpret_cast<const uint32_t*>(qrow);
                        qf[kk][nt][1] = *reinterpret_cast<const uint32_t*>(qrow + 8);
                    } else {
                        qf[kk][nt][0] = 0u;
                        qf[kk][nt][1] = 0u;
                    }
                }
            }
        }
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            m[nt][0] = m[nt][1] = -INFINITY;
            l[nt][0] = l[nt][1] = 0.f;
            vs = 1.f;
#pragma unroll
            for (int mt = 0; mt < KS; ++mt)
#pragma unroll
                for (int i = 0; i < 4; ++i) acc[mt][nt][i] = 0.f;
        }
    }

    // One tile of 16-bit K and V.  scale_log2 multiplies q.k (with any K
    // dequantisation scale folded in); vscale multiplies the V rows.  P
    // stays in [0, 1] for the 16-bit fragments; the V scale goes into the
    // fp32 accumulator instead, which is kept in units of the current
    // tile's scale (rescaled by old / new scale with the softmax factor).
    __device__ __forceinline__ void tile(const uint8_t* kt, const uint8_t* vt, int valid,
                                         float scale_log2, int lane, float vscale = 1.f) {
        const uint32_t kbase = smem_addr(kt), vbase = smem_addr(vt);
        const int j = lane >> 3;
        // S^T[token][head] = K Q^T over head_dim
        // two independent accumulator chains (even / odd k-steps) halve the
        // dependent MMA latency, then add
        float sacc[NT][4], sacc2[NT][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int i = 0; i < 4; ++i) sacc[nt][i] = sacc2[nt][i] = 0.f;
        if constexpr (E4) {
            // kt is the e4m3 tile (16 rows of 128 codes, 16-byte chunks
            // swizzled).  One ldmatrix (read as 16-bit pairs) gives the lane
            // codes 4j .. 4j+3 of chunks 2pp and 2pp + 1 for rows g and
            // g + 8; converted pairwise to f16x2 they are the A fragments of
            // k-steps 2pp and 2pp + 1 with the dims of each k-step in the
            // order init gave the queries.
#pragma unroll
            for (int pp = 0; pp < KS / 2; ++pp) {
                uint32_t r[4];
                const int row = token_of_row((lane & 7) + (j & 1) * 8);
                const int chunk = 2 * pp + (j >> 1);
                ldmatrix_x4(r, kbase + row * 128 + ((chunk ^ (row & 7)) << 4));
                const uint32_t a0[4] = {e4m3x2_to_f16x2((uint16_t)r[0]),
                                        e4m3x2_to_f16x2((uint16_t)r[1]),
                                        e4m3x2_to_f16x2((uint16_t)(r[0] >> 16)),
                                        e4m3x2_to_f16x2((uint16_t)(r[1] >> 16))};
                const uint32_t a1[4] = {e4m3x2_to_f16x2((uint16_t)r[2]),
                                        e4m3x2_to_f16x2((uint16_t)r[3]),
                                        e4m3x2_to_f16x2((uint16_t)(r[2] >> 16)),
                                        e4m3x2_to_f16x2((uint16_t)(r[3] >> 16))};
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    Mma<MT>::m16n8k16(sacc[nt], a0, qf[2 * pp][nt][0], qf[2 * pp][nt][1]);
                    Mma<MT>::m16n8k16(sacc2[nt], a1, qf[2 * pp + 1][nt][0],
                                      qf[2 * pp + 1][nt][1]);
                }
            }
        } else {
#pragma unroll
            for (int kk = 0; kk < KS; ++kk) {
                uint32_t a[4];
                const int row = (lane & 7) + (j & 1) * 8;
                ldmatrix_x4(a, kbase + swz(row, kk * 2 + (j >> 1)));
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    if (kk & 1)
                        Mma<MT>::m16n8k16(sacc2[nt], a, qf[kk][nt][0], qf[kk][nt][1]);
                    else
                        Mma<MT>::m16n8k16(sacc[nt], a, qf[kk][nt][0], qf[kk][nt][1]);
                }
            }
        }
        scale_log2 *= qinv;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int i = 0; i < 4; ++i) sacc[nt][i] += sacc2[nt][i];
        // online softmax per head; the lane holds tokens r0, r0 + 8
        const int r0 = lane >> 2;
        const bool v0 = (E4 ? token_of_row(r0) : r0) < valid;
        const bool v1 = (E4 ? token_of_row(r0 + 8) : r0 + 8) < valid;
        const float ratio = vscale == vs ? 1.f : vs / vscale;
        vs = vscale;
        uint32_t pb[NT][2], pl[NT][2];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const float s0 = v0 ? sacc[nt][0] * scale_log2 : -INFINITY;
            const float s1 = v0 ? sacc[nt][1] * scale_log2 : -INFINITY;
            const float s2 = v1 ? sacc[nt][2] * scale_log2 : -INFINITY;
            const float s3 = v1 ? sacc[nt][3] * scale_log2 : -INFINITY;
            float mx0 = fmaxf(s0, s2), mx1 = fmaxf(s1, s3);
#pragma unroll
            for (int x = 4; x < 32; x <<= 1) {
                mx0 = fmaxf(mx0, __shfl_xor_sync(kFull, mx0, x));
                mx1 = fmaxf(mx1, __shfl_xor_sync(kFull, mx1, x));
            }
            const float mn0 = fmaxf(m[nt][0], mx0), mn1 = fmaxf(m[nt][1], mx1);
            const float a0 = exp2f(m[nt][0] - mn0), a1 = exp2f(m[nt][1] - mn1);
            const float p0 = exp2f(s0 - mn0), p1 = exp2f(s1 - mn1);
            const float p2 = exp2f(s2 - mn0), p3 = exp2f(s3 - mn1);
            l[nt][0] = l[nt][0] * a0 + (p0 + p2);
            l[nt][1] = l[nt][1] * a1 + (p1 + p3);
            m[nt][0] = mn0;
            m[nt][1] = mn1;
            const float c0 = a0 * ratio, c1 = a1 * ratio;
#pragma unroll
            for (int mt = 0; mt < KS; ++mt) {
                acc[mt][nt][0] *= c0;
                acc[mt][nt][1] *= c1;
                acc[mt][nt][2] *= c0;
                acc[mt][nt][3] *= c1;
            }
            // P[token][head] as 16-bit fragments, transposed to P^T
            // B-fragments.  Over 16-bit caches P is split into a rounded high
            // part and the rounded remainder, so the PV product sees P to
            // ~16 bits of mantissa instead of the 8 of one bf16 rounding.
            const uint32_t h01 = Storage<MT>::from_float2(p0, p1);
            const uint32_t h23 = Storage<MT>::from_float2(p2, p3);
            const float2 b01 = Storage<MT>::to_float2(h01), b23 = Storage<MT>::to_float2(h23);
            pb[nt][0] = movmatrix_trans(h01);
            pb[nt][1] = movmatrix_trans(h23);
            if constexpr (kPRem) {
                pl[nt][0] = movmatrix_trans(Storage<MT>::from_float2(p0 - b01.x, p1 - b01.y));
                pl[nt][1] = movmatrix_trans(Storage<MT>::from_float2(p2 - b23.x, p3 - b23.y));
            }
        }
        // O^T[d][head] += V^T P^T over the 16 tokens
        if constexpr (E4) {
            // vt is the e4m3 tile.  The transposing byte load gives the lane
            // tokens 4j .. 4j+3 of dims g and g + 8 of two 16-dim m-tiles;
            // converted pairwise they are the A fragments with the token
            // order of P's fragments (token_of_row).
            const int tok = lane & 15;
#pragma unroll
            for (int mp = 0; mp < KS / 2; ++mp) {
                uint32_t r[4];
                const int chunk = 2 * mp + (lane >> 4);
                ldmatrix_b8_x2_trans(r, vbase + tok * 128 + ((chunk ^ (tok & 7)) << 4));
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const uint32_t a[4] = {e4m3x2_to_f16x2((uint16_t)r[2 * h]),
                                           e4m3x2_to_f16x2((uint16_t)r[2 * h + 1]),
                                           e4m3x2_to_f16x2((uint16_t)(r[2 * h] >> 16)),
                                           e4m3x2_to_f16x2((uint16_t)(r[2 * h + 1] >> 16))};
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) {
                        Mma<MT>::m16n8k16(acc[2 * mp + h][nt], a, pb[nt][0], pb[nt][1]);
                        if constexpr (kPRem)
                            Mma<MT>::m16n8k16(acc[2 * mp + h][nt], a, pl[nt][0], pl[nt][1]);
                    }
                }
            }
        } else {
#pragma unroll
            for (int mt = 0; mt < KS; ++mt) {
                uint32_t a[4];
                const int row = (lane & 7) + (j >> 1) * 8;
                ldmatrix_x4_trans(a, vbase + swz(row, mt * 2 + (j & 1)));
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    Mma<MT>::m16n8k16(acc[mt][nt], a, pb[nt][0], pb[nt][1]);
                    Mma<MT>::m16n8k16(acc[mt][nt], a, pl[nt][0], pl[nt][1]);
                }
            }
        }
    }

    __device__ __forceinline__ void finish() {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int x = 4; x < 32; x <<= 1) {
                l[nt][0] += __shfl_xor_sync(kFull, l[nt][0], x);
                l[nt][1] += __shfl_xor_sync(kFull, l[nt][1], x);
            }
    }

    __device__ __forceinline__ void store_ml(float* sm_m, float* sm_l, int warp, int lane,
                                             int G) {
        if (lane < 4) {
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int i = 0; i < 2; ++i) {
                    const int h = nt * 8 + lane * 2 + i;
                    sm_m[warp * GP + h] = m[nt][i];
                    sm_l[warp * GP + h] = l[nt][i];
                }
        }
    }

    __device__ __forceinline__ void store_o(float* sm_o, const float* M, int warp, int lane,
                                            int G) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int h = nt * 8 + (lane & 3) * 2 + (i & 1);
                if (h >= G) continue;
                const float f = M[h] == -INFINITY ? 0.f : exp2f(m[nt][i & 1] - M[h]) * vs;
#pragma unroll
                for (int mt = 0; mt < KS; ++mt) {
                    const int d = mt * 16 + (lane >> 2) + (i >> 1) * 8;
                    sm_o[(warp * G + h) * D + d] = acc[mt][nt][i] * f;
                }
            }
    }
};

// ---------------------------------------------------------------------------
// Shared-memory plan of one CTA: per warp a ring of stages (the K and V tiles
// as stored), then the mbarriers, the per-stage dequantisation scales (e4m3)
// and the partition's table slice.  The ring is reused by the epilogue once
// every load has landed.
// ---------------------------------------------------------------------------
template <int D, bool FP8, bool MMA>
struct Plan {
    static_assert(!FP8 || D == 128, "e4m3 caches are built for head_dim 128");
    static_assert(!FP8 || MMA, "e4m3 caches run on the tensor-core path");
    static constexpr int kStages = FP8 ? 2 : Geom<D>::kStages;
    static constexpr int kTileBytes = FP8 ? kTile * D : Geom<D>::kKBytes;  // K (or V) as stored
    static constexpr int kStageBytes = 2 * kTileBytes;
    static constexpr size_t kRing = (size_t)kWarps * kStages * kStageBytes;
    // the warps' merge reuses the ring: per warp m and l of up to 16 (padded)
    // heads, the common max, and per warp G x D partial outputs (G <= 16)
    static constexpr size_t kMerge = ((size_t)kWarps * 2 * 16 + 16 + (size_t)kWarps * 16 * D) * 4;
    static constexpr size_t kEpilogue = kRing > kMerge ? kRing : kMerge;
    static constexpr size_t kBarOff = kEpilogue;
    static constexpr size_t kScaleOff = kBarOff + (size_t)kWarps * kStages * 8;
    static constexpr size_t kTableOff = kScaleOff + (FP8 ? (size_t)kWarps * kStages * 32 : 0);
    static constexpr uint32_t kTx = kStageBytes + (FP8 ? 32 : 0);  // bytes landing per stage
};

// ---------------------------------------------------------------------------
// The attention kernel (single pass or one partition of split-K)
// ---------------------------------------------------------------------------
// The body of one CTA; the kernels below differ only in their launch bounds.
template <typename T, int D, typename Warp, bool FP8>
__device__ __forceinline__ void decode_cta(const CUtensorMap& kmap, const CUtensorMap& vmap,
                                           const DecodeParams& p) {
    using Gm = Geom<D>;
    using Pl = Plan<D, FP8, Warp::kMma>;
    constexpr int STAGES = Pl::kStages;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);
    uint8_t* stages = smem;  // [warp][stage][K tile | V tile]
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Pl::kBarOff);
    float* scales = reinterpret_cast<float*>(smem + Pl::kScaleOff);  // [warp][stage][K 4 | V 4]
    int32_t* table = reinterpret_cast<int32_t*>(smem + Pl::kTableOff);

    // Flat grid, partition fastest: the partitions of one (sequence, KV
    // head) run side by side, so their merge happens early and in parallel
    // with the other CTAs' streaming rather than all at the end.  With a
    // work list the CTA takes its item from the list instead (the host
    // orders the items longest first and leaves out empty partitions).
    unsigned item = blockIdx.x;
    if (p.work_items != nullptr) {
        item = (unsigned)__ldg(p.work_items + blockIdx.x);
        if (item >= (unsigned)p.num_seqs * (unsigned)p.num_kv_heads *
                        (unsigned)p.num_partitions) {
            if (threadIdx.x == 0) report_error(p.dev_error, PKV_DEVERR_WORK_ITEM, blockIdx.x);
            return;
        }
    }
    const int part = (int)(item % (unsigned)p.num_partitions);
    const int rest = (int)(item / (unsigned)p.num_partitions);
    const int kvh = rest % p.num_kv_heads;
    const int s = rest / p.num_kv_heads;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = p.group, bs = p.block_size, P = p.partition_size;

    // The partition's first table entries are read together with the
    // context length (the row index does not depend on it), so the two
    // global loads overlap instead of forming a chain before the first TMA.
    const int lb0 = part * P / bs;
    const int32_t* trow = p.block_tables + (int64_t)s * p.max_blocks_per_seq + lb0;
    const int row_left = p.max_blocks_per_seq - lb0;  // > 0: part < NP
    const int32_t spec = threadIdx.x < row_left ? __ldg(trow + threadIdx.x) : -1;

    bool bad_len;
    const int L = checked_len(p, s, &bad_len);
    if (bad_len && part == 0 && kvh == 0 && threadIdx.x == 0)
        report_error(p.dev_error, PKV_DEVERR_CONTEXT_LEN, s);
    const int np = L > 0 ? (L + P - 1) / P : 1;
    if (part >= np) return;  // a partition past this sequence's end

    uint64_t* my_bars = bars + warp * STAGES;
    uint8_t* my_stages = stages + warp * STAGES * Pl::kStageBytes;
    float* my_scales = scales + warp * STAGES * 8;
    if (lane == 0) {
#pragma unroll
        for (int st = 0; st < STAGES; ++st) mbar_init(&my_bars[st], 1);
        fence_barrier_init();
    }
    if (threadIdx.x == 0) {
        prefetch_tensormap(&kmap);
        prefetch_tensormap(&vmap);
    }
    const int t_begin = part * P;
    const int t_end = min(L, t_begin + P);
    // Tiles of 16 tokens per block (block_size is a multiple of 16, at most
    // 256) and a multiplier that divides a tile index by it: the high word
    // of ti * ceil(2^32 / tpb) is floor(ti / tpb) for every ti below 2^28,
    // and tile indexes stay below 2^27, so the loop needs no division.
    const unsigned tpb = (unsigned)(bs / kTile);
    const unsigned tpb_mul = tpb == 1 ? 0u : 0xFFFFFFFFu / tpb + 1u;
    const unsigned ti0 = (unsigned)(t_begin / kTile);
    auto block_of = [&](unsigned ti) -> unsigned { return tpb_mul ? __umulhi(ti, tpb_mul) : ti; };
    const int ntiles = t_end > t_begin ? (t_end - t_begin + kTile - 1) / kTile : 0;
    const int nlb = t_end > t_begin ? (t_end - 1) / bs - lb0 + 1 : 0;

    // this partition's slice of the Block Table, one entry per logical block
    for (int i = threadIdx.x; i < nlb; i += kWarps * 32) {
        const int32_t b = i < kWarps * 32 ? spec : __ldg(trow + i);
        if (b < 0 || b >= p.num_blocks) report_error(p.dev_error, PKV_DEVERR_BLOCK_ID, s);
        table[i] = b;
    }
    __syncthreads();

    // TMA of tile `tile` (K and V, all boxes) into stage `st`; lane 0 only
    // index of the (block, KV head) scale of a tile; a block id outside the
    // pool (reported above, its tile read as zeros) takes block 0's
    auto scale_index = [&](int phys) -> int64_t {
        return (int64_t)(phys >= 0 && phys < p.num_blocks ? phys : 0) * p.num_kv_heads + kvh;
    };
    auto issue = [&](int st, int tile) {
        const unsigned ti = ti0 + (unsigned)tile;
        const unsigned lb = block_of(ti);
        const int phys = table[lb - (unsigned)lb0];
        const int off = (int)(ti - lb * tpb) * kTile;
        uint8_t* kdst = my_stages + st * Pl::kStageBytes;
        uint8_t* vdst = kdst + Pl::kTileBytes;
        mbar_arrive_expect_tx(&my_bars[st], Pl::kTx);
        if constexpr (FP8) {
            // one box of 16 rows x 128 codes per cache, and the 16-byte
            // aligned groups of 4 scales holding this (block, head)'s
            tma_load_4d(kdst, &kmap, &my_bars[st], 0, kvh, off, phys);
            tma_load_4d(vdst, &vmap, &my_bars[st], 0, kvh, off, phys);
            const int64_t g = scale_index(phys) & ~int64_t(3);
            bulk_load(my_scales + st * 8, p.k_scale + g, 16, &my_bars[st]);
            bulk_load(my_scales + st * 8 + 4, p.v_scale + g, 16, &my_bars[st]);
        } else {
            // one instruction per tile and cache: all head_dim / 64 boxes
            tma_load_5d(kdst, &kmap, &my_bars[st], 0, kvh, off, 0, phys);
            tma_load_5d(vdst, &vmap, &my_bars[st], 0, kvh, off, 0, phys);
        }
    };

    const int my_tiles = ntiles > warp ? (ntiles - warp + kWarps - 1) / kWarps : 0;
    if (lane == 0) {
#pragma unroll
        for (int st = 0; st < STAGES; ++st)
            if (st < my_tiles) issue(st, warp + st * kWarps);
    }
    __syncwarp();

    Warp w;
    w.init(p, s, kvh, lane);
    int it = 0;
    bool failed = false;
    for (; it < my_tiles; ++it) {
        const int st = it % STAGES;
        const int tile = warp + it * kWarps;
        if (!mbar_wait_bounded(&my_bars[st], (it / STAGES) & 1)) {
            failed = true;
            break;
        }
        uint8_t* kt = my_stages + st * Pl::kStageBytes;
        uint8_t* vt = kt + Pl::kTileBytes;
        const int valid = min(kTile, t_end - (t_begin + tile * kTile));
        float kscale = 1.f, vscale = 1.f;
        if constexpr (FP8) {
            const int64_t si = scale_index(table[block_of(ti0 + (unsigned)tile) - (unsigned)lb0]) & 3;
            kscale = my_scales[st * 8 + si];
            vscale = my_scales[st * 8 + 4 + si];

        }
        if (valid < kTile) {
            // rows past the context may hold anything (NaN included): zero
            // the V rows so that their zero weights contribute exactly 0
            if constexpr (FP8) {
                for (int c = lane; c < (kTile - valid) * 8; c += 32)
                    *reinterpret_cast<uint4*>(vt + (valid + c / 8) * 128 + (c % 8) * 16) =
                        make_uint4(0, 0, 0, 0);
            } else {
                const int nchunks = (kTile - valid) * Gm::kBoxes * 8;
                for (int c = lane; c < nchunks; c += 32) {
                    const int r = valid + c / (Gm::kBoxes * 8);
                    const int ch = c % (Gm::kBoxes * 8);
                    *reinterpret_cast<uint4*>(vt + swz(r, ch)) = make_uint4(0, 0, 0, 0);
                }
            }
            __syncwarp();
        }
        w.tile(kt, vt, valid, p.scale_log2 * kscale, lane, vscale);
        // Every shared-memory read of this stage feeds an instruction that
        // precedes the next TMA issue in program order, so the reads are
        // complete before the stage is rewritten.
        __syncwarp();
        const int next = it + STAGES;
        if (lane == 0 && next < my_tiles) issue(st, warp + next * kWarps);
    }
    if (failed) {
        // drain this warp's loads still in flight before giving up
        for (int k = it; k < my_tiles && k < it + STAGES; ++k)
            mbar_wait_bounded(&my_bars[k % STAGES], (k / STAGES) & 1);
    }
    if (__syncthreads_or(failed)) {
        if (threadIdx.x == 0) report_error(p.dev_error, PKV_DEVERR_TIMEOUT, 0);
        return;
    }

    // ---- merge the warps' partial softmax states through shared memory ----
    w.finish();
    constexpr int GP = Warp::GP;
    float* sm_m = reinterpret_cast<float*>(stages);  // [warp][GP]
    float* sm_l = sm_m + kWarps * GP;                // [warp][GP]
    float* sm_M = sm_l + kWarps * GP;                // [GP]
    float* sm_o = sm_M + GP;                         // [warp][G][D]
    w.store_ml(sm_m, sm_l, warp, lane, G);
    __syncthreads();
    if (threadIdx.x < G) {
        float M = -INFINITY;
#pragma unroll
        for (int k = 0; k < kWarps; ++k) M = fmaxf(M, sm_m[k * GP + threadIdx.x]);
        sm_M[threadIdx.x] = M;
    }
    __syncthreads();
    w.store_o(sm_o, sm_M, warp, lane, G);
    __syncthreads();

    const int Hq = p.num_q_heads;
    const int64_t qh0 = (int64_t)s * Hq + (int64_t)kvh * G;  // first query head
    for (int idx = threadIdx.x; idx < G * D; idx += kWarps * 32) {
        const int h = idx / D, d = idx - h * D;
        const float M = sm_M[h];
        float Lsum = 0.f, O = 0.f;
#pragma unroll
        for (int k = 0; k < kWarps; ++k) {
            const float mk = sm_m[k * GP + h];
            Lsum += M == -INFINITY ? 0.f : sm_l[k * GP + h] * exp2f(mk - M);
            O += sm_o[(k * G + h) * D + d];
        }
        if (np == 1) {
            static_cast<T*>(p.out)[(qh0 + h) * D + d] =
                Storage<T>::from_float(Lsum > 0.f ? O / Lsum : 0.f);
        } else {
            const int64_t wi = (qh0 + h) * p.num_partitions + part;
            p.ws_o[wi * D + d] = O;
            if (d == 0) {
                p.ws_m[wi] = M;
                p.ws_l[wi] = Lsum;
            }
        }
    }
    if (np == 1) return;

    // ---- split-K merge, done by the last partition to finish ----------------
    // Each CTA publishes its partial (m, l, o), then counts itself in; the
    // CTA that brings the count to np merges all np partials of this
    // (sequence, KV head):  M = max_p m_p,  w_p = 2^(m_p - M),
    // out = sum_p w_p o_p / sum_p w_p l_p.
    // The barrier orders every thread's partial stores before thread 0's
    // fence, and a fence is cumulative, so one fence publishes them all
    // before the count; symmetrically the merging CTA's thread 0 fences
    // after the count and the barrier passes that on to its readers.
    __shared__ int sm_last;
    __syncthreads();
    int32_t* count = p.ws_count + (int64_t)s * p.num_kv_heads + kvh;
    if (threadIdx.x == 0) {
        __threadfence();
        sm_last = atomicAdd(count, 1) == np - 1;
        if (sm_last) __threadfence();
    }
    __syncthreads();
    if (!sm_last) return;
    float* w_m = reinterpret_cast<float*>(stages);  // [G][np]: m, then the weights
    float* w_l = w_m + G * np;                      // [G][np]
    float* h_M = w_l + G * np;                      // [G]
    float* h_L = h_M + G;                           // [G]
    for (int i = threadIdx.x; i < G * np; i += kWarps * 32) {
        const int h = i / np, pp = i - h * np;
        const int64_t wi = (qh0 + h) * p.num_partitions + pp;
        w_m[i] = __ldcg(p.ws_m + wi);
        w_l[i] = __ldcg(p.ws_l + wi);
    }
    __syncthreads();
    if (threadIdx.x < G) {
        const float* mh = w_m + threadIdx.x * np;
        float M = -INFINITY;
        for (int pp = 0; pp < np; ++pp) M = fmaxf(M, mh[pp]);
        h_M[threadIdx.x] = M;
    }
    __syncthreads();
    for (int i = threadIdx.x; i < G * np; i += kWarps * 32) {
        const float wgt = exp2f(w_m[i] - h_M[i / np]);
        w_m[i] = wgt;
        w_l[i] *= wgt;
    }
    __syncthreads();
    if (threadIdx.x < G) {
        const float* lh = w_l + threadIdx.x * np;
        float Lsum = 0.f;
        for (int pp = 0; pp < np; ++pp) Lsum += lh[pp];
        h_L[threadIdx.x] = Lsum;
    }
    __syncthreads();
    // four consecutive dims per thread: float4 loads of the partials
    for (int idx = threadIdx.x; idx < G * D / 4; idx += kWarps * 32) {
        const int h = idx / (D / 4), d4 = (idx - h * (D / 4)) * 4;
        const float* wh = w_m + h * np;
        const float4* o = reinterpret_cast<const float4*>(
            p.ws_o + ((qh0 + h) * p.num_partitions) * D + d4);
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 8
        for (int pp = 0; pp < np; ++pp) {
            const float4 v = __ldcg(o + (int64_t)pp * (D / 4));
            const float wgt = wh[pp];
            acc.x = fmaf(wgt, v.x, acc.x);
            acc.y = fmaf(wgt, v.y, acc.y);
            acc.z = fmaf(wgt, v.z, acc.z);
            acc.w = fmaf(wgt, v.w, acc.w);
        }
        const float inv = 1.f / h_L[h];
        T* dst = static_cast<T*>(p.out) + (qh0 + h) * D + d4;
        uint2 packed;
        packed.x = Storage<T>::from_float2(acc.x * inv, acc.y * inv);
        packed.y = Storage<T>::from_float2(acc.z * inv, acc.w * inv);
        *reinterpret_cast<uint2*>(dst) = packed;
    }
    if (threadIdx.x == 0) *count = 0;  // ready for the next launch
}

template <typename T, int D, typename Warp, bool FP8>
__global__ void __launch_bounds__(kWarps * 32)
paged_decode_kernel(const __grid_constant__ CUtensorMap kmap,
                    const __grid_constant__ CUtensorMap vmap, const DecodeParams p) {
    decode_cta<T, D, Warp, FP8>(kmap, vmap, p);
}

// e4m3 caches with up to 8 query heads per KV head: registers capped at
// 128 per thread so that 4 CTAs fit per SM without a spill (under a cap of
// 96 for 5 CTAs the body spills, and 4 unspilled CTAs measured 2-3 % faster).
template <typename T, typename Warp>
__global__ void __launch_bounds__(kWarps * 32, 4)
paged_decode_kernel_e4m3(const __grid_constant__ CUtensorMap kmap,
                         const __grid_constant__ CUtensorMap vmap, const DecodeParams p) {
    decode_cta<T, 128, Warp, true>(kmap, vmap, p);
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000,
                                             cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    });
    return fn;
}

// 5-D view of one cache: (64 dims, kv head, slot in block, 64-dim half,
// physical block).  The halves are 128 bytes apart; putting them after the
// slot makes one box of 64 x 1 x 16 x (head_dim / 64) x 1 elements land in
// shared memory as head_dim / 64 swizzled 16-row x 128-byte sub-tiles, so a
// single TMA instruction fetches a whole K (or V) tile.
int encode_cache_map(CUtensorMap* map, const void* cache, pkv_dtype dtype, int head_dim,
                     int num_kv_heads, int block_size, int num_blocks, int64_t block_stride) {
    auto fn = encode_fn();
    if (!fn) return fail(PKV_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
    const cuuint64_t dims[5] = {(cuuint64_t)kBoxD, (cuuint64_t)num_kv_heads,
                                (cuuint64_t)block_size, (cuuint64_t)(head_dim / kBoxD),
                                (cuuint64_t)num_blocks};
    const cuuint64_t strides[4] = {(cuuint64_t)head_dim * 2,
                                   (cuuint64_t)num_kv_heads * head_dim * 2,
                                   (cuuint64_t)kBoxD * 2, (cuuint64_t)block_stride * 2};
    const cuuint32_t box[5] = {kBoxD, 1, kTile, (cuuint32_t)(head_dim / kBoxD), 1};
    const cuuint32_t estr[5] = {1, 1, 1, 1, 1};
    const CUtensorMapDataType ty = dtype == PKV_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                                     : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
    CUresult r = fn(map, ty, 5, const_cast<void*>(cache), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(PKV_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
    return PKV_OK;
}

struct WorkspaceLayout {
    size_t count_off, m_off, l_off, o_off, total;
};

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// int32 partition counters (one per (seq, KV head); room for S * Hq) |
// m [S, Hq, NP] | l [S, Hq, NP] | o [S, Hq, NP, D], each 256-byte aligned
WorkspaceLayout workspace_layout(int64_t S, int64_t Hq, int64_t NP, int64_t D) {
    WorkspaceLayout w;
    const size_t cnt = align256((size_t)(S * Hq) * sizeof(int32_t));
    const size_t ml = align256((size_t)(S * Hq * NP) * sizeof(float));
    w.count_off = 0;
    w.m_off = cnt;
    w.l_off = cnt + ml;
    w.o_off = cnt + 2 * ml;
    w.total = cnt + 2 * ml + align256((size_t)(S * Hq * NP * D) * sizeof(float));
    return w;
}

template <typename T, int D, typename Warp, bool FP8>
int launch_decode(const CUtensorMap& kmap, const CUtensorMap& vmap, const DecodeParams& p,
                  int num_kv_heads, int num_items, cudaStream_t stream) {
    using Pl = Plan<D, FP8, Warp::kMma>;
    const int table_cap = (p.partition_size + p.block_size - 1) / p.block_size + 1;
    const size_t smem = 1024 + Pl::kTableOff + (size_t)table_cap * sizeof(int32_t);
    if (smem > 227 * 1024)
        return fail(PKV_ERR_UNSUPPORTED,
                    "pkv_decode_attention: %d tokens per partition need %zu bytes of shared "
                    "memory; use a smaller partition_size",
                    p.partition_size, smem);
    // the merging CTA keeps the partials' m and l of its G heads in the
    // (then idle) stage buffers
    const size_t merge_smem = (size_t)p.group * (2 * p.num_partitions + 2) * sizeof(float);
    if (p.num_partitions > 1 && merge_smem > Pl::kEpilogue)
        return fail(PKV_ERR_UNSUPPORTED,
                    "pkv_decode_attention: %d partitions of %d query heads are too many to "
                    "merge in one CTA; use a larger partition_size",
                    p.num_partitions, p.group);
    void (*kern)(CUtensorMap, CUtensorMap, DecodeParams) = nullptr;
    if constexpr (FP8 && Warp::GP <= 8)
        kern = paged_decode_kernel_e4m3<T, Warp>;
    else
        kern = paged_decode_kernel<T, D, Warp, FP8>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess)
        return fail(PKV_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
    if (p.num_partitions > 1) {
        e = cudaMemsetAsync(p.ws_count, 0, (size_t)p.num_seqs * num_kv_heads * sizeof(int32_t),
                            stream);
        if (e != cudaSuccess)
            return fail(PKV_ERR_CUDA, "pkv_decode_attention: clearing the partition counters: %s",
                        cudaGetErrorString(e));
    }
    const int64_t ctas = p.work_items != nullptr
                             ? (int64_t)num_items
                             : (int64_t)p.num_seqs * num_kv_heads * p.num_partitions;
    if (ctas >= (1ll << 31))
        return fail(PKV_ERR_UNSUPPORTED, "pkv_decode_attention: %lld CTAs", (long long)ctas);
    kern<<<(unsigned)ctas, kWarps * 32, smem, stream>>>(kmap, vmap, p);
    return launch_status("pkv_decode_attention");
}

template <typename T, int D, bool FP8>
int dispatch_group(const CUtensorMap& kmap, const CUtensorMap& vmap, const DecodeParams& p,
                   int num_kv_heads, int num_items, cudaStream_t stream) {
    // e4m3 caches take the tensor-core path for every group size: its
    // conversions are cheaper per tile than the GEMV's, and the tensor pipe
    // is otherwise idle (G = 1 uses one of the eight MMA columns)
    if constexpr (!FP8) {
        if (p.group == 1)
            return launch_decode<T, D, GemvWarp<T, D>, FP8>(kmap, vmap, p, num_kv_heads,
                                                            num_items, stream);
    }
    if (p.group <= 8)
        return launch_decode<T, D, MmaWarp<T, D, 1, FP8>, FP8>(kmap, vmap, p, num_kv_heads,
                                                               num_items, stream);
    return launch_decode<T, D, MmaWarp<T, D, 2, FP8>, FP8>(kmap, vmap, p, num_kv_heads,
                                                           num_items, stream);
}

// 4-D view of one e4m3 cache: (head_dim codes, kv head, slot, block), boxes
// of 128 x 1 x 16 x 1 codes (one 128-byte row per token) with 128-byte
// swizzling.  block_stride is in bytes.
int encode_cache_map_fp8(CUtensorMap* map, const void* cache, int head_dim, int num_kv_heads,
                         int block_size, int num_blocks, int64_t block_stride) {
    auto fn = encode_fn();
    if (!fn) return fail(PKV_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
    const cuuint64_t dims[4] = {(cuuint64_t)head_dim, (cuuint64_t)num_kv_heads,
                                (cuuint64_t)block_size, (cuuint64_t)num_blocks};
    const cuuint64_t strides[3] = {(cuuint64_t)head_dim, (cuuint64_t)num_kv_heads * head_dim,
                                   (cuuint64_t)block_stride};
    const cuuint32_t box[4] = {(cuuint32_t)head_dim, 1, kTile, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, const_cast<void*>(cache), dims,
                    strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(PKV_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
    return PKV_OK;
}

}  // namespace
}  // namespace pkv

extern "C" size_t pkv_decode_workspace_bytes(int num_seqs, int num_q_heads, int max_context_len,
                                             int partition_size, int head_dim) {
    using namespace pkv;
    if (num_seqs <= 0 || num_q_heads <= 0 || head_dim <= 0 || max_context_len <= 0) return 0;
    int P, NP;
    plan_partitions(max_context_len, partition_size, &P, &NP);
    if (NP <= 1) return 0;
    return workspace_layout(num_seqs, num_q_heads, NP, head_dim).total;
}

namespace pkv {
namespace {

// Both entry points: 16-bit caches (fp8 false) or e4m3 caches with their
// per-(block, KV head) scales (fp8 true; block_stride then in bytes).
int decode_impl(void* out, const void* query, const void* key_cache, const void* value_cache,
                const float* k_scale, const float* v_scale, bool fp8,
                const int32_t* block_tables, int max_blocks_per_seq,
                const int32_t* context_lens, int num_seqs, int max_context_len, int num_q_heads,
                int num_kv_heads, int head_dim, int num_blocks, int block_size,
                int64_t block_stride, float scale, int partition_size, void* workspace,
                size_t workspace_bytes, const int32_t* work_items, int num_items,
                pkv_dtype dtype, int32_t* dev_error, cudaStream_t stream) {
    PKV_REQUIRE(dtype == PKV_F16 || dtype == PKV_BF16, PKV_ERR_UNSUPPORTED,
                "pkv_decode_attention: dtype %d", (int)dtype);
    PKV_REQUIRE(head_dim == 128 || (head_dim == 64 && !fp8), PKV_ERR_UNSUPPORTED,
                "pkv_decode_attention: head_dim %d (built: 64, 128; e4m3 caches: 128)",
                head_dim);
    PKV_REQUIRE(block_size > 0 && block_size % kTile == 0 && block_size <= 256,
                PKV_ERR_UNSUPPORTED,
                "pkv_decode_attention: block_size %d (built: multiples of 16 up to 256)",
                block_size);
    PKV_REQUIRE(num_seqs >= 0 && num_q_heads > 0 && num_kv_heads > 0 && num_blocks >= 0 &&
                    max_blocks_per_seq >= 0 && max_context_len >= 0,
                PKV_ERR_INVALID, "pkv_decode_attention: bad sizes");
    PKV_REQUIRE(num_q_heads % num_kv_heads == 0, PKV_ERR_INVALID,
                "pkv_decode_attention: %d query heads over %d KV heads", num_q_heads,
                num_kv_heads);
    const int group = num_q_heads / num_kv_heads;
    PKV_REQUIRE(group <= 16, PKV_ERR_UNSUPPORTED,
                "pkv_decode_attention: group size %d (built: up to 16)", group);
    PKV_REQUIRE(partition_size >= 0 && partition_size % kTile == 0, PKV_ERR_INVALID,
                "pkv_decode_attention: partition_size %d is not a multiple of 16",
                partition_size);
    PKV_REQUIRE((int64_t)max_context_len <= (int64_t)max_blocks_per_seq * block_size,
                PKV_ERR_INVALID,
                "pkv_decode_attention: max_context_len %d exceeds the table (%d x %d)",
                max_context_len, max_blocks_per_seq, block_size);
    const int64_t block_elems = (int64_t)block_size * num_kv_heads * head_dim;
    PKV_REQUIRE(block_stride >= block_elems && block_stride % (fp8 ? 16 : 8) == 0,
                PKV_ERR_INVALID, "pkv_decode_attention: block_stride %lld",
                (long long)block_stride);
    PKV_REQUIRE(num_kv_heads <= 65535, PKV_ERR_UNSUPPORTED, "too many KV heads");
    PKV_REQUIRE(num_items >= 0, PKV_ERR_INVALID, "pkv_decode_attention_items: %d items",
                num_items);
    if (num_seqs == 0 || (work_items != nullptr && num_items == 0)) return PKV_OK;
    PKV_REQUIRE(out && query && key_cache && value_cache && context_lens &&
                    (block_tables || max_blocks_per_seq == 0),
                PKV_ERR_INVALID, "pkv_decode_attention: NULL pointer");
    PKV_REQUIRE(aligned16(out) && aligned16(query) && aligned16(key_cache) &&
                    aligned16(value_cache),
                PKV_ERR_INVALID, "pkv_decode_attention: pointers must be 16-byte aligned");
    PKV_REQUIRE(num_blocks > 0, PKV_ERR_INVALID, "pkv_decode_attention: empty pool");
    PKV_REQUIRE(!fp8 || (k_scale && v_scale && aligned16(k_scale) && aligned16(v_scale)),
                PKV_ERR_INVALID,
                "pkv_decode_attention_fp8: scales must be 16-byte aligned device arrays");

    DecodeParams p{};
    p.out = out;
    p.query = query;
    p.block_tables = block_tables;
    p.context_lens = context_lens;
    p.dev_error = dev_error;
    p.num_seqs = num_seqs;
    p.num_kv_heads = num_kv_heads;
    p.max_blocks_per_seq = max_blocks_per_seq;
    p.max_context_len = max_context_len;
    p.num_q_heads = num_q_heads;
    p.group = group;
    p.num_blocks = num_blocks;
    p.block_size = block_size;
    p.scale_log2 = scale * kLog2e;
    p.k_scale = k_scale;
    p.v_scale = v_scale;
    p.work_items = work_items;
    plan_partitions(max_context_len, partition_size, &p.partition_size, &p.num_partitions);
    PKV_REQUIRE(p.num_partitions <= 65535, PKV_ERR_UNSUPPORTED,
                "pkv_decode_attention: %d partitions (max 65535)", p.num_partitions);
    PKV_REQUIRE(work_items == nullptr ||
                    (int64_t)num_items <= (int64_t)num_seqs * num_kv_heads * p.num_partitions,
                PKV_ERR_INVALID,
                "pkv_decode_attention_items: %d items for a grid of %lld", num_items,
                (long long)num_seqs * num_kv_heads * p.num_partitions);
    if (p.num_partitions > 1) {
        WorkspaceLayout w = workspace_layout(num_seqs, num_q_heads, p.num_partitions, head_dim);
        PKV_REQUIRE(workspace != nullptr && workspace_bytes >= w.total && aligned16(workspace),
                    PKV_ERR_WORKSPACE,
                    "pkv_decode_attention: needs %zu bytes of 16-byte aligned workspace, got %zu",
                    w.total, workspace ? workspace_bytes : (size_t)0);
        uint8_t* base = static_cast<uint8_t*>(workspace);
        p.ws_m = reinterpret_cast<float*>(base + w.m_off);
        p.ws_l = reinterpret_cast<float*>(base + w.l_off);
        p.ws_o = reinterpret_cast<float*>(base + w.o_off);
        p.ws_count = reinterpret_cast<int32_t*>(base + w.count_off);
    }

    CUtensorMap kmap, vmap;
    int st = fp8 ? encode_cache_map_fp8(&kmap, key_cache, head_dim, num_kv_heads, block_size,
                                        num_blocks, block_stride)
                 : encode_cache_map(&kmap, key_cache, dtype, head_dim, num_kv_heads, block_size,
                                    num_blocks, block_stride);
    if (st != PKV_OK) return st;
    st = fp8 ? encode_cache_map_fp8(&vmap, value_cache, head_dim, num_kv_heads, block_size,
                                    num_blocks, block_stride)
             : encode_cache_map(&vmap, value_cache, dtype, head_dim, num_kv_heads, block_size,
                                num_blocks, block_stride);
    if (st != PKV_OK) return st;

    DeviceGuard guard(stream, key_cache);
    const int n = num_items;
    if (fp8) {
        return dtype == PKV_BF16
                   ? dispatch_group<__nv_bfloat16, 128, true>(kmap, vmap, p, num_kv_heads, n, stream)
                   : dispatch_group<__half, 128, true>(kmap, vmap, p, num_kv_heads, n, stream);
    }
    if (dtype == PKV_BF16) {
        return head_dim == 128
                   ? dispatch_group<__nv_bfloat16, 128, false>(kmap, vmap, p, num_kv_heads, n,
                                                               stream)
                   : dispatch_group<__nv_bfloat16, 64, false>(kmap, vmap, p, num_kv_heads, n,
                                                              stream);
    }
    return head_dim == 128
               ? dispatch_group<__half, 128, false>(kmap, vmap, p, num_kv_heads, n, stream)
               : dispatch_group<__half, 64, false>(kmap, vmap, p, num_kv_heads, n, stream);
}

}  // namespace
}  // namespace pkv

extern "C" int pkv_decode_attention(void* out, const void* query, const void* key_cache,
                                    const void* value_cache, const int32_t* block_tables,
                                    int max_blocks_per_seq, const int32_t* context_lens,
                                    int num_seqs, int max_context_len, int num_q_heads,
                                    int num_kv_heads, int head_dim, int num_blocks,
                                    int block_size, int64_t block_stride, float scale,
                                    int partition_size, void* workspace, size_t workspace_bytes,
                                    pkv_dtype dtype, int32_t* dev_error, cudaStream_t stream) {
    PKV_NVTX_RANGE("pkv_decode_attention");
    return pkv::decode_impl(out, query, key_cache, value_cache, nullptr, nullptr, false,
                            block_tables, max_blocks_per_seq, context_lens, num_seqs,
                            max_context_len, num_q_heads, num_kv_heads, head_dim, num_blocks,
                            block_size, block_stride, scale, partition_size, workspace,
                            workspace_bytes, nullptr, 0, dtype, dev_error, stream);
}

extern "C" int pkv_decode_attention_fp8(void* out, const void* query, const void* key_cache,
                                        const void* value_cache, const float* k_scale,
                                        const float* v_scale, const int32_t* block_tables,
                                        int max_blocks_per_seq, const int32_t* context_lens,
                                        int num_seqs, int max_context_len, int num_q_heads,
                                        int num_kv_heads, int head_dim, int num_blocks,
                                        int block_size, int64_t block_stride, float scale,
                                        int partition_size, void* workspace,
                                        size_t workspace_bytes, pkv_dtype dtype,
                                        int32_t* dev_error, cudaStream_t stream) {
    PKV_NVTX_RANGE("pkv_decode_attention_fp8");
    return pkv::decode_impl(out, query, key_cache, value_cache, k_scale, v_scale, true,
                            block_tables, max_blocks_per_seq, context_lens, num_seqs,
                            max_context_len, num_q_heads, num_kv_heads, head_dim, num_blocks,
                            block_size, block_stride, scale, partition_size, workspace,
                            workspace_bytes, nullptr, 0, dtype, dev_error, stream);
}

extern "C" int pkv_decode_attention_items(void* out, const void* query, const void* key_cache,
                                          const void* value_cache, const int32_t* block_tables,
                                          int max_blocks_per_seq, const int32_t* context_lens,
                                          int num_seqs, int max_context_len, int num_q_heads,
                                          int num_kv_heads, int head_dim, int num_blocks,
                                          int block_size, int64_t block_stride, float scale,
                                          int partition_size, void* workspace,
                                          size_t workspace_bytes, const int32_t* work_items,
                                          int num_items, pkv_dtype dtype, int32_t* dev_error,
                                          cudaStream_t stream) {
    PKV_NVTX_RANGE("pkv_decode_attention_items");
    PKV_REQUIRE(work_items != nullptr || num_items == 0, PKV_ERR_INVALID,
                "pkv_decode_attention_items: NULL work list");
    if (num_items == 0) return PKV_OK;
    return pkv::decode_impl(out, query, key_cache, value_cache, nullptr, nullptr, false,
                            block_tables, max_blocks_per_seq, context_lens, num_seqs,
                            max_context_len, num_q_heads, num_kv_heads, head_dim, num_blocks,
                            block_size, block_stride, scale, partition_size, workspace,
                            workspace_bytes, work_items, num_items, dtype, dev_error, stream);
}

extern "C" int pkv_decode_attention_fp8_items(
    void* out, const void* query, const void* key_cache, const void* value_cache,
    const float* k_scale, const float* v_scale, const int32_t* block_tables,
    int max_blocks_per_seq, const int32_t* context_lens, int num_seqs, int max_context_len,
    int num_q_heads, int num_kv_heads, int head_dim, int num_blocks, int block_size,
    int64_t block_stride, float scale, int partition_size, void* workspace,
    size_t workspace_bytes, const int32_t* work_items, int num_items, pkv_dtype dtype,
    int32_t* dev_error, cudaStream_t stream) {
    PKV_NVTX_RANGE("pkv_decode_attention_fp8_items");
    PKV_REQUIRE(work_items != nullptr || num_items == 0, PKV_ERR_INVALID,
                "pkv_decode_attention_fp8_items: NULL work list");
    if (num_items == 0) return PKV_OK;
    return pkv::decode_impl(out, query, key_cache, value_cache, k_scale, v_scale, true,
                            block_tables, max_blocks_per_seq, context_lens, num_seqs,
                            max_context_len, num_q_heads, num_kv_heads, head_dim, num_blocks,
                            block_size, block_stride, scale, partition_size, workspace,
                            workspace_bytes, work_items, num_items, dtype, dev_error, stream);
}
