/*
 * pkv_oracle.c — plain, slow, obviously correct CPU oracle for the paged KV
 * cache hot path.  TEST INFRASTRUCTURE ONLY: the tests, the smoke check and
 * the CPU-baseline leg of the benchmark call it; the product library never
 * links, includes or calls anything here, and nothing here is shared with the
 * CUDA path.
 *
 * Every floating-point result is computed in IEEE binary64.  The 16-bit cache
 * values are widened to double exactly (both fp16 and bf16 are subsets of
 * binary64), so the only rounding in this file is the fp64 arithmetic itself.
 *
 * Sources (web pages on PagedAttention):
 *  - "Paged KV" wiki page, section "实现原理 / 初始化阶段": every physical
 *    block holds K and V of shape [block_size, num_kv_heads, head_dim].
 *  - same page, section "实现原理 / 运行阶段": a per-sequence Block Table maps
 *    logical block i to a physical block; during decode each new token is
 *    written to the next slot of the current block.
 *  - same page, section "Attention Kernel 的适配": the kernel takes the Block
 *    Table and block_size and reads K/V block by block through indirection.
 *  - "一文读懂vLLM的…PagedAttention" page, opening paragraphs: PagedAttention
 *    is a cache-management scheme, not a new attention algorithm, so the
 *    result is ordinary softmax attention over the sequence's tokens in
 *    logical order.
 *  - "PagedAttention 动态内存分页" page, section "写时复制与内存共享": a block
 *    shared by several sequences is copied before one of them writes into it.
 *
 * Readings where the pages are silent (each also listed in the design notes):
 *  - a query head h reads KV head h / (Hq / Hkv)  (contiguous GQA groups);
 *  - context_lens[s] counts every cached token including the one just
 *    written; the query attends to all of them;
 *  - the score is scale * dot(q, k), taken before the softmax max;
 *  - context_lens[s] == 0 gives an all-zero output (empty sum);
 *  - a negative slot in slot_mapping means "no write" (padding).
 *
 * Status codes: 0 ok, -1 invalid argument or metadata.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#include "pkv_oracle.h"

/* ---- exact widening of the 16-bit storage formats ----------------------- */

/* bfloat16 is the upper half of an IEEE binary32: shift it back into place. */
double pkv_oracle_bf16_to_f64(uint16_t bits) {
    uint32_t w = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &w, sizeof f);
    return (double)f;
}

/* IEEE binary16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits. */
double pkv_oracle_f16_to_f64(uint16_t bits) {
    int sign = (bits >> 15) & 1;
    int expo = (bits >> 10) & 0x1f;
    int frac = bits & 0x3ff;
    double mag;
    if (expo == 0) {
        mag = ldexp((double)frac, -24);          /* zero or subnormal */
    } else if (expo == 31) {
        mag = frac ? NAN : INFINITY;
    } else {
        mag = ldexp((double)(1024 + frac), expo - 25);
    }
    return sign ? -mag : mag;
}

static double widen(uint16_t bits, int dtype) {
    return dtype == PKV_ORACLE_BF16 ? pkv_oracle_bf16_to_f64(bits)
                                    : pkv_oracle_f16_to_f64(bits);
}

/* ---- addressing through the block table -------------------------------- */

/* Element offset of (physical block b, slot o, kv head h, dim 0): a block is
 * [block_size, num_kv_heads, head_dim] contiguous; blocks sit block_stride
 * elements apart. */
static int64_t slot_offset(int64_t b, int64_t o, int64_t h, int64_t Hkv,
                           int64_t D, int64_t block_stride) {
    return b * block_stride + (o * Hkv + h) * D;
}

static int check_shapes(int S, int Hq, int Hkv, int D, int NB, int bs,
                        int64_t block_stride, int MB) {
    if (S < 0 || Hq <= 0 || Hkv <= 0 || D <= 0 || NB < 0 || bs <= 0 || MB < 0)
        return -1;
    if (Hq % Hkv != 0) return -1;
    if (block_stride < (int64_t)bs * Hkv * D) return -1;
    return 0;
}

/* Check that sequence s's first ceil(L/bs) table entries name real blocks. */
static int check_seq(const int32_t* tables, int MB, const int32_t* lens,
                     int s, int NB, int bs) {
    int L = lens[s];
    if (L < 0 || (int64_t)L > (int64_t)MB * bs) return -1;
    int nblk = (L + bs - 1) / bs;
    for (int i = 0; i < nblk; ++i) {
        int32_t b = tables[(int64_t)s * MB + i];
        if (b < 0 || b >= NB) return -1;
    }
    return 0;
}

/*
 * Attention of one query head over tokens [t0, t1) of sequence s, gathered
 * in logical order.  Writes the running maximum m, the sum of exponentials
 * l = sum_t exp(s_t - m) and the unnormalised o = sum_t exp(s_t - m) v_t.
 * With t0 == t1 it writes m = -inf, l = 0, o = 0.
 */
static void attend_range(double* m_out, double* l_out, double* o_out,
                         const uint16_t* q, const uint16_t* kc,
                         const uint16_t* vc, const int32_t* table, int t0,
                         int t1, int kvh, int Hkv, int D, int bs,
                         int64_t block_stride, double scale, int dtype,
                         double* scores /* scratch, >= t1 - t0 */) {
    /* step 1: scores s_t = scale * <q, k_t> over the gathered keys */
    double m = -INFINITY;
    for (int t = t0; t < t1; ++t) {
        int64_t b = table[t / bs];
        int64_t o = t % bs;
        const uint16_t* k = kc + slot_offset(b, o, kvh, Hkv, D, block_stride);
        double dot = 0.0;
        for (int d = 0; d < D; ++d) dot += widen(q[d], dtype) * widen(k[d], dtype);
        double st = scale * dot;
        scores[t - t0] = st;
        if (st > m) m = st;
    }
    /* step 2: exponentials relative to the maximum, and their sum */
    double l = 0.0;
    for (int d = 0; d < D; ++d) o_out[d] = 0.0;
    for (int t = t0; t < t1; ++t) {
        double w = exp(scores[t - t0] - m);
        l += w;
        int64_t b = table[t / bs];
        int64_t o = t % bs;
        const uint16_t* v = vc + slot_offset(b, o, kvh, Hkv, D, block_stride);
        /* step 3: weighted sum of the gathered values */
        for (int d = 0; d < D; ++d) o_out[d] += w * widen(v[d], dtype);
    }
    *m_out = m;
    *l_out = l;
}

int pkv_oracle_decode_attention(double* out, const uint16_t* query,
                                const uint16_t* key_cache,
                                const uint16_t* value_cache,
                                const int32_t* block_tables,
                                int max_blocks_per_seq,
                                const int32_t* context_lens, int num_seqs,
                                int num_q_heads, int num_kv_heads, int head_dim,
                                int num_blocks, int block_size,
                                int64_t block_stride, double scale, int dtype,
                                int num_threads) {
    const int S = num_seqs, Hq = num_q_heads, Hkv = num_kv_heads, D = head_dim;
    const int MB = max_blocks_per_seq, bs = block_size;
    if (check_shapes(S, Hq, Hkv, D, num_blocks, bs, block_stride, MB)) return -1;
    int max_len = 0;
    for (int s = 0; s < S; ++s) {
        if (check_seq(block_tables, MB, context_lens, s, num_blocks, bs)) return -1;
        if (context_lens[s] > max_len) max_len = context_lens[s];
    }
    const int G = Hq / Hkv;
    int bad = 0;
#ifdef _OPENMP
    omp_set_num_threads(num_threads > 0 ? num_threads : omp_get_num_procs());
#else
    (void)num_threads;
#endif
#pragma omp parallel reduction(| : bad)
    {
        double* scores = (double*)malloc(sizeof(double) * (size_t)(max_len > 0 ? max_len : 1));
        if (!scores) bad = 1;
#pragma omp for schedule(dynamic, 1)
        for (int64_t sh = 0; sh < (int64_t)S * Hq; ++sh) {
            if (!scores) continue;
            int s = (int)(sh / Hq), h = (int)(sh % Hq);
            int kvh = h / G; /* contiguous GQA groups */
            double* o = out + sh * D;
            const uint16_t* q = query + sh * D;
            int L = context_lens[s];
            double m, l;
            attend_range(&m, &l, o, q, key_cache, value_cache,
                         block_tables + (int64_t)s * MB, 0, L, kvh, Hkv, D, bs,
                         block_stride, scale, dtype, scores);
            /* normalise; an empty context leaves o at zero */
            if (L > 0)
                for (int d = 0; d < D; ++d) o[d] /= l;
        }
        free(scores);
    }
    return bad ? -1 : 0;
}

/* Paged prefill attention ("Paged KV" wiki page, 实现原理 / 运行阶段: prefill
 * takes blocks in order and fills them with the prompt's K/V; the prompt's
 * tokens then attend to the sequence through the same Block Table).  The
 * query rows of sequence s are query_start[s] .. query_start[s+1]-1: the
 * last n_s of its L_s = context_lens[s] cached tokens (a prompt, or a later
 * chunk of one after L_s - n_s tokens already cached).  Row query_start[s]
 * + i is token p = L_s - n_s + i and attends causally, to tokens 0 .. p:
 *     out[row, h] = sum_{t <= p} softmax_t(scale * <query[row, h], K_t>) V_t. */
int pkv_oracle_prefill_attention(double* out, const uint16_t* query,
                                 const uint16_t* key_cache, const uint16_t* value_cache,
                                 const int32_t* block_tables, int max_blocks_per_seq,
                                 const int32_t* context_lens, const int32_t* query_start,
                                 int num_seqs, int num_q_heads, int num_kv_heads,
                                 int head_dim, int num_blocks, int block_size,
                                 int64_t block_stride, double scale, int dtype,
                                 int num_threads) {
    const int S = num_seqs, Hq = num_q_heads, Hkv = num_kv_heads, D = head_dim;
    const int MB = max_blocks_per_seq, bs = block_size;
    if (check_shapes(S, Hq, Hkv, D, num_blocks, bs, block_stride, MB)) return -1;
    if (query_start[0] != 0) return -1;
    int max_len = 0;
    for (int s = 0; s < S; ++s) {
        if (check_seq(block_tables, MB, context_lens, s, num_blocks, bs)) return -1;
        const int n = query_start[s + 1] - query_start[s];
        if (n < 0 || n > context_lens[s]) return -1;
        if (context_lens[s] > max_len) max_len = context_lens[s];
    }
    const int64_t rows = query_start[S];
    const int G = Hq / Hkv;
    int bad = 0;
#ifdef _OPENMP
    omp_set_num_threads(num_threads > 0 ? num_threads : omp_get_num_procs());
#else
    (void)num_threads;
#endif
#pragma omp parallel reduction(| : bad)
    {
        double* scores = (double*)malloc(sizeof(double) * (size_t)(max_len > 0 ? max_len : 1));
        if (!scores) bad = 1;
#pragma omp for schedule(dynamic, 4)
        for (int64_t rh = 0; rh < rows * Hq; ++rh) {
            if (!scores) continue;
            const int64_t row = rh / Hq;
            const int h = (int)(rh % Hq);
            int s = 0; /* the sequence holding this row */
            while (query_start[s + 1] <= row) ++s;
            const int n = query_start[s + 1] - query_start[s];
            const int p = context_lens[s] - n + (int)(row - query_start[s]);
            double m, l;
            double* o = out + rh * D;
            attend_range(&m, &l, o, query + rh * D, key_cache, value_cache,
                         block_tables + (int64_t)s * MB, 0, p + 1, h / G, Hkv, D, bs,
                         block_stride, scale, dtype, scores);
            for (int d = 0; d < D; ++d) o[d] /= l;
        }
        free(scores);
    }
    return bad ? -1 : 0;
}

int pkv_oracle_decode_partials(double* m_out, double* l_out, double* o_out,
                               const uint16_t* query, const uint16_t* key_cache,
                               const uint16_t* value_cache,
                               const int32_t* block_tables,
                               int max_blocks_per_seq,
                               const int32_t* context_lens, int num_seqs,
                               int num_q_heads, int num_kv_heads, int head_dim,
                               int num_blocks, int block_size,
                               int64_t block_stride, double scale, int dtype,
                               int partition_size, int num_partitions) {
    const int S = num_seqs, Hq = num_q_heads, Hkv = num_kv_heads, D = head_dim;
    const int MB = max_blocks_per_seq, bs = block_size, P = partition_size;
    const int NP = num_partitions;
    if (check_shapes(S, Hq, Hkv, D, num_blocks, bs, block_stride, MB)) return -1;
    if (P <= 0 || NP <= 0) return -1;
    for (int s = 0; s < S; ++s) {
        if (check_seq(block_tables, MB, context_lens, s, num_blocks, bs)) return -1;
        if ((int64_t)context_lens[s] > (int64_t)P * NP) return -1;
    }
    const int G = Hq / Hkv;
    double* scores = (double*)malloc(sizeof(double) * (size_t)P);
    if (!scores) return -1;
    for (int s = 0; s < S; ++s) {
        int L = context_lens[s];
        for (int h = 0; h < Hq; ++h) {
            for (int p = 0; p < NP; ++p) {
                int64_t idx = ((int64_t)s * Hq + h) * NP + p;
                int t0 = p * P;
                int t1 = t0 + P < L ? t0 + P : L;
                if (t1 < t0) t1 = t0;
                attend_range(m_out + idx, l_out + idx, o_out + idx * D,
                             query + ((int64_t)s * Hq + h) * D, key_cache,
                             value_cache, block_tables + (int64_t)s * MB, t0,
                             t1, h / G, Hkv, D, bs, block_stride, scale, dtype,
                             scores);
            }
        }
    }
    free(scores);
    return 0;
}

/*
 * Merge of per-partition partials (m_p, l_p, o_p): with M = max_p m_p and
 * w_p = exp(m_p - M), out = sum_p w_p o_p / sum_p w_p l_p.  Only the
 * partitions that hold tokens (p < ceil(L / P)) take part.
 */
int pkv_oracle_merge_partials(double* out, const double* m, const double* l,
                              const double* o, const int32_t* context_lens,
                              int num_seqs, int num_q_heads, int head_dim,
                              int partition_size, int num_partitions) {
    const int S = num_seqs, Hq = num_q_heads, D = head_dim;
    const int P = partition_size, NP = num_partitions;
    if (P <= 0 || NP <= 0) return -1;
    for (int s = 0; s < S; ++s) {
        int L = context_lens[s];
        if (L < 0 || (int64_t)L > (int64_t)P * NP) return -1;
        int np = (L + P - 1) / P;
        for (int h = 0; h < Hq; ++h) {
            int64_t base = ((int64_t)s * Hq + h) * NP;
            double* dst = out + ((int64_t)s * Hq + h) * D;
            for (int d = 0; d < D; ++d) dst[d] = 0.0;
            if (np == 0) continue;
            double M = -INFINITY;
            for (int p = 0; p < np; ++p)
                if (m[base + p] > M) M = m[base + p];
            double den = 0.0;
            for (int p = 0; p < np; ++p) {
                double w = exp(m[base + p] - M);
                den += w * l[base + p];
                for (int d = 0; d < D; ++d) dst[d] += w * o[(base + p) * D + d];
            }
            for (int d = 0; d < D; ++d) dst[d] /= den;
        }
    }
    return 0;
}

/*
 * Slot write: token t's K and V rows go to physical block slot / block_size,
 * offset slot % block_size ("Paged KV" wiki, 运行阶段: a decoded token is
 * written into the next slot of the current block).  Negative slots are
 * skipped.  Slots must be distinct and below num_blocks * block_size.
 */
int pkv_oracle_write_slots(uint16_t* key_cache, uint16_t* value_cache,
                           const uint16_t* key, const uint16_t* value,
                           const int64_t* slot_mapping, int num_tokens,
                           int num_blocks, int block_size, int num_kv_heads,
                           int head_dim, int64_t block_stride) {
    const int64_t row = (int64_t)num_kv_heads * head_dim;
    const int64_t nslots = (int64_t)num_blocks * block_size;
    if (num_tokens < 0 || block_size <= 0 || row <= 0) return -1;
    if (block_stride < (int64_t)block_size * row) return -1;
    for (int t = 0; t < num_tokens; ++t) {
        int64_t st = slot_mapping[t];
        if (st < 0) continue;
        if (st >= nslots) return -1;
        for (int u = 0; u < t; ++u)
            if (slot_mapping[u] == st) return -1; /* slots must be distinct */
    }
    for (int t = 0; t < num_tokens; ++t) {
        int64_t st = slot_mapping[t];
        if (st < 0) continue;
        int64_t dst = slot_offset(st / block_size, st % block_size, 0,
                                  num_kv_heads, head_dim, block_stride);
        memcpy(key_cache + dst, key + (int64_t)t * row, sizeof(uint16_t) * row);
        memcpy(value_cache + dst, value + (int64_t)t * row, sizeof(uint16_t) * row);
    }
    return 0;
}

/*
 * Copy-on-write block copy: for each pair (src, dst) in order, the whole
 * block dst of K and of V becomes a copy of block src ("PagedAttention 动态
 * 内存分页" page, 写时复制与内存共享).
 */
int pkv_oracle_copy_blocks(uint16_t* key_cache, uint16_t* value_cache,
                           const int32_t* block_pairs, int num_pairs,
                           int num_blocks, int block_size, int num_kv_heads,
                           int head_dim, int64_t block_stride) {
    const int64_t elems = (int64_t)block_size * num_kv_heads * head_dim;
    if (num_pairs < 0 || elems <= 0 || block_stride < elems) return -1;
    for (int i = 0; i < num_pairs; ++i) {
        int32_t src = block_pairs[2 * i], dst = block_pairs[2 * i + 1];
        if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks) return -1;
    }
    for (int i = 0; i < num_pairs; ++i) {
        int64_t src = block_pairs[2 * i], dst = block_pairs[2 * i + 1];
        memmove(key_cache + dst * block_stride, key_cache + src * block_stride,
                sizeof(uint16_t) * elems);
        memmove(value_cache + dst * block_stride, value_cache + src * block_stride,
                sizeof(uint16_t) * elems);
    }
    return 0;
}

/* Block swap between two pools ("PagedAttention 动态内存分页" page, 动态块分配
 * 与回收: under memory pressure a sequence's KV blocks move to CPU memory and
 * come back when it runs again).  For every pair (src, dst), the block_bytes
 * bytes of block src of the source pool become block dst of the destination
 * pool.  The pools are distinct arrays; blocks are block_bytes long at their
 * own strides.  Any pair outside its pool: nothing is copied, -1. */
int pkv_oracle_swap_blocks(uint8_t* dst, const uint8_t* src, const int32_t* block_pairs,
                           int num_pairs, int src_num_blocks, int dst_num_blocks,
                           int64_t block_bytes, int64_t src_block_stride,
                           int64_t dst_block_stride) {
    if (num_pairs < 0 || block_bytes < 0 || src_block_stride < block_bytes ||
        dst_block_stride < block_bytes)
        return -1;
    for (int i = 0; i < num_pairs; ++i) {
        int32_t s = block_pairs[2 * i], d = block_pairs[2 * i + 1];
        if (s < 0 || s >= src_num_blocks || d < 0 || d >= dst_num_blocks) return -1;
    }
    for (int i = 0; i < num_pairs; ++i) {
        int64_t s = block_pairs[2 * i], d = block_pairs[2 * i + 1];
        memcpy(dst + d * dst_block_stride, src + s * src_block_stride, (size_t)block_bytes);
    }
    return 0;
}

/* Bytes of one physical block, as the "Paged KV" wiki page's 初始化阶段
 * section gives them: block_size x num_kv_heads x head_dim x 2 (K and V)
 * x num_layers x dtype_bytes. */
int64_t pkv_oracle_block_bytes(int block_size, int num_kv_heads, int head_dim,
                               int num_layers, int dtype_bytes) {
    return (int64_t)block_size * num_kv_heads * head_dim * 2 * num_layers *
           dtype_bytes;
}

int pkv_oracle_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ======================================================================== */
/* FP8 (e4m3) KV cache with a scale per (block, KV head)                     */
/* ======================================================================== */
/*
 * "Paged KV" wiki page, section 局限性: some KV quantisation schemes, such as
 * FP8 with a scale per block, tie the block size to the quantisation.  The
 * reading taken here: K and V are stored as e4m3 codes (1 sign, 4 exponent
 * bits with bias 7, 3 fraction bits; no infinities; S.1111.111 is NaN;
 * largest finite 448), and every (physical block, KV head) has one fp32 scale
 * for K and one for V: value = decode(code) * scale.  A value is stored as
 * the e4m3 code nearest to (fp32) x / scale, ties to an even code, with
 * magnitudes beyond 448 saturating to 448.
 */

double pkv_oracle_e4m3_to_f64(uint8_t code) {
    int sign = (code >> 7) & 1;
    int expo = (code >> 3) & 0xf;
    int frac = code & 0x7;
    double mag;
    if (expo == 0xf && frac == 0x7) {
        mag = NAN;
    } else if (expo == 0) {
        mag = ldexp((double)frac, -9);               /* zero or subnormal */
    } else {
        mag = ldexp((double)(8 + frac), expo - 10);  /* (1 + f/8) 2^(e-7) */
    }
    return sign ? -mag : mag;
}

/* Nearest e4m3 code by exhaustive search over the 127 finite magnitudes. */
uint8_t pkv_oracle_f32_to_e4m3_sat(float x) {
    if (x != x) return 0x7f;
    const double a = fabs((double)x);
    int best = 0;
    double best_err = INFINITY;
    for (int c = 0; c <= 0x7e; ++c) {
        const double err = fabs(pkv_oracle_e4m3_to_f64((uint8_t)c) - a);
        /* strictly better, or as good with an even code (ties to even) */
        if (err < best_err || (err == best_err && (c & 1) == 0)) {
            best = c;
            best_err = err;
        }
    }
    return (uint8_t)(best | (signbit(x) ? 0x80 : 0));  /* -0 keeps its sign */
}

static double fp8_elem(const uint8_t* cache, int64_t idx, const float* scales,
                       int64_t scale_idx) {
    return pkv_oracle_e4m3_to_f64(cache[idx]) * (double)scales[scale_idx];
}

/* Slot write into e4m3 caches: token t, KV head h goes to block b = slot /
 * block_size with the code of (float)x / scale[b * Hkv + h]. */
int pkv_oracle_write_slots_fp8(uint8_t* key_cache, uint8_t* value_cache,
                               const uint16_t* key, const uint16_t* value,
                               const int64_t* slot_mapping, int num_tokens,
                               int num_blocks, int block_size, int num_kv_heads,
                               int head_dim, int64_t block_stride,
                               const float* k_scale, const float* v_scale,
                               int dtype) {
    const int Hkv = num_kv_heads, D = head_dim;
    const int64_t nslots = (int64_t)num_blocks * block_size;
    if (num_tokens < 0 || block_size <= 0 || Hkv <= 0 || D <= 0) return -1;
    if (block_stride < (int64_t)block_size * Hkv * D) return -1;
    for (int t = 0; t < num_tokens; ++t) {
        int64_t st = slot_mapping[t];
        if (st < 0) continue;
        if (st >= nslots) return -1;
        for (int u = 0; u < t; ++u)
            if (slot_mapping[u] == st) return -1;
    }
    for (int t = 0; t < num_tokens; ++t) {
        int64_t st = slot_mapping[t];
        if (st < 0) continue;
        int64_t b = st / block_size, o = st % block_size;
        for (int h = 0; h < Hkv; ++h) {
            const float ks = k_scale[b * Hkv + h], vs = v_scale[b * Hkv + h];
            const int64_t dst = slot_offset(b, o, h, Hkv, D, block_stride);
            const int64_t src = ((int64_t)t * Hkv + h) * D;
            for (int d = 0; d < D; ++d) {
                const float kx = (float)widen(key[src + d], dtype);
                const float vx = (float)widen(value[src + d], dtype);
                key_cache[dst + d] = pkv_oracle_f32_to_e4m3_sat(kx / ks);
                value_cache[dst + d] = pkv_oracle_f32_to_e4m3_sat(vx / vs);
            }
        }
    }
    return 0;
}

/* Paged decode attention over e4m3 caches: the same definition as
 * pkv_oracle_decode_attention with K and V dequantised exactly in fp64. */
int pkv_oracle_decode_attention_fp8(double* out, const uint16_t* query,
                                    const uint8_t* key_cache,
                                    const uint8_t* value_cache,
                                    const float* k_scale, const float* v_scale,
                                    const int32_t* block_tables,
                                    int max_blocks_per_seq,
                                    const int32_t* context_lens, int num_seqs,
                                    int num_q_heads, int num_kv_heads, int head_dim,
                                    int num_blocks, int block_size,
                                    int64_t block_stride, double scale, int dtype,
                                    int num_threads) {
    const int S = num_seqs, Hq = num_q_heads, Hkv = num_kv_heads, D = head_dim;
    const int MB = max_blocks_per_seq, bs = block_size;
    if (check_shapes(S, Hq, Hkv, D, num_blocks, bs, block_stride, MB)) return -1;
    int max_len = 0;
    for (int s = 0; s < S; ++s) {
        if (check_seq(block_tables, MB, context_lens, s, num_blocks, bs)) return -1;
        if (context_lens[s] > max_len) max_len = context_lens[s];
    }
    const int G = Hq / Hkv;
    int bad = 0;
#ifdef _OPENMP
    omp_set_num_threads(num_threads > 0 ? num_threads : omp_get_num_procs());
#else
    (void)num_threads;
#endif
#pragma omp parallel reduction(| : bad)
    {
        double* scores = (double*)malloc(sizeof(double) * (size_t)(max_len > 0 ? max_len : 1));
        if (!scores) bad = 1;
#pragma omp for schedule(dynamic, 1)
        for (int64_t sh = 0; sh < (int64_t)S * Hq; ++sh) {
            if (!scores) continue;
            int s = (int)(sh / Hq), h = (int)(sh % Hq);
            int kvh = h / G;
            const int32_t* table = block_tables + (int64_t)s * MB;
            const uint16_t* q = query + sh * D;
            double* o = out + sh * D;
            int L = context_lens[s];
            double m = -INFINITY;
            for (int t = 0; t < L; ++t) {
                int64_t b = table[t / bs], off = t % bs;
                int64_t base = slot_offset(b, off, kvh, Hkv, D, block_stride);
                double dot = 0.0;
                for (int d = 0; d < D; ++d)
                    dot += widen(q[d], dtype) * fp8_elem(key_cache, base + d, k_scale, b * Hkv + kvh);
                scores[t] = scale * dot;
                if (scores[t] > m) m = scores[t];
            }
            double l = 0.0;
            for (int d = 0; d < D; ++d) o[d] = 0.0;
            for (int t = 0; t < L; ++t) {
                double w = exp(scores[t] - m);
                l += w;
                int64_t b = table[t / bs], off = t % bs;
                int64_t base = slot_offset(b, off, kvh, Hkv, D, block_stride);
                for (int d = 0; d < D; ++d)
                    o[d] += w * fp8_elem(value_cache, base + d, v_scale, b * Hkv + kvh);
            }
            if (L > 0)
                for (int d = 0; d < D; ++d) o[d] /= l;
        }
        free(scores);
    }
    return bad ? -1 : 0;
}
