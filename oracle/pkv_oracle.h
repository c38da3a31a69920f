/*
 * pkv_oracle.h — declarations of the fp64 CPU oracle (test infrastructure
 * only; see pkv_oracle.c).  This header is private to oracle/ and shares
 * nothing with the product library's headers.
 */
#ifndef PKV_ORACLE_H
#define PKV_ORACLE_H
#include <stdint.h>

#define PKV_ORACLE_F16 0
#define PKV_ORACLE_BF16 1

#ifdef __cplusplus
extern "C" {
#endif

double pkv_oracle_bf16_to_f64(uint16_t bits);
double pkv_oracle_f16_to_f64(uint16_t bits);

int pkv_oracle_decode_attention(double* out, const uint16_t* query,
                                const uint16_t* key_cache,
                                const uint16_t* value_cache,
                                const int32_t* block_tables,
                                int max_blocks_per_seq,
                                const int32_t* context_lens, int num_seqs,
                                int num_q_heads, int num_kv_heads, int head_dim,
                                int num_blocks, int block_size,
                                int64_t block_stride, double scale, int dtype,
                                int num_threads);

int pkv_oracle_prefill_attention(double* out, const uint16_t* query,
                                 const uint16_t* key_cache, const uint16_t* value_cache,
                                 const int32_t* block_tables, int max_blocks_per_seq,
                                 const int32_t* context_lens, const int32_t* query_start,
                                 int num_seqs, int num_q_heads, int num_kv_heads,
                                 int head_dim, int num_blocks, int block_size,
                                 int64_t block_stride, double scale, int dtype,
                                 int num_threads);

int pkv_oracle_decode_partials(double* m_out, double* l_out, double* o_out,
                               const uint16_t* query, const uint16_t* key_cache,
                               const uint16_t* value_cache,
                               const int32_t* block_tables,
                               int max_blocks_per_seq,
                               const int32_t* context_lens, int num_seqs,
                               int num_q_heads, int num_kv_heads, int head_dim,
                               int num_blocks, int block_size,
                               int64_t block_stride, double scale, int dtype,
                               int partition_size, int num_partitions);

int pkv_oracle_merge_partials(double* out, const double* m, const double* l,
                              const double* o, const int32_t* context_lens,
                              int num_seqs, int num_q_heads, int head_dim,
                              int partition_size, int num_partitions);

int pkv_oracle_write_slots(uint16_t* key_cache, uint16_t* value_cache,
                           const uint16_t* key, const uint16_t* value,
                           const int64_t* slot_mapping, int num_tokens,
                           int num_blocks, int block_size, int num_kv_heads,
                           int head_dim, int64_t block_stride);

int pkv_oracle_copy_blocks(uint16_t* key_cache, uint16_t* value_cache,
                           const int32_t* block_pairs, int num_pairs,
                           int num_blocks, int block_size, int num_kv_heads,
                           int head_dim, int64_t block_stride);

int pkv_oracle_swap_blocks(uint8_t* dst, const uint8_t* src, const int32_t* block_pairs,
                           int num_pairs, int src_num_blocks, int dst_num_blocks,
                           int64_t block_bytes, int64_t src_block_stride,
                           int64_t dst_block_stride);

int64_t pkv_oracle_block_bytes(int block_size, int num_kv_heads, int head_dim,
                               int num_layers, int dtype_bytes);

int pkv_oracle_max_threads(void);

double pkv_oracle_e4m3_to_f64(uint8_t code);
uint8_t pkv_oracle_f32_to_e4m3_sat(float x);
int pkv_oracle_write_slots_fp8(uint8_t* key_cache, uint8_t* value_cache,
                               const uint16_t* key, const uint16_t* value,
                               const int64_t* slot_mapping, int num_tokens,
                               int num_blocks, int block_size, int num_kv_heads,
                               int head_dim, int64_t block_stride,
                               const float* k_scale, const float* v_scale,
                               int dtype);
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
                                    int num_threads);

#ifdef __cplusplus
}
#endif
#endif
