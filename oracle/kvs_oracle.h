/*
 * kvs_oracle.h -- declarations of the CPU oracle (test infrastructure only;
 * the product library never includes this header).
 */
#ifndef KVS_ORACLE_H
#define KVS_ORACLE_H
#include <stdint.h>

#define ORACLE_PAGE_ABSENT   (-1)
#define ORACLE_PAGE_RESIDENT 1
#define ORACLE_PAGE_STREAMED 2

double   oracle_half_to_double(uint16_t h);
float    oracle_half_to_float(uint16_t h);
uint16_t oracle_float_to_half(float f);

void oracle_q8_0_block(const uint16_t x_h[32], uint8_t out[34]);
void oracle_q4_0_block(const uint16_t x_h[32], uint8_t out[18]);
void oracle_dequant_q8_0(const uint8_t blk[34], double out[32]);
void oracle_dequant_q4_0(const uint8_t blk[18], double out[32]);
void oracle_q5_0_block(const uint16_t x_h[32], uint8_t out[22]);
void oracle_dequant_q5_0(const uint8_t blk[22], double out[32]);
void oracle_q4_1_block(const uint16_t x_h[32], uint8_t out[20]);
void oracle_dequant_q4_1(const uint8_t blk[20], double out[32]);
void oracle_q5_1_block(const uint16_t x_h[32], uint8_t out[24]);
void oracle_dequant_q5_1(const uint8_t blk[24], double out[32]);
void oracle_quantize_rows(int n_rows, int dim, const uint16_t* k, const uint16_t* v,
                          uint8_t* k_blocks, uint8_t* v_blocks);

int oracle_attention(int n_kv, int n_qh, int dim, const uint8_t* k_blocks,
                     const uint8_t* v_blocks, int n_q, int pos0, const uint16_t* q,
                     double* out, double* lse);

/* the same with the V block type explicit: 1 = F16 (64-byte blocks of the
 * values), 2 = Q4_0 (18), 3 = Q4_1 (20), 6 = Q5_0 (22), 7 = Q5_1 (24),
 * 8 = Q8_0 (34); -1 for any other */
int oracle_quantize_rows_t(int n_rows, int dim, const uint16_t* k, const uint16_t* v,
                           uint8_t* k_blocks, uint8_t* v_blocks, int v_type);
int oracle_attention_t(int n_kv, int n_qh, int dim, const uint8_t* k_blocks,
                       const uint8_t* v_blocks, int n_q, int pos0, const uint16_t* q,
                       double* out, double* lse, int v_type);

/* the same with the K block type explicit as well: 8 = Q8_0 (34-byte blocks)
 * or 1 = F16 (64-byte blocks of the values); -1 for any other */
int oracle_quantize_rows_kv(int n_rows, int dim, const uint16_t* k, const uint16_t* v,
                            uint8_t* k_blocks, uint8_t* v_blocks, int k_type, int v_type);
int oracle_attention_kv(int n_kv, int n_qh, int dim, const uint8_t* k_blocks,
                        const uint8_t* v_blocks, int n_q, int pos0, const uint16_t* q,
                        double* out, double* lse, int k_type, int v_type);

long oracle_pages_for(long n_tokens, int page_tokens);
long oracle_auto_resident_pages(long max_ctx, int page_tokens, long page_bytes, int n_layers);
int  oracle_page_location(long n_tokens, int page_tokens, long n_resident, long page,
                          int* kind, long* index);
#endif
