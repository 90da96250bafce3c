/*
 * CPU oracle for MoE expert-parallel dispatch / combine.
 *
 * TEST INFRASTRUCTURE ONLY.  The tests, the package's smoke check and the
 * benchmark's CPU-baseline leg are the only code that may load this library.
 * It shares no code, header, table or constant with the CUDA library, and the
 * CUDA library never calls it.
 *
 * Everything is single-threaded plain C on host memory.  bf16 values travel as
 * their 16-bit patterns (uint16_t), e4m3 values as their 8-bit codes.
 * Sizes are int64_t so that T*k*H never overflows.
 *
 * Return codes of this oracle (its own numbering):
 *   EPO_OK 0, EPO_BAD_INDEX 1 (an expert id outside [-1, E); the pair is then
 *   treated like a masked (-1) pair), EPO_INVALID 2 (bad shape).
 */
#ifndef EP_ORACLE_H
#define EP_ORACLE_H

#include <stdint.h>

#define EPO_OK 0
#define EPO_BAD_INDEX 1
#define EPO_INVALID 2
#define EPO_CAPACITY 4  /* padded layout: a pair beyond max_tokens_per_rank (bit, may combine with BAD_INDEX) */

#ifdef __cplusplus
extern "C" {
#endif

/* number formats */
double   epo_e4m3_value(uint8_t code);
uint8_t  epo_e4m3_encode(float v);
uint16_t epo_bf16_from_f32(float f);
float    epo_f32_from_bf16(uint16_t b);

/* element-wise helpers over arrays, for the tests */
void epo_e4m3_encode_array(const float* v, int64_t n, uint8_t* out);
void epo_e4m3_value_array(const uint8_t* c, int64_t n, double* out);
void epo_bf16_from_f32_array(const float* v, int64_t n, uint16_t* out);

int epo_layout(int64_t T, int64_t k, int64_t E, int64_t R, const int64_t* topk_idx,
               int32_t* num_tokens_per_expert, int32_t* expert_offset,
               int32_t* num_tokens_per_rank, int32_t* count_src_rank_expert,
               int32_t* src_rank_expert_offset, uint8_t* is_token_in_rank,
               int32_t* slot_of_pair, int32_t* src_of_slot);

/* Padded ("low-latency") layout: receive rows [E][R][M]; pair (t, j) with
 * expert e from source rank r = t / (T/R) takes row (e*R + r)*M + i, i its
 * position among rank r's pairs to e in (t, j) order.  i >= M: no row,
 * EPO_CAPACITY.  src_of_row has E*R*M entries, -1 where no pair landed.
 * expert_offset[e] = e*R*M, src_rank_expert_offset[r*E+e] = (e*R+r)*M. */
int epo_layout_padded(int64_t T, int64_t k, int64_t E, int64_t R, int64_t M, const int64_t* topk_idx,
                      int32_t* num_tokens_per_expert, int32_t* expert_offset,
                      int32_t* num_tokens_per_rank, int32_t* count_src_rank_expert,
                      int32_t* src_rank_expert_offset, uint8_t* is_token_in_rank,
                      int32_t* slot_of_pair, int32_t* src_of_row);

/* Group-limited top-k routing of scores [T,E] (E experts in n_groups groups of
 * E/n_groups consecutive experts): group score = max of its experts' scores;
 * the topk_groups best groups are kept, then the k best experts inside them.
 * Ties go to the lower index.  topk_idx lists the experts by descending score;
 * topk_weights = softmax of their scores (computed in double). */
int epo_route_group_limited(int64_t T, int64_t E, int64_t k, int64_t n_groups, int64_t topk_groups,
                            const float* scores, int64_t* topk_idx, float* topk_weights);

void epo_dispatch_bf16(int64_t T, int64_t H, int64_t k, const uint16_t* x,
                       const float* topk_weights, const int32_t* slot_of_pair,
                       uint16_t* recv_x, float* recv_weight);

void epo_dispatch_fp8(int64_t T, int64_t H, int64_t k, const uint16_t* x,
                      const float* topk_weights, const int32_t* slot_of_pair,
                      uint8_t* recv_x, float* recv_scale, float* recv_weight);

void epo_combine(int64_t T, int64_t H, int64_t k, const uint16_t* y,
                 const float* topk_weights, const int32_t* slot_of_pair, uint16_t* out);

void epo_combine_backward(int64_t T, int64_t H, int64_t k, const uint16_t* grad_out,
                          const uint16_t* y, const float* topk_weights,
                          const int32_t* slot_of_pair, uint16_t* grad_y, float* grad_w);

void epo_dispatch_backward(int64_t T, int64_t H, int64_t k, const uint16_t* grad_recv,
                           const int32_t* slot_of_pair, uint16_t* grad_x);

#ifdef __cplusplus
}
#endif
#endif
