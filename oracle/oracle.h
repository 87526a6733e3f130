/*
 * Oracle declarations.  TEST INFRASTRUCTURE ONLY: used by the test-suite, the
 * package smoke check and the CPU-baseline leg of the benchmark; never by the
 * CUDA library.  See oracle.c for what each function computes and which
 * passage of the pages it follows.
 */
#ifndef MOE_ORACLE_H
#define MOE_ORACLE_H
#include <stdint.h>

float orc_bf16_to_f32(uint16_t h);
uint16_t orc_f32_to_bf16(float f);
float orc_exp_portable(float x);
void orc_exp_portable_range(const float* x, int64_t n, float* out);
void orc_exp_portable_neg_bits(uint32_t start, int64_t n, float* out);
void orc_route(const float* logits, int32_t T, int32_t E, int32_t k, float L, const int32_t* slot_table,
               int32_t* ids, double* w, float* u_out);
void orc_sort(const int32_t* ids, int32_t T, int32_t k, int32_t E, int32_t* offsets, int32_t* pairs,
              int32_t* active, int32_t* n_active);
void orc_slot_lookup(const int32_t* table, const int32_t* active, int32_t n_active, int32_t pass_begin,
                     int32_t pass_len, int32_t n_slots, int32_t* slots, int32_t* miss, int32_t* n_miss,
                     int32_t* bad);
int orc_bits_supported(int32_t b);
int64_t orc_row_bytes(int32_t K, int32_t b);
int64_t orc_row_groups(int32_t K, int32_t g);
void orc_slot_layout(int32_t H, int32_t I, int32_t g, int32_t b_gu, int32_t b_d, int64_t* off);
int32_t orc_get_code(const uint8_t* proj, int32_t K, int32_t g, int32_t row, int32_t k, int32_t b);
void orc_set_code(uint8_t* proj, int32_t K, int32_t g, int32_t row, int32_t k, int32_t b, int32_t q);
int64_t orc_tile_bytes(int32_t K, int32_t g, int32_t b);
int32_t orc_gate_up_row(int32_t R, int32_t I);
int64_t orc_sb_offset(int32_t row, int64_t gi, int32_t K, int32_t g, int32_t b);
void orc_quantize_rows(const float* w, int32_t rows, int32_t K, int32_t g, int32_t b, uint8_t* proj);
void orc_dequant_rows(const uint8_t* proj, int32_t rows, int32_t K, int32_t g, int32_t b, float* out);
void orc_dequant_slot(const uint8_t* slot, int32_t H, int32_t I, int32_t g, int32_t b_gu, int32_t b_d,
                      float* gate_up, float* down);
void orc_expert_ffn(const uint16_t* x, int32_t H, int32_t I, int32_t g, int32_t b_gu, int32_t b_d,
                    int32_t k, const uint8_t* const* expert_slot, const int32_t* ids, const double* w,
                    const int32_t* tok, int32_t n_tok, double* y);
int32_t orc_lru_step(int32_t E, int32_t n_slots, int32_t slot_base, int32_t* table, int32_t* owner,
                     int64_t* stamp, int64_t* clock, const int32_t* pass_experts, int32_t n_pass,
                     int32_t* assigned, int32_t* n_assigned);
#endif
