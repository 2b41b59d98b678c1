/*
 * stq_oracle.h -- declarations of the CPU oracle (test infrastructure only; see stq_oracle.c).
 * This header belongs to the oracle alone: the CUDA library neither includes nor mirrors it.
 */
#ifndef STQ_ORACLE_H
#define STQ_ORACLE_H

#include <stddef.h>
#include <stdint.h>

#define ORC_OK 0
#define ORC_EINVAL 1
#define ORC_ENONFINITE 4

#define ORC_GATE_SCALAR 0
#define ORC_GATE_CHANNEL 1
#define ORC_GATE_CHANNEL_DECAY_FIRST 2

/* storage format of the row and column scales */
#define ORC_SCALE_F32 0
#define ORC_SCALE_BF16 1

int orc_qmax(int bits);
double orc_round_half_even(double y);

size_t orc_codes_bytes(int bits, int dk, int dv);
size_t orc_scale_offset(int bits, int dk, int dv);
size_t orc_block_bytes(int bits, int dk, int dv);
size_t orc_block_bytes_s(int bits, int sfmt, int dk, int dv);

void orc_pack(int bits, size_t n, const int32_t *u, uint8_t *out);
void orc_unpack(int bits, size_t n, const uint8_t *in, int32_t *u);

double orc_half_to_double(uint16_t h);
uint16_t orc_double_to_half(double x);
double orc_bf16_to_double(uint16_t h);
uint16_t orc_double_to_bf16(double x);

int orc_quantize(int bits, int dk, int dv, const double *S, const double *w, uint8_t *block,
                 double *x_out, uint8_t *tie_out, double delta);
int orc_dequantize(int bits, int dk, int dv, const uint8_t *block, double *S);
int orc_quantize_s(int bits, int sfmt, int dk, int dv, const double *S, const double *w,
                   const double *c_given, const double *r_given, uint8_t *block, double *x_out,
                   uint8_t *tie_out, uint8_t *stie_out, double delta);
int orc_dequantize_s(int bits, int sfmt, int dk, int dv, const uint8_t *block, double *S);
int orc_quantize_fit(int bits, int sfmt, int rounds, int dk, int dv, const double *S, const double *w,
                     uint8_t *block, double *x_out, uint8_t *tie_out, uint8_t *stie_out, double delta);

void orc_update(int dk, int dv, int gate, double *S, const double *q, const double *k,
                const double *v, double beta, const double *alpha, double *o);
int orc_decode_step(int bits, int dk, int dv, int gate, uint8_t *block, const double *q,
                    const double *k, const double *v, double beta, const double *alpha,
                    const double *w, float *o, double *S_new_out, double *x_out,
                    uint8_t *tie_out, double delta);
int orc_decode_step_s(int bits, int sfmt, int rounds, int dk, int dv, int gate, uint8_t *block, const double *q,
                      const double *k, const double *v, double beta, const double *alpha,
                      const double *w, float *o, double *S_new_out, double *x_out,
                      uint8_t *tie_out, uint8_t *stie_out, double delta);
int orc_prefill_seq(int bits, int dk, int dv, int gate, uint8_t *block, int T, int chunk,
                    const double *q, const double *k, const double *v, const double *beta,
                    const double *alpha, const double *w, float *o, double *x_out,
                    uint8_t *tie_out, double delta);
int orc_prefill_seq_s(int bits, int sfmt, int rounds, int dk, int dv, int gate, uint8_t *block, int T, int chunk,
                      const double *q, const double *k, const double *v, const double *beta,
                      const double *alpha, const double *w, float *o, double *x_out,
                      uint8_t *tie_out, uint8_t *stie_out, double delta);
int orc_chunk_wy(int dk, int dv, int C, const double *S0, const double *q, const double *k,
                 const double *v, const double *beta, const double *alpha, double *S_end,
                 double *O);

size_t orc_uniform_block_bytes(int bits, int dk, int dv);
int orc_quantize_uniform(int bits, int dk, int dv, const double *S, uint8_t *block, double *x_out,
                         uint8_t *tie_out, double delta);
int orc_dequantize_uniform(int bits, int dk, int dv, const uint8_t *block, double *S);
int orc_decode_step_uniform(int bits, int dk, int dv, int gate, uint8_t *block, const double *q,
                            const double *k, const double *v, double beta, const double *alpha,
                            float *o, double *x_out, uint8_t *tie_out, double delta);

#endif
