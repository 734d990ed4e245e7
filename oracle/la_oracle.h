/*
 * la_oracle.h -- declarations of the CPU oracle (test infrastructure only; see
 * la_oracle.c for what each function computes and which passage it follows).
 * Independent of the CUDA library: it has its own constants and includes nothing of it.
 */
#ifndef LA_ORACLE_H
#define LA_ORACLE_H

#include <stddef.h>

#define LAO_RULE_LINEAR 0
#define LAO_RULE_GATED 1
#define LAO_RULE_DELTA 2
#define LAO_RULE_GATED_DELTA 3
#define LAO_RULE_KDA 4

#define LAO_F64 0
#define LAO_F32 1
#define LAO_BF16 2
#define LAO_Q8 3

#ifdef __cplusplus
extern "C" {
#endif

double lao_round_bf16(double x);
double lao_round_to(double x, int dtype);

int lao_step(int rule, int n_qk_heads, int n_v_heads, int dk, int dv,
             const double *src_pool, int src_slots,
             double *dst_pool, int dst_slots, int dst_dtype,
             const int *read_slot, const int *write_slot, int B,
             const double *q, const double *k, const double *v, int io_dtype,
             const double *g, const double *beta, double scale, double *o);

void lao_readout_rearranged(int rule, int n_qk_heads, int n_v_heads, int dk, int dv,
                            const double *src_pool, int B,
                            const double *q, const double *k, const double *v,
                            const double *g, const double *beta, double scale, double *o);

int lao_scan(int rule, int n_qk_heads, int n_v_heads, int dk, int dv,
             const double *src_pool, int src_slots, const int *read_slot,
             double *dst_pool, int dst_slots, int dst_dtype, const int *write_slot,
             int n_seqs, const int *cu_seqlens, int total_tokens,
             const double *q, const double *k, const double *v, int io_dtype,
             const double *g, const double *beta, double scale, double *o);

int lao_scan_ckpt(int rule, int n_qk_heads, int n_v_heads, int dk, int dv,
                  const double *src_pool, int src_slots, const int *read_slot,
                  double *dst_pool, int dst_slots, int dst_dtype, const int *write_slot,
                  int n_seqs, const int *cu_seqlens, int total_tokens,
                  const double *q, const double *k, const double *v, int io_dtype,
                  const double *g, const double *beta, double scale, double *o,
                  int ckpt_every, const int *ckpt_cu, const int *ckpt_slots);

int lao_step_qgroups(int rule, int n_q_heads, int n_v_heads, int dk, int dv,
                     const double *src_pool, int src_slots,
                     double *dst_pool, int dst_slots, int dst_dtype,
                     const int *read_slot, const int *write_slot, int B,
                     const double *q, const double *k, const double *v, int io_dtype,
                     const double *g, const double *beta, double scale, double *o);

int lao_scan_qgroups(int rule, int n_q_heads, int n_v_heads, int dk, int dv,
                     const double *src_pool, int src_slots, const int *read_slot,
                     double *dst_pool, int dst_slots, int dst_dtype, const int *write_slot,
                     int n_seqs, const int *cu_seqlens, int total_tokens,
                     const double *q, const double *k, const double *v, int io_dtype,
                     const double *g, const double *beta, double scale, double *o);

size_t lao_q8_tile_bytes(int dk, int dv, int n_hp);
int lao_q8_encode(const float *x, int n, int H, int dk, int dv, int n_hp, const unsigned *masks,
                  unsigned char *out);
int lao_q8_decode(const unsigned char *in, int n, int H, int dk, int dv, int n_hp, const unsigned *masks, float *x);
int lao_step_q8(int rule, int n_qk_heads, int n_v_heads, int dk, int dv,
                const double *src_pool, int src_slots, double *dst_pool, int dst_slots,
                const int *read_slot, const int *write_slot, int B,
                const double *q, const double *k, const double *v, int io_dtype,
                const double *g, const double *beta, double scale, double *o, const unsigned *q8_masks);
int lao_scan_q8(int rule, int n_qk_heads, int n_v_heads, int dk, int dv,
                const double *src_pool, int src_slots, const int *read_slot,
                double *dst_pool, int dst_slots, const int *write_slot,
                int n_seqs, const int *cu_seqlens, int total_tokens,
                const double *q, const double *k, const double *v, int io_dtype,
                const double *g, const double *beta, double scale, double *o,
                int ckpt_every, const int *ckpt_cu, const int *ckpt_slots, const unsigned *q8_masks);

void lao_conv(int n_qk_heads, int n_v_heads, int dk, int dv, int W, int act, int l2norm, int B,
              const double *xq, const double *xk, const double *xv, const double *wq, const double *wk,
              const double *wv, const double *hist, double *hist_out, double *q, double *k, double *v);
int lao_step_conv(int rule, int n_qk_heads, int n_v_heads, int dk, int dv,
                  const double *src_pool, int src_slots, double *dst_pool, int dst_slots, int dst_dtype,
                  const int *read_slot, const int *write_slot, int B,
                  const double *xq, const double *xk, const double *xv, int io_dtype,
                  const double *g, const double *beta, double scale, double *o,
                  int W, int act, int l2norm, const double *wq, const double *wk, const double *wv,
                  const double *conv_src, double *conv_dst);

int lao_scan_conv(int rule, int n_qk_heads, int n_v_heads, int dk, int dv,
                  const double *src_pool, int src_slots, const int *read_slot,
                  double *dst_pool, int dst_slots, int dst_dtype, const int *write_slot,
                  int n_seqs, const int *cu_seqlens, int total_tokens,
                  const double *xq, const double *xk, const double *xv, int io_dtype,
                  const double *g, const double *beta, double scale, double *o,
                  int W, int act, int l2norm, const double *wq, const double *wk, const double *wv,
                  const double *conv_src, double *conv_dst);

int lao_pool_copy(unsigned char *pool, size_t slot_bytes, int n_slots, int n,
                  const int *src_slots, const int *dst_slots);
int lao_pool_gather(const unsigned char *pool, size_t slot_bytes, int n_slots, int n,
                    const int *slots, unsigned char *dense);
int lao_pool_scatter(unsigned char *pool, size_t slot_bytes, int n_slots, int n,
                     const int *slots, const unsigned char *dense);
int lao_pool_zero(unsigned char *pool, size_t slot_bytes, int n_slots, int n, const int *slots);

int lao_num_threads(void);
void lao_set_threads(int n);

#ifdef __cplusplus
}
#endif

#endif
