/*
 * moe_oracle.h -- declarations of the CPU oracle (moe_oracle.c).
 * TEST INFRASTRUCTURE ONLY: private to oracle/, never included by the CUDA
 * library.  Each function's definition cites the passage it restates.
 */
#ifndef MOE_ORACLE_H
#define MOE_ORACLE_H
#include <stddef.h>
#include <stdint.h>

double orc_f16_to_f64(uint16_t h);
float orc_bf16_to_f32(uint16_t b);
double orc_gelu_tanh(double v);

size_t orc_blob_bytes(int D, int F);
double orc_weight(const uint8_t *blob, int D, int F, int m, int n, int k);
void orc_dequant(const uint8_t *blob, int D, int F, int m, double *W);
void orc_expert_ffn(const uint8_t *blob, int D, int F, const double *x, double *y);

void orc_router_logits(const uint16_t *x_bf16, const int8_t *wq, const uint16_t *ws_f16,
                       const float *bias, int E, int D, int G, float *logits);
int orc_topk(const float *logits, int E, int K, int32_t *ids);
void orc_gate_weights(const float *logits, const int32_t *ids, int K, double *w);

int orc_moe_token(int D, int E, int K, int F, int FS, int G,
                  const uint16_t *x_bf16,
                  const int8_t *wq, const uint16_t *ws_f16, const float *bias,
                  const uint8_t *shared_blob, const uint8_t *const *expert_blobs,
                  int32_t *ids, double *gate_w, float *logits, double *y);

#define ORC_POLICY_LFU 0
#define ORC_POLICY_LRU 1
#define ORC_POLICY_LFU_DECAY 2
#define ORC_POLICY_LFU_IN_CACHE 3

int orc_cache_plan(int E, int S, int policy, uint32_t decay_period,
                   uint32_t *count, uint32_t *last_use,
                   int32_t *slot_of, int32_t *expert_in,
                   const int32_t *ids, int T, int K, uint32_t step,
                   int32_t *pair_slot, int32_t *u_expert, int32_t *u_slot,
                   int32_t *u_hit, int32_t *u_victim, int32_t *u_wave, int *n_u);

int orc_lfu_plan(int E, int S, uint32_t *count, uint32_t *last_use,
                 int32_t *slot_of, int32_t *expert_in,
                 const int32_t *ids, int T, int K, uint32_t step,
                 int32_t *pair_slot, int32_t *u_expert, int32_t *u_slot,
                 int32_t *u_hit, int32_t *u_victim, int32_t *u_wave, int *n_u);

uint16_t orc_f64_to_bf16(double v);
void orc_residual_rmsnorm(const double *r_in, const double *y, int D, double *r_out, uint16_t *x_next);

int orc_group_by_expert(const int32_t *ids, int T, int K, int E,
                        int32_t *offsets, int32_t *pairs);

int orc_attn_decode(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                    int Hq, int Hkv, int hd, int cap, int n, double scale, double *o);
#endif
