/*
 * moe_oracle.h -- declarations of the scalar fp64 CPU oracle.
 * TEST INFRASTRUCTURE ONLY (see moe_oracle.c); the product library never
 * includes this header.
 */
#ifndef MOE_ORACLE_H
#define MOE_ORACLE_H
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum { ORC_Q4_SYM_G32 = 1, ORC_Q2_ASYM_G64 = 2 };

double orc_f16_to_f64(uint16_t b);
uint16_t orc_f64_to_f16(double v);
double orc_bf16_to_f64(uint16_t b);
uint16_t orc_f64_to_bf16(double v);

int orc_group_size(int fmt);
long orc_code_bytes(int fmt, int R, int K);
long orc_group_count(int fmt, int R, int K);
int orc_dequant(int fmt, const uint8_t *codes, const uint16_t *scales,
                const uint16_t *mins, int R, int K, double *W);
int orc_quantize(int fmt, const double *W, int R, int K, uint8_t *codes,
                 uint16_t *scales, uint16_t *mins);

void orc_rmsnorm(const uint16_t *x, const float *gamma, double eps, int T, int d,
                 uint16_t *h);
void orc_router(const uint16_t *h, const float *W, const float *bias, int T,
                int d, int E, double *logits);
int orc_topk(const double *logits, int T, int E, int k, int32_t *idx, double *w,
             double *margin);
int orc_bucket(const int32_t *idx, int T, int k, int E, int32_t *cnt,
               int32_t *off, int32_t *perm);
double orc_silu(double z);
void orc_expert(const double *Wg, const double *Wu, const double *Wd, int d,
                int f, const uint16_t *h, int n, double *y);
int orc_dequant_expert(int fmt, int d, int f, const uint8_t *codes,
                       const uint16_t *scales, const uint16_t *mins, double *Wg,
                       double *Wu, double *Wd);

typedef struct {
  int T, d, f, E, k, fmt;
  const uint16_t *x;         /* bf16 [T, d] residual input */
  int use_norm;              /* 1: h = RMSNorm(x); 0: h = x */
  const float *gamma;        /* [d] or NULL (= 1) */
  double eps;
  const float *router_w;     /* fp32 [E, d] */
  const float *router_bias;  /* fp32 [E] or NULL */
  const uint8_t *const *codes_of;    /* [E] pointers, packed expert codes */
  const uint16_t *const *scales_of;  /* [E] pointers, fp16 scales */
  const uint16_t *const *mins_of;    /* [E] pointers (Q2) or NULL */
  const uint8_t *shared_codes;       /* NULL = no shared expert */
  const uint16_t *shared_scales;
  const uint16_t *shared_mins;
} orc_layer_in;

typedef struct {
  uint16_t *h;
  double *logits;
  int32_t *idx;
  double *w;
  double *margin;
  int32_t *cnt;
  int32_t *off;
  int32_t *perm;
  double *delta;
  uint16_t *x_out;
} orc_layer_out;

int orc_moe_layer(const orc_layer_in *in, orc_layer_out *out);

#ifdef __cplusplus
}
#endif
#endif
