/*
 * moe_oracle.c -- plain, slow, scalar CPU oracle for the sparse MoE expert
 * layer.  TEST INFRASTRUCTURE ONLY: nothing in the product library links,
 * includes or calls this file; only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg load it.  It shares no code, header, table or
 * helper with the CUDA path.
 *
 * Every floating-point step is done in IEEE double (fp64).  The code follows
 * the plain definitions, in the order the method states them:
 *
 *   Strata engine analysis article, "93 token/s on one 8 GB card"
 *   (m.lqnn.cn/news/264700), section "Architecture overview": per layer the
 *   router picks the 10 experts of 512 that a token activates, the chosen
 *   experts are computed, and their outputs are combined and written back
 *   into the residual.
 *
 *   Same article, section "Doorbell handshake": each block is split at the
 *   router; "pre" ends with the router (expert ids + routing weights),
 *   "post" combines the expert outputs and writes the residual back.
 *
 *   Same article, section "Expert cache": the residency table answers
 *   (layer, expert) -> slot or -1 and does no computing; cached and
 *   uncached experts compute the same function, so the oracle has no notion
 *   of residency at all.
 *
 *   lcz.me topic 2059 (X99 + RX 7900 XTX report), section 2 "Model and
 *   principles": 48 layers, 512 experts, 10 routed + 1 shared per token.
 *
 * The pages print no router formula, no softmax and no quantised bit layout;
 * the readings this file implements are:
 *   - router logits  l[t,e] = sum_i W[e,i] * h[t,i] (+ bias[e]);
 *   - top-k: the k largest logits, ties broken towards the lower expert id;
 *   - weights: softmax over the k selected logits (renormalised);
 *   - expert: y = Wd * ( SiLU(Wg*h) (.) (Wu*h) ),  SiLU(z) = z / (1+e^-z);
 *   - shared expert: same SwiGLU, weight 1, added for every token;
 *   - combine: delta[t] = sum_{j=0..k-1} w[t,j]*y[t,j] + y_shared[t],
 *              x[t] <- bf16_rne( x[t] + delta[t] );
 *   - RMSNorm (stack only): h = bf16_rne( x * (mean(x^2)+eps)^-1/2 * gamma ).
 *   - Q4 (4-bit symmetric, group 32 along K, fp16 scale):
 *        stored nibble c in [0,15], value = s * (c - 8); two nibbles per
 *        byte, lower k in the low nibble; scales fp16 [rows, K/32].
 *   - Q2 (2-bit asymmetric, group 64 along K, fp16 scale + fp16 min):
 *        stored code q in [0,3], value = s * q + m; four codes per byte,
 *        element k in bits 2*(k%4); scales and mins fp16 [rows, K/64].
 *   - expert matrices: Wg, Wu are [f, d], Wd is [d, f], row-major, groups
 *     contiguous along the reduction dimension.  One expert = the codes of
 *     Wg, then Wu, then Wd (same order for scales and mins).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#include "moe_oracle.h"

/* ------------------------------------------------------------------ */
/* 16-bit float encodings, written out from their IEEE / bfloat16      */
/* definitions.                                                        */
/* ------------------------------------------------------------------ */

double orc_f16_to_f64(uint16_t b) {
  int sign = (b >> 15) & 1;
  int ex = (b >> 10) & 0x1f;
  int man = b & 0x3ff;
  double v;
  if (ex == 0)
    v = ldexp((double)man, -24); /* subnormal: man * 2^-24 */
  else if (ex == 31)
    v = man ? NAN : INFINITY;
  else
    v = ldexp((double)(1024 + man), ex - 25); /* (1 + man/1024) * 2^(ex-15) */
  return sign ? -v : v;
}

/* round-to-nearest-even of a double into IEEE binary16, returned as bits */
uint16_t orc_f64_to_f16(double v) {
  uint16_t sign = 0;
  if (isnan(v)) return 0x7e00;
  if (signbit(v)) { sign = 0x8000; v = -v; }
  if (v == 0.0) return sign;
  if (v >= 65520.0) return sign | 0x7c00; /* rounds to infinity */
  int e;
  frexp(v, &e);         /* v = m * 2^e, m in [0.5,1) -> v = 1.x * 2^(e-1) */
  int E = e - 1;
  if (E < -14) E = -14; /* subnormal range shares the quantum 2^-24 */
  double q = ldexp(1.0, E - 10);
  double n = rint(v / q); /* exact scaling, then RNE to an integer */
  double r = n * q;       /* representable value */
  if (r < ldexp(1.0, -14)) return sign | (uint16_t)(r / ldexp(1.0, -24));
  frexp(r, &e);
  E = e - 1;
  uint16_t man = (uint16_t)(r / ldexp(1.0, E - 10) - 1024.0);
  return sign | (uint16_t)((E + 15) << 10) | man;
}

double orc_bf16_to_f64(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, 4);
  return (double)f;
}

/* round-to-nearest-even of a double into bfloat16 (8 exponent bits, 7
 * stored mantissa bits), returned as bits; done directly from the double so
 * there is no intermediate rounding to float. */
uint16_t orc_f64_to_bf16(double v) {
  uint16_t sign = 0;
  if (isnan(v)) return 0x7fc0;
  if (signbit(v)) { sign = 0x8000; v = -v; }
  if (v == 0.0) return sign;
  /* largest finite bf16 is (2 - 2^-7) * 2^127; halfway to 2^128 rounds up */
  if (v >= ldexp(2.0 - ldexp(1.0, -8), 127)) return sign | 0x7f80;
  int e;
  frexp(v, &e);
  int E = e - 1;
  if (E < -126) E = -126;
  double q = ldexp(1.0, E - 7);
  double r = rint(v / q) * q;
  if (r < ldexp(1.0, -126)) return sign | (uint16_t)(r / ldexp(1.0, -133));
  frexp(r, &e);
  E = e - 1;
  uint16_t man = (uint16_t)(r / ldexp(1.0, E - 7) - 128.0);
  return sign | (uint16_t)((E + 127) << 7) | man;
}

/* ------------------------------------------------------------------ */
/* Quantised formats                                                    */
/* ------------------------------------------------------------------ */

int orc_group_size(int fmt) {
  return fmt == ORC_Q4_SYM_G32 ? 32 : fmt == ORC_Q2_ASYM_G64 ? 64 : 0;
}

/* packed bytes of one [R, K] matrix */
long orc_code_bytes(int fmt, int R, int K) {
  return fmt == ORC_Q4_SYM_G32 ? (long)R * K / 2 : (long)R * K / 4;
}

long orc_group_count(int fmt, int R, int K) {
  return (long)R * (K / orc_group_size(fmt));
}

/* Dequantise one [R, K] matrix into doubles. */
int orc_dequant(int fmt, const uint8_t *codes, const uint16_t *scales,
                const uint16_t *mins, int R, int K, double *W) {
  int G = orc_group_size(fmt);
  if (!G || K % G) return -1;
  int ng = K / G;
  for (int r = 0; r < R; ++r) {
    for (int k = 0; k < K; ++k) {
      double s = orc_f16_to_f64(scales[(long)r * ng + k / G]);
      if (fmt == ORC_Q4_SYM_G32) {
        uint8_t byte = codes[(long)r * (K / 2) + k / 2];
        int c = (k % 2 == 0) ? (byte & 0xf) : (byte >> 4);
        W[(long)r * K + k] = s * (double)(c - 8);
      } else {
        if (!mins) return -1;
        uint8_t byte = codes[(long)r * (K / 4) + k / 4];
        int q = (byte >> (2 * (k % 4))) & 3;
        double m = orc_f16_to_f64(mins[(long)r * ng + k / G]);
        W[(long)r * K + k] = s * (double)q + m;
      }
    }
  }
  return 0;
}

/* Quantise one [R, K] matrix (the encoder of each format).
 * Q4: s = fp16(max|w| / 7); q = clamp(rne(w / s), -8, 7); nibble = q + 8.
 * Q2: m = fp16(min w); s = fp16((max w - m) / 3);
 *     q = clamp(rne((w - m) / s), 0, 3).
 * A zero scale encodes the whole group as q = 0 (Q4 nibble 8). */
int orc_quantize(int fmt, const double *W, int R, int K, uint8_t *codes,
                 uint16_t *scales, uint16_t *mins) {
  int G = orc_group_size(fmt);
  if (!G || K % G) return -1;
  int ng = K / G;
  memset(codes, 0, (size_t)orc_code_bytes(fmt, R, K));
  for (int r = 0; r < R; ++r) {
    for (int g = 0; g < ng; ++g) {
      const double *w = W + (long)r * K + (long)g * G;
      if (fmt == ORC_Q4_SYM_G32) {
        double amax = 0.0;
        for (int i = 0; i < G; ++i)
          if (fabs(w[i]) > amax) amax = fabs(w[i]);
        uint16_t sb = orc_f64_to_f16(amax / 7.0);
        double s = orc_f16_to_f64(sb);
        scales[(long)r * ng + g] = sb;
        for (int i = 0; i < G; ++i) {
          int q = 0;
          if (s != 0.0) {
            double t = rint(w[i] / s);
            q = t < -8.0 ? -8 : t > 7.0 ? 7 : (int)t;
          }
          int k = g * G + i;
          uint8_t c = (uint8_t)(q + 8);
          codes[(long)r * (K / 2) + k / 2] |= (k % 2 == 0) ? c : (uint8_t)(c << 4);
        }
      } else {
        if (!mins) return -1;
        double mn = w[0], mx = w[0];
        for (int i = 1; i < G; ++i) {
          if (w[i] < mn) mn = w[i];
          if (w[i] > mx) mx = w[i];
        }
        uint16_t mb = orc_f64_to_f16(mn);
        double m = orc_f16_to_f64(mb);
        uint16_t sb = orc_f64_to_f16((mx - m) / 3.0);
        double s = orc_f16_to_f64(sb);
        mins[(long)r * ng + g] = mb;
        scales[(long)r * ng + g] = sb;
        for (int i = 0; i < G; ++i) {
          int q = 0;
          if (s != 0.0) {
            double t = rint((w[i] - m) / s);
            q = t < 0.0 ? 0 : t > 3.0 ? 3 : (int)t;
          }
          int k = g * G + i;
          codes[(long)r * (K / 4) + k / 4] |= (uint8_t)(q << (2 * (k % 4)));
        }
      }
    }
  }
  return 0;
}

/* ------------------------------------------------------------------ */
/* Layer steps                                                          */
/* ------------------------------------------------------------------ */

/* RMSNorm: h = bf16( x * (mean(x^2) + eps)^-1/2 * gamma ), fp64 inside. */
void orc_rmsnorm(const uint16_t *x, const float *gamma, double eps, int T, int d,
                 uint16_t *h) {
  for (int t = 0; t < T; ++t) {
    double ss = 0.0;
    for (int i = 0; i < d; ++i) {
      double v = orc_bf16_to_f64(x[(long)t * d + i]);
      ss += v * v;
    }
    double inv = 1.0 / sqrt(ss / (double)d + eps);
    for (int i = 0; i < d; ++i) {
      double v = orc_bf16_to_f64(x[(long)t * d + i]) * inv;
      if (gamma) v *= (double)gamma[i];
      h[(long)t * d + i] = orc_f64_to_bf16(v);
    }
  }
}

/* Router logits: l[t,e] = sum_i W[e,i] h[t,i] + bias[e]. */
void orc_router(const uint16_t *h, const float *W, const float *bias, int T,
                int d, int E, double *logits) {
  for (int t = 0; t < T; ++t)
    for (int e = 0; e < E; ++e) {
      double acc = 0.0;
      for (int i = 0; i < d; ++i)
        acc += (double)W[(long)e * d + i] * orc_bf16_to_f64(h[(long)t * d + i]);
      if (bias) acc += (double)bias[e];
      logits[(long)t * E + e] = acc;
    }
}

/* Top-k by repeated selection of the largest remaining logit; a later
 * candidate replaces the current best only when strictly larger, so equal
 * logits go to the lower expert id.  Weights: softmax over the k selected.
 * margin[t] = (k-th largest) - ((k+1)-th largest), +inf when k == E. */
int orc_topk(const double *logits, int T, int E, int k, int32_t *idx, double *w,
             double *margin) {
  if (k < 1 || k > E) return -1;
  unsigned char *taken = (unsigned char *)malloc((size_t)E);
  if (!taken) return -2;
  for (int t = 0; t < T; ++t) {
    const double *l = logits + (long)t * E;
    memset(taken, 0, (size_t)E);
    for (int j = 0; j < k; ++j) {
      int best = -1;
      for (int e = 0; e < E; ++e)
        if (!taken[e] && (best < 0 || l[e] > l[best])) best = e;
      taken[best] = 1;
      idx[(long)t * k + j] = best;
    }
    if (margin) {
      if (k == E) {
        margin[t] = INFINITY;
      } else {
        int nxt = -1;
        for (int e = 0; e < E; ++e)
          if (!taken[e] && (nxt < 0 || l[e] > l[nxt])) nxt = e;
        margin[t] = l[idx[(long)t * k + k - 1]] - l[nxt];
      }
    }
    double lmax = l[idx[(long)t * k]];
    double den = 0.0;
    for (int j = 0; j < k; ++j) den += exp(l[idx[(long)t * k + j]] - lmax);
    for (int j = 0; j < k; ++j)
      w[(long)t * k + j] = exp(l[idx[(long)t * k + j]] - lmax) / den;
  }
  free(taken);
  return 0;
}

/* Bucketing by expert (a counting sort): cnt[e] = number of (t,j) routed to
 * e; off = exclusive prefix sum of cnt (E+1 entries); perm lists the pair
 * ids p = t*k + j grouped by expert, ascending t inside each expert. */
int orc_bucket(const int32_t *idx, int T, int k, int E, int32_t *cnt,
               int32_t *off, int32_t *perm) {
  for (int e = 0; e < E; ++e) cnt[e] = 0;
  for (long p = 0; p < (long)T * k; ++p) {
    int e = idx[p];
    if (e < 0 || e >= E) return -1;
    cnt[e]++;
  }
  off[0] = 0;
  for (int e = 0; e < E; ++e) off[e + 1] = off[e] + cnt[e];
  int32_t *fill = (int32_t *)calloc((size_t)E, sizeof(int32_t));
  if (!fill) return -2;
  for (int t = 0; t < T; ++t)
    for (int j = 0; j < k; ++j) {
      int e = idx[(long)t * k + j];
      perm[off[e] + fill[e]++] = t * k + j;
    }
  free(fill);
  return 0;
}

double orc_silu(double z) { return z / (1.0 + exp(-z)); }

/* One SwiGLU expert on n token rows: y = Wd (SiLU(Wg h) .* (Wu h)).
 * Wg, Wu: [f, d]; Wd: [d, f]; h: bf16 [n, d]; y: [n, d]. */
void orc_expert(const double *Wg, const double *Wu, const double *Wd, int d,
                int f, const uint16_t *h, int n, double *y) {
  double *a = (double *)malloc((size_t)f * sizeof(double));
  double *hv = (double *)malloc((size_t)d * sizeof(double));
  for (int t = 0; t < n; ++t) {
    for (int i = 0; i < d; ++i) hv[i] = orc_bf16_to_f64(h[(long)t * d + i]);
    for (int r = 0; r < f; ++r) {
      double g = 0.0, u = 0.0;
      for (int i = 0; i < d; ++i) {
        g += Wg[(long)r * d + i] * hv[i];
        u += Wu[(long)r * d + i] * hv[i];
      }
      a[r] = orc_silu(g) * u;
    }
    for (int o = 0; o < d; ++o) {
      double acc = 0.0;
      for (int r = 0; r < f; ++r) acc += Wd[(long)o * f + r] * a[r];
      y[(long)t * d + o] = acc;
    }
  }
  free(a);
  free(hv);
}

/* Dequantise a packed expert (Wg, Wu, Wd back to back) into three buffers. */
int orc_dequant_expert(int fmt, int d, int f, const uint8_t *codes,
                       const uint16_t *scales, const uint16_t *mins, double *Wg,
                       double *Wu, double *Wd) {
  long cb = orc_code_bytes(fmt, f, d); /* same for [f,d] and [d,f] */
  long ng = orc_group_count(fmt, f, d);
  int rc = 0;
  rc |= orc_dequant(fmt, codes, scales, mins, f, d, Wg);
  rc |= orc_dequant(fmt, codes + cb, scales + ng, mins ? mins + ng : NULL, f, d, Wu);
  rc |= orc_dequant(fmt, codes + 2 * cb, scales + 2 * ng, mins ? mins + 2 * ng : NULL,
                    d, f, Wd);
  return rc;
}

/* One MoE layer on T token rows, in the order of the method:
 *   [RMSNorm] -> router -> top-k + softmax -> bucketing -> experts
 *   (+ shared) -> combine + residual.
 * Expert e's packed bytes are codes_of[e] / scales_of[e] / mins_of[e]; only
 * the experts that some token selects are touched (NULL elsewhere is fine).
 * Outputs (any may be NULL except x_out): h [T,d] bf16, logits [T,E],
 * idx [T,k], w [T,k], margin [T], cnt [E], off [E+1], perm [T*k],
 * delta [T,d] (the fp64 MoE output before the residual add),
 * x_out [T,d] bf16. */
int orc_moe_layer(const orc_layer_in *in, orc_layer_out *out) {
  const int T = in->T, d = in->d, f = in->f, E = in->E, k = in->k, fmt = in->fmt;
  if (T < 0 || d <= 0 || f <= 0 || E <= 0 || k < 1 || k > E) return -1;
  int G = orc_group_size(fmt);
  if (!G || d % G || f % G) return -1;
  long wsz = (long)f * d;
  int rc = 0;

  uint16_t *h = (uint16_t *)malloc((size_t)T * d * 2 + 2);
  double *logits = (double *)malloc((size_t)T * E * sizeof(double) + 8);
  int32_t *idx = (int32_t *)malloc((size_t)T * k * 4 + 4);
  double *w = (double *)malloc((size_t)T * k * sizeof(double) + 8);
  double *margin = (double *)malloc((size_t)T * sizeof(double) + 8);
  int32_t *cnt = (int32_t *)malloc((size_t)E * 4);
  int32_t *off = (int32_t *)malloc((size_t)(E + 1) * 4);
  int32_t *perm = (int32_t *)malloc((size_t)T * k * 4 + 4);
  double *ypair = (double *)calloc((size_t)T * k * d + 1, sizeof(double));
  double *yshared = (double *)calloc((size_t)T * d + 1, sizeof(double));
  double *Wg = (double *)malloc((size_t)wsz * sizeof(double));
  double *Wu = (double *)malloc((size_t)wsz * sizeof(double));
  double *Wd = (double *)malloc((size_t)wsz * sizeof(double));
  if (!h || !logits || !idx || !w || !margin || !cnt || !off || !perm || !ypair ||
      !yshared || !Wg || !Wu || !Wd) {
    rc = -2;
    goto done;
  }

  /* RMSNorm (only when a norm is configured), else h = x */
  if (in->use_norm)
    orc_rmsnorm(in->x, in->gamma, in->eps, T, d, h);
  else
    memcpy(h, in->x, (size_t)T * d * 2);

  /* router, top-k, softmax */
  orc_router(h, in->router_w, in->router_bias, T, d, E, logits);
  if (orc_topk(logits, T, E, k, idx, w, margin)) { rc = -3; goto done; }

  /* bucketing */
  if (orc_bucket(idx, T, k, E, cnt, off, perm)) { rc = -4; goto done; }

  /* routed experts: each selected expert is dequantised once and applied to
   * every token in its bucket */
  for (int e = 0; e < E; ++e) {
    if (cnt[e] == 0) continue;
    if (!in->codes_of[e] || !in->scales_of[e] ||
        (fmt == ORC_Q2_ASYM_G64 && !in->mins_of[e])) {
      rc = -5;
      goto done;
    }
    if (orc_dequant_expert(fmt, d, f, in->codes_of[e], in->scales_of[e],
                           in->mins_of ? in->mins_of[e] : NULL, Wg, Wu, Wd)) {
      rc = -6;
      goto done;
    }
    for (int p = off[e]; p < off[e + 1]; ++p) {
      int pair = perm[p];
      int t = pair / k;
      orc_expert(Wg, Wu, Wd, d, f, h + (long)t * d, 1, ypair + (long)pair * d);
    }
  }

  /* shared expert: every token, weight 1 */
  if (in->shared_codes) {
    if (orc_dequant_expert(fmt, d, f, in->shared_codes, in->shared_scales,
                           in->shared_mins, Wg, Wu, Wd)) {
      rc = -7;
      goto done;
    }
    orc_expert(Wg, Wu, Wd, d, f, h, T, yshared);
  }

  /* combine in j order, then the shared expert, then the residual add */
  for (int t = 0; t < T; ++t) {
    for (int o = 0; o < d; ++o) {
      double acc = 0.0;
      for (int j = 0; j < k; ++j)
        acc += w[(long)t * k + j] * ypair[((long)t * k + j) * d + o];
      acc += yshared[(long)t * d + o];
      if (out->delta) out->delta[(long)t * d + o] = acc;
      double xv = orc_bf16_to_f64(in->x[(long)t * d + o]);
      if (out->x_out) out->x_out[(long)t * d + o] = orc_f64_to_bf16(xv + acc);
    }
  }

  if (out->h) memcpy(out->h, h, (size_t)T * d * 2);
  if (out->logits) memcpy(out->logits, logits, (size_t)T * E * sizeof(double));
  if (out->idx) memcpy(out->idx, idx, (size_t)T * k * 4);
  if (out->w) memcpy(out->w, w, (size_t)T * k * sizeof(double));
  if (out->margin) memcpy(out->margin, margin, (size_t)T * sizeof(double));
  if (out->cnt) memcpy(out->cnt, cnt, (size_t)E * 4);
  if (out->off) memcpy(out->off, off, (size_t)(E + 1) * 4);
  if (out->perm) memcpy(out->perm, perm, (size_t)T * k * 4);

done:
  free(h); free(logits); free(idx); free(w); free(margin); free(cnt); free(off);
  free(perm); free(ypair); free(yshared); free(Wg); free(Wu); free(Wd);
  return rc;
}
