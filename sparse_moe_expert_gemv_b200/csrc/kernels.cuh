// kernels.cuh -- the decode-path kernels of libmoe (sm_100a).
//
// Per layer and window of T tokens (Strata engine analysis article
// "93 token/s on one 8 GB card", section "Architecture overview": router ->
// selected experts -> combine into the residual):
//   rmsnorm_kernel      (optional)  h = RMSNorm(x)
//   router_logits_kernel            logits[t,e] = W[e,:] . h[t,:] + b[e]
//   route_finish_kernel             top-k + softmax, bucketing by expert,
//                                   residency lookup, expert work list
//   expert_gemv_kernel<GATED=1>     a = SiLU(Wg h) * (Wu h)   per (expert, token)
//   expert_gemv_kernel<GATED=0>     y = Wd a                   per (expert, token)
//   combine_kernel                  x += sum_j w_j y_j + y_shared
// Consecutive kernels overlap through programmatic dependent launch: each
// kernel waits (griddepcontrol.wait) before touching its predecessor's
// output; the down-projection kernel streams its weights in before that wait.
#pragma once

#include "common.cuh"
#include "gemv.cuh"
#include "route.cuh"

namespace moe {

// ============================================================ repack (load)
struct RepackParams {
  const uint8_t *codes;    // canonical packed codes of n experts
  const uint16_t *scales;  // canonical fp16 scales
  const uint16_t *mins;    // canonical fp16 mins (Q2) or null
  uint8_t *dst;            // device arena address of the first expert
  int n_experts;
  Layout L;
};

// First reduction column of k-step `st` held by lane quad position `tig`:
// within each 32-column block, lane tig owns columns [8 tig, 8 tig + 8): the
// first four feed k-step 2q (fragment columns 2tig, 2tig+1, 2tig+8, 2tig+9
// in that order), the next four k-step 2q+1.  The same permutation of the
// reduction applies to the codes and to the B operand, so one 16-byte load
// of a B row gives a lane both fragments of two consecutive k-steps.
MOE_HOST_DEV_INLINE int kb_step(int st, int tig) { return 32 * (st >> 1) + 8 * tig + 4 * (st & 1); }

// One thread per 32-bit code word of the device layout, then one per scale
// entry.  Canonical layout: per expert Wg [f,d], Wu [f,d], Wd [d,f] codes
// back to back (Q4: 2 per byte, low nibble first; Q2: 4 per byte, element i
// in bits 2*(i%4)); scales/mins [rows, K/G] per matrix in the same order.
__global__ void repack_kernel(RepackParams p) {
  const Layout &L = p.L;
  const int d = L.d, f = L.f, TK = L.TK, G = L.G;
  const bool q4 = L.fmt == 1;
  const long long mat_codes = q4 ? (long long)f * d / 2 : (long long)f * d / 4;
  const long long mat_groups = (long long)f * d / G;
  const int sblk = q4 ? 8 : 16;  // bytes of scale data per lane-group g
  // words per matrix tile: 32 lanes x 4 words; scale entries per tile:
  const int nse = q4 ? 4 : 8;
  // items: for each expert, matrix m in {0,1,2}, rb, tile, (lane, word) / (g, e)
  const int tiles_p1 = (f / 16) * (d / TK);  // per gate or up matrix
  const int tiles_p2 = (d / 16) * (f / TK);
  const long long tiles_expert = 2LL * tiles_p1 + tiles_p2;
  const long long words_per_tile = 128, scales_per_tile = 8LL * nse;
  const long long per_tile = words_per_tile + scales_per_tile;
  const long long total = (long long)p.n_experts * tiles_expert * per_tile;
  for (long long it = blockIdx.x * (long long)blockDim.x + threadIdx.x; it < total;
       it += (long long)gridDim.x * blockDim.x) {
    long long x = it;
    const int e = (int)(x / (tiles_expert * per_tile));
    x -= (long long)e * tiles_expert * per_tile;
    long long tile = x / per_tile;
    const int within = (int)(x - tile * per_tile);
    int m, K;
    if (tile < tiles_p1) { m = 0; }
    else if (tile < 2 * tiles_p1) { m = 1; tile -= tiles_p1; }
    else { m = 2; tile -= 2 * tiles_p1; }
    K = m < 2 ? d : f;
    const int ntile = K / TK;
    const int rb = (int)(tile / ntile), t = (int)(tile % ntile);
    const uint8_t *src = p.codes + (long long)e * 3 * mat_codes + m * mat_codes;
    const uint16_t *ssrc = p.scales + (long long)e * 3 * mat_groups + m * mat_groups;
    const uint16_t *msrc = p.mins ? p.mins + (long long)e * 3 * mat_groups + m * mat_groups : nullptr;
    uint8_t *tb = p.dst + (long long)e * L.expert_bytes +
                  (m < 2 ? ((long long)rb * ntile + t) * 2 * L.tile_bytes + (m == 1 ? L.tile_bytes : 0)
                         : L.p1_bytes + ((long long)rb * ntile + t) * L.tile_bytes);
    if (within < words_per_tile) {
      const int lane = within >> 2, word = within & 3;
      const int g = lane >> 2, tig = lane & 3;
      const int r0 = rb * 16 + g, r1 = r0 + 8;
      uint32_t v = 0;
      if (q4) {
        const int kb = t * 64 + kb_step(word, tig);
        for (int fr = 0; fr < 4; ++fr) {
          const int row = (fr & 1) ? r1 : r0, col = kb + ((fr & 2) ? 2 : 0);
          const uint32_t lo = (src[(long long)row * (K / 2) + col / 2] >> (4 * (col & 1))) & 0xF;
          const uint32_t hi = (src[(long long)row * (K / 2) + (col + 1) / 2] >> (4 * ((col + 1) & 1))) & 0xF;
          v |= lo << (4 * fr);
          v |= hi << (16 + 4 * fr);
        }
      } else {
        for (int r = 0; r < 8; ++r) {
          const int st = 2 * word + (r >> 2), fr = r & 3;
          const int kb = t * 128 + kb_step(st, tig);
          const int row = (fr & 1) ? r1 : r0, col = kb + ((fr & 2) ? 2 : 0);
          const uint32_t lo = (src[(long long)row * (K / 4) + col / 4] >> (2 * (col & 3))) & 3;
          const uint32_t hi = (src[(long long)row * (K / 4) + (col + 1) / 4] >> (2 * ((col + 1) & 3))) & 3;
          v |= lo << (2 * r);
          v |= hi << (16 + 2 * r);
        }
      }
      reinterpret_cast<uint32_t *>(tb)[lane * 4 + word] = v;
    } else {
      const int s = within - (int)words_per_tile;
      const int g = s / nse, ent = s % nse;
      const int row = rb * 16 + g + ((ent & 1) ? 8 : 0);
      const int grp = 2 * t + ((ent >> 1) & 1);
      const int ng = K / G;
      uint16_t v;
      if (q4 || ent < 4) v = ssrc[(long long)row * ng + grp];
      else v = msrc[(long long)row * ng + grp];
      reinterpret_cast<uint16_t *>(tb + 512 + g * sblk)[ent] = v;
    }
  }
}

// ================================================================ RMSNorm
struct NormParams {
  const uint16_t *x;
  const float *gamma;  // [d] or null
  float eps;
  int T, d;
  uint16_t *h;
};

// one CTA per token; sum of squares in fp32, IEEE sqrt and divide.
__global__ void __launch_bounds__(256) rmsnorm_kernel(NormParams p) {
  pdl_wait();
  const int t = blockIdx.x;
  const uint16_t *xr = p.x + (long long)t * p.d;
  float ss = 0.f;
  for (int i = threadIdx.x * 4; i < p.d; i += blockDim.x * 4) {
    uint2 v = ldcg_u2(xr + i);
    float a = __uint_as_float(v.x << 16), b = __uint_as_float(v.x & 0xFFFF0000u);
    float c = __uint_as_float(v.y << 16), e = __uint_as_float(v.y & 0xFFFF0000u);
    ss += a * a + b * b + c * c + e * e;
  }
  __shared__ float red[32];
  ss = warp_sum(ss);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
  __syncthreads();
  if (threadIdx.x < 32) {
    float v = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0.f;
    v = warp_sum(v);
    if (threadIdx.x == 0) red[0] = v;
  }
  __syncthreads();
  pdl_launch_dependents();
  const float inv = 1.0f / sqrtf(red[0] / (float)p.d + p.eps);
  for (int i = threadIdx.x * 4; i < p.d; i += blockDim.x * 4) {
    uint2 v = ldcg_u2(xr + i);
    float in[4] = {__uint_as_float(v.x << 16), __uint_as_float(v.x & 0xFFFF0000u),
                   __uint_as_float(v.y << 16), __uint_as_float(v.y & 0xFFFF0000u)};
    unsigned short o[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      float r = in[j] * inv;
      if (p.gamma) r *= p.gamma[i + j];
      o[j] = __bfloat16_as_ushort(__float2bfloat16_rn(r));
    }
    uint2 w;
    w.x = o[0] | ((uint32_t)o[1] << 16);
    w.y = o[2] | ((uint32_t)o[3] << 16);
    *reinterpret_cast<uint2 *>(p.h + (long long)t * p.d + i) = w;
  }
}

// =========================================================== router logits
struct RouterParams {
  const uint16_t *h;   // bf16 [T, d]
  const float *W;      // fp32 [E, d]
  const float *bias;   // fp32 [E] or null
  int T, d, E;
  float *logits;       // fp32 [T, E]
};

constexpr int kRouterWarps = 4;
constexpr int kRouterSmem = 48 * 1024;  // bytes of h staged per pass

// One warp per expert row: the row of W stays in registers (d/32 floats per
// lane, d <= 4096) and is dotted with the h rows of the CTA's token chunks
// (chunks blockIdx.y, + gridDim.y, ...), which the CTA stages in shared
// memory one chunk at a time; fp32 accumulate, four tokens in flight per
// warp.
template <int VPL>  // float4 vectors per lane = d / 128
__global__ void __launch_bounds__(kRouterWarps * 32) router_logits_kernel(RouterParams p) {
  extern __shared__ __align__(16) unsigned char rsm[];
  const int lane = threadIdx.x & 31;
  const int e = blockIdx.x * kRouterWarps + (threadIdx.x >> 5);
  const int d = p.d;
  float4 wv[VPL];
  if (e < p.E) {
    const float4 *wr = reinterpret_cast<const float4 *>(p.W + (long long)e * d);
#pragma unroll
    for (int i = 0; i < VPL; ++i) wv[i] = __ldg(wr + lane + 32 * i);
  }
  const float b = (e < p.E && p.bias) ? p.bias[e] : 0.f;
  pdl_wait();
  pdl_launch_dependents();
  const int tc = kRouterSmem / (2 * d);  // tokens per pass
  for (int t0 = blockIdx.y * tc; t0 < p.T; t0 += gridDim.y * tc) {
    const int nt = min(tc, p.T - t0);
    __syncthreads();
    const int n16 = nt * d / 8;  // 16-byte vectors, 8 loads in flight per thread
    const uint4 *src = reinterpret_cast<const uint4 *>(p.h + (long long)t0 * d);
    for (int i0 = threadIdx.x; i0 < n16; i0 += 8 * blockDim.x) {
      uint4 v[8];
#pragma unroll
      for (int q = 0; q < 8; ++q)
        if (i0 + q * (int)blockDim.x < n16) v[q] = ldcg_u4(src + i0 + q * blockDim.x);
#pragma unroll
      for (int q = 0; q < 8; ++q)
        if (i0 + q * (int)blockDim.x < n16) reinterpret_cast<uint4 *>(rsm)[i0 + q * blockDim.x] = v[q];
    }
    __syncthreads();
    if (e >= p.E) continue;
    for (int t = 0; t < nt; t += 4) {
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        if (t + q >= nt) break;
        const uint32_t hb = smem_addr(rsm) + (uint32_t)(t + q) * d * 2;
#pragma unroll
        for (int i = 0; i < VPL; ++i) {
          const uint2 v = lds_u2(hb + 8 * (lane + 32 * i));
          acc[q] = fmaf(wv[i].x, __uint_as_float(v.x << 16), acc[q]);
          acc[q] = fmaf(wv[i].y, __uint_as_float(v.x & 0xFFFF0000u), acc[q]);
          acc[q] = fmaf(wv[i].z, __uint_as_float(v.y << 16), acc[q]);
          acc[q] = fmaf(wv[i].w, __uint_as_float(v.y & 0xFFFF0000u), acc[q]);
        }
      }
#pragma unroll
      for (int o = 16; o; o >>= 1)
#pragma unroll
        for (int q = 0; q < 4; ++q) acc[q] += __shfl_xor_sync(0xffffffffu, acc[q], o);
      if (lane < 4 && t + lane < nt) {
        const float v = lane == 0 ? acc[0] : lane == 1 ? acc[1] : lane == 2 ? acc[2] : acc[3];
        p.logits[(long long)(t0 + t + lane) * p.E + e] = v + b;
      }
    }
  }
}

// ================================================================ combine
struct CombineParams {
  const float *y;      // [P_total][d]
  const float *w;      // [T][k]
  int T, k, d, has_shared;
  uint16_t *x;         // bf16 [T][d] residual (mode 0)
  float *delta;        // fp32 [T][d] (mode 1)
};

// x[t] <- bf16(x[t] + sum_j w[t,j] y[t*k+j] + y_shared[t]), j in order.
// Each thread owns 4 columns of one token and issues every load it needs
// (x, the k weights, the k + 1 rows of y) before the first use, 16 rows at a
// time, so their L2 latencies overlap; the sum is still taken in j order.
constexpr int kCombineBatch = 16;

__global__ void __launch_bounds__(128) combine_kernel(CombineParams p) {
  MOE_TRACE(kTrCombStart);
  pdl_wait();
  pdl_launch_dependents();
  const int per_t = p.d / 4;
  const long long n = (long long)p.T * per_t;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n;
       i += (long long)gridDim.x * blockDim.x) {
    const int t = (int)(i / per_t), o = (int)(i - (long long)t * per_t) * 4;
    uint16_t *xr = p.x ? p.x + (long long)t * p.d + o : nullptr;
    const uint2 xv = xr ? *reinterpret_cast<const uint2 *>(xr) : make_uint2(0u, 0u);
    const float4 sh = p.has_shared ? ldcg_f4(p.y + ((long long)p.T * p.k + t) * p.d + o)
                                   : make_float4(0.f, 0.f, 0.f, 0.f);
    float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
    for (int j0 = 0; j0 < p.k; j0 += kCombineBatch) {
      float4 v[kCombineBatch];
      float wj[kCombineBatch];
#pragma unroll
      for (int q = 0; q < kCombineBatch; ++q) {
        const int j = j0 + q;
        if (j < p.k) {
          wj[q] = __ldcg(p.w + (long long)t * p.k + j);
          v[q] = ldcg_f4(p.y + ((long long)t * p.k + j) * p.d + o);
        }
      }
#pragma unroll
      for (int q = 0; q < kCombineBatch; ++q) {
        if (j0 + q < p.k) {
          a0 = fmaf(wj[q], v[q].x, a0);
          a1 = fmaf(wj[q], v[q].y, a1);
          a2 = fmaf(wj[q], v[q].z, a2);
          a3 = fmaf(wj[q], v[q].w, a3);
        }
      }
    }
    a0 += sh.x;
    a1 += sh.y;
    a2 += sh.z;
    a3 += sh.w;
    if (p.delta) {
      *reinterpret_cast<float4 *>(p.delta + (long long)t * p.d + o) = make_float4(a0, a1, a2, a3);
    } else {
      const float r0 = __uint_as_float(xv.x << 16) + a0;
      const float r1 = __uint_as_float(xv.x & 0xFFFF0000u) + a1;
      const float r2 = __uint_as_float(xv.y << 16) + a2;
      const float r3 = __uint_as_float(xv.y & 0xFFFF0000u) + a3;
      uint2 o2;
      o2.x = __bfloat16_as_ushort(__float2bfloat16_rn(r0)) |
             ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(r1)) << 16);
      o2.y = __bfloat16_as_ushort(__float2bfloat16_rn(r2)) |
             ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(r3)) << 16);
      *reinterpret_cast<uint2 *>(xr) = o2;
    }
  }
  if ((threadIdx.x & 31) == 0) trace_point(kTrCombEnd);
}

}  // namespace moe
