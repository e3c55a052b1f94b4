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
    int m, R, K;
    if (tile < tiles_p1) { m = 0; }
    else if (tile < 2 * tiles_p1) { m = 1; tile -= tiles_p1; }
    else { m = 2; tile -= 2 * tiles_p1; }
    if (m < 2) { R = f; K = d; } else { R = d; K = f; }
    (void)R;
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
        const int kb = t * 64 + 16 * word + 4 * tig;
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
          const int kb = t * 128 + 16 * st + 4 * tig;
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

// One warp per expert row: the row of W stays in registers (d/32 floats per
// lane, d <= 4096) and is dotted with every token's h; fp32 accumulate.
template <int VPL>  // float4 vectors per lane = d / 128
__global__ void __launch_bounds__(kRouterWarps * 32) router_logits_kernel(RouterParams p) {
  const int lane = threadIdx.x & 31;
  const int e = blockIdx.x * kRouterWarps + (threadIdx.x >> 5);
  float4 wv[VPL];
  if (e < p.E) {
    const float4 *wr = reinterpret_cast<const float4 *>(p.W + (long long)e * p.d);
#pragma unroll
    for (int i = 0; i < VPL; ++i) wv[i] = __ldg(wr + lane + 32 * i);
  }
  pdl_wait();
  pdl_launch_dependents();
  if (e >= p.E) return;
  const float b = p.bias ? p.bias[e] : 0.f;
  for (int t = 0; t < p.T; ++t) {
    const uint16_t *hr = p.h + (long long)t * p.d;
    float acc = 0.f;
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      uint2 v = ldcg_u2(hr + 4 * (lane + 32 * i));
      acc = fmaf(wv[i].x, __uint_as_float(v.x << 16), acc);
      acc = fmaf(wv[i].y, __uint_as_float(v.x & 0xFFFF0000u), acc);
      acc = fmaf(wv[i].z, __uint_as_float(v.y << 16), acc);
      acc = fmaf(wv[i].w, __uint_as_float(v.y & 0xFFFF0000u), acc);
    }
    acc = warp_sum(acc);
    if (lane == 0) p.logits[(long long)t * p.E + e] = acc + b;
  }
}

// ============================================ top-k, bucketing, work list
struct FinishParams {
  // inputs
  const float *logits;     // [T, E] or null (bucket-only mode)
  const int *idx_in;       // [T, k] when logits == null
  int T, E, k, layer;
  // routing outputs
  int *idx;                // [T, k]
  float *w;                // [T, k] (unused in bucket-only mode)
  int *off;                // [E+1] (may alias scratch)
  int *perm;               // [T*k]
  // work list (only when build_jobs)
  int build_jobs;
  int chunk;               // tokens per job
  int *plist;              // [T*k + T]
  unsigned long long *job_ptr;
  int *job_beg, *job_n, *n_jobs;
  int max_jobs;
  const int *slot_of;      // [L*E] residency table
  int n_slots;
  const uint8_t *arena;    // backing experts [L*E]
  const uint8_t *pool;     // slot pool [n_slots]
  const uint8_t *shared;   // shared expert of this layer or null
  long long expert_bytes;
  // statistics / status
  int *cnt_out;            // [E] tokens per expert (stats copy)
  unsigned long long *stats;  // [0]=calls [1]=tokens [2]=hits [3]=misses [4]=near_ties
  int *last;               // [0]=T [1]=active [2]=layer
  int *status;
};

constexpr int kFinishThreads = 1024;

// Single CTA.  Phase A: one warp per token selects the k largest logits by
// repeated warp arg-max (equal logits: lower expert id wins), then the
// softmax over the selected k.  Phase B: counting sort of the T*k pairs by
// expert (histogram, exclusive scan, stable scatter with ascending t).
// Phase C: the residency lookup (slot table -> slot pool or backing arena)
// and the list of expert jobs (<= chunk tokens each) for the expert kernels.
template <int NPL>  // logits per lane = ceil(E / 32)
__global__ void __launch_bounds__(kFinishThreads) route_finish_kernel(FinishParams p) {
  extern __shared__ int sm[];
  int *cnt = sm;                 // [E]
  int *off = cnt + p.E;          // [E+1]
  int *fill = off + p.E + 1;     // [E]
  int *jscan = fill + p.E;       // [E+1]
  __shared__ int red[32];
  __shared__ unsigned long long hit_miss[2];
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5, nw = blockDim.x >> 5;
  const int T = p.T, E = p.E, k = p.k, P = T * k;

  pdl_wait();
  pdl_launch_dependents();

  // ---------------- phase A: top-k + softmax
  if (p.logits) {
    for (int t = wid; t < T; t += nw) {
      float v[NPL];
      const float *lr = p.logits + (long long)t * E;
#pragma unroll
      for (int i = 0; i < NPL; ++i) {
        const int e = lane + 32 * i;
        v[i] = e < E ? __ldcg(lr + e) : -INFINITY;
      }
      uint32_t taken = 0;
      float my_v = 0.f, v0 = 0.f, vk = 0.f;
      int my_i = 0;
      for (int j = 0; j <= k; ++j) {
        if (j == k && k == E) break;
        float bv = -INFINITY;
        int bi = 0x7fffffff;
#pragma unroll
        for (int i = 0; i < NPL; ++i) {
          const int e = lane + 32 * i;
          if (e < E && !((taken >> i) & 1u) && (v[i] > bv || bi == 0x7fffffff)) {
            bv = v[i];
            bi = e;
          }
        }
#pragma unroll
        for (int o = 16; o; o >>= 1) {
          const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
          const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
          if (ov > bv || (ov == bv && oi < bi)) {
            bv = ov;
            bi = oi;
          }
        }
        if (j == k) {  // the (k+1)-th logit: near-tie count only
          if (lane == 0 && vk - bv < 1e-5f) atomicAdd(&p.stats[4], 1ULL);
          break;
        }
        if ((bi & 31) == lane) taken |= 1u << (bi >> 5);
        if (lane == j) {
          my_v = bv;
          my_i = bi;
        }
        if (j == 0) v0 = bv;
        vk = bv;
      }
      const float ex = lane < k ? expf(my_v - v0) : 0.f;
      const float den = warp_sum(ex);
      if (lane < k) {
        p.idx[(long long)t * k + lane] = my_i;
        p.w[(long long)t * k + lane] = ex / den;
      }
    }
  }
  __syncthreads();
  const int *idx = p.logits ? p.idx : p.idx_in;

  // ---------------- phase B: bucketing
  for (int e = tid; e < E; e += blockDim.x) {
    cnt[e] = 0;
    fill[e] = 0;
  }
  __syncthreads();
  for (int q = tid; q < P; q += blockDim.x) {
    const int e = idx[q];
    if (e >= 0 && e < E) atomicAdd(&cnt[e], 1);
    else atomicOr(p.status, kErrBadExpert);
  }
  __syncthreads();
  // exclusive scan of cnt -> off (E <= 1024 = blockDim)
  {
    const int v = tid < E ? cnt[tid] : 0;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) red[wid] = x;
    __syncthreads();
    if (wid == 0) {
      int s = lane < nw ? red[lane] : 0;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, s, o);
        if (lane >= o) s += y;
      }
      red[lane] = s;  // inclusive over warps
    }
    __syncthreads();
    const int base = wid ? red[wid - 1] : 0;
    if (tid < E) off[tid] = base + x - v;
    if (tid == 0) off[E] = red[nw - 1];
  }
  __syncthreads();
  // stable scatter: warp 0 walks the pairs in order, 32 at a time
  if (wid == 0) {
    for (int base = 0; base < P; base += 32) {
      const int q = base + lane;
      int e = q < P ? idx[q] : -1;
      if (e >= E) e = -1;
      const unsigned mask = __match_any_sync(0xffffffffu, e);
      const int rank = __popc(mask & ((1u << lane) - 1u));
      if (e >= 0) p.perm[off[e] + fill[e] + rank] = q;
      __syncwarp();
      if (e >= 0 && rank == 0) fill[e] += __popc(mask);
      __syncwarp();
    }
  }
  for (int e = tid; e <= E; e += blockDim.x) p.off[e] = off[e];
  if (!p.build_jobs) return;
  __syncthreads();

  // ---------------- phase C: residency lookup + expert jobs
  if (tid < 2) hit_miss[tid] = 0;
  {
    const int nch = tid < E ? (cnt[tid] + p.chunk - 1) / p.chunk : 0;
    int x = nch;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    __syncthreads();
    if (lane == 31) red[wid] = x;
    __syncthreads();
    if (wid == 0) {
      int s = lane < nw ? red[lane] : 0;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, s, o);
        if (lane >= o) s += y;
      }
      red[lane] = s;
    }
    __syncthreads();
    const int base = wid ? red[wid - 1] : 0;
    if (tid < E) jscan[tid] = base + x - nch;
    if (tid == 0) jscan[E] = red[nw - 1];
  }
  __syncthreads();
  const int routed_jobs = jscan[E];
  const int shared_jobs = p.shared ? (T + p.chunk - 1) / p.chunk : 0;
  if (routed_jobs + shared_jobs > p.max_jobs) {
    if (tid == 0) {
      atomicOr(p.status, kErrJobOverflow);
      *p.n_jobs = 0;
    }
    return;
  }
  int active = 0;
  for (int e = tid; e < E; e += blockDim.x) {
    const int c = cnt[e];
    p.cnt_out[e] = c;
    if (!c) continue;
    active++;
    const long long le = (long long)p.layer * E + e;
    const int slot = p.slot_of ? p.slot_of[le] : -1;
    const uint8_t *ptr;
    if (slot >= 0 && slot < p.n_slots) {
      ptr = p.pool + (long long)slot * p.expert_bytes;
      atomicAdd(&hit_miss[0], (unsigned long long)c);
    } else {
      if (slot >= p.n_slots) atomicOr(p.status, kErrBadSlot);
      ptr = p.arena + le * p.expert_bytes;
      atomicAdd(&hit_miss[1], (unsigned long long)c);
    }
    for (int j = jscan[e], b = 0; b < c; ++j, b += p.chunk) {
      p.job_ptr[j] = (unsigned long long)ptr;
      p.job_beg[j] = off[e] + b;
      p.job_n[j] = min(p.chunk, c - b);
    }
  }
  for (int q = tid; q < P; q += blockDim.x) p.plist[q] = p.perm[q];
  if (p.shared) {
    for (int t = tid; t < T; t += blockDim.x) p.plist[P + t] = P + t;
    for (int s = tid; s < shared_jobs; s += blockDim.x) {
      const int j = routed_jobs + s;
      p.job_ptr[j] = (unsigned long long)p.shared;
      p.job_beg[j] = P + s * p.chunk;
      p.job_n[j] = min(p.chunk, T - s * p.chunk);
    }
  }
  // statistics
  {
    int a = active;
#pragma unroll
    for (int o = 16; o; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
    if (lane == 0) red[wid] = a;
  }
  __syncthreads();
  if (tid == 0) {
    int a = 0;
    for (int i = 0; i < nw; ++i) a += red[i];
    *p.n_jobs = routed_jobs + shared_jobs;
    p.stats[0] += 1;
    p.stats[1] += (unsigned long long)T;
    p.stats[2] += hit_miss[0];
    p.stats[3] += hit_miss[1];
    p.last[0] = T;
    p.last[1] = a;
    p.last[2] = p.layer;
  }
}

// ================================================== grouped dequant GEMV
struct GemvParams {
  const unsigned long long *job_ptr;  // expert base address per job
  const int *job_beg, *job_n, *n_jobs;
  const int *plist;    // pair ids; pair < Tk: routed (token = pair / k), else shared (token = pair - Tk)
  int Tk, k;
  const uint16_t *src; // bf16 B-operand rows: h [T][K] (gated) or a [pairs][K]
  int src_by_pair;
  int K, R;            // reduction length, output rows of this phase
  long long region_off;
  uint16_t *out_a;     // gated: bf16 a [pairs][R]
  float *out_y;        // down: fp32 y [pairs][R]
  int *status;
};

template <int FMT, bool GATED>
struct GemvCfg {
  static constexpr int TK = FMT == 1 ? 64 : 128;
  static constexpr int TILE = FMT == 1 ? 576 : 640;
  static constexpr int NM = GATED ? 2 : 1;
  static constexpr int STRIDE = NM * TILE;
  static constexpr int D = 8;       // tiles in flight per warp
  static constexpr int NT = 2;      // 8-token mma column tiles per job
  static constexpr int WARPS = 8;
  static constexpr int SMEM = WARPS * D * STRIDE + WARPS * D * 8;
};

// Persistent kernel.  Work items are (job, 16-row block); items are dealt
// round-robin to warps so consecutive items land on different SMs.  Each
// warp streams the tiles of its items through a private ring of D shared-
// memory slots filled by 1-D bulk (TMA) copies, so up to D tiles are in
// flight per warp across item boundaries.  Every weight byte is read once
// per job; the 4-bit/2-bit codes are turned into exact bf16 integers in
// registers and multiplied on the tensor cores (mma m16n8k16, fp32
// accumulate) against the job's token rows; each quantisation group's
// partial sum is scaled in fp32 (Q2 adds min * sum(h) from a second mma
// against a ones matrix).
template <int FMT, bool GATED>
__global__ void __launch_bounds__(256) expert_gemv_kernel(GemvParams p) {
  using C = GemvCfg<FMT, GATED>;
  extern __shared__ __align__(128) unsigned char smem[];
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int g = lane >> 2, tig = lane & 3;
  unsigned char *ring = smem + wid * C::D * C::STRIDE;
  const uint32_t ring_s = smem_addr(ring);
  const uint32_t bar_s = smem_addr(smem + C::WARPS * C::D * C::STRIDE) + wid * C::D * 8;

  if (GATED) {
    pdl_wait();
    pdl_launch_dependents();
  }
  if (lane == 0) {
    for (int u = 0; u < C::D; ++u) mbar_init(bar_s + 8 * u, 1);
    fence_mbar_init();
  }
  __syncwarp();

  const int n_jobs = ldcg_i32(p.n_jobs);
  const int RB = p.R / 16, NTILE = p.K / C::TK;
  const long long n_items = (long long)n_jobs * RB;
  const int W = gridDim.x * C::WARPS;
  const int w = wid * gridDim.x + blockIdx.x;
  const int my_items = n_items > w ? (int)((n_items - w + W - 1) / W) : 0;
  const int total = my_items * NTILE;

  auto tile_src = [&](int q) -> const unsigned char * {
    const int j = q / NTILE, t = q - j * NTILE;
    const long long item = w + (long long)j * W;
    const int job = (int)(item / RB), rb = (int)(item - (long long)job * RB);
    const unsigned long long base = ldcg_u64(p.job_ptr + job);
    return reinterpret_cast<const unsigned char *>(base) + p.region_off +
           ((long long)rb * NTILE + t) * C::STRIDE;
  };
  auto issue = [&](int u, int q) {
    if (lane == 0) {
      fence_proxy_async_smem();
      mbar_expect_tx(bar_s + 8 * u, C::STRIDE);
      bulk_g2s(ring_s + u * C::STRIDE, tile_src(q), C::STRIDE, bar_s + 8 * u);
    }
  };
  for (int u = 0; u < C::D && u < total; ++u) issue(u, u);
  if (!GATED) pdl_wait();

  float acc[C::NM][C::NT][4];
  float tmp[C::NM][C::NT][4];
  float tH[C::NT][4];
  const uint16_t *brow[C::NT];
  int epair[C::NT][2];
  int ntA = 0, rb = 0;
  const float zero4[4] = {0.f, 0.f, 0.f, 0.f};
  const uint32_t ones[4] = {0x3F803F80u, 0x3F803F80u, 0x3F803F80u, 0x3F803F80u};

  for (int q = 0; q < total; ++q) {
    const int j = q / NTILE, t = q - j * NTILE;
    if (t == 0) {  // ---- start of an item
      const long long item = w + (long long)j * W;
      const int job = (int)(item / RB);
      rb = (int)(item - (long long)job * RB);
      const int n = ldcg_i32(p.job_n + job), beg = ldcg_i32(p.job_beg + job);
      ntA = (n + 7) >> 3;
#pragma unroll
      for (int nt = 0; nt < C::NT; ++nt) {
        const int ni = nt * 8 + g;
        brow[nt] = nullptr;
        if (ni < n) {
          const int pair = ldcg_i32(p.plist + beg + ni);
          const int row = p.src_by_pair ? pair : (pair < p.Tk ? pair / p.k : pair - p.Tk);
          brow[nt] = p.src + (long long)row * p.K;
        }
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          const int nc = nt * 8 + 2 * tig + c;
          epair[nt][c] = nc < n ? ldcg_i32(p.plist + beg + nc) : -1;
        }
#pragma unroll
        for (int m = 0; m < C::NM; ++m)
#pragma unroll
          for (int c = 0; c < 4; ++c) acc[m][nt][c] = 0.f;
      }
    }
    const int u = q & (C::D - 1);
    if (!mbar_wait_bounded(bar_s + 8 * u, (q / C::D) & 1)) {
      if (lane == 0) atomicOr(p.status, kErrTimeout);
      return;
    }
    const uint32_t tile_s = ring_s + u * C::STRIDE;
    uint4 cw[C::NM];
#pragma unroll
    for (int m = 0; m < C::NM; ++m) cw[m] = lds_u4(tile_s + m * C::TILE + lane * 16);

    if constexpr (FMT == 1) {
      uint2 sc[C::NM];
#pragma unroll
      for (int m = 0; m < C::NM; ++m) sc[m] = lds_u2(tile_s + m * C::TILE + 512 + g * 8);
      // B fragments for the tile: 4 steps x 8 bytes per 8-token column tile
      uint2 bq[C::NT][4];
#pragma unroll
      for (int nt = 0; nt < C::NT; ++nt)
#pragma unroll
        for (int s = 0; s < 4; ++s)
          bq[nt][s] = (nt < ntA && brow[nt]) ? ldcg_u2(brow[nt] + t * 64 + 16 * s + 4 * tig)
                                             : make_uint2(0u, 0u);
#pragma unroll
      for (int s = 0; s < 4; ++s) {
        uint32_t a[C::NM][4];
#pragma unroll
        for (int m = 0; m < C::NM; ++m) {
          const uint32_t word = s == 0 ? cw[m].x : s == 1 ? cw[m].y : s == 2 ? cw[m].z : cw[m].w;
          unpack_q4(word, a[m]);
        }
#pragma unroll
        for (int nt = 0; nt < C::NT; ++nt) {
          if (nt < ntA) {
#pragma unroll
            for (int m = 0; m < C::NM; ++m) {
              if (s & 1) mma_bf16_16816(tmp[m][nt], a[m], bq[nt][s].x, bq[nt][s].y, tmp[m][nt]);
              else mma_bf16_16816(tmp[m][nt], a[m], bq[nt][s].x, bq[nt][s].y, zero4);
            }
          }
        }
        if (s & 1) {  // end of a 32-wide group: scale and accumulate
#pragma unroll
          for (int m = 0; m < C::NM; ++m) {
            const uint32_t sv = (s >> 1) ? sc[m].y : sc[m].x;
            const float slo = half_lo(sv), shi = half_hi(sv);
#pragma unroll
            for (int nt = 0; nt < C::NT; ++nt) {
              acc[m][nt][0] = fmaf(slo, tmp[m][nt][0], acc[m][nt][0]);
              acc[m][nt][1] = fmaf(slo, tmp[m][nt][1], acc[m][nt][1]);
              acc[m][nt][2] = fmaf(shi, tmp[m][nt][2], acc[m][nt][2]);
              acc[m][nt][3] = fmaf(shi, tmp[m][nt][3], acc[m][nt][3]);
            }
          }
        }
      }
    } else {
      uint4 sc[C::NM];
#pragma unroll
      for (int m = 0; m < C::NM; ++m) sc[m] = lds_u4(tile_s + m * C::TILE + 512 + g * 16);
#pragma unroll
      for (int half = 0; half < 2; ++half) {  // two groups of 64 per tile
        uint2 bq[C::NT][4];
#pragma unroll
        for (int nt = 0; nt < C::NT; ++nt)
#pragma unroll
          for (int s = 0; s < 4; ++s)
            bq[nt][s] = (nt < ntA && brow[nt])
                            ? ldcg_u2(brow[nt] + t * 128 + 64 * half + 16 * s + 4 * tig)
                            : make_uint2(0u, 0u);
#pragma unroll
        for (int wv = 0; wv < 2; ++wv) {
          uint32_t a8[C::NM][8];
#pragma unroll
          for (int m = 0; m < C::NM; ++m) {
            const int wi = 2 * half + wv;
            const uint32_t word = wi == 0 ? cw[m].x : wi == 1 ? cw[m].y : wi == 2 ? cw[m].z : cw[m].w;
            unpack_q2(word, a8[m]);
          }
#pragma unroll
          for (int hs = 0; hs < 2; ++hs) {
            const int s = 2 * wv + hs;  // step within the group
#pragma unroll
            for (int nt = 0; nt < C::NT; ++nt) {
              if (nt < ntA) {
#pragma unroll
                for (int m = 0; m < C::NM; ++m) {
                  const uint32_t af[4] = {a8[m][4 * hs], a8[m][4 * hs + 1], a8[m][4 * hs + 2],
                                          a8[m][4 * hs + 3]};
                  if (s) mma_bf16_16816(tmp[m][nt], af, bq[nt][s].x, bq[nt][s].y, tmp[m][nt]);
                  else mma_bf16_16816(tmp[m][nt], af, bq[nt][s].x, bq[nt][s].y, zero4);
                }
                if (s) mma_bf16_16816(tH[nt], ones, bq[nt][s].x, bq[nt][s].y, tH[nt]);
                else mma_bf16_16816(tH[nt], ones, bq[nt][s].x, bq[nt][s].y, zero4);
              }
            }
          }
        }
        // end of group `half`: acc += s * sum(q h) + m * sum(h)
#pragma unroll
        for (int m = 0; m < C::NM; ++m) {
          const uint32_t sv = half ? sc[m].y : sc[m].x;
          const uint32_t mv = half ? sc[m].w : sc[m].z;
          const float slo = half_lo(sv), shi = half_hi(sv);
          const float mlo = half_lo(mv), mhi = half_hi(mv);
#pragma unroll
          for (int nt = 0; nt < C::NT; ++nt) {
            acc[m][nt][0] = fmaf(slo, tmp[m][nt][0], fmaf(mlo, tH[nt][0], acc[m][nt][0]));
            acc[m][nt][1] = fmaf(slo, tmp[m][nt][1], fmaf(mlo, tH[nt][1], acc[m][nt][1]));
            acc[m][nt][2] = fmaf(shi, tmp[m][nt][2], fmaf(mhi, tH[nt][2], acc[m][nt][2]));
            acc[m][nt][3] = fmaf(shi, tmp[m][nt][3], fmaf(mhi, tH[nt][3], acc[m][nt][3]));
          }
        }
      }
    }
    __syncwarp();
    if (q + C::D < total) issue(u, q + C::D);

    if (t == NTILE - 1) {  // ---- end of an item: epilogue
#pragma unroll
      for (int nt = 0; nt < C::NT; ++nt) {
        if (nt >= ntA) continue;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int pair = epair[nt][c & 1];
          if (pair < 0) continue;
          const int row = rb * 16 + g + (c >= 2 ? 8 : 0);
          if constexpr (GATED) {
            const float gv = acc[0][nt][c], uv = acc[1][nt][c];
            const float av = gv / (1.0f + __expf(-gv)) * uv;
            p.out_a[(long long)pair * p.R + row] = __bfloat16_as_ushort(__float2bfloat16_rn(av));
          } else {
            p.out_y[(long long)pair * p.R + row] = acc[0][nt][c];
          }
        }
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
__global__ void __launch_bounds__(256) combine_kernel(CombineParams p) {
  pdl_wait();
  pdl_launch_dependents();
  const int per_t = p.d / 4;
  const long long n = (long long)p.T * per_t;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n;
       i += (long long)gridDim.x * blockDim.x) {
    const int t = (int)(i / per_t), o = (int)(i - (long long)t * per_t) * 4;
    float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
    for (int j = 0; j < p.k; ++j) {
      const float wj = __ldcg(p.w + (long long)t * p.k + j);
      const float4 v = ldcg_f4(p.y + ((long long)t * p.k + j) * p.d + o);
      a0 = fmaf(wj, v.x, a0);
      a1 = fmaf(wj, v.y, a1);
      a2 = fmaf(wj, v.z, a2);
      a3 = fmaf(wj, v.w, a3);
    }
    if (p.has_shared) {
      const float4 v = ldcg_f4(p.y + ((long long)p.T * p.k + t) * p.d + o);
      a0 += v.x;
      a1 += v.y;
      a2 += v.z;
      a3 += v.w;
    }
    if (p.delta) {
      *reinterpret_cast<float4 *>(p.delta + (long long)t * p.d + o) = make_float4(a0, a1, a2, a3);
    } else {
      uint16_t *xr = p.x + (long long)t * p.d + o;
      const uint2 xv = *reinterpret_cast<const uint2 *>(xr);
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
}

}  // namespace moe
