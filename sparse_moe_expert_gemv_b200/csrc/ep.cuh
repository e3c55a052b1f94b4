// ep.cuh -- the two ends of an expert-parallel layer's exchange.
//
// The layer's experts are sharded by id over R ranks: rank r owns experts
// [r E/R, (r+1) E/R).  Each rank routes its own tokens (the engine article
// "93 token/s on one 8 GB card", section "Architecture overview": 10 of 512
// experts per token), sends the router-input row of every (token, expert)
// pair to the expert's owner, the owner runs its experts on the rows it
// receives, and the expert outputs travel back to the source rank, which
// combines them in j order exactly as the one-GPU layer does.  The
// exchange itself is the caller's collective (an all-to-all); these
// kernels build the send buffer and consume what comes back.
#pragma once

#include "route.cuh"

namespace moe {

constexpr int kEpMaxRanks = 64;

// Pairs are placed in blocks of kEpBlockPairs consecutive pair ids, one
// per lane of the block's warps.
constexpr int kEpWarps = 8, kEpBlockPairs = kEpWarps * 32;

struct EpPlanParams {
  const int *idx;       // [N, k] expert ids
  const uint16_t *h;    // bf16 [N, d] router input
  int N, k, d, E, R;
  int blocks;           // blocks of kEpBlockPairs pairs
  int *blk_cnt;         // [blocks][R] pairs of each block for each rank
  int *blk_off;         // [blocks][R] first send position of the block's pairs for each rank
  int *counts;          // [R] rows for each rank
  int *row_of;          // [N*k] send position of pair q = t k + j (-1: invalid id, not sent)
  int *send_e;          // [N*k] expert id of the row at each send position
  uint16_t *send_h;     // bf16 [rows sent, d]
  int *status;
};

// Owner rank of pair q's expert, or -1 for an id outside [0, E).
MOE_DEV int ep_owner(const EpPlanParams &p, long long q, int *e_out) {
  const int e = __ldg(p.idx + q);
  *e_out = e;
  return (e >= 0 && e < p.E) ? e / (p.E / p.R) : -1;
}

// Pass 1: each block's pair count for every rank (order does not matter).
__global__ void __launch_bounds__(kEpBlockPairs) ep_count_kernel(EpPlanParams p) {
  __shared__ int s_cnt[kEpMaxRanks];
  pdl_wait();
  for (int r = threadIdx.x; r < p.R; r += blockDim.x) s_cnt[r] = 0;
  __syncthreads();
  const long long P = (long long)p.N * p.k;
  const long long q = (long long)blockIdx.x * kEpBlockPairs + threadIdx.x;
  if (q < P) {
    int e;
    const int r = ep_owner(p, q, &e);
    if (r >= 0)
      atomicAdd(&s_cnt[r], 1);
    else
      atomicOr(p.status, kErrBadExpert);
  }
  __syncthreads();
  for (int r = threadIdx.x; r < p.R; r += blockDim.x) p.blk_cnt[(long long)blockIdx.x * p.R + r] = s_cnt[r];
  pdl_launch_dependents();
}

// Pass 2, one CTA: per rank, an exclusive scan of the blocks' counts in
// block order (the rank segments one after another) and the rank totals.
__global__ void __launch_bounds__(1024) ep_offsets_kernel(EpPlanParams p) {
  const int blocks = p.blocks;
  __shared__ int s_cnt[1025];
  __shared__ int s_red[32];
  pdl_wait();
  int base = 0;
  for (int r = 0; r < p.R; ++r) {
    const int start = base;
    for (int b0 = 0; b0 < blocks; b0 += 1024) {
      const int nb = min(1024, blocks - b0);
      for (int i = threadIdx.x; i < nb; i += blockDim.x) s_cnt[i] = p.blk_cnt[(long long)(b0 + i) * p.R + r];
      block_exclusive_scan(s_cnt, s_cnt, nb, s_red);
      for (int i = threadIdx.x; i < nb; i += blockDim.x) p.blk_off[(long long)(b0 + i) * p.R + r] = base + s_cnt[i];
      base += s_cnt[nb];
      __syncthreads();  // s_cnt is rewritten by the next range
    }
    if (threadIdx.x == 0) p.counts[r] = base - start;
  }
  pdl_launch_dependents();
}

// Pass 3: each pair's send position, stable in pair id inside a rank's
// segment (the block's offset, the earlier warps' counts, the earlier lanes
// with the same owner), then the warp copies the pairs' token rows to their
// positions, 16 bytes per lane per step.
__global__ void __launch_bounds__(kEpBlockPairs) ep_place_kernel(EpPlanParams p) {
  __shared__ int s_wcnt[kEpWarps][kEpMaxRanks];
  __shared__ int s_pos[kEpWarps][32];
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  pdl_wait();
  for (int i = threadIdx.x; i < kEpWarps * kEpMaxRanks; i += blockDim.x) (&s_wcnt[0][0])[i] = 0;
  __syncthreads();
  const long long P = (long long)p.N * p.k;
  const long long q = (long long)blockIdx.x * kEpBlockPairs + threadIdx.x;
  int e = -1, r = -1;
  if (q < P) r = ep_owner(p, q, &e);
  const unsigned same = __match_any_sync(0xffffffffu, r);
  const int before = __popc(same & ((1u << lane) - 1u));
  if (r >= 0 && before == 0) s_wcnt[wid][r] = __popc(same);
  __syncthreads();
  int pos = -1;
  if (r >= 0) {
    pos = p.blk_off[(long long)blockIdx.x * p.R + r] + before;
    for (int w = 0; w < wid; ++w) pos += s_wcnt[w][r];
    p.send_e[pos] = e;
  }
  if (q < P) p.row_of[q] = pos;
  s_pos[wid][lane] = pos;
  __syncwarp();
  const int n8 = p.d / 8;
  const long long q0 = (long long)blockIdx.x * kEpBlockPairs + wid * 32;
  for (int i = 0; i < 32 && q0 + i < P; ++i) {
    const int at = s_pos[wid][i];
    if (at < 0) continue;
    const uint4 *src = reinterpret_cast<const uint4 *>(p.h + ((q0 + i) / p.k) * p.d);
    uint4 *dst = reinterpret_cast<uint4 *>(p.send_h + (long long)at * p.d);
    for (int c = lane; c < n8; c += 32) dst[c] = __ldg(src + c);
  }
  pdl_launch_dependents();
}

struct EpCombineParams {
  const __half *y;        // fp16 [rows][d] expert outputs, in send order
  const int *row_of;      // [N*k] row of pair q in y (negative: contributes nothing)
  const float *w;         // [N, k]
  const float *y_shared;  // fp32 [N, d] or null
  int N, k, d;
  uint16_t *x;            // bf16 [N, d] residual (when delta is null)
  float *delta;           // fp32 [N, d] or null
};

// x[t] <- bf16(x[t] + sum_j w[t,j] y[row(t,j)] + y_shared[t]), j in order,
// with the one-GPU combine's arithmetic (one fused multiply-add per pair in
// j order, the shared expert's output added last), so a sharded layer
// reproduces the one-GPU result bit for bit.
__global__ void __launch_bounds__(256) ep_combine_kernel(EpCombineParams p) {
  pdl_wait();
  const int per_t = p.d / 4;
  const long long n = (long long)p.N * per_t;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n;
       i += (long long)gridDim.x * blockDim.x) {
    const int t = (int)(i / per_t), o = (int)(i - (long long)t * per_t) * 4;
    float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
    for (int j = 0; j < p.k; ++j) {
      const int row = __ldg(p.row_of + (long long)t * p.k + j);
      if (row < 0) continue;
      const float wj = __ldg(p.w + (long long)t * p.k + j);
      const uint2 q = __ldcs(reinterpret_cast<const uint2 *>(p.y + (long long)row * p.d + o));
      const float4 v = make_float4(half_lo(q.x), half_hi(q.x), half_lo(q.y), half_hi(q.y));
      a0 = fmaf(wj, v.x, a0);
      a1 = fmaf(wj, v.y, a1);
      a2 = fmaf(wj, v.z, a2);
      a3 = fmaf(wj, v.w, a3);
    }
    if (p.y_shared) {
      const float4 sh = __ldcs(reinterpret_cast<const float4 *>(p.y_shared + (long long)t * p.d + o));
      a0 += sh.x;
      a1 += sh.y;
      a2 += sh.z;
      a3 += sh.w;
    }
    if (p.delta) {
      *reinterpret_cast<float4 *>(p.delta + (long long)t * p.d + o) = make_float4(a0, a1, a2, a3);
    } else {
      uint16_t *xr = p.x + (long long)t * p.d + o;
      const uint2 xv = *reinterpret_cast<const uint2 *>(xr);
      uint2 o2;
      o2.x = __bfloat16_as_ushort(__float2bfloat16_rn(__uint_as_float(xv.x << 16) + a0)) |
             ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(__uint_as_float(xv.x & 0xFFFF0000u) + a1)) << 16);
      o2.y = __bfloat16_as_ushort(__float2bfloat16_rn(__uint_as_float(xv.y << 16) + a2)) |
             ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(__uint_as_float(xv.y & 0xFFFF0000u) + a3)) << 16);
      *reinterpret_cast<uint2 *>(xr) = o2;
    }
  }
  pdl_launch_dependents();
}

}  // namespace moe
