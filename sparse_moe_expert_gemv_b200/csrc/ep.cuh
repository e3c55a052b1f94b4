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

struct EpPlanParams {
  const int *idx;  // [N, k] expert ids
  int N, k, E, R;
  int *row_of;     // [N*k] send position of pair q = t k + j (-1: invalid id, not sent)
  int *send_e;     // [N*k] expert id of the row at each send position
  int *counts;     // [R] rows for each rank
  int *status;
};

// One CTA of 1024 threads.  Each thread takes a run of consecutive pairs;
// for each rank in turn a block scan over the runs' counts gives every
// run's first position inside that rank's segment, so each segment lists
// its pairs in ascending pair id (t, then j).  An id outside [0, E) sets
// the device status and its pair is left out (row_of = -1).
__global__ void __launch_bounds__(1024) ep_plan_kernel(EpPlanParams p) {
  __shared__ int s_cnt[1025];
  __shared__ int s_red[32];
  pdl_wait();
  const int tid = threadIdx.x;
  const int P = p.N * p.k, per = p.E / p.R;
  const int ept = (P + blockDim.x - 1) / blockDim.x;
  const int q0 = min(P, tid * ept), q1 = min(P, q0 + ept);
  bool bad = false;
  for (int q = q0; q < q1; ++q) {
    const int e = __ldg(p.idx + q);
    if (e < 0 || e >= p.E) {
      p.row_of[q] = -1;
      bad = true;
    }
  }
  if (bad) atomicOr(p.status, kErrBadExpert);
  int base = 0;
  for (int r = 0; r < p.R; ++r) {
    int n = 0;
    for (int q = q0; q < q1; ++q) {
      const int e = __ldg(p.idx + q);
      n += (e >= 0 && e < p.E && e / per == r);
    }
    s_cnt[tid] = n;
    block_exclusive_scan(s_cnt, s_cnt, blockDim.x, s_red);
    int pos = base + s_cnt[tid];
    for (int q = q0; q < q1; ++q) {
      const int e = __ldg(p.idx + q);
      if (e >= 0 && e < p.E && e / per == r) {
        p.row_of[q] = pos;
        p.send_e[pos] = e;
        ++pos;
      }
    }
    const int total = s_cnt[blockDim.x];
    if (tid == 0) p.counts[r] = total;
    base += total;
    __syncthreads();  // s_cnt is rewritten by the next rank's counts
  }
  pdl_launch_dependents();
}

struct EpGatherParams {
  const uint16_t *h;   // bf16 [N, d] router input
  const int *row_of;   // [N*k]
  int N, k, d;
  uint16_t *send_h;    // bf16 [rows sent, d]
};

// One warp per pair: the token's row to the pair's send position, 16 bytes
// per lane per step.
__global__ void __launch_bounds__(256) ep_gather_kernel(EpGatherParams p) {
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const long long P = (long long)p.N * p.k;
  const int n8 = p.d / 8;
  const long long nw = ((long long)gridDim.x * blockDim.x) >> 5;
  for (long long q = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5; q < P; q += nw) {
    const int pos = __ldg(p.row_of + q);
    if (pos < 0) continue;
    const uint4 *src = reinterpret_cast<const uint4 *>(p.h + (q / p.k) * p.d);
    uint4 *dst = reinterpret_cast<uint4 *>(p.send_h + (long long)pos * p.d);
    for (int i = lane; i < n8; i += 32) dst[i] = __ldg(src + i);
  }
  pdl_launch_dependents();
}

struct EpCombineParams {
  const float *y;         // fp32 [rows][d] expert outputs, in send order
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
      const float4 v = __ldcs(reinterpret_cast<const float4 *>(p.y + (long long)row * p.d + o));
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
