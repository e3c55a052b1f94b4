// prefill.cuh -- the MoE layer for a prefill chunk of up to 8192 tokens
// (sm_100a).
//
// A chunk is a real dense contraction per expert (the engine article "93
// token/s on one 8 GB card", section "Architecture overview": prefill runs
// in chunks of up to 8192 tokens), so the experts run as a grouped GEMM on
// the 5th-generation tensor cores:
//
//   prefill_topk_kernel     one warp per token: top-k + softmax (candidate
//                           filter, warp_topk_fast); per block of
//                           kPfTok tokens, each expert's token set (a bitmask)
//   prefill_colscan_kernel  per expert: each block of tokens' first row
//                           relative to the expert's (a scan down the
//                           expert's column of block masks) and its tokens
//   prefill_scan_kernel     the experts' first rows in grouped order and the
//                           list of 256-row tiles (expert, first row, rows)
//   prefill_scatter_kernel  pair -> row in grouped order (stable: ascending t
//                           within an expert) and the gather of every pair's
//                           token row into the grouped A matrix (fp16)
//   prefill_gemm_kernel     on CTA pairs: A tiles (TMA, 128B swizzle) x
//                           dequantised weight tiles (written by each CTA's
//                           warps straight into the swizzled fp16 layout) ->
//                           tcgen05.mma.cta_group::2 m256n256k16, fp32
//                           accumulators in both CTAs' TMEM; gate/up pass writes
//                           SiLU(G) * U (fp16), down pass writes y (fp16)
//   prefill_combine_kernel  x += sum_j w_j y[row(t, j)] + y_shared[t]
//
// Operands are fp16: a Q4 weight s*(c-8) with its fp16 scale is one
// rounding away from exact in fp16, and bf16 activations convert to fp16
// exactly in fp16's normal range (values beyond +-65504 saturate).
#pragma once

#include <cuda.h>

#include "common.cuh"
#include "route.cuh"

namespace moe {

// Tokens per block of the top-k / scatter kernels (one warp each; a block's
// per-expert token set is a 16-bit mask).  Eight rather than 16: a top-k
// CTA waits for its slowest token (the few with an exact refinement), and
// 8-warp CTAs fit three to an SM instead of one.
constexpr int kPfTok = 8;
constexpr int kPfBM = 128;       // rows of one MMA (an M-half of a GEMM tile)
constexpr int kPfTileRows = 2 * kPfBM;  // rows of one GEMM tile of an expert (two M-halves)
constexpr int kPfBN = 128;       // GEMM tile columns (output features)
constexpr int kPfBK = 64;        // reduction per stage (one 128-byte swizzle row of fp16)
constexpr int kPfMaxE = 1024;

struct PfTile {                  // one tile of up to 256 rows of one expert
  const uint8_t *w;              // expert base (repacked layout)
  int row0, rows;                // first row in grouped order, rows <= 256
};

// logits[t, e] = sum_z part[z][t, e] (z = 0, 1, ... in order) + bias[e]: the
// partial sums of a router whose reduction was split over ksplit CTAs.  One
// thread per four logits, every partial load in flight at once.
constexpr int kMaxRouterSplit = 16;
struct RouterSumParams {
  const float *part;  // [ksplit][T][E]
  int ksplit;
  const float *bias;  // [E] or null
  int T, E;           // E a multiple of 4
  float *logits;      // [T][E]
};

__global__ void __launch_bounds__(256) router_sum_kernel(RouterSumParams p) {
  const float *part = p.part, *bias = p.bias;
  const int ksplit = p.ksplit, E = p.E;
  float *logits = p.logits;
  pdl_wait();
  const long long n4 = (long long)p.T * E / 4, plane = (long long)p.T * E;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n4;
       i += (long long)gridDim.x * blockDim.x) {
    float4 v[kMaxRouterSplit];
#pragma unroll
    for (int z = 0; z < kMaxRouterSplit; ++z)
      if (z < ksplit) v[z] = __ldcg(reinterpret_cast<const float4 *>(part + z * plane) + i);
    float4 s = v[0];
#pragma unroll
    for (int z = 1; z < kMaxRouterSplit; ++z)
      if (z < ksplit) {
        s.x += v[z].x;
        s.y += v[z].y;
        s.z += v[z].z;
        s.w += v[z].w;
      }
    if (bias) {
      const int e = (int)((i * 4) % E);
      s.x += bias[e];
      s.y += bias[e + 1];
      s.z += bias[e + 2];
      s.w += bias[e + 3];
    }
    reinterpret_cast<float4 *>(logits)[i] = s;
  }
  pdl_launch_dependents();
}

struct PfRouteParams {
  float *logits;        // [T, E]
  int T, E, k;
  int *idx;             // [T, k]
  float *w;             // [T, k]
  unsigned short *bmask;  // [blocks][E]: bit i = token 16 b + i selected the expert
  unsigned long long *near_ties;
  const float *bias;    // [E] or null (for the boundary refinement)
  const uint16_t *h;    // bf16 [T, d] router input and
  const float *W;       // fp32 [E, d] router rows, for the boundary refinement
  int d;
};

// Logits within this distance of a token's selection boundary (its k-th and
// (k+1)-th logits) are recomputed exactly before the final selection.  The
// chunk routers accumulate in fp32 in an order of their own (the tensor-core
// router inside its MMAs); their error stays far below this band, so outside
// it no two logits can change order.
constexpr float kRefineBand = 2e-3f;

// One warp: the exact logit of expert e for token row h (fp64 sum of the
// exact fp32 x bf16 products, then the bias), rounded once to fp32.
// d a multiple of 128; loads four columns per lane at a time, eight in flight.
MOE_DEV float exact_logit(const float *W, const uint16_t *h, const float *bias, int d, int e, int lane) {
  const float4 *wr = reinterpret_cast<const float4 *>(W + (long long)e * d);
  const uint2 *hr = reinterpret_cast<const uint2 *>(h);
  const int n4 = d / 4;
  double acc = 0.0;
  for (int i0 = lane; i0 < n4; i0 += 32 * 8) {
    float4 wv[8];
    uint2 hv[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const int i = i0 + 32 * q;
      wv[q] = i < n4 ? __ldg(wr + i) : make_float4(0.f, 0.f, 0.f, 0.f);
      hv[q] = i < n4 ? __ldg(hr + i) : make_uint2(0u, 0u);
    }
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      acc += (double)wv[q].x * (double)__uint_as_float(hv[q].x << 16);
      acc += (double)wv[q].y * (double)__uint_as_float(hv[q].x & 0xFFFF0000u);
      acc += (double)wv[q].z * (double)__uint_as_float(hv[q].y << 16);
      acc += (double)wv[q].w * (double)__uint_as_float(hv[q].y & 0xFFFF0000u);
    }
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  return (float)(acc + (bias ? (double)bias[e] : 0.0));
}

// One warp per token; then the block's per-expert token sets.
template <int NPL>
__global__ void __launch_bounds__(kPfTok * 32) prefill_topk_kernel(PfRouteParams p) {
  __shared__ unsigned s_mask[kPfMaxE];
  __shared__ unsigned long long s_cand[kPfTok][64];  // each warp's top-k candidates
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  pdl_wait();
  for (int e = threadIdx.x; e < p.E; e += blockDim.x) s_mask[e] = 0u;
  __syncthreads();
  const int t = blockIdx.x * kPfTok + wid;
  if (t < p.T) {
    int e;
    float w, lk, lk1;
    float *lr = p.logits + (long long)t * p.E;
    if (!warp_topk_fast<NPL>(lr, p.E, p.k, lane, s_cand[wid], e, w, nullptr, &lk, &lk1))
      warp_topk<NPL>(lr, p.E, p.k, lane, false, e, w, nullptr, &lk, &lk1);
    if (lk - lk1 < kRefineBand) {
      // the boundary is close: recompute the logits in the band around it
      // exactly, then select again (and count a near tie on exact values)
      const uint16_t *hrow = p.h + (long long)t * p.d;
      for (int i = 0; i < (p.E + 31) / 32; ++i) {
        const int ei = lane + 32 * i;
        const float v = ei < p.E ? __ldcg(lr + ei) : -INFINITY;
        unsigned band = __ballot_sync(0xffffffffu, ei < p.E && v >= lk1 - kRefineBand && v <= lk + kRefineBand);
        while (band) {
          const int src = __ffs(band) - 1;
          band &= band - 1;
          const float x = exact_logit(p.W, hrow, p.bias, p.d, src + 32 * i, lane);
          if (lane == src) lr[ei] = x;
        }
      }
      __threadfence();
      __syncwarp();
      warp_topk<NPL>(lr, p.E, p.k, lane, false, e, w, p.near_ties);
    }
    if (lane < p.k) {
      p.idx[(long long)t * p.k + lane] = e;
      p.w[(long long)t * p.k + lane] = w;
      atomicOr(&s_mask[e], 1u << wid);
    }
  }
  __syncthreads();
  for (int e = threadIdx.x; e < p.E; e += blockDim.x)
    p.bmask[(long long)blockIdx.x * p.E + e] = (unsigned short)s_mask[e];
  pdl_launch_dependents();
}

// Caller-given routing (idx [T, k], distinct ids in [0, E) per token,
// checked on the host): the block masks prefill_topk_kernel would have
// written for it, so the chunk path's bucketing can run without the router.
struct PfMaskParams {
  const int *idx;         // [T, k]
  int T, E, k;
  unsigned short *bmask;  // [blocks][E]
};

__global__ void __launch_bounds__(kPfTok * 32) prefill_mask_kernel(PfMaskParams p) {
  __shared__ unsigned s_mask[kPfMaxE];
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  pdl_wait();
  for (int e = threadIdx.x; e < p.E; e += blockDim.x) s_mask[e] = 0u;
  __syncthreads();
  const int t = blockIdx.x * kPfTok + wid;
  if (t < p.T && lane < p.k) atomicOr(&s_mask[__ldg(p.idx + (long long)t * p.k + lane)], 1u << wid);
  __syncthreads();
  for (int e = threadIdx.x; e < p.E; e += blockDim.x)
    p.bmask[(long long)blockIdx.x * p.E + e] = (unsigned short)s_mask[e];
  pdl_launch_dependents();
}

struct PfScanParams {
  const unsigned short *bmask;  // [blocks][E]
  int blocks, E, T, k;
  int *boff;                    // [blocks][E] first row of (block, expert) relative to the expert's
  int *col_part;                // [kPfColSplitMax][E] per-range token counts (split column scan)
  int *eoff;                    // [E + 1] token counts (colscan), then first rows (scan)
  const int *slot_of;           // residency table [L*E]
  int n_slots, layer;
  const uint8_t *arena, *pool, *shared;
  long long expert_bytes;
  PfTile *tiles;                // [max_tiles]
  int *n_tiles;
  int max_tiles;
  // experts with fewer than hot_min tokens become GEMV jobs instead of GEMM
  // tiles (hot_min <= 1: every expert is a GEMM expert)
  int hot_min, chunk;           // chunk: tokens per GEMV job
  int *hot;                     // [E] 1 = GEMM expert
  unsigned long long *job_ptr;  // [max_jobs] expert base address per GEMV job
  int *job_beg, *job_n, *n_jobs;  // first grouped row, rows; job count
  int max_jobs;
  int *cnt_out;                 // [E] statistics
  unsigned long long *stats;
  int *last;
  int *status;
};

// Down each expert's column of block masks (block order = token order, so
// rows stay in ascending t): every block's first row relative to the
// expert's first row (boff), and the expert's token count (eoff[e], turned
// into the expert's first row by prefill_scan_kernel).  A CTA takes 32
// experts (one per lane) and one of gridDim.y contiguous ranges of blocks,
// its 16 warps contiguous sub-ranges.  With more than one range,
// prefill_colcount_kernel has left each range's counts in col_part, and a
// range starts from the sum of the earlier ranges' counts.
constexpr int kPfColWarps = 16, kPfColSplitMax = 32;

MOE_DEV void colscan_range(const PfScanParams &p, int *b0_out, int *b1_out) {
  const int per_s = (p.blocks + gridDim.y - 1) / gridDim.y;
  *b0_out = min(p.blocks, (int)blockIdx.y * per_s);
  *b1_out = min(p.blocks, *b0_out + per_s);
}

__global__ void __launch_bounds__(kPfColWarps * 32) prefill_colcount_kernel(PfScanParams p) {
  __shared__ int s_part[kPfColWarps][33];
  pdl_wait();
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int e = blockIdx.x * 32 + lane;
  int sb0, sb1;
  colscan_range(p, &sb0, &sb1);
  const int per = (sb1 - sb0 + kPfColWarps - 1) / kPfColWarps;
  const int b0 = min(sb1, sb0 + wid * per), b1 = min(sb1, b0 + per);
  int run = 0;
  if (e < p.E) {
#pragma unroll 8
    for (int b = b0; b < b1; ++b) run += __popc(p.bmask[(long long)b * p.E + e]);
  }
  s_part[wid][lane] = run;
  __syncthreads();
  if (wid == 0 && e < p.E) {
    int tot = 0;
    for (int w = 0; w < kPfColWarps; ++w) tot += s_part[w][lane];
    p.col_part[(long long)blockIdx.y * p.E + e] = tot;
  }
  pdl_launch_dependents();
}

__global__ void __launch_bounds__(kPfColWarps * 32) prefill_colscan_kernel(PfScanParams p) {
  __shared__ int s_part[kPfColWarps][33];
  pdl_wait();
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int e = blockIdx.x * 32 + lane;
  int sb0, sb1;
  colscan_range(p, &sb0, &sb1);
  const int per = (sb1 - sb0 + kPfColWarps - 1) / kPfColWarps;
  const int b0 = min(sb1, sb0 + wid * per), b1 = min(sb1, b0 + per);
  int run = 0;
  if (e < p.E) {
#pragma unroll 8
    for (int b = b0; b < b1; ++b) run += __popc(p.bmask[(long long)b * p.E + e]);
  }
  s_part[wid][lane] = run;
  __syncthreads();
  int base = 0;
  if (e < p.E)
    for (int s = 0; s < (int)blockIdx.y; ++s) base += p.col_part[(long long)s * p.E + e];
  for (int w = 0; w < wid; ++w) base += s_part[w][lane];
  if (e < p.E) {
    for (int b = b0; b < b1; ++b) {
      p.boff[(long long)b * p.E + e] = base;
      base += __popc(p.bmask[(long long)b * p.E + e]);
    }
    // the last range's last warp: all blocks, the expert's tokens
    if (wid == kPfColWarps - 1 && blockIdx.y == gridDim.y - 1) p.eoff[e] = base;
  }
  pdl_launch_dependents();
}

// One CTA of 1024 threads: block scans over the experts' token counts give
// their first rows, their first GEMM tiles and their first GEMV jobs; then
// the tile and job lists, with the residency lookup.  An expert with at
// least hot_min tokens is a GEMM expert (256-row tiles); one with fewer is
// cut into GEMV jobs of at most `chunk` tokens, which stream its weights
// once per job instead of dequantising a mostly empty tile.
__global__ void __launch_bounds__(1024) prefill_scan_kernel(PfScanParams p) {
  __shared__ int s_cnt[3 * kPfMaxE + 3];
  __shared__ int s_red[32];
  __shared__ unsigned long long s_hm[3];
  pdl_wait();
  const int tid = threadIdx.x;
  int *cnt = s_cnt, *tl = s_cnt + kPfMaxE + 1, *jl = s_cnt + 2 * kPfMaxE + 2;
  if (tid < 3) s_hm[tid] = 0;
  for (int e = tid; e < p.E; e += blockDim.x) {
    const int run = p.eoff[e];  // token count from prefill_colscan_kernel
    const bool hot = run >= p.hot_min;
    cnt[e] = run;
    tl[e] = hot ? (run + kPfTileRows - 1) / kPfTileRows : 0;
    jl[e] = hot ? 0 : (run + p.chunk - 1) / p.chunk;
  }
  block_exclusive_scan(cnt, cnt, p.E, s_red);
  block_exclusive_scan(tl, tl, p.E, s_red);
  block_exclusive_scan(jl, jl, p.E, s_red);
  const int routed_tiles = tl[p.E], P = cnt[p.E], n_jobs = jl[p.E];
  const int shared_tiles = p.shared ? (p.T + kPfTileRows - 1) / kPfTileRows : 0;
  if (routed_tiles + shared_tiles > p.max_tiles || n_jobs > p.max_jobs) {
    if (tid == 0) {
      atomicOr(p.status, kErrJobOverflow);
      *p.n_tiles = 0;
      *p.n_jobs = 0;
    }
    return;
  }
  for (int e = tid; e < p.E; e += blockDim.x) {
    p.eoff[e] = cnt[e];
    const int n = cnt[e + 1] - cnt[e];
    const bool hot = n >= p.hot_min;
    p.cnt_out[e] = n;
    p.hot[e] = hot;
    if (!n) continue;
    const int slot = p.slot_of ? p.slot_of[(long long)p.layer * p.E + e] : -1;
    const bool hit = slot >= 0 && slot < p.n_slots;
    if (!hit && slot >= p.n_slots) atomicOr(p.status, kErrBadSlot);
    const uint8_t *ptr = hit ? p.pool + (long long)slot * p.expert_bytes
                             : p.arena + ((long long)p.layer * p.E + e) * p.expert_bytes;
    atomicAdd(&s_hm[hit ? 0 : 1], (unsigned long long)n);
    atomicAdd(&s_hm[2], 1ull);
    if (hot) {
      for (int m = 0, ti = tl[e]; m < n; m += kPfTileRows, ++ti) {
        p.tiles[ti].w = ptr;
        p.tiles[ti].row0 = cnt[e] + m;
        p.tiles[ti].rows = min(kPfTileRows, n - m);
      }
    } else {
      for (int m = 0, j = jl[e]; m < n; m += p.chunk, ++j) {
        p.job_ptr[j] = (unsigned long long)ptr;
        p.job_beg[j] = cnt[e] + m;
        p.job_n[j] = min(p.chunk, n - m);
      }
    }
  }
  if (tid == 0) p.eoff[p.E] = P;
  for (int q = tid; q < shared_tiles; q += blockDim.x) {
    p.tiles[routed_tiles + q].w = p.shared;
    p.tiles[routed_tiles + q].row0 = P + q * kPfTileRows;
    p.tiles[routed_tiles + q].rows = min(kPfTileRows, p.T - q * kPfTileRows);
  }
  __syncthreads();
  if (tid == 0) {
    *p.n_tiles = routed_tiles + shared_tiles;
    *p.n_jobs = n_jobs;
    atomicAdd(&p.stats[0], 1ULL);
    atomicAdd(&p.stats[1], (unsigned long long)p.T);
    atomicAdd(&p.stats[2], s_hm[0]);
    atomicAdd(&p.stats[3], s_hm[1]);
    p.last[0] = p.T;
    p.last[1] = (int)s_hm[2];
    p.last[2] = p.layer;
  }
  pdl_launch_dependents();
}

struct PfScatterParams {
  const int *idx;               // [T, k]
  const unsigned short *bmask;  // [blocks][E]
  const int *boff, *eoff;
  const uint16_t *h;            // bf16 [T, d]
  int T, E, k, d, has_shared;
  int *row_of;                  // [T*k + T]: grouped row of pair (shared pair P + t);
                                // ~pair (negative) for a pair of a GEMV expert
  __half *hg;                   // fp16 [rows][d] grouped A matrix (rows of GEMM experts)
  int *perm;                    // [T*k] or null: pair id of each routed grouped row
  const int *hot;               // [E] or null (null: every expert is a GEMM expert)
};

// One warp per token: its k pairs (and its shared-expert pair) get their
// grouped rows, and the token's row is copied (fp16, saturating) to each.
// blockIdx.y splits the row's columns (small chunks: more CTAs); the CTAs
// with blockIdx.y == 0 write the row map and the permutation.
// With perm set, the routed rows' pair ids are also written in grouped
// order: the bucket permutation (each expert's pairs in ascending t).
__global__ void __launch_bounds__(kPfTok * 32) prefill_scatter_kernel(PfScatterParams p) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  pdl_wait();
  const int t = blockIdx.x * kPfTok + wid;
  if (t >= p.T) return;
  const int P = p.T * p.k;
  int rows[33];
  unsigned long long copy = 0;  // bit j: row j feeds the GEMM (its A row is needed)
  const int nr = p.k + (p.has_shared ? 1 : 0);
  for (int j = 0; j < p.k; ++j) {
    const int e = __ldg(p.idx + (long long)t * p.k + j);
    const unsigned m = p.bmask[(long long)blockIdx.x * p.E + e];
    const int rank = __popc(m & ((1u << wid) - 1u));
    rows[j] = p.eoff[e] + p.boff[(long long)blockIdx.x * p.E + e] + rank;
    if (!p.hot || p.hot[e]) copy |= 1ull << j;
  }
  if (p.has_shared) {
    rows[p.k] = P + t;
    copy |= 1ull << p.k;
  }
  if (lane < p.k && blockIdx.y == 0) {
    const int q = t * p.k + lane;
    p.row_of[q] = (copy >> lane) & 1 ? rows[lane] : ~q;
    // the bucket permutation: grouped row -> pair id (rows < P are routed)
    if (p.perm) p.perm[rows[lane]] = q;
  }
  if (lane == 0 && p.has_shared && blockIdx.y == 0) p.row_of[P + t] = P + t;
  // copy the token row's column slice to every destination, 8 elements per
  // lane per step
  const uint4 *src = reinterpret_cast<const uint4 *>(p.h + (long long)t * p.d);
  const int n8 = p.d / 8, per = (n8 + gridDim.y - 1) / gridDim.y;
  const int i0 = blockIdx.y * per, i1 = min(n8, i0 + per);
  for (int i = i0 + lane; i < i1; i += 32) {
    const uint4 v = __ldg(src + i);
    const uint32_t in[4] = {v.x, v.y, v.z, v.w};
    uint32_t out[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float lo = __uint_as_float(in[q] << 16), hi = __uint_as_float(in[q] & 0xFFFF0000u);
      uint32_t r;
      asm("cvt.rn.satfinite.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
      out[q] = r;
    }
    const uint4 o = make_uint4(out[0], out[1], out[2], out[3]);
    for (int j = 0; j < nr; ++j)
      if ((copy >> j) & 1) reinterpret_cast<uint4 *>(p.hg + (long long)rows[j] * p.d)[i] = o;
  }
  pdl_launch_dependents();
}

// ------------------------------------------------------------ router GEMM
// logits[t, e] = sum_i W[e, i] h[t, i] (+ b[e]) for a whole chunk, fp32 FMA
// (routing decisions are compared bit-exactly, so no reduced-precision
// tensor-core path).  Small chunks split the reduction over blockIdx.z
// (columns [z kchunk, (z+1) kchunk)) so the grid fills the GPU; each split
// writes its partial sums, which router_sum_kernel adds in split order.
// CTA tile: 128 tokens x 128 experts, 256 threads, each
// an 8 x 8 block of outputs made of two 4-row and two 4-column halves 64
// apart (so a warp's 16-byte shared-memory reads are contiguous: no bank
// conflicts); the reduction walks i in order, 16 at a time through shared
// memory (h converted from bf16 on the way in).
struct RouterGemmParams {
  const uint16_t *h;   // bf16 [T, d]
  const float *W;      // fp32 [E, d]
  const float *bias;   // [E] or null
  int T, d, E;
  float *logits;       // [T, E]; with gridDim.z > 1 partial sums [gridDim.z][T][E], no bias
  int kchunk;          // reduction columns of one CTA (blockIdx.z); d when unsplit
};

constexpr int kRgBM = 128, kRgBN = 128, kRgBK = 16;

__global__ void __launch_bounds__(256) router_gemm_kernel(RouterGemmParams p) {
  __shared__ __align__(16) float As[2][kRgBK][kRgBM + 4];
  __shared__ __align__(16) float Ws[2][kRgBK][kRgBN + 4];
  pdl_wait();
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  const int t0 = blockIdx.x * kRgBM, e0 = blockIdx.y * kRgBN;
  // loaders: thread -> (row = tid / 2, 8 columns at (tid % 2) * 8)
  const int lr = tid >> 1, lc = (tid & 1) * 8;
  const int ta = t0 + lr, ew = e0 + lr;
  float acc[8][8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;
  auto load = [&](int k0, uint4 &hv, float4 &w0, float4 &w1) {
    hv = ta < p.T ? __ldg(reinterpret_cast<const uint4 *>(p.h + (long long)ta * p.d + k0 + lc))
                  : make_uint4(0u, 0u, 0u, 0u);
    if (ew < p.E) {
      const float4 *wp = reinterpret_cast<const float4 *>(p.W + (long long)ew * p.d + k0 + lc);
      w0 = __ldg(wp);
      w1 = __ldg(wp + 1);
    } else {
      w0 = w1 = make_float4(0.f, 0.f, 0.f, 0.f);
    }
  };
  auto store = [&](int buf, const uint4 &hv, const float4 &w0, const float4 &w1) {
    const uint32_t hw[4] = {hv.x, hv.y, hv.z, hv.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      As[buf][lc + 2 * q][lr] = __uint_as_float(hw[q] << 16);
      As[buf][lc + 2 * q + 1][lr] = __uint_as_float(hw[q] & 0xFFFF0000u);
    }
    const float wv[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
#pragma unroll
    for (int q = 0; q < 8; ++q) Ws[buf][lc + q][lr] = wv[q];
  };
  uint4 hv;
  float4 w0, w1;
  const int kbase = blockIdx.z * p.kchunk;
  load(kbase, hv, w0, w1);
  store(0, hv, w0, w1);
  __syncthreads();
  const int nk = p.kchunk / kRgBK;
  for (int kt = 0; kt < nk; ++kt) {
    const int buf = kt & 1;
    if (kt + 1 < nk) load(kbase + (kt + 1) * kRgBK, hv, w0, w1);
#pragma unroll
    for (int k = 0; k < kRgBK; ++k) {
      const float4 a0 = *reinterpret_cast<const float4 *>(&As[buf][k][ty * 4]);
      const float4 a1 = *reinterpret_cast<const float4 *>(&As[buf][k][64 + ty * 4]);
      const float4 b0 = *reinterpret_cast<const float4 *>(&Ws[buf][k][tx * 4]);
      const float4 b1 = *reinterpret_cast<const float4 *>(&Ws[buf][k][64 + tx * 4]);
      const float a[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
      const float b[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    if (kt + 1 < nk) store(buf ^ 1, hv, w0, w1);
    __syncthreads();
  }
  pdl_launch_dependents();
  const bool split = gridDim.z > 1;
  float *out = p.logits + (long long)blockIdx.z * p.T * p.E;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int t = t0 + (i < 4 ? ty * 4 + i : 64 + ty * 4 + i - 4);
    if (t >= p.T) continue;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int e = e0 + (j < 4 ? tx * 4 + j : 64 + tx * 4 + j - 4);
      if (e < p.E) out[(long long)t * p.E + e] = acc[i][j] + (!split && p.bias ? p.bias[e] : 0.f);
    }
  }
}

// ---------------------------------------------------------- tcgen05 helpers
// Shared-memory matrix descriptor (sm_100): start address >> 4 in bits
// [0,14), leading byte offset >> 4 in [16,30), stride byte offset >> 4 in
// [32,46), descriptor version 1 in [46,48), layout in [61,64) (2 = 128-byte
// swizzle).  A K-major tile of rows x 64 fp16 with 128-byte swizzle: rows of
// 128 B, 8-row groups 1024 B apart (SBO); LBO is unused.
MOE_DEV uint64_t umma_desc_sw128(uint32_t saddr) {
  return (uint64_t)((saddr >> 4) & 0x3FFF) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
         ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

// Instruction descriptor of kind::f16: D fp32 (bits 4-5 = 1), A and B fp16
// (bits 7-9, 10-12 = 0), both K-major, N >> 3 in [17,23), M >> 4 in [24,29).
constexpr uint32_t umma_idesc_f16(int M, int N) {
  return (1u << 4) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

MOE_DEV void umma_f16(uint32_t tmem_d, uint64_t da, uint64_t db, uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(tmem_d),
      "l"(da), "l"(db), "r"(idesc), "r"(accumulate));
}
// Arrive on an mbarrier once every tcgen05 operation this thread issued so far
// has completed.
MOE_DEV void umma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
               : "memory");
}
MOE_DEV void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
MOE_DEV void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// 32 TMEM columns of this warp's 32 lanes (thread i = lane 32 (warp % 4) + i)
MOE_DEV void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
        "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
        "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),
        "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// The same 32 columns, issued without waiting: the registers hold the data
// only after tmem_ld32_wait on them (which names them as operands, so no
// use can move above the wait).
#define MOE_R32(r)                                                                                         \
  "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),        \
      "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15]), \
      "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]), "+r"(r[22]),          \
      "+r"(r[23]), "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]), "+r"(r[29]),          \
      "+r"(r[30]), "+r"(r[31])
MOE_DEV void tmem_ld32_issue(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
        "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
        "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),
        "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}
MOE_DEV void tmem_ld32_wait(uint32_t (&r)[32]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;" : MOE_R32(r)::"memory");
}

// 2-D TMA tile load (x = element offset along the contiguous dimension, y = row)
MOE_DEV void tma_load_2d(uint32_t dst, const CUtensorMap *map, int x, int y, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
          dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
      : "memory");
}

MOE_DEV uint32_t h2_dup(uint32_t v, bool hi) {  // (h, h) from one fp16 half of v
  const uint32_t h = hi ? (v >> 16) : (v & 0xFFFFu);
  return h | (h << 16);
}
MOE_DEV uint32_t hsub2(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}
MOE_DEV uint32_t hmul2(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}
MOE_DEV uint32_t hfma2(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t r;
  asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(c));
  return r;
}

// One code-word pair of a k-step pair: rows r0 (fp16 halves at nibble bits
// 0/16 and 8/24) and r1 (bits 4/20 and 12/28), columns kb .. kb+7 from words
// wa (kb .. kb+3) and wb (kb+4 .. kb+7).
MOE_DEV void dq_pair(uint32_t wa, uint32_t wb, uint32_t s0, uint32_t s1, uint4 &row0, uint4 &row1) {
  const uint32_t c1032 = 0x64086408u, c72 = 0x54805480u;  // fp16 1032.0, 72.0
  const uint32_t a8 = wa >> 8, b8 = wb >> 8;
  row0.x = hmul2(hsub2(lop3_and_or(wa, 0x000F000Fu, 0x64006400u), c1032), s0);
  row0.y = hmul2(hsub2(lop3_and_or(a8, 0x000F000Fu, 0x64006400u), c1032), s0);
  row0.z = hmul2(hsub2(lop3_and_or(wb, 0x000F000Fu, 0x64006400u), c1032), s0);
  row0.w = hmul2(hsub2(lop3_and_or(b8, 0x000F000Fu, 0x64006400u), c1032), s0);
  row1.x = hmul2(hsub2(lop3_and_or(wa, 0x00F000F0u, 0x54005400u), c72), s1);
  row1.y = hmul2(hsub2(lop3_and_or(a8, 0x00F000F0u, 0x54005400u), c72), s1);
  row1.z = hmul2(hsub2(lop3_and_or(wb, 0x00F000F0u, 0x54005400u), c72), s1);
  row1.w = hmul2(hsub2(lop3_and_or(b8, 0x00F000F0u, 0x54005400u), c72), s1);
}

// Dequantise the four code words of one lane (g, tig) of a repacked Q4 tile
// into the swizzled fp16 B tile.  Word st of the lane holds reduction columns
// kb_step(st, tig) .. +3 of rows r0 = 16 rb + g and r0 + 8, so words 0 and 1
// fill 16-byte chunk tig of both rows (group 0) and words 2 and 3 chunk
// 4 + tig (group 1); sc holds the rows' scales of the two groups.  Lanes
// with odd g store their group-1 chunk first: in each store instruction the
// eight lanes of a wavefront (rows g, g+1 of one tile, tig 0..3) then cover
// all eight swizzled 16-byte positions of the 128-byte bank window.
MOE_DEV void dequant_q4_lane(uint4 w, uint2 sc, uint32_t dst_s, int r0, int g, int tig) {
  const int r1 = r0 + 8;
  const uint32_t base0 = dst_s + (uint32_t)(r0 >> 3) * 1024 + (uint32_t)(r0 & 7) * 128;
  const uint32_t base1 = dst_s + (uint32_t)(r1 >> 3) * 1024 + (uint32_t)(r1 & 7) * 128;
  uint4 a0, b0, a1, b1;
  dq_pair(w.x, w.y, h2_dup(sc.x, false), h2_dup(sc.x, true), a0, b0);  // group 0
  dq_pair(w.z, w.w, h2_dup(sc.y, false), h2_dup(sc.y, true), a1, b1);  // group 1
  const bool odd = g & 1;
  const uint32_t cf = (uint32_t)((odd ? 4 : 0) + tig), cs = (uint32_t)((odd ? 0 : 4) + tig);
  const uint4 f0 = odd ? a1 : a0, s0 = odd ? a0 : a1, f1 = odd ? b1 : b0, s1 = odd ? b0 : b1;
  asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(base0 + ((cf ^ (r0 & 7)) << 4)),
               "r"(f0.x), "r"(f0.y), "r"(f0.z), "r"(f0.w) : "memory");
  asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(base0 + ((cs ^ (r0 & 7)) << 4)),
               "r"(s0.x), "r"(s0.y), "r"(s0.z), "r"(s0.w) : "memory");
  asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(base1 + ((cf ^ (r1 & 7)) << 4)),
               "r"(f1.x), "r"(f1.y), "r"(f1.z), "r"(f1.w) : "memory");
  asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(base1 + ((cs ^ (r1 & 7)) << 4)),
               "r"(s1.x), "r"(s1.y), "r"(s1.z), "r"(s1.w) : "memory");
}

// Q2 codes of one k-step half of a repacked tile into the swizzled fp16 B
// tile.  A Q2 tile spans 128 reduction columns, two groups of 64; half h of
// it is group h and sits in words 2h and 2h+1 of each lane (g, tig): word
// 2h holds rows r0 = 16 rb + g and r0 + 8 at reduction columns
// [8 tig, 8 tig + 8) of the half (16-byte chunk tig of both rows), word
// 2h + 1 the same rows at chunk 4 + tig.  In a word, fragment register r
// (r = 0..7) holds columns 2 (r >> 1) and 2 (r >> 1) + 1 -- row r0 for even
// r, r0 + 8 for odd r -- at bits [2r, 2r + 2) and [16 + 2r, 18 + 2r).  A code
// q placed at mantissa bit p of fp16 1024 gives 1024 + q 2^p; subtracting
// 1024 is exact, and one fp16 FMA with s 2^-p (exact) and the min gives
// s q + m, rounded once.  s and mn hold the group's (row r0, row r0 + 8)
// fp16 scales and mins.  Stores as in dequant_q4_lane.
MOE_DEV void dq_q2_word(uint32_t w, uint32_t sa, uint32_t sb, uint32_t ma, uint32_t mb, uint4 &row0,
                        uint4 &row1) {
  const uint32_t c1024 = 0x64006400u;
  const uint32_t w4 = w >> 4, w8 = w >> 8, w12 = w >> 12;
  // row r0: codes at p = 0 of w, w >> 4, w >> 8, w >> 12; row r1: p = 2
  row0.x = hfma2(hsub2(lop3_and_or(w, 0x00030003u, c1024), c1024), sa, ma);
  row0.y = hfma2(hsub2(lop3_and_or(w4, 0x00030003u, c1024), c1024), sa, ma);
  row0.z = hfma2(hsub2(lop3_and_or(w8, 0x00030003u, c1024), c1024), sa, ma);
  row0.w = hfma2(hsub2(lop3_and_or(w12, 0x00030003u, c1024), c1024), sa, ma);
  row1.x = hfma2(hsub2(lop3_and_or(w, 0x000C000Cu, c1024), c1024), sb, mb);
  row1.y = hfma2(hsub2(lop3_and_or(w4, 0x000C000Cu, c1024), c1024), sb, mb);
  row1.z = hfma2(hsub2(lop3_and_or(w8, 0x000C000Cu, c1024), c1024), sb, mb);
  row1.w = hfma2(hsub2(lop3_and_or(w12, 0x000C000Cu, c1024), c1024), sb, mb);
}

MOE_DEV void dequant_q2_lane(uint2 w, uint32_t s, uint32_t mn, uint32_t dst_s, int r0, int g, int tig) {
  const int r1 = r0 + 8;
  const uint32_t base0 = dst_s + (uint32_t)(r0 >> 3) * 1024 + (uint32_t)(r0 & 7) * 128;
  const uint32_t base1 = dst_s + (uint32_t)(r1 >> 3) * 1024 + (uint32_t)(r1 & 7) * 128;
  const uint32_t sa = h2_dup(s, false), sb = hmul2(h2_dup(s, true), 0x34003400u);  // s_r1 / 4
  const uint32_t ma = h2_dup(mn, false), mb = h2_dup(mn, true);
  uint4 a0, b0, a1, b1;
  dq_q2_word(w.x, sa, sb, ma, mb, a0, b0);  // chunk tig
  dq_q2_word(w.y, sa, sb, ma, mb, a1, b1);  // chunk 4 + tig
  const bool odd = g & 1;
  const uint32_t cf = (uint32_t)((odd ? 4 : 0) + tig), cs = (uint32_t)((odd ? 0 : 4) + tig);
  const uint4 f0 = odd ? a1 : a0, s0 = odd ? a0 : a1, f1 = odd ? b1 : b0, s1 = odd ? b0 : b1;
  asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(base0 + ((cf ^ (r0 & 7)) << 4)),
               "r"(f0.x), "r"(f0.y), "r"(f0.z), "r"(f0.w) : "memory");
  asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(base0 + ((cs ^ (r0 & 7)) << 4)),
               "r"(s0.x), "r"(s0.y), "r"(s0.z), "r"(s0.w) : "memory");
  asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(base1 + ((cf ^ (r1 & 7)) << 4)),
               "r"(f1.x), "r"(f1.y), "r"(f1.z), "r"(f1.w) : "memory");
  asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(base1 + ((cs ^ (r1 & 7)) << 4)),
               "r"(s1.x), "r"(s1.y), "r"(s1.z), "r"(s1.w) : "memory");
}

// ------------------------------------------------------- CTA-pair helpers
// The grouped GEMM runs on clusters of two CTAs (a CTA pair on two SMs) that
// issue one tcgen05.mma.cta_group::2 per 16-column step: the pair's MMA is
// m256n256k16, each CTA holding 128 of the A rows and 128 of the B rows in
// its own shared memory (at the same offsets) and 128 accumulator rows in its
// own TMEM.  Per SM that halves the shared-memory bytes per FLOP of the
// one-CTA m128n128 form.
MOE_DEV uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
MOE_DEV uint32_t cluster_id_x() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%clusterid.x;" : "=r"(r));
  return r;
}
MOE_DEV uint32_t cluster_count_x() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%nclusterid.x;" : "=r"(r));
  return r;
}
// shared::cluster address of the variable at shared::cta address `a` in the
// cluster's CTA `rank`
MOE_DEV uint32_t mapa_shared(uint32_t a, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(rank));
  return r;
}
// All threads of both CTAs; orders everything before it (release) against
// everything after it (acquire) across the pair.
MOE_DEV void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// One arrival on an mbarrier of either CTA of the pair (shared::cluster
// address), with the instruction's default release semantics.  Waits on the
// pair's barriers use the ordinary try_wait: the tensor-core and TMA
// pipelines of the pair synchronise this way, and the release/acquire forms
// at cluster scope made every step of this kernel a third slower.
MOE_DEV void mbar_arrive_remote(uint32_t bar_cl) {
  asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(bar_cl) : "memory");
}
// 2-D TMA tile load into this CTA's shared memory whose completion is
// counted on an mbarrier of either CTA of the pair (bar_cl: shared::cluster
// address).  No multicast: the tile lands in this CTA only.
MOE_DEV void tma_load_2d_pair(uint32_t dst, const CUtensorMap *map, int x, int y, uint32_t bar_cl) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, "
      "%3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar_cl)
      : "memory");
}
// 2-D TMA tile store from this CTA's shared memory (bulk-group completion).
MOE_DEV void tma_store_2d(const CUtensorMap *map, uint32_t src, int x, int y) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(src), "r"(x), "r"(y)
               : "memory");
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// 3-D TMA tile store from this CTA's shared memory (bulk-group completion).
MOE_DEV void tma_store_3d(const CUtensorMap *map, uint32_t src, int x, int y, int z) {
  asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(src), "r"(x), "r"(y), "r"(z)
               : "memory");
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// Wait until at most N of this thread's bulk groups still read shared memory.
template <int N>
MOE_DEV void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
// Wait until all of this thread's bulk groups are complete.
MOE_DEV void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// The pair's MMA, issued by one thread of the even CTA: D (both CTAs' TMEM at
// tmem_d) (+)= A (both CTAs' shared memory at da) x B (both at db)^T.
MOE_DEV void umma_f16_pair(uint32_t tmem_d, uint64_t da, uint64_t db, uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(tmem_d),
      "l"(da), "l"(db), "r"(idesc), "r"(accumulate));
}
// One arrival on the mbarrier at shared::cta offset `bar` in both CTAs of the
// pair once every tcgen05 operation this thread issued has completed.
MOE_DEV void umma_commit_pair(uint32_t bar) {
  const uint16_t both = 3;
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(bar),
      "h"(both)
      : "memory");
}

struct PfGemmParams {
  const PfTile *tiles;
  const int *n_tiles;
  int K;                 // reduction (d for gate/up, f for down)
  int N;                 // output features (f for gate/up, d for down)
  int ntile_k;           // repacked tiles along K: K / 64 (Q4) or K / 128 (Q2)
  long long region_off;  // 0 (gate/up) or the down region's offset
  __half *out_a;         // gate/up: SiLU(G) * U, fp16 [rows][N]
  __half *out_y;         // down: y, fp16 (round to nearest, saturating) [rows][N]
  int *status;
};

constexpr int kPfGemmThreads = 512;  // 16 warps
constexpr int kPfOutRows = 32, kPfOutCols = 32;  // epilogue TMA store box (one warp's rows x 64 B)
constexpr uint32_t kPfOutStage = kPfOutRows * kPfOutCols * 2;  // 2 KB
constexpr int kPfDeqWarp0 = 8;       // warps 8..15 dequantise
constexpr int kPfEpiWarp0 = 4;       // warps 4..7 drain the accumulators (TMEM lane quarters 0..3)

// A work item is one tile of up to 256 rows of one expert times one output
// slice: 128 features of the gate/up pass or 256 features of the down pass.
// Each CTA dequantises 128 weight rows of the slice -- gate/up: the gate and
// up rows of 64 features (the even CTA features [0, 64) of the slice, the odd
// CTA [64, 128)); down: 128 output features -- and holds 128 of the tile's
// rows: the even CTA rows [0, 128), the odd CTA rows [128, 256).  The pair's
// accumulator columns are then [gate | up] of the even CTA's 64 features and
// [gate | up] of the odd CTA's (gate/up), or the slice's 256 features in
// order (down).  Per step of 128 reduction columns each CTA loads its A tile
// (32 KB) and dequantises its 128 weight rows (32 KB of fp16) once for all
// 256 token rows.  The A tiles and the code tiles travel in two rings: an A
// stage is released when the pair's MMAs complete, a code stage when the
// CTA's dequantising warps have read it.  A code stage holds CT consecutive
// repacked tiles of each of the CTA's row blocks (two steps): the tiles of a
// row block along the reduction are contiguous in memory (gate/up: gate and
// up tile of each column side by side), so one bulk copy per row block fills
// it -- issuing a copy costs the producer about 100 cycles, and one copy per
// tile (8 per 64 columns) was the pipeline's bottleneck.
template <int FMT>
struct PfCfg {
  static constexpr int TILE = FMT == 1 ? 576 : 640;         // repacked code tile (+ scales)
  static constexpr int APT = FMT == 1 ? 1 : 2;              // 64-column atoms per tile (64 / 128 columns)
  static constexpr int CT = FMT == 1 ? 4 : 2;               // tiles per row block per code stage
  static constexpr int APC = CT * APT;                      // atoms per code stage (4: two steps)
  static constexpr int SA = 3;                              // A ring (stages of one step)
  static constexpr int SC = FMT == 1 ? 2 : 3;               // code ring
  static constexpr int NBB = 2;                             // B buffers (dequantised weights of one step)
  static constexpr int NB_ROWS = 128;                       // weight rows per CTA per item
  static constexpr uint32_t ATOM_A = kPfBM * kPfBK * 2;     // 16 KB: this CTA's 128 rows x 64 columns
  static constexpr uint32_t TILE_A = 2 * ATOM_A;            // one step: 128 columns
  static constexpr uint32_t ATOM_B = NB_ROWS * kPfBK * 2;   // 16 KB
  static constexpr uint32_t BBUF = 2 * ATOM_B;              // one step
  static constexpr uint32_t CODES = (8 * CT * TILE + 1023) / 1024 * 1024;  // 8 row blocks x CT tiles
  static constexpr uint32_t OUT = 4 * 2 * kPfOutStage;       // epilogue staging: 2 per epilogue warp
  static constexpr uint32_t SMEM = SA * TILE_A + SC * CODES + NBB * BBUF + OUT + 1024;  // + alignment slack
  static constexpr uint32_t ACC_COLS = 2 * NB_ROWS;         // TMEM columns per buffer (MMA N = 256)
  static constexpr uint32_t TMEM_COLS = 2 * ACC_COLS;       // double buffered: all 512
};

// Grouped GEMM over the tile list, warp-specialised, on CTA pairs; the
// persistent pairs walk the items clusterid.x, +nclusterid.x.  Both CTAs:
//  warp 0 lane 0   A producer: per step (128 reduction columns, two 64-column
//                  atoms) this CTA's A tile (two 2-D TMA boxes, 128-byte
//                  swizzle; the odd CTA only when the tile has more than 128
//                  rows) into a free stage of the A ring, counted on the even
//                  CTA's stage barrier
//  warp 2 lane 0   code producer: every two steps the next code stage (one
//                  1-D bulk copy per row block) into the code ring; apart
//                  from the A producer so that neither ring waits on the other
//  warps 8..15     one row block each: dequantise a step's codes into one of
//                  two swizzled fp16 B buffers, arrive on the even CTA's
//                  buffer barrier, release the code stage after its last step
//  warps 4..7      drain an accumulator buffer (TMEM lanes = the CTA's rows)
//                  while the next item accumulates into the other one, then
//                  arrive on the even CTA's buffer-empty barrier
// Even CTA only:
//  warp 1 lane 0   issues the pair's MMAs (8 x m256n256k16 per step, fp32 in
//                  TMEM) and commits the release of the A stage, the B buffer
//                  and the accumulator to the barriers of both CTAs
// A step of 128 columns (rather than one 64-column atom) halves the barrier
// waits and commits per MMA: the issuing thread's per-wait overhead left the
// tensor pipe idle between atoms.
// Every wait is bounded; a timeout raises kErrTimeout and stops both CTAs.
template <int FMT, bool GATED>
__global__ void __launch_bounds__(kPfGemmThreads, 1)
    prefill_gemm_kernel(const __grid_constant__ CUtensorMap amap, const __grid_constant__ CUtensorMap omap,
                        PfGemmParams p) {
  using C = PfCfg<FMT>;
  constexpr int SA = C::SA, SC = C::SC, APT = C::APT, CT = C::CT, APC = C::APC, TILE = C::TILE,
                NBB = C::NBB;
  constexpr int SPS = APC / 2;  // steps per code stage
  constexpr int COLS = GATED ? C::NB_ROWS : 2 * C::NB_ROWS;  // output features per item
  extern __shared__ __align__(128) unsigned char pf_smem[];  // stages start at the next 1024 B
  __shared__ __align__(8) unsigned long long s_afull[SA], s_aempty[SA], s_cfull[SC], s_cempty[SC],
      s_bfull[NBB], s_bempty[NBB], s_accf[2], s_acce[2];
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort;
  const int tid = threadIdx.x, wid = tid >> 5, lane = tid & 31;
  const uint32_t rank = cluster_ctarank();  // 0: the even CTA (issues the MMAs)
  const uint32_t base = smem_addr(pf_smem), stage0 = base + ((1024 - (base & 1023)) & 1023);
  if (tid == 0) {
    for (int i = 0; i < SA; ++i) {
      mbar_init(smem_addr(&s_afull[i]), 1);   // the even CTA's expect_tx; both CTAs' bytes
      mbar_init(smem_addr(&s_aempty[i]), 1);  // the pair's MMA commit
    }
    for (int i = 0; i < SC; ++i) {
      mbar_init(smem_addr(&s_cfull[i]), 1);
      mbar_init(smem_addr(&s_cempty[i]), 8);  // one arrival per dequantising warp
    }
    for (int b = 0; b < NBB; ++b) {
      mbar_init(smem_addr(&s_bfull[b]), 16);  // 8 dequantising warps of each CTA
      mbar_init(smem_addr(&s_bempty[b]), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_addr(&s_accf[b]), 1);
      mbar_init(smem_addr(&s_acce[b]), 8);  // 4 epilogue warps of each CTA
    }
    s_abort = 0;
    fence_mbar_init();
  }
  if (wid == 0) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_addr(&s_tmem)),
                 "r"(C::TMEM_COLS));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // both CTAs' barriers exist before either signals the other's
  tc_fence_after();
  const uint32_t tmem = s_tmem;
  pdl_wait();
  const int ntiles = ldcg_i32(p.n_tiles);
  const int nslices = p.N / COLS, nsteps = p.K / (2 * kPfBK);  // K is a multiple of 128
  const int items = ntiles * nslices;
  const int pair = (int)cluster_id_x(), npairs = (int)cluster_count_x();
  auto stage_a = [&](uint32_t st) { return stage0 + st * C::TILE_A; };
  auto stage_c = [&](uint32_t cs) { return stage0 + SA * C::TILE_A + cs * C::CODES; };
  auto bbuf = [&](uint32_t b) { return stage0 + SA * C::TILE_A + SC * C::CODES + b * C::BBUF; };
  const uint32_t out0 = stage0 + SA * C::TILE_A + SC * C::CODES + NBB * C::BBUF;  // 1024-aligned
  auto lead = [&](const void *v) { return mapa_shared(smem_addr(v), 0); };  // the even CTA's copy
  auto aborted = [&]() { return *reinterpret_cast<volatile int *>(&s_abort) != 0; };
  auto give_up = [&]() {  // stop both CTAs' roles
    *reinterpret_cast<volatile int *>(&s_abort) = 1;
    asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(mapa_shared(smem_addr(&s_abort), rank ^ 1u)),
                 "r"(1)
                 : "memory");
    atomicOr(p.status, kErrTimeout);
  };

  if (wid == 0) {
    // ------------------------------------------------------------ A producer
    if (lane == 0) {
      uint32_t it = 0;  // steps issued
      bool ok = true;
      for (int item = pair; item < items && ok && !aborted(); item += npairs) {
        const PfTile tile = p.tiles[item / nslices];
        const bool two = tile.rows > kPfBM;  // the odd CTA's rows exist
        const bool mine = rank == 0 || two;  // this CTA loads A rows
        for (int ks = 0; ks < nsteps; ++ks, ++it) {
          const uint32_t st = it % SA, use = it / SA;
          if (use > 0 && !mbar_wait_bounded(smem_addr(&s_aempty[st]), (use - 1) & 1)) {
            ok = false;
            break;
          }
          if (rank == 0) mbar_expect_tx(smem_addr(&s_afull[st]), two ? 2 * C::TILE_A : C::TILE_A);
          if (mine)
#pragma unroll
            for (int s = 0; s < 2; ++s)
              tma_load_2d_pair(stage_a(st) + s * C::ATOM_A, &amap, (2 * ks + s) * kPfBK,
                               tile.row0 + (int)rank * kPfBM, lead(&s_afull[st]));
        }
      }
      if (!ok) give_up();
      // no copy may land in shared memory after the pair has moved on (a
      // give-up leaves stages in flight): the even CTA's stage barriers count
      // both CTAs' A bytes; consumed stages pass at once
      if (rank == 0)
        for (uint32_t j = it > SA ? it - SA : 0; j < it; ++j)
          (void)mbar_wait_bounded(smem_addr(&s_afull[j % SA]), (j / SA) & 1);
    }
  } else if (wid == 2) {
    // ------------------------------------------------------------ code producer
    if (lane == 0) {
      uint32_t ct = 0;  // code stages issued
      bool ok = true;
      for (int item = pair; item < items && ok && !aborted(); item += npairs) {
        const PfTile tile = p.tiles[item / nslices];
        const int slice = item % nslices;
        const uint8_t *wbase = tile.w + p.region_off;
        for (int ks = 0; ks < nsteps; ks += SPS) {  // code stage: tiles tk0 .. tk0 + nt - 1
          const uint32_t cs = ct % SC, cuse = ct / SC;
          const int tk0 = 2 * ks / APT, nt = min(CT, p.ntile_k - tk0);
          if (cuse > 0 && !mbar_wait_bounded(smem_addr(&s_cempty[cs]), (cuse - 1) & 1)) {
            ok = false;
            break;
          }
          const uint32_t cbar = smem_addr(&s_cfull[cs]);
          mbar_expect_tx(cbar, 8 * nt * TILE);
          if constexpr (GATED) {
            // row block r of the CTA's 64 features: its gate and up tiles of
            // columns tk0 .. are one contiguous run
            for (int r = 0; r < 4; ++r)
              bulk_g2s(stage_c(cs) + r * 2 * CT * TILE,
                       wbase + ((long long)(slice * 8 + (int)rank * 4 + r) * p.ntile_k + tk0) * 2 * TILE,
                       2 * nt * TILE, cbar);
          } else {
            for (int q = 0; q < 8; ++q)  // row block q of the CTA's half of the slice
              bulk_g2s(stage_c(cs) + q * CT * TILE,
                       wbase + ((long long)(slice * 16 + (int)rank * 8 + q) * p.ntile_k + tk0) * TILE,
                       nt * TILE, cbar);
          }
          ++ct;
        }
      }
      if (!ok) give_up();
      for (uint32_t j = ct > SC ? ct - SC : 0; j < ct; ++j)
        (void)mbar_wait_bounded(smem_addr(&s_cfull[j % SC]), (j / SC) & 1);
    }
  } else if (wid == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && rank == 0) {
      constexpr uint32_t IDESC = umma_idesc_f16(2 * kPfBM, C::ACC_COLS);
      uint32_t it = 0, ii = 0;
      for (int item = pair; item < items && !aborted(); item += npairs, ++ii) {
        const uint32_t buf = ii & 1, acc = tmem + buf * C::ACC_COLS;
        if (ii >= 2 && !mbar_wait_bounded(smem_addr(&s_acce[buf]), ((ii >> 1) - 1) & 1)) {
          give_up();
          break;
        }
        tc_fence_after();
        bool ok = true;
        for (int ks = 0; ks < nsteps; ++ks, ++it) {
          const uint32_t st = it % SA, use = it / SA, bb = it % NBB, buse = it / NBB;
          if (!mbar_wait_bounded(smem_addr(&s_bfull[bb]), buse & 1) ||
              !mbar_wait_bounded(smem_addr(&s_afull[st]), use & 1)) {
            ok = false;
            break;
          }
          tc_fence_after();
#pragma unroll
          for (int s = 0; s < 2; ++s)
#pragma unroll
            for (int kk = 0; kk < kPfBK / 16; ++kk)
              umma_f16_pair(acc, umma_desc_sw128(stage_a(st) + s * C::ATOM_A + kk * 32),
                            umma_desc_sw128(bbuf(bb) + s * C::ATOM_B + kk * 32), IDESC, (ks | s | kk) != 0);
          umma_commit_pair(smem_addr(&s_aempty[st]));
          umma_commit_pair(smem_addr(&s_bempty[bb]));
        }
        if (!ok) {
          give_up();
          break;
        }
        umma_commit_pair(smem_addr(&s_accf[buf]));
      }
      // every committed MMA must be complete before either CTA releases TMEM
      if (it > 0) (void)mbar_wait_bounded(smem_addr(&s_aempty[(it - 1) % SA]), ((it - 1) / SA) & 1);
    }
  } else if (wid >= kPfEpiWarp0 && wid < kPfEpiWarp0 + 4) {
    // ------------------------------------------------------------ epilogue
    // A warp whose 32 rows all belong to the tile stages each 32-column
    // chunk (fp16, 64-byte swizzle: conflict-free lane stores) and writes it
    // with one TMA store, two stages in flight; rows at a tile's ragged end
    // are stored lane by lane, so no store reaches another expert's rows.
    const int quarter = wid & 3;  // TMEM lanes [32 quarter, +32) = the warp's rows of this CTA
    const uint32_t stg = out0 + (uint32_t)quarter * 2 * kPfOutStage;
    uint32_t ii = 0, ob = 0;  // items, staged stores
    for (int item = pair; item < items; item += npairs, ++ii) {
      const uint32_t buf = ii & 1;
      const bool ok = mbar_wait_bounded(smem_addr(&s_accf[buf]), (ii >> 1) & 1);
      if (__any_sync(0xffffffffu, !ok) || aborted()) {
        if (lane == 0) give_up();
        break;
      }
      tc_fence_after();
      const PfTile tile = p.tiles[item / nslices];
      const int n0 = (item % nslices) * COLS;
      const int r0 = (int)rank * kPfBM + quarter * 32;  // the warp's first row in the tile
      const int r = r0 + lane;
      const bool full = r0 + 32 <= tile.rows;  // warp-uniform
      const uint32_t lane_addr = tmem + buf * C::ACC_COLS + ((uint32_t)(quarter * 32) << 16);
      __half *const out = GATED ? p.out_a : p.out_y;
      auto emit = [&](const uint32_t (&pk)[16], int col) {
        if (full) {
          const uint32_t sb = stg + (ob & 1) * kPfOutStage;
          if (lane == 0 && ob >= 2) bulk_wait_read<1>();  // the store of two chunks ago has read its stage
          __syncwarp();
#pragma unroll
          for (int v = 0; v < 4; ++v)
            asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(sb + lane * 64 +
                                                                      ((v ^ ((lane >> 1) & 3)) << 4)),
                         "r"(pk[4 * v]), "r"(pk[4 * v + 1]), "r"(pk[4 * v + 2]), "r"(pk[4 * v + 3])
                         : "memory");
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) tma_store_2d(&omap, sb, col, tile.row0 + r0);
          ++ob;
        } else if (r < tile.rows) {
          uint4 *dst = reinterpret_cast<uint4 *>(out + (long long)(tile.row0 + r) * p.N + col);
#pragma unroll
          for (int v = 0; v < 4; ++v) dst[v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
        }
      };
      if (r0 < tile.rows) {  // warp-uniform: the warp has rows in this tile
        if constexpr (GATED) {
          // accumulator columns [128 h, 128 h + 64) = gate, [128 h + 64,
          // 128 h + 128) = up of features n0 + 64 h ..
          for (int c = 0; c < COLS; c += 32) {
            const int h = c >> 6, c0 = c & 63;
            float g[32], u[32];
            tmem_ld32(lane_addr + h * 128 + c0, g);
            tmem_ld32(lane_addr + h * 128 + 64 + c0, u);
            uint32_t pk[16];
            // SiLU(g) u with the fast divide: a is rounded to fp16 next, so
            // its few-ulp fp32 error is invisible, and the IEEE divide made
            // this epilogue as slow as the item's MMAs (for g below about
            // -88 the denominator is inf and the quotient the correct 0)
#pragma unroll
            for (int q = 0; q < 16; ++q) {
              const float a0 = __fdividef(g[2 * q], 1.0f + __expf(-g[2 * q])) * u[2 * q];
              const float a1 = __fdividef(g[2 * q + 1], 1.0f + __expf(-g[2 * q + 1])) * u[2 * q + 1];
              asm("cvt.rn.satfinite.f16x2.f32 %0, %1, %2;" : "=r"(pk[q]) : "f"(a1), "f"(a0));
            }
            emit(pk, n0 + c);
          }
        } else {
          // the next chunk's TMEM load is in flight while this one is
          // converted and stored
          uint32_t ra[32], rb[32];
          auto put = [&](const uint32_t (&r)[32], int col) {
            uint32_t pk[16];
#pragma unroll
            for (int q = 0; q < 16; ++q)
              asm("cvt.rn.satfinite.f16x2.f32 %0, %1, %2;"
                  : "=r"(pk[q])
                  : "f"(__uint_as_float(r[2 * q + 1])), "f"(__uint_as_float(r[2 * q])));
            emit(pk, col);
          };
          tmem_ld32_issue(lane_addr, ra);
          tmem_ld32_wait(ra);
          for (int c0 = 0; c0 < COLS; c0 += 64) {  // COLS is a multiple of 64
            tmem_ld32_issue(lane_addr + c0 + 32, rb);
            put(ra, n0 + c0);
            tmem_ld32_wait(rb);
            if (c0 + 64 < COLS) tmem_ld32_issue(lane_addr + c0 + 64, ra);
            put(rb, n0 + c0 + 32);
            if (c0 + 64 < COLS) tmem_ld32_wait(ra);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(lead(&s_acce[buf]));
    }
    if (lane == 0) bulk_wait_all();  // every staged store has landed before the CTA exits
  } else if (wid >= kPfDeqWarp0) {
    // ------------------------------------------------------------ dequantise
    // warp -> one row block of the CTA's 128 weight rows (gate/up: row
    // block q >> 1 of matrix q & 1, i.e. B rows (q & 1) 64 + (q >> 1) 16 ..;
    // down: row block q), lane -> the tile's lane: contiguous code reads,
    // conflict-free stores (dequant_q4_lane / dequant_q2_lane)
    const int q = wid - kPfDeqWarp0;  // 0..7
    const int brow0 = GATED ? (q & 1) * 64 + (q >> 1) * 16 : q * 16;  // B row of its row 0
    // its tiles in a code stage: tile j at tbase + j * tstep
    const uint32_t tbase = GATED ? (uint32_t)(((q >> 1) * 2 * CT + (q & 1)) * TILE) : (uint32_t)(q * CT * TILE);
    constexpr uint32_t tstep = GATED ? 2 * TILE : TILE;
    const int g = lane >> 2, tig = lane & 3;
    uint32_t it = 0, ct = 0;
    bool ok = true;
    for (int item = pair; item < items && ok; item += npairs) {
      for (int ks = 0; ks < nsteps; ++ks, ++it) {
        const uint32_t cs = ct % SC, cuse = ct / SC, bb = it % NBB, buse = it / NBB;
        bool got = mbar_wait_bounded(smem_addr(&s_cfull[cs]), cuse & 1);
        if (got && buse > 0) got = mbar_wait_bounded(smem_addr(&s_bempty[bb]), (buse - 1) & 1);
        if (__any_sync(0xffffffffu, !got) || aborted()) {
          if (lane == 0) give_up();
          ok = false;
          break;
        }
#pragma unroll
        for (int s = 0; s < 2; ++s) {  // the step's two 64-column atoms
          const int at = (2 * ks + s) % APC, half = at % APT, j = at / APT;
          const uint32_t tsm = stage_c(cs) + tbase + j * tstep, dst = bbuf(bb) + s * C::ATOM_B;
          if constexpr (FMT == 1) {
            dequant_q4_lane(lds_u4(tsm + lane * 16), lds_u2(tsm + 512 + g * 8), dst, brow0 + g, g, tig);
          } else {
            const uint4 sc = lds_u4(tsm + 512 + g * 16);
            dequant_q2_lane(lds_u2(tsm + lane * 16 + 8 * half), half ? sc.y : sc.x, half ? sc.w : sc.z, dst,
                            brow0 + g, g, tig);
          }
        }
        fence_proxy_async_smem();  // the tensor core reads B through the async proxy
        __syncwarp();
        if (lane == 0) mbar_arrive_remote(lead(&s_bfull[bb]));
        if (ks % SPS == SPS - 1 || ks == nsteps - 1) {  // the code stage's last step: release it
          if (lane == 0) mbar_arrive(smem_addr(&s_cempty[cs]));
          ++ct;
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // the pair's MMAs, remote arrivals and copies are done
  tc_fence_after();
  if (wid == 0)
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(C::TMEM_COLS));
  pdl_launch_dependents();
}

// ------------------------------------------------ router on the tensor cores
// logits[t, e] = sum_i W[e, i] h[t, i] (+ b[e]) for a whole chunk.  The fp32
// router rows are split once, exactly, into three bf16 parts W = Wh + Wm + Wl
// (8 significand bits each: router_split_kernel), and h is bf16, so the sum
// runs as one bf16 GEMM with the reduction tripled: [h | h | h] x
// [Wh | Wm | Wl]^T.  Every product is exact and the tensor core accumulates
// in fp32, so the logits keep fp32 accuracy: this is not a reduced-precision
// router.  One 128-token x 256-expert tile per CTA: warp 0 lane 0 loads the h
// and W tiles of each 64-column step by TMA (128-byte swizzle) into a 4-deep
// ring, warp 1 lane 0 issues the m128n256k16 MMAs (fp32 in TMEM), warps 4..7
// read the accumulator back and add the bias.  Every wait is bounded.
constexpr int kRtBM = 128, kRtBN = 256, kRtStages = 4;

struct RtCfg {
  static constexpr uint32_t TILE_A = kRtBM * 64 * 2;   // 16 KB
  static constexpr uint32_t TILE_B = kRtBN * 64 * 2;   // 32 KB
  static constexpr uint32_t STAGE = TILE_A + TILE_B;   // a multiple of 1024 B
  static constexpr uint32_t SMEM = kRtStages * STAGE + 1024;  // + alignment slack
};

struct RouterTcParams {
  const float *bias;  // [E] or null (null with a split reduction: router_sum_kernel adds it)
  float *logits;      // [T, E] (written through the output map)
  int T, E, d;
  int ksteps;         // 64-column reduction steps per split (blockIdx.z): 3 d / 64 / splits
  int *status;
};

// W3[e] = [Wh | Wm | Wl] (bf16, 3d per row) with W[e] = Wh + Wm + Wl exactly:
// each part is the bf16 rounding of what the parts before it left, and each
// difference is exact in fp32.
__global__ void router_split_kernel(const float *W, long long n, int d, __nv_bfloat16 *W3) {
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n;
       i += (long long)gridDim.x * blockDim.x) {
    const long long e = i / d, c = i - e * d;
    const float w = W[i];
    const __nv_bfloat16 hi = __float2bfloat16_rn(w);
    const float r1 = w - __bfloat162float(hi);
    const __nv_bfloat16 mid = __float2bfloat16_rn(r1);
    const __nv_bfloat16 lo = __float2bfloat16_rn(r1 - __bfloat162float(mid));
    __nv_bfloat16 *row = W3 + e * 3 * d;
    row[c] = hi;
    row[d + c] = mid;
    row[2 * d + c] = lo;
  }
}

// Instruction descriptor of kind::f16 with bf16 A and B (formats 1).
constexpr uint32_t umma_idesc_bf16(int M, int N) { return umma_idesc_f16(M, N) | (1u << 7) | (1u << 10); }

__global__ void __launch_bounds__(256, 1)
    router_tc_kernel(const __grid_constant__ CUtensorMap hmap, const __grid_constant__ CUtensorMap wmap,
                     const __grid_constant__ CUtensorMap lmap, RouterTcParams p) {
  using C = RtCfg;
  constexpr int S = kRtStages;
  extern __shared__ __align__(128) unsigned char rt_smem[];
  __shared__ __align__(8) unsigned long long s_full[S], s_empty[S], s_accf;
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort;
  const int tid = threadIdx.x, wid = tid >> 5, lane = tid & 31;
  const uint32_t base = smem_addr(rt_smem), stage0 = base + ((1024 - (base & 1023)) & 1023);
  if (tid == 0) {
    for (int i = 0; i < S; ++i) {
      mbar_init(smem_addr(&s_full[i]), 1);
      mbar_init(smem_addr(&s_empty[i]), 1);
    }
    mbar_init(smem_addr(&s_accf), 1);
    s_abort = 0;
    fence_mbar_init();
  }
  if (wid == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_addr(&s_tmem)),
                 "r"(kRtBN));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;
  pdl_wait();
  const int m0 = blockIdx.x * kRtBM, n0 = blockIdx.y * kRtBN;
  // this CTA's reduction steps [k0, k0 + nk) of the tripled reduction
  const int nkh = p.d / 64, nk = p.ksteps, k0 = blockIdx.z * p.ksteps;
  auto stage_a = [&](int st) { return stage0 + (uint32_t)st * C::STAGE; };
  auto stage_b = [&](int st) { return stage0 + (uint32_t)st * C::STAGE + C::TILE_A; };
  auto aborted = [&]() { return *reinterpret_cast<volatile int *>(&s_abort) != 0; };
  auto give_up = [&]() {
    *reinterpret_cast<volatile int *>(&s_abort) = 1;
    atomicOr(p.status, kErrTimeout);
  };
  if (wid == 0) {
    if (lane == 0) {  // producer
      int issued = 0;
      for (int ks = 0; ks < nk && !aborted(); ++ks) {
        const int st = ks % S, use = ks / S;
        if (use > 0 && !mbar_wait_bounded(smem_addr(&s_empty[st]), (use - 1) & 1)) {
          give_up();
          break;
        }
        const uint32_t bar = smem_addr(&s_full[st]);
        mbar_expect_tx(bar, C::STAGE);
        tma_load_2d(stage_a(st), &hmap, ((k0 + ks) % nkh) * 64, m0, bar);
        tma_load_2d(stage_b(st), &wmap, (k0 + ks) * 64, n0, bar);
        issued = ks + 1;
      }
      // no tile may land in shared memory after the CTA has moved on
      for (int ks = max(0, issued - S); ks < issued; ++ks)
        (void)mbar_wait_bounded(smem_addr(&s_full[ks % S]), (ks / S) & 1);
    }
  } else if (wid == 1) {
    if (lane == 0) {  // MMA issuer
      constexpr uint32_t IDESC = umma_idesc_bf16(kRtBM, kRtBN);
      bool ok = true;
      for (int ks = 0; ks < nk; ++ks) {
        const int st = ks % S, use = ks / S;
        if (!mbar_wait_bounded(smem_addr(&s_full[st]), use & 1)) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          umma_f16(tmem, umma_desc_sw128(stage_a(st) + kk * 32), umma_desc_sw128(stage_b(st) + kk * 32), IDESC,
                   (ks | kk) != 0);
        umma_commit(smem_addr(&s_empty[st]));
      }
      if (!ok) give_up();
      umma_commit(smem_addr(&s_accf));
      // every issued MMA is complete before TMEM is released
      (void)mbar_wait_bounded(smem_addr(&s_accf), 0);
    }
  } else if (wid >= 4) {  // epilogue: TMEM lane = tile row
    const bool ok = mbar_wait_bounded(smem_addr(&s_accf), 0);
    tc_fence_after();
    if (__all_sync(0xffffffffu, ok && !aborted())) {  // warp-uniform: tcgen05.ld is collective
      // Every MMA is complete, so the ring is free: each warp stages its 32
      // rows x 32 logits (128-byte swizzle: conflict-free lane stores) in
      // two 4 KB buffers there and writes each block with one TMA store
      // (rows past T are clipped by the tensor map).
      const int quarter = wid & 3, r0 = m0 + quarter * 32;
      const uint32_t lane_addr = tmem + ((uint32_t)(quarter * 32) << 16);
      const uint32_t stg = stage0 + (uint32_t)quarter * 2 * 4096;
      for (int c0 = 0, ob = 0; c0 < kRtBN; c0 += 32, ++ob) {
        float v[32];
        tmem_ld32(lane_addr + c0, v);
        if (p.bias) {
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] += __ldg(p.bias + n0 + c0 + j);
        }
        const uint32_t sb = stg + (uint32_t)(ob & 1) * 4096;
        if (lane == 0 && ob >= 2) bulk_wait_read<1>();  // the store of two blocks ago has read its buffer
        __syncwarp();
#pragma unroll
        for (int q = 0; q < 8; ++q)
          asm volatile("st.shared.v4.f32 [%0], {%1,%2,%3,%4};" ::"r"(sb + lane * 128 + ((q ^ (lane & 7)) << 4)),
                       "f"(v[4 * q]), "f"(v[4 * q + 1]), "f"(v[4 * q + 2]), "f"(v[4 * q + 3])
                       : "memory");
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0 && r0 < p.T) tma_store_3d(&lmap, sb, n0 + c0, r0, blockIdx.z);
      }
      if (lane == 0) bulk_wait_all();
    } else if (lane == 0) {
      give_up();
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (wid == 0) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kRtBN));
  pdl_launch_dependents();
}

struct PfCombineParams {
  const __half *y;    // fp16 [rows][d] grouped order (GEMM experts)
  const __half *yp;   // fp16 [T*k][d] by pair id (GEMV experts: row_of < 0)
  const float *w;     // [T][k]
  const int *row_of;  // [T*k + T]
  int T, k, d, has_shared;
  uint16_t *x;        // bf16 [T][d] residual (mode 0)
  float *delta;       // fp32 [T][d] (mode 1)
};

// x[t] <- bf16(x[t] + sum_j w[t,j] y[row(t,j)] + y[row(shared, t)]), j in order;
// a pair of a GEMV expert reads its y by pair id instead (fp16 as well).
__global__ void __launch_bounds__(256) prefill_combine_kernel(PfCombineParams p) {
  pdl_wait();
  const int per_t = p.d / 4, P = p.T * p.k;
  const long long n = (long long)p.T * per_t;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n;
       i += (long long)gridDim.x * blockDim.x) {
    const int t = (int)(i / per_t), o = (int)(i - (long long)t * per_t) * 4;
    float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
    // four fp16 y values of a row: one 8-byte load
    auto y4 = [&](const __half *base, long long row) {
      const uint2 v = __ldcg(reinterpret_cast<const uint2 *>(base + row * p.d + o));
      return make_float4(half_lo(v.x), half_hi(v.x), half_lo(v.y), half_hi(v.y));
    };
    for (int j = 0; j < p.k; ++j) {
      const float wj = __ldg(p.w + (long long)t * p.k + j);
      const int row = __ldg(p.row_of + (long long)t * p.k + j);
      const float4 v = row >= 0 ? y4(p.y, row) : y4(p.yp, ~row);
      a0 = fmaf(wj, v.x, a0);
      a1 = fmaf(wj, v.y, a1);
      a2 = fmaf(wj, v.z, a2);
      a3 = fmaf(wj, v.w, a3);
    }
    if (p.has_shared) {
      const float4 sh = y4(p.y, P + t);
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
}

// One expert per row (given routing with kk = 1, weight 1): row t's output
// y in fp16, in row order, copied from the GEMM's grouped rows or the GEMV's
// pair rows (an expert-parallel owner's result).
struct PfRowsParams {
  const __half *y;    // fp16 [rows][d] grouped order (GEMM experts)
  const __half *yp;   // fp16 [T][d] by pair id (GEMV experts: row_of < 0)
  const int *row_of;  // [T]
  int T, d;
  __half *out;        // fp16 [T][d]
};

__global__ void __launch_bounds__(256) prefill_rows_kernel(PfRowsParams p) {
  pdl_wait();
  const int per_t = p.d / 8;
  const long long n = (long long)p.T * per_t;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n;
       i += (long long)gridDim.x * blockDim.x) {
    const int t = (int)(i / per_t), o = (int)(i - (long long)t * per_t) * 8;
    const int row = __ldg(p.row_of + t);
    const __half *src = row >= 0 ? p.y + (long long)row * p.d : p.yp + (long long)~row * p.d;
    *reinterpret_cast<uint4 *>(p.out + (long long)t * p.d + o) = __ldcg(reinterpret_cast<const uint4 *>(src + o));
  }
  pdl_launch_dependents();
}

}  // namespace moe
