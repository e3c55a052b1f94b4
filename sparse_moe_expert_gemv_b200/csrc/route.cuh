// route.cuh -- top-k + renormalised softmax, bucketing by expert, residency
// lookup and the expert job list (sm_100a).
//
// The router picks the k of E experts a token activates and their routing
// weights; the selected experts are then computed from wherever they reside
// (Strata engine analysis article "93 token/s on one 8 GB card", sections
// "Architecture overview" and "Expert cache": (layer, expert) -> slot or -1).
// The grouped expert kernels want the tokens bucketed by expert, so the
// routing step also builds, per call, the list of expert jobs.
//
// Two entry kernels share one block-level body:
//  * route_fused_kernel (windows of <= 32 tokens): each CTA stages the window
//    (RMSNorm applied when configured), computes the logits of its experts,
//    and the last CTA to finish runs the body;
//  * route_finish_kernel: the body alone, after router_logits_kernel.
#pragma once

#include "common.cuh"

namespace moe {

struct FinishParams {
  // inputs
  const float *logits;     // [T, E] or null (bucket-only mode)
  const int *idx_in;       // [T, k] when logits == null
  int T, E, k, layer;
  // routing outputs
  int *idx;                // [T, k]
  float *w;                // [T, k] (unused in bucket-only mode)
  int *off;                // [E+1]
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

// pairs whose routing ids and bucket order are kept in shared memory
constexpr int kSmemPairs = 4096;
constexpr int kMaxSlotPrefetch = 4;  // E <= kMaxSlotPrefetch * blockDim.x

// Exclusive prefix sum over n ints: out[i] = sum in[0..i), out[n] = total.
// in and out may alias; red: 32 ints of scratch.  All threads of the block
// call it; it begins and ends with a barrier, so `in` may have been written
// by any thread just before the call.  Each thread scans a run of
// ceil(n / blockDim.x) consecutive entries.
MOE_DEV void block_exclusive_scan(const int *in, int *out, int n, int *red) {
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5, nw = blockDim.x >> 5;
  const int ept = (n + blockDim.x - 1) / blockDim.x;
  __syncthreads();
  const int i0 = tid * ept;
  int run = 0;
  for (int i = 0; i < ept; ++i)
    if (i0 + i < n) run += in[i0 + i];
  int x = run;
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
    red[lane] = s;
  }
  __syncthreads();
  int excl = (wid ? red[wid - 1] : 0) + x - run;
  const int total = red[nw - 1];
  __syncthreads();  // everyone has read in[] and red[] before out[] is written
  for (int i = 0; i < ept; ++i)
    if (i0 + i < n) {
      const int v = in[i0 + i];
      out[i0 + i] = excl;
      excl += v;
    }
  if (tid == 0) out[n] = total;
  __syncthreads();
}

// Largest of n packed values by a balanced tournament (depth log2 n).
template <int N>
MOE_DEV unsigned long long tournament_max(const unsigned long long (&v)[N]) {
  constexpr int LOG2N = N >= 32 ? 5 : N >= 16 ? 4 : N >= 8 ? 3 : N >= 4 ? 2 : N >= 2 ? 1 : 0;
  unsigned long long m[N];
#pragma unroll
  for (int i = 0; i < N; ++i) m[i] = v[i];
#pragma unroll
  for (int l = 0; l < LOG2N; ++l) {
#pragma unroll
    for (int i = 0; i < (N >> (l + 1)); ++i) {
      const unsigned long long b = m[i + (N >> (l + 1))];
      m[i] = m[i] > b ? m[i] : b;
    }
  }
  return m[0];
}

// Top-k + renormalised softmax of one token by one warp (Strata engine
// analysis article "93 token/s on one 8 GB card", section "Architecture
// overview": the router picks the top 10 of 512 experts per token).  A lane
// holds logits lane + 32 i as 64-bit (order-preserving key << 32 | ~expert)
// values, so the larger value is the larger logit and equal logits favour
// the lower id.  Each selection round: a register tournament gives every
// lane its best, one redux.max over the warp gives the winning key and a
// second one the lowest id holding it; the winner's entry is cleared.  Lane
// j < k returns the j-th selection (descending logit) and its weight
// exp(l_j - l_0) / sum_j' exp(l_j' - l_0).  When near_ties is non-null, a
// (k+1)-th logit within 1e-5 of the k-th counts one near tie.
// When lk is non-null, *lk and *lk1 receive (in every lane) the k-th and the
// (k+1)-th largest logits (-inf when k == E).
template <int NPL>
MOE_DEV void warp_topk(const float *lr, int E, int k, int lane, bool trace, int &sel_e,
                       float &sel_w, unsigned long long *near_ties, float *lk = nullptr,
                       float *lk1 = nullptr) {
  unsigned long long pk[NPL];
#pragma unroll
  for (int i = 0; i < NPL; ++i) {
    const int e = lane + 32 * i;
    pk[i] = e < E ? ((unsigned long long)order_key(__ldcg(lr + e)) << 32) | (uint32_t)~e : 0ull;
  }
  if (trace && lane == 0 && pk[0] != 1ull) trace_point(kTrRouteLoaded);
  uint32_t my_key = 0, k0 = 0, kk = 0;
  int my_i = 0;
  if (lk1) *lk1 = -INFINITY;
  for (int j = 0; j <= k; ++j) {
    if (j == k && k == E) break;
    const unsigned long long best = tournament_max<NPL>(pk);
    const uint32_t hi = (uint32_t)(best >> 32);
    const uint32_t wmax = __reduce_max_sync(0xffffffffu, hi);
    const uint32_t wlo = __reduce_max_sync(0xffffffffu, hi == wmax ? (uint32_t)best : 0u);
    const int wi = (int)~wlo;
    if (j == k) {  // the (k+1)-th logit: near-tie count only
      if (near_ties && lane == 0 && key_to_float(kk) - key_to_float(wmax) < 1e-5f)
        atomicAdd(near_ties, 1ULL);
      if (lk1) *lk1 = key_to_float(wmax);
      break;
    }
    const bool mine = (wi & 31) == lane;
#pragma unroll
    for (int i = 0; i < NPL; ++i) pk[i] = (mine && (wi >> 5) == i) ? 0ull : pk[i];
    if (lane == j) {
      my_key = wmax;
      my_i = wi;
    }
    if (j == 0) k0 = wmax;
    kk = wmax;
  }
  if (trace && lane == 0) trace_point(kTrRouteSelected);
  if (lk) *lk = key_to_float(kk);
  const float ex = lane < k ? expf(key_to_float(my_key) - key_to_float(k0)) : 0.f;
  const float den = warp_sum(ex);
  sel_e = my_i;
  sel_w = ex / den;
}

// The kk best of a warp's packed values (lane + 32 i holds pk[i]; 0 =
// empty), in descending order: lane j < kk returns the j-th, 0 if fewer
// exist.  Same round as warp_topk, with the winner cleared by value (the
// packed values are distinct).
template <int NPL>
MOE_DEV unsigned long long warp_top_packed(unsigned long long (&pk)[NPL], int kk, int lane) {
  unsigned long long mine = 0ull;
  for (int j = 0; j < kk; ++j) {
    const unsigned long long best = tournament_max<NPL>(pk);
    const uint32_t hi = (uint32_t)(best >> 32);
    const uint32_t wmax = __reduce_max_sync(0xffffffffu, hi);
    const uint32_t wlo = __reduce_max_sync(0xffffffffu, hi == wmax ? (uint32_t)best : 0u);
    const unsigned long long win = ((unsigned long long)wmax << 32) | wlo;
    if (lane == j) mine = win;
#pragma unroll
    for (int i = 0; i < NPL; ++i) pk[i] = pk[i] == win ? 0ull : pk[i];
  }
  return mine;
}

// Top-k of one token split over `parts` warps (part 1): warp q of the token
// keeps the kk = k + 1 best of experts [q per, (q+1) per) as packed values
// in cand[q][kk].  The union of the parts' k + 1 best holds the token's
// k + 1 best, so the merge (warp_topk_merge) selects exactly what warp_topk
// selects over all E logits, in the same order.
template <int NPL>
MOE_DEV void warp_topk_part(const float *lr, int E, int per, int q, int kk, int lane,
                            unsigned long long *cand) {
  unsigned long long pk[NPL];
  const int e0 = q * per, e1 = min(E, e0 + per);
#pragma unroll
  for (int i = 0; i < NPL; ++i) {
    const int e = e0 + lane + 32 * i;
    pk[i] = e < e1 ? ((unsigned long long)order_key(__ldcg(lr + e)) << 32) | (uint32_t)~e : 0ull;
  }
  const unsigned long long v = warp_top_packed<NPL>(pk, kk, lane);
  if (lane < kk) cand[lane] = v;
}

// Part 2: one warp merges the n <= 64 candidates of a token (cand[0..n))
// and returns, like warp_topk, selection j and its weight in lane j < k,
// counting a near tie of the k-th and (k+1)-th logits when near_ties is set.
MOE_DEV void warp_topk_merge(const unsigned long long *cand, int n, int E, int k, int lane,
                             int &sel_e, float &sel_w, unsigned long long *near_ties) {
  unsigned long long pk[2];
#pragma unroll
  for (int i = 0; i < 2; ++i) pk[i] = lane + 32 * i < n ? cand[lane + 32 * i] : 0ull;
  const int kk = k < E ? k + 1 : k;
  const unsigned long long v = warp_top_packed<2>(pk, kk, lane);
  const uint32_t key = (uint32_t)(v >> 32);
  const uint32_t k0 = __shfl_sync(0xffffffffu, key, 0);
  const uint32_t kth = __shfl_sync(0xffffffffu, key, k - 1);
  const uint32_t next = __shfl_sync(0xffffffffu, key, kk - 1);
  if (k < E && near_ties && lane == 0 && key_to_float(kth) - key_to_float(next) < 1e-5f)
    atomicAdd(near_ties, 1ULL);
  const float ex = lane < k ? expf(key_to_float(key) - key_to_float(k0)) : 0.f;
  const float den = warp_sum(ex);
  sel_e = (int)~(uint32_t)v;
  sel_w = ex / den;
}

// Top-k of one token by one warp through a candidate filter; same result
// as warp_topk (selections, weights, *lk, *lk1).  The (k+1)-th largest of
// the lanes' maxima is a threshold that at least k + 1 logits reach, so the
// k + 1 best are among the values at or above it: those (usually a few
// dozen) are compacted into cand[0..64) (this warp's shared memory) and the
// k + 1 best of them are selected two per lane.  A full selection round over
// all NPL values per lane runs only once (the lane maxima) instead of k + 1
// times.  Returns false, with nothing written, when k + 1 > 32, k >= E or
// more than 64 values pass; the caller then runs warp_topk.  Near ties are
// counted as warp_topk counts them.
template <int NPL>
MOE_DEV bool warp_topk_fast(const float *lr, int E, int k, int lane, unsigned long long *cand, int &sel_e,
                            float &sel_w, unsigned long long *near_ties, float *lk, float *lk1) {
  if (k + 1 > 32 || k >= E) return false;
  unsigned long long pk[NPL];
#pragma unroll
  for (int i = 0; i < NPL; ++i) {
    const int e = lane + 32 * i;
    pk[i] = e < E ? ((unsigned long long)order_key(__ldcg(lr + e)) << 32) | (uint32_t)~e : 0ull;
  }
  // the (k+1)-th largest lane maximum: min(E, 32) >= k + 1 lanes hold one
  unsigned long long m = tournament_max<NPL>(pk), thr = 0ull;
  for (int j = 0; j <= k; ++j) {
    const uint32_t hi = (uint32_t)(m >> 32);
    const uint32_t wmax = __reduce_max_sync(0xffffffffu, hi);
    const uint32_t wlo = __reduce_max_sync(0xffffffffu, hi == wmax ? (uint32_t)m : 0u);
    thr = ((unsigned long long)wmax << 32) | wlo;
    m = m == thr ? 0ull : m;
  }
  int c = 0;
#pragma unroll
  for (int i = 0; i < NPL; ++i) c += (pk[i] != 0ull && pk[i] >= thr) ? 1 : 0;
  int incl = c;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  const int total = __shfl_sync(0xffffffffu, incl, 31);
  if (total > 64) return false;
  int pos = incl - c;
#pragma unroll
  for (int i = 0; i < NPL; ++i)
    if (pk[i] != 0ull && pk[i] >= thr) cand[pos++] = pk[i];
  __syncwarp();
  unsigned long long pc[2];
#pragma unroll
  for (int i = 0; i < 2; ++i) pc[i] = lane + 32 * i < total ? cand[lane + 32 * i] : 0ull;
  __syncwarp();  // cand[] may be rewritten by this warp's next token
  const unsigned long long v = warp_top_packed<2>(pc, k + 1, lane);  // lane j <= k: the j-th best
  const uint32_t key = (uint32_t)(v >> 32);
  const uint32_t k0 = __shfl_sync(0xffffffffu, key, 0);
  const uint32_t kth = __shfl_sync(0xffffffffu, key, k - 1);
  const uint32_t next = __shfl_sync(0xffffffffu, key, k);
  if (near_ties && lane == 0 && key_to_float(kth) - key_to_float(next) < 1e-5f) atomicAdd(near_ties, 1ULL);
  if (lk) *lk = key_to_float(kth);
  if (lk1) *lk1 = key_to_float(next);
  const float ex = lane < k ? expf(key_to_float(key) - key_to_float(k0)) : 0.f;
  const float den = warp_sum(ex);
  sel_e = lane < k ? (int)~(uint32_t)v : 0;
  sel_w = ex / den;
  return true;
}

// Shared-memory words the body needs (dynamic smem of the finish kernel;
// the fused kernel reuses its staging area).
MOE_HOST_DEV_INLINE int finish_smem_ints(int E, int P) {
  return 4 * E + 2 + (P <= kSmemPairs ? 2 * P : 0);
}

// The routing body, run by one CTA after the logits exist.
//  Phase A: one warp per token selects the k largest logits (warp_topk).
//  Phase B: counting sort of the T*k pairs by expert (histogram, exclusive
//    scan, stable scatter with ascending t).
//  Phase C: the residency lookup (slot table -> slot pool or backing arena)
//    and the list of expert jobs (<= chunk tokens each).
// slot_pref holds slot_of[layer*E + tid + i*blockDim] (prefetched).
template <int NPL>
MOE_DEV void finish_body(const FinishParams &p, int *sm, const int (&slot_pref)[kMaxSlotPrefetch]) {
  __shared__ int red[32];
  __shared__ unsigned long long hit_miss[2];
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5, nw = blockDim.x >> 5;
  const int T = p.T, E = p.E, k = p.k, P = T * k;
  const bool smem_pairs = P <= kSmemPairs;
  int *cnt = sm;                 // [E]
  int *off = cnt + E;            // [E+1]
  int *fill = off + E + 1;       // [E]
  int *jscan = fill + E;         // [E+1]
  int *sidx = jscan + E + 1;     // [P]  (smem_pairs)
  int *sperm = sidx + P;         // [P]  (smem_pairs)

  // ---------------- phase A: top-k + softmax
  if (p.logits) {
    for (int t = wid; t < T; t += nw) {
      int sel_e;
      float sel_w;
      warp_topk<NPL>(p.logits + (long long)t * E, E, k, lane, t == 0, sel_e, sel_w, &p.stats[4]);
      if (lane < k) {
        p.idx[(long long)t * k + lane] = sel_e;
        p.w[(long long)t * k + lane] = sel_w;
        if (smem_pairs) sidx[t * k + lane] = sel_e;
      }
    }
  } else if (smem_pairs) {
    for (int q = tid; q < P; q += blockDim.x) sidx[q] = p.idx_in[q];
  }
  const int *idx = smem_pairs ? sidx : (p.logits ? p.idx : p.idx_in);
  int *perm = smem_pairs ? sperm : p.perm;

  // ---------------- phase B: bucketing
  for (int e = tid; e < E; e += blockDim.x) {
    cnt[e] = 0;
    fill[e] = 0;
  }
  __syncthreads();
  MOE_TRACE(kTrRouteTopk);
  for (int q = tid; q < P; q += blockDim.x) {
    const int e = idx[q];
    if (e >= 0 && e < E) atomicAdd(&cnt[e], 1);
    else atomicOr(p.status, kErrBadExpert);
  }
  block_exclusive_scan(cnt, off, E, red);
  // stable scatter: warp 0 walks the pairs in order, 32 at a time
  if (wid == 0) {
    for (int base = 0; base < P; base += 32) {
      const int q = base + lane;
      int e = q < P ? idx[q] : -1;
      if (e >= E) e = -1;
      const unsigned mask = __match_any_sync(0xffffffffu, e);
      const int rank = __popc(mask & ((1u << lane) - 1u));
      if (e >= 0) perm[off[e] + fill[e] + rank] = q;
      __syncwarp();
      if (e >= 0 && rank == 0) fill[e] += __popc(mask);
      __syncwarp();
    }
  }
  __syncthreads();
  for (int e = tid; e <= E; e += blockDim.x) p.off[e] = off[e];
  if (smem_pairs)
    for (int q = tid; q < P; q += blockDim.x) p.perm[q] = sperm[q];
  MOE_TRACE(kTrRouteBucket);
  if (!p.build_jobs) return;

  // ---------------- phase C: residency lookup + expert jobs
  if (tid < 2) hit_miss[tid] = 0;
  for (int e = tid; e < E; e += blockDim.x) fill[e] = (cnt[e] + p.chunk - 1) / p.chunk;
  block_exclusive_scan(fill, jscan, E, red);
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
#pragma unroll
  for (int i = 0; i < kMaxSlotPrefetch; ++i) {
    const int e = tid + i * blockDim.x;
    if (e >= E) break;
    const int c = cnt[e];
    p.cnt_out[e] = c;
    if (!c) continue;
    active++;
    const long long le = (long long)p.layer * E + e;
    const int slot = slot_pref[i];
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
  for (int q = tid; q < P; q += blockDim.x) p.plist[q] = perm[q];
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
    atomicAdd(&p.stats[0], 1ULL);
    atomicAdd(&p.stats[1], (unsigned long long)T);
    atomicAdd(&p.stats[2], hit_miss[0]);
    atomicAdd(&p.stats[3], hit_miss[1]);
    p.last[0] = T;
    p.last[1] = a;
    p.last[2] = p.layer;
  }
}

MOE_DEV void prefetch_slots(const FinishParams &p, int (&slot_pref)[kMaxSlotPrefetch]) {
#pragma unroll
  for (int i = 0; i < kMaxSlotPrefetch; ++i) {
    const int e = threadIdx.x + i * blockDim.x;
    slot_pref[i] = (p.slot_of && e < p.E) ? p.slot_of[(long long)p.layer * p.E + e] : -1;
  }
}

constexpr int kFinishThreads = 512;

template <int NPL>  // logits per lane = ceil(E / 32) rounded up to a power of 2
__global__ void __launch_bounds__(kFinishThreads) route_finish_kernel(FinishParams p) {
  extern __shared__ int sm[];
  int slot_pref[kMaxSlotPrefetch];
  prefetch_slots(p, slot_pref);
  pdl_wait();
  finish_body<NPL>(p, sm, slot_pref);
  __syncthreads();
  pdl_launch_dependents();  // late: see route_fused_kernel
}

// ---------------------------------------------------------- fused routing
struct RouteFusedParams {
  const uint16_t *x;       // bf16 [T, d] layer input
  const float *gamma;      // RMSNorm weight [d] or null (gamma = 1)
  float eps;
  int use_norm;            // h = RMSNorm(x) (else h = x)
  uint16_t *h_out;         // normalised h for the expert kernels (use_norm)
  const float *W;          // fp32 [E, d]
  const float *bias;       // fp32 [E] or null
  int d;
  float *logits;           // fp32 [T, E]
  unsigned int *ticket;    // [0] CTA completion counter, [1] abort flag; both
                           // zero between calls (the last CTA resets them)
  FinishParams f;
};

constexpr int kFusedWarps = 8;  // at most; 4 for windows of <= 8 tokens
constexpr int kFusedMaxT = 32;
constexpr int kFusedSmem = 160 * 1024;
constexpr int kFusedMaxV = 16;  // router row in registers: d <= 16 * 128

// Whole routing step of a decode window in one launch.  Each CTA stages the
// window in shared memory (applying RMSNorm when configured: fp32 sum of
// squares, IEEE sqrt and divide, bf16 round-to-nearest-even), and each warp
// dots one router row (loaded into registers before the dependency wait)
// with every token, four tokens at a time, fp32 accumulate.  The last CTA to finish (atomic ticket) runs the
// routing body on the complete logits and resets the ticket.  A CTA whose
// staging wait gives up reports kErrTimeout, raises the abort flag and still
// takes its ticket, so the count completes: the last CTA then leaves the
// outputs unwritten and resets both words, and the next call starts clean.
template <int NPL>
__global__ void __launch_bounds__(kFusedWarps * 32) route_fused_kernel(RouteFusedParams p) {
  extern __shared__ __align__(128) unsigned char fsm[];
  __shared__ int s_last;
  __shared__ __align__(8) unsigned long long s_bar;
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;
  const int E = p.f.E, T = p.f.T, d = p.d, nv = d / 128;
  const int e = blockIdx.x * nw + wid;
  MOE_TRACE(kTrRouteStart);
  // the router row does not depend on earlier kernels: registers, before the wait
  const float4 *wr = reinterpret_cast<const float4 *>(p.W + (long long)(e < E ? e : 0) * d);
  float4 wv[kFusedMaxV];
#pragma unroll
  for (int i = 0; i < kFusedMaxV; ++i)
    wv[i] = (e < E && i < nv) ? __ldg(wr + lane + 32 * i) : make_float4(0.f, 0.f, 0.f, 0.f);
  const float b = (e < E && p.bias) ? p.bias[e] : 0.f;
  int slot_pref[kMaxSlotPrefetch];
  prefetch_slots(p.f, slot_pref);
  if (threadIdx.x == 0) {
    mbar_init(smem_addr(&s_bar), 1);
    fence_mbar_init();
  }
  __syncthreads();
  pdl_wait();
  MOE_TRACE(kTrRouteWaited);

  // stage the window: one bulk copy of the T contiguous rows
  if (threadIdx.x == 0) {
    const uint32_t bytes = (uint32_t)T * d * 2;
    mbar_expect_tx(smem_addr(&s_bar), bytes);
    bulk_g2s(smem_addr(fsm), p.x, bytes, smem_addr(&s_bar));
  }
  // the whole CTA agrees on the outcome of the wait (no thread leaves alone)
  const bool staged = !__syncthreads_or(!mbar_wait_bounded(smem_addr(&s_bar), 0));
  if (!staged && threadIdx.x == 0) {
    atomicOr(p.f.status, kErrTimeout);
    atomicOr(p.ticket + 1, 1u);
  }
  if (staged && p.use_norm) {
    for (int t = wid; t < T; t += nw) {
      uint16_t *hr = reinterpret_cast<uint16_t *>(fsm) + (long long)t * d;
      float ss = 0.f;
      for (int i = lane * 4; i < d; i += 128) {
        const uint2 v = *reinterpret_cast<const uint2 *>(hr + i);
        const float a0 = __uint_as_float(v.x << 16), a1 = __uint_as_float(v.x & 0xFFFF0000u);
        const float a2 = __uint_as_float(v.y << 16), a3 = __uint_as_float(v.y & 0xFFFF0000u);
        ss += a0 * a0 + a1 * a1 + a2 * a2 + a3 * a3;
      }
      ss = warp_sum(ss);
      const float inv = 1.0f / sqrtf(ss / (float)d + p.eps);
      for (int i = lane * 4; i < d; i += 128) {
        uint2 v = *reinterpret_cast<const uint2 *>(hr + i);
        float in[4] = {__uint_as_float(v.x << 16), __uint_as_float(v.x & 0xFFFF0000u),
                       __uint_as_float(v.y << 16), __uint_as_float(v.y & 0xFFFF0000u)};
        unsigned short o[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          float r = in[j] * inv;
          if (p.gamma) r *= p.gamma[i + j];
          o[j] = __bfloat16_as_ushort(__float2bfloat16_rn(r));
        }
        v.x = o[0] | ((uint32_t)o[1] << 16);
        v.y = o[2] | ((uint32_t)o[3] << 16);
        *reinterpret_cast<uint2 *>(hr + i) = v;
        if (blockIdx.x == 0) *reinterpret_cast<uint2 *>(p.h_out + (long long)t * d + i) = v;
      }
    }
    __syncthreads();
  }

  // logits of this warp's expert for every token
  if (staged && e < E) {
    const uint32_t hb0 = smem_addr(fsm);
    for (int t = 0; t < T; t += 4) {
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int i = 0; i < kFusedMaxV; ++i) {
        if (i >= nv) break;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          if (t + q < T) {
            const uint2 v = lds_u2(hb0 + (uint32_t)(t + q) * d * 2 + 8 * (lane + 32 * i));
            acc[q] = fmaf(wv[i].x, __uint_as_float(v.x << 16), acc[q]);
            acc[q] = fmaf(wv[i].y, __uint_as_float(v.x & 0xFFFF0000u), acc[q]);
            acc[q] = fmaf(wv[i].z, __uint_as_float(v.y << 16), acc[q]);
            acc[q] = fmaf(wv[i].w, __uint_as_float(v.y & 0xFFFF0000u), acc[q]);
          }
        }
      }
#pragma unroll
      for (int o = 16; o; o >>= 1)
#pragma unroll
        for (int q = 0; q < 4; ++q) acc[q] += __shfl_xor_sync(0xffffffffu, acc[q], o);
      if (lane < 4 && t + lane < T) {
        const float v = lane == 0 ? acc[0] : lane == 1 ? acc[1] : lane == 2 ? acc[2] : acc[3];
        p.logits[(long long)(t + lane) * E + e] = v + b;
      }
    }
  }

  // the last CTA routes: the CTA barrier orders every thread's logits before
  // thread 0's device-scope fence and ticket; the last CTA's thread 0 fences
  // again before the CTA reads the other CTAs' logits (through L2)
  __syncthreads();
  MOE_TRACE(kTrRouteLogits);
  if (threadIdx.x == 0) {
    __threadfence();
    s_last = atomicAdd(p.ticket, 1u) == gridDim.x - 1;
    if (s_last) {
      __threadfence();
      // a CTA gave up: some logits are missing, route nothing
      if (atomicAdd(p.ticket + 1, 0u) != 0u) s_last = 2;
    }
  }
  __syncthreads();
  if (!s_last) return;
  MOE_TRACE(kTrRouteLastStart);
  if (s_last == 1) finish_body<NPL>(p.f, reinterpret_cast<int *>(fsm), slot_pref);
  MOE_TRACE(kTrRouteEnd);
  if (threadIdx.x == 0) {
    p.ticket[1] = 0u;
    p.ticket[0] = 0u;
  }
  // the expert kernels may launch now (not earlier: CTAs parked in their
  // dependency wait would compete with this CTA, the critical path)
  __syncthreads();
  pdl_launch_dependents();
}

}  // namespace moe
