// decode.cuh -- the whole MoE layer of one decode window in one launch
// (sm_100a).
//
// Per window of T <= 32 tokens (Strata engine analysis article "93 token/s on
// one 8 GB card", section "Architecture overview": router -> the selected
// experts, from wherever they reside -> combine into the residual), one
// persistent CTA per SM runs five phases separated by grid-wide barriers:
//
//   1  stage the window in shared memory (RMSNorm applied when configured)
//      and compute this CTA's slice of the router logits;       barrier
//   2  every CTA reads all logits and, redundantly, selects the top-k of
//      each token, buckets the pairs by expert, looks every selected expert
//      up in the residency table and builds the job list in shared memory
//      (no second barrier is needed: every CTA derives the same list);
//   3  gate/up GEMV: the job list's weight units are split evenly over all
//      warps of the grid (stream-K); an item cut between warps is finished
//      by the warp holding its first unit, which adds the later warps'
//      partial sums in warp order (deterministic), then a = SiLU(g) * u;
//   4  the down projection's weight stream starts before the barrier that
//      makes a visible;                                         barrier
//      down GEMV, split the same way;                           barrier
//   5  combine: x += sum_j w_j y_j + y_shared (j in order).
//
// Compared with one launch per step, this removes three kernel boundaries
// and the single-CTA routing tail from the critical path, and no warp idles
// while another still streams: every warp gets the same number of weight
// bytes.  The grid is one CTA per SM (all co-resident); every wait is
// bounded and reports kErrTimeout.
#pragma once

#include "common.cuh"
#include "gemv.cuh"
#include "route.cuh"

namespace moe {

constexpr int kDecMaxT = 32;        // tokens per window (token sets are 32-bit masks)
constexpr int kDecMaxPairs = 512;   // T * k
constexpr int kDecMaxE = 1024;      // experts (top-k holds <= 32 logits per lane)
constexpr int kDecMaxK = 32;        // lane j of the top-k warp returns selection j
constexpr int kDecSmem = 226 * 1024;
constexpr int kDecWv = 8;           // router-row float4s per lane held in registers
constexpr int kHandFloats = 8;      // partial-sum floats per lane (2 matrices x 4)

// ------------------------------------------------ memory-model helpers
MOE_DEV unsigned long long ld_acquire_u64(const unsigned long long *p) {
  unsigned long long v;
  asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}
MOE_DEV void st_release_u64(unsigned long long *p, unsigned long long v) {
  asm volatile("st.release.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}
MOE_DEV void red_release_add_u64(unsigned long long *p, unsigned long long v) {
  asm volatile("red.release.gpu.global.add.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}
// Orders this thread's earlier generic-proxy global accesses (and those it
// has observed) before its later bulk-copy (async-proxy) reads of global memory.
MOE_DEV void fence_proxy_async_global() { asm volatile("fence.proxy.async.global;" ::: "memory"); }

// Grid-wide barrier of a launch whose CTAs are all resident.  *count only
// grows (one arrival per CTA per barrier); a launch reads it once after its
// dependency wait (a multiple of gridDim.x, every earlier barrier being
// complete), so its n-th barrier completes when the counter reaches
// base + n * gridDim.x: the arrival needs no reply.  Returns false if the
// wait gave up.
// The arrival is a release and the poll an acquire at gpu scope; both are
// cumulative over the CTA's accesses ordered by the CTA barriers around
// them, so no separate fences are needed.
// Split form: grid_arrive, then work that only touches this CTA's shared
// memory, then grid_wait.
MOE_DEV void grid_arrive(unsigned long long *count) {
  __syncthreads();
  if (threadIdx.x == 0) red_release_add_u64(count, 1ull);
}
MOE_DEV bool grid_wait(unsigned long long *count, unsigned long long target, uint32_t limit = 1u << 22) {
  __shared__ int s_ok;
  if (threadIdx.x == 0) {
    bool ok = false;
    for (uint32_t i = 0; !ok && i < limit; ++i) ok = ld_acquire_u64(count) >= target;
    s_ok = ok;
  }
  __syncthreads();
  return s_ok != 0;
}
MOE_DEV bool grid_sync(unsigned long long *count, unsigned long long target) {
  grid_arrive(count);
  return grid_wait(count, target);
}

// Bounded wait for a partial-sum flag to carry this barrier epoch.
MOE_DEV bool wait_flag(const unsigned long long *f, unsigned long long epoch) {
  for (uint32_t i = 0; i < (1u << 20); ++i) {
    if (ld_acquire_u64(f) == epoch) return true;
    if (i >= 64) __nanosleep(64);
  }
  return false;
}

// ------------------------------------------------ shared-memory carve
// Byte offsets from the dynamic shared-memory base: tables first, then the
// warps' weight rings, then the staging area (contiguous with the rings, so
// a wide window can span both while the rings are still idle).
struct DecSmem {
  int ring;          // the warps' weight rings (directly before the staging area)
  int win;           // phase 1 window rows: the staging area, or ring + staging for wide windows
  int restage;       // 1: after routing each CTA re-stages only its gate/up jobs' token rows
  int rowmap;        // int [T]: staging row of token t for the gate/up pass, or -1 (global)
  int bars;          // ring mbarriers of every warp, then the window, staging and restage barriers
  int slot;          // int [E]      residency slots of this layer
  int mask;          // u32 [E]      token set of every expert
  int cnt;           // int [E+1]    per expert (jobs << 16 | tokens), then its exclusive scan
  int idx, w;        // int / float [T*k] selections and weights
  int plist;         // int [T*k + T] pair ids in job order
  int jptr, jbeg, jn;  // job list: u64 expert address, first pair, tokens
  int part;          // float [rpc * qp * T] router partial dots
  int hg, ngd;       // float [T][ngd]   group sums of the window rows (gate/up B)
  int hd, ngf;       // float [rows][ngf] group sums of the staged a rows (down B)
  int hd_rows;
  int hand, hflag;   // partial sums handed to a warp of the same CTA: float [warps][32][8], u64 [warps]
  int stage;         // window rows (phase 1-3), then down-projection B rows
  int stage_bytes;
  int rsh, rsa;      // padded row strides (bytes) of staged h and a rows
  int rpc, qp;       // router rows per CTA, parts per row
  int max_jobs;
  int npl;           // logits per lane of the top-k warp
  int tk_parts;      // warps per token of the split top-k (1: one warp per token)
  int tk_npl;        // logits per lane of a split top-k part
  int cand;          // u64 [warps][k + 1] the parts' candidates
};

MOE_HOST_DEV_INLINE int dec_align(int x, int a) { return (x + a - 1) / a * a; }

// The carve for one launch shape; ring = bytes of the warps' rings.  The
// caller checks T * rsh <= kDecSmem - win.
inline DecSmem dec_layout(int ring, int warps, int chunk, int T, int d, int f, int E, int k,
                          int grid, int group) {
  DecSmem L{};
  int off = 0;
  auto carve = [&](int bytes, int align) {
    off = dec_align(off, align);
    const int at = off;
    off += bytes;
    return at;
  };
  const int P = T * k;
  L.max_jobs = P + (T + chunk - 1) / chunk;
  L.bars = carve((warps * kRingD + 3) * 8, 8);
  L.rowmap = carve(T * 4, 16);
  L.slot = carve(E * 4, 16);
  L.mask = carve(E * 4, 16);
  L.cnt = carve((E + 1) * 4, 16);
  L.idx = carve(P * 4, 16);
  L.w = carve(P * 4, 16);
  L.plist = carve((P + T) * 4, 16);
  L.jptr = carve(L.max_jobs * 8, 16);
  L.jbeg = carve(L.max_jobs * 4, 16);
  L.jn = carve(L.max_jobs * 4, 16);
  L.rpc = (E + grid - 1) / grid;
  const int nch = d / 128;
  L.qp = 1;
  while (L.rpc * L.qp * 2 <= warps && nch % (L.qp * 2) == 0) L.qp *= 2;
  L.part = carve(L.rpc * L.qp * T * 4, 16);
  L.ngd = d / group;
  L.ngf = f / group;
  L.hg = carve(T * L.ngd * 4, 16);
  L.hd_rows = kMaxStagedJobs * chunk;
  L.hd = carve(L.hd_rows * L.ngf * 4, 16);
  // split top-k: parts (a power of two) warps per token, each keeping k + 1
  // candidates of E / parts logits, while T * parts <= warps and the merge
  // sees at most 64 candidates
  L.tk_parts = 1;
  while (L.tk_parts * 2 * T <= warps && L.tk_parts * 2 * (k + 1) <= 64 && E / (L.tk_parts * 2) >= k + 1)
    L.tk_parts *= 2;
  {
    const int per = (E + L.tk_parts - 1) / L.tk_parts;
    L.tk_npl = 1;
    while (L.tk_npl * 32 < per) L.tk_npl *= 2;
    if (L.tk_npl > 8) L.tk_parts = 1;
  }
  L.cand = carve(warps * (k + 1) * 8, 16);
  L.hand = carve(warps * 32 * kHandFloats * 4, 16);
  L.hflag = carve(warps * 8, 8);
  L.ring = carve(ring, 128);
  L.stage = carve(0, 128);
  L.stage_bytes = kDecSmem - L.stage;
  L.rsh = 2 * d + 64;
  L.rsa = 2 * f + 64;
  L.restage = T * L.rsh > L.stage_bytes;
  L.win = L.restage ? L.ring : L.stage;
  L.npl = E <= 128 ? 4 : E <= 512 ? 16 : 32;
  return L;
}

struct DecodeParams {
  uint16_t *x;          // bf16 [T, d] layer input; residual mode: x += moe(x)
  float *delta;         // fp32 [T, d] or null; when set, moe(x) goes here and x is untouched
  const float *gamma;   // RMSNorm weight [d] or null (gamma = 1)
  float eps;
  int use_norm;
  const float *W;       // router fp32 [E, d]
  const float *bias;    // fp32 [E] or null
  int T, d, f, E, k, layer, chunk;
  const int *slot_of;   // [L*E] residency table
  int n_slots;
  const uint8_t *arena, *pool, *shared;
  long long expert_bytes, p1_bytes;
  float *logits;        // [T, E]
  uint16_t *hbuf;       // bf16 [T, d]: the normalised window (written by CTA 0 with RMSNorm)
  uint16_t *abuf;       // bf16 [T*k + T, f]
  float *ybuf;          // fp32 [T*k + T, d]
  float *ws;            // stream-K partial sums [warps of the grid][32][16]
  unsigned long long *flags;  // [2][warps of the grid]
  unsigned long long *bar;    // grid barrier counter
  int *cnt_out;
  unsigned long long *stats;  // [0]=calls [1]=tokens [2]=hits [3]=misses [4]=near_ties
  int *last;
  int *status;
  unsigned long long bar1_extra;  // added to the first grid barrier's target (0; a test
                                  // sets it so that the bounded wait runs out)
  uint32_t bar1_polls;  // poll limit of the first grid barrier
  DecSmem sm;
};

// Group sums of staged bf16 rows: tab[r][q] = scale * sum of the G entries
// of group q of row r (fp32, in order), for r < rows.  All threads.
MOE_DEV void group_sums(const unsigned char *rows_g, int rs, int rows, int ng, int G, float scale,
                        float *tab) {
  for (int i = threadIdx.x; i < rows * ng; i += blockDim.x) {
    const int r = i / ng, q = i - r * ng;
    const uint4 *src = reinterpret_cast<const uint4 *>(rows_g + (size_t)r * rs + (size_t)q * G * 2);
    float acc = 0.f;
    for (int j = 0; j < G / 8; ++j) {
      const uint4 v = src[j];
      acc += __uint_as_float(v.x << 16);
      acc += __uint_as_float(v.x & 0xFFFF0000u);
      acc += __uint_as_float(v.y << 16);
      acc += __uint_as_float(v.y & 0xFFFF0000u);
      acc += __uint_as_float(v.z << 16);
      acc += __uint_as_float(v.z & 0xFFFF0000u);
      acc += __uint_as_float(v.w << 16);
      acc += __uint_as_float(v.w & 0xFFFF0000u);
    }
    tab[i] = scale * acc;
  }
}

// ------------------------------------------------ phase 2: routing
// Top-k of every token, one warp per token; selections and weights into
// shared memory and the token into its experts' token sets.
template <int NPL>
__device__ __noinline__ void decode_topk(const float *logits, int T, int E, int k, int nw,
                                         int *s_idx, float *s_w, unsigned *s_mask,
                                         unsigned long long *near_ties) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  for (int t = wid; t < T; t += nw) {
    int e;
    float w;
    warp_topk<NPL>(logits + (long long)t * E, E, k, lane, t == 0 && near_ties != nullptr, e, w,
                   near_ties);
    if (lane < k) {
      s_idx[t * k + lane] = e;
      s_w[t * k + lane] = w;
      atomicOr(&s_mask[e], 1u << t);
    }
  }
}

// Top-k of every token with `parts` warps per token (warp_topk_part, then
// warp_topk_merge by warp t): the same selections and weights as
// decode_topk in fewer dependent rounds per warp.  All threads.
template <int NPL>
__device__ __noinline__ void decode_topk_split(const float *logits, int T, int E, int k, int parts,
                                               int *s_idx, float *s_w, unsigned *s_mask,
                                               unsigned long long *s_cand,
                                               unsigned long long *near_ties) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int kk = k < E ? k + 1 : k, per = (E + parts - 1) / parts;
  const int t = wid / parts, q = wid - t * parts;
  if (t < T)
    warp_topk_part<NPL>(logits + (long long)t * E, E, per, q, kk, lane, s_cand + (t * parts + q) * kk);
  __syncthreads();
  if (wid < T) {
    int e;
    float w;
    warp_topk_merge(s_cand + wid * parts * kk, parts * kk, E, k, lane, e, w, near_ties);
    if (lane < k) {
      s_idx[wid * k + lane] = e;
      s_w[wid * k + lane] = w;
      atomicOr(&s_mask[e], 1u << wid);
    }
  }
}

// All threads of the CTA: the job list.  Experts come in ascending id, each
// split into jobs of <= chunk tokens in ascending t; one exclusive scan over
// the experts' packed (jobs, tokens) counts gives every expert its first job
// and first pair.  Each selected expert is looked up in the residency table
// (slot pool, else the backing arena; Strata engine analysis article "93
// token/s on one 8 GB card", section "Expert cache").  The shared expert's
// jobs come last.  Ends with a CTA barrier: the weight streams can start
// from here, before the pair list (decode_pairs) exists.
MOE_DEV int decode_jobs(const DecodeParams &p, const int *s_slot, const unsigned *s_mask, int *s_cnt,
                        unsigned long long *s_jptr, int *s_jbeg, int *s_jn) {
  __shared__ int s_red[32];
  const int tid = threadIdx.x;
  const int E = p.E, T = p.T, P = T * p.k, CH = p.chunk;
  for (int e = tid; e < E; e += blockDim.x) {
    const int n = __popc(s_mask[e]);
    s_cnt[e] = (((n + CH - 1) / CH) << 16) | n;
  }
  block_exclusive_scan(s_cnt, s_cnt, E, s_red);
  const int routed_jobs = s_cnt[E] >> 16;
  for (int e = tid; e < E; e += blockDim.x) {
    const int n = __popc(s_mask[e]);
    if (!n) continue;
    int jx = s_cnt[e] >> 16;
    const int px = s_cnt[e] & 0xFFFF;
    const int slot = s_slot[e];
    const uint8_t *ptr;
    if (slot >= 0 && slot < p.n_slots) {
      ptr = p.pool + (long long)slot * p.expert_bytes;
    } else {
      if (slot >= p.n_slots && blockIdx.x == 0) atomicOr(p.status, kErrBadSlot);
      ptr = p.arena + ((long long)p.layer * E + e) * p.expert_bytes;
    }
    for (int c0 = 0; c0 < n; c0 += CH, ++jx) {
      s_jptr[jx] = (unsigned long long)ptr;
      s_jbeg[jx] = px + c0;
      s_jn[jx] = min(CH, n - c0);
    }
  }
  int shared_jobs = 0;
  if (p.shared) {
    shared_jobs = (T + CH - 1) / CH;
    for (int q = tid; q < shared_jobs; q += blockDim.x) {
      s_jptr[routed_jobs + q] = (unsigned long long)p.shared;
      s_jbeg[routed_jobs + q] = P + q * CH;
      s_jn[routed_jobs + q] = min(CH, T - q * CH);
    }
  }
  __syncthreads();
  return routed_jobs + shared_jobs;
}

// All threads of the CTA, after decode_jobs: the pair list (each expert's
// tokens in ascending t, as pair ids t*k + j; the shared expert's pairs
// P + t last) and, in CTA 0, the statistics (per-expert token counts,
// residency hits and misses, warp-reduced).  Ends with a CTA barrier.
MOE_DEV void decode_pairs(const DecodeParams &p, const int *s_slot, const unsigned *s_mask,
                          const int *s_idx, const int *s_cnt, int *s_plist) {
  __shared__ unsigned long long s_hm[3];  // hits, misses, active experts (CTA 0)
  const int tid = threadIdx.x;
  const int E = p.E, k = p.k, T = p.T, P = T * k;
  const bool cta0 = blockIdx.x == 0;
  if (tid < 3) s_hm[tid] = 0;
  unsigned my_hits = 0, my_misses = 0, my_active = 0;
  for (int e = tid; e < E; e += blockDim.x) {
    unsigned m = s_mask[e];
    const int n = __popc(m);
    if (cta0) p.cnt_out[e] = n;
    if (!n) continue;
    const int px = s_cnt[e] & 0xFFFF;
    const int slot = s_slot[e];
    (slot >= 0 && slot < p.n_slots ? my_hits : my_misses) += (unsigned)n;
    ++my_active;
    for (int b = 0; m; ++b) {
      const int t = __ffs(m) - 1;
      m &= m - 1;
      int j = k - 1;  // the token's selection slot of e (independent loads)
#pragma unroll 4
      for (int jj = k - 2; jj >= 0; --jj) j = s_idx[t * k + jj] == e ? jj : j;
      s_plist[px + b] = t * k + j;
    }
  }
  if (p.shared)
    for (int t = tid; t < T; t += blockDim.x) s_plist[P + t] = P + t;
  __syncthreads();  // s_hm cleared before any warp adds to it
  if (cta0) {
    const unsigned h = __reduce_add_sync(0xffffffffu, my_hits);
    const unsigned mi = __reduce_add_sync(0xffffffffu, my_misses);
    const unsigned a = __reduce_add_sync(0xffffffffu, my_active);
    if ((tid & 31) == 0) {
      atomicAdd(&s_hm[0], (unsigned long long)h);
      atomicAdd(&s_hm[1], (unsigned long long)mi);
      atomicAdd(&s_hm[2], (unsigned long long)a);
    }
  }
  __syncthreads();
  if (cta0 && tid == 0) {
    atomicAdd(&p.stats[0], 1ULL);
    atomicAdd(&p.stats[1], (unsigned long long)T);
    atomicAdd(&p.stats[2], s_hm[0]);
    atomicAdd(&p.stats[3], s_hm[1]);
    p.last[0] = T;
    p.last[1] = (int)s_hm[2];
    p.last[2] = p.layer;
  }
}

// ------------------------------------------------ phases 3 and 4: stream-K GEMV
// The phase's U weight units (job-major, then row block, then unit) are
// split over the W warps of the grid: warp w owns [U w / W, U (w+1) / W).
struct SKCtx {
  int U, W, gw;
  int q, rm;                  // U = q W + rm: start(w) = q w + (rm w) / W in 32 bits
  unsigned long long epoch;   // this phase's barrier number
  float *ws;                  // [W][32 lanes][16] partial sums (hand-over between CTAs)
  unsigned long long *flags;  // [W] this phase's hand-over flags (between CTAs)
  float *s_hand;              // [warps][32][kHandFloats] same hand-over within the CTA
  unsigned long long *s_flag; // [warps]
  int warps;                  // warps per CTA
  int cta_start;              // first unit of this CTA's range
};

MOE_DEV SKCtx sk_make(int U, int W, int gw, unsigned long long epoch, float *ws,
                      unsigned long long *flags, float *s_hand, unsigned long long *s_flag,
                      int warps) {
  SKCtx sk{U, W, gw, U / W, U % W, epoch, ws, flags, s_hand, s_flag, warps, 0};
  sk.cta_start = sk.q * (gw - gw % warps) + (sk.rm * (gw - gw % warps)) / W;
  return sk;
}

// First unit of warp w's range (= floor(U w / W)).
MOE_DEV int sk_start(const SKCtx &sk, int w) { return sk.q * w + (sk.rm * w) / sk.W; }

// One item of the warp's range: units [ua, ub) of item `it`.
//  ua > 0   the item began in an earlier warp's range: publish the partial
//           sum for that warp to add -- in shared memory when it runs in
//           this CTA, else in ws[gw] with flags[gw] = epoch;
//  ub < UPI the item continues in later warps' ranges: add their partial
//           sums in warp order, then store;
//  else     the whole item is here: store.
template <int FMT, bool GATED, int NTA, bool HTAB>
MOE_DEV bool sk_item(WarpRing &r, const Phase &ph, const SKCtx &sk, int ubase, int ua, int ub,
                     int lane, int rb, const BRows &br, const int (&epair)[2][2], int R,
                     uint16_t *out_a, float *out_y) {
  using Run = ItemRun<FMT, GATED, NTA, HTAB>;
  constexpr int NM = Run::C::NM;
  float acc[NM][NTA][4];
  if (!Run::run(r, ph, lane, ua, ub, br, acc)) return false;
  static_assert(NM * NTA * 4 <= kHandFloats || NTA > 1, "hand-over slot too small");
  const int cta_w0 = sk.gw - sk.gw % sk.warps;  // first warp of this CTA
  if (ua > 0) {
    // the item's first unit (ubase) lies in this CTA's range iff its owner runs here
    const bool local = NM * NTA * 4 <= kHandFloats && ubase >= sk.cta_start;
    float4 *mine = local ? reinterpret_cast<float4 *>(sk.s_hand + ((sk.gw - cta_w0) * 32 + lane) * kHandFloats)
                         : reinterpret_cast<float4 *>(sk.ws + ((long long)sk.gw * 32 + lane) * 16);
#pragma unroll
    for (int m = 0; m < NM; ++m)
#pragma unroll
      for (int nt = 0; nt < NTA; ++nt)
        mine[m * NTA + nt] = make_float4(acc[m][nt][0], acc[m][nt][1], acc[m][nt][2], acc[m][nt][3]);
    __syncwarp();
    if (lane == 0) {
      if (local) {
        __threadfence_block();
        *reinterpret_cast<volatile unsigned long long *>(sk.s_flag + (sk.gw - cta_w0)) = sk.epoch;
      } else {
        st_release_u64(sk.flags + sk.gw, sk.epoch);  // release covers the lanes' stores (syncwarp)
      }
    }
    return true;
  }
  if (ub < ph.UPI) {
    const int iend = ubase + ph.UPI;
    for (int w2 = sk.gw + 1; w2 < sk.W; ++w2) {
      const int s2 = sk_start(sk, w2);
      if (s2 >= iend) break;
      if (sk_start(sk, w2 + 1) == s2) continue;  // empty range: nothing to add
      const bool local = NM * NTA * 4 <= kHandFloats && w2 < cta_w0 + sk.warps;
      const float *src;
      if (local) {
        bool ok = false;
        for (uint32_t i = 0; !ok && i < (1u << 24); ++i)
          ok = *reinterpret_cast<volatile unsigned long long *>(sk.s_flag + (w2 - cta_w0)) == sk.epoch;
        if (__any_sync(0xffffffffu, !ok)) return false;
        __threadfence_block();
        src = sk.s_hand + ((w2 - cta_w0) * 32 + lane) * kHandFloats;
      } else {
        if (__any_sync(0xffffffffu, !wait_flag(sk.flags + w2, sk.epoch))) return false;
        src = sk.ws + ((long long)w2 * 32 + lane) * 16;
      }
#pragma unroll
      for (int m = 0; m < NM; ++m)
#pragma unroll
        for (int nt = 0; nt < NTA; ++nt) {
          float4 v;
          if (local) {  // asm load: not moved above the fence
            const uint4 q = ld_v4(src + 4 * (m * NTA + nt));
            v = make_float4(__uint_as_float(q.x), __uint_as_float(q.y), __uint_as_float(q.z),
                            __uint_as_float(q.w));
          } else {
            v = ldcg_f4(src + 4 * (m * NTA + nt));
          }
          acc[m][nt][0] += v.x;
          acc[m][nt][1] += v.y;
          acc[m][nt][2] += v.z;
          acc[m][nt][3] += v.w;
        }
    }
  }
  Run::store(acc, epair, rb, lane, R, out_a, out_y);
  return true;
}

// Gate/up pass over this warp's units.  B rows are the window's token rows:
// token t at staging row s_rowmap[t] (row stride rsh) at stage_g, or in
// global memory (gsrc) when s_rowmap[t] < 0.
template <int FMT, int NTM>
MOE_DEV bool decode_gated(WarpRing &r, const Phase &ph, const SKCtx &sk, int u0, int u1,
                          const DecodeParams &p, const int *s_plist, const int *s_jbeg,
                          const int *s_jn, const unsigned char *stage_g, const float *s_hg,
                          const int *s_rowmap, const uint16_t *gsrc) {
  const int lane = threadIdx.x & 31, g = lane >> 2, tig = lane & 3;
  const int P = p.T * p.k;
  if (u1 <= u0) return true;
  const int it0 = u0 / ph.UPI;
  int job = it0 / ph.RB, rb = it0 - job * ph.RB;
  for (int ubase = it0 * ph.UPI; ubase < u1; ubase += ph.UPI) {
    const int ua = max(u0, ubase) - ubase, ub = min(u1, ubase + ph.UPI) - ubase;
    const int n = s_jn[job], beg = s_jbeg[job];
    BRows br;
    int epair[2][2];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      br.row[nt] = nullptr;
      br.hc[nt][0] = br.hc[nt][1] = nullptr;
      epair[nt][0] = epair[nt][1] = -1;
    }
#pragma unroll
    for (int nt = 0; nt < NTM; ++nt) {
      const int ni = nt * 8 + g;
      if (ni < n) {
        const int pair = s_plist[beg + ni];
        const int tok = pair < P ? pair / p.k : pair - P;
        const int sr = s_rowmap[tok];
        br.row[nt] = sr >= 0 ? reinterpret_cast<const uint16_t *>(stage_g + (size_t)sr * p.sm.rsh)
                             : gsrc + (long long)tok * p.d;
      }
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        const int nc = nt * 8 + 2 * tig + c;
        epair[nt][c] = nc < n ? s_plist[beg + nc] : -1;
        if (nc < n) {
          const int pc = epair[nt][c];
          br.hc[nt][c] = s_hg + (pc < P ? pc / p.k : pc - P) * p.sm.ngd;
        }
      }
    }
    const bool ok =
        (NTM == 1 || n <= 8)
            ? sk_item<FMT, true, 1, true>(r, ph, sk, ubase, ua, ub, lane, rb, br, epair, p.f, p.abuf, nullptr)
            : sk_item<FMT, true, NTM, true>(r, ph, sk, ubase, ua, ub, lane, rb, br, epair, p.f, p.abuf, nullptr);
    if (!ok) return false;
    if (++rb == ph.RB) {
      rb = 0;
      ++job;
    }
  }
  return true;
}

// Down pass over this warp's units.  B rows are rows of a: the CTA's first
// jobs are staged in shared memory at stage_g (nst jobs; job jfirst + i
// starts at staged row row0 of lane i), later ones are read from global
// memory.
template <int FMT, int NTM>
MOE_DEV bool decode_down(WarpRing &r, const Phase &ph, const SKCtx &sk, int u0, int u1,
                         const DecodeParams &p, const int *s_plist, const int *s_jbeg,
                         const int *s_jn, const unsigned char *stage_g, const float *s_hd, int jfirst,
                         int nst, int row0) {
  const int lane = threadIdx.x & 31, g = lane >> 2, tig = lane & 3;
  if (u1 <= u0) return true;
  const int it0 = u0 / ph.UPI;
  int job = it0 / ph.RB, rb = it0 - job * ph.RB;
  for (int ubase = it0 * ph.UPI; ubase < u1; ubase += ph.UPI) {
    const int ua = max(u0, ubase) - ubase, ub = min(u1, ubase + ph.UPI) - ubase;
    const int n = s_jn[job], beg = s_jbeg[job];
    const int sj = job - jfirst;
    const bool staged = sj >= 0 && sj < nst;
    const int jrow0 = __shfl_sync(0xffffffffu, row0, staged ? sj : 0);
    BRows br;
    int epair[2][2];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      br.row[nt] = nullptr;
      br.hc[nt][0] = br.hc[nt][1] = nullptr;
      epair[nt][0] = epair[nt][1] = -1;
    }
#pragma unroll
    for (int nt = 0; nt < NTM; ++nt) {
      const int ni = nt * 8 + g;
      if (ni < n)
        br.row[nt] = staged ? reinterpret_cast<const uint16_t *>(stage_g + (size_t)(jrow0 + ni) * p.sm.rsa)
                            : p.abuf + (long long)s_plist[beg + ni] * p.f;
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        const int nc = nt * 8 + 2 * tig + c;
        epair[nt][c] = nc < n ? s_plist[beg + nc] : -1;
        if (staged && nc < n) br.hc[nt][c] = s_hd + (jrow0 + nc) * p.sm.ngf;
      }
    }
    bool ok;
    if (staged)
      ok = (NTM == 1 || n <= 8)
               ? sk_item<FMT, false, 1, true>(r, ph, sk, ubase, ua, ub, lane, rb, br, epair, p.d, nullptr, p.ybuf)
               : sk_item<FMT, false, NTM, true>(r, ph, sk, ubase, ua, ub, lane, rb, br, epair, p.d, nullptr, p.ybuf);
    else  // rows read from global memory: group sums from the tensor core
      ok = (NTM == 1 || n <= 8)
               ? sk_item<FMT, false, 1, false>(r, ph, sk, ubase, ua, ub, lane, rb, br, epair, p.d, nullptr, p.ybuf)
               : sk_item<FMT, false, NTM, false>(r, ph, sk, ubase, ua, ub, lane, rb, br, epair, p.d, nullptr, p.ybuf);
    if (!ok) return false;
    if (++rb == ph.RB) {
      rb = 0;
      ++job;
    }
  }
  return true;
}

// dot of one 128-column chunk of a router row (w: this lane's 4 columns)
// with up to 8 staged token rows
MOE_DEV void dot8(float (&acc)[8], const float4 w, uint32_t hcol, int t0, int T, int rsh) {
#pragma unroll
  for (int tt = 0; tt < 8; ++tt) {
    if (t0 + tt < T) {
      const uint2 v = lds_u2(hcol + (uint32_t)(t0 + tt) * rsh);
      acc[tt] = fmaf(w.x, __uint_as_float(v.x << 16), acc[tt]);
      acc[tt] = fmaf(w.y, __uint_as_float(v.x & 0xFFFF0000u), acc[tt]);
      acc[tt] = fmaf(w.z, __uint_as_float(v.y << 16), acc[tt]);
      acc[tt] = fmaf(w.w, __uint_as_float(v.y & 0xFFFF0000u), acc[tt]);
    }
  }
}

// The decode kernel.  NTM = 8-token column tiles per job (jobs of <= 8 NTM
// tokens); one CTA per SM.
template <int FMT, int NTM>
__global__ void __launch_bounds__(GemvCfg<FMT, true, NTM>::WARPS * 32, 1)
    decode_kernel(DecodeParams p) {
  using CG = GemvCfg<FMT, true, NTM>;
  using CD = GemvCfg<FMT, false, NTM>;
  constexpr int WARPS = CG::WARPS;
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ int s_njobs;
  __shared__ unsigned long long s_bar0;  // grid barrier counter at launch
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  const int T = p.T, d = p.d, f = p.f, E = p.E, k = p.k;
  const DecSmem &L = p.sm;
  int *s_slot = reinterpret_cast<int *>(smem + L.slot);
  unsigned *s_mask = reinterpret_cast<unsigned *>(smem + L.mask);
  int *s_cnt = reinterpret_cast<int *>(smem + L.cnt);
  int *s_idx = reinterpret_cast<int *>(smem + L.idx);
  float *s_w = reinterpret_cast<float *>(smem + L.w);
  int *s_plist = reinterpret_cast<int *>(smem + L.plist);
  unsigned long long *s_jptr = reinterpret_cast<unsigned long long *>(smem + L.jptr);
  int *s_jbeg = reinterpret_cast<int *>(smem + L.jbeg);
  int *s_jn = reinterpret_cast<int *>(smem + L.jn);
  float *s_part = reinterpret_cast<float *>(smem + L.part);
  float *s_hg = reinterpret_cast<float *>(smem + L.hg);
  float *s_hd = reinterpret_cast<float *>(smem + L.hd);
  float *s_hand = reinterpret_cast<float *>(smem + L.hand);
  unsigned long long *s_hflag = reinterpret_cast<unsigned long long *>(smem + L.hflag);
  constexpr int GQ = FMT == 1 ? 32 : 64;            // quantisation group
  constexpr float kSumScale = FMT == 1 ? -136.f : 1.f;  // see ItemRun::tile
  const uint32_t stage_s = smem_addr(smem + L.stage);
  const unsigned char *stage_g = smem + L.stage;
  const uint32_t win_s = smem_addr(smem + L.win);
  unsigned char *win_g = smem + L.win;
  int *s_rowmap = reinterpret_cast<int *>(smem + L.rowmap);
  const uint32_t bars = smem_addr(smem + L.bars);
  const uint32_t h_bar = bars + WARPS * kRingD * 8, st_bar = h_bar + 8, rs_bar = h_bar + 16;

  MOE_TRACE(kTrRouteStart);
  WarpRing r;
  ring_init(r, smem_addr(smem + L.ring) + wid * kRingD * CG::SLOT, bars + wid * kRingD * 8, CG::SLOT);
  if (lane == 0) {
    for (int u = 0; u < kRingD; ++u) mbar_init(r.bar_s + 8 * u, 1);
    if (wid == 0) {
      mbar_init(h_bar, 1);
      mbar_init(st_bar, 1);
      mbar_init(rs_bar, 1);
    }
    fence_mbar_init();
  }
  // Router rows of this CTA: rpc rows, each dotted in qp parts of cpp
  // 128-column chunks by one warp per (row, part).  The first task's row
  // part goes into registers before the dependency wait (the router weights
  // do not depend on earlier kernels).
  const int RPC = L.rpc, QP = L.qp, CPP = (d / 128) / QP, ntask = RPC * QP;
  float4 wv[kDecWv];
  {
    const int rr = wid / QP, q = wid - rr * QP, e = blockIdx.x * RPC + rr;
    const bool has = wid < ntask && e < E;
    const float4 *wr = reinterpret_cast<const float4 *>(p.W + (long long)(has ? e : 0) * d) +
                       q * CPP * 32 + lane;
#pragma unroll
    for (int i = 0; i < kDecWv; ++i)
      wv[i] = (has && i < CPP) ? __ldg(wr + 32 * i) : make_float4(0.f, 0.f, 0.f, 0.f);
  }
  for (int e = tid; e < E; e += blockDim.x) {
    s_slot[e] = p.slot_of ? p.slot_of[(long long)p.layer * E + e] : -1;
    s_mask[e] = 0u;
  }
  if (tid < WARPS) s_hflag[tid] = 0ull;  // epochs start at 1
  __syncthreads();
  pdl_wait();
  MOE_TRACE(kTrRouteWaited);
  if (tid == 0) s_bar0 = ld_acquire_u64(p.bar);  // read by all after the next barrier

  // ---------------- phase 1: the window, RMSNorm, router logits
  if (tid == 0) {
    mbar_expect_tx(h_bar, (uint32_t)T * d * 2);
    for (int t = 0; t < T; ++t)
      bulk_g2s(win_s + (uint32_t)t * L.rsh, p.x + (long long)t * d, (uint32_t)d * 2, h_bar);
  }
  if (__syncthreads_or(!mbar_wait_bounded(h_bar, 0))) {
    if (tid == 0) atomicOr(p.status, kErrTimeout);
    return;
  }
  if (p.use_norm) {  // fp32 sum of squares, IEEE sqrt and divide, bf16 RNE
    for (int t = wid; t < T; t += WARPS) {
      uint16_t *hr = reinterpret_cast<uint16_t *>(win_g + (long long)t * L.rsh);
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
        const float in[4] = {__uint_as_float(v.x << 16), __uint_as_float(v.x & 0xFFFF0000u),
                             __uint_as_float(v.y << 16), __uint_as_float(v.y & 0xFFFF0000u)};
        unsigned short o[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          float rv = in[j] * inv;
          if (p.gamma) rv *= p.gamma[i + j];
          o[j] = __bfloat16_as_ushort(__float2bfloat16_rn(rv));
        }
        v.x = o[0] | ((uint32_t)o[1] << 16);
        v.y = o[2] | ((uint32_t)o[3] << 16);
        *reinterpret_cast<uint2 *>(hr + i) = v;
        // CTA 0 publishes the normalised rows: wide windows re-stage them
        // after routing (visible to every CTA after the first barrier), and
        // moe_debug_last_h reads them back
        if (blockIdx.x == 0) *reinterpret_cast<uint2 *>(p.hbuf + (long long)t * d + i) = v;
      }
    }
    __syncthreads();
  }
  for (int task = wid, it = 0; task < ntask; task += WARPS, ++it) {
    const int rr = task / QP, q = task - rr * QP, e = blockIdx.x * RPC + rr;
    if (e >= E) continue;
    const float4 *wr = reinterpret_cast<const float4 *>(p.W + (long long)e * d) + q * CPP * 32 + lane;
    const uint32_t hcol = win_s + 2u * (uint32_t)(q * CPP * 128 + lane * 4);
    for (int t0 = 0; t0 < T; t0 += 8) {
      float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int i = 0; i < kDecWv; ++i)
        if (i < CPP) dot8(acc, it == 0 ? wv[i] : __ldg(wr + 32 * i), hcol + 256u * i, t0, T, L.rsh);
      for (int i = kDecWv; i < CPP; ++i) dot8(acc, __ldg(wr + 32 * i), hcol + 256u * i, t0, T, L.rsh);
#pragma unroll
      for (int tt = 0; tt < 8; ++tt) {
        if (t0 + tt >= T) break;
        const float v = warp_sum(acc[tt]);
        if (lane == tt) s_part[task * T + t0 + tt] = v;
      }
    }
  }
  __syncthreads();
  for (int i = tid; i < RPC * T; i += blockDim.x) {
    const int rr = i / T, t = i - rr * T, e = blockIdx.x * RPC + rr;
    if (e < E) {
      float s = 0.f;
      for (int q = 0; q < QP; ++q) s += s_part[(rr * QP + q) * T + t];
      if (p.bias) s += p.bias[e];
      p.logits[(long long)t * E + e] = s;
    }
  }
  MOE_TRACE(kTrRouteLogits);
  const unsigned long long G = gridDim.x, ep0 = s_bar0 / G;
  const unsigned long long ep1 = ep0 + 1;
  grid_arrive(p.bar);
  // group sums of the window rows for the gate/up pass, while the grid syncs
  group_sums(win_g, L.rsh, T, L.ngd, GQ, kSumScale, s_hg);
  if (!grid_wait(p.bar, ep1 * G + p.bar1_extra, p.bar1_polls)) {
    if (tid == 0) atomicOr(p.status, kErrTimeout);
    return;
  }
  MOE_TRACE(kTrRouteLastStart);

  // ---------------- phase 2: routing (every CTA, redundantly)
  unsigned long long *near = blockIdx.x == 0 ? &p.stats[4] : nullptr;
  unsigned long long *s_cand = reinterpret_cast<unsigned long long *>(smem + L.cand);
  if (L.tk_parts > 1) {
    if (L.tk_npl == 1) decode_topk_split<1>(p.logits, T, E, k, L.tk_parts, s_idx, s_w, s_mask, s_cand, near);
    else if (L.tk_npl == 2) decode_topk_split<2>(p.logits, T, E, k, L.tk_parts, s_idx, s_w, s_mask, s_cand, near);
    else if (L.tk_npl == 4) decode_topk_split<4>(p.logits, T, E, k, L.tk_parts, s_idx, s_w, s_mask, s_cand, near);
    else decode_topk_split<8>(p.logits, T, E, k, L.tk_parts, s_idx, s_w, s_mask, s_cand, near);
  } else if (L.npl == 4) {
    decode_topk<4>(p.logits, T, E, k, WARPS, s_idx, s_w, s_mask, near);
  } else if (L.npl == 16) {
    decode_topk<16>(p.logits, T, E, k, WARPS, s_idx, s_w, s_mask, near);
  } else {
    decode_topk<32>(p.logits, T, E, k, WARPS, s_idx, s_w, s_mask, near);
  }
  __syncthreads();
  MOE_TRACE(kTrRouteTopk);
  {
    const int nj = decode_jobs(p, s_slot, s_mask, s_cnt, s_jptr, s_jbeg, s_jn);
    if (tid == 0) s_njobs = nj;
  }
  __syncthreads();
  MOE_TRACE(kTrRouteEnd);
  const int n_jobs = s_njobs;
  const int W = gridDim.x * WARPS, gw = blockIdx.x * WARPS + wid;

  // ---------------- phase 3: gate/up
  const Phase ph1 = make_phase(s_jptr, f, d, CG::TK, CG::STRIDE, 0);
  const SKCtx sk1 = sk_make(n_jobs * ph1.RB * ph1.UPI, W, gw, ep1, p.ws, p.flags, s_hand, s_hflag, WARPS);
  // The warp's first weight units go in flight as soon as the job list
  // exists; the pair list and the token rows are built while they land.
  const int u0 = sk_start(sk1, gw), u1 = sk_start(sk1, gw + 1);
  {
    const int i0 = u0 / ph1.UPI;
    ring_start(r, ph1, i0 / ph1.RB, i0 % ph1.RB, u0 - i0 * ph1.UPI, u1 - u0, 1);
    if (lane == 0) fence_proxy_async_smem();  // a wide window occupied the rings until now
    __syncwarp();
    ring_prologue(r, ph1, lane);
  }
  decode_pairs(p, s_slot, s_mask, s_idx, s_cnt, s_plist);
  // Token rows for the gate/up B operand.  A window that fits the staging
  // area stays there (row t at staging row t).  A wide window was staged
  // over the rings and the staging area; now that the rings are needed, the
  // CTA copies only the tokens of its own gate/up jobs into the staging
  // area (as many as fit), and reads any others from global memory.
  const uint16_t *gsrc = p.use_norm ? p.hbuf : p.x;
  if (!L.restage) {
    for (int t = tid; t < T; t += blockDim.x) s_rowmap[t] = t;
  } else {
    for (int t = tid; t < T; t += blockDim.x) s_rowmap[t] = -1;
    __syncthreads();
    if (tid == 0) {
      const int c0 = sk_start(sk1, blockIdx.x * WARPS), c1 = sk_start(sk1, (blockIdx.x + 1) * WARPS);
      const int cap = L.stage_bytes / L.rsh, P = T * k;
      int rows = 0;
      if (c1 > c0) {
        const int jf = c0 / ph1.UPI / ph1.RB, jl = (c1 - 1) / ph1.UPI / ph1.RB;
        for (int j = jf; j <= jl; ++j)
          for (int i = 0; i < s_jn[j]; ++i) {
            const int pr = s_plist[s_jbeg[j] + i], tok = pr < P ? pr / k : pr - P;
            if (s_rowmap[tok] < 0 && rows < cap) s_rowmap[tok] = rows++;
          }
      }
      // the normalised rows came from generic stores before the first barrier;
      // the window area was last read by this CTA's generic loads
      fence_proxy_async_global();
      fence_proxy_async_smem();
      mbar_expect_tx(rs_bar, (uint32_t)rows * d * 2);
      for (int t = 0; t < T; ++t)
        if (s_rowmap[t] >= 0)
          bulk_g2s(stage_s + (uint32_t)s_rowmap[t] * L.rsh, gsrc + (long long)t * d, (uint32_t)d * 2,
                   rs_bar);
    }
    if (__syncthreads_or(!mbar_wait_bounded(rs_bar, 0))) {
      ring_drain(r);  // the first weight units are in flight
      if (tid == 0) atomicOr(p.status, kErrTimeout);
      return;
    }
  }
  __syncthreads();
  if (!decode_gated<FMT, NTM>(r, ph1, sk1, u0, u1, p, s_plist, s_jbeg, s_jn, stage_g, s_hg, s_rowmap,
                              gsrc)) {
    if (lane == 0) atomicOr(p.status, kErrTimeout);
    ring_drain(r);
  }
  if (lane == 0) trace_point(kTrGateEnd);

  // ---------------- phase 4: down projection
  // down units of up to four tiles: the ring slots hold a gate/up unit (two
  // tiles of both matrices), so a down unit may fill the same bytes
  const Phase ph2 = make_phase(s_jptr, d, f, CD::TK, CD::STRIDE, p.p1_bytes, CG::SLOT);
  const SKCtx sk2 = sk_make(n_jobs * ph2.RB * ph2.UPI, W, gw, ep0 + 2, p.ws, p.flags + W, s_hand,
                            s_hflag, WARPS);
  const int v0 = sk_start(sk2, gw), v1 = sk_start(sk2, gw + 1);
  {
    const int i0 = v0 / ph2.UPI;
    ring_start(r, ph2, i0 / ph2.RB, i0 % ph2.RB, v0 - i0 * ph2.UPI, v1 - v0, 1);
  }
  ring_prologue(r, ph2, lane);  // weights stream in while the grid syncs
  if (!grid_sync(p.bar, (ep0 + 2) * G)) {
    ring_drain(r);
    if (tid == 0) atomicOr(p.status, kErrTimeout);
    return;
  }
  MOE_TRACE(kTrDownWaited);
  // Stage the a rows of this CTA's first down jobs (whole jobs, at most
  // kMaxStagedJobs, as many as fit).  Every warp derives the same plan; lane
  // i describes job jfirst + i.
  int jfirst = 0, njobs_cta = 0;
  {
    const int c0 = sk_start(sk2, blockIdx.x * WARPS), c1 = sk_start(sk2, (blockIdx.x + 1) * WARPS);
    if (c1 > c0) {
      jfirst = c0 / ph2.UPI / ph2.RB;
      njobs_cta = (c1 - 1) / ph2.UPI / ph2.RB - jfirst + 1;
    }
  }
  int pn = 0, pbeg = 0;
  if (lane < njobs_cta && lane < kMaxStagedJobs) {
    pn = s_jn[jfirst + lane];
    pbeg = s_jbeg[jfirst + lane];
  }
  int incl = pn;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  const int row0 = incl - pn;
  const int cap = L.stage_bytes / L.rsa;
  const int nst = __popc(__ballot_sync(0xffffffffu, pn > 0 && incl <= cap && incl <= L.hd_rows));
  const int used = nst ? __shfl_sync(0xffffffffu, incl, nst - 1) : 0;
  if (wid == 0) {
    // a was written by other CTAs' generic stores before the barrier; the
    // window rows in the staging area were last read before it
    fence_proxy_async_global();
    fence_proxy_async_smem();
    if (lane == 0) mbar_expect_tx(st_bar, (uint32_t)used * f * 2);
    __syncwarp();
    for (int r0 = 0; r0 < used; r0 += 32) {
      const int rr = r0 + lane;
      int sj = 0;
      for (int q = 1; q < nst; ++q) sj += rr >= __shfl_sync(0xffffffffu, row0, q) ? 1 : 0;
      const int beg = __shfl_sync(0xffffffffu, pbeg, sj);
      const int rj = rr - __shfl_sync(0xffffffffu, row0, sj);
      if (rr < used)
        bulk_g2s(stage_s + (uint32_t)rr * L.rsa, p.abuf + (long long)s_plist[beg + rj] * f,
                 (uint32_t)f * 2, st_bar);
    }
  }
  // every thread: the staged rows, then their group sums
  if (__syncthreads_or(!mbar_wait_bounded(st_bar, 0))) {
    ring_drain(r);
    if (tid == 0) atomicOr(p.status, kErrTimeout);
    return;
  }
  group_sums(stage_g, L.rsa, used, L.ngf, GQ, kSumScale, s_hd);
  __syncthreads();
  if (!decode_down<FMT, NTM>(r, ph2, sk2, v0, v1, p, s_plist, s_jbeg, s_jn, stage_g, s_hd, jfirst,
                             nst, row0)) {
    if (lane == 0) atomicOr(p.status, kErrTimeout);
    ring_drain(r);
  }
  if (lane == 0) trace_point(kTrDownEnd);
  if (!grid_sync(p.bar, (ep0 + 3) * G)) {
    if (tid == 0) atomicOr(p.status, kErrTimeout);
    return;
  }
  pdl_launch_dependents();

  // ---------------- phase 5: combine + residual
  MOE_TRACE(kTrCombStart);
  const int P = T * k, per_t = d / 4;
  for (int i = blockIdx.x * blockDim.x + tid; i < T * per_t; i += gridDim.x * blockDim.x) {
    const int t = i / per_t, o = (i - t * per_t) * 4;
    const float4 sh = p.shared ? ldcg_f4(p.ybuf + ((long long)P + t) * d + o) : make_float4(0.f, 0.f, 0.f, 0.f);
    float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
    for (int j0 = 0; j0 < k; j0 += 16) {
      float4 v[16];
#pragma unroll
      for (int q = 0; q < 16; ++q)
        if (j0 + q < k) v[q] = ldcg_f4(p.ybuf + ((long long)t * k + j0 + q) * d + o);
#pragma unroll
      for (int q = 0; q < 16; ++q) {
        if (j0 + q < k) {
          const float wj = s_w[t * k + j0 + q];
          a0 = fmaf(wj, v[q].x, a0);
          a1 = fmaf(wj, v[q].y, a1);
          a2 = fmaf(wj, v[q].z, a2);
          a3 = fmaf(wj, v[q].w, a3);
        }
      }
    }
    a0 += sh.x;
    a1 += sh.y;
    a2 += sh.z;
    a3 += sh.w;
    if (p.delta) {
      *reinterpret_cast<float4 *>(p.delta + (long long)t * d + o) = make_float4(a0, a1, a2, a3);
    } else {
      uint16_t *xr = p.x + (long long)t * d + o;
      const uint2 xv = *reinterpret_cast<const uint2 *>(xr);
      uint2 o2;
      o2.x = __bfloat16_as_ushort(__float2bfloat16_rn(__uint_as_float(xv.x << 16) + a0)) |
             ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(__uint_as_float(xv.x & 0xFFFF0000u) + a1)) << 16);
      o2.y = __bfloat16_as_ushort(__float2bfloat16_rn(__uint_as_float(xv.y << 16) + a2)) |
             ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(__uint_as_float(xv.y & 0xFFFF0000u) + a3)) << 16);
      *reinterpret_cast<uint2 *>(xr) = o2;
    }
  }
  if (lane == 0) trace_point(kTrCombEnd);
}

}  // namespace moe
