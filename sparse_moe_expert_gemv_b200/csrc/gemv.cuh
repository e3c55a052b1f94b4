// gemv.cuh -- grouped dequant-GEMV of the decode path (sm_100a).
//
// One launch computes, for every job (an expert with up to 8*NTM of its
// tokens), either the gated half of the SwiGLU expert, a = SiLU(Wg h) *
// (Wu h), or the down projection y = Wd a.  The expert weights dominate the
// layer's HBM traffic (Strata engine analysis article "93 token/s on one 8 GB
// card", section "Expert cache": the expert bytes are the largest single cost
// and the kernel is memory-bound), so the kernel is built around streaming
// each selected expert's packed codes exactly once:
//
//  * Work items are (job, block of 16 output rows), ordered job-major.  Each
//    CTA (one per SM, 16 warps) owns a contiguous range of items, so it
//    touches only a few jobs; its warps take the range's items round-robin.
//  * The B operand of those jobs (their token rows of h, or their rows of a)
//    is copied once into shared memory with 1-D bulk copies; a job that does
//    not fit is read from L2 instead, one tile ahead.
//  * Each warp streams the weight tiles of its items through a private ring
//    of D shared-memory slots filled by 1-D bulk (TMA) copies, D tiles in
//    flight across item boundaries.  A tile is one 16-row x TK-column block
//    of codes (512 B, laid out so each lane's 16 bytes are its own mma
//    fragments) followed by the block's fp16 scales (and mins).
//  * Codes become exact bf16 values in registers (a LOP3 per pair of codes,
//    plus shifts) and go through mma.m16n8k16 with fp32 accumulation against
//    up to 8*NTM token columns; each quantisation group's partial sum is
//    scaled in fp32.  Even and odd k-steps accumulate in separate chains so
//    consecutive mma's are independent.
#pragma once

#include "common.cuh"

namespace moe {

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

constexpr int kGemvSmem = 220 * 1024;  // dynamic shared memory per CTA
constexpr int kMaxStagedJobs = 8;

template <int FMT, bool GATED, int NTM = 1>
struct GemvCfg {
  static constexpr int TK = FMT == 1 ? 64 : 128;
  static constexpr int TILE = FMT == 1 ? 576 : 640;
  static constexpr int NM = GATED ? 2 : 1;
  static constexpr int STRIDE = NM * TILE;
  static constexpr int D = 3;       // ring slots per warp (each 1 or 2 tiles)
  static constexpr int NT = NTM;    // 8-token mma column tiles per job (max)
  static constexpr int WARPS = NTM == 1 ? 16 : 8;  // register file: 128 / 255 per thread
  static constexpr int STEPS = TK / 16;  // mma k-steps per tile
  static constexpr int RING = WARPS * D * 2 * STRIDE;
  static constexpr int BARS = WARPS * D * 8 + 8;  // ring barriers + staging barrier
  static constexpr int STAGE_OFF = (RING + BARS + 127) / 128 * 128;
  static constexpr int STAGE_BYTES = kGemvSmem - STAGE_OFF;
};

// Per-warp streaming state.  The producer (lane 0) always runs exactly D
// tiles ahead of the consumer, so it refills the slot just consumed.
struct WarpRing {
  uint32_t data_s, bar_s;
  int u;             // slot of the next tile to consume
  uint32_t phase;    // its mbarrier parity
  int pj, pt;        // producer cursor: my-item index and tile
  const unsigned char *pbase;
};

struct ItemGeom {
  int first, step, my_items;  // my items: first + j * step, j < my_items
  int RB, NTILE;
  int tps;                    // tiles per ring slot (2 when NTILE is even)
  long long stride;           // bytes per tile of this phase (all matrices)
  long long region_off;
};

MOE_DEV const unsigned char *item_base(const GemvParams &p, const ItemGeom &g, int j) {
  const int item = g.first + j * g.step;
  const int job = item / g.RB, rb = item - job * g.RB;
  const unsigned long long base = ldcg_u64(p.job_ptr + job);
  return reinterpret_cast<const unsigned char *>(base) + g.region_off +
         (long long)rb * g.NTILE * g.stride;
}

// lane 0: issue the producer's next tps tiles into slot `slot` and advance
MOE_DEV void ring_issue(WarpRing &r, const GemvParams &p, const ItemGeom &g, int slot) {
  if (r.pj >= g.my_items) return;
  const uint32_t bar = r.bar_s + 8 * slot;
  const uint32_t bytes = (uint32_t)(g.tps * g.stride);
  fence_proxy_async_smem();
  mbar_expect_tx(bar, bytes);
  bulk_g2s(r.data_s + slot * bytes, r.pbase, bytes, bar);
  r.pbase += bytes;
  r.pt += g.tps;
  if (r.pt == g.NTILE) {
    r.pt = 0;
    if (++r.pj < g.my_items) r.pbase = item_base(p, g, r.pj);
  }
}

// Where a lane's B rows live for the current item: shared memory (staged
// job) or global memory (L2).
struct BRows {
  bool smem;
  uint32_t s[2];               // shared addresses of the lane's rows (0 = none)
  const uint16_t *gp[2];       // global rows (nullptr = none)
};

// One item (16 output rows of one job) of the streaming GEMV.
//  NTA    8-token column tiles of the job (1 or 2)
//  ONECOL the job has a single token: only accumulator column 0 is live, so
//         the per-group scaling and the epilogue skip the other column
//  BSMEM  the job's B rows are staged in shared memory (else read from L2)
template <int FMT, bool GATED, int NTA, bool ONECOL, bool BSMEM>
struct ItemRun {
  using C = GemvCfg<FMT, GATED>;  // tile geometry does not depend on NTM or WARPS

  // B fragments of tile t: per column tile, STEPS x (b0, b1)
  static MOE_DEV void load_b(uint2 (&b)[NTA][C::STEPS], const BRows &br, int t, int tig) {
#pragma unroll
    for (int nt = 0; nt < NTA; ++nt)
#pragma unroll
      for (int s = 0; s < C::STEPS; ++s) {
        const int col = t * C::TK + 16 * s + 4 * tig;
        if constexpr (BSMEM)
          b[nt][s] = br.s[nt] ? lds_u2(br.s[nt] + 2 * col) : make_uint2(0u, 0u);
        else
          b[nt][s] = br.gp[nt] ? ldcg_u2(br.gp[nt] + col) : make_uint2(0u, 0u);
      }
  }

  // acc += this tile's contribution.  c runs over the live accumulator
  // entries: (row g, col 2tig), (row g, col 2tig+1), (row g+8, ...) ...
  static MOE_DEV void tile(uint32_t tile_s, int lane, const uint2 (&b)[NTA][C::STEPS],
                           float (&acc)[C::NM][NTA][4]) {
    const int g = lane >> 2;
    const uint32_t ones[4] = {0x3F803F80u, 0x3F803F80u, 0x3F803F80u, 0x3F803F80u};
    uint4 cw[C::NM];
#pragma unroll
    for (int m = 0; m < C::NM; ++m) cw[m] = lds_u4(tile_s + m * C::TILE + lane * 16);
    // [chain][m][nt][4]: chain 0 takes even k-steps, chain 1 odd ones
    float tmp[2][C::NM][NTA][4];
    float tH[2][NTA][4];
    if constexpr (FMT == 1) {
      // codes enter the mma as exact bf16 128 + c; sum((c - 8) h) is
      // tmp - 136 * sum(h), and sum(h) comes from an mma against ones
      uint2 sc[C::NM];
#pragma unroll
      for (int m = 0; m < C::NM; ++m) sc[m] = lds_u2(tile_s + m * C::TILE + 512 + g * 8);
#pragma unroll
      for (int s = 0; s < 4; ++s) {
        const int ch = s & 1;
        uint32_t a[C::NM][4];
#pragma unroll
        for (int m = 0; m < C::NM; ++m) {
          const uint32_t word = s == 0 ? cw[m].x : s == 1 ? cw[m].y : s == 2 ? cw[m].z : cw[m].w;
          a[m][0] = lop3_and_or(word, 0x000F000Fu, 0x43004300u);
          a[m][1] = lop3_and_or(word >> 4, 0x000F000Fu, 0x43004300u);
          a[m][2] = lop3_and_or(word >> 8, 0x000F000Fu, 0x43004300u);
          a[m][3] = lop3_and_or(word >> 12, 0x000F000Fu, 0x43004300u);
        }
#pragma unroll
        for (int nt = 0; nt < NTA; ++nt) {
#pragma unroll
          for (int m = 0; m < C::NM; ++m)
            mma_bf16_acc(tmp[ch][m][nt], a[m], b[nt][s].x, b[nt][s].y, true);
          mma_bf16_acc(tH[ch][nt], ones, b[nt][s].x, b[nt][s].y, true);
        }
        if (s & 1) {  // end of a 32-wide group
#pragma unroll
          for (int nt = 0; nt < NTA; ++nt) {
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              if (ONECOL && (c & 1)) continue;
              const float corr = 136.f * (tH[0][nt][c] + tH[1][nt][c]);
#pragma unroll
              for (int m = 0; m < C::NM; ++m) {
                const uint32_t sv = (s >> 1) ? sc[m].y : sc[m].x;
                const float sf = c < 2 ? half_lo(sv) : half_hi(sv);
                acc[m][nt][c] = fmaf(sf, (tmp[0][m][nt][c] + tmp[1][m][nt][c]) - corr, acc[m][nt][c]);
              }
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
            const int st = 4 * half + 2 * wv + hs;  // step within the tile
            const bool first = wv == 0;             // first use of chain hs in this group
#pragma unroll
            for (int nt = 0; nt < NTA; ++nt) {
#pragma unroll
              for (int m = 0; m < C::NM; ++m) {
                const uint32_t af[4] = {a8[m][4 * hs], a8[m][4 * hs + 1], a8[m][4 * hs + 2],
                                        a8[m][4 * hs + 3]};
                mma_bf16_acc(tmp[hs][m][nt], af, b[nt][st].x, b[nt][st].y, first);
              }
              mma_bf16_acc(tH[hs][nt], ones, b[nt][st].x, b[nt][st].y, first);
            }
          }
        }
        // end of group `half`: acc += s * sum(q h) + m * sum(h)
#pragma unroll
        for (int nt = 0; nt < NTA; ++nt) {
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            if (ONECOL && (c & 1)) continue;
            const float hsum = tH[0][nt][c] + tH[1][nt][c];
#pragma unroll
            for (int m = 0; m < C::NM; ++m) {
              const uint32_t sv = half ? sc[m].y : sc[m].x;
              const uint32_t mv = half ? sc[m].w : sc[m].z;
              const float sf = c < 2 ? half_lo(sv) : half_hi(sv);
              const float mf = c < 2 ? half_lo(mv) : half_hi(mv);
              acc[m][nt][c] = fmaf(sf, tmp[0][m][nt][c] + tmp[1][m][nt][c], fmaf(mf, hsum, acc[m][nt][c]));
            }
          }
        }
      }
    }
  }

  // Consume the item's NTILE tiles, `tps` tiles per ring slot; returns false
  // on a wait timeout.
  static MOE_DEV bool run(WarpRing &r, const GemvParams &p, const ItemGeom &geo, int lane, int rb,
                          const BRows &br, const int (&epair)[NTA][2]) {
    const int tig = lane & 3, g = lane >> 2;
    const int tps = geo.tps;
    const uint32_t slot_bytes = (uint32_t)(tps * C::STRIDE);
    float acc[C::NM][NTA][4];
#pragma unroll
    for (int m = 0; m < C::NM; ++m)
#pragma unroll
      for (int nt = 0; nt < NTA; ++nt)
#pragma unroll
        for (int c = 0; c < 4; ++c) acc[m][nt][c] = 0.f;
    for (int t0 = 0; t0 < geo.NTILE; t0 += tps) {
      if (!mbar_wait_bounded(r.bar_s + 8 * r.u, r.phase)) return false;
      const uint32_t slot_s = r.data_s + r.u * slot_bytes;
      for (int tt = 0; tt < tps; ++tt) {
        uint2 b[NTA][C::STEPS];
        load_b(b, br, t0 + tt, tig);
        tile(slot_s + tt * C::STRIDE, lane, b, acc);
      }
      __syncwarp();
      if (lane == 0) ring_issue(r, p, geo, r.u);
      if (++r.u == C::D) {
        r.u = 0;
        r.phase ^= 1u;
      }
    }
#pragma unroll
    for (int nt = 0; nt < NTA; ++nt) {
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        if (ONECOL && (c & 1)) continue;
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
    return true;
  }
};

// Persistent grouped dequant-GEMV kernel (see the top of this file).  NTM is
// the largest number of 8-token column tiles of a job (jobs hold <= 8*NTM
// tokens); windows of <= 8 tokens use NTM = 1, 16 warps and a register file
// of 128 per thread.
template <int FMT, bool GATED, int NTM>
__global__ void __launch_bounds__(GemvCfg<FMT, GATED, NTM>::WARPS * 32, 1)
    expert_gemv_kernel(GemvParams p) {
  using C = GemvCfg<FMT, GATED, NTM>;
  extern __shared__ __align__(128) unsigned char smem[];
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int g = lane >> 2, tig = lane & 3;

  MOE_TRACE(GATED ? kTrGateStart : kTrDownStart);
  if (GATED) {
    pdl_wait();
    pdl_launch_dependents();
    MOE_TRACE(kTrGateWaited);
  }
  WarpRing r;
  r.data_s = smem_addr(smem + wid * C::D * 2 * C::STRIDE);
  r.bar_s = smem_addr(smem + C::RING) + wid * C::D * 8;
  r.u = 0;
  r.phase = 0;
  const uint32_t stage_bar = smem_addr(smem + C::RING) + C::WARPS * C::D * 8;
  const uint32_t stage_s = smem_addr(smem + C::STAGE_OFF);
  if (lane == 0) {
    for (int u = 0; u < C::D; ++u) mbar_init(r.bar_s + 8 * u, 1);
    if (wid == 0) mbar_init(stage_bar, 1);
    fence_mbar_init();
  }
  __syncthreads();

  // this CTA's contiguous range of (job, row-block) items
  const int n_jobs = ldcg_i32(p.n_jobs);
  const int RB = p.R / 16, NTILE = p.K / C::TK;
  const long long n_items = (long long)n_jobs * RB;
  const int i0 = (int)(n_items * blockIdx.x / gridDim.x);
  const int i1 = (int)(n_items * (blockIdx.x + 1) / gridDim.x);
  ItemGeom geo;
  geo.first = i0 + wid;
  geo.step = C::WARPS;
  geo.my_items = i1 > geo.first ? (i1 - geo.first + C::WARPS - 1) / C::WARPS : 0;
  geo.RB = RB;
  geo.NTILE = NTILE;
  geo.tps = NTILE % 2 == 0 ? 2 : 1;
  geo.stride = C::STRIDE;
  geo.region_off = p.region_off;

  // weight stream: D tiles in flight per warp (weights do not depend on the
  // previous kernel, so the down projection starts streaming before its wait)
  r.pj = 0;
  r.pt = 0;
  r.pbase = geo.my_items ? item_base(p, geo, 0) : nullptr;
  if (lane == 0)
    for (int u = 0; u < C::D; ++u) ring_issue(r, p, geo, u);
  if (!GATED) {
    pdl_wait();
    MOE_TRACE(kTrDownWaited);
  }

  // Stage the B rows of this CTA's first jobs (as many whole jobs as fit, at
  // most kMaxStagedJobs).  Every warp derives the same plan from one
  // parallel read of the job sizes: lane l describes job jfirst + l.
  const uint32_t RS = (uint32_t)p.K * 2 + 32;  // padded row stride (bank spread)
  const int jfirst = i0 / RB;
  const int njobs_cta = i1 > i0 ? (i1 - 1) / RB - jfirst + 1 : 0;
  int pn = 0, pbeg = 0;
  if (lane < njobs_cta && lane < kMaxStagedJobs) {
    pn = ldcg_i32(p.job_n + jfirst + lane);
    pbeg = ldcg_i32(p.job_beg + jfirst + lane);
  }
  int incl = pn;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  const int row0 = incl - pn;  // first staging row of job jfirst + lane
  const int cap = C::STAGE_BYTES / (int)RS;
  const int nst = __popc(__ballot_sync(0xffffffffu, pn > 0 && incl <= cap));
  const int used = nst ? __shfl_sync(0xffffffffu, incl, nst - 1) : 0;
  if (wid == 0) {
    if (lane == 0) mbar_expect_tx(stage_bar, (uint32_t)used * p.K * 2);  // the one arrival
    __syncwarp();
    for (int r0 = 0; r0 < used; r0 += 32) {  // uniform trip count: shuffles inside
      const int r = r0 + lane;
      int sj = 0;
      for (int q = 1; q < nst; ++q) sj += r >= __shfl_sync(0xffffffffu, row0, q) ? 1 : 0;
      const int beg = __shfl_sync(0xffffffffu, pbeg, sj);
      const int rj = r - __shfl_sync(0xffffffffu, row0, sj);
      if (r < used) {
        const int pair = ldcg_i32(p.plist + beg + rj);
        const int row = p.src_by_pair ? pair : (pair < p.Tk ? pair / p.k : pair - p.Tk);
        bulk_g2s(stage_s + (uint32_t)r * RS, p.src + (long long)row * p.K, (uint32_t)p.K * 2,
                 stage_bar);
      }
    }
  }
  bool staged_ready = false;

  for (int j = 0; j < geo.my_items; ++j) {
    const int item = geo.first + j * geo.step;
    const int job = item / RB, rb = item - job * RB;
    const int n = ldcg_i32(p.job_n + job), beg = ldcg_i32(p.job_beg + job);
    const int sj = job - jfirst;
    BRows br;
    br.smem = sj >= 0 && sj < nst;
    const int jrow0 = __shfl_sync(0xffffffffu, row0, br.smem ? sj : 0);
    if (br.smem && !staged_ready) {
      if (!mbar_wait_bounded(stage_bar, 0)) {
        if (lane == 0) atomicOr(p.status, kErrTimeout);
        return;
      }
      staged_ready = true;
    }
    int epair[C::NT][2];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      br.s[nt] = 0;
      br.gp[nt] = nullptr;
    }
#pragma unroll
    for (int nt = 0; nt < C::NT; ++nt) {
      const int ni = nt * 8 + g;
      if (ni < n) {
        if (br.smem) {
          br.s[nt] = stage_s + (uint32_t)(jrow0 + ni) * RS;
        } else {
          const int pair = ldcg_i32(p.plist + beg + ni);
          const int row = p.src_by_pair ? pair : (pair < p.Tk ? pair / p.k : pair - p.Tk);
          br.gp[nt] = p.src + (long long)row * p.K;
        }
      }
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        const int nc = nt * 8 + 2 * tig + c;
        epair[nt][c] = nc < n ? ldcg_i32(p.plist + beg + nc) : -1;
      }
    }
    bool ok;
    if (NTM == 1 || n <= 8) {
      const int e1[1][2] = {{epair[0][0], epair[0][1]}};
      if (n == 1)
        ok = br.smem ? ItemRun<FMT, GATED, 1, true, true>::run(r, p, geo, lane, rb, br, e1)
                     : ItemRun<FMT, GATED, 1, true, false>::run(r, p, geo, lane, rb, br, e1);
      else
        ok = br.smem ? ItemRun<FMT, GATED, 1, false, true>::run(r, p, geo, lane, rb, br, e1)
                     : ItemRun<FMT, GATED, 1, false, false>::run(r, p, geo, lane, rb, br, e1);
    } else {
      ok = br.smem ? ItemRun<FMT, GATED, NTM, false, true>::run(r, p, geo, lane, rb, br, epair)
                   : ItemRun<FMT, GATED, NTM, false, false>::run(r, p, geo, lane, rb, br, epair);
    }
    if (!ok) {
      if (lane == 0) atomicOr(p.status, kErrTimeout);
      return;
    }
    if (j == 0 && GATED) MOE_TRACE(kTrGateFirstTile);
  }
  if (lane == 0) trace_point(GATED ? kTrGateEnd : kTrDownEnd);
}

}  // namespace moe
