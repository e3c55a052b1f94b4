// gemv.cuh -- grouped dequant-GEMV of the decode path (sm_100a).
//
// Computes, for every job (an expert with up to 8*NTM of its tokens), either
// the gated half of the SwiGLU expert, a = SiLU(Wg h) * (Wu h), or the down
// projection y = Wd a.  The expert weights dominate the layer's HBM traffic
// (Strata engine analysis article "93 token/s on one 8 GB card", section
// "Expert cache": the expert bytes are the largest single cost and the
// kernel is memory-bound), so everything is built around streaming each
// selected expert's packed codes exactly once:
//
//  * Work items are (job, block of 16 output rows), ordered job-major; an
//    item is NTILE tiles of the reduction, streamed as UPI units of tps
//    tiles (one ring slot each).
//  * Each warp streams the weight tiles of its units through a private ring
//    of kRingD shared-memory slots filled by 1-D bulk (TMA) copies, kRingD
//    units in flight across item boundaries.  A tile is one 16-row x
//    TK-column block of codes (512 B, laid out so each lane's 16 bytes are
//    its own mma fragments) followed by the block's fp16 scales (and mins).
//  * Codes become exact bf16 values in registers (one LOP3 per pair of Q4
//    codes: 128 + c) and go through mma.m16n8k16 with fp32 accumulation
//    against up to 8*NTM token columns.  The offset is removed inside the
//    mma: the accumulator of each quantisation group starts at -136 * sum(h)
//    (from an mma of the same B fragments against ones), so the group sum
//    leaves the tensor core as sum((c - 8) h) and one FFMA per output entry
//    applies the group's scale.
//  * The B operand (token rows of h, or rows of a) is read from shared memory
//    with one 16-byte load per lane per two k-steps: the tile layout assigns
//    lane t of a quad the reduction columns [8t, 8t+8) of every 32-column
//    block, so those 16 bytes are exactly its two B fragments.
//
// expert_gemv_kernel gives every warp whole items (round-robin over the
// CTA's contiguous item range); the single-launch decode kernel in decode.cuh
// splits the unit stream evenly over all warps instead.
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
  __half *out_y16;     // down, instead of out_y when set: fp16 y [pairs][R]
  int *status;
};

constexpr int kGemvSmem = 220 * 1024;  // dynamic shared memory per CTA
constexpr int kMaxStagedJobs = 8;
constexpr int kRingD = 3;              // ring slots per warp

template <int FMT, bool GATED, int NTM = 1>
struct GemvCfg {
  static constexpr int TK = FMT == 1 ? 64 : 128;
  static constexpr int TILE = FMT == 1 ? 576 : 640;
  static constexpr int NM = GATED ? 2 : 1;
  static constexpr int STRIDE = NM * TILE;
  static constexpr int SLOT = 2 * STRIDE;  // a slot holds up to two tiles
  static constexpr int NT = NTM;           // 8-token mma column tiles per job (max)
  static constexpr int WARPS = NTM == 1 ? 16 : 8;  // register file: 128 / 255 per thread
  static constexpr int STEPS = TK / 16;    // mma k-steps per tile
  static constexpr int RING = WARPS * kRingD * SLOT;
  static constexpr int BARS = WARPS * kRingD * 8 + 8;  // ring barriers + staging barrier
  static constexpr int STAGE_OFF = (RING + BARS + 127) / 128 * 128;
  static constexpr int STAGE_BYTES = kGemvSmem - STAGE_OFF;
};

// One GEMV pass over the job list (gate/up or down).
struct Phase {
  const unsigned long long *job_ptr;  // expert base address per job (global or shared)
  int RB;                // 16-row blocks per job
  int NTILE;             // tiles per item
  int tps;               // tiles per unit (ring slot)
  int UPI;               // units per item
  int stride;            // bytes per tile, all matrices of the pass
  long long region_off;  // byte offset of the pass's region inside an expert
};

// Units are 4, 2 or 1 tiles: the most that divide the item's tiles and fit
// one ring slot of slot_bytes (0: two tiles' worth).
MOE_DEV Phase make_phase(const unsigned long long *job_ptr, int R, int K, int TK, int stride,
                         long long region_off, int slot_bytes = 0) {
  Phase ph;
  ph.job_ptr = job_ptr;
  ph.RB = R / 16;
  ph.NTILE = K / TK;
  if (slot_bytes <= 0) slot_bytes = 2 * stride;
  ph.tps = ph.NTILE % 4 == 0 && 4 * stride <= slot_bytes ? 4 : ph.NTILE % 2 == 0 ? 2 : 1;
  ph.UPI = ph.NTILE / ph.tps;
  ph.stride = stride;
  ph.region_off = region_off;
  return ph;
}

// First byte of item (job, rb) of the pass.
MOE_DEV const unsigned char *item_base(const Phase &ph, int job, int rb) {
  return reinterpret_cast<const unsigned char *>(ph.job_ptr[job]) + ph.region_off +
         (long long)rb * ph.NTILE * ph.stride;
}

// A walk over consecutive weight units: n units from unit `unit` of item
// (job, rb); the next item is istep row blocks further.  Only increments and
// compares: no division per unit or item.
struct UnitCursor {
  int rem, job, rb, unit;
  const unsigned char *addr;
};

MOE_DEV void cursor_start(UnitCursor &c, const Phase &ph, int job, int rb, int unit, int n) {
  c.rem = n;
  c.job = job;
  c.rb = rb;
  c.unit = unit;
  c.addr = n > 0 ? item_base(ph, job, rb) + (long long)unit * ph.tps * ph.stride : nullptr;
}

MOE_DEV void cursor_advance(UnitCursor &c, const Phase &ph, int istep) {
  --c.rem;
  c.addr += ph.tps * ph.stride;
  if (++c.unit == ph.UPI) {
    c.unit = 0;
    c.rb += istep;
    while (c.rb >= ph.RB) {
      c.rb -= ph.RB;
      ++c.job;
    }
    if (c.rem > 0) c.addr = item_base(ph, c.job, c.rb);
  }
}

// Per-warp streaming state.  The consumer fields (u, phase) are kept by
// every lane; the producer cursor only by lane 0, which issues each unit
// into the slot the consumer has just released, kRingD units ahead.  The
// loads carry an evict-first L2 policy: a weight line is read once.
struct WarpRing {
  uint32_t data_s, bar_s, slot_stride;
  int u;             // slot of the next unit to consume
  uint32_t phase;    // its mbarrier parity
  int inflight;      // units issued and not yet consumed
  int istep;
  UnitCursor ld;      // next unit to load into the ring
  uint64_t policy;   // L2 policy of the ring loads (evict first)
};

MOE_DEV void ring_init(WarpRing &r, uint32_t data_s, uint32_t bar_s, uint32_t slot_stride) {
  r.data_s = data_s;
  r.bar_s = bar_s;
  r.slot_stride = slot_stride;
  r.u = 0;
  r.phase = 0;
  r.inflight = 0;
  r.istep = 1;
  r.ld.rem = 0;
  r.policy = l2_evict_first();
}

// Point the producer at n units starting at unit `unit` of item (job, rb);
// consecutive items are istep row blocks apart.
MOE_DEV void ring_start(WarpRing &r, const Phase &ph, int job, int rb, int unit, int n, int istep) {
  r.istep = istep;
  cursor_start(r.ld, ph, job, rb, unit, n);
}

// Every lane: the producer's next unit into slot `slot`, issued by lane 0
// alone (predicated, no divergent branch); every lane keeps the cursor.  The
// slot's previous unit was read with ld.shared by every lane, and those reads
// are ordered before this copy by the __syncwarp that precedes the call (the
// values were consumed by then), as in a TMA pipeline's consumer release.
MOE_DEV void ring_issue_warp(WarpRing &r, const Phase &ph, int slot, int lane) {
  if (r.ld.rem <= 0) return;
  const uint32_t bytes = (uint32_t)(ph.tps * ph.stride);
  bulk_g2s_hint_pred(lane == 0, r.data_s + slot * r.slot_stride, r.ld.addr, bytes, r.bar_s + 8 * slot,
                     r.policy);
  ++r.inflight;
  cursor_advance(r.ld, ph, r.istep);
}

// Every lane: fill the kRingD slots that follow the consumer position
// (lane 0 issues).
MOE_DEV void ring_prologue(WarpRing &r, const Phase &ph, int lane) {
  for (int i = 0; i < kRingD; ++i) ring_issue_warp(r, ph, (r.u + i) % kRingD, lane);
}

// After a failed wait (all lanes of the warp): wait, bounded, for the units
// still in flight so no bulk copy lands in shared memory after the warp has
// moved on, and leave the ring empty and consistent.
MOE_DEV void ring_drain(WarpRing &r) {
  const int n = __shfl_sync(0xffffffffu, r.inflight, 0);
  for (int i = 0; i < n; ++i) {
    (void)mbar_wait_bounded(r.bar_s + 8 * r.u, r.phase);
    if (++r.u == kRingD) {
      r.u = 0;
      r.phase ^= 1u;
    }
  }
  r.inflight = 0;
  r.ld.rem = 0;
}

// The lane's B rows for the current item (its token column g of each 8-token
// column tile): generic addresses of rows staged in shared memory or of rows
// in global memory; null = no token.  With a sum table (HTAB), hc[nt][c] is
// the table row of the token in accumulator column 2 tig + c: one float per
// quantisation group of the reduction (see ItemRun::tile); null = no token.
struct BRows {
  const uint16_t *row[2];
  const float *hc[2][2];
};

MOE_DEV float2 ld_f2(const float *p) {
  float2 r;
  asm volatile("ld.v2.f32 {%0,%1}, [%2];" : "=f"(r.x), "=f"(r.y) : "l"(p));
  return r;
}

MOE_DEV uint4 ld_v4(const void *p) {
  uint4 r;
  asm volatile("ld.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
  return r;
}

// One item (16 output rows of one job) of the streaming GEMV; NTA = 8-token
// column tiles of the job (1 or 2).  The per-group sums of the B rows that
// the tile math needs come either from a table (HTAB: -136 sum(h) for Q4,
// sum(h) for Q2, per row and group, computed once per call) or from an mma
// of the B fragments against ones.
template <int FMT, bool GATED, int NTA, bool HTAB = false>
struct ItemRun {
  using C = GemvCfg<FMT, GATED>;  // tile geometry does not depend on NTM or WARPS
  static constexpr int NB = C::STEPS / 2;  // 16-byte B loads per tile and column tile

  // B fragments of tile t: b[nt][q] holds k-steps 2q (x, y) and 2q+1 (z, w);
  // with HTAB, hv[nt][c] = the table entries of the tile's groups 2t, 2t+1
  // for accumulator column 2 tig + c
  static MOE_DEV void load_b(uint4 (&b)[NTA][NB], float2 (&hv)[NTA][2], const BRows &br, int t,
                             int tig) {
#pragma unroll
    for (int nt = 0; nt < NTA; ++nt) {
#pragma unroll
      for (int q = 0; q < NB; ++q) {
        const int col = t * C::TK + 32 * q + 8 * tig;
        b[nt][q] = br.row[nt] ? ld_v4(br.row[nt] + col) : make_uint4(0u, 0u, 0u, 0u);
      }
      if constexpr (HTAB) {
#pragma unroll
        for (int c = 0; c < 2; ++c)
          hv[nt][c] = br.hc[nt][c] ? ld_f2(br.hc[nt][c] + 2 * t) : make_float2(0.f, 0.f);
      }
    }
  }

  // acc += this tile's contribution.  c runs over the accumulator entries:
  // (row g, col 2tig), (row g, col 2tig+1), (row g+8, col 2tig), (row g+8, col 2tig+1).
  static MOE_DEV void tile(uint32_t tile_s, int lane, const uint4 (&b)[NTA][NB],
                           const float2 (&hv)[NTA][2], float (&acc)[C::NM][NTA][4]) {
    const int g = lane >> 2;
    const uint32_t ones[4] = {0x3F803F80u, 0x3F803F80u, 0x3F803F80u, 0x3F803F80u};
    uint4 cw[C::NM];
#pragma unroll
    for (int m = 0; m < C::NM; ++m) cw[m] = lds_u4(tile_s + m * C::TILE + lane * 16);
    if constexpr (FMT == 1) {
      // two groups of 32 columns per tile, two k-steps each
      uint2 sc[C::NM];
#pragma unroll
      for (int m = 0; m < C::NM; ++m) sc[m] = lds_u2(tile_s + m * C::TILE + 512 + g * 8);
#pragma unroll
      for (int grp = 0; grp < 2; ++grp) {
        uint32_t a[C::NM][2][4];  // bf16 128 + c
#pragma unroll
        for (int m = 0; m < C::NM; ++m)
#pragma unroll
          for (int st = 0; st < 2; ++st) {
            const uint32_t w = grp == 0 ? (st == 0 ? cw[m].x : cw[m].y) : (st == 0 ? cw[m].z : cw[m].w);
#pragma unroll
            for (int i = 0; i < 4; ++i) a[m][st][i] = lop3_and_or(w >> (4 * i), 0x000F000Fu, 0x43004300u);
          }
#pragma unroll
        for (int nt = 0; nt < NTA; ++nt) {
          const uint4 bb = b[nt][grp];
          float ci[4];
          if constexpr (HTAB) {
            const float h0 = grp ? hv[nt][0].y : hv[nt][0].x, h1 = grp ? hv[nt][1].y : hv[nt][1].x;
            ci[0] = h0;
            ci[1] = h1;
            ci[2] = h0;
            ci[3] = h1;
          } else {
            float hs[4];
            mma_bf16_acc(hs, ones, bb.x, bb.y, true);
            mma_bf16_16816(hs, ones, bb.z, bb.w, hs);
#pragma unroll
            for (int c = 0; c < 4; ++c) ci[c] = -136.f * hs[c];
          }
#pragma unroll
          for (int m = 0; m < C::NM; ++m) {
            float tmp[4];
            mma_bf16_16816(tmp, a[m][0], bb.x, bb.y, ci);
            mma_bf16_16816(tmp, a[m][1], bb.z, bb.w, tmp);
            const uint32_t sv = grp ? sc[m].y : sc[m].x;
            const float s0 = half_lo(sv), s1 = half_hi(sv);
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              acc[m][nt][c] = fmaf(c < 2 ? s0 : s1, tmp[c], acc[m][nt][c]);
            }
          }
        }
      }
    } else {
      // two groups of 64 columns per tile, four k-steps (two code words) each;
      // y += s * sum(q h) + min * sum(h)
      uint4 sc[C::NM];
#pragma unroll
      for (int m = 0; m < C::NM; ++m) sc[m] = lds_u4(tile_s + m * C::TILE + 512 + g * 16);
#pragma unroll
      for (int grp = 0; grp < 2; ++grp) {
        float hs[NTA][4], tmp[C::NM][NTA][4];
#pragma unroll
        for (int wv = 0; wv < 2; ++wv) {
          uint32_t a8[C::NM][8];
#pragma unroll
          for (int m = 0; m < C::NM; ++m) {
            const int wi = 2 * grp + wv;
            const uint32_t w = wi == 0 ? cw[m].x : wi == 1 ? cw[m].y : wi == 2 ? cw[m].z : cw[m].w;
            unpack_q2(w, a8[m]);
          }
#pragma unroll
          for (int nt = 0; nt < NTA; ++nt) {
            const uint4 bb = b[nt][2 * grp + wv];
#pragma unroll
            for (int hs2 = 0; hs2 < 2; ++hs2) {
              const bool first = wv == 0 && hs2 == 0;
              const uint32_t b0 = hs2 ? bb.z : bb.x, b1 = hs2 ? bb.w : bb.y;
              if constexpr (!HTAB) mma_bf16_acc(hs[nt], ones, b0, b1, first);
#pragma unroll
              for (int m = 0; m < C::NM; ++m) {
                const uint32_t af[4] = {a8[m][4 * hs2], a8[m][4 * hs2 + 1], a8[m][4 * hs2 + 2],
                                        a8[m][4 * hs2 + 3]};
                mma_bf16_acc(tmp[m][nt], af, b0, b1, first);
              }
            }
          }
        }
        if constexpr (HTAB) {
#pragma unroll
          for (int nt = 0; nt < NTA; ++nt) {
            const float h0 = grp ? hv[nt][0].y : hv[nt][0].x, h1 = grp ? hv[nt][1].y : hv[nt][1].x;
            hs[nt][0] = h0;
            hs[nt][1] = h1;
            hs[nt][2] = h0;
            hs[nt][3] = h1;
          }
        }
#pragma unroll
        for (int m = 0; m < C::NM; ++m) {
          const uint32_t sv = grp ? sc[m].y : sc[m].x, mv = grp ? sc[m].w : sc[m].z;
          const float s0 = half_lo(sv), s1 = half_hi(sv), m0 = half_lo(mv), m1 = half_hi(mv);
#pragma unroll
          for (int nt = 0; nt < NTA; ++nt)
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              acc[m][nt][c] = fmaf(c < 2 ? s0 : s1, tmp[m][nt][c],
                                   fmaf(c < 2 ? m0 : m1, hs[nt][c], acc[m][nt][c]));
            }
        }
      }
    }
  }

  // Consume units [ua, ub) of the current item (acc starts at zero).
  // Returns false on a wait timeout.
  static MOE_DEV bool run(WarpRing &r, const Phase &ph, int lane, int ua, int ub, const BRows &br,
                          float (&acc)[C::NM][NTA][4]) {
    const int tig = lane & 3;
#pragma unroll
    for (int m = 0; m < C::NM; ++m)
#pragma unroll
      for (int nt = 0; nt < NTA; ++nt)
#pragma unroll
        for (int c = 0; c < 4; ++c) acc[m][nt][c] = 0.f;
    for (int u = ua; u < ub; ++u) {
      const bool ok = mbar_wait_bounded(r.bar_s + 8 * r.u, r.phase);
      if (__any_sync(0xffffffffu, !ok)) return false;  // warp-uniform
      const uint32_t slot_s = r.data_s + r.u * r.slot_stride;
      if (ph.tps == 4) {
        // two straight-line blocks of two tiles each
#pragma unroll 1
        for (int hp = 0; hp < 2; ++hp) {
          uint4 b0[NTA][NB], b1[NTA][NB];
          float2 hv0[NTA][2], hv1[NTA][2];
          load_b(b0, hv0, br, 4 * u + 2 * hp, tig);
          load_b(b1, hv1, br, 4 * u + 2 * hp + 1, tig);
          tile(slot_s + 2 * hp * C::STRIDE, lane, b0, hv0, acc);
          tile(slot_s + (2 * hp + 1) * C::STRIDE, lane, b1, hv1, acc);
        }
      } else if (ph.tps == 2) {
        // both tiles of the unit in one block of straight-line code, so the
        // scheduler can overlap one tile's unpack with the other's mma chains
        uint4 b0[NTA][NB], b1[NTA][NB];
        float2 hv0[NTA][2], hv1[NTA][2];
        load_b(b0, hv0, br, 2 * u, tig);
        load_b(b1, hv1, br, 2 * u + 1, tig);
        tile(slot_s, lane, b0, hv0, acc);
        tile(slot_s + C::STRIDE, lane, b1, hv1, acc);
      } else {
        uint4 b[NTA][NB];
        float2 hv[NTA][2];
        load_b(b, hv, br, u, tig);
        tile(slot_s, lane, b, hv, acc);
      }
      __syncwarp();
      --r.inflight;
      ring_issue_warp(r, ph, r.u, lane);
      if (++r.u == kRingD) {
        r.u = 0;
        r.phase ^= 1u;
      }
    }
    return true;
  }

  // Write the item's outputs: a = bf16(SiLU(g) * u) (gated) or y (down).
  static MOE_DEV void store(const float (&acc)[C::NM][NTA][4], const int (&epair)[2][2], int rb,
                            int lane, int R, uint16_t *out_a, float *out_y, __half *out_y16 = nullptr) {
    const int g = lane >> 2;
#pragma unroll
    for (int nt = 0; nt < NTA; ++nt) {
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int pair = epair[nt][c & 1];
        if (pair < 0) continue;
        const int row = rb * 16 + g + (c >= 2 ? 8 : 0);
        if constexpr (GATED) {
          const float gv = acc[0][nt][c], uv = acc[C::NM - 1][nt][c];
          const float av = gv / (1.0f + __expf(-gv)) * uv;
          out_a[(long long)pair * R + row] = __bfloat16_as_ushort(__float2bfloat16_rn(av));
        } else {
          if (out_y16)
            out_y16[(long long)pair * R + row] = __float2half_rn(acc[0][nt][c]);
          else
            out_y[(long long)pair * R + row] = acc[0][nt][c];
        }
      }
    }
  }
};

// Runs one whole item and stores it (expert_gemv_kernel).
template <int FMT, bool GATED, int NTA>
MOE_DEV bool whole_item(WarpRing &r, const Phase &ph, const GemvParams &p, int lane, int rb,
                        const BRows &br, const int (&epair)[2][2]) {
  using Run = ItemRun<FMT, GATED, NTA>;
  float acc[Run::C::NM][NTA][4];
  if (!Run::run(r, ph, lane, 0, ph.UPI, br, acc)) return false;
  Run::store(acc, epair, rb, lane, p.R, p.out_a, p.out_y, p.out_y16);
  return true;
}

// Grouped dequant-GEMV over a job list built by the routing kernels (windows
// of more than 32 tokens).  NTM is the largest number of 8-token column tiles
// of a job (jobs hold <= 8*NTM tokens); windows of <= 8 tokens use NTM = 1,
// 16 warps and a register file of 128 per thread.
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
  ring_init(r, smem_addr(smem + wid * kRingD * C::SLOT), smem_addr(smem + C::RING) + wid * kRingD * 8,
            C::SLOT);
  const uint32_t stage_bar = smem_addr(smem + C::RING) + C::WARPS * kRingD * 8;
  const uint32_t stage_s = smem_addr(smem + C::STAGE_OFF);
  if (lane == 0) {
    for (int u = 0; u < kRingD; ++u) mbar_init(r.bar_s + 8 * u, 1);
    if (wid == 0) mbar_init(stage_bar, 1);
    fence_mbar_init();
  }
  __syncthreads();

  // this CTA's contiguous range of (job, row-block) items
  const int n_jobs = ldcg_i32(p.n_jobs);
  const Phase ph = make_phase(p.job_ptr, p.R, p.K, C::TK, C::STRIDE, p.region_off);
  const int RB = ph.RB;
  const long long n_items = (long long)n_jobs * RB;
  const int i0 = (int)(n_items * blockIdx.x / gridDim.x);
  const int i1 = (int)(n_items * (blockIdx.x + 1) / gridDim.x);
  const int first = i0 + wid;
  const int my_items = i1 > first ? (i1 - first + C::WARPS - 1) / C::WARPS : 0;

  // weight stream: kRingD units in flight per warp (weights do not depend on
  // the previous kernel, so the down projection starts streaming before its
  // wait)
  ring_start(r, ph, first / RB, first % RB, 0, my_items * ph.UPI, C::WARPS);
  ring_prologue(r, ph, lane);
  if (!GATED) {
    pdl_wait();
    MOE_TRACE(kTrDownWaited);
  }

  // Stage the B rows of this CTA's first jobs (as many whole jobs as fit, at
  // most kMaxStagedJobs).  Every warp derives the same plan from one
  // parallel read of the job sizes: lane l describes job jfirst + l.
  const uint32_t RS = (uint32_t)p.K * 2 + 64;  // padded row stride (bank spread)
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
      const int rr = r0 + lane;
      int sj = 0;
      for (int q = 1; q < nst; ++q) sj += rr >= __shfl_sync(0xffffffffu, row0, q) ? 1 : 0;
      const int beg = __shfl_sync(0xffffffffu, pbeg, sj);
      const int rj = rr - __shfl_sync(0xffffffffu, row0, sj);
      if (rr < used) {
        const int pair = ldcg_i32(p.plist + beg + rj);
        const int row = p.src_by_pair ? pair : (pair < p.Tk ? pair / p.k : pair - p.Tk);
        bulk_g2s(stage_s + (uint32_t)rr * RS, p.src + (long long)row * p.K, (uint32_t)p.K * 2,
                 stage_bar);
      }
    }
  }
  bool staged_ready = false;

  for (int j = 0; j < my_items; ++j) {
    const int item = first + j * C::WARPS;
    const int job = item / RB, rb = item - job * RB;
    const int n = ldcg_i32(p.job_n + job), beg = ldcg_i32(p.job_beg + job);
    const int sj = job - jfirst;
    const bool staged = sj >= 0 && sj < nst;
    const int jrow0 = __shfl_sync(0xffffffffu, row0, staged ? sj : 0);
    if (staged && !staged_ready) {
      if (__any_sync(0xffffffffu, !mbar_wait_bounded(stage_bar, 0))) {
        if (lane == 0) atomicOr(p.status, kErrTimeout);
        ring_drain(r);
        return;
      }
      staged_ready = true;
    }
    BRows br;
    int epair[2][2];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      br.row[nt] = nullptr;
      br.hc[nt][0] = br.hc[nt][1] = nullptr;
      epair[nt][0] = epair[nt][1] = -1;
    }
#pragma unroll
    for (int nt = 0; nt < C::NT; ++nt) {
      const int ni = nt * 8 + g;
      if (ni < n) {
        if (staged) {
          br.row[nt] = reinterpret_cast<const uint16_t *>(smem + C::STAGE_OFF + (size_t)(jrow0 + ni) * RS);
        } else {
          const int pair = ldcg_i32(p.plist + beg + ni);
          const int row = p.src_by_pair ? pair : (pair < p.Tk ? pair / p.k : pair - p.Tk);
          br.row[nt] = p.src + (long long)row * p.K;
        }
      }
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        const int nc = nt * 8 + 2 * tig + c;
        epair[nt][c] = nc < n ? ldcg_i32(p.plist + beg + nc) : -1;
      }
    }
    const bool ok = (NTM == 1 || n <= 8) ? whole_item<FMT, GATED, 1>(r, ph, p, lane, rb, br, epair)
                                         : whole_item<FMT, GATED, NTM>(r, ph, p, lane, rb, br, epair);
    if (!ok) {
      if (lane == 0) atomicOr(p.status, kErrTimeout);
      ring_drain(r);
      return;
    }
    if (j == 0 && GATED) MOE_TRACE(kTrGateFirstTile);
  }
  if (lane == 0) trace_point(GATED ? kTrGateEnd : kTrDownEnd);
}

}  // namespace moe
