// moe_api.cu -- host side of libmoe.so: the C ABI declared in include/moe.h.
//
// The context owns, in device memory (HBM):
//   arena   [L * E] experts in the repacked tile layout (every expert has a
//           backing copy here),
//   shared  [L] shared experts,
//   pool    [n_slots] residency slot pool; slot_of[l*E+e] >= 0 makes the
//           kernels read expert (l,e) from its slot (the "expert cache" of
//           the Strata engine analysis article, section "Expert cache":
//           (layer, expert) -> slot or -1),
//   router  fp32 W [L, E, d] and bias [L, E],
//   scratch sized for max_tokens tokens per call.
#include <cuda_runtime.h>

#include <algorithm>
#include <chrono>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <map>
#include <mutex>
#include <string>
#include <thread>
#include <utility>
#include <vector>

#include "../../include/moe.h"
#include "decode.cuh"
#include "kernels.cuh"
#include "prefill.cuh"
#include "ep.cuh"
#include "tier.h"

using namespace moe;

struct moe_ctx {
  int device = 0;
  int d = 0, f = 0, E = 0, k = 0, fmt = 0;
  int L = 1, n_shared = 0, n_slots = 0, max_tokens = 64;
  bool configured = false, any_loaded = false;
  Layout lay{};
  int n_sm = 0;
  int chunk_min = 8;  // smallest job size (sizes the job list)
  int max_jobs = 0;
  cudaStream_t io = nullptr;  // private stream for loads and status reads
  cudaStream_t last_stream = nullptr;  // stream of the most recent compute call

  uint8_t *arena = nullptr, *shared = nullptr, *pool = nullptr;
  int *d_slot_of = nullptr;
  std::vector<int> h_slot_of;
  // host tier: the backing arena in pinned, mapped host memory and the slot
  // pool as a cache over it (moe_set_host_tier)
  int host_tier = 0, tier_policy = 0;
  double tier_half_life = 64.0;
  uint8_t *h_arena = nullptr;            // host address of the arena (host tier)
  moe::TierCache tier;
  cudaStream_t tier_stream = nullptr;    // host -> HBM expert copies
  cudaStream_t pf_side = nullptr;        // the chunk's GEMV experts, beside the GEMM
  cudaEvent_t pf_fork = nullptr, pf_join = nullptr;
  cudaEvent_t tier_done = nullptr;       // the latest copies and slot-table update
  int32_t *tier_idx = nullptr;           // device [max_tokens * k] routing of the tiered forward
  float *tier_w = nullptr;
  int32_t *h_tier_idx = nullptr;         // pinned host copy of a window's routing
  long long tier_bytes = 0, tier_calls = 0;
  std::vector<int> tier_trace;           // per request: call, layer, n, then n expert ids
  float *d_router = nullptr, *d_bias = nullptr, *d_gamma = nullptr;
  __nv_bfloat16 *d_router3 = nullptr;  // [L][E][3d] exact bf16 parts of the router (prefill)
  std::vector<char> has_router, has_bias, has_norm, has_gamma, shared_loaded;
  std::vector<float> eps;
  std::vector<std::vector<char>> expert_loaded;
  std::vector<int> n_loaded;

  // scratch: views into one allocation (do_configure)
  uint8_t *scratch = nullptr;
  float *logits = nullptr, *w = nullptr, *ybuf = nullptr;
  int *idx = nullptr, *off = nullptr, *perm = nullptr, *plist = nullptr;
  unsigned long long *job_ptr = nullptr;
  int *job_beg = nullptr, *job_n = nullptr, *n_jobs = nullptr;
  uint16_t *hbuf = nullptr, *abuf = nullptr;
  int *status = nullptr, *cnt_out = nullptr, *last = nullptr;
  int *ep_counts = nullptr;  // expert-parallel dispatch: [kEpMaxRanks] rows per rank, then the
                             // blocks' per-rank counts and offsets
  long long ep_scratch_n = 0;
  unsigned int *ticket = nullptr;    // fused routing: [0] CTA counter, [1] abort flag
  // single-launch decode kernel: grid barrier counter, hand-over flags and
  // partial sums (one slot per warp of the grid)
  unsigned long long *dec_bar = nullptr, *dec_flags = nullptr;
  float *dec_ws = nullptr;
  size_t dec_sync_bytes = 0;  // bytes of the counter + flags block (cleared after a timeout)
  // prefill (grouped GEMM) buffers, present when max_tokens > kDecMaxT
  uint8_t *pf = nullptr;
  __half *pf_hg = nullptr;              // grouped A rows, fp16 [rows][d]
  int *pf_row_of = nullptr, *pf_boff = nullptr, *pf_eoff = nullptr, *pf_ntiles = nullptr;
  unsigned short *pf_bmask = nullptr;
  float *pf_part = nullptr;             // split router partial sums
  __half *pf_a16 = nullptr, *pf_y16 = nullptr;  // GEMM a and y, fp16 [rows][f], [rows][d]
  int *pf_perm = nullptr, *pf_hot = nullptr;     // bucket permutation [T*k], GEMM-expert flags [E]
  int *pf_colpart = nullptr;                     // [kPfColSplitMax][E] split column-scan counts
  long long pf_part_floats = 0;
  PfTile *pf_tiles = nullptr;
  int pf_max_tiles = 0, pf_rows = 0;
  CUtensorMap pf_map_h{}, pf_map_a{};   // TMA maps of the grouped A matrices
  CUtensorMap pf_omap_a{}, pf_omap_y{};  // TMA maps of the GEMMs' outputs (a, y)
  bool pf_maps = false;
  int pf_pairs = 0;  // co-resident CTA pairs of the grouped GEMM (0: it cannot run)
  unsigned long long *trace = nullptr;  // moe_set_trace buffer
  unsigned long long *stats = nullptr;
  std::vector<int32_t> host_counts;

  int gemv_blocks[2][2][2] = {};  // [fmt][gated][NTM-1]
  bool dec_fits = true;           // one decode_kernel CTA fits on every SM (checked at create)
  int dec_coop = -1;              // decode launches cooperative: -1 untried, 0 no, 1 yes
  int dec_stall_next = 0;         // test hook: the next decode launch's first barrier cannot complete
  uint32_t dec_stall_polls = 0;
  // profiling: 4 events per call slot
  bool profiling = false;
  std::vector<cudaEvent_t> prof_ev;
  int prof_next = 0, prof_pending = 0;
  std::map<std::pair<void *, int>, cudaGraphExec_t> stack_graphs;
  std::string err;
};

namespace {

moe_status fail(moe_ctx *c, moe_status s, const char *fmt, ...) {
  if (c) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    c->err = buf;
  }
  return s;
}

#define CUDA_TRY(c, expr)                                                              \
  do {                                                                                 \
    cudaError_t e_ = (expr);                                                           \
    if (e_ != cudaSuccess) {                                                           \
      (void)cudaGetLastError();                                                        \
      return fail(c, e_ == cudaErrorMemoryAllocation ? MOE_ERR_OOM : MOE_ERR_CUDA,     \
                  "%s: %s", #expr, cudaGetErrorString(e_));                            \
    }                                                                                  \
  } while (0)

template <typename P>
cudaError_t launch(void (*kern)(P), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                   const P &params, bool pdl = true) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, params);
}

template <int FMT, bool GATED, int NTM>
cudaError_t setup_gemv(int n_sm, int *blocks) {
  using C = GemvCfg<FMT, GATED, NTM>;
  cudaError_t e = cudaFuncSetAttribute(expert_gemv_kernel<FMT, GATED, NTM>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, kGemvSmem);
  if (e != cudaSuccess) return e;
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, expert_gemv_kernel<FMT, GATED, NTM>,
                                                    C::WARPS * 32, kGemvSmem);
  if (e != cudaSuccess) return e;
  *blocks = n_sm * (per_sm > 0 ? per_sm : 1);
  return cudaSuccess;
}

template <int FMT, bool GATED, int NTM>
cudaError_t launch_gemv(moe_ctx *c, cudaStream_t s, const GemvParams &gp) {
  using C = GemvCfg<FMT, GATED, NTM>;
  return launch(expert_gemv_kernel<FMT, GATED, NTM>,
                dim3(c->gemv_blocks[FMT - 1][GATED][NTM - 1]), dim3(C::WARPS * 32), kGemvSmem, s,
                gp);
}

// tokens per expert job: 8 for windows of <= 8 tokens (NTM = 1), else 16
int job_chunk(int T) { return T <= 8 ? 8 : 16; }

template <int FMT>
cudaError_t launch_experts(moe_ctx *c, cudaStream_t s, int T, const GemvParams &g1,
                           const GemvParams &g2) {
  cudaError_t e;
  if (job_chunk(T) == 8) {
    e = launch_gemv<FMT, true, 1>(c, s, g1);
    if (e == cudaSuccess) e = launch_gemv<FMT, false, 1>(c, s, g2);
  } else {
    e = launch_gemv<FMT, true, 2>(c, s, g1);
    if (e == cudaSuccess) e = launch_gemv<FMT, false, 2>(c, s, g2);
  }
  return e;
}

bool valid_layer(const moe_ctx *c, int layer) { return layer >= 0 && layer < c->L; }

// activations are read with 16-byte vector loads and bulk copies
bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }

template <typename T>
void dfree(T *&p) {
  if (p) cudaFree((void *)p);
  p = nullptr;
}

moe_status do_configure(moe_ctx *c) {
  const Layout &L = c->lay;
  const long long Be = L.expert_bytes;
  const int T = c->max_tokens, E = c->E, k = c->k, d = c->d, f = c->f;
  if (c->host_tier) {
    // every expert's backing copy in pinned host memory, mapped so that the
    // kernels can still address it; the HBM slot pool caches it
    CUDA_TRY(c, cudaHostAlloc((void **)&c->h_arena, (size_t)c->L * E * Be,
                              cudaHostAllocMapped | cudaHostAllocPortable));
    CUDA_TRY(c, cudaHostGetDevicePointer((void **)&c->arena, c->h_arena, 0));
    CUDA_TRY(c, cudaStreamCreateWithFlags(&c->tier_stream, cudaStreamNonBlocking));
    CUDA_TRY(c, cudaEventCreateWithFlags(&c->tier_done, cudaEventDisableTiming));
    CUDA_TRY(c, cudaMalloc(&c->tier_idx, (size_t)T * k * sizeof(int32_t)));
    CUDA_TRY(c, cudaMalloc(&c->tier_w, (size_t)T * k * sizeof(float)));
    CUDA_TRY(c, cudaHostAlloc((void **)&c->h_tier_idx, (size_t)T * k * sizeof(int32_t), cudaHostAllocDefault));
    c->tier.init(c->n_slots, c->tier_policy, c->tier_half_life, (long long)c->L * E);
  } else {
    CUDA_TRY(c, cudaMalloc(&c->arena, (size_t)c->L * E * Be));
  }
  if (c->n_shared) CUDA_TRY(c, cudaMalloc(&c->shared, (size_t)c->L * Be));
  if (c->n_slots) CUDA_TRY(c, cudaMalloc(&c->pool, (size_t)c->n_slots * Be));
  CUDA_TRY(c, cudaMalloc(&c->d_slot_of, (size_t)c->L * E * sizeof(int)));
  c->h_slot_of.assign((size_t)c->L * E, -1);
  CUDA_TRY(c, cudaMemset(c->d_slot_of, 0xFF, (size_t)c->L * E * sizeof(int)));
  CUDA_TRY(c, cudaMalloc(&c->d_router, (size_t)c->L * E * d * sizeof(float)));
  CUDA_TRY(c, cudaMalloc(&c->d_bias, (size_t)c->L * E * sizeof(float)));
  CUDA_TRY(c, cudaMalloc(&c->d_gamma, (size_t)c->L * d * sizeof(float)));
  const long long P = (long long)T * k, Ptot = P + T;
  c->max_jobs = (int)(P + E + (T + c->chunk_min - 1) / c->chunk_min + 8);
  // All per-call scratch lives in one allocation, small and hot buffers
  // first, so a call touches few pages (the expert stream evicts the
  // translations of scattered small buffers between calls).
  size_t off = 0;
  auto carve = [&](size_t bytes) {
    const size_t at = off;
    off += (bytes + 255) / 256 * 256;
    return at;
  };
  const size_t o_status = carve(sizeof(int)), o_ticket = carve(2 * sizeof(unsigned int));
  const size_t dec_warps = (size_t)c->n_sm * GemvCfg<1, true, 1>::WARPS;  // decode_kernel warps
  const size_t o_dbar = carve(sizeof(unsigned long long) * (1 + 2 * dec_warps));
  const size_t o_dws = carve(sizeof(float) * dec_warps * 32 * 16);
  const size_t o_njobs = carve(sizeof(int)), o_last = carve(4 * sizeof(int));
  const size_t o_stats = carve(8 * sizeof(unsigned long long));
  const size_t o_jptr = carve((size_t)c->max_jobs * sizeof(unsigned long long));
  const size_t o_jbeg = carve((size_t)c->max_jobs * sizeof(int));
  const size_t o_jn = carve((size_t)c->max_jobs * sizeof(int));
  const size_t o_idx = carve((size_t)P * sizeof(int)), o_w = carve((size_t)P * sizeof(float));
  const size_t o_off = carve((size_t)(E + 1) * sizeof(int)), o_perm = carve((size_t)P * sizeof(int));
  const size_t o_plist = carve((size_t)Ptot * sizeof(int)), o_cnt = carve((size_t)E * sizeof(int));
  const size_t o_logits = carve((size_t)T * E * sizeof(float));
  const size_t o_h = carve((size_t)T * d * 2), o_a = carve((size_t)Ptot * f * 2);
  const size_t o_y = carve((size_t)Ptot * d * sizeof(float));
  CUDA_TRY(c, cudaMalloc(&c->scratch, off));
  CUDA_TRY(c, cudaMemset(c->scratch, 0, off));
  uint8_t *b = c->scratch;
  c->status = (int *)(b + o_status);
  c->ticket = (unsigned int *)(b + o_ticket);
  c->dec_bar = (unsigned long long *)(b + o_dbar);
  c->dec_flags = c->dec_bar + 1;
  c->dec_sync_bytes = sizeof(unsigned long long) * (1 + 2 * dec_warps);
  c->dec_ws = (float *)(b + o_dws);
  c->n_jobs = (int *)(b + o_njobs);
  c->last = (int *)(b + o_last);
  c->stats = (unsigned long long *)(b + o_stats);
  c->job_ptr = (unsigned long long *)(b + o_jptr);
  c->job_beg = (int *)(b + o_jbeg);
  c->job_n = (int *)(b + o_jn);
  c->idx = (int *)(b + o_idx);
  c->w = (float *)(b + o_w);
  c->off = (int *)(b + o_off);
  c->perm = (int *)(b + o_perm);
  c->plist = (int *)(b + o_plist);
  c->cnt_out = (int *)(b + o_cnt);
  c->logits = (float *)(b + o_logits);
  c->hbuf = (uint16_t *)(b + o_h);
  c->abuf = (uint16_t *)(b + o_a);
  c->ybuf = (float *)(b + o_y);
  if (T > kDecMaxT) {  // prefill-capable: grouped-GEMM buffers
    CUDA_TRY(c, cudaStreamCreateWithFlags(&c->pf_side, cudaStreamNonBlocking));
    CUDA_TRY(c, cudaEventCreateWithFlags(&c->pf_fork, cudaEventDisableTiming));
    CUDA_TRY(c, cudaEventCreateWithFlags(&c->pf_join, cudaEventDisableTiming));
    const long long rows = Ptot;
    const int blocks = (T + kPfTok - 1) / kPfTok;
    c->pf_rows = (int)rows;
    c->pf_max_tiles = (int)((P + kPfBM - 1) / kPfBM + E + (T + kPfBM - 1) / kPfBM + 4);
    size_t po = 0;
    auto pcarve = [&](size_t bytes) {
      const size_t at = po;
      po += (bytes + 1023) / 1024 * 1024;
      return at;
    };
    const size_t o_hg = pcarve((size_t)rows * d * 2), o_row = pcarve((size_t)rows * 4);
    const size_t o_bm = pcarve((size_t)blocks * E * 2), o_bo = pcarve((size_t)blocks * E * 4);
    const size_t o_eo = pcarve((size_t)(E + 1) * 4), o_nt = pcarve(4);
    const size_t o_tl = pcarve((size_t)c->pf_max_tiles * sizeof(PfTile));
    // a split reduction uses at most 2 n_sm 128 x 128 tiles of partial sums
    c->pf_part_floats = 2LL * c->n_sm * kRgBM * kRgBN;
    const size_t o_part = pcarve((size_t)c->pf_part_floats * sizeof(float));
    const size_t o_a16 = pcarve((size_t)rows * f * 2), o_y16 = pcarve((size_t)rows * d * 2);
    const size_t o_perm = pcarve((size_t)P * 4), o_hot = pcarve((size_t)E * 4);
    const size_t o_colp = pcarve((size_t)kPfColSplitMax * E * 4);
    CUDA_TRY(c, cudaMalloc(&c->pf, po));
    CUDA_TRY(c, cudaMemset(c->pf, 0, po));
    c->pf_hg = (__half *)(c->pf + o_hg);
    c->pf_row_of = (int *)(c->pf + o_row);
    c->pf_bmask = (unsigned short *)(c->pf + o_bm);
    c->pf_boff = (int *)(c->pf + o_bo);
    c->pf_eoff = (int *)(c->pf + o_eo);
    c->pf_ntiles = (int *)(c->pf + o_nt);
    c->pf_tiles = (PfTile *)(c->pf + o_tl);
    c->pf_part = (float *)(c->pf + o_part);
    c->pf_a16 = (__half *)(c->pf + o_a16);
    c->pf_y16 = (__half *)(c->pf + o_y16);
    c->pf_perm = (int *)(c->pf + o_perm);
    c->pf_hot = (int *)(c->pf + o_hot);
    c->pf_colpart = (int *)(c->pf + o_colp);
    // the router rows as three exact bf16 parts, for the tensor-core router
    CUDA_TRY(c, cudaMalloc(&c->d_router3, (size_t)c->L * E * 3 * d * sizeof(__nv_bfloat16)));
  }
  c->has_router.assign(c->L, 0);
  c->has_bias.assign(c->L, 0);
  c->has_norm.assign(c->L, 0);
  c->has_gamma.assign(c->L, 0);
  c->shared_loaded.assign(c->L, 0);
  c->eps.assign(c->L, 1e-6f);
  c->expert_loaded.assign(c->L, std::vector<char>(E, 0));
  c->n_loaded.assign(c->L, 0);
  c->host_counts.assign(E, 0);
  c->configured = true;
  return MOE_OK;
}

moe_status ensure_configured(moe_ctx *c) {
  if (c->configured) return MOE_OK;
  return do_configure(c);
}

int finish_npl(int E) {
  int n = (E + 31) / 32;
  int p = 1;
  while (p < n) p <<= 1;
  return p;
}

cudaError_t launch_finish(moe_ctx *c, cudaStream_t s, const FinishParams &fp) {
  const size_t smem = (size_t)finish_smem_ints(c->E, fp.T * c->k) * sizeof(int);
  switch (finish_npl(c->E)) {
    case 1: return launch(route_finish_kernel<1>, dim3(1), dim3(kFinishThreads), smem, s, fp);
    case 2: return launch(route_finish_kernel<2>, dim3(1), dim3(kFinishThreads), smem, s, fp);
    case 4: return launch(route_finish_kernel<4>, dim3(1), dim3(kFinishThreads), smem, s, fp);
    case 8: return launch(route_finish_kernel<8>, dim3(1), dim3(kFinishThreads), smem, s, fp);
    case 16: return launch(route_finish_kernel<16>, dim3(1), dim3(kFinishThreads), smem, s, fp);
    default: return launch(route_finish_kernel<32>, dim3(1), dim3(kFinishThreads), smem, s, fp);
  }
}

// The one-launch routing step (route_fused_kernel) serves windows whose
// tokens fit its shared-memory staging.
bool use_fused_route(const moe_ctx *c, int T) {
  const size_t need = std::max((size_t)T * c->d * 2,
                               (size_t)finish_smem_ints(c->E, T * c->k) * sizeof(int));
  return T <= kFusedMaxT && c->d <= kFusedMaxV * 128 && need <= (size_t)kFusedSmem;
}

cudaError_t launch_route_fused(moe_ctx *c, cudaStream_t s, const RouteFusedParams &rp) {
  const int warps = rp.f.T <= 8 ? 4 : kFusedWarps;
  const dim3 grid((c->E + warps - 1) / warps), block(warps * 32);
  const size_t sm = std::max((size_t)rp.f.T * c->d * 2,
                             (size_t)finish_smem_ints(c->E, rp.f.T * c->k) * sizeof(int));
  switch (finish_npl(c->E)) {
    case 1: return launch(route_fused_kernel<1>, grid, block, sm, s, rp);
    case 2: return launch(route_fused_kernel<2>, grid, block, sm, s, rp);
    case 4: return launch(route_fused_kernel<4>, grid, block, sm, s, rp);
    case 8: return launch(route_fused_kernel<8>, grid, block, sm, s, rp);
    case 16: return launch(route_fused_kernel<16>, grid, block, sm, s, rp);
    default: return launch(route_fused_kernel<32>, grid, block, sm, s, rp);
  }
}

cudaError_t setup_route_fused() {
  cudaError_t e = cudaSuccess;
  void (*ks[])(RouteFusedParams) = {route_fused_kernel<1>, route_fused_kernel<2>,
                                    route_fused_kernel<4>, route_fused_kernel<8>,
                                    route_fused_kernel<16>, route_fused_kernel<32>};
  for (auto k : ks)
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, kFusedSmem);
  return e;
}

cudaError_t setup_finish() {
  cudaError_t e = cudaSuccess;
  void (*ks[])(FinishParams) = {route_finish_kernel<1>, route_finish_kernel<2>,
                                route_finish_kernel<4>, route_finish_kernel<8>,
                                route_finish_kernel<16>, route_finish_kernel<32>};
  for (auto k : ks)
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, 64 * 1024);
  return e;
}

cudaError_t setup_decode() {
  cudaError_t e = cudaSuccess;
  void (*ks[])(DecodeParams) = {decode_kernel<1, 1>, decode_kernel<2, 1>};
  for (auto k : ks)
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, kDecSmem);
  return e;
}

// Shared-memory carve of the decode kernel for a window of T tokens.  The
// decode kernel always runs 16 warps with jobs of <= 8 tokens: a window of
// up to 32 tokens rarely puts more than 8 on one expert, and 16 warps hide
// the GEMV's latency better than 8 warps with two column tiles.
DecSmem decode_layout(const moe_ctx *c, int T) {
  const bool q4 = c->fmt == MOE_Q4_SYM_G32_F16;
  const int ring = q4 ? GemvCfg<1, true, 1>::RING : GemvCfg<2, true, 1>::RING;
  return dec_layout(ring, GemvCfg<1, true, 1>::WARPS, 8, T, c->d, c->f, c->E, c->k, c->n_sm,
                    c->lay.G);
}

// Windows the single-launch decode kernel serves: token sets fit a 32-bit
// mask, the pairs and the window fit its shared memory.
bool use_decode_kernel(const moe_ctx *c, int T) {
  if (!c->dec_fits || T < 1 || T > kDecMaxT || T * c->k > kDecMaxPairs || c->E > kDecMaxE ||
      c->k > kDecMaxK)
    return false;
  const DecSmem L = decode_layout(c, T);
  return L.stage_bytes >= L.rsh && (long long)T * L.rsh <= kDecSmem - L.win &&
         L.rsa <= L.stage_bytes;
}

// The decode kernel's CTAs wait on one another (grid barriers), so all of
// them must be resident: one per SM.  Outside a stream capture the launch is
// cooperative, so the driver refuses a grid that cannot be co-resident
// instead of leaving the waits to run out; it is combined with programmatic
// dependent launch when the driver accepts both (tried once per context,
// else PDL alone).  Captured launches use PDL alone.
cudaError_t launch_decode(moe_ctx *c, cudaStream_t s, const DecodeParams &dp) {
  void (*k)(DecodeParams) = c->fmt == MOE_Q4_SYM_G32_F16 ? decode_kernel<1, 1> : decode_kernel<2, 1>;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(c->n_sm);
  cfg.blockDim = dim3(GemvCfg<1, true, 1>::WARPS * 32);
  cfg.dynamicSmemBytes = kDecSmem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeCooperative;
  attr[1].val.cooperative = 1;
  cfg.attrs = attr;
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(s, &cs) != cudaSuccess) {
    (void)cudaGetLastError();
    cs = cudaStreamCaptureStatusActive;  // unknown: take the plain launch
  }
  if (c->dec_coop != 0 && cs == cudaStreamCaptureStatusNone) {
    cfg.numAttrs = 2;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, k, dp);
    if (e == cudaSuccess || c->dec_coop == 1) {
      c->dec_coop = e == cudaSuccess ? 1 : c->dec_coop;
      return e;
    }
    (void)cudaGetLastError();  // not accepted together: PDL alone from now on
    c->dec_coop = 0;
  }
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, k, dp);
}

// Top-k of every token, one warp per token over ceil(T / 16) CTAs: idx, w and
// the per-block token masks.
cudaError_t launch_pf_topk(moe_ctx *c, cudaStream_t s, const PfRouteParams &tp) {
  const dim3 tg((tp.T + kPfTok - 1) / kPfTok), tb(kPfTok * 32);
  if (c->E <= 128) return launch(prefill_topk_kernel<4>, tg, tb, 0, s, tp);
  if (c->E <= 512) return launch(prefill_topk_kernel<16>, tg, tb, 0, s, tp);
  return launch(prefill_topk_kernel<32>, tg, tb, 0, s, tp);
}

// Router logits: CTA (x, y) takes expert rows [4x, 4x + 4) and every
// gridDim.y-th chunk of tokens from chunk y.
cudaError_t launch_router(moe_ctx *c, cudaStream_t s, const RouterParams &rp) {
  const int tc = kRouterSmem / (2 * c->d);
  const dim3 grid((c->E + kRouterWarps - 1) / kRouterWarps, std::min((rp.T + tc - 1) / tc, 64)),
      block(kRouterWarps * 32);
  const size_t sm = (size_t)std::min(rp.T, tc) * c->d * 2;
  switch (c->d / 128) {
    case 1: return launch(router_logits_kernel<1>, grid, block, sm, s, rp);
    case 2: return launch(router_logits_kernel<2>, grid, block, sm, s, rp);
    case 4: return launch(router_logits_kernel<4>, grid, block, sm, s, rp);
    case 8: return launch(router_logits_kernel<8>, grid, block, sm, s, rp);
    case 12: return launch(router_logits_kernel<12>, grid, block, sm, s, rp);
    case 16: return launch(router_logits_kernel<16>, grid, block, sm, s, rp);
    case 24: return launch(router_logits_kernel<24>, grid, block, sm, s, rp);
    case 32: return launch(router_logits_kernel<32>, grid, block, sm, s, rp);
    default: return cudaErrorInvalidValue;
  }
}

bool router_d_supported(int d) {
  const int v = d / 128;
  return d % 128 == 0 && (v == 1 || v == 2 || v == 4 || v == 8 || v == 12 || v == 16 ||
                          v == 24 || v == 32);
}

// Router input for `layer`: either x itself or RMSNorm(x) in scratch.
const uint16_t *router_input(moe_ctx *c, int layer, const uint16_t *x, int T, cudaStream_t s,
                             cudaError_t *e) {
  if (!c->has_norm[layer]) return x;
  NormParams np{x, c->has_gamma[layer] ? c->d_gamma + (size_t)layer * c->d : nullptr,
                c->eps[layer], T, c->d, c->hbuf};
  *e = launch(rmsnorm_kernel, dim3(T), dim3(256), 0, s, np);
  return c->hbuf;
}

FinishParams finish_params(moe_ctx *c, int layer, int T) {
  FinishParams fp{};
  fp.logits = c->logits;
  fp.T = T;
  fp.E = c->E;
  fp.k = c->k;
  fp.layer = layer;
  fp.idx = c->idx;
  fp.w = c->w;
  fp.off = c->off;
  fp.perm = c->perm;
  fp.chunk = job_chunk(T);
  fp.plist = c->plist;
  fp.job_ptr = c->job_ptr;
  fp.job_beg = c->job_beg;
  fp.job_n = c->job_n;
  fp.n_jobs = c->n_jobs;
  fp.max_jobs = c->max_jobs;
  fp.slot_of = c->d_slot_of;
  fp.n_slots = c->n_slots;
  fp.arena = c->arena;
  fp.pool = c->pool;
  fp.shared = c->n_shared ? c->shared + (size_t)layer * c->lay.expert_bytes : nullptr;
  fp.expert_bytes = c->lay.expert_bytes;
  fp.cnt_out = c->cnt_out;
  fp.stats = c->stats;
  fp.last = c->last;
  fp.status = c->status;
  return fp;
}

moe_status check_ready(moe_ctx *c, int layer) {
  if (!c->configured) return fail(c, MOE_ERR_STATE, "nothing loaded");
  if (!c->has_router[layer]) return fail(c, MOE_ERR_STATE, "router of layer %d not set", layer);
  if (c->n_loaded[layer] != c->E)
    return fail(c, MOE_ERR_STATE, "layer %d: %d of %d experts loaded", layer, c->n_loaded[layer],
                c->E);
  if (c->n_shared && !c->shared_loaded[layer])
    return fail(c, MOE_ERR_STATE, "shared expert of layer %d not loaded", layer);
  return MOE_OK;
}

constexpr int kProfSlots = 8192;

// Event i (0..3) of the current profiled call, or nullptr when off.
cudaEvent_t prof_event(moe_ctx *c, int i) {
  return c->profiling ? c->prof_ev[(size_t)c->prof_next * 4 + i] : nullptr;
}

cudaError_t prof_mark(moe_ctx *c, int i, cudaStream_t s) {
  cudaEvent_t ev = prof_event(c, i);
  if (!ev) return cudaSuccess;
  // inside a stream capture the event becomes an external graph node (so a
  // replay records it again); outside one it is an ordinary record
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  cudaError_t e = cudaStreamIsCapturing(s, &cs);
  if (e != cudaSuccess) return e;
  return cs == cudaStreamCaptureStatusActive ? cudaEventRecordWithFlags(ev, s, cudaEventRecordExternal)
                                            : cudaEventRecord(ev, s);
}

// The whole decode chain for one layer.  delta == nullptr: residual mode.
// Routing for `layer` (norm + logits + top-k + buckets + jobs when
// build_jobs); returns the router input h (x, or the normalised copy).
bool launch_router_tc(moe_ctx *c, cudaStream_t s, const uint16_t *h, int N, int layer, cudaError_t *err);

// Router logits of a chunk of N > 32 tokens by fp32 FMA (router_gemm_kernel).
// A chunk too small to give every SM a 128 x 128 tile splits the reduction
// over blockIdx.z (a power of two dividing d / 128, partial sums bounded by
// the pf_part buffer); *ksplit receives the split count.  Either way the
// logits (with bias) end in c->logits: a split writes partial sums to
// c->pf_part and router_sum_kernel adds them in split order.
cudaError_t launch_router_fma(moe_ctx *c, cudaStream_t s, const uint16_t *h, int N, int layer, int *ksplit) {
  const int E = c->E, d = c->d;
  const int tiles = ((N + kRgBM - 1) / kRgBM) * ((E + kRgBN - 1) / kRgBN);
  int ks = 1;
  while (ks * tiles < c->n_sm && 2 * ks <= kMaxRouterSplit && (d / 128) % (2 * ks) == 0 &&
         (long long)2 * ks * N * E <= c->pf_part_floats && E % 4 == 0)
    ks *= 2;
  *ksplit = ks;
  const float *bias = c->has_bias[layer] ? c->d_bias + (size_t)layer * E : nullptr;
  RouterGemmParams rp{h, c->d_router + (size_t)layer * E * d, bias, N, d, E, ks > 1 ? c->pf_part : c->logits,
                      d / ks};
  cudaError_t e = launch(router_gemm_kernel, dim3((N + kRgBM - 1) / kRgBM, (E + kRgBN - 1) / kRgBN, ks),
                         dim3(256), 0, s, rp);
  if (e == cudaSuccess && ks > 1) {
    const long long n4 = (long long)N * E / 4;
    RouterSumParams sp{c->pf_part, ks, bias, N, E, c->logits};
    e = launch(router_sum_kernel, dim3((unsigned)std::min<long long>((n4 + 255) / 256, 8LL * c->n_sm)),
               dim3(256), 0, s, sp);
  }
  return e;
}

moe_status route_impl(moe_ctx *c, int layer, const uint16_t *x, int T, const FinishParams &fp,
                      cudaStream_t s, const uint16_t **h_out) {
  if (use_fused_route(c, T)) {
    RouteFusedParams rp{};
    rp.x = x;
    rp.gamma = c->has_gamma[layer] ? c->d_gamma + (size_t)layer * c->d : nullptr;
    rp.eps = c->eps[layer];
    rp.use_norm = c->has_norm[layer];
    rp.h_out = c->hbuf;
    rp.W = c->d_router + (size_t)layer * c->E * c->d;
    rp.bias = c->has_bias[layer] ? c->d_bias + (size_t)layer * c->E : nullptr;
    rp.d = c->d;
    rp.logits = c->logits;
    rp.ticket = c->ticket;
    rp.f = fp;
    CUDA_TRY(c, launch_route_fused(c, s, rp));
    if (h_out) *h_out = rp.use_norm ? c->hbuf : x;
    return MOE_OK;
  }
  cudaError_t e = cudaSuccess;
  const uint16_t *h = router_input(c, layer, x, T, s, &e);
  CUDA_TRY(c, e);
  const float *bias = c->has_bias[layer] ? c->d_bias + (size_t)layer * c->E : nullptr;
  if (T > kDecMaxT && c->pf_bmask) {
    // many tokens: logits on the tensor cores (large windows) or by a split
    // fp32 GEMM, the top-k one warp per token across the grid, and the
    // single routing CTA only buckets the selections and builds the jobs
    int ks = 1;
    if (launch_router_tc(c, s, h, T, layer, &e))
      CUDA_TRY(c, e);
    else
      CUDA_TRY(c, launch_router_fma(c, s, h, T, layer, &ks));
    PfRouteParams tp{c->logits, T, c->E, c->k, fp.idx, fp.w, c->pf_bmask, &c->stats[4], bias, h,
                     c->d_router + (size_t)layer * c->E * c->d, c->d};
    CUDA_TRY(c, launch_pf_topk(c, s, tp));
    FinishParams fb = fp;
    fb.logits = nullptr;
    fb.idx_in = fp.idx;
    CUDA_TRY(c, launch_finish(c, s, fb));
  } else {
    RouterParams rp{h, c->d_router + (size_t)layer * c->E * c->d, bias, T, c->d, c->E, c->logits};
    CUDA_TRY(c, launch_router(c, s, rp));
    CUDA_TRY(c, launch_finish(c, s, fp));
  }
  if (h_out) *h_out = h;
  return MOE_OK;
}

// 2-D TMA map of a row-major fp16 matrix [rows][cols]: boxes of 64 columns x
// 128 rows, 128-byte swizzle (the layout the tcgen05 descriptors expect).
// The driver's tensor-map encoder, looked up through the runtime so the
// library has no link-time dependency on the driver library.
using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                   const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                   const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_tiled_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
    else
      (void)cudaGetLastError();
  });
  return fn;
}

// 2-D map of a row-major matrix of 16-bit elements [rows][cols]: boxes of 64
// columns (one 128-byte swizzle row) x box_rows rows, out-of-range rows read
// as zeros.
bool encode_map_16b(CUtensorMap *map, CUtensorMapDataType type, const void *base, int rows, int cols,
                    int box_rows) {
  EncodeTiledFn enc = encode_tiled_fn();
  if (!enc) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
  const cuuint32_t box[2] = {64u, (cuuint32_t)box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return enc(map, type, 2, const_cast<void *>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// fp32 logits [planes][rows][cols] (planes = the splits of a split
// reduction, else 1) in boxes of 32 x 32 x 1 with the 128-byte swizzle of
// the router's staging tiles; a plane clips its own rows.
bool encode_logit_map(CUtensorMap *map, const void *base, int planes, int rows, int cols) {
  EncodeTiledFn enc = encode_tiled_fn();
  if (!enc) return false;
  const cuuint64_t dims[3] = {(cuuint64_t)cols, (cuuint64_t)rows, (cuuint64_t)planes};
  const cuuint64_t strides[2] = {(cuuint64_t)cols * 4, (cuuint64_t)rows * cols * 4};
  const cuuint32_t box[3] = {32u, 32u, 1u};
  const cuuint32_t estr[3] = {1, 1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<void *>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Output map of the grouped GEMM's epilogue: fp16 [rows][cols], boxes of
// 32 rows x 32 columns (64 B) with the 64-byte swizzle of the staging tiles.
bool encode_out_map_f16(CUtensorMap *map, const void *base, int rows, int cols) {
  EncodeTiledFn enc = encode_tiled_fn();
  if (!enc) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
  const cuuint32_t box[2] = {(cuuint32_t)kPfOutCols, (cuuint32_t)kPfOutRows};
  const cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void *>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool encode_map_f16(CUtensorMap *map, const void *base, int rows, int cols) {
  static_assert(kPfBK == 64, "one swizzle row per box row");
  return encode_map_16b(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, base, rows, cols, kPfBM);
}

// How many CTA pairs of the grouped GEMM fit on the device at once (the
// persistent grid launches exactly that many, at most one CTA per SM).
template <int FMT>
cudaError_t prefill_pairs(int n_sm, int *pairs) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(n_sm / 2 * 2);
  cfg.blockDim = dim3(kPfGemmThreads);
  cfg.dynamicSmemBytes = PfCfg<FMT>::SMEM;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  const cudaError_t e = cudaOccupancyMaxActiveClusters(&n, (const void *)prefill_gemm_kernel<FMT, true>, &cfg);
  *pairs = e == cudaSuccess ? std::min(n, n_sm / 2) : 0;
  return e;
}

cudaError_t setup_prefill() {
  cudaError_t e = cudaFuncSetAttribute(router_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       RtCfg::SMEM);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(prefill_gemm_kernel<1, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             PfCfg<1>::SMEM);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(prefill_gemm_kernel<1, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             PfCfg<1>::SMEM);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(prefill_gemm_kernel<2, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             PfCfg<2>::SMEM);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(prefill_gemm_kernel<2, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             PfCfg<2>::SMEM);
  return e;
}

// The two grouped GEMM launches of a prefill chunk (gate/up, then down).
template <int FMT>
cudaError_t launch_prefill_gemms(moe_ctx *c, cudaStream_t s) {
  const int d = c->d, f = c->f, TK = c->lay.TK;
  PfGemmParams g1{c->pf_tiles, c->pf_ntiles, d, f, d / TK, 0, c->pf_a16, nullptr, c->status};
  PfGemmParams g2{c->pf_tiles, c->pf_ntiles, f, d, f / TK, c->lay.p1_bytes, nullptr, c->pf_y16, c->status};
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * c->pf_pairs);  // persistent CTA pairs, all co-resident
  cfg.blockDim = dim3(kPfGemmThreads);
  cfg.dynamicSmemBytes = PfCfg<FMT>::SMEM;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = 2;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  cudaError_t e = cudaLaunchKernelEx(&cfg, prefill_gemm_kernel<FMT, true>, c->pf_map_h, c->pf_omap_a, g1);
  if (e == cudaSuccess)
    e = cudaLaunchKernelEx(&cfg, prefill_gemm_kernel<FMT, false>, c->pf_map_a, c->pf_omap_y, g2);
  return e;
}

// Prefill through the grouped tcgen05 GEMM: more tokens than a decode
// window, f a multiple of the gate/up item (128 features) and d of the down
// item (256 features); Q4 and Q2 experts.
// Router logits of N tokens on the tensor cores (router_tc_kernel) when the
// context holds the router's bf16 parts and E and d fit its tiles; returns
// false (nothing launched) otherwise.  A chunk with fewer 128 x 256 tiles
// than SMs splits the reduction over blockIdx.z (each split at least four
// 64-column steps) and router_sum_kernel adds the partial sums, in split
// order, with the bias.
bool launch_router_tc(moe_ctx *c, cudaStream_t s, const uint16_t *h, int N, int layer, cudaError_t *err) {
  const int E = c->E, d = c->d;
  if (!c->d_router3 || E % kRtBN != 0 || d % 64 != 0) return false;
  const int tiles = ((N + kRtBM - 1) / kRtBM) * (E / kRtBN), nk = 3 * d / 64;
  int splits = 1;
  while (2 * splits * tiles <= c->n_sm && 2 * splits <= kMaxRouterSplit && nk % (2 * splits) == 0 &&
         nk / (2 * splits) >= 4 && (long long)2 * splits * N * E <= c->pf_part_floats)
    splits *= 2;
  const float *bias = c->has_bias[layer] ? c->d_bias + (size_t)layer * E : nullptr;
  CUtensorMap hm, wm, lm;
  if (!encode_map_16b(&hm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, h, N, d, kRtBM) ||
      !encode_map_16b(&wm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, c->d_router3 + (size_t)layer * E * 3 * d, E,
                      3 * d, kRtBN) ||
      !encode_logit_map(&lm, splits > 1 ? c->pf_part : c->logits, splits, N, E))
    return false;
  RouterTcParams tp{splits > 1 ? nullptr : bias, c->logits, N, E, d, nk / splits, c->status};
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((N + kRtBM - 1) / kRtBM, E / kRtBN, splits);
  cfg.blockDim = dim3(256);
  cfg.dynamicSmemBytes = RtCfg::SMEM;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  *err = cudaLaunchKernelEx(&cfg, router_tc_kernel, hm, wm, lm, tp);
  if (*err == cudaSuccess && splits > 1) {
    const long long n4 = (long long)N * E / 4;
    RouterSumParams sp{c->pf_part, splits, bias, N, E, c->logits};
    *err = launch(router_sum_kernel, dim3((unsigned)std::min<long long>((n4 + 255) / 256, 8LL * c->n_sm)),
                  dim3(256), 0, s, sp);
  }
  return true;
}

// Experts with at least this many tokens in a chunk run on the grouped GEMM
// (256-row tiles); fewer tokens would leave most of a tile empty, and the
// GEMV streams such an expert once per job of <= 8 tokens instead (its
// later jobs mostly from L2).  The GEMV runs beside the GEMM, so moving the
// experts of 16-23 tokens to it shortens the GEMM's rounds of items on small
// chunks (256 tokens: 176 us per call against 184 with a threshold of 16)
// without slowing the 8192-token chunk.
constexpr int kHotMinTokens = 24;
// The chunk path's GEMV experts (fewer than kHotMinTokens tokens: most have
// one to three) run as jobs of <= 8 tokens through the one-column-tile GEMV;
// jobs of 16 doubled its tensor work per weight byte, and the pass is
// weight-bound (a chunk of 8192 tokens touched about 106 such experts with
// 401 tokens between them: 281 MB of weights).
constexpr int kColdChunk = 8;

bool use_prefill_gemm(const moe_ctx *c, int N) {
  return c->pf && c->pf_pairs > 0 && N > kDecMaxT && c->d % (2 * kPfBN) == 0 && c->f % kPfBN == 0 &&
         c->E <= kPfMaxE;
}

// The prefill chunk's routing on router input h: logits, top-k + softmax
// (idx, w), the sort of the chunk's pairs by expert (each expert's rows in
// ascending t), the 256-row tile list with the residency lookup, and the
// gather of the grouped fp16 A rows.  perm (or null) receives the bucket
// permutation; the bucket offsets are left in c->pf_eoff.
moe_status pf_bucket_impl(moe_ctx *c, int layer, const uint16_t *h, int N, int kk, const int32_t *idx,
                          bool with_shared, int32_t *perm, cudaStream_t s, int hot_min);

moe_status prefill_route_impl(moe_ctx *c, int layer, const uint16_t *h, int N, int32_t *idx, float *w,
                              int32_t *perm, cudaStream_t s, int hot_min) {
  const int E = c->E, k = c->k, d = c->d;
  cudaError_t e = cudaSuccess;
  const float *bias = c->has_bias[layer] ? c->d_bias + (size_t)layer * E : nullptr;
  int ks = 1;
  if (launch_router_tc(c, s, h, N, layer, &e))
    CUDA_TRY(c, e);
  else  // small expert counts or chunks: fp32 FMA
    CUDA_TRY(c, launch_router_fma(c, s, h, N, layer, &ks));
  PfRouteParams tp{c->logits, N, E, k, idx, w, c->pf_bmask, &c->stats[4], bias, h,
                   c->d_router + (size_t)layer * E * d, d};
  CUDA_TRY(c, launch_pf_topk(c, s, tp));
  return pf_bucket_impl(c, layer, h, N, k, idx, c->n_shared != 0, perm, s, hot_min);
}

// The chunk's pairs sorted by expert from the block masks in c->pf_bmask
// (the top-k's, or prefill_mask_kernel's for given routing): bucket
// offsets, the GEMM tile and GEMV job lists with the residency lookup, and
// the grouped fp16 A rows.  kk: experts per token; with_shared adds the
// shared expert's T rows after the routed ones.
moe_status pf_bucket_impl(moe_ctx *c, int layer, const uint16_t *h, int N, int kk, const int32_t *idx,
                          bool with_shared, int32_t *perm, cudaStream_t s, int hot_min) {
  const int E = c->E, d = c->d;
  const int blocks = (N + kPfTok - 1) / kPfTok;
  PfScanParams sp{};
  sp.bmask = c->pf_bmask;
  sp.blocks = blocks;
  sp.E = E;
  sp.T = N;
  sp.k = kk;
  sp.boff = c->pf_boff;
  sp.eoff = c->pf_eoff;
  sp.slot_of = c->d_slot_of;
  sp.n_slots = c->n_slots;
  sp.layer = layer;
  sp.arena = c->arena;
  sp.pool = c->pool;
  sp.shared = with_shared ? c->shared + (size_t)layer * c->lay.expert_bytes : nullptr;
  sp.expert_bytes = c->lay.expert_bytes;
  sp.tiles = c->pf_tiles;
  sp.n_tiles = c->pf_ntiles;
  sp.max_tiles = c->pf_max_tiles;
  sp.hot_min = hot_min;
  sp.chunk = kColdChunk;
  sp.hot = c->pf_hot;
  sp.job_ptr = c->job_ptr;
  sp.job_beg = c->job_beg;
  sp.job_n = c->job_n;
  sp.n_jobs = c->n_jobs;
  sp.max_jobs = c->max_jobs;
  sp.cnt_out = c->cnt_out;
  sp.stats = c->stats;
  sp.last = c->last;
  sp.status = c->status;
  // long chunks: the column scan split over ranges of about 64 blocks
  const int splits = std::max(1, std::min(kPfColSplitMax, blocks / 64));
  sp.col_part = c->pf_colpart;
  if (splits > 1)
    CUDA_TRY(c, launch(prefill_colcount_kernel, dim3((E + 31) / 32, splits), dim3(kPfColWarps * 32), 0, s, sp));
  CUDA_TRY(c, launch(prefill_colscan_kernel, dim3((E + 31) / 32, splits), dim3(kPfColWarps * 32), 0, s, sp));
  CUDA_TRY(c, launch(prefill_scan_kernel, dim3(1), dim3(1024), 0, s, sp));
  PfScatterParams cp{idx, c->pf_bmask, c->pf_boff, c->pf_eoff, h, N, E, kk, d, with_shared ? 1 : 0,
                     c->pf_row_of, c->pf_hg, perm ? perm : c->pf_perm, c->pf_hot};
  // small chunks split each token row's columns over more CTAs
  const int ysplit = std::max(1, std::min(d / 256, (2 * c->n_sm + blocks - 1) / blocks));
  CUDA_TRY(c, launch(prefill_scatter_kernel, dim3(blocks, ysplit), dim3(kPfTok * 32), 0, s, cp));
  return MOE_OK;
}

// Tensor maps of the grouped GEMM's operands (encoded once per context).
moe_status pf_maps(moe_ctx *c) {
  if (c->pf_maps) return MOE_OK;
  const int d = c->d, f = c->f;
  if (!encode_map_f16(&c->pf_map_h, c->pf_hg, c->pf_rows, d) ||
      !encode_map_f16(&c->pf_map_a, c->pf_a16, c->pf_rows, f) ||
      !encode_out_map_f16(&c->pf_omap_a, c->pf_a16, c->pf_rows, f) ||
      !encode_out_map_f16(&c->pf_omap_y, c->pf_y16, c->pf_rows, d))
    return fail(c, MOE_ERR_CUDA, "cuTensorMapEncodeTiled failed");
  c->pf_maps = true;
  return MOE_OK;
}

// The experts of a bucketed chunk: experts with many tokens run as the
// grouped GEMM over 256-row tiles, the others as the GEMV over jobs of <= 8
// tokens, rows read through the bucket permutation (grouped row -> pair
// id).  h: the router input the pairs' rows come from; kk: experts per token.
moe_status pf_experts_impl(moe_ctx *c, const uint16_t *h, int N, int kk, cudaStream_t s) {
  GemvParams g1{};
  g1.job_ptr = c->job_ptr;
  g1.job_beg = c->job_beg;
  g1.job_n = c->job_n;
  g1.n_jobs = c->n_jobs;
  g1.plist = c->pf_perm;
  g1.Tk = N * kk;
  g1.k = kk > 0 ? kk : 1;  // kk == 0: no routed pairs, so no GEMV jobs
  g1.src = h;
  g1.src_by_pair = 0;
  g1.K = c->d;
  g1.R = c->f;
  g1.region_off = 0;
  g1.out_a = c->abuf;
  g1.status = c->status;
  GemvParams g2 = g1;
  g2.src = c->abuf;
  g2.src_by_pair = 1;
  g2.K = c->f;
  g2.R = c->d;
  g2.region_off = c->lay.p1_bytes;
  g2.out_a = nullptr;
  g2.out_y = nullptr;
  g2.out_y16 = reinterpret_cast<__half *>(c->ybuf);  // fp16 y by pair id, as the GEMM's
  // the GEMV experts run on a second stream beside the grouped GEMM: their
  // CTAs take the SMs that GEMM pairs leave idle in its last round of items
  // (they read the same grouped inputs and write other buffers)
  CUDA_TRY(c, cudaEventRecord(c->pf_fork, s));
  CUDA_TRY(c, cudaStreamWaitEvent(c->pf_side, c->pf_fork, 0));
  if (c->fmt == MOE_Q4_SYM_G32_F16) {
    CUDA_TRY(c, launch_prefill_gemms<1>(c, s));
    CUDA_TRY(c, launch_experts<1>(c, c->pf_side, kColdChunk, g1, g2));
  } else {
    CUDA_TRY(c, launch_prefill_gemms<2>(c, s));
    CUDA_TRY(c, launch_experts<2>(c, c->pf_side, kColdChunk, g1, g2));
  }
  CUDA_TRY(c, cudaEventRecord(c->pf_join, c->pf_side));
  CUDA_TRY(c, cudaStreamWaitEvent(s, c->pf_join, 0));
  return MOE_OK;
}

// x[t] <- bf16(x[t] + sum_j w[t,j] y(t,j) + y_shared[t]) (delta == null) or
// delta[t] <- the same sum, from the chunk's grouped outputs.
moe_status pf_combine_impl(moe_ctx *c, int N, int kk, const float *w, bool with_shared, uint16_t *x,
                           float *delta, cudaStream_t s) {
  const int d = c->d;
  PfCombineParams mp{c->pf_y16, reinterpret_cast<const __half *>(c->ybuf), w, c->pf_row_of, N, kk, d,
                     with_shared ? 1 : 0, x, delta};
  const long long n4 = (long long)N * d / 4;
  const int cblocks = (int)std::min<long long>((n4 + 255) / 256, 8LL * c->n_sm);
  CUDA_TRY(c, launch(prefill_combine_kernel, dim3(cblocks), dim3(256), 0, s, mp));
  return MOE_OK;
}

moe_status prefill_impl(moe_ctx *c, int layer, uint16_t *x, int N, float *delta, cudaStream_t s) {
  const int k = c->k;
  moe_status st = pf_maps(c);
  if (st) return st;
  CUDA_TRY(c, prof_mark(c, 0, s));
  cudaError_t e = cudaSuccess;
  const uint16_t *h = router_input(c, layer, x, N, s, &e);
  CUDA_TRY(c, e);
  st = prefill_route_impl(c, layer, h, N, c->idx, c->w, c->pf_perm, s, kHotMinTokens);
  if (st) return st;
  CUDA_TRY(c, prof_mark(c, 1, s));
  st = pf_experts_impl(c, h, N, k, s);
  if (st) return st;
  CUDA_TRY(c, prof_mark(c, 2, s));
  st = pf_combine_impl(c, N, k, c->w, c->n_shared != 0, x, delta, s);
  if (st) return st;
  CUDA_TRY(c, prof_mark(c, 3, s));
  if (c->profiling) {
    c->prof_next = (c->prof_next + 1) % kProfSlots;
    c->prof_pending = std::min(c->prof_pending + 1, kProfSlots);
  }
  return MOE_OK;
}

// The experts of a chunk on caller-given routing (the rows an
// expert-parallel owner received, or any precomputed routing): block masks
// from idx, then the chunk path's bucketing, experts and combine into
// delta.  idx was checked on the host (ids in [0, E), distinct per token).
moe_status given_impl(moe_ctx *c, int layer, const uint16_t *h, int N, int kk, const int32_t *idx,
                      const float *w, bool with_shared, float *delta, cudaStream_t s, __half *rows16 = nullptr) {
  moe_status st = pf_maps(c);
  if (st) return st;
  const int blocks = (N + kPfTok - 1) / kPfTok;
  PfMaskParams mp{idx, N, c->E, kk, c->pf_bmask};
  CUDA_TRY(c, launch(prefill_mask_kernel, dim3(blocks), dim3(kPfTok * 32), 0, s, mp));
  st = pf_bucket_impl(c, layer, h, N, kk, idx, with_shared, c->pf_perm, s, kHotMinTokens);
  if (st) return st;
  st = pf_experts_impl(c, h, N, kk, s);
  if (st) return st;
  if (rows16) {  // kk == 1, no weights, no shared expert: each row's y as it is
    PfRowsParams rp{c->pf_y16, reinterpret_cast<const __half *>(c->ybuf), c->pf_row_of, N, c->d, rows16};
    const long long n8 = (long long)N * c->d / 8;
    const int blocks = (int)std::min<long long>((n8 + 255) / 256, 8LL * c->n_sm);
    CUDA_TRY(c, launch(prefill_rows_kernel, dim3(blocks), dim3(256), 0, s, rp));
    return MOE_OK;
  }
  return pf_combine_impl(c, N, kk, w, with_shared, nullptr, delta, s);
}

// The whole decode chain for one layer.  delta == nullptr: residual mode.
// Windows of <= kFusedMaxT tokens take four launches: fused routing, the
// gated expert GEMV, the down GEMV and the combine + residual.
moe_status forward_impl(moe_ctx *c, int layer, uint16_t *x, int T, float *delta, cudaStream_t s) {
  CUDA_TRY(c, prof_mark(c, 0, s));
  if (use_decode_kernel(c, T)) {
    DecodeParams dp{};
    dp.x = x;
    dp.delta = delta;
    dp.gamma = c->has_gamma[layer] ? c->d_gamma + (size_t)layer * c->d : nullptr;
    dp.eps = c->eps[layer];
    dp.use_norm = c->has_norm[layer];
    dp.W = c->d_router + (size_t)layer * c->E * c->d;
    dp.bias = c->has_bias[layer] ? c->d_bias + (size_t)layer * c->E : nullptr;
    dp.T = T;
    dp.d = c->d;
    dp.f = c->f;
    dp.E = c->E;
    dp.k = c->k;
    dp.layer = layer;
    dp.chunk = 8;
    dp.slot_of = c->d_slot_of;
    dp.n_slots = c->n_slots;
    dp.arena = c->arena;
    dp.pool = c->pool;
    dp.shared = c->n_shared ? c->shared + (size_t)layer * c->lay.expert_bytes : nullptr;
    dp.expert_bytes = c->lay.expert_bytes;
    dp.p1_bytes = c->lay.p1_bytes;
    dp.logits = c->logits;
    dp.hbuf = c->hbuf;
    dp.abuf = c->abuf;
    dp.ybuf = c->ybuf;
    dp.ws = c->dec_ws;
    dp.flags = c->dec_flags;
    dp.bar = c->dec_bar;
    dp.cnt_out = c->cnt_out;
    dp.stats = c->stats;
    dp.last = c->last;
    dp.status = c->status;
    dp.sm = decode_layout(c, T);
    dp.bar1_extra = c->dec_stall_next ? (unsigned long long)c->n_sm : 0ull;
    dp.bar1_polls = c->dec_stall_next ? c->dec_stall_polls : (1u << 22);
    c->dec_stall_next = 0;
    CUDA_TRY(c, launch_decode(c, s, dp));
    // one kernel: the profile's route / experts / combine marks coincide
    CUDA_TRY(c, prof_mark(c, 1, s));
    CUDA_TRY(c, prof_mark(c, 2, s));
    CUDA_TRY(c, prof_mark(c, 3, s));
    if (c->profiling) {
      c->prof_next = (c->prof_next + 1) % kProfSlots;
      c->prof_pending = std::min(c->prof_pending + 1, kProfSlots);
    }
    return MOE_OK;
  }
  // more tokens than a decode window: GEMM for the experts that many tokens
  // share, GEMV for the rest (prefill_impl)
  if (use_prefill_gemm(c, T)) return prefill_impl(c, layer, x, T, delta, s);
  FinishParams fp = finish_params(c, layer, T);
  fp.build_jobs = 1;
  const uint16_t *h = nullptr;
  moe_status st = route_impl(c, layer, x, T, fp, s, &h);
  if (st) return st;

  GemvParams g1{};
  g1.job_ptr = c->job_ptr;
  g1.job_beg = c->job_beg;
  g1.job_n = c->job_n;
  g1.n_jobs = c->n_jobs;
  g1.plist = c->plist;
  g1.Tk = T * c->k;
  g1.k = c->k;
  g1.src = h;
  g1.src_by_pair = 0;
  g1.K = c->d;
  g1.R = c->f;
  g1.region_off = 0;
  g1.out_a = c->abuf;
  g1.status = c->status;
  GemvParams g2 = g1;
  g2.src = c->abuf;
  g2.src_by_pair = 1;
  g2.K = c->f;
  g2.R = c->d;
  g2.region_off = c->lay.p1_bytes;
  g2.out_a = nullptr;
  g2.out_y = c->ybuf;
  CUDA_TRY(c, prof_mark(c, 1, s));
  if (c->fmt == MOE_Q4_SYM_G32_F16)
    CUDA_TRY(c, launch_experts<1>(c, s, T, g1, g2));
  else
    CUDA_TRY(c, launch_experts<2>(c, s, T, g1, g2));
  CUDA_TRY(c, prof_mark(c, 2, s));
  {
    CombineParams cp{c->ybuf, c->w, T, c->k, c->d, c->n_shared, x, delta};
    const long long n4 = (long long)T * c->d / 4;
    const int blocks = (int)std::min<long long>((n4 + 127) / 128, 8LL * c->n_sm);
    CUDA_TRY(c, launch(combine_kernel, dim3(blocks), dim3(128), 0, s, cp));
  }
  CUDA_TRY(c, prof_mark(c, 3, s));
  if (c->profiling) {
    c->prof_next = (c->prof_next + 1) % kProfSlots;
    c->prof_pending = std::min(c->prof_pending + 1, kProfSlots);
  }
  return MOE_OK;
}

moe_status load_impl(moe_ctx *c, uint8_t *dst, int n, const void *codes, const void *scales,
                     const void *mins, int src_is_device) {
  const Layout &L = c->lay;
  const long long per_codes = L.fmt == 1 ? 3LL * c->f * c->d / 2 : 3LL * c->f * c->d / 4;
  const long long per_groups = 3LL * c->f * c->d / L.G;
  const size_t nc = (size_t)n * per_codes, ns = (size_t)n * per_groups * 2;
  const uint8_t *dc = (const uint8_t *)codes;
  const uint16_t *ds = (const uint16_t *)scales, *dm = (const uint16_t *)mins;
  uint8_t *staging = nullptr;
  if (!src_is_device) {
    const size_t tot = nc + ns + (mins ? ns : 0);
    CUDA_TRY(c, cudaMalloc(&staging, tot));
    cudaError_t e = cudaMemcpyAsync(staging, codes, nc, cudaMemcpyHostToDevice, c->io);
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(staging + nc, scales, ns, cudaMemcpyHostToDevice, c->io);
    if (e == cudaSuccess && mins)
      e = cudaMemcpyAsync(staging + nc + ns, mins, ns, cudaMemcpyHostToDevice, c->io);
    if (e != cudaSuccess) {
      cudaFree(staging);
      CUDA_TRY(c, e);
    }
    dc = staging;
    ds = (const uint16_t *)(staging + nc);
    dm = mins ? (const uint16_t *)(staging + nc + ns) : nullptr;
  }
  RepackParams rp{dc, ds, dm, dst, n, L};
  cudaError_t e = launch(repack_kernel, dim3(4 * c->n_sm), dim3(256), 0, c->io, rp, false);
  if (e == cudaSuccess) e = cudaStreamSynchronize(c->io);
  if (staging) cudaFree(staging);
  CUDA_TRY(c, e);
  return MOE_OK;
}

moe_status refresh_slots(moe_ctx *c, int layer, int first, int n) {
  const long long Be = c->lay.expert_bytes;
  for (int e = first; e < first + n; ++e) {
    const int slot = c->h_slot_of[(size_t)layer * c->E + e];
    if (slot >= 0)
      CUDA_TRY(c, cudaMemcpyAsync(c->pool + (size_t)slot * Be,
                                  c->arena + ((size_t)layer * c->E + e) * Be, (size_t)Be,
                                  cudaMemcpyDefault, c->io));
  }
  CUDA_TRY(c, cudaStreamSynchronize(c->io));
  return MOE_OK;
}

// One request of the host tier.  The window's routing (idx_dev [T, k], on
// stream s) is read back once the stream's work is done; its distinct
// experts are the request.  Each miss takes a slot by the cache's policy, its
// expert is copied from the host arena into the slot on the tier stream, and
// the slot-table rows that changed follow on the same stream.  With wait,
// stream s waits for those copies; otherwise (a prefetch) they stay in
// flight and the next request's wait covers them, and the previous
// request's slots are protected from eviction (its window may still run).
moe_status tier_request(moe_ctx *c, int layer, const int32_t *idx_dev, int T, cudaStream_t s, bool wait) {
  const int E = c->E, k = c->k;
  const long long Be = c->lay.expert_bytes;
  CUDA_TRY(c, cudaMemcpyAsync(c->h_tier_idx, idx_dev, (size_t)T * k * sizeof(int32_t), cudaMemcpyDeviceToHost, s));
  CUDA_TRY(c, cudaStreamSynchronize(s));
  std::vector<char> seen(E, 0);
  std::vector<long long> keys;
  for (int i = 0; i < T * k; ++i) {
    const int e = c->h_tier_idx[i];
    if (e < 0 || e >= E) return fail(c, MOE_ERR_DEVICE, "routing id %d out of range", e);
    if (!seen[e]) {
      seen[e] = 1;
      keys.push_back((long long)layer * E + e);
    }
  }
  std::sort(keys.begin(), keys.end());
  std::vector<long long> fill_key, fill_ev;
  std::vector<int> fill_slot;
  if (!c->tier.request(keys, c->h_slot_of, !wait, fill_key, fill_slot, fill_ev))
    return fail(c, MOE_ERR_INVALID_ARG, "the window needs %zu experts resident; the pool has %d slots",
                keys.size(), c->n_slots);
  ++c->tier_calls;
  c->tier_trace.push_back((int)c->tier_calls);
  c->tier_trace.push_back(layer);
  c->tier_trace.push_back((int)keys.size());
  for (long long key : keys) c->tier_trace.push_back((int)(key - (long long)layer * E));
  std::vector<char> dirty(c->L, 0);
  for (size_t i = 0; i < fill_key.size(); ++i) {
    CUDA_TRY(c, cudaMemcpyAsync(c->pool + (size_t)fill_slot[i] * Be, c->h_arena + (size_t)fill_key[i] * Be,
                                (size_t)Be, cudaMemcpyHostToDevice, c->tier_stream));
    c->tier_bytes += Be;
    dirty[fill_key[i] / E] = 1;
    if (fill_ev[i] >= 0) dirty[fill_ev[i] / E] = 1;
  }
  // pageable source: the call returns once the row has been staged
  for (int l = 0; l < c->L; ++l)
    if (dirty[l])
      CUDA_TRY(c, cudaMemcpyAsync(c->d_slot_of + (size_t)l * E, c->h_slot_of.data() + (size_t)l * E,
                                  (size_t)E * sizeof(int), cudaMemcpyHostToDevice, c->tier_stream));
  CUDA_TRY(c, cudaEventRecord(c->tier_done, c->tier_stream));
  if (wait) CUDA_TRY(c, cudaStreamWaitEvent(s, c->tier_done, 0));
  return MOE_OK;
}

}  // namespace

extern "C" {

const char *moe_status_string(int s) {
  switch (s) {
    case MOE_OK: return "MOE_OK";
    case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG";
    case MOE_ERR_OOM: return "MOE_ERR_OOM";
    case MOE_ERR_CUDA: return "MOE_ERR_CUDA";
    case MOE_ERR_STATE: return "MOE_ERR_STATE";
    case MOE_ERR_BAD_SLOT: return "MOE_ERR_BAD_SLOT";
    case MOE_ERR_DEVICE: return "MOE_ERR_DEVICE";
    case MOE_ERR_TIMEOUT: return "MOE_ERR_TIMEOUT";
    case MOE_ERR_NOT_SUPPORTED: return "MOE_ERR_NOT_SUPPORTED";
    default: return "MOE_ERR_UNKNOWN";
  }
}

int64_t moe_expert_bytes(int d, int f, int fmt) {
  if (d <= 0 || f <= 0 || d % 128 || f % 128) return -1;
  if (fmt != MOE_Q4_SYM_G32_F16 && fmt != MOE_Q2_ASYM_G64_F16) return -1;
  return make_layout(fmt, d, f).expert_bytes;
}

const char *moe_last_error(const moe_ctx *c) { return c ? c->err.c_str() : ""; }

moe_status moe_create(int d, int f, int E, int k, int fmt, moe_ctx **out) {
  if (!out) return MOE_ERR_INVALID_ARG;
  *out = nullptr;
  if (d <= 0 || f <= 0 || d % 128 || f % 128 || E < 1 || E > 1024 || k < 1 || k > E || k > 32 ||
      (fmt != MOE_Q4_SYM_G32_F16 && fmt != MOE_Q2_ASYM_G64_F16) || d > 4096 ||
      !router_d_supported(d))
    return MOE_ERR_INVALID_ARG;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    (void)cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  moe_ctx *c = new moe_ctx();
  c->device = dev;
  c->d = d;
  c->f = f;
  c->E = E;
  c->k = k;
  c->fmt = fmt;
  c->lay = make_layout(fmt, d, f);
  cudaError_t e = cudaDeviceGetAttribute(&c->n_sm, cudaDevAttrMultiProcessorCount, dev);
  if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&c->io, cudaStreamNonBlocking);
  if (e == cudaSuccess) e = setup_route_fused();
  if (e == cudaSuccess) e = setup_finish();
  if (e == cudaSuccess) e = setup_decode();
  if (e == cudaSuccess) e = setup_prefill();
  if (e == cudaSuccess) e = setup_gemv<1, true, 1>(c->n_sm, &c->gemv_blocks[0][1][0]);
  if (e == cudaSuccess) e = setup_gemv<1, false, 1>(c->n_sm, &c->gemv_blocks[0][0][0]);
  if (e == cudaSuccess) e = setup_gemv<2, true, 1>(c->n_sm, &c->gemv_blocks[1][1][0]);
  if (e == cudaSuccess) e = setup_gemv<2, false, 1>(c->n_sm, &c->gemv_blocks[1][0][0]);
  if (e == cudaSuccess) e = setup_gemv<1, true, 2>(c->n_sm, &c->gemv_blocks[0][1][1]);
  if (e == cudaSuccess) e = setup_gemv<1, false, 2>(c->n_sm, &c->gemv_blocks[0][0][1]);
  if (e == cudaSuccess) e = setup_gemv<2, true, 2>(c->n_sm, &c->gemv_blocks[1][1][1]);
  if (e == cudaSuccess) e = setup_gemv<2, false, 2>(c->n_sm, &c->gemv_blocks[1][0][1]);
  if (e == cudaSuccess) {
    // the single-launch decode kernel needs one resident CTA per SM; where
    // it does not fit (a smaller part, or shared-memory carve-outs), windows
    // take the multi-launch path instead
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, decode_kernel<1, 1>,
                                                      GemvCfg<1, true, 1>::WARPS * 32, kDecSmem);
    c->dec_fits = e == cudaSuccess && per_sm >= 1;
  }
  if (e == cudaSuccess)
    e = fmt == MOE_Q4_SYM_G32_F16 ? prefill_pairs<1>(c->n_sm, &c->pf_pairs) : prefill_pairs<2>(c->n_sm, &c->pf_pairs);
  if (e != cudaSuccess) {
    (void)cudaGetLastError();
    moe_destroy(c);
    return MOE_ERR_CUDA;
  }
  *out = c;
  return MOE_OK;
}

moe_status moe_configure(moe_ctx *c, int n_layers, int n_shared, int n_slots, int max_tokens) {
  if (!c) return MOE_ERR_INVALID_ARG;
  if (c->configured) return fail(c, MOE_ERR_STATE, "moe_configure after configuration/loads");
  if (n_layers < 1 || n_layers > 4096 || (n_shared != 0 && n_shared != 1) || n_slots < 0 ||
      max_tokens < 1 || max_tokens > (1 << 20))
    return fail(c, MOE_ERR_INVALID_ARG, "bad configuration");
  c->L = n_layers;
  c->n_shared = n_shared;
  c->n_slots = n_slots;
  c->max_tokens = max_tokens;
  return do_configure(c);
}

moe_status moe_destroy(moe_ctx *c) {
  if (!c) return MOE_OK;
  cudaDeviceSynchronize();
  for (auto &kv : c->stack_graphs) cudaGraphExecDestroy(kv.second);
  for (cudaEvent_t ev : c->prof_ev) cudaEventDestroy(ev);
  dfree(c->pf);
  dfree(c->ep_counts);
  if (c->h_arena) {
    cudaFreeHost(c->h_arena);
    c->h_arena = nullptr;
    c->arena = nullptr;
  }
  dfree(c->arena);
  dfree(c->tier_idx);
  dfree(c->tier_w);
  if (c->h_tier_idx) cudaFreeHost(c->h_tier_idx);
  if (c->tier_done) cudaEventDestroy(c->tier_done);
  if (c->tier_stream) cudaStreamDestroy(c->tier_stream);
  if (c->pf_side) cudaStreamDestroy(c->pf_side);
  if (c->pf_fork) cudaEventDestroy(c->pf_fork);
  if (c->pf_join) cudaEventDestroy(c->pf_join);
  dfree(c->shared);
  dfree(c->pool);
  dfree(c->d_slot_of);
  dfree(c->d_router);
  dfree(c->d_router3);
  dfree(c->d_bias);
  dfree(c->d_gamma);
  dfree(c->scratch);
  if (c->trace) {
    unsigned long long *null_ptr = nullptr;
    cudaMemcpyToSymbol(g_trace, &null_ptr, sizeof null_ptr);
    dfree(c->trace);
  }
  if (c->io) cudaStreamDestroy(c->io);
  (void)cudaGetLastError();
  delete c;
  return MOE_OK;
}

moe_status moe_load_experts(moe_ctx *c, int layer, int first, int n, const void *codes,
                            const void *scales, const void *mins, int src_is_device) {
  if (!c) return MOE_ERR_INVALID_ARG;
  moe_status st = ensure_configured(c);
  if (st) return st;
  if (!valid_layer(c, layer) || first < 0 || n < 1 || first + n > c->E || !codes || !scales ||
      (c->fmt == MOE_Q2_ASYM_G64_F16 && !mins))
    return fail(c, MOE_ERR_INVALID_ARG, "moe_load_experts: bad arguments");
  if (c->fmt == MOE_Q4_SYM_G32_F16) mins = nullptr;
  uint8_t *dst = c->arena + ((size_t)layer * c->E + first) * c->lay.expert_bytes;
  st = load_impl(c, dst, n, codes, scales, mins, src_is_device);
  if (st) return st;
  for (int e = first; e < first + n; ++e)
    if (!c->expert_loaded[layer][e]) {
      c->expert_loaded[layer][e] = 1;
      c->n_loaded[layer]++;
    }
  c->any_loaded = true;
  return refresh_slots(c, layer, first, n);
}

moe_status moe_load_shared(moe_ctx *c, int layer, const void *codes, const void *scales,
                           const void *mins, int src_is_device) {
  if (!c) return MOE_ERR_INVALID_ARG;
  moe_status st = ensure_configured(c);
  if (st) return st;
  if (!c->n_shared) return fail(c, MOE_ERR_STATE, "configured without a shared expert");
  if (!valid_layer(c, layer) || !codes || !scales || (c->fmt == MOE_Q2_ASYM_G64_F16 && !mins))
    return fail(c, MOE_ERR_INVALID_ARG, "moe_load_shared: bad arguments");
  if (c->fmt == MOE_Q4_SYM_G32_F16) mins = nullptr;
  st = load_impl(c, c->shared + (size_t)layer * c->lay.expert_bytes, 1, codes, scales, mins,
                 src_is_device);
  if (st) return st;
  c->shared_loaded[layer] = 1;
  c->any_loaded = true;
  return MOE_OK;
}

moe_status moe_set_router(moe_ctx *c, int layer, const float *W, const float *bias,
                          int src_is_device) {
  if (!c) return MOE_ERR_INVALID_ARG;
  moe_status st = ensure_configured(c);
  if (st) return st;
  if (!valid_layer(c, layer) || !W) return fail(c, MOE_ERR_INVALID_ARG, "moe_set_router");
  const cudaMemcpyKind kind = src_is_device ? cudaMemcpyDeviceToDevice : cudaMemcpyHostToDevice;
  CUDA_TRY(c, cudaMemcpyAsync(c->d_router + (size_t)layer * c->E * c->d, W,
                              (size_t)c->E * c->d * sizeof(float), kind, c->io));
  if (bias)
    CUDA_TRY(c, cudaMemcpyAsync(c->d_bias + (size_t)layer * c->E, bias, (size_t)c->E * sizeof(float),
                                kind, c->io));
  if (c->d_router3) {
    const long long n = (long long)c->E * c->d;
    router_split_kernel<<<(unsigned)std::min<long long>((n + 255) / 256, 4096), 256, 0, c->io>>>(
        c->d_router + (size_t)layer * c->E * c->d, n, c->d,
        c->d_router3 + (size_t)layer * c->E * 3 * c->d);
    CUDA_TRY(c, cudaGetLastError());
  }
  CUDA_TRY(c, cudaStreamSynchronize(c->io));
  c->has_router[layer] = 1;
  c->has_bias[layer] = bias != nullptr;
  return MOE_OK;
}

moe_status moe_set_norm(moe_ctx *c, int layer, const float *gamma, float eps) {
  if (!c) return MOE_ERR_INVALID_ARG;
  moe_status st = ensure_configured(c);
  if (st) return st;
  if (!valid_layer(c, layer) || !(eps >= 0.f)) return fail(c, MOE_ERR_INVALID_ARG, "moe_set_norm");
  if (gamma)
    CUDA_TRY(c, cudaMemcpy(c->d_gamma + (size_t)layer * c->d, gamma, (size_t)c->d * sizeof(float),
                           cudaMemcpyHostToDevice));
  c->has_norm[layer] = 1;
  c->has_gamma[layer] = gamma != nullptr;
  c->eps[layer] = eps;
  return MOE_OK;
}

moe_status moe_set_slots(moe_ctx *c, const int32_t *slot_of) {
  if (!c || !slot_of) return fail(c, MOE_ERR_INVALID_ARG, "moe_set_slots: NULL");
  moe_status st = ensure_configured(c);
  if (st) return st;
  const size_t n = (size_t)c->L * c->E;
  std::vector<char> used(c->n_slots, 0);
  for (size_t i = 0; i < n; ++i) {
    const int s = slot_of[i];
    if (s < -1 || s >= c->n_slots) return fail(c, MOE_ERR_INVALID_ARG, "slot %d out of range", s);
    if (s >= 0) {
      if (used[s]) return fail(c, MOE_ERR_INVALID_ARG, "slot %d used twice", s);
      used[s] = 1;
    }
  }
  c->h_slot_of.assign(slot_of, slot_of + n);
  if (c->host_tier) c->tier.adopt(c->h_slot_of);
  CUDA_TRY(c, cudaMemcpy(c->d_slot_of, slot_of, n * sizeof(int), cudaMemcpyHostToDevice));
  for (int l = 0; l < c->L; ++l) {
    st = refresh_slots(c, l, 0, c->E);
    if (st) return st;
  }
  return MOE_OK;
}

moe_status moe_route(moe_ctx *c, int layer, const void *h, int T, int32_t *idx, float *w,
                     int32_t *boff, int32_t *bperm, void *stream) {
  if (!c) return MOE_ERR_INVALID_ARG;
  if (!c->configured) return fail(c, MOE_ERR_STATE, "nothing loaded");
  if (!valid_layer(c, layer) || !h || !idx || !w || T < 1 || T > c->max_tokens || !aligned16(h))
    return fail(c, MOE_ERR_INVALID_ARG, "moe_route: bad arguments (T=%d max=%d)", T, c->max_tokens);
  if (!c->has_router[layer]) return fail(c, MOE_ERR_STATE, "router of layer %d not set", layer);
  cudaStream_t s = (cudaStream_t)stream;
  c->last_stream = s;
  if (use_prefill_gemm(c, T)) {
    // a chunk in a chunk-configured context: the chunk path's routing, whose
    // parallel sort by expert gives the same buckets as the one-CTA sort below
    moe_status st = prefill_route_impl(c, layer, (const uint16_t *)h, T, idx, w, bperm, s, kHotMinTokens);
    if (st) return st;
    if (boff)
      CUDA_TRY(c, cudaMemcpyAsync(boff, c->pf_eoff, (size_t)(c->E + 1) * sizeof(int32_t),
                                  cudaMemcpyDeviceToDevice, s));
    return MOE_OK;
  }
  FinishParams fp = finish_params(c, layer, T);
  fp.idx = idx;
  fp.w = w;
  fp.off = boff ? boff : c->off;
  fp.perm = bperm ? bperm : c->perm;
  fp.build_jobs = 0;
  // moe_route takes the router input directly: no RMSNorm here
  const char saved = c->has_norm[layer];
  c->has_norm[layer] = 0;
  moe_status st = route_impl(c, layer, (const uint16_t *)h, T, fp, s, nullptr);
  c->has_norm[layer] = saved;
  return st;
}

moe_status moe_set_host_tier(moe_ctx *c, int enable, int policy, double half_life) {
  if (!c) return MOE_ERR_INVALID_ARG;
  if (c->configured) return fail(c, MOE_ERR_STATE, "moe_set_host_tier after configuration/loads");
  if ((enable != 0 && enable != 1) || (policy != moe::kLru && policy != moe::kAdaptive) || !(half_life > 0))
    return fail(c, MOE_ERR_INVALID_ARG, "moe_set_host_tier: bad arguments");
  c->host_tier = enable;
  c->tier_policy = policy;
  c->tier_half_life = half_life;
  return MOE_OK;
}

moe_status moe_tier_prepare(moe_ctx *c, int layer, const int32_t *idx_dev, int T, void *stream) {
  if (!c) return MOE_ERR_INVALID_ARG;
  if (!c->configured || !c->host_tier) return fail(c, MOE_ERR_STATE, "moe_tier_prepare: no host tier");
  if (!valid_layer(c, layer) || !idx_dev || T < 1 || T > c->max_tokens)
    return fail(c, MOE_ERR_INVALID_ARG, "moe_tier_prepare: bad arguments");
  return tier_request(c, layer, idx_dev, T, (cudaStream_t)stream, true);
}

moe_status moe_tier_prefetch(moe_ctx *c, int layer, const int32_t *idx_dev, int T, void *stream) {
  if (!c) return MOE_ERR_INVALID_ARG;
  if (!c->configured || !c->host_tier) return fail(c, MOE_ERR_STATE, "moe_tier_prefetch: no host tier");
  if (!valid_layer(c, layer) || !idx_dev || T < 1 || T > c->max_tokens)
    return fail(c, MOE_ERR_INVALID_ARG, "moe_tier_prefetch: bad arguments");
  return tier_request(c, layer, idx_dev, T, (cudaStream_t)stream, false);
}

moe_status moe_forward_tiered(moe_ctx *c, int layer, void *x, int T, void *stream) {
  if (!c) return MOE_ERR_INVALID_ARG;
  if (!c->configured || !c->host_tier) return fail(c, MOE_ERR_STATE, "moe_forward_tiered: no host tier");
  if (!valid_layer(c, layer) || !x || T < 1 || T > c->max_tokens || !aligned16(x))
    return fail(c, MOE_ERR_INVALID_ARG, "moe_forward_tiered: bad arguments");
  moe_status st = check_ready(c, layer);
  if (st) return st;
  cudaStream_t s = (cudaStream_t)stream;
  c->last_stream = s;
  // the window's routing (with the layer's RMSNorm, as the forward computes it)
  FinishParams fp = finish_params(c, layer, T);
  fp.idx = c->tier_idx;
  fp.w = c->tier_w;
  fp.off = c->off;
  fp.perm = c->perm;
  fp.build_jobs = 0;
  st = route_impl(c, layer, (const uint16_t *)x, T, fp, s, nullptr);
  if (st) return st;
  st = tier_request(c, layer, c->tier_idx, T, s, true);
  if (st) return st;
  return forward_impl(c, layer, (uint16_t *)x, T, nullptr, s);
}

moe_status moe_tier_stats(moe_ctx *c, long long *out) {
  if (!c || !out) return MOE_ERR_INVALID_ARG;
  if (!c->host_tier) return fail(c, MOE_ERR_STATE, "moe_tier_stats: no host tier");
  int used = 0;
  for (long long o : c->tier.owner) used += o >= 0 ? 1 : 0;
  out[0] = c->tier.hits;
  out[1] = c->tier.misses;
  out[2] = c->tier.evictions;
  out[3] = c->tier_bytes;
  out[4] = c->tier_calls;
  out[5] = used;
  return MOE_OK;
}

moe_status moe_tier_dump_trace(moe_ctx *c, const char *path) {
  if (!c || !path) return MOE_ERR_INVALID_ARG;
  if (!c->host_tier) return fail(c, MOE_ERR_STATE, "moe_tier_dump_trace: no host tier");
  FILE *fh = fopen(path, "w");
  if (!fh) return fail(c, MOE_ERR_INVALID_ARG, "cannot open %s", path);
  fprintf(fh, "# request layer n_experts experts...\n");
  const std::vector<int> &tr = c->tier_trace;
  for (size_t i = 0; i + 3 <= tr.size();) {
    const int n = tr[i + 2];
    fprintf(fh, "%d %d %d", tr[i], tr[i + 1], n);
    for (int j = 0; j < n; ++j) fprintf(fh, " %d", tr[i + 3 + j]);
    fprintf(fh, "\n");
    i += 3 + (size_t)n;
  }
  const bool ok = fclose(fh) == 0;
  return ok ? MOE_OK : fail(c, MOE_ERR_INVALID_ARG, "cannot write %s", path);
}

// Host-only model of the tier's replacement policy (no device needed).
typedef std::pair<moe::TierCache, std::vector<int>> TierSim;

void *moe_tier_sim_create(int n_slots, int policy, double half_life, long long n_keys) {
  if (n_slots < 1 || n_keys < 1 || (policy != moe::kLru && policy != moe::kAdaptive) || !(half_life > 0))
    return nullptr;
  TierSim *sim = new TierSim();
  sim->first.init(n_slots, policy, half_life, n_keys);
  sim->second.assign((size_t)n_keys, -1);
  return sim;
}

int moe_tier_sim_request(void *h, const long long *keys, int n, int protect_prev, int *slots_out) {
  TierSim *sim = static_cast<TierSim *>(h);
  if (!sim || (!keys && n > 0) || n < 0) return -1;
  std::vector<long long> ks;
  std::vector<char> seen(sim->second.size(), 0);
  for (int i = 0; i < n; ++i) {
    if (keys[i] < 0 || keys[i] >= (long long)sim->second.size() || seen[(size_t)keys[i]]) return -1;
    seen[(size_t)keys[i]] = 1;
    ks.push_back(keys[i]);
  }
  std::vector<long long> fk, fe;
  std::vector<int> fs;
  if (!sim->first.request(ks, sim->second, protect_prev != 0, fk, fs, fe)) return -2;
  if (slots_out)
    for (int i = 0; i < n; ++i) slots_out[i] = sim->second[(size_t)keys[i]];
  return (int)fk.size();  // misses of this request
}

void moe_tier_sim_counts(void *h, long long *out) {
  TierSim *sim = static_cast<TierSim *>(h);
  if (!sim || !out) return;
  out[0] = sim->first.hits;
  out[1] = sim->first.misses;
  out[2] = sim->first.evictions;
}

void moe_tier_sim_destroy(void *h) { delete static_cast<TierSim *>(h); }

moe_status moe_bucket(moe_ctx *c, const int32_t *idx, int T, int32_t *boff, int32_t *bperm,
                      void *stream) {
  if (!c) return MOE_ERR_INVALID_ARG;
  moe_status st = ensure_configured(c);
  if (st) return st;
  if (!idx || !boff || !bperm || T < 1 || T > c->max_tokens)
    return fail(c, MOE_ERR_INVALID_ARG, "moe_bucket: bad arguments");
  FinishParams fp = finish_params(c, 0, T);
  fp.logits = nullptr;
  fp.idx_in = idx;
  fp.off = boff;
  fp.perm = bperm;
  fp.build_jobs = 0;
  c->last_stream = (cudaStream_t)stream;
  CUDA_TRY(c, launch_finish(c, (cudaStream_t)stream, fp));
  return MOE_OK;
}

moe_status moe_forward(moe_ctx *c, int layer, void *x, int T, void *stream) {
  if (!c) return MOE_ERR_INVALID_ARG;
  if (!c->configured) return fail(c, MOE_ERR_STATE, "nothing loaded");
  if (!valid_layer(c, layer) || !x || T < 1 || T > c->max_tokens || !aligned16(x))
    return fail(c, MOE_ERR_INVALID_ARG, "moe_forward: bad arguments (T=%d max=%d)", T,
                c->max_tokens);
  moe_status st = check_ready(c, layer);
  if (st) return st;
  c->last_stream = (cudaStream_t)stream;
  return forward_impl(c, layer, (uint16_t *)x, T, nullptr, (cudaStream_t)stream);
}

moe_status moe_forward_delta(moe_ctx *c, int layer, const void *x, int T, float *delta,
                             void *stream) {
  if (!c) return MOE_ERR_INVALID_ARG;
  if (!c->configured) return fail(c, MOE_ERR_STATE, "nothing loaded");
  if (!valid_layer(c, layer) || !x || !delta || T < 1 || T > c->max_tokens || !aligned16(x) ||
      !aligned16(delta))
    return fail(c, MOE_ERR_INVALID_ARG, "moe_forward_delta: bad arguments");
  moe_status st = check_ready(c, layer);
  if (st) return st;
  c->last_stream = (cudaStream_t)stream;
  return forward_impl(c, layer, (uint16_t *)const_cast<void *>(x), T, delta,
                      (cudaStream_t)stream);
}

moe_status moe_forward_stack(moe_ctx *c, void *x, int T, void *stream) {
  if (!c) return MOE_ERR_INVALID_ARG;
  if (!c->configured) return fail(c, MOE_ERR_STATE, "nothing loaded");
  if (!x || T < 1 || T > c->max_tokens || !aligned16(x))
    return fail(c, MOE_ERR_INVALID_ARG, "moe_forward_stack");
  for (int l = 0; l < c->L; ++l) {
    moe_status st = check_ready(c, l);
    if (st) return st;
  }
  cudaStream_t s = (cudaStream_t)stream;
  auto key = std::make_pair(x, T);
  auto it = c->stack_graphs.find(key);
  if (it == c->stack_graphs.end()) {
    cudaStream_t cap = nullptr;
    CUDA_TRY(c, cudaStreamCreateWithFlags(&cap, cudaStreamNonBlocking));
    cudaGraph_t graph = nullptr;
    cudaError_t e = cudaStreamBeginCapture(cap, cudaStreamCaptureModeThreadLocal);
    moe_status st = MOE_OK;
    if (e == cudaSuccess) {
      for (int l = 0; l < c->L && st == MOE_OK; ++l)
        st = forward_impl(c, l, (uint16_t *)x, T, nullptr, cap);
      e = cudaStreamEndCapture(cap, &graph);
    }
    cudaGraphExec_t exec = nullptr;
    if (e == cudaSuccess && st == MOE_OK) e = cudaGraphInstantiate(&exec, graph, 0);
    if (graph) cudaGraphDestroy(graph);
    cudaStreamDestroy(cap);
    if (st != MOE_OK) return st;
    CUDA_TRY(c, e);
    it = c->stack_graphs.emplace(key, exec).first;
  }
  c->last_stream = s;
  CUDA_TRY(c, cudaGraphLaunch(it->second, s));
  return MOE_OK;
}

moe_status moe_prefill(moe_ctx *c, int layer, void *x, int N, void *stream) {
  if (!c) return MOE_ERR_INVALID_ARG;
  if (!c->configured) return fail(c, MOE_ERR_STATE, "nothing loaded");
  if (!valid_layer(c, layer) || !x || N < 1 || N > c->max_tokens || !aligned16(x))
    return fail(c, MOE_ERR_INVALID_ARG, "moe_prefill: bad arguments (N=%d max=%d)", N,
                c->max_tokens);
  moe_status st = check_ready(c, layer);
  if (st) return st;
  c->last_stream = (cudaStream_t)stream;
  if (!use_prefill_gemm(c, N))
    return forward_impl(c, layer, (uint16_t *)x, N, nullptr, (cudaStream_t)stream);
  return prefill_impl(c, layer, (uint16_t *)x, N, nullptr, (cudaStream_t)stream);
}

moe_status moe_prefill_delta(moe_ctx *c, int layer, const void *x, int N, float *delta,
                             void *stream) {
  if (!c) return MOE_ERR_INVALID_ARG;
  if (!c->configured) return fail(c, MOE_ERR_STATE, "nothing loaded");
  if (!valid_layer(c, layer) || !x || !delta || N < 1 || N > c->max_tokens || !aligned16(x) ||
      !aligned16(delta))
    return fail(c, MOE_ERR_INVALID_ARG, "moe_prefill_delta: bad arguments");
  moe_status st = check_ready(c, layer);
  if (st) return st;
  c->last_stream = (cudaStream_t)stream;
  uint16_t *xp = (uint16_t *)const_cast<void *>(x);
  if (!use_prefill_gemm(c, N)) return forward_impl(c, layer, xp, N, delta, (cudaStream_t)stream);
  return prefill_impl(c, layer, xp, N, delta, (cudaStream_t)stream);
}

moe_status moe_prefill_route(moe_ctx *c, int layer, const void *h, int N, int32_t *idx, float *w,
                             int32_t *boff, int32_t *bperm, void *stream) {
  if (!c) return MOE_ERR_INVALID_ARG;
  if (!c->configured) return fail(c, MOE_ERR_STATE, "nothing loaded");
  if (!valid_layer(c, layer) || !h || !idx || !w || N < 1 || N > c->max_tokens || !aligned16(h))
    return fail(c, MOE_ERR_INVALID_ARG, "moe_prefill_route: bad arguments (N=%d max=%d)", N,
                c->max_tokens);
  if (!c->pf)
    return fail(c, MOE_ERR_NOT_SUPPORTED,
                "moe_prefill_route: context configured for decode windows only (max_tokens <= 32)");
  if (!c->has_router[layer]) return fail(c, MOE_ERR_STATE, "router of layer %d not set", layer);
  cudaStream_t s = (cudaStream_t)stream;
  c->last_stream = s;
  moe_status st = prefill_route_impl(c, layer, (const uint16_t *)h, N, idx, w, bperm, s, kHotMinTokens);
  if (st) return st;
  if (boff)
    CUDA_TRY(c, cudaMemcpyAsync(boff, c->pf_eoff, (size_t)(c->E + 1) * sizeof(int32_t),
                                cudaMemcpyDeviceToDevice, s));
  return MOE_OK;
}

moe_status moe_rmsnorm(moe_ctx *c, int layer, const void *x, int T, void *h, void *stream) {
  if (!c) return MOE_ERR_INVALID_ARG;
  if (!c->configured) return fail(c, MOE_ERR_STATE, "nothing loaded");
  if (!valid_layer(c, layer) || !x || !h || T < 1 || !aligned16(x) || !aligned16(h))
    return fail(c, MOE_ERR_INVALID_ARG, "moe_rmsnorm: bad arguments");
  cudaStream_t s = (cudaStream_t)stream;
  c->last_stream = s;
  if (!c->has_norm[layer]) {
    CUDA_TRY(c, cudaMemcpyAsync(h, x, (size_t)T * c->d * 2, cudaMemcpyDeviceToDevice, s));
    return MOE_OK;
  }
  NormParams np{(const uint16_t *)x, c->has_gamma[layer] ? c->d_gamma + (size_t)layer * c->d : nullptr,
                c->eps[layer], T, c->d, (uint16_t *)h};
  CUDA_TRY(c, launch(rmsnorm_kernel, dim3(T), dim3(256), 0, s, np));
  return MOE_OK;
}

// Checks shared by the calls on given routing; the ids are copied to the
// host and checked before any launch (one stream synchronisation).
static moe_status given_check(moe_ctx *c, int layer, const void *h, int N, int kk, const int32_t *idx,
                              int with_shared, const void *out, cudaStream_t s, const char *who) {
  if (!c->configured) return fail(c, MOE_ERR_STATE, "nothing loaded");
  if (!valid_layer(c, layer) || !h || !out || N < 1 || N > c->max_tokens || kk < 0 || kk > c->k ||
      (kk > 0 && !idx) || (kk == 0 && !with_shared) || !aligned16(h) || !aligned16(out))
    return fail(c, MOE_ERR_INVALID_ARG, "%s: bad arguments (N=%d max=%d kk=%d k=%d)", who, N, c->max_tokens,
                kk, c->k);
  if (with_shared && !c->n_shared) return fail(c, MOE_ERR_INVALID_ARG, "%s: no shared expert configured", who);
  if (!c->pf || c->pf_pairs <= 0 || c->d % (2 * kPfBN) != 0 || c->f % kPfBN != 0 || c->E > kPfMaxE)
    return fail(c, MOE_ERR_NOT_SUPPORTED,
                "%s: needs a chunk-configured context (max_tokens > 32) and the grouped GEMM's shapes", who);
  if (with_shared && !c->shared_loaded[layer])
    return fail(c, MOE_ERR_STATE, "shared expert of layer %d not loaded", layer);
  if (kk > 0) {
    // the ids index the kernels' tables: check them before any launch
    std::vector<int32_t> ids((size_t)N * kk);
    CUDA_TRY(c, cudaMemcpyAsync(ids.data(), idx, ids.size() * sizeof(int32_t), cudaMemcpyDeviceToHost, s));
    CUDA_TRY(c, cudaStreamSynchronize(s));
    const auto &loaded = c->expert_loaded[layer];
    for (int t = 0; t < N; ++t)
      for (int j = 0; j < kk; ++j) {
        const int e = ids[(size_t)t * kk + j];
        if (e < 0 || e >= c->E)
          return fail(c, MOE_ERR_INVALID_ARG, "%s: id %d of row %d outside [0, %d)", who, e, t, c->E);
        if (!loaded[e]) return fail(c, MOE_ERR_STATE, "%s: expert %d of layer %d not loaded", who, e, layer);
        for (int i = 0; i < j; ++i)
          if (ids[(size_t)t * kk + i] == e)
            return fail(c, MOE_ERR_INVALID_ARG, "%s: row %d selects expert %d twice", who, t, e);
      }
  }
  return MOE_OK;
}

moe_status moe_experts_given(moe_ctx *c, int layer, const void *h, int N, int kk, const int32_t *idx,
                             const float *w, int with_shared, float *delta, void *stream) {
  if (!c) return MOE_ERR_INVALID_ARG;
  cudaStream_t s = (cudaStream_t)stream;
  if (kk > 0 && !w) return fail(c, MOE_ERR_INVALID_ARG, "moe_experts_given: weights missing");
  moe_status st = given_check(c, layer, h, N, kk, idx, with_shared, delta, s, "moe_experts_given");
  if (st) return st;
  c->last_stream = s;
  return given_impl(c, layer, (const uint16_t *)h, N, kk, idx, w, with_shared != 0, delta, s);
}

moe_status moe_experts_rows(moe_ctx *c, int layer, const void *h, int M, const int32_t *e, void *y_dev,
                            void *stream) {
  if (!c) return MOE_ERR_INVALID_ARG;
  cudaStream_t s = (cudaStream_t)stream;
  if (!e) return fail(c, MOE_ERR_INVALID_ARG, "moe_experts_rows: expert ids missing");
  moe_status st = given_check(c, layer, h, M, 1, e, 0, y_dev, s, "moe_experts_rows");
  if (st) return st;
  c->last_stream = s;
  return given_impl(c, layer, (const uint16_t *)h, M, 1, e, nullptr, false, nullptr, s,
                    reinterpret_cast<__half *>(y_dev));
}

moe_status moe_ep_dispatch(moe_ctx *c, const int32_t *idx, int N, int n_ranks, const void *h,
                           void *send_h, int32_t *send_e, int32_t *row_of, int32_t *counts_host,
                           void *stream) {
  if (!c) return MOE_ERR_INVALID_ARG;
  if (!idx || !h || !send_h || !send_e || !row_of || !counts_host || N < 1 || n_ranks < 1 ||
      n_ranks > kEpMaxRanks || c->E % n_ranks != 0 || !aligned16(h) || !aligned16(send_h) ||
      (long long)N * c->k > (1LL << 30))
    return fail(c, MOE_ERR_INVALID_ARG, "moe_ep_dispatch: bad arguments (N=%d ranks=%d E=%d)", N, n_ranks,
                c->E);
  if (!c->configured) return fail(c, MOE_ERR_STATE, "nothing loaded");
  cudaStream_t s = (cudaStream_t)stream;
  c->last_stream = s;
  const long long P = (long long)N * c->k;
  const int blocks = (int)((P + kEpBlockPairs - 1) / kEpBlockPairs);
  const long long need = kEpMaxRanks + 2LL * blocks * n_ranks;
  if (need > c->ep_scratch_n) {  // grows to the largest dispatch seen
    CUDA_TRY(c, cudaStreamSynchronize(s));
    dfree(c->ep_counts);
    CUDA_TRY(c, cudaMalloc(&c->ep_counts, (size_t)need * sizeof(int)));
    c->ep_scratch_n = need;
  }
  EpPlanParams pp{idx, (const uint16_t *)h, N, c->k, c->d, c->E, n_ranks, blocks,
                  c->ep_counts + kEpMaxRanks, c->ep_counts + kEpMaxRanks + (long long)blocks * n_ranks,
                  c->ep_counts, row_of, send_e, (uint16_t *)send_h, c->status};
  CUDA_TRY(c, launch(ep_count_kernel, dim3(blocks), dim3(kEpBlockPairs), 0, s, pp));
  CUDA_TRY(c, launch(ep_offsets_kernel, dim3(1), dim3(1024), 0, s, pp));
  CUDA_TRY(c, launch(ep_place_kernel, dim3(blocks), dim3(kEpBlockPairs), 0, s, pp));
  CUDA_TRY(c, cudaMemcpyAsync(counts_host, c->ep_counts, n_ranks * sizeof(int), cudaMemcpyDeviceToHost, s));
  CUDA_TRY(c, cudaStreamSynchronize(s));
  return MOE_OK;
}

moe_status moe_ep_combine(moe_ctx *c, int N, const float *w, const void *y, const int32_t *row_of,
                          const float *y_shared, void *x, float *delta, void *stream) {
  if (!c) return MOE_ERR_INVALID_ARG;
  if (N < 1 || !w || !y || !row_of || (!x == !delta) || !aligned16(y) ||
      (y_shared && !aligned16(y_shared)) || (x && !aligned16(x)) || (delta && !aligned16(delta)))
    return fail(c, MOE_ERR_INVALID_ARG, "moe_ep_combine: bad arguments");
  cudaStream_t s = (cudaStream_t)stream;
  c->last_stream = s;
  EpCombineParams mp{reinterpret_cast<const __half *>(y), row_of, w, y_shared, N, c->k, c->d, (uint16_t *)x,
                     delta};
  const long long n4 = (long long)N * c->d / 4;
  const int cblocks = (int)std::min<long long>((n4 + 255) / 256, 8LL * c->n_sm);
  CUDA_TRY(c, launch(ep_combine_kernel, dim3(cblocks), dim3(256), 0, s, mp));
  return MOE_OK;
}

moe_status moe_sync(moe_ctx *c, int timeout_ms) {
  if (!c) return MOE_ERR_INVALID_ARG;
  if (!c->configured) return MOE_OK;
  // poll the stream of the most recent compute call, with a bound
  const auto t0 = std::chrono::steady_clock::now();
  for (;;) {
    cudaError_t e = cudaStreamQuery(c->last_stream);
    if (e == cudaSuccess) break;
    if (e != cudaErrorNotReady) CUDA_TRY(c, e);
    if (timeout_ms >= 0 &&
        std::chrono::steady_clock::now() - t0 > std::chrono::milliseconds(timeout_ms))
      return fail(c, MOE_ERR_TIMEOUT, "moe_sync: not done after %d ms", timeout_ms);
    std::this_thread::sleep_for(std::chrono::microseconds(50));
  }
  int st = 0;
  CUDA_TRY(c, cudaMemcpyAsync(&st, c->status, sizeof(int), cudaMemcpyDeviceToHost, c->io));
  CUDA_TRY(c, cudaMemsetAsync(c->status, 0, sizeof(int), c->io));
  // a kernel that gave up a wait may have left a counter mid-count: start
  // the decode grid barrier, its hand-over flags and the fused-routing
  // ticket again from zero
  if (st & kErrTimeout) {
    CUDA_TRY(c, cudaMemsetAsync(c->dec_bar, 0, c->dec_sync_bytes, c->io));
    CUDA_TRY(c, cudaMemsetAsync(c->ticket, 0, 2 * sizeof(unsigned int), c->io));
  }
  CUDA_TRY(c, cudaStreamSynchronize(c->io));
  if (st & kErrBadSlot) return fail(c, MOE_ERR_BAD_SLOT, "device status 0x%x: bad slot", st);
  if (st) return fail(c, MOE_ERR_DEVICE, "device status 0x%x", st);
  return MOE_OK;
}

moe_status moe_get_stats(moe_ctx *c, moe_stats *out) {
  if (!c || !out) return MOE_ERR_INVALID_ARG;
  std::memset(out, 0, sizeof *out);
  if (!c->configured) return MOE_OK;
  CUDA_TRY(c, cudaStreamSynchronize(c->last_stream));
  unsigned long long s[8];
  int last[4];
  CUDA_TRY(c, cudaMemcpyAsync(s, c->stats, sizeof s, cudaMemcpyDeviceToHost, c->io));
  CUDA_TRY(c, cudaMemcpyAsync(last, c->last, sizeof last, cudaMemcpyDeviceToHost, c->io));
  CUDA_TRY(c, cudaMemcpyAsync(c->host_counts.data(), c->cnt_out, (size_t)c->E * sizeof(int),
                              cudaMemcpyDeviceToHost, c->io));
  CUDA_TRY(c, cudaStreamSynchronize(c->io));
  out->calls = (int64_t)s[0];
  out->tokens = (int64_t)s[1];
  out->hits = (int64_t)s[2];
  out->misses = (int64_t)s[3];
  out->near_ties = (int64_t)s[4];
  out->last_T = last[0];
  out->last_active = last[1];
  out->last_layer = last[2];
  out->E = c->E;
  out->expert_count = c->host_counts.data();
  return MOE_OK;
}

moe_status moe_set_profiling(moe_ctx *c, int enable) {
  if (!c) return MOE_ERR_INVALID_ARG;
  if (enable && c->prof_ev.empty()) {
    c->prof_ev.resize((size_t)kProfSlots * 4, nullptr);
    for (auto &ev : c->prof_ev) CUDA_TRY(c, cudaEventCreate(&ev));
  }
  c->profiling = enable != 0;
  c->prof_next = 0;
  c->prof_pending = 0;
  return MOE_OK;
}

moe_status moe_read_profile(moe_ctx *c, double ms[3], int64_t *n_calls) {
  if (!c || !ms || !n_calls) return MOE_ERR_INVALID_ARG;
  *n_calls = 0;
  if (c->prof_ev.empty()) return MOE_OK;
  // the pending calls are the prof_pending slots ending at prof_next - 1;
  // for replayed graphs every recorded slot is re-read
  const int n = c->prof_pending;
  for (int i = 0; i < n; ++i) {
    const int slot = ((c->prof_next - n + i) % kProfSlots + kProfSlots) % kProfSlots;
    float seg[3];
    CUDA_TRY(c, cudaEventSynchronize(c->prof_ev[(size_t)slot * 4 + 3]));
    for (int j = 0; j < 3; ++j)
      CUDA_TRY(c, cudaEventElapsedTime(&seg[j], c->prof_ev[(size_t)slot * 4 + j],
                                       c->prof_ev[(size_t)slot * 4 + j + 1]));
    for (int j = 0; j < 3; ++j) ms[j] += seg[j];
  }
  *n_calls = n;
  return MOE_OK;
}

moe_status moe_set_trace(moe_ctx *c, int enable) {
  if (!c) return MOE_ERR_INVALID_ARG;
  unsigned long long *buf = nullptr;
  if (enable) {
    if (!c->trace) CUDA_TRY(c, cudaMalloc(&c->trace, 2 * kTrCount * sizeof(unsigned long long)));
    CUDA_TRY(c, cudaMemset(c->trace, 0xFF, kTrCount * sizeof(unsigned long long)));
    CUDA_TRY(c, cudaMemset(c->trace + kTrCount, 0, kTrCount * sizeof(unsigned long long)));
    buf = c->trace;
  }
  CUDA_TRY(c, cudaDeviceSynchronize());
  CUDA_TRY(c, cudaMemcpyToSymbol(g_trace, &buf, sizeof buf));
  return MOE_OK;
}

moe_status moe_read_trace(moe_ctx *c, int64_t *out, int n) {
  if (!c || !out || n < 2 * kTrCount) return fail(c, MOE_ERR_INVALID_ARG, "moe_read_trace");
  if (!c->trace) return fail(c, MOE_ERR_STATE, "tracing was never enabled");
  CUDA_TRY(c, cudaDeviceSynchronize());
  CUDA_TRY(c, cudaMemcpy(out, c->trace, 2 * kTrCount * sizeof(int64_t), cudaMemcpyDeviceToHost));
  CUDA_TRY(c, cudaMemset(c->trace, 0xFF, kTrCount * sizeof(unsigned long long)));
  CUDA_TRY(c, cudaMemset(c->trace + kTrCount, 0, kTrCount * sizeof(unsigned long long)));
  return MOE_OK;
}

// Debug hook: write one raw slot-table entry on the device without host
// validation, so tests can check the device-side detection of a corrupted
// residency table (kErrBadSlot -> MOE_ERR_BAD_SLOT from moe_sync).
moe_status moe_debug_poke_slot(moe_ctx *c, int layer, int expert, int32_t slot) {
  if (!c || !c->configured || !valid_layer(c, layer) || expert < 0 || expert >= c->E)
    return fail(c, MOE_ERR_INVALID_ARG, "moe_debug_poke_slot");
  CUDA_TRY(c, cudaMemcpy(c->d_slot_of + (size_t)layer * c->E + expert, &slot, sizeof slot,
                         cudaMemcpyHostToDevice));
  return MOE_OK;
}

// Test hook: the next single-launch decode (moe_forward / moe_forward_delta
// of a window of <= 32 tokens) gets a first grid barrier that cannot
// complete, with a poll limit of `polls`; its bounded wait runs out, the
// kernel reports kErrTimeout and leaves, and moe_sync reports it.
moe_status moe_debug_stall_next_decode(moe_ctx *c, uint32_t polls) {
  if (!c || polls < 1) return fail(c, MOE_ERR_INVALID_ARG, "moe_debug_stall_next_decode");
  c->dec_stall_next = 1;
  c->dec_stall_polls = polls;
  return MOE_OK;
}

// Debug hook: the normalised router input h (bf16 [T, d]) that the most
// recent forward or prefill call of a layer with RMSNorm computed, copied on
// `stream` into caller memory.
moe_status moe_debug_last_h(moe_ctx *c, void *out, int T, void *stream) {
  if (!c || !out || !c->configured || T < 1 || T > c->max_tokens)
    return fail(c, MOE_ERR_INVALID_ARG, "moe_debug_last_h");
  CUDA_TRY(c, cudaMemcpyAsync(out, c->hbuf, (size_t)T * c->d * 2, cudaMemcpyDeviceToDevice,
                              (cudaStream_t)stream));
  return MOE_OK;
}

}  // extern "C"

// ======================================================================
// Routing with no allocation at all.
//
// Some callers cannot call cudaMalloc: code running inside a CUDA graph
// that is being captured or re-instantiated under a fixed memory budget,
// engines that hand every byte of device memory to their own pool up front
// and forbid the driver allocator afterwards, or plugins that are given only
// raw device pointers by a host framework.  moe_route_static serves them:
// it needs no context, takes the router weights as a device pointer, and
// keeps its only scratch -- the fp32 logits, the CTA completion ticket and a
// status word -- in the file-scope device array below.  Every GPU that loads
// this library holds that array (kStaticScratchBytes) until the process
// exits.  The array is shared by every call on a device and keeps the last
// call's contents; each call clears the words that must start at zero.  Two
// calls whose execution overlaps on the GPU race on it.
namespace {

constexpr int kStaticMaxT = kFusedMaxT;  // tokens per call
constexpr int kStaticMaxE = 1024;        // experts
constexpr int kStaticMaxD = kFusedMaxV * 128;
constexpr size_t kStaticHeader = 256;    // ticket + abort flag, status, statistics words
constexpr size_t kStaticStatusOff = 16;  // the status word, inside the header
constexpr size_t kStaticScratchBytes =
    kStaticHeader + (size_t)kStaticMaxT * kStaticMaxE * sizeof(float);

static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_static_mu;
unsigned char *g_static_addr[kMaxDevices] = {};  // device address, per device

// Once per device, with that device current: the device address of the
// scratch array (a host-side name of a __device__ array is not a device
// address) and the shared-memory limit of the routing kernels.
cudaError_t static_scratch(int dev, unsigned char **out) {
  std::lock_guard<std::mutex> lock(g_static_mu);
  if (!g_static_addr[dev]) {
    void *p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_static_scratch);
    if (e != cudaSuccess) return e;
    e = setup_route_fused();
    if (e != cudaSuccess) return e;
    g_static_addr[dev] = static_cast<unsigned char *>(p);
  }
  *out = g_static_addr[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" {

moe_status moe_route_static(const void *h, int T, int d, int E, int k, const float *W,
                            const float *bias, int32_t *idx, float *w, int32_t *boff,
                            int32_t *bperm, void *stream) {
  if (!h || !W || !idx || !w || !boff || !bperm || T < 1 || T > kStaticMaxT || d < 128 ||
      d % 128 || d > kStaticMaxD || E < 1 || E > kStaticMaxE || k < 1 || k > E || k > 32 ||
      !aligned16(h) || !aligned16(W))
    return MOE_ERR_INVALID_ARG;
  const size_t smem = std::max((size_t)T * d * 2, (size_t)finish_smem_ints(E, T * k) * sizeof(int));
  if (smem > (size_t)kFusedSmem) return MOE_ERR_INVALID_ARG;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    (void)cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  unsigned char *base = nullptr;
  if (static_scratch(dev, &base) != cudaSuccess) {
    (void)cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  cudaStream_t s = (cudaStream_t)stream;
  // ticket, status and the statistics words must start at zero
  if (cudaMemsetAsync(base, 0, kStaticHeader, s) != cudaSuccess) {
    (void)cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  RouteFusedParams rp{};
  rp.x = (const uint16_t *)h;
  rp.use_norm = 0;
  rp.W = W;
  rp.bias = bias;
  rp.d = d;
  rp.logits = reinterpret_cast<float *>(base + kStaticHeader);
  rp.ticket = reinterpret_cast<unsigned int *>(base);
  FinishParams &fp = rp.f;
  fp.T = T;
  fp.E = E;
  fp.k = k;
  fp.logits = rp.logits;
  fp.idx = idx;
  fp.w = w;
  fp.off = boff;
  fp.perm = bperm;
  fp.build_jobs = 0;
  fp.status = reinterpret_cast<int *>(base + kStaticStatusOff);
  fp.stats = reinterpret_cast<unsigned long long *>(base + 64);
  const int warps = T <= 8 ? 4 : kFusedWarps;
  const dim3 grid((E + warps - 1) / warps), block(warps * 32);
  cudaError_t e;
  switch (finish_npl(E)) {
    case 1: e = launch(route_fused_kernel<1>, grid, block, smem, s, rp); break;
    case 2: e = launch(route_fused_kernel<2>, grid, block, smem, s, rp); break;
    case 4: e = launch(route_fused_kernel<4>, grid, block, smem, s, rp); break;
    case 8: e = launch(route_fused_kernel<8>, grid, block, smem, s, rp); break;
    case 16: e = launch(route_fused_kernel<16>, grid, block, smem, s, rp); break;
    default: e = launch(route_fused_kernel<32>, grid, block, smem, s, rp); break;
  }
  if (e != cudaSuccess) {
    (void)cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  return MOE_OK;
}

moe_status moe_route_static_status(int *status_out, void *stream) {
  if (!status_out) return MOE_ERR_INVALID_ARG;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    (void)cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  unsigned char *base = nullptr;
  if (static_scratch(dev, &base) != cudaSuccess) {
    (void)cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  cudaStream_t s = (cudaStream_t)stream;
  int st = 0;
  cudaError_t e = cudaMemcpyAsync(&st, base + kStaticStatusOff, sizeof(int), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) {
    (void)cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  *status_out = st;
  return st ? MOE_ERR_DEVICE : MOE_OK;
}

}  // extern "C"
