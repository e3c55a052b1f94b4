/*
 * moe.h -- C ABI of libmoe.so, a single-GPU (sm_100a) implementation of the
 * sparse Mixture-of-Experts expert layer: router -> top-k -> residency
 * lookup -> bucketing -> dequantised SwiGLU experts -> weighted combine +
 * residual write-back.
 *
 * The problem statement these calls follow is the per-layer flow of the
 * Strata engine analysis article "93 token/s on one 8 GB card"
 * (m.lqnn.cn/news/264700), section "Architecture overview": prompts are cut
 * into chunks of at most 8,192 tokens for prefill; then, layer by layer, the
 * router picks the 10 of 512 experts a token activates, the selected experts
 * are computed, and their outputs are combined into the residual.  The
 * "Doorbell handshake" section splits each block at the router ("pre" ends
 * with router ids + weights, "post" combines expert outputs and writes the
 * residual back); the "Expert cache" section defines the residency table
 * (layer, expert) -> slot or -1.  The model shape (48 layers, 512 experts,
 * 10 routed + 1 shared) is from lcz.me topic 2059, section 2 "Model and
 * principles".
 *
 * Conventions (all calls):
 *  - Every call returns a moe_status; no exception or exit() crosses the ABI.
 *    moe_last_error(ctx) gives a one-line description of the last failure.
 *  - Pointers named *_dev are device pointers the caller owns (for example
 *    torch tensors' data_ptr()); the library never frees them.  Weight-load
 *    calls take host or device pointers (src_is_device) and COPY the data;
 *    the caller may free its buffers as soon as the call returns.
 *  - `stream` is a cudaStream_t passed as void*; NULL means the legacy
 *    default stream.  Compute calls are asynchronous on that stream; the
 *    caller must keep its buffers alive until the stream passes the call.
 *  - Layouts are row-major and densely packed unless stated otherwise.
 *    Activations are bfloat16 bit patterns (uint16), router weights fp32.
 *  - A context is used from one host thread at a time and on the device that
 *    was current when it was created.  Its compute calls share the context's
 *    scratch memory, so calls on different streams must not overlap: issue
 *    them on one stream, or order the streams.  (Chunk calls fork internal
 *    work to a stream of the context's own and join it before they return
 *    to the caller's stream.)
 *
 * Packed expert format (input of moe_load_experts / moe_load_shared).  The
 * pages print no bit layout; these formats are this library's own:
 *  - One expert is the triple Wg [f,d], Wu [f,d], Wd [d,f] (row-major; the
 *    reduction dimension is contiguous).  y = Wd (SiLU(Wg h) * (Wu h)),
 *    SiLU(z) = z / (1 + exp(-z)).
 *  - MOE_Q4_SYM_G32_F16: groups of 32 along the reduction dimension;
 *    value = s * (c - 8), c a 4-bit code, two codes per byte with the lower
 *    index in the low nibble; s is an fp16 scale per (row, group).
 *  - MOE_Q2_ASYM_G64_F16: groups of 64; value = s * q + m, q a 2-bit code,
 *    four per byte with element i in bits 2*(i%4); s and m are fp16 per
 *    (row, group).
 *  - codes: for each expert, Wg's codes, then Wu's, then Wd's; experts back
 *    to back.  scales (and mins) follow the same order, [rows, K/group] per
 *    matrix.  Per expert: Q4 3*f*d/2 code bytes + 3*f*d/32 scales;
 *    Q2 3*f*d/4 code bytes + 3*f*d/64 scales + as many mins.
 */
#ifndef MOE_H
#define MOE_H

#include <stdint.h>

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct moe_ctx moe_ctx; /* opaque, library-owned */

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1, /* bad size, index or pointer; nothing was done */
  MOE_ERR_OOM = 2,         /* device allocation failed */
  MOE_ERR_CUDA = 3,        /* a CUDA runtime call failed (see last_error) */
  MOE_ERR_STATE = 4,       /* call order violated (e.g. forward before load) */
  MOE_ERR_BAD_SLOT = 5,    /* device saw a slot id outside the slot pool */
  MOE_ERR_DEVICE = 6,      /* device saw another bad value (expert id, ...) */
  MOE_ERR_TIMEOUT = 7,     /* moe_sync gave up waiting */
  MOE_ERR_NOT_SUPPORTED = 8 /* valid request this build does not handle */
} moe_status;

enum { MOE_Q4_SYM_G32_F16 = 1, MOE_Q2_ASYM_G64_F16 = 2 };

/* Statistics of the most recent routed call (moe_get_stats). */
typedef struct {
  int64_t calls;            /* routed calls since create / last reset */
  int64_t tokens;           /* tokens routed since create */
  int64_t hits;             /* (token, expert) pairs served from the slot pool */
  int64_t misses;           /* pairs served from the backing arena */
  int64_t near_ties;        /* tokens whose k-th and (k+1)-th fp32 logits
                               differ by less than 1e-5 */
  int32_t last_T;           /* tokens of the last routed call */
  int32_t last_active;      /* distinct experts of the last call */
  int32_t last_layer;
  int32_t E;                /* number of entries written to expert_count */
  const int32_t *expert_count; /* host array [E]: tokens per expert, last call;
                                  owned by the context, valid until the next
                                  moe_get_stats or moe_destroy */
} moe_stats;

/* moe_create: a context for a layer of hidden size d, SwiGLU width f,
 * E experts, top-k routing and the given quant format.  Defaults: 1 layer,
 * no shared expert, no slot pool, up to 64 tokens per call; change them with
 * moe_configure before the first load.
 * Errors: INVALID_ARG if d or f is not a multiple of 128, E < 1 or E > 1024,
 * k < 1, k > E or k > 32, or quant_fmt unknown; CUDA if no device. */
MOE_API moe_status moe_create(int d, int f, int E, int k, int quant_fmt, moe_ctx **out);

/* moe_configure: model size and call limits; allocates all device memory
 * (weights arena for n_layers * E experts, n_shared shared experts per layer
 * (0 or 1), a slot pool of n_slots experts, scratch for max_tokens tokens per
 * call).  Must come before any load; may be called once.
 * Errors: INVALID_ARG on n_layers < 1, n_shared not 0/1, n_slots < 0,
 * max_tokens < 1; STATE if weights were already loaded; OOM. */
MOE_API moe_status moe_configure(moe_ctx *ctx, int n_layers, int n_shared, int n_slots,
                         int max_tokens);

/* moe_destroy: frees everything the context owns (synchronises the device
 * first).  NULL is accepted and ignored. */
MOE_API moe_status moe_destroy(moe_ctx *ctx);

/* moe_load_experts: copy n_experts packed experts (format above) into
 * (the backing copy of every (layer, expert) that the residency table of the
 * engine article "93 token/s on one 8 GB card", section "Expert cache",
 * points at when an expert is not in a slot)
 * experts [first_expert, first_expert + n_experts) of `layer`, repacking them
 * into the library's device layout.  Also refreshes any slot-pool copies of
 * those experts.  Synchronous.  Errors: INVALID_ARG on a bad range or NULL
 * codes/scales (or NULL mins for Q2); OOM; CUDA. */
MOE_API moe_status moe_load_experts(moe_ctx *ctx, int layer, int first_expert,
                            int n_experts, const void *codes,
                            const void *scales, const void *mins,
                            int src_is_device);

/* moe_load_shared: the shared expert of `layer` (same format, one expert).
 * Errors: STATE if configured with n_shared = 0; else as moe_load_experts. */
MOE_API moe_status moe_load_shared(moe_ctx *ctx, int layer, const void *codes,
                           const void *scales, const void *mins,
                           int src_is_device);

/* moe_set_router: router weight W fp32 [E, d] and optional bias fp32 [E]
 * (NULL = no bias) of `layer`.  Synchronous copy.  In a context configured
 * with max_tokens > 32 it also stores W as three bf16 parts whose sum is W
 * exactly (L * E * 3d * 2 bytes for the context), from which chunks of 512
 * or more tokens compute the logits on the tensor cores at fp32 accuracy. */
MOE_API moe_status moe_set_router(moe_ctx *ctx, int layer, const float *W,
                          const float *bias, int src_is_device);

/* moe_set_norm: RMSNorm before the router for `layer`: h = x * (mean(x^2) +
 * eps)^-1/2 * gamma.  gamma is a HOST fp32 [d] array or NULL for gamma = 1.
 * Without this call a layer uses h = x (no norm). */
MOE_API moe_status moe_set_norm(moe_ctx *ctx, int layer, const float *gamma, float eps);

/* moe_set_slots: the residency table of the engine article "93 token/s on
 * one 8 GB card", section "Expert cache": (layer, expert) -> slot or -1.
 * HOST int32 [n_layers * E]: slot id of
 * (layer, expert) in the slot pool, or -1 when it is served from the backing
 * arena (every expert always has a backing copy, so results do not depend on
 * the table).  Copies the experts into their slots (synchronous).
 * Errors: INVALID_ARG on a slot >= n_slots or a slot used twice. */
MOE_API moe_status moe_set_slots(moe_ctx *ctx, const int32_t *slot_of);

/* moe_route: router logits + top-k + softmax + bucketing for T tokens of
 * `layer` (the engine article "93 token/s on one 8 GB card", section
 * "Architecture overview": the router picks 10 of 512 experts per token;
 * the "Doorbell handshake" section ends the "pre" half of a block with the
 * router's ids and weights).  Windows of more than 32 tokens select the
 * top-k one warp per token; in a context configured for chunks
 * (max_tokens > 32) whose shapes the grouped GEMM takes, they route exactly
 * as moe_prefill_route (logits on the tensor cores when E is a multiple of
 * 256, see moe_set_router; the sort by expert over many CTAs).  h_dev: bf16 [T, d] router input.  idx_dev int32 [T, k] and
 * w_dev fp32 [T, k] receive each token's experts and renormalised weights,
 * ordered by descending logit (equal logits: lower expert id first).
 * bucket_off_dev int32 [E+1] (exclusive prefix of tokens per expert) and
 * bucket_perm_dev int32 [T*k] (pair ids t*k+j grouped by expert, ascending t
 * inside an expert) may be NULL.  Errors: INVALID_ARG if T < 1 or T >
 * max_tokens or a required pointer is NULL. */
MOE_API moe_status moe_route(moe_ctx *ctx, int layer, const void *h_dev, int T,
                     int32_t *idx_dev, float *w_dev, int32_t *bucket_off_dev,
                     int32_t *bucket_perm_dev, void *stream);

/* moe_bucket: bucketing alone, for caller-provided routing idx_dev int32
 * [T, k] (distinct expert ids per token).  Outputs as in moe_route.  An id
 * outside [0, E) sets the device error status (moe_sync returns DEVICE). */
MOE_API moe_status moe_bucket(moe_ctx *ctx, const int32_t *idx_dev, int T,
                      int32_t *bucket_off_dev, int32_t *bucket_perm_dev,
                      void *stream);

/* moe_forward: one decode window of T tokens through `layer`, in place
 * (the engine article "93 token/s on one 8 GB card", section "Architecture
 * overview": route, compute each selected expert from wherever it resides,
 * combine into the residual):
 * x <- x + MoE(norm(x)).  x_dev: bf16 [T, d].  Runs router, top-k, residency
 * lookup, bucketing, the grouped dequant-SwiGLU experts (+ shared expert)
 * and the combine + residual kernel.  Errors: INVALID_ARG, STATE (router or
 * experts not loaded). */
MOE_API moe_status moe_forward(moe_ctx *ctx, int layer, void *x_dev, int T,
                       void *stream);

/* moe_forward_delta: as moe_forward but leaves x unchanged and writes the
 * fp32 MoE output delta_dev [T, d] (the value added to the residual). */
MOE_API moe_status moe_forward_delta(moe_ctx *ctx, int layer, const void *x_dev, int T,
                             float *delta_dev, void *stream);

/* moe_forward_stack: moe_forward through layers 0..n_layers-1 in order.  The
 * first call for a given (x_dev, T) records the whole stack as one CUDA
 * graph; later calls replay it.  Do not call it while `stream` is being
 * captured by the caller. */
MOE_API moe_status moe_forward_stack(moe_ctx *ctx, void *x_dev, int T, void *stream);

/* moe_prefill: a prefill chunk of N tokens (N <= max_tokens) through
 * `layer`, in place (x <- x + MoE(norm(x))).  The engine article "93 token/s
 * on one 8 GB card", section "Architecture overview", runs prefill in chunks
 * of up to 8192 tokens; per expert such a chunk is a dense contraction.  For
 * N > 32 the experts (Q4 or Q2) run as a grouped GEMM on the tensor cores
 * (tcgen05): tokens sorted by expert, 256-token tiles, weights dequantised
 * to fp16 tile by tile in shared memory (Q4: s (c - 8); Q2: s q + m, one
 * fp16 rounding), fp32 accumulation in tensor memory.  Activations enter as
 * fp16 (exact for |h| < 65504; larger values saturate), and the experts'
 * outputs y are kept in fp16 until the combine.  Router logits: fp32
 * accuracy, on the tensor cores when E is a multiple of 256 (see
 * moe_set_router), else fp32 FMA.  N <= 32 takes the moe_forward path.
 * Requires a context configured with max_tokens >= N.  Errors: INVALID_ARG,
 * STATE; device faults through moe_sync. */
MOE_API moe_status moe_prefill(moe_ctx *ctx, int layer, void *x_dev, int N,
                       void *stream);

/* moe_prefill_delta: as moe_prefill but leaves x unchanged and writes the
 * fp32 MoE output delta_dev [N, d]. */
MOE_API moe_status moe_prefill_delta(moe_ctx *ctx, int layer, const void *x_dev, int N,
                                     float *delta_dev, void *stream);

/* moe_prefill_route: the routing half of moe_prefill alone, on router
 * input h_dev bf16 [N, d] (no RMSNorm here, as in moe_route): the chunk's
 * router logits (tensor cores when E is a multiple of 256, else fp32
 * FMA), top-k + softmax one warp per token, and the sort of the
 * chunk's pairs by expert that feeds the grouped GEMM (the engine article
 * "93 token/s on one 8 GB card", section "Architecture overview": prefill in
 * chunks of up to 8192 tokens).  It launches exactly the kernels moe_prefill
 * launches before its GEMMs.  Outputs as in moe_route: idx_dev int32
 * [N, k], w_dev fp32 [N, k], bucket_off_dev int32 [E+1] (may be NULL),
 * bucket_perm_dev int32 [N*k] (pair ids grouped by expert, ascending t
 * inside an expert; may be NULL).  Errors: INVALID_ARG (N < 1, N >
 * max_tokens, NULL idx/w, h not 16-byte aligned), STATE (router not set),
 * NOT_SUPPORTED in a context configured with max_tokens <= 32. */
MOE_API moe_status moe_prefill_route(moe_ctx *ctx, int layer, const void *h_dev, int N,
                                     int32_t *idx_dev, float *w_dev, int32_t *bucket_off_dev,
                                     int32_t *bucket_perm_dev, void *stream);

/* moe_rmsnorm: the router input of `layer` for T tokens, h = RMSNorm(x)
 * as moe_forward and moe_prefill compute it (h = bf16(x (mean(x^2) +
 * eps)^-1/2 gamma), fp32 inside), or a copy of x when the layer has no
 * norm.  x_dev, h_dev: bf16 [T, d], 16-byte aligned, caller-owned; T >= 1
 * (no scratch is used).  Errors: INVALID_ARG, STATE (not configured). */
MOE_API moe_status moe_rmsnorm(moe_ctx *ctx, int layer, const void *x_dev, int T, void *h_dev,
                               void *stream);

/* moe_experts_given: the experts of `layer` on caller-given routing, with
 * the chunk path's kernels (bucketing by expert, grouped tcgen05 GEMM for
 * experts with at least 24 rows, GEMV for the others, combine): the
 * "experts by residency, then combine" half of the engine article's
 * per-layer flow ("93 token/s on one 8 GB card", section "Architecture
 * overview") without its router.  It is what an expert-parallel owner runs
 * on the rows it receives.
 *   h_dev    bf16 [N, d] router input rows (already normalised; no RMSNorm here)
 *   idx_dev  int32 [N, kk] expert ids, distinct within a row, each expert loaded
 *   w_dev    fp32 [N, kk] weights
 *   kk       0..k experts per row (0: shared expert only)
 *   with_shared  1: add the shared expert's output (the context must have one)
 *   delta_dev fp32 [N, d] receives sum_j w[t,j] y_j(h_t) (+ y_shared(h_t)),
 *            j in order, with the arithmetic of moe_prefill_delta.
 * Every buffer is caller-owned device memory, 16-byte aligned where it
 * holds rows.  N <= max_tokens.  The ids are copied to the host and checked
 * before any launch (the call synchronizes `stream` once).  Errors:
 * INVALID_ARG (bad sizes or pointers, an id outside [0, E), a repeated id
 * in a row), STATE (an expert or the shared expert not loaded),
 * NOT_SUPPORTED (context configured with max_tokens <= 32, or shapes the
 * grouped GEMM does not take: d a multiple of 256, f of 128, E <= 1024). */
MOE_API moe_status moe_experts_given(moe_ctx *ctx, int layer, const void *h_dev, int N, int kk,
                                     const int32_t *idx_dev, const float *w_dev, int with_shared,
                                     float *delta_dev, void *stream);

/* moe_experts_rows: the owner's step of an expert-parallel layer.  Row t
 * of h_dev (bf16 [M, d], router input) goes through the one expert
 * e_dev[t] (int32 [M], loaded, in [0, E)) with weight 1 and no shared
 * expert, with the chunk path's kernels (as moe_experts_given with kk = 1);
 * y_dev (fp16 [M, d], caller-owned, 16-byte aligned) receives each row's
 * output y in row order, in the fp16 the chunk path keeps expert outputs in
 * before its combine.  M <= max_tokens.  The ids are checked on the host
 * first (one stream synchronisation).  Errors as moe_experts_given. */
MOE_API moe_status moe_experts_rows(moe_ctx *ctx, int layer, const void *h_dev, int M,
                                    const int32_t *e_dev, void *y_dev, void *stream);

/* Expert parallelism over n_ranks ranks: expert e belongs to rank
 * e / (E / n_ranks) (E a multiple of n_ranks, n_ranks <= 64).
 *
 * moe_ep_dispatch: the send side of the exchange for N tokens routed by
 * idx_dev int32 [N, k] (this context's k and E): every pair q = t k + j is
 * sent to its expert's owner.  Writes, in device memory the caller owns:
 *   send_h_dev  bf16 [N k, d]: the router-input row h_dev[t] of each sent
 *               pair, grouped by destination rank (rank 0 first), ascending
 *               pair id inside a rank's segment;
 *   send_e_dev  int32 [N k]: the pair's expert id at the same position;
 *   row_of_dev  int32 [N k]: the send position of pair q (-1: id outside
 *               [0, E), not sent; the device status is set and moe_sync
 *               reports DEVICE);
 * and counts_host int32 [n_ranks] (host memory): rows for each rank, the
 * all-to-all's send split.  h_dev bf16 [N, d].  Synchronizes `stream`
 * (the counts are read back).  Errors: INVALID_ARG, STATE. */
MOE_API moe_status moe_ep_dispatch(moe_ctx *ctx, const int32_t *idx_dev, int N, int n_ranks,
                                   const void *h_dev, void *send_h_dev, int32_t *send_e_dev,
                                   int32_t *row_of_dev, int32_t *counts_host, void *stream);

/* moe_ep_combine: the receive side.  y_dev fp16 [rows, d]: the expert
 * outputs returned by the owners (moe_experts_rows), in send order (row_of_dev from
 * moe_ep_dispatch maps pair q to its row); w_dev fp32 [N, k];
 * y_shared_dev fp32 [N, d] (the shared expert's output, e.g. from
 * moe_experts_given with kk = 0) or NULL.  Exactly one of x_dev (bf16
 * [N, d], updated in place: x <- bf16(x + acc)) and delta_dev (fp32 [N, d]
 * <- acc) is non-NULL; acc = sum_j w[t,j] y[row_of(t,j)] + y_shared[t],
 * j in order, the one-GPU combine's arithmetic, so an expert-parallel layer
 * matches moe_prefill bit for bit.  row_of_dev must be the one
 * moe_ep_dispatch wrote for the same routing (its entries are rows of y_dev
 * or -1; they are not checked again).  Errors: INVALID_ARG. */
MOE_API moe_status moe_ep_combine(moe_ctx *ctx, int N, const float *w_dev, const void *y_dev,
                                  const int32_t *row_of_dev, const float *y_shared_dev, void *x_dev,
                                  float *delta_dev, void *stream);

/* moe_sync: wait (polling cudaEventQuery, at most timeout_ms; < 0 = no
 * limit) until the work queued by this context has finished, then read and
 * clear the device error status.  Returns TIMEOUT, BAD_SLOT, DEVICE, CUDA or
 * OK. */
MOE_API moe_status moe_sync(moe_ctx *ctx, int timeout_ms);

/* moe_get_stats: synchronises and fills *out (see moe_stats). */
MOE_API moe_status moe_get_stats(moe_ctx *ctx, moe_stats *out);

/* moe_route_static: the routing step of moe_route (router logits, top-k
 * with renormalised softmax, bucketing) with NO allocation and no context,
 * for callers that cannot call cudaMalloc (for example code that runs under
 * a fixed device-memory budget handed to its own pool, or a plugin that is
 * only given raw device pointers).  The pages this library follows have no
 * counterpart of this call; it is a deployment convenience.
 *  h_dev     bf16 [T, d] router input (16-byte aligned)
 *  W_dev     fp32 [E, d] router weights (16-byte aligned); bias_dev fp32 [E]
 *            or NULL
 *  idx_dev, w_dev, bucket_off_dev, bucket_perm_dev: outputs exactly as in
 *            moe_route (none may be NULL).
 * Limits: 1 <= T <= 32, d a multiple of 128 and <= 2048, 1 <= E <= 1024,
 * 1 <= k <= min(E, 32); anything else returns MOE_ERR_INVALID_ARG before any
 * GPU work.  Scratch (logits, a completion ticket, a status word) lives in a
 * static device array of about 129 KB that every GPU loading this library
 * holds until the process exits.  The first call on a device, with that
 * device current, looks up the array's device address and sets the routing
 * kernels' shared-memory limit; make that first call before any stream
 * capture.  Each call clears the array's counters on `stream` before use;
 * calls whose execution overlaps on the GPU (other streams, other threads)
 * race on the array.  Returns MOE_OK, MOE_ERR_INVALID_ARG or MOE_ERR_CUDA at
 * launch; an out-of-range routing id cannot occur (ids come from the
 * top-k).  If a bounded wait inside the kernel gives up (the window's copy
 * into shared memory never completed), the call routes nothing: idx, w and
 * the buckets keep their previous contents, and moe_route_static_status
 * reports it. */
MOE_API moe_status moe_route_static(const void *h_dev, int T, int d, int E, int k,
                                    const float *W_dev, const float *bias_dev,
                                    int32_t *idx_dev, float *w_dev,
                                    int32_t *bucket_off_dev, int32_t *bucket_perm_dev,
                                    void *stream);

/* moe_route_static_status: synchronises `stream`, then stores in
 * *status_out the device status word of the most recent moe_route_static
 * call on the current device (0, or the OR of its fault bits: 8 = a bounded
 * wait gave up and nothing was routed).  Returns MOE_OK for 0, MOE_ERR_DEVICE
 * for a non-zero word, MOE_ERR_CUDA or MOE_ERR_INVALID_ARG (NULL).  The
 * word is cleared by the next moe_route_static call. */
MOE_API moe_status moe_route_static_status(int *status_out, void *stream);

/* Host tier (the engine article "93 token/s on one 8 GB card", section
 * "Expert cache": a model larger than the GPU keeps its hot experts in a
 * fixed set of device slots, (layer, expert) -> slot or -1, and brings
 * misses in while other work runs; the user report "EPYC 7B13 + 2x RTX 3090"
 * makes that cache adaptive).  With the host tier, every expert's backing
 * copy lives in pinned, mapped host memory, and the n_slots slots of
 * moe_configure form an HBM cache over it.  The shared experts, routers and
 * scratch stay in HBM.  Results are those of the all-HBM context bit for bit:
 * residency only moves where an expert is read from.
 *
 * moe_set_host_tier: before moe_configure.  enable 0/1; policy 0 = least
 * recently used, 1 = adaptive (an exponentially decayed use count with the
 * given half-life in requests, ties by recency).  Errors: INVALID_ARG,
 * STATE (already configured). */
MOE_API moe_status moe_set_host_tier(moe_ctx *ctx, int enable, int policy, double half_life);

/* moe_tier_prepare: make the experts a window selects resident.  idx_dev is
 * the window's routing, int32 [T, k] on the device (e.g. from moe_route),
 * written by work already queued on `stream`: the call waits for the stream,
 * reads the ids back, gives each selected expert without a slot a slot (by
 * the policy; never one the window itself uses), copies the missed experts
 * host -> HBM on the context's copy stream with the changed slot-table rows
 * after them, and makes `stream` wait for those copies.  A later forward of
 * this window on `stream` then reads only HBM.  Errors: INVALID_ARG (bad
 * arguments, or more distinct experts than slots), STATE (no host tier),
 * DEVICE (an id outside [0, E)), CUDA. */
MOE_API moe_status moe_tier_prepare(moe_ctx *ctx, int layer, const int32_t *idx_dev, int T,
                                    void *stream);

/* moe_tier_prefetch: as moe_tier_prepare, but the copies stay in flight
 * (no stream waits for them; the next prepare or prefetch is ordered after
 * them), so they overlap whatever runs meanwhile -- the pages stream the
 * next layer's misses during the current layer's work.  The previous
 * request's slots are not evicted either, since its window may still be
 * running; other work in flight must only use experts of that request. */
MOE_API moe_status moe_tier_prefetch(moe_ctx *ctx, int layer, const int32_t *idx_dev, int T,
                                     void *stream);

/* moe_forward_tiered: moe_forward with the miss path in front: the window's
 * routing (with the layer's RMSNorm, as the forward computes it),
 * moe_tier_prepare on it, then the forward.  Same arguments, results and
 * errors as moe_forward, plus those of moe_tier_prepare. */
MOE_API moe_status moe_forward_tiered(moe_ctx *ctx, int layer, void *x_dev, int T, void *stream);

/* moe_tier_stats: out[0] hits, out[1] misses, out[2] evictions (distinct
 * experts per request), out[3] bytes copied host -> HBM, out[4] requests,
 * out[5] slots in use.  Errors: INVALID_ARG, STATE (no host tier). */
MOE_API moe_status moe_tier_stats(moe_ctx *ctx, long long *out);

/* moe_tier_dump_trace: write the routing trace of every request so far to a
 * text file, one line per request: "request layer n expert...".  Errors:
 * INVALID_ARG (cannot open or write), STATE (no host tier). */
MOE_API moe_status moe_tier_dump_trace(moe_ctx *ctx, const char *path);

/* Host-only model of the tier's replacement policy (no device involved), for
 * policy studies and tests: a cache of n_slots slots over keys [0, n_keys).
 * moe_tier_sim_request takes one request of n distinct keys, writes each
 * key's slot into slots_out[n] (may be NULL) and returns the request's misses,
 * -1 for bad arguments, -2 when the misses outnumber the slots that may be
 * taken.  moe_tier_sim_counts writes hits, misses, evictions. */
MOE_API void *moe_tier_sim_create(int n_slots, int policy, double half_life, long long n_keys);
MOE_API int moe_tier_sim_request(void *sim, const long long *keys, int n, int protect_prev,
                                 int *slots_out);
MOE_API void moe_tier_sim_counts(void *sim, long long *out);
MOE_API void moe_tier_sim_destroy(void *sim);

/* Profiling: when enabled, every forward call records CUDA events on its
 * stream around its three segments -- routing (norm + router + top-k +
 * bucketing), experts (the two grouped dequant-GEMV kernels) and combine --
 * into a pool of 8192 call slots.  The events sit between the kernels, so a
 * profiled call loses the launch overlap at those three points.  Events are
 * recorded as external graph nodes, so profiled calls may be captured. */
MOE_API moe_status moe_set_profiling(moe_ctx *ctx, int enable);

/* Synchronises, then adds the elapsed milliseconds of the profiled calls
 * made since profiling was last enabled (at most the 8192 most recent) to
 * ms[0] (routing), ms[1] (experts), ms[2] (combine) and returns their number
 * in *n_calls.  Reading does not consume the slots: after a replay of a
 * captured graph, a new read gives that replay's times.  moe_set_profiling
 * (ctx, 1) starts a new set.  ms is caller-owned host memory. */
MOE_API moe_status moe_read_profile(moe_ctx *ctx, double ms[3], int64_t *n_calls);

/* Device timeline tracing (diagnostics).  When enabled, kernels record the
 * earliest and latest %globaltimer (ns) at which any CTA reached each of a
 * fixed list of trace points (kernel start, dependency wait passed, phase
 * ends, kernel end of the routing, expert and combine kernels).  The trace
 * buffer is shared by every context of the process on this device; enabling
 * it synchronises the device.  Costs a few atomics per CTA while on. */
MOE_API moe_status moe_set_trace(moe_ctx *ctx, int enable);

/* Synchronises, copies the 2 * n_points trace values (first all minima, then
 * all maxima; unset minima read as -1, unset maxima as 0) into out[0 .. n)
 * and resets them.  n must be at least 2 * 18. */
MOE_API moe_status moe_read_trace(moe_ctx *ctx, int64_t *out, int n);

/* Last error message of ctx (never NULL; "" when none). */
MOE_API const char *moe_last_error(const moe_ctx *ctx);

/* Static name of a status code. */
MOE_API const char *moe_status_string(int status);

/* Debug hook for fault-injection tests: writes one raw entry of the device
 * residency table WITHOUT the host validation of moe_set_slots.  A slot id
 * outside the pool is then caught by the routing kernel, which falls back to
 * the backing copy and sets the device status that moe_sync reports as
 * MOE_ERR_BAD_SLOT.  Not for production use. */
MOE_API moe_status moe_debug_poke_slot(moe_ctx *ctx, int layer, int expert, int32_t slot);

/* Test hook for the device's bounded waits: the next single-launch decode
 * (moe_forward or moe_forward_delta of a window of <= 32 tokens) runs with
 * a first grid barrier that cannot complete and a poll limit of `polls`
 * (about a microsecond each), so that wait runs out.  The kernel then sets
 * the device status (a bounded wait gave up), skips the layer and leaves;
 * moe_sync returns MOE_ERR_DEVICE and resets the barrier counters, and the
 * next call runs normally.  No fault, trap or hang is involved.  Errors:
 * INVALID_ARG (NULL ctx, polls < 1). */
MOE_API moe_status moe_debug_stall_next_decode(moe_ctx *ctx, uint32_t polls);

/* Debug hook: copies on `stream` the normalised router input h (bf16
 * [T, d], h = RMSNorm(x) as the kernels computed it) of the most recent
 * moe_forward / moe_forward_delta / moe_prefill call on a layer with
 * RMSNorm into out_dev.  Lets tests compare the device's RMSNorm with a
 * reference.  Errors: INVALID_ARG (NULL, T out of range). */
MOE_API moe_status moe_debug_last_h(moe_ctx *ctx, void *out_dev, int T, void *stream);

/* Bytes one packed expert occupies in the given format (codes + scales +
 * mins), or -1 for bad arguments. */
MOE_API int64_t moe_expert_bytes(int d, int f, int quant_fmt);

#ifdef __cplusplus
}
#endif
#endif
