// common.cuh -- device helpers shared by the libmoe kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#define MOE_DEV __device__ __forceinline__
#define MOE_HOST_DEV_INLINE __host__ __device__ __forceinline__

namespace moe {

// ---------------------------------------------------------------- status bits
// Device-detected faults; OR-ed into the context's status word and reported
// (then cleared) by moe_sync.  No kernel traps.
enum : int {
  kErrBadExpert = 1 << 0,  // expert id outside [0, E)
  kErrBadSlot = 1 << 1,    // residency slot outside the slot pool
  kErrJobOverflow = 1 << 2,
  kErrTimeout = 1 << 3,    // a bounded wait gave up
};

// ------------------------------------------------------------ format layout
// Device layout of one expert after moe_load_experts repacks it.
//
// An expert is stored as two regions.  Region 1 (gate+up) holds, for every
// block of 16 rows of Wg/Wu, the K = d reduction split into tiles of TK
// columns; each tile is a Wg tile followed by the Wu tile of the same rows
// and columns.  Region 2 holds the Wd tiles (16 rows of d, K = f).  A tile is
// 512 bytes of codes (16 bytes per lane of a warp, already in the order the
// tensor-core fragments want) followed by the scales (and mins) of its 16
// rows: 64 B for Q4 (TK = 64, two groups of 32), 128 B for Q2 (TK = 128, two
// groups of 64).  So one warp streams each tile with one contiguous copy.
struct Layout {
  int fmt, d, f;
  int G;          // quantisation group
  int TK;         // reduction columns per tile
  int tile_bytes; // codes + scale block of one 16-row tile of one matrix
  long long p1_bytes, p2_bytes, expert_bytes;
};

inline Layout make_layout(int fmt, int d, int f) {
  Layout L;
  L.fmt = fmt;
  L.d = d;
  L.f = f;
  L.G = fmt == 1 ? 32 : 64;
  L.TK = fmt == 1 ? 64 : 128;
  L.tile_bytes = fmt == 1 ? 512 + 64 : 512 + 128;
  L.p1_bytes = (long long)(f / 16) * (d / L.TK) * 2 * L.tile_bytes;
  L.p2_bytes = (long long)(d / 16) * (f / L.TK) * L.tile_bytes;
  L.expert_bytes = L.p1_bytes + L.p2_bytes;
  return L;
}

// ----------------------------------------------------------------- tracing
// Device timeline of one forward call (moe_set_trace): each trace point
// keeps the earliest and latest %globaltimer (ns) any CTA recorded there.
// Null when tracing is off; then a trace point costs one load and a branch.
enum TracePoint : int {
  kTrRouteStart = 0, kTrRouteWaited, kTrRouteLogits, kTrRouteLastStart, kTrRouteTopk,
  kTrRouteBucket, kTrRouteEnd,
  kTrGateStart, kTrGateWaited, kTrGateFirstTile, kTrGateEnd,
  kTrDownStart, kTrDownWaited, kTrDownEnd,
  kTrCombStart, kTrCombEnd,
  kTrRouteLoaded, kTrRouteSelected,
  kTrCount
};
// [2 * kTrCount]: minima then maxima; the library is one translation unit
__device__ unsigned long long *g_trace = nullptr;

MOE_DEV unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
MOE_DEV void trace_point(int i) {
  unsigned long long *tr = g_trace;
  if (tr) {
    const unsigned long long t = global_ns();
    atomicMin(tr + i, t);
    atomicMax(tr + kTrCount + i, t);
  }
}
#define MOE_TRACE(i)                       \
  do {                                     \
    if (threadIdx.x == 0) trace_point(i);  \
  } while (0)

// ------------------------------------------------------- PDL (griddepcontrol)
MOE_DEV void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
MOE_DEV void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// --------------------------------------------------------------- raw loads
MOE_DEV uint2 ldcg_u2(const void *p) {
  uint2 r;
  asm volatile("ld.global.cg.v2.u32 {%0,%1}, [%2];" : "=r"(r.x), "=r"(r.y) : "l"(p));
  return r;
}
MOE_DEV uint4 ldcg_u4(const void *p) {
  uint4 r;
  asm volatile("ld.global.cg.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}
MOE_DEV float4 ldcg_f4(const void *p) {
  float4 r;
  asm volatile("ld.global.cg.v4.f32 {%0,%1,%2,%3}, [%4];"
               : "=f"(r.x), "=f"(r.y), "=f"(r.z), "=f"(r.w)
               : "l"(p));
  return r;
}
MOE_DEV int ldcg_i32(const int *p) { return __ldcg(p); }
MOE_DEV unsigned long long ldcg_u64(const unsigned long long *p) { return __ldcg(p); }

MOE_DEV uint4 lds_u4(uint32_t a) {
  uint4 r;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "r"(a));
  return r;
}
MOE_DEV uint2 lds_u2(uint32_t a) {
  uint2 r;
  asm volatile("ld.shared.v2.u32 {%0,%1}, [%2];" : "=r"(r.x), "=r"(r.y) : "r"(a));
  return r;
}

MOE_DEV uint32_t smem_addr(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ------------------------------------------------ mbarrier + bulk (TMA) copy
MOE_DEV void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
MOE_DEV void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
MOE_DEV void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
MOE_DEV void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}
// expect_tx + 1-D bulk copy with an L2 cache policy (l2_evict_first), issued
// by the calling lane only when `issue`; every lane may execute it
// (predicated, no branch).
MOE_DEV void bulk_g2s_hint_pred(bool issue, uint32_t dst, const void *src, uint32_t bytes, uint32_t bar,
                                uint64_t policy) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.u32 p, %5, 0;\n\t"
      "@p mbarrier.arrive.expect_tx.shared::cta.b64 _, [%3], %2;\n\t"
      "@p cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;\n\t}" ::"r"(
          dst),
      "l"(src), "r"(bytes), "r"(bar), "l"(policy), "r"((uint32_t)issue)
      : "memory");
}
// One arrival (this thread) on an mbarrier.
MOE_DEV void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
// 1-D bulk copy global -> this CTA's shared memory, completing on `bar`.
// dst/src 16-byte aligned, bytes a multiple of 16.
MOE_DEV void bulk_g2s(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}

// Policy for data read once: its L2 lines are the first to be evicted, so a
// stream of them does not push other data (or code) out of L2.
MOE_DEV uint64_t l2_evict_first() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}
MOE_DEV bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait: returns false (and the caller reports kErrTimeout) if the
// phase never completes within the iteration limit.
MOE_DEV bool mbar_wait_bounded(uint32_t bar, uint32_t parity) {
  for (uint32_t i = 0; i < (1u << 24); ++i)
    if (mbar_try_wait(bar, parity)) return true;
  return false;
}

// ----------------------------------------------------------- tensor-core mma
// D = A(16x16, row) * B(16x8, col) + C, bf16 inputs, fp32 accumulate.
MOE_DEV void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1,
                            const float (&c)[4]) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%10,%11,%12,%13};"
      : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "f"(c[0]), "f"(c[1]),
        "f"(c[2]), "f"(c[3]));
}

// D = A * B (zero accumulator) when `first`, else D += A * B.
MOE_DEV void mma_bf16_acc(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1,
                          bool first) {
  if (first) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%10,%10,%10,%10};"
        : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "f"(0.f));
  } else {
    mma_bf16_16816(d, a, b0, b1, d);
  }
}

// ------------------------------------------------------------- code unpack
MOE_DEV uint32_t lop3_and_or(uint32_t x, uint32_t m, uint32_t c) {
  uint32_t r;  // (x & m) | c
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(r) : "r"(x), "r"(m), "r"(c));
  return r;
}
MOE_DEV uint32_t bf16x2_fma(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t r;
  asm("fma.rn.bf16x2 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(c));
  return r;
}

// Q2: one word holds the 16 codes of two mma steps; fragment register r
// (r = 0..7; step = r / 4) takes its low code from bits [2r, 2r+2) and its
// high code from bits [16+2r, 18+2r).  The code lands at mantissa bit p of
// bf16 128.0 (p = 0, 2 or 4 after a shift of 0, 6 or 12) giving 128 + q*2^p;
// an exact bf16x2 FMA (x * 2^-p - 128 * 2^-p) recovers q in {0,1,2,3}.
MOE_DEV void unpack_q2(uint32_t w, uint32_t (&a)[8]) {
  const uint32_t C = 0x43004300u;
  const uint32_t s0 = 0x3F803F80u, o0 = 0xC300C300u;  // 1, -128
  const uint32_t s2 = 0x3E803E80u, o2 = 0xC200C200u;  // 1/4, -32
  const uint32_t s4 = 0x3D803D80u, o4 = 0xC100C100u;  // 1/16, -8
  const uint32_t w6 = w >> 6, w12 = w >> 12;
  a[0] = bf16x2_fma(lop3_and_or(w, 0x00030003u, C), s0, o0);
  a[1] = bf16x2_fma(lop3_and_or(w, 0x000C000Cu, C), s2, o2);
  a[2] = bf16x2_fma(lop3_and_or(w, 0x00300030u, C), s4, o4);
  a[3] = bf16x2_fma(lop3_and_or(w6, 0x00030003u, C), s0, o0);
  a[4] = bf16x2_fma(lop3_and_or(w6, 0x000C000Cu, C), s2, o2);
  a[5] = bf16x2_fma(lop3_and_or(w6, 0x00300030u, C), s4, o4);
  a[6] = bf16x2_fma(lop3_and_or(w12, 0x00030003u, C), s0, o0);
  a[7] = bf16x2_fma(lop3_and_or(w12, 0x000C000Cu, C), s2, o2);
}

MOE_DEV float half_lo(uint32_t v) { return __half2float(__ushort_as_half((unsigned short)(v & 0xFFFF))); }
MOE_DEV float half_hi(uint32_t v) { return __half2float(__ushort_as_half((unsigned short)(v >> 16))); }

MOE_DEV float bf16_bits_to_float(unsigned short b) { return __uint_as_float((uint32_t)b << 16); }

// Order-preserving map of a float to an unsigned key (-0 and +0 equal):
// a > b  <=>  order_key(a) > order_key(b) for non-NaN a, b.  0 is below every
// real value's key, so it marks a used or absent entry.
MOE_DEV uint32_t order_key(float f) {
  if (f == 0.f) f = 0.f;
  const uint32_t b = __float_as_uint(f);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
MOE_DEV float key_to_float(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

MOE_DEV float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

}  // namespace moe
