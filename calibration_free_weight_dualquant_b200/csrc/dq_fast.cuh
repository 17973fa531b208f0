// dq_fast.cuh -- fp32 fast paths of the per-iteration pass and the TMA
// (bulk-copy) pipeline primitives.
//
// Every fast path here either returns the exact answer of the definitions in
// dq_device.cuh or raises a flag, and the caller then takes the exact path:
//  * grid decisions: the fp32 candidate x~ for W/(a b) carries a relative error
//    below 7 * 2^-24; an element whose x~ lies within kGuard of a rounding
//    boundary is flagged;
//  * block inverse-scale updates: num and den are fp32 sums of at most 8 + 5
//    roundings each, so num/den is known to a relative 2^-19 (kAmbUlps units of
//    the fp32 significand); a value that close to a projection midpoint, or
//    outside the target format's normal range, is flagged.
#pragma once

#include "dq_device.cuh"
#include "dq_internal.h"

namespace dq {

// Static schedule of the persistent passes: CTA k owns the strip-major row
// units [k L / P, (k+1) L / P); cta_of(u) is the CTA owning unit u.
__device__ __forceinline__ int64_t cta_of(int64_t u, int64_t P, int64_t L) { return ((u + 1) * P - 1) / L; }
__device__ __forceinline__ int64_t range_begin(int64_t k, int64_t P, int64_t L) { return k * L / P; }

// Fast-path scale factors are trusted when they stay inside [2^-50, 2^50]:
// then every product that lands near a rounding boundary, and every a*b the
// exact fp32 decision forms, is a normal fp32 number, so the relative error
// bound behind kGuard holds and the exact sign tests below cannot underflow.
__device__ __forceinline__ bool in_range(float x) { return x >= 0x1p-50f && x <= 0x1p50f; }

// ---------------------------------------------------------------------------
// Approximate reciprocal (max error 1 ulp), used for fast-path factors only.
__device__ __forceinline__ float rcp_approx(float x) {
  float r;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}

// Exact integer-grid decision in fp32 for an element the fast path flagged.
// ab = a*b is exact in fp32 (fp16*fp16, fp16*bf16 or 2^k*bf16), h*ab too (h
// has at most 9 significant bits on the INT8 grid), and w - h*a*b is formed
// inside one fma, so its sign says on which side of the boundary h nearest the
// candidate W/(a b) lies; zero is a tie (to even).
template <int FMT>
static __device__ __noinline__ float qexact32_int(float w, float u, float ia, float ab) {
  const float xt = u * ia;
  const float qu = __fsub_rn(__fadd_rn(xt, 12582912.f), 12582912.f);
  const float h = qu + copysignf(0.5f, xt - qu);
  const float d = fmaf(-h, ab, w);
  float q;
  if (d > 0.f) {
    q = h + 0.5f;
  } else if (d < 0.f) {
    q = h - 0.5f;
  } else {
    q = __fsub_rn(__fadd_rn(h, 12582912.f), 12582912.f);  // the even neighbour
  }
  return fminf(fmaxf(q, grid_lo(FMT)), grid_hi(FMT));
}

// Exact E2M1 decision in fp32: a*b = c1 * sT with c1 = e*b exact (<= 15 bits),
// h*c1 exact, and |w| - (h*c1)*sT formed exactly inside one fma.
static __device__ __noinline__ float qexact32_e2m1(float w, float u, float ia, float c1, float sT) {
  const float xt = u * ia;
  const float ax = fminf(fabsf(xt), 6.f);
  const float p2 = __uint_as_float(max(__float_as_uint(ax) & 0x7F800000u, 0x3F800000u));
  const float magic = p2 * 6291456.f;
  float qm = __fsub_rn(__fadd_rn(ax, magic), magic);
  const float h = qm + copysignf(0.25f * p2, ax - qm);
  const float half = h < 2.f ? 0.25f : (h < 4.f ? 0.5f : 1.f);
  const float lo = h - half, hi = h + half;
  const float d = fmaf(-(h * c1), sT, fabsf(w));
  const bool lo_even = (lo == 0.f || lo == 1.f || lo == 2.f || lo == 4.f);
  qm = d > 0.f ? hi : (d < 0.f ? lo : (lo_even ? lo : hi));
  return copysignf(fminf(qm, 6.f), w);
}

// Exact E4M3 decision in fp32 (power-of-two a): ab = a*b is exact, h*ab too
// (h has at most 5 significant bits), and |w| - h*ab is formed inside one fma.
// Spacing p2/8 in the binade [p2, 2 p2) (2^-9 below 2^-6); 448 is the top.
static __device__ __noinline__ float qexact32_e4m3(float w, float u, float ia, float ab) {
  const float xt = u * ia;
  const float ax = fminf(fabsf(xt), 448.f);
  const float p2 = __uint_as_float(max(__float_as_uint(ax) & 0x7F800000u, 0x3C800000u));
  const float magic = p2 * 1572864.f;
  float qm = __fsub_rn(__fadd_rn(ax, magic), magic);
  const float half = p2 * 0.0625f;
  const float h = qm + copysignf(half, ax - qm);
  const float lo = h - half, hi = h + half;
  const float d = fmaf(-h, ab, fabsf(w));
  const bool lo_even = fmodf(lo / (2.f * half), 2.f) == 0.f;
  qm = d > 0.f ? hi : (d < 0.f ? lo : (lo_even ? lo : hi));
  return copysignf(fminf(qm, 448.f), w);
}

// ---------------------------------------------------------------------------
// Projection of a block inverse-scale value known to a relative 2^-19.

constexpr int kAmbUlps = 34;

// Nearest value with MB mantissa bits, certified when v lies in [lo, hi] (the
// target's normal range) and at least kAmbUlps fp32 ulps from a midpoint.
template <int MB>
__device__ __forceinline__ float proj_fast(float v, float lo, float hi, bool& amb) {
  constexpr int SH = 23 - MB;
  constexpr uint32_t HALF = 1u << (SH - 1), MASK = (1u << SH) - 1u;
  const uint32_t bits = __float_as_uint(v);
  const int dist = (int)(bits & MASK) - (int)HALF;
  amb |= (abs(dist) <= kAmbUlps) || !(v >= lo && v <= hi);
  return __uint_as_float((bits + (HALF - 1u) + ((bits >> SH) & 1u)) & ~MASK);
}

// Stored factor of the new block inverse scale (fp16 value, 2^k, or E4M3 e).
// num and den must lie in [2^-60, 2^100]: then rounding of underflowing or
// overflowing terms cannot matter at the 2^-19 level; a zero den (possibly an
// all-zero code slice, possibly underflow) is settled by the exact path too.
template <int FMT>
__device__ __forceinline__ float a_fast(float num, float den, float isT, bool& amb) {
  if (!(num >= 0x1p-60f && num <= 0x1p100f && den >= 0x1p-60f && den <= 0x1p100f)) {
    amb = true;
    return 1.f;
  }
  float v = num * rcp_approx(den);
  if (FMT == FMT_INT4) return proj_fast<10>(v, 0x1p-14f, 65504.f, amb);
  if (fmt_pow2(FMT)) return proj_fast<0>(v, 0x1p-126f, 0x1p126f, amb);
  v *= isT;
  return proj_fast<3>(v, 0x1p-6f, 448.f, amb);
}

template <int FMT>
__device__ __forceinline__ void a_store_f(void* store, int64_t idx, float v) {
  if (FMT == FMT_INT4) {
    reinterpret_cast<__half*>(store)[idx] = __float2half_rn(v);
  } else if (fmt_pow2(FMT)) {
    reinterpret_cast<uint8_t*>(store)[idx] = (uint8_t)(__float_as_uint(v) >> 23);
  } else {
    reinterpret_cast<uint8_t*>(store)[idx] = (uint8_t)__nv_cvt_float_to_fp8(v, __NV_SATFINITE, __NV_E4M3);
  }
}

// ---------------------------------------------------------------------------
// Packed f32x2 arithmetic (one instruction for a pair of elements).
typedef unsigned long long f2;
__device__ __forceinline__ f2 pk(float lo, float hi) {
  f2 r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ float lo_of(f2 v) {
  float a;
  asm("{\n.reg .f32 t;\nmov.b64 {%0, t}, %1;\n}" : "=f"(a) : "l"(v));
  return a;
}
__device__ __forceinline__ float hi_of(f2 v) {
  float b;
  asm("{\n.reg .f32 t;\nmov.b64 {t, %0}, %1;\n}" : "=f"(b) : "l"(v));
  return b;
}
__device__ __forceinline__ f2 mul2(f2 a, f2 b) {
  f2 d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ f2 fma2(f2 a, f2 b, f2 c) {
  f2 d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ f2 add2(f2 a, f2 b) {
  f2 d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ f2 splat(float v) { return pk(v, v); }

// ---------------------------------------------------------------------------
// mbarrier and bulk-copy (TMA) primitives.  No multicast anywhere.

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, unsigned count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_fence_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, unsigned bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, unsigned parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Wall-clock bound of every wait in the solver's kernels (1 s): a wait that
// runs out records kFlagTimeout in the workspace header and returns, so a lost
// arrival ends in a status instead of a hung GPU.
constexpr unsigned long long kWaitLimitNs = 1000000000ull;

__device__ __forceinline__ unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ unsigned ld_volatile(const unsigned* a) { return *reinterpret_cast<const volatile unsigned*>(a); }

// True when a bounded wait begun at t0 must give up (its time is over, or some
// other wait already gave up); then kFlagTimeout is recorded.
__device__ __forceinline__ bool wait_expired(unsigned* flags, unsigned long long t0) {
  if (global_ns() - t0 > kWaitLimitNs || (ld_volatile(flags) & kFlagTimeout)) {
    atomicOr(flags, kFlagTimeout);
    return true;
  }
  return false;
}

__device__ __forceinline__ unsigned ld_acquire_gpu(const unsigned* a) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(a) : "memory");
  return v;
}

// Bounded wait for the phase of `parity` of a ring barrier: polls until it
// completes, or until kWaitLimitNs of wall time have passed or another wait has
// given up (checked every 256 polls), then records kFlagTimeout and returns
// false.  The first poll usually succeeds, so the timer is read only after it
// fails.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, unsigned parity, unsigned* flags) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = global_ns();
  for (unsigned i = 1;; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 255u) == 0u && wait_expired(flags, t0)) return false;
  }
}

// Wait for a copy this CTA issued to land before the CTA exits: bounded by
// kWaitLimitNs alone (a copy in flight completes whatever other waits did).
__device__ __forceinline__ void mbar_drain(uint64_t* bar, unsigned parity) {
  const unsigned long long t0 = global_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_ns() - t0 > kWaitLimitNs) return;
  }
}

// Orders this thread's earlier generic-proxy accesses to shared memory (the
// consumers' loads of a ring slot) before later async-proxy accesses (the
// tensor copy that refills the slot once the release is observed): without it
// a copy may overwrite a slot whose loads are not yet performed.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Copy `bytes` (multiple of 16, both addresses 16-byte aligned) from global
// memory into this CTA's shared memory, completing on `bar`.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, unsigned bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_u32(dst)),
               "l"(src), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}

// Tiled tensor copy (TMA) of the box at (x = column, y = row) of the 2-D
// tensor map `map` into this CTA's shared memory, completing on `bar`.  The
// column coordinate times the element size must be a multiple of 16 bytes;
// out-of-range rows and columns of the box are filled with zeros.
__device__ __forceinline__ void tma_load_2d(void* dst, const void* map, int x, int y, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
          smem_u32(dst)),
      "l"(map), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}

// Tiled tensor copy (TMA) of the box at (x, y, z) of the 3-D tensor map `map`
// into this CTA's shared memory, completing on `bar`; x times the element size
// must be a multiple of 16 bytes.
__device__ __forceinline__ void tma_load_3d(void* dst, const void* map, int x, int y, int z, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(
          smem_u32(dst)),
      "l"(map), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar))
      : "memory");
}

// L2 prefetch of the box at (x = column, y = row) of the 2-D tensor map `map`
// (no shared memory written, no completion to wait for).
__device__ __forceinline__ void tma_prefetch_2d(const void* map, int x, int y) {
  asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global.tile [%0, {%1, %2}];" ::"l"(map), "r"(x), "r"(y)
               : "memory");
}

// Programmatic dependent launch.  A grid launched with programmatic stream
// serialization may start while the grid before it in the stream is still
// running; griddep_wait() returns once every grid it depends on has completed
// and its memory operations are visible, so it must come before the first
// read of anything an earlier kernel wrote, in every CTA (a CTA that exits
// without it would let the next grid overtake the unfinished one).
// griddep_launch_dependents() lets the next grid begin launching early.
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

__device__ __forceinline__ void consumer_sync(int nthreads) {
  asm volatile("bar.sync 1, %0;" ::"r"(nthreads) : "memory");
}

}  // namespace dq
