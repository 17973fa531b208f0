// dq_iter.cuh -- the per-iteration pass k_iter: one BCD iteration in one read
// of W (included by dq_solver.cu).
//
// CTA = 15 consumer warps + 1 producer warp (16 warps, 4 per SM sub-partition,
// so each thread may hold 128 registers).  The producer streams the CTA's rows
// of the current column strip, one row per bulk (TMA) copy, into a ring of
// shared-memory tiles of kRowsPerTile rows, guarded by full/empty mbarriers.
// Consumer warp w takes rows w and w + 15 of every tile; lane l takes the 8
// consecutive columns 8l..8l+7 of the strip.  Per element the consumers run the
// fp32 fast paths and fall back to the exact definitions where those flag.
// Column sums run in fp32 for kRun rows of a lane and are then added into fp64
// accumulators kept in shared memory.
#pragma once

#include "dq_device.cuh"
#include "dq_fast.cuh"
#include "dq_internal.h"

namespace dq {

constexpr int kConsumerWarps = 15;
constexpr int kConsumers = kConsumerWarps * 32;
constexpr int kIterThreads = kConsumers + 32;
constexpr int kConsumerTreeTop = 256;  // largest power of two below kConsumers
static_assert(kConsumerTreeTop < kConsumers && 2 * kConsumerTreeTop >= kConsumers, "tree reduction shape");
constexpr int kRowsPerWarp = 2;
constexpr int kRowsPerTile = kConsumerWarps * kRowsPerWarp;
constexpr int kRun = 8;
constexpr int kRingBytes = 96 * 1024;
// relative error bound of the fp64 column totals built from fp32 runs of kRun
// rows (kRun roundings per run, fp64 beyond), plus the oracle's own fp64 error
constexpr double kColErr = 2.0 * kRun * 0x1p-24 + 1e-11;
// Relative bracket of the E2M1 candidate: the fp32 candidate W*(1/b)*(1/e)*(1/s_T)
// is within 7 * 2^-24 of W/(a b), the bracket factors add two more roundings.
constexpr float kRelGuard = 0x1p-20f;

__host__ __device__ constexpr int ring_stages(int es) { return kRingBytes / (kRowsPerTile * kStripMax * es); }
__host__ __device__ constexpr size_t iter_col_acc_bytes() {
  return (size_t)kConsumerWarps * kStripMax * sizeof(double2);
}
__host__ __device__ constexpr size_t iter_smem_bytes(int es) {
  return (size_t)kRingBytes + iter_col_acc_bytes() + 2 * sizeof(uint64_t) * ring_stages(es) +
         (2 + kStripMax + 4) * sizeof(int);
}

// ---------------------------------------------------------------------------
// E2M1 fast path with the hardware conversion: both ends of the bracket
// [x~ (1 - g), x~ (1 + g)] are converted (round to nearest even, saturating);
// equal codes prove the exact quotient has that code too (rounding is
// monotone), different codes flag the pair for the exact path.
__device__ __forceinline__ uint32_t cvt_e2m1x2(float hi, float lo) {
  uint32_t r;
  asm("{\n.reg .b8 t;\ncvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\ncvt.u32.u8 %0, t;\n}" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}
__device__ __forceinline__ float2 dec_e2m1x2(uint32_t code) {  // low nibble -> .x, high nibble -> .y
  uint32_t h;
  asm("{\n.reg .b8 t;\ncvt.u8.u32 t, %1;\ncvt.rn.f16x2.e2m1x2 %0, t;\n}" : "=r"(h) : "r"(code));
  return __half22float2(*reinterpret_cast<const __half2*>(&h));
}

__device__ __forceinline__ void req8_e2m1(const float uw[8], float ia, float q[8], bool& near) {
  const float ilo = ia * (1.f - kRelGuard), ihi = ia * (1.f + kRelGuard);
#pragma unroll
  for (int c = 0; c < 8; c += 2) {
    const uint32_t lo = cvt_e2m1x2(uw[c + 1] * ilo, uw[c] * ilo);
    const uint32_t hi = cvt_e2m1x2(uw[c + 1] * ihi, uw[c] * ihi);
    near |= lo != hi;
    const float2 d = dec_e2m1x2(lo);
    q[c] = d.x;
    q[c + 1] = d.y;
  }
}

// Per-lane state of a column strip segment: b, the candidate factor cb = 1/b
// (times 1/s_T for NVFP4), the guard threshold per column (MXINT4 columns with a
// power-of-two b have an exact candidate and need no guard), fp32 column runs.
struct ColState {
  float bj[8], cb[8], thr[8], cn[8], cd[8];
  bool ok;
};

// Exact fp64 decision for one element (factors outside the fast range).
template <int FMT>
__device__ __noinline__ float qexact64(float w, float a, float b, double sTd) {
  const double ab = ab_exact<FMT>(a, b, sTd);
  const float xt = (float)((double)w / ab);
  if (FMT == FMT_NVFP4) return q_e2m1<FMT>(xt, w, a, b, sTd);
  return q_int4<FMT>(xt, w, a, b, sTd);
}

// Requantize the 8 elements of a lane with block factor a (stored value).
// Fast path for all lanes; a lane with a flagged element re-derives which
// elements are close to a boundary and settles only those exactly.
template <int FMT>
__device__ __forceinline__ void requant8(const float w[8], const float uw[8], float a, const ColState& cs, float sT,
                                         double sTd, bool active, float q[8], unsigned* s_cnt) {
  const float ia = rcp_approx(a);
  const bool ok = cs.ok && in_range(ia);
  bool near = !ok;
  if (FMT == FMT_NVFP4) {
    req8_e2m1(uw, ia, q, near);
  } else {
#pragma unroll
    for (int c = 0; c < 8; ++c) q[c] = qfast_int4(uw[c], ia, FMT == FMT_MXINT4 ? cs.thr[c] : 0.5f - kGuard, near);
  }
  if (near && active) {
    atomicAdd(&s_cnt[0], 1u);
    if (!ok) {
#pragma unroll
      for (int c = 0; c < 8; ++c) q[c] = qexact64<FMT>(w[c], a, cs.bj[c], sTd);
    } else if (FMT == FMT_NVFP4) {
      const float ilo = ia * (1.f - kRelGuard), ihi = ia * (1.f + kRelGuard);
#pragma unroll
      for (int c = 0; c < 8; c += 2) {
        const uint32_t lo = cvt_e2m1x2(uw[c + 1] * ilo, uw[c] * ilo);
        const uint32_t hi = cvt_e2m1x2(uw[c + 1] * ihi, uw[c] * ihi);
        const uint32_t diff = lo ^ hi;
        if (diff & 0x0Fu) q[c] = qexact32_e2m1(w[c], uw[c], ia, a * cs.bj[c], sT);
        if (diff & 0xF0u) q[c + 1] = qexact32_e2m1(w[c + 1], uw[c + 1], ia, a * cs.bj[c + 1], sT);
      }
    } else {
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const float qu = fmaf(uw[c], ia, 12582912.f) - 12582912.f;
        const float thr = FMT == FMT_MXINT4 ? cs.thr[c] : 0.5f - kGuard;
        if (fabsf(fmaf(uw[c], ia, -qu)) > thr) q[c] = qexact32_int4(w[c], uw[c], ia, a * cs.bj[c]);
      }
    }
  }
}

// ---------------------------------------------------------------------------
// Exact fp64 column sums of one column over all rows (ambiguous-projection
// fallback), run by the consumer threads of the finalizing CTA.
template <int FMT, int WDT>
__device__ double2 column_exact(const Problem& p, int64_t j, float bj, double sTd, double* scratch) {
  const float isT = FMT == FMT_NVFP4 ? (float)(1.0 / sTd) : 1.f;
  const float cb = __frcp_rn(bj) * isT;
  double cn = 0.0, cd = 0.0;
  for (int64_t i = threadIdx.x; i < p.M; i += kConsumers) {
    float w;
    if (WDT == DT_F32) {
      w = __ldg(reinterpret_cast<const float*>(p.W) + i * p.N + j);
    } else if (WDT == DT_BF16) {
      w = __uint_as_float((uint32_t)__ldg(reinterpret_cast<const unsigned short*>(p.W) + i * p.N + j) << 16);
    } else {
      w = __half2float(__ushort_as_half(__ldg(reinterpret_cast<const unsigned short*>(p.W) + i * p.N + j)));
    }
    const int64_t bidx = i * p.nb + j / p.G;
    float a;
    if (FMT == FMT_INT4) {
      a = __half2float(__ushort_as_half(__ldcg(reinterpret_cast<const unsigned short*>(p.a_store) + bidx)));
    } else {
      const uint32_t v = __ldcg(reinterpret_cast<const unsigned char*>(p.a_store) + bidx);
      a = FMT == FMT_MXINT4 ? __uint_as_float(v << 23) : e4m3_value(v);
    }
    const float ia = __frcp_rn(a);
    const bool ok = in_range(cb) && in_range(ia);
    const float q = quant<FMT>(w, w * cb, ia, ok, a, bj, sTd);
    const double sv = (double)q * (double)a;
    cn = fma((double)w, sv, cn);
    cd = fma(sv, sv, cd);
  }
  scratch[2 * threadIdx.x] = cn;
  scratch[2 * threadIdx.x + 1] = cd;
  consumer_sync(kConsumers);
  for (int o = kConsumerTreeTop; o > 0; o >>= 1) {  // fixed-order tree
    if (threadIdx.x < o && threadIdx.x + o < kConsumers) {
      scratch[2 * threadIdx.x] += scratch[2 * (threadIdx.x + o)];
      scratch[2 * threadIdx.x + 1] += scratch[2 * (threadIdx.x + o) + 1];
    }
    consumer_sync(kConsumers);
  }
  const double2 r = make_double2(scratch[0], scratch[1]);
  consumer_sync(kConsumers);
  return r;
}


template <int WDT>
__device__ __forceinline__ void smem_row8(const unsigned char* src, float w[8]) {
  if (WDT == DT_F32) {
    const float4 x = *reinterpret_cast<const float4*>(src);
    const float4 y = *reinterpret_cast<const float4*>(src + 16);
    w[0] = x.x; w[1] = x.y; w[2] = x.z; w[3] = x.w;
    w[4] = y.x; w[5] = y.y; w[6] = y.z; w[7] = y.w;
  } else {
    const uint4 v = *reinterpret_cast<const uint4*>(src);
    const uint32_t uu[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      if (WDT == DT_BF16) {
        w[2 * i] = __uint_as_float(uu[i] << 16);
        w[2 * i + 1] = __uint_as_float(uu[i] & 0xFFFF0000u);
      } else {
        const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&uu[i]));
        w[2 * i] = f.x;
        w[2 * i + 1] = f.y;
      }
    }
  }
}

// One row of one lane: requantize the incoming iterate, block sums and update,
// requantize, column sums.  Warp-collective (shuffles); `active` lanes hold
// real columns.  Returns nothing; updates cs, mse_acc and the counters.
template <int FMT>
__device__ __forceinline__ void row_step(const Problem& p, const float w[8], float aold, int64_t bidx, bool active,
                                         bool leader, int lpb, ColState& cs, float sT, float isT, double sTd,
                                         double& mse_acc, unsigned* s_cnt) {
  float uw[8], q[8];
#pragma unroll
  for (int c = 0; c < 8; ++c) uw[c] = w[c] * cs.cb[c];
  requant8<FMT>(w, uw, aold, cs, sT, sTd, active, q, s_cnt);
  float num = 0.f, den = 0.f;
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    const float pq = q[c] * cs.bj[c];
    num = fmaf(w[c], pq, num);
    den = fmaf(pq, pq, den);
  }
  for (int o = 1; o < lpb; o <<= 1) {
    num += __shfl_xor_sync(0xffffffffu, num, o);
    den += __shfl_xor_sync(0xffffffffu, den, o);
  }
  bool amb = false;
  float anew = a_fast<FMT>(num, den, isT, amb);
  double nsum = (double)num, dsum = (double)den;
  if (__any_sync(0xffffffffu, amb && active)) {
    double n64 = 0.0, d64 = 0.0;
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const double pd = (double)(q[c] * cs.bj[c]);
      n64 = fma((double)w[c], pd, n64);
      d64 = fma(pd, pd, d64);
    }
    for (int o = 1; o < lpb; o <<= 1) {
      n64 += __shfl_xor_sync(0xffffffffu, n64, o);
      d64 += __shfl_xor_sync(0xffffffffu, d64, o);
    }
    if (amb) {
      if (active && leader) atomicAdd(&s_cnt[1], 1u);
      anew = d64 == 0.0 ? 1.f : (float)a_project<FMT>(n64 / d64, sTd);
      nsum = n64;
      dsum = d64;
    }
  }
  if (active && leader) {
    const double av = FMT == FMT_NVFP4 ? sTd * (double)aold : (double)aold;
    mse_acc += av * (av * dsum - 2.0 * nsum);
    a_store_f<FMT>(p.a_store, bidx, anew);
  }
  requant8<FMT>(w, uw, anew, cs, sT, sTd, active, q, s_cnt);
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    const float sv = q[c] * anew;  // exact; NVFP4 leaves s_T out
    cs.cn[c] = fmaf(w[c], sv, cs.cn[c]);
    cs.cd[c] = fmaf(sv, sv, cs.cd[c]);
  }
}

// fp32 column runs into the warp's fp64 accumulators (layout [warp][c][lane]).
__device__ __forceinline__ void flush_runs(ColState& cs, double2* acc, int warp, int lane) {
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    double2& a = acc[(warp * 8 + c) * 32 + lane];
    double2 v = a;
    v.x += (double)cs.cn[c];
    v.y += (double)cs.cd[c];
    a = v;
    cs.cn[c] = cs.cd[c] = 0.f;
  }
}

template <int FMT, int WDT>
__global__ void __launch_bounds__(kIterThreads, 1) k_iter(Problem p, int t) {
  if (p.hdr->flags & kFlagNonFinite) return;
  constexpr int ES = WDT == DT_F32 ? 4 : 2;
  constexpr int S = ring_stages(ES);
  extern __shared__ __align__(128) unsigned char smem[];
  unsigned char* ring = smem;
  double2* acc = reinterpret_cast<double2*>(smem + kRingBytes);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kRingBytes + iter_col_acc_bytes());
  uint64_t* empty = full + S;
  int* s_misc = reinterpret_cast<int*>(empty + S);  // [0] ticket result, [1] #ambiguous, [2..] columns
  unsigned* s_cnt = reinterpret_cast<unsigned*>(s_misc + 2 + kStripMax);  // exact-path counters
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row_bytes = p.TS * ES;  // ring slot per row
  const int stage_bytes = kRowsPerTile * row_bytes;

  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], kConsumerWarps);
    }
    mbar_fence_init();
    s_cnt[0] = s_cnt[1] = s_cnt[2] = 0u;
  }
  __syncthreads();

  const int64_t k = blockIdx.x;
  const int64_t u_begin = range_begin(k, p.P, p.L), u_end = range_begin(k + 1, p.P, p.L);

  if (warp == kConsumerWarps) {
    // ---------------- producer warp ----------------
    int64_t tile = 0;
    for (int64_t u = u_begin; u < u_end;) {
      const int64_t s = u / p.M;
      const int64_t r0 = u - s * p.M;
      const int64_t r1 = min(p.M, r0 + (u_end - u));
      const int64_t c0 = s * p.TS;
      const int width = (int)min((int64_t)p.TS, p.N - c0);
      const unsigned bytes = (unsigned)(width * ES);
      for (int64_t tr = r0; tr < r1; tr += kRowsPerTile, ++tile) {
        const int st = (int)(tile % S);
        const unsigned par = (unsigned)((tile / S) & 1) ^ 1u;
        mbar_wait(&empty[st], par, &p.hdr->flags);
        const int nr = (int)min((int64_t)kRowsPerTile, r1 - tr);
        if (lane == 0) mbar_arrive_expect_tx(&full[st], (unsigned)nr * bytes);
        __syncwarp();
        if (lane < nr) {
          const unsigned char* src =
              reinterpret_cast<const unsigned char*>(p.W) + ((tr + lane) * p.N + c0) * (int64_t)ES;
          bulk_g2s(ring + st * stage_bytes + lane * row_bytes, src, bytes, &full[st]);
        }
      }
      u = (s + 1) * p.M;
    }
    return;
  }

  // ---------------- consumer warps ----------------
  const int lpb = p.G / 8;  // lanes per block
  const bool leader = (lane & (lpb - 1)) == 0;
  const float sT = p.hdr->sT;
  const double sTd = (double)sT;
  const float isT = FMT == FMT_NVFP4 ? __frcp_rn(sT) : 1.f;
  const bool sT_ok = FMT != FMT_NVFP4 || in_range(isT);
  const int64_t s_first = u_begin / p.M;
  double mse_acc = 0.0;
  int64_t tile = 0;

  for (int64_t u = u_begin; u < u_end;) {
    const int64_t s = u / p.M;
    const int64_t r0 = u - s * p.M;
    const int64_t r1 = min(p.M, r0 + (u_end - u));
    const int64_t c0 = s * p.TS;
    const int width = (int)min((int64_t)p.TS, p.N - c0);
    const bool active = lane * 8 < width;
    const int64_t col = c0 + lane * 8;
    const int64_t blk_col = col / p.G;

    ColState cs;
    cs.ok = sT_ok;
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      cs.bj[c] = 1.f;
      cs.cb[c] = 1.f;
      cs.thr[c] = 0.5f - kGuard;
      cs.cn[c] = cs.cd[c] = 0.f;
      acc[(warp * 8 + c) * 32 + lane] = make_double2(0.0, 0.0);
    }
    if (active) {
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        cs.bj[c] = b_decode(p.b_store, p.col_dt, col + c);
        cs.cb[c] = __frcp_rn(cs.bj[c]) * isT;
        cs.ok = cs.ok && in_range(cs.cb[c]);
        // MXINT4: a = 2^k, so a power-of-two b makes the candidate exact
        if (FMT == FMT_MXINT4 && (__float_as_uint(cs.bj[c]) & 0x007FFFFFu) == 0u) cs.thr[c] = 2.f;
      }
    }
    int run = 0;
    // block scales of this warp's rows, one tile ahead
    float an0 = 1.f, an1 = 1.f;
    if (active && r0 + warp < r1) an0 = a_decode<FMT>(p.a_store, (r0 + warp) * p.nb + blk_col);
    if (active && r0 + warp + kConsumerWarps < r1)
      an1 = a_decode<FMT>(p.a_store, (r0 + warp + kConsumerWarps) * p.nb + blk_col);

    for (int64_t tr = r0; tr < r1; tr += kRowsPerTile, ++tile) {
      const int st = (int)(tile % S);
      const unsigned par = (unsigned)((tile / S) & 1);
      const int64_t ra = tr + warp, rb = ra + kConsumerWarps;
      const bool has_a = ra < r1, has_b = rb < r1;  // warp-uniform
      const float aa = an0, ab = an1;
      if (active && ra + kRowsPerTile < r1) an0 = a_decode<FMT>(p.a_store, (ra + kRowsPerTile) * p.nb + blk_col);
      if (active && rb + kRowsPerTile < r1) an1 = a_decode<FMT>(p.a_store, (rb + kRowsPerTile) * p.nb + blk_col);
      mbar_wait(&full[st], par, &p.hdr->flags);
      float wa[8], wb[8];
#pragma unroll
      for (int c = 0; c < 8; ++c) wa[c] = wb[c] = 0.f;
      const unsigned char* base = ring + st * stage_bytes + lane * 8 * ES;
      if (active && has_a) smem_row8<WDT>(base + warp * row_bytes, wa);
      if (active && has_b) smem_row8<WDT>(base + (warp + kConsumerWarps) * row_bytes, wb);
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[st]);
      if (has_a) {
        row_step<FMT>(p, wa, aa, ra * p.nb + blk_col, active, leader, lpb, cs, sT, isT, sTd, mse_acc, s_cnt);
        ++run;
      }
      if (has_b) {
        row_step<FMT>(p, wb, ab, rb * p.nb + blk_col, active, leader, lpb, cs, sT, isT, sTd, mse_acc, s_cnt);
        ++run;
      }
      if (run >= kRun) {
        run = 0;
        flush_runs(cs, acc, warp, lane);
      }
    }
    flush_runs(cs, acc, warp, lane);

    // CTA reduction of the column sums over the consumer warps, fixed order.
    // Thread t sums entry (c, l) = (t / 32, t % 32), i.e. column 8 (t % 32) + t / 32.
    consumer_sync(kConsumers);
    const int64_t slot = k * p.segmax + (s - s_first);
    if (threadIdx.x < kStripMax) {
      const int cc = threadIdx.x >> 5, ll = threadIdx.x & 31;
      const int colw = ll * 8 + cc;
      if (colw < width) {
        double2 tot = acc[cc * 32 + ll];
        for (int wi = 1; wi < kConsumerWarps; ++wi) {
          const double2 v = acc[(wi * 8 + cc) * 32 + ll];
          tot.x += v.x;
          tot.y += v.y;
        }
        p.col_part[slot * p.TS + colw] = tot;
      }
    }
    __threadfence();
    consumer_sync(kConsumers);
    const int64_t k_first = cta_of(s * p.M, p.P, p.L);
    const int64_t k_last = cta_of((s + 1) * p.M - 1, p.P, p.L);
    if (threadIdx.x == 0) {
      const unsigned prev = atomicAdd(&p.strip_counter[s], 1u);
      s_misc[0] = prev == (unsigned)(k_last - k_first) ? 1 : 0;
      s_misc[1] = 0;
    }
    consumer_sync(kConsumers);
    if (s_misc[0]) {
      __threadfence();
      // totals in CTA order, certified projection
      double bnew = 1.0;
      if (threadIdx.x < width) {
        double2 tot = make_double2(0.0, 0.0);
        for (int64_t kk = k_first; kk <= k_last; ++kk) {
          const int64_t sl = kk * p.segmax + (s - range_begin(kk, p.P, p.L) / p.M);
          const double2 v = __ldcg(&p.col_part[sl * p.TS + threadIdx.x]);
          tot.x += v.x;
          tot.y += v.y;
        }
        // certified only when the fp32 runs stayed well inside the normal
        // range (no overflow; underflowed terms negligible); a zero total may
        // be underflow and is settled exactly as well
        const bool safe = tot.x >= 0x1p-60 && tot.x <= 0x1p100 && tot.y >= 0x1p-60 && tot.y <= 0x1p100;
        const double v = FMT == FMT_NVFP4 ? (tot.x / tot.y) / sTd : tot.x / tot.y;
        const double lo = safe ? b_project(v * (1.0 - kColErr), p.col_dt) : 0.0;
        const double hi = safe ? b_project(v * (1.0 + kColErr), p.col_dt) : 1.0;
        if (lo == hi) {
          bnew = lo;
        } else {
          const int slot_a = atomicAdd(&s_misc[1], 1);
          s_misc[2 + slot_a] = threadIdx.x;
        }
      }
      consumer_sync(kConsumers);
      const int namb = s_misc[1];
      if (threadIdx.x == 0) s_cnt[2] += (unsigned)namb;
      double* scratch = reinterpret_cast<double*>(acc);
      for (int ia = 0; ia < namb; ++ia) {
        const int cidx = s_misc[2 + ia];
        const float bold = b_decode(p.b_store, p.col_dt, c0 + cidx);
        const double2 ex = column_exact<FMT, WDT>(p, c0 + cidx, bold, sTd, scratch);
        if (threadIdx.x == cidx) {
          const double v = FMT == FMT_NVFP4 ? (ex.x / ex.y) / sTd : ex.x / ex.y;
          bnew = ex.y == 0.0 ? 1.0 : b_project(v, p.col_dt);
        }
      }
      consumer_sync(kConsumers);
      if (threadIdx.x < width) b_encode(p.b_store, p.col_dt, c0 + threadIdx.x, bnew);
      if (threadIdx.x == 0) p.strip_counter[s] = 0u;
    }
    consumer_sync(kConsumers);
    u = (s + 1) * p.M;
  }

  // MSE of the incoming iterate: CTA sum, then CTA-ordered total
  double* mred = reinterpret_cast<double*>(acc);
  mred[threadIdx.x] = mse_acc;
  consumer_sync(kConsumers);
  for (int o = kConsumerTreeTop; o > 0; o >>= 1) {
    if (threadIdx.x < o && threadIdx.x + o < kConsumers) mred[threadIdx.x] += mred[threadIdx.x + o];
    consumer_sync(kConsumers);
  }
  if (threadIdx.x == 0) {
    if (s_cnt[0]) atomicAdd(&p.hdr->n_quant_exact, (unsigned long long)s_cnt[0]);
    if (s_cnt[1]) atomicAdd(&p.hdr->n_block_exact, (unsigned long long)s_cnt[1]);
    if (s_cnt[2]) atomicAdd(&p.hdr->n_col_exact, (unsigned long long)s_cnt[2]);
    p.cta_part[k] = mred[0];
    __threadfence();
    const unsigned prev = atomicAdd(&p.hdr->cta_counter, 1u);
    if (prev == (unsigned)p.P - 1u) {
      __threadfence();
      double tot = p.hdr->sumW2;
      for (int64_t kk = 0; kk < p.P; ++kk) tot += __ldcg(&p.cta_part[kk]);
      p.mse[t - 1] = tot / ((double)p.M * (double)p.N);
      p.hdr->cta_counter = 0u;
    }
  }
}

}  // namespace dq
