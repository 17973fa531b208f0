// dq_iter.cuh -- the per-iteration pass k_iter: one BCD iteration in one read
// of the block-columns that can still change (included by dq_solver.cu).
//
// Block-columns.  A block-column is the M x G slab of W under one column of
// blocks.  Its block scales a_{:,g} and its column scales b_j (j in the
// block-column) interact only with each other: the block update of a_ig reads
// the G elements of block (i, g) and their column scales, and the column
// update of b_j reads column j and the block scales of the blocks holding it
// (reproduction README, "Core equations"; the NVFP4 tensor scale is fixed at
// init).  One BCD iteration therefore maps each block-column's state to its
// next state by itself, and a block-column whose scales all come out of an
// iteration unchanged is at a fixed point: every later iteration repeats the
// same sums, the same updates and the same residuals.  Such a block-column is
// dropped from the later passes; its share of the reconstruction MSE is kept
// from the pass that last computed it.  The results are those of the full
// iteration, bit for bit.
//
// Schedule of a pass.  The active block-columns (all of them in the first pass
// and the final pass) are taken in increasing order, 15 at a time, into
// strips; the (strip, row) units are laid out strip-major and split into
// equal contiguous ranges, one per CTA.  A CTA is 15 consumer warps + 1
// producer warp (512 threads, 128 registers each).  Consumer warp w owns
// block-column w of the strip; its lanes are (row-lane rho, octet o): lane
// rho * (G/8) + o takes the 8 columns 8o..8o+7 of the block-column in rows rho
// and rho + 32/(G/8) of every tile, so a tile is 2 * 32/(G/8) rows (512
// elements per block-column).  The producer fills a shared-memory ring with
// one 2-D tensor copy (TMA) per block-column and tile, wherever the active
// block-columns lie; a warp's 32 lanes read 512 contiguous bytes of its slot.
// The pair arithmetic runs as packed f32x2 instructions.  Column sums and the
// reconstruction residuals run in fp32 for run_rows<FMT>() rows of a lane and
// are then added into fp64 accumulators kept in shared memory.
#pragma once

#include <cuda.h>  // CUtensorMap

#include "dq_device.cuh"
#include "dq_fast.cuh"
#include "dq_internal.h"

namespace dq {

constexpr int kConsumerTreeTop = 256;  // largest power of two below kConsumers
static_assert(kConsumerTreeTop < kConsumers && 2 * kConsumerTreeTop >= kConsumers, "tree reduction shape");
// kinds of k_iter pass: a BCD iteration; a BCD iteration that also tracks the
// codes between iterates (changed-code counts); the final pass (codes of the
// final iterate and the last MSE)
enum : int { PASS_ITER = 0, PASS_COUNT = 1, PASS_FINAL = 2 };
// rows of a lane's fp32 column-sum and residual runs before they are added
// into fp64: shorter runs tighten the certified column projection (fewer
// columns need the exact update) at the cost of more fp64 adds; NVFP4, whose
// exact updates cost most, takes 4, the other formats 8 (measured)
template <int FMT>
constexpr int run_rows() { return FMT == FMT_NVFP4 ? 4 : 8; }
// relative error bound of the fp64 column totals built from fp32 runs of
// run_rows rows (that many roundings per run, fp64 beyond), plus the oracle's
// own fp64 error
template <int FMT>
constexpr double col_err() { return 2.0 * run_rows<FMT>() * 0x1p-24 + 1e-11; }
// Relative bracket of the E2M1 candidate: the fp32 candidate W*(1/b)*(1/e)*(1/s_T)
// is within 7 * 2^-24 of W/(a b), the bracket factors add two more roundings.
constexpr float kRelGuard = 0x1p-20f;

// CTA-ordered schedule of one pass, computed by every CTA from the same flags.
struct Sched {
  long long L;                // (strip, row) units of the pass
  long long u_begin, u_end;   // this CTA's units
  int nact;                   // active block-columns
  int Pt;                     // CTAs that get units (a multiple of the strip count when that keeps 90%)
  int v_first;                // first strip of this CTA's range
  int ident;                  // the active list is 0 .. nb-1 (first and final pass)
};

// ---------------------------------------------------------------------------
// E2M1 conversions (round to nearest even, saturating) and decode.
__device__ __forceinline__ uint32_t cvt_e2m1x2(float hi, float lo) {
  uint32_t r;
  asm("{\n.reg .b8 t;\ncvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\ncvt.u32.u8 %0, t;\n}" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}
__device__ __forceinline__ f2 dec_e2m1x2(uint32_t code) {  // low nibble -> low float, high nibble -> high float
  uint32_t h;
  asm("{\n.reg .b8 t;\ncvt.u8.u32 t, %1;\ncvt.rn.f16x2.e2m1x2 %0, t;\n}" : "=r"(h) : "r"(code));
  const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&h));
  return pk(f.x, f.y);
}

// E4M3 conversions of four values (pairs p, q): byte k of the word is element k
// (the low element of p in the low byte); round to nearest even, saturating
// at 448.  The decode is exact (every E4M3 value is an fp16 value).
__device__ __forceinline__ uint32_t cvt_e4m3x4(f2 p, f2 q) {
  uint32_t r;
  asm("{\n.reg .b16 l, h;\n"
      "cvt.rn.satfinite.e4m3x2.f32 l, %2, %1;\n"
      "cvt.rn.satfinite.e4m3x2.f32 h, %4, %3;\n"
      "mov.b32 %0, {l, h};\n}"
      : "=r"(r)
      : "f"(lo_of(p)), "f"(hi_of(p)), "f"(lo_of(q)), "f"(hi_of(q)));
  return r;
}
__device__ __forceinline__ void dec_e4m3x4(uint32_t c, f2& p, f2& q) {
  uint32_t h0, h1;
  asm("{\n.reg .b16 l, h;\n"
      "mov.b32 {l, h}, %2;\n"
      "cvt.rn.f16x2.e4m3x2 %0, l;\n"
      "cvt.rn.f16x2.e4m3x2 %1, h;\n}"
      : "=r"(h0), "=r"(h1)
      : "r"(c));
  const float2 f0 = __half22float2(*reinterpret_cast<const __half2*>(&h0));
  const float2 f1 = __half22float2(*reinterpret_cast<const __half2*>(&h1));
  p = pk(f0.x, f0.y);
  q = pk(f1.x, f1.y);
}

// Stored block scale as loaded (fp16 bits or an 8-bit code), fetched a tile
// ahead of its use and decoded only there, so the warp does not wait for the
// load right after issuing it.
// Block scales are rewritten inside the kernel, so the load goes to L2
// (ld.global.cg), never through the read-only or L1 path.
template <int FMT>
__device__ __forceinline__ uint32_t a_fetch(const void* store, int64_t idx) {
  if (FMT == FMT_INT4) return __ldcg(reinterpret_cast<const unsigned short*>(store) + idx);
  return __ldcg(reinterpret_cast<const unsigned char*>(store) + idx);
}

// Column scale from storage through L2 (other CTAs rewrite it inside the kernel).
__device__ __forceinline__ float b_decode_cg(const void* store, int col_dt, int64_t j) {
  const unsigned short h = __ldcg(reinterpret_cast<const unsigned short*>(store) + j);
  return col_dt == DT_F16 ? __half2float(__ushort_as_half(h)) : __uint_as_float((uint32_t)h << 16);
}

// Stores a block scale in its storage format from its stored bits.
template <int FMT>
__device__ __forceinline__ void a_put_raw(void* store, int64_t idx, uint32_t raw) {
  if (FMT == FMT_INT4) {
    reinterpret_cast<unsigned short*>(store)[idx] = (unsigned short)raw;
  } else {
    reinterpret_cast<uint8_t*>(store)[idx] = (uint8_t)raw;
  }
}

// the stored form of the factor 1 (fp16 1.0, 2^0, E4M3 1.0)
template <int FMT>
__device__ __forceinline__ constexpr uint32_t a_raw_one() {
  return FMT == FMT_INT4 ? 0x3C00u : (fmt_pow2(FMT) ? 127u : 0x38u);
}

template <int FMT>
__device__ __forceinline__ float a_dec(uint32_t v) {
  if (FMT == FMT_INT4) return __half2float(__ushort_as_half((unsigned short)v));
  if (fmt_pow2(FMT)) return __uint_as_float(v << 23);
  uint32_t h;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h) : "h"((unsigned short)v));
  return __half2float(__ushort_as_half((unsigned short)(h & 0xFFFFu)));
}

// Column table of a warp's block-column in shared memory: for each octet o
// of the block, 4 column pairs of (b) and 4 of (cb); lane (rho, o) points at
// its octet's entries and lanes of one octet read the same word (broadcast).
// Loads are volatile so the compiler re-reads the table at each use instead of
// holding 16 registers.
__device__ __forceinline__ f2 col_ld(const f2* tab, int i) {
  f2 v;
  asm volatile("ld.shared.b64 %0, [%1];" : "=l"(v) : "r"(smem_u32(tab + i)));
  return v;
}

// Per-lane state of a block-column segment, as 4 column pairs: b, the
// candidate factor cb = 1/b (times 1/s_T for NVFP4), fp32 column runs, and the
// guard threshold per column (MXINT4/MXINT8 columns with a power-of-two b have an exact
// candidate and need no guard).
struct ColState {
  const f2* tb;   // this lane's 4 b pairs in the warp's table
  const f2* tcb;  // this lane's 4 cb pairs
  int lane;
  f2 cn2[4], cd2[4];
  float thr[8];
  f2 res2;  // fp32 run of squared reconstruction residuals
  bool ok;
  bool tie_ok;  // a flagged element of this lane can only be an exact tie (see tie_certified)
};

// Significant bits of a positive normal float (1 + index of the lowest set
// mantissa bit counted from the top): 1 for a power of two, 24 at most.
__device__ __forceinline__ int sig_bits(float v) {
  return 25 - __ffs((int)((__float_as_uint(v) & 0x007FFFFFu) | 0x00800000u));
}

// Tie certification.  Write W = w 2^g with w an odd integer below 2^11 (bf16 or
// fp16 W), the element's scale product P = a b = p 2^h with p odd and at most k
// bits long, and a rounding boundary B of the grid as an odd integer over a
// power of two: at most 4 bits on the INT4 grid (the boundaries that matter
// after clipping are +-1/2 .. +-15/2; 8 bits on the INT8 grid, +-1/2 ..
// +-255/2), 3 bits on E2M1 (1/4 .. 5), 5 bits on E4M3 (midpoints of
// neighbours with 3 mantissa bits, 2^-10 .. 432).  Then B P = n 2^f with n
// odd, and if W != B P, |W - B P| >= 2^min(g, f):
//  * g >= f: |x - B| >= |B| / n >= 1 / (2 p) on the integer grids (absolute,
//    whatever the boundary's own bits), and |x - B| / |B| >= 1 / n > 2^-(3 + k)
//    on E2M1, > 2^-(5 + k) on E4M3 (relative);
//  * g < f:  |x - B| >= x / 2^11, i.e. 2^-13 absolute (|B| >= 1/2) or 2^-11
//    relative.
// The fast paths flag an element only when x lies within 2^-14 + 2^-19 of a
// boundary (INT4 grid, absolute; candidate error included), within
// 2^-14 + 4.6e-5 < 2^-13 of it (INT8 grid, |x| <= 128.5), or within
// 1.5 * 2^-20 of it relative (E2M1 and E4M3 brackets plus candidate error).
// So with k <= 12 (integer grids), k <= 15 (E2M1) or k <= 14 (E4M3) every
// flagged element is an exact tie x == B, whose answer is the even neighbour
// (round half to even).
template <int FMT, int WDT>
__device__ __forceinline__ bool tie_certified(int k_bits) {
  if (WDT == DT_F32 || FMT == FMT_INT4) return false;  // INT4: fp16 a and b give k up to 22
  if (fmt_e4m3(FMT)) return k_bits <= 14;
  return fmt_e2m1(FMT) ? k_bits <= 15 : k_bits <= 12;
}

// Exact fp64 decision for one element (factors outside the fast range).
template <int FMT>
__device__ __noinline__ float qexact64(float w, float a, float b, double sTd) {
  const double ab = ab_exact<FMT>(a, b, sTd);
  const float xt = (float)((double)w / ab);
  if (fmt_e2m1(FMT)) return q_e2m1<FMT>(xt, w, a, b, sTd);
  if (fmt_e4m3(FMT)) return q_e4m3<FMT>(xt, w, a, b, sTd);
  return q_int4<FMT>(xt, w, a, b, sTd);
}

// Fast requantization of the 8 elements (4 pairs u2 = W * cb) of a lane with
// block factor a; `near` is raised for a lane with an element too close to a
// rounding boundary (or factors outside the fast range).
template <int FMT>
__device__ __forceinline__ void req_fast(const f2 u2[4], float a, const ColState& cs, float& ia, bool& ok, f2 q2[4],
                                         bool& near, bool& tie) {
  ia = rcp_approx(a);
  // fp16 a (INT4) and E4M3 e (NVFP4) keep 1/a inside [2^-50, 2^50]; 2^k may not
  ok = cs.ok && (!fmt_pow2(FMT) || in_range(ia));
  near = !ok;
  tie = false;
  if (fmt_e2m1(FMT)) {
    const f2 ilo = splat(ia * (1.f - kRelGuard)), ihi = splat(ia * (1.f + kRelGuard));
    f2 lo[4], hi[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      lo[i] = mul2(u2[i], ilo);
      hi[i] = mul2(u2[i], ihi);
    }
    uint32_t clo, chi, h0, h1, h2, h3;
    asm("{\n.reg .b8 l0, l1, l2, l3, g0, g1, g2, g3;\n"
        "cvt.rn.satfinite.e2m1x2.f32 l0, %3, %2;\n"
        "cvt.rn.satfinite.e2m1x2.f32 l1, %5, %4;\n"
        "cvt.rn.satfinite.e2m1x2.f32 l2, %7, %6;\n"
        "cvt.rn.satfinite.e2m1x2.f32 l3, %9, %8;\n"
        "cvt.rn.satfinite.e2m1x2.f32 g0, %11, %10;\n"
        "cvt.rn.satfinite.e2m1x2.f32 g1, %13, %12;\n"
        "cvt.rn.satfinite.e2m1x2.f32 g2, %15, %14;\n"
        "cvt.rn.satfinite.e2m1x2.f32 g3, %17, %16;\n"
        "mov.b32 %0, {l0, l1, l2, l3};\n"
        "mov.b32 %1, {g0, g1, g2, g3};\n}"
        : "=r"(clo), "=r"(chi)
        : "f"(lo_of(lo[0])), "f"(hi_of(lo[0])), "f"(lo_of(lo[1])), "f"(hi_of(lo[1])), "f"(lo_of(lo[2])),
          "f"(hi_of(lo[2])), "f"(lo_of(lo[3])), "f"(hi_of(lo[3])), "f"(lo_of(hi[0])), "f"(hi_of(hi[0])),
          "f"(lo_of(hi[1])), "f"(hi_of(hi[1])), "f"(lo_of(hi[2])), "f"(hi_of(hi[2])), "f"(lo_of(hi[3])),
          "f"(hi_of(hi[3])));
    // The bracket codes differ only at elements within the bracket of a
    // boundary, where they are the two neighbours (adjacent codes, one of them
    // with an even mantissa bit).  On a tie-certified lane such an element is
    // an exact tie: keep the neighbour whose low code bit is 0.
    const uint32_t diff = clo ^ chi;
    const uint32_t tmask = cs.tie_ok ? 0xFFFFFFFFu : 0u;
    near |= (diff & ~tmask) != 0u;
    const uint32_t code = clo ^ (diff & ((clo & 0x11111111u) * 15u) & tmask);
    tie = (diff & tmask) != 0u;
    // each byte is extracted explicitly (cvt.u8.u32) before its decode
    asm("{\n.reg .b8 c0, c1, c2, c3;\n"
        "cvt.u8.u32 c0, %4;\n"
        "cvt.u8.u32 c1, %5;\n"
        "cvt.u8.u32 c2, %6;\n"
        "cvt.u8.u32 c3, %7;\n"
        "cvt.rn.f16x2.e2m1x2 %0, c0;\n"
        "cvt.rn.f16x2.e2m1x2 %1, c1;\n"
        "cvt.rn.f16x2.e2m1x2 %2, c2;\n"
        "cvt.rn.f16x2.e2m1x2 %3, c3;\n}"
        : "=r"(h0), "=r"(h1), "=r"(h2), "=r"(h3)
        : "r"(code & 0xFFu), "r"((code >> 8) & 0xFFu), "r"((code >> 16) & 0xFFu), "r"(code >> 24));
    const uint32_t hh[4] = {h0, h1, h2, h3};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&hh[i]));
      q2[i] = pk(f.x, f.y);
    }
  } else if (fmt_e4m3(FMT)) {
    // E4M3 codes of the bracket ends, four to a word; as for E2M1, differing
    // codes are neighbours, and a certified tie keeps the one whose low bit
    // (mantissa bit) is 0
    const f2 ilo = splat(ia * (1.f - kRelGuard)), ihi = splat(ia * (1.f + kRelGuard));
    const uint32_t tmask = cs.tie_ok ? 0xFFFFFFFFu : 0u;
    uint32_t anyd = 0u;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const uint32_t clo = cvt_e4m3x4(mul2(u2[2 * h], ilo), mul2(u2[2 * h + 1], ilo));
      const uint32_t chi = cvt_e4m3x4(mul2(u2[2 * h], ihi), mul2(u2[2 * h + 1], ihi));
      const uint32_t diff = clo ^ chi;
      anyd |= diff;
      dec_e4m3x4(clo ^ (diff & ((clo & 0x01010101u) * 0xFFu) & tmask), q2[2 * h], q2[2 * h + 1]);
    }
    near |= (anyd & ~tmask) != 0u;
    tie = (anyd & tmask) != 0u;
  } else {
    const f2 ia2 = splat(ia), nia2 = splat(-ia), m2 = splat(12582912.f), nm2 = splat(-12582912.f);
    bool flagged = false;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const f2 qu = add2(fma2(u2[i], ia2, m2), nm2);  // round half even
      const f2 r = fma2(u2[i], nia2, qu);             // qu - x~
      const float t0 = fmt_mxint(FMT) ? cs.thr[2 * i] : 0.5f - kGuard;
      const float t1 = fmt_mxint(FMT) ? cs.thr[2 * i + 1] : 0.5f - kGuard;
      flagged |= fabsf(lo_of(r)) > t0;
      flagged |= fabsf(hi_of(r)) > t1;
      q2[i] = pk(fminf(fmaxf(lo_of(qu), grid_lo(FMT)), grid_hi(FMT)),
                 fminf(fmaxf(hi_of(qu), grid_lo(FMT)), grid_hi(FMT)));
    }
    if (flagged && cs.tie_ok) {
      // certified exact ties x~ ~ n + 1/2: the even neighbour is 2 rint(x~ / 2)
      tie = true;
      const f2 hia2 = splat(0.5f * ia);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const f2 qu = add2(fma2(u2[i], ia2, m2), nm2);
        const f2 r = fma2(u2[i], nia2, qu);
        const f2 h = add2(fma2(u2[i], hia2, m2), nm2);
        const f2 qe = add2(h, h);
        const float t0 = fmt_mxint(FMT) ? cs.thr[2 * i] : 0.5f - kGuard;
        const float t1 = fmt_mxint(FMT) ? cs.thr[2 * i + 1] : 0.5f - kGuard;
        const float q0 = fabsf(lo_of(r)) > t0 ? lo_of(qe) : lo_of(qu);
        const float q1 = fabsf(hi_of(r)) > t1 ? hi_of(qe) : hi_of(qu);
        q2[i] = pk(fminf(fmaxf(q0, grid_lo(FMT)), grid_hi(FMT)), fminf(fmaxf(q1, grid_lo(FMT)), grid_hi(FMT)));
      }
    } else {
      near |= flagged;
    }
  }
}

// Exact settling of a flagged lane: re-derive which elements are close to a
// boundary and decide only those exactly (all 8 in fp64 when the factors are
// outside the fast range).
template <int FMT>
__device__ __forceinline__ void req_slow(const f2 w2[4], const f2 u2[4], float a, float ia, bool ok, const ColState& cs,
                                         float sT, double sTd, f2 q2[4]) {
  float q[8], w[8], u[8], b[8];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    q[2 * i] = lo_of(q2[i]);
    q[2 * i + 1] = hi_of(q2[i]);
    w[2 * i] = lo_of(w2[i]);
    w[2 * i + 1] = hi_of(w2[i]);
    u[2 * i] = lo_of(u2[i]);
    u[2 * i + 1] = hi_of(u2[i]);
    const f2 bi = col_ld(cs.tb, i);
    b[2 * i] = lo_of(bi);
    b[2 * i + 1] = hi_of(bi);
  }
  if (!ok) {
#pragma unroll
    for (int c = 0; c < 8; ++c) q[c] = qexact64<FMT>(w[c], a, b[c], sTd);
  } else if (fmt_e2m1(FMT)) {
    const float ilo = ia * (1.f - kRelGuard), ihi = ia * (1.f + kRelGuard);
#pragma unroll
    for (int c = 0; c < 8; c += 2) {
      const uint32_t lo = cvt_e2m1x2(u[c + 1] * ilo, u[c] * ilo);
      const uint32_t hi = cvt_e2m1x2(u[c + 1] * ihi, u[c] * ihi);
      const uint32_t diff = lo ^ hi;
      if (diff & 0x0Fu) q[c] = qexact32_e2m1(w[c], u[c], ia, a * b[c], sT);
      if (diff & 0xF0u) q[c + 1] = qexact32_e2m1(w[c + 1], u[c + 1], ia, a * b[c + 1], sT);
    }
  } else if (fmt_e4m3(FMT)) {
    const float ilo = ia * (1.f - kRelGuard), ihi = ia * (1.f + kRelGuard);
#pragma unroll
    for (int c = 0; c < 8; c += 4) {
      const uint32_t lo = cvt_e4m3x4(pk(u[c] * ilo, u[c + 1] * ilo), pk(u[c + 2] * ilo, u[c + 3] * ilo));
      const uint32_t hi = cvt_e4m3x4(pk(u[c] * ihi, u[c + 1] * ihi), pk(u[c + 2] * ihi, u[c + 3] * ihi));
      const uint32_t diff = lo ^ hi;
#pragma unroll
      for (int k = 0; k < 4; ++k)
        if ((diff >> (8 * k)) & 0xFFu) q[c + k] = qexact32_e4m3(w[c + k], u[c + k], ia, a * b[c + k]);
    }
  } else {
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const float qu = fmaf(u[c], ia, 12582912.f) - 12582912.f;
      const float thr = fmt_mxint(FMT) ? cs.thr[c] : 0.5f - kGuard;
      if (fabsf(fmaf(u[c], ia, -qu)) > thr) q[c] = qexact32_int<FMT>(w[c], u[c], ia, a * b[c]);
    }
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) q2[i] = pk(q[2 * i], q[2 * i + 1]);
}

// Requantize two rows of a lane (x = row a, y = row b) with block factors fa, fb.
template <int FMT>
__device__ __forceinline__ void req_pair(const f2 wx[4], const f2 ux[4], float fa, bool actx, const f2 wy[4],
                                         const f2 uy[4], float fb, bool acty, const ColState& cs, float sT, double sTd,
                                         f2 qx[4], f2 qy[4], unsigned* s_cnt, unsigned& tcnt) {
  float iax, iay;
  bool okx, oky, nx, ny, tx, ty;
  req_fast<FMT>(ux, fa, cs, iax, okx, qx, nx, tx);
  req_fast<FMT>(uy, fb, cs, iay, oky, qy, ny, ty);
  nx = nx && actx;
  ny = ny && acty;
  tcnt += (unsigned)(tx && actx) + (unsigned)(ty && acty);  // lane-rows settled as certified ties
  if (nx || ny) {
    if (nx) {
      atomicAdd(&s_cnt[0], 1u);
      req_slow<FMT>(wx, ux, fa, iax, okx, cs, sT, sTd, qx);
    }
    if (ny) {
      atomicAdd(&s_cnt[0], 1u);
      req_slow<FMT>(wy, uy, fb, iay, oky, cs, sT, sTd, qy);
    }
  }
}

// ---------------------------------------------------------------------------
// One row of W for one lane (8 elements as 4 pairs, exact fp32 values).
template <int WDT>
__device__ __forceinline__ void smem_row(const unsigned char* src, f2 w2[4]) {
  if (WDT == DT_F32) {
    const float4 x = *reinterpret_cast<const float4*>(src);
    const float4 y = *reinterpret_cast<const float4*>(src + 16);
    w2[0] = pk(x.x, x.y);
    w2[1] = pk(x.z, x.w);
    w2[2] = pk(y.x, y.y);
    w2[3] = pk(y.z, y.w);
  } else {
    const uint4 v = *reinterpret_cast<const uint4*>(src);
    const uint32_t uu[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      if (WDT == DT_BF16) {
        w2[i] = pk(__uint_as_float(uu[i] << 16), __uint_as_float(uu[i] & 0xFFFF0000u));
      } else {
        const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&uu[i]));
        w2[i] = pk(f.x, f.y);
      }
    }
  }
}

// Block sums and residuals of the incoming iterate for the two rows of a lane
// (x, y; an absent row holds zeros and adds nothing).  The residual W - a q b
// is taken with the product q b a exact inside fmas: q b is exact in fp32, and
// so is a for INT4/MX; the NVFP4 factor a = e s_T is split as hi + lo (hi =
// fl(e s_T), lo its exact rounding error), so the only rounding is that of the
// (small) residual itself.  With `scaled` the residual is multiplied by the
// power of two rscale before it is squared (a W whose max |W| is far from 1);
// otherwise its square cannot leave the fp32 range.
template <int FMT>
__device__ __forceinline__ void row_sums2(const f2 wx[4], const f2 qx[4], float ax, const f2 wy[4], const f2 qy[4],
                                          float ay, const ColState& cs, float sT, bool scaled, f2 rscale2, float& nx,
                                          float& dx, float& ny, float& dy, f2& res2) {
  const float axh = FMT == FMT_NVFP4 ? ax * sT : ax;
  const float ayh = FMT == FMT_NVFP4 ? ay * sT : ay;
  const f2 nax2 = splat(-axh), nay2 = splat(-ayh);
  const f2 nlox2 = splat(FMT == FMT_NVFP4 ? -fmaf(ax, sT, -axh) : 0.f);
  const f2 nloy2 = splat(FMT == FMT_NVFP4 ? -fmaf(ay, sT, -ayh) : 0.f);
  f2 nx2 = 0ull, dx2 = 0ull, ny2 = 0ull, dy2 = 0ull;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const f2 bi = col_ld(cs.tb, i);
    const f2 px = mul2(qx[i], bi), py = mul2(qy[i], bi);
    nx2 = fma2(wx[i], px, nx2);
    dx2 = fma2(px, px, dx2);
    ny2 = fma2(wy[i], py, ny2);
    dy2 = fma2(py, py, dy2);
    f2 rx = fma2(px, nax2, wx[i]), ry = fma2(py, nay2, wy[i]);
    if (FMT == FMT_NVFP4) {
      rx = fma2(px, nlox2, rx);
      ry = fma2(py, nloy2, ry);
    }
    if (scaled) {
      rx = mul2(rx, rscale2);
      ry = mul2(ry, rscale2);
    }
    res2 = fma2(rx, rx, res2);
    res2 = fma2(ry, ry, res2);
  }
  nx = lo_of(nx2) + hi_of(nx2);
  dx = lo_of(dx2) + hi_of(dx2);
  ny = lo_of(ny2) + hi_of(ny2);
  dy = lo_of(dy2) + hi_of(dy2);
}

// Exact fp64 block sums of one row of one lane (warp-collective reduction).
__device__ __forceinline__ void row_sums64(const f2 w2[4], const f2 q2[4], const ColState& cs, int lpb, double& n64,
                                           double& d64) {
  n64 = 0.0;
  d64 = 0.0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const f2 pq = mul2(q2[i], col_ld(cs.tb, i));  // exact products
    n64 = fma((double)lo_of(w2[i]), (double)lo_of(pq), n64);
    d64 = fma((double)lo_of(pq), (double)lo_of(pq), d64);
    n64 = fma((double)hi_of(w2[i]), (double)hi_of(pq), n64);
    d64 = fma((double)hi_of(pq), (double)hi_of(pq), d64);
  }
  for (int o = 1; o < lpb; o <<= 1) {
    n64 += __shfl_xor_sync(0xffffffffu, n64, o);
    d64 += __shfl_xor_sync(0xffffffffu, d64, o);
  }
}

// The 8 codes of a lane's row.  Integer grids: q + 1.5 * 2^23 holds q in the
// low mantissa bits (two's complement).  INT8 and E4M3 grids: one byte per
// code, column order from the low byte of .x to the high byte of .y (E4M3:
// the bit pattern, zero as 0x00).  Other grids: packed
// nibbles in .x (even column in the low nibble; zero is always the 0x0
// nibble), .y = 0.
template <int FMT>
__device__ __forceinline__ uint2 pack8(const f2 q2[4]) {
  uint2 r = make_uint2(0u, 0u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float lo = __fadd_rn(lo_of(q2[i]), 0.f), hi = __fadd_rn(hi_of(q2[i]), 0.f);  // -0 becomes +0
    if (fmt_e4m3(FMT)) {  // grid values convert exactly; zero is always 0x00
      if (i & 1) {
        const uint32_t four = cvt_e4m3x4(pk(__fadd_rn(lo_of(q2[i - 1]), 0.f), __fadd_rn(hi_of(q2[i - 1]), 0.f)),
                                         pk(lo, hi));
        if (i == 1) {
          r.x = four;
        } else {
          r.y = four;
        }
      }
    } else if (fmt_byte_codes(FMT)) {
      const uint32_t two = (__float_as_uint(lo + 12582912.f) & 255u) | ((__float_as_uint(hi + 12582912.f) & 255u) << 8);
      if (i < 2) {
        r.x |= two << (16 * i);
      } else {
        r.y |= two << (16 * (i - 2));
      }
    } else {
      uint32_t byte;
      if (fmt_e2m1(FMT)) {
        byte = cvt_e2m1x2(hi, lo);  // grid values convert exactly
      } else {
        byte = (__float_as_uint(lo + 12582912.f) & 15u) | ((__float_as_uint(hi + 12582912.f) & 15u) << 4);
      }
      r.x |= byte << (8 * i);
    }
  }
  return r;
}

// Number of codes that differ, for x = new ^ old (nonzero bytes or nibbles).
template <int FMT>
__device__ __forceinline__ uint32_t changed_codes(uint2 x) {
  if (fmt_byte_codes(FMT)) {
    x.x |= x.x >> 1;
    x.x |= x.x >> 2;
    x.x |= x.x >> 4;
    x.y |= x.y >> 1;
    x.y |= x.y >> 2;
    x.y |= x.y >> 4;
    return (uint32_t)(__popc(x.x & 0x01010101u) + __popc(x.y & 0x01010101u));
  }
  x.x |= x.x >> 1;
  x.x |= x.x >> 2;
  return (uint32_t)__popc(x.x & 0x11111111u);
}

// The code group (8 codes) at index cix: a 32-bit word, or 8 bytes for the
// INT8 grid.  Codes are rewritten inside the kernel: loads go through L2.
template <int FMT>
__device__ __forceinline__ uint2 load_codes(const void* codes, int64_t cix) {
  if (fmt_byte_codes(FMT)) return __ldcg(reinterpret_cast<const uint2*>(codes) + cix);
  return make_uint2(__ldcg(reinterpret_cast<const uint32_t*>(codes) + cix), 0u);
}

template <int FMT>
__device__ __forceinline__ void store_codes(void* codes, int64_t cix, uint2 c) {
  if (fmt_byte_codes(FMT)) {
    reinterpret_cast<uint2*>(codes)[cix] = c;
  } else {
    reinterpret_cast<uint32_t*>(codes)[cix] = c.x;
  }
}

// Code tracking for two rows of a lane: the codes replace the groups at cix
// (row x) and cix + code_step (row y); with `cmp` the codes that differ from
// the previous groups oldx, oldy are counted into nchg.
template <int FMT>
__device__ __forceinline__ void track_codes(const Problem& p, const f2 qx[4], const f2 qy[4], bool actx, bool acty,
                                            int64_t cix, int64_t code_step, uint2 oldx, uint2 oldy, bool cmp,
                                            unsigned& nchg) {
  if (actx) {
    const uint2 c = pack8<FMT>(qx);
    if (cmp) nchg += changed_codes<FMT>(make_uint2(c.x ^ oldx.x, c.y ^ oldx.y));
    store_codes<FMT>(p.codes, cix, c);
  }
  if (acty) {
    const uint2 c = pack8<FMT>(qy);
    if (cmp) nchg += changed_codes<FMT>(make_uint2(c.x ^ oldy.x, c.y ^ oldy.y));
    store_codes<FMT>(p.codes, cix + code_step, c);
  }
}

// Two rows of one lane (x = row a, y = row b; a row outside the segment holds
// zeros and nothing of it is written): requantize the incoming iterate; block
// sums, residuals and block updates; requantize with the new block scales
// where they changed; column sums.  Warp-collective (shuffles and votes);
// actx / acty say which of the lane's rows are real.  achg is raised when a
// block scale of the lane's rows changed.
template <int FMT, int PASS>
__device__ __forceinline__ void row_pair(const Problem& p, const f2 wx[4], float ax_old, int64_t bidx_x,
                                         const f2 wy[4], float ay_old, int64_t bidx_y, bool actx, bool acty,
                                         bool leader, int lpb, ColState& cs, float sT, float isT, double sTd,
                                         bool scaled, f2 rscale2, unsigned* s_cnt, unsigned& tcnt, int64_t cix,
                                         int64_t code_step, uint2 oldx, uint2 oldy, bool cmp, unsigned& nchg,
                                         bool& achg) {
  f2 ux[4], uy[4], qx[4], qy[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const f2 cbi = col_ld(cs.tcb, i);
    ux[i] = mul2(wx[i], cbi);
    uy[i] = mul2(wy[i], cbi);
  }
  req_pair<FMT>(wx, ux, ax_old, actx, wy, uy, ay_old, acty, cs, sT, sTd, qx, qy, s_cnt, tcnt);
  if (PASS == PASS_COUNT) track_codes<FMT>(p, qx, qy, actx, acty, cix, code_step, oldx, oldy, cmp, nchg);
  float nx, dx, ny, dy;
  row_sums2<FMT>(wx, qx, ax_old, wy, qy, ay_old, cs, sT, scaled, rscale2, nx, dx, ny, dy, cs.res2);
  float anx, any;
  if (p.mode == DQ_MODE_COL) {  // column scales only: the block scales keep their values
    anx = ax_old;
    any = ay_old;
  } else if (lpb == 1) {  // a block within one lane: both rows here
    bool ambx = false, amby = false;
    anx = a_fast<FMT>(nx, dx, isT, ambx);
    any = a_fast<FMT>(ny, dy, isT, amby);
    ambx = ambx && actx;
    amby = amby && acty;
    if (__any_sync(0xffffffffu, ambx || amby)) {
      double n64, d64;
      row_sums64(wx, qx, cs, lpb, n64, d64);
      if (ambx) {
        atomicAdd(&s_cnt[1], 1u);
        anx = d64 == 0.0 ? 1.f : (float)a_project<FMT>(n64 / d64, sTd);
      }
      row_sums64(wy, qy, cs, lpb, n64, d64);
      if (amby) {
        atomicAdd(&s_cnt[1], 1u);
        any = d64 == 0.0 ? 1.f : (float)a_project<FMT>(n64 / d64, sTd);
      }
    }
  } else {
    // the lanes of a block split the two rows: even lanes finish row x, odd
    // lanes row y (one reduce-scatter step, then the usual xor tree), so each
    // lane projects one block value; the partner's result comes back by shuffle
    const bool odd = (cs.lane & 1) != 0;
    float kn = odd ? ny : nx, kd = odd ? dy : dx;
    kn += __shfl_xor_sync(0xffffffffu, odd ? nx : ny, 1);
    kd += __shfl_xor_sync(0xffffffffu, odd ? dx : dy, 1);
    for (int o = 2; o < lpb; o <<= 1) {
      kn += __shfl_xor_sync(0xffffffffu, kn, o);
      kd += __shfl_xor_sync(0xffffffffu, kd, o);
    }
    bool amb = false;
    float an = a_fast<FMT>(kn, kd, isT, amb);
    amb = amb && (odd ? acty : actx);
    if (__any_sync(0xffffffffu, amb)) {
      double n64x, d64x, n64y, d64y;
      row_sums64(wx, qx, cs, lpb, n64x, d64x);
      row_sums64(wy, qy, cs, lpb, n64y, d64y);
      if (amb) {
        if ((cs.lane & (lpb - 1)) <= 1) atomicAdd(&s_cnt[1], 1u);  // once per block row
        const double n64 = odd ? n64y : n64x, d64 = odd ? d64y : d64x;
        an = d64 == 0.0 ? 1.f : (float)a_project<FMT>(n64 / d64, sTd);
      }
    }
    const float ao = __shfl_xor_sync(0xffffffffu, an, 1);
    anx = odd ? ao : an;
    any = odd ? an : ao;
  }
  // the storage already holds the old factors; with a block scale unchanged the
  // codes are unchanged too (same a, same b), so requantize only where it changed
  const bool chx = anx != ax_old && actx, chy = any != ay_old && acty;
  achg = achg || chx || chy;
  if (chx && leader) a_store_f<FMT>(p.a_work, bidx_x, anx);
  if (chy && leader) a_store_f<FMT>(p.a_work, bidx_y, any);
  if (__any_sync(0xffffffffu, chx || chy)) {
    // recomputed rather than kept live across the block update (registers)
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const f2 cbi = col_ld(cs.tcb, i);
      ux[i] = mul2(wx[i], cbi);
      uy[i] = mul2(wy[i], cbi);
    }
    req_pair<FMT>(wx, ux, anx, actx, wy, uy, any, acty, cs, sT, sTd, qx, qy, s_cnt, tcnt);
  }
  const f2 anx2 = splat(anx), any2 = splat(any);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const f2 svx = mul2(qx[i], anx2);  // exact; NVFP4 leaves s_T out
    const f2 svy = mul2(qy[i], any2);
    cs.cn2[i] = fma2(wx[i], svx, cs.cn2[i]);
    cs.cd2[i] = fma2(svx, svx, cs.cd2[i]);
    cs.cn2[i] = fma2(wy[i], svy, cs.cn2[i]);
    cs.cd2[i] = fma2(svy, svy, cs.cd2[i]);
  }
}

// Final pass for two rows of a lane (x, y; a row outside the segment holds
// zeros and is not written): codes of the final iterate, written packed, and
// the residuals of that iterate for its MSE.
template <int FMT>
__device__ __forceinline__ void final_pair(const Problem& p, const f2 wx[4], float ax, const f2 wy[4], float ay,
                                           bool actx, bool acty, ColState& cs, float sT, double sTd, bool scaled,
                                           f2 rscale2, unsigned* s_cnt, unsigned& tcnt, int64_t cix,
                                           int64_t code_step, uint2 oldx, uint2 oldy, bool cmp, unsigned& nchg) {
  f2 ux[4], uy[4], qx[4], qy[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const f2 cbi = col_ld(cs.tcb, i);
    ux[i] = mul2(wx[i], cbi);
    uy[i] = mul2(wy[i], cbi);
  }
  req_pair<FMT>(wx, ux, ax, actx, wy, uy, ay, acty, cs, sT, sTd, qx, qy, s_cnt, tcnt);
  float nx, dx, ny, dy;  // block sums: not needed here
  row_sums2<FMT>(wx, qx, ax, wy, qy, ay, cs, sT, scaled, rscale2, nx, dx, ny, dy, cs.res2);
  track_codes<FMT>(p, qx, qy, actx, acty, cix, code_step, oldx, oldy, cmp, nchg);
}

// fp32 runs into the warp's fp64 accumulators (layout [warp][c][lane], then
// [warp][lane] for the residuals).
__device__ __forceinline__ void flush_runs(ColState& cs, double2* acc, double* racc, int warp, int lane,
                                           bool active) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      double2& a = acc[(warp * 8 + 2 * i + h) * 32 + lane];
      double2 v = a;
      v.x += (double)(h ? hi_of(cs.cn2[i]) : lo_of(cs.cn2[i]));
      v.y += (double)(h ? hi_of(cs.cd2[i]) : lo_of(cs.cd2[i]));
      a = v;
    }
    cs.cn2[i] = cs.cd2[i] = 0ull;
  }
  if (active) racc[warp * 32 + lane] += (double)lo_of(cs.res2) + (double)hi_of(cs.res2);
  cs.res2 = 0ull;
}

// ---------------------------------------------------------------------------
// Grid-wide barrier of the consumer threads of every CTA.  k_iter is launched
// cooperatively, so all its CTAs are resident at once.  Arrivals are counted
// in hdr->gbar over the whole solve; a use waits for the next multiple of the
// grid size.  The wait is bounded: it gives up after kWaitLimitNs of wall
// time (or at once when some wait already gave up), records kFlagTimeout and
// goes on.
// MSE of a finished pass from its n partial residual totals `part` (one per
// CTA, or one per block-column): a fixed-order tree over the index, so the
// value does not depend on which CTA sums it.  Run by the consumer threads of
// one CTA; `red` holds kConsumers doubles.
__device__ void mse_total(const Problem& p, const double* part, int64_t n, double* out, double rscale_d,
                          double* red) {
  double v = 0.0;
  for (int64_t kk = threadIdx.x; kk < n; kk += kConsumers) v += __ldcg(part + kk);
  red[threadIdx.x] = v;
  consumer_sync(kConsumers);
  for (int o = kConsumerTreeTop; o > 0; o >>= 1) {
    if (threadIdx.x < o && threadIdx.x + o < kConsumers) red[threadIdx.x] += red[threadIdx.x + o];
    consumer_sync(kConsumers);
  }
  if (threadIdx.x == 0) *out = red[0] / (rscale_d * rscale_d) / ((double)p.M * (double)p.N);
  consumer_sync(kConsumers);
}

// Per-CTA residual totals of the final pass t live in cta_part[(t % 3) P + k].
__device__ __forceinline__ double* mse_part(const Problem& p, int t) { return p.cta_part + (int64_t)(t % 3) * p.P; }

// Residual total of each block-column for the incoming iterate of BCD pass t:
// mse_bc[(t % 3) nb + g].  Three buffers, so the totals of pass t - 1 stay
// intact while pass t + 1 runs (the MSE of pass t - 1 is summed during pass t).
__device__ __forceinline__ double* mse_bcs(const Problem& p, int t) { return p.mse_bc + (int64_t)(t % 3) * p.nb; }

// Grid barrier at the end of pass t.  The first CTA to arrive has the most
// time to spare: it sums the MSE of pass t - 1 (all of whose block-column
// totals were written before the barrier that ended it) while the others
// finish.
__device__ void grid_sync(const Problem& p, int t, double rscale_d, double* red, int* s_flag) {
  WsHeader* hdr = p.hdr;
  consumer_sync(kConsumers);
  unsigned target = 0u;
  if (threadIdx.x == 0) {
    __threadfence();
    const unsigned ticket = atomicAdd(&hdr->gbar, 1u);
    target = (ticket / gridDim.x + 1u) * gridDim.x;
    *s_flag = (ticket % gridDim.x == 0u && t >= 2) ? 1 : 0;
  }
  consumer_sync(kConsumers);
  if (*s_flag) mse_total(p, mse_bcs(p, t - 1), p.nb, p.mse + (t - 2), rscale_d, red);
  if (threadIdx.x == 0) {
    const unsigned long long t0 = global_ns();
    for (;;) {
      if ((int)(ld_acquire_gpu(&hdr->gbar) - target) >= 0) break;
      if (wait_expired(&hdr->flags, t0)) break;
      __nanosleep(64);
    }
    __threadfence();
  }
  consumer_sync(kConsumers);
}

// Plain grid barrier (no MSE duty).
__device__ void grid_sync_plain(WsHeader* hdr) {
  consumer_sync(kConsumers);
  if (threadIdx.x == 0) {
    __threadfence();
    const unsigned ticket = atomicAdd(&hdr->gbar, 1u);
    const unsigned target = (ticket / gridDim.x + 1u) * gridDim.x;
    const unsigned long long t0 = global_ns();
    for (;;) {
      if ((int)(ld_acquire_gpu(&hdr->gbar) - target) >= 0) break;
      if (wait_expired(&hdr->flags, t0)) break;
      __nanosleep(64);
    }
    __threadfence();
  }
  consumer_sync(kConsumers);
}

constexpr int kXRows = 8;

// Exact column sums by one warp of a group of `nw` warps sharing the column:
// fp64 sums of W a q and (a q)^2 of column j over rows i_begin + 32 wi + lane,
// + 32 nw, ... below i_end (wi: the warp's index in the group; 8 loads in
// flight each), with q decided exactly, added over the lanes in a fixed xor
// tree; every lane returns the warp's totals.
template <int FMT, int WDT>
__device__ double2 column_rows_exact_warp(const Problem& p, int64_t j, int64_t i_begin, int64_t i_end, int wi, int nw,
                                          double sTd, float isT) {
  const int lane = threadIdx.x & 31;
  const int64_t step = (int64_t)32 * nw;
  const unsigned short braw = __ldcg(reinterpret_cast<const unsigned short*>(p.b_store) + j);
  const float bj = p.col_dt == DT_F16 ? __half2float(__ushort_as_half(braw)) : __uint_as_float((uint32_t)braw << 16);
  const float cb = __frcp_rn(bj) * isT;
  const int64_t jb = j / p.G;  // block column
  double cn = 0.0, cd = 0.0;
  for (int64_t i0 = i_begin + 32 * wi + lane; i0 < i_end; i0 += (int64_t)kXRows * step) {
    float w[kXRows];
    uint32_t araw[kXRows];
#pragma unroll
    for (int k = 0; k < kXRows; ++k) {
      const int64_t i = i0 + (int64_t)k * step;
      w[k] = 0.f;
      araw[k] = a_raw_one<FMT>();
      if (i < i_end) {
        const int64_t e = i * p.N + j;
        if (WDT == DT_F32) {
          w[k] = __ldg(reinterpret_cast<const float*>(p.W) + e);
        } else if (WDT == DT_BF16) {
          w[k] = __uint_as_float((uint32_t)__ldg(reinterpret_cast<const unsigned short*>(p.W) + e) << 16);
        } else {
          w[k] = __half2float(__ushort_as_half(__ldg(reinterpret_cast<const unsigned short*>(p.W) + e)));
        }
        araw[k] = a_fetch<FMT>(p.a_work, jb * p.M + i);
      }
    }
#pragma unroll
    for (int k = 0; k < kXRows; ++k) {  // absent rows hold w = 0, which adds nothing
      const float a = a_dec<FMT>(araw[k]);
      const float ia = __frcp_rn(a);
      const bool ok = in_range(cb) && in_range(ia);
      const float q = quant<FMT>(w[k], w[k] * cb, ia, ok, a, bj, sTd);
      const double sv = (double)q * (double)a;
      cn = fma((double)w[k], sv, cn);
      cd = fma(sv, sv, cd);
    }
  }
  for (int o = 16; o > 0; o >>= 1) {
    cn += __shfl_xor_sync(0xffffffffu, cn, o);
    cd += __shfl_xor_sync(0xffffffffu, cd, o);
  }
  return make_double2(cn, cd);
}

// Bounded wait of thread 0 until *c reaches `target` (ld.acquire; gives up
// with kFlagTimeout after kWaitLimitNs).  The caller synchronizes the CTA
// afterwards, which orders the other threads' later loads after the acquire.
__device__ void wait_count(unsigned* c, unsigned target, unsigned* flags) {
  if (threadIdx.x == 0) {
    const unsigned long long t0 = global_ns();
    for (;;) {
      if ((int)(ld_acquire_gpu(c) - target) >= 0) break;
      if (wait_expired(flags, t0)) break;
      __nanosleep(64);
    }
  }
}

// Sum of the column partials (sum W a q, sum (a q)^2) of strip column vc over
// the CTAs kb0 .. kb1-1 of strip v, in CTA order, 4 loads in flight.
__device__ __forceinline__ double2 col_total(const Problem& p, int vc, int64_t v, int64_t kb0, int64_t kb1,
                                             const int* s_sfirst) {
  double2 tot = make_double2(0.0, 0.0);
  for (int64_t kb = kb0; kb < kb1; kb += 4) {
    double2 x[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int64_t kk = kb + q;
      x[q] = make_double2(0.0, 0.0);
      if (kk < kb1) x[q] = __ldcg(&p.col_part[(kk * p.segmax + (v - s_sfirst[kk])) * p.TSv + vc]);
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      tot.x += x[q].x;
      tot.y += x[q].y;
    }
  }
  return tot;
}

// Finalization of the strip slots w = w0, w0 + step, ... < nbc of strip v in
// pass t, by the consumer threads of one CTA, once all K CTAs of the strip
// (k_first ..) have written their partial sums; slots are taken in groups whose
// loads are all issued together.  For each column: its totals from the K CTAs
// (sp threads per column, each adding a contiguous slice in CTA order, the
// slices then added in slice order) and the certified projection of its new
// scale; a column whose projection is ambiguous is added to the strip's list
// (strip column index) for the exact update that follows, and its block-column
// counts as changed.  For each slot: its block-column's residual total (in CTA
// order) and change flag.  `scr` is scratch shared memory of at least 2048
// doubles; `ctab` the CTA's column tables of the strip (its last segment),
// which hold the old scales.
template <int FMT>
__device__ void finalize_slots(const Problem& p, int t, int64_t v, int w0, int step, int nbc, const int* act,
                               bool ident, int i0, int64_t k_first, int K, const int* s_sfirst, double sTd,
                               double* scr, const f2* ctab, int* amb_list, unsigned* amb_cnt, int* s_chg) {
  const int G = p.G;
  const bool cols = p.mode != DQ_MODE_ROW;  // in the row mode b keeps its values
  const int nw_all = w0 < nbc ? (nbc - w0 + step - 1) / step : 0;
  const int grp_max = max(1, kConsumers / G);
  for (int g0 = 0; g0 < nw_all; g0 += grp_max) {
    const int nw = min(grp_max, nw_all - g0);
    const int sp = max(1, min(min(K, 16), kConsumers / (G * nw)));
    double* mpart = scr;                                                          // [nw][K]
    double2* cpart = reinterpret_cast<double2*>(scr + ((nw * K + 1) & ~1));      // [nw][sp][G]
    if (threadIdx.x < nw) s_chg[threadIdx.x] = 0;
    for (int e = threadIdx.x; e < nw * K; e += kConsumers) {
      const int iw = e / K;
      const int w = w0 + (g0 + iw) * step;
      const int64_t kk = k_first + (e - iw * K);
      mpart[e] = __ldcg(&p.mse_seg[(kk * p.segmax + (v - s_sfirst[kk])) * kBcPerStrip + w]);
    }
    if (cols) {
      for (int e = threadIdx.x; e < nw * sp * G; e += kConsumers) {
        const int iw = e / (sp * G), rem = e - iw * (sp * G), part = rem / G, c = rem - part * G;
        const int w = w0 + (g0 + iw) * step;
        cpart[e] = col_total(p, w * G + c, v, k_first + (int64_t)part * K / sp,
                             k_first + (int64_t)(part + 1) * K / sp, s_sfirst);
      }
    }
    consumer_sync(kConsumers);
    if (cols) {
      for (int e = threadIdx.x; e < nw * G; e += kConsumers) {
        const int iw = e / G, c = e - iw * G;
        const int w = w0 + (g0 + iw) * step;
        double2 tot = cpart[iw * sp * G + c];
        for (int part = 1; part < sp; ++part) {
          const double2 x = cpart[(iw * sp + part) * G + c];
          tot.x += x.x;
          tot.y += x.y;
        }
        const int64_t j = (int64_t)(ident ? i0 + w : act[i0 + w]) * G + c;
        // certified only when the fp32 runs stayed well inside the normal range
        // (no overflow; underflowed terms negligible); a zero total may be
        // underflow and is settled exactly as well
        const bool safe = tot.x >= 0x1p-60 && tot.x <= 0x1p100 && tot.y >= 0x1p-60 && tot.y <= 0x1p100;
        const double ratio = FMT == FMT_NVFP4 ? (tot.x / tot.y) / sTd : tot.x / tot.y;
        const double lo = safe ? b_project(ratio * (1.0 - col_err<FMT>()), p.col_dt) : 0.0;
        const double hi = safe ? b_project(ratio * (1.0 + col_err<FMT>()), p.col_dt) : 1.0;
        // the old scale: this CTA's column table of the strip (warp w, octet
        // c / 8, pair (c % 8) / 2), loaded when its segment of the strip began
        const f2 bp = ctab[w * 8 * (G / 8) + (c >> 3) * 4 + ((c & 7) >> 1)];
        const double bold = (double)((c & 1) ? hi_of(bp) : lo_of(bp));
        if (lo == hi) {
          if (lo != bold) {
            b_encode(p.b_store, p.col_dt, j, lo);
            s_chg[iw] = 1;
          }
        } else {
          amb_list[atomicAdd(amb_cnt, 1u)] = w * G + c;  // b keeps its value until the exact update
          s_chg[iw] = 1;
        }
      }
      consumer_sync(kConsumers);
    }
    for (int iw = threadIdx.x; iw < nw; iw += kConsumers) {
      const int w = w0 + (g0 + iw) * step;
      const int gw = ident ? i0 + w : act[i0 + w];
      double m = 0.0;  // the block-column's residual total, in CTA order
      for (int kq = 0; kq < K; ++kq) m += mpart[iw * K + kq];
      mse_bcs(p, t)[gw] = m;
      if (s_chg[iw]) p.chg[(int64_t)(t % 3) * p.nb + gw] = 1u;
    }
    consumer_sync(kConsumers);  // the scratch is reused
  }
}

// Exact update of the columns of strip v listed as ambiguous (amb_list[0 ..
// n)), shared by the nfin finalizing CTAs of the strip: finalizer q sums the
// columns exactly (fp64, exact grid decisions) over rows [q M / nfin,
// (q+1) M / nfin) and stores the two sums in its own partial slot `myslot` of
// the strip (whose values every finalizer has read by now); the last of them
// to finish adds the nfin sums of each column in finalizer order and writes
// the projected scale.  `red` holds 3 kConsumers doubles; s_flag one int.
template <int FMT, int WDT>
__device__ void exact_columns(const Problem& p, int64_t v, const int* act, bool ident, int i0_strip, int q, int nfin,
                              int64_t k_first, int64_t myslot, const int* s_sfirst, const int* amb_list, int n,
                              unsigned* ticket, double sTd, float isT, double* red, int* s_flag, unsigned* s_cnt) {
  const int G = p.G;
  const int64_t lo = (int64_t)q * p.M / nfin, hi = (int64_t)(q + 1) * p.M / nfin;
  // the 15 warps are shared evenly by the listed columns (all of them on one
  // column when it is the only one), so each column's rows take about one
  // round of loads; the warps' sums of a column are added in warp order
  const int warp = threadIdx.x >> 5;
  const int wpc = max(1, kConsumerWarps / n);     // warps per column
  const int ncw = kConsumerWarps / wpc;           // columns handled at once
  double2* wsum = reinterpret_cast<double2*>(red);  // [kConsumerWarps]
  for (int i0 = 0; i0 < n; i0 += ncw) {
    const int i = i0 + warp / wpc, wi = warp % wpc;
    const bool mine = warp < ncw * wpc && i < n;
    double2 s2 = make_double2(0.0, 0.0);
    int vc = 0;
    if (mine) {
      vc = __ldcg(amb_list + i);
      const int w = vc / G;
      const int64_t j = (int64_t)(ident ? i0_strip + w : act[i0_strip + w]) * G + (vc - w * G);
      s2 = column_rows_exact_warp<FMT, WDT>(p, j, lo, hi, wi, wpc, sTd, isT);
    }
    if ((threadIdx.x & 31) == 0) wsum[warp] = s2;
    consumer_sync(kConsumers);
    if (mine && wi == 0 && (threadIdx.x & 31) == 0) {
      double2 tot = wsum[warp];
      for (int k = 1; k < wpc; ++k) {
        tot.x += wsum[warp + k].x;
        tot.y += wsum[warp + k].y;
      }
      p.col_part[myslot * p.TSv + vc] = tot;
    }
    consumer_sync(kConsumers);  // wsum is reused
  }
  if (threadIdx.x == 0) {
    __threadfence();
    *s_flag = atomicAdd(ticket, 1u) == (unsigned)nfin - 1u ? 1 : 0;
  }
  consumer_sync(kConsumers);
  if (*s_flag == 0) return;
  __threadfence();
  // every share of every listed column loaded at once (into the idle column
  // accumulators, 2 kConsumers doubles), then each column's shares added in
  // finalizer order
  double2* sh = reinterpret_cast<double2*>(red) + kConsumers;
  for (int i0 = 0; i0 < n; i0 += max(1, kConsumers / nfin)) {
    const int nc = min(n - i0, max(1, kConsumers / nfin));
    for (int e = threadIdx.x; e < nc * nfin; e += kConsumers) {
      const int i = e / nfin, qq = e - i * nfin;
      const int vc = __ldcg(amb_list + i0 + i);
      const int64_t kk = k_first + qq;
      sh[e] = __ldcg(&p.col_part[(kk * p.segmax + (v - s_sfirst[kk])) * p.TSv + vc]);
    }
    consumer_sync(kConsumers);
    for (int i = threadIdx.x; i < nc; i += kConsumers) {
      const int vc = __ldcg(amb_list + i0 + i);
      const int w = vc / G;
      const int64_t j = (int64_t)(ident ? i0_strip + w : act[i0_strip + w]) * G + (vc - w * G);
      double tn = 0.0, td = 0.0;
      for (int qq = 0; qq < nfin; ++qq) {
        tn += sh[i * nfin + qq].x;
        td += sh[i * nfin + qq].y;
      }
      const double r = FMT == FMT_NVFP4 ? (tn / td) / sTd : tn / td;
      const double bnew = td == 0.0 ? 1.0 : b_project(r, p.col_dt);
      if (bnew != (double)b_decode_cg(p.b_store, p.col_dt, j)) b_encode(p.b_store, p.col_dt, j, bnew);
    }
    consumer_sync(kConsumers);
  }
  if (threadIdx.x == 0) s_cnt[2] += (unsigned)n;
}

// True when a strip's nbc block-columns g_first .. g_last are consecutive and
// W has the 3-D tensor map: then one tensor copy brings a whole tile.
__device__ __forceinline__ bool strip_contiguous(const Problem& p, bool ident, int g_first, int g_last, int nbc) {
  return p.use_tmap3 && (ident || g_last - g_first == nbc - 1);
}

// Named barrier of the whole CTA (consumers and producer): the schedule of a
// pass is handed to the producer through it.
__device__ __forceinline__ void cta_sync_all() { asm volatile("bar.sync 2, %0;" ::"r"(kIterThreads) : "memory"); }

// Schedule of pass t, computed by the consumer threads of every CTA from the
// same flags (so every CTA finds the same strips and ranges): the active
// block-columns, this CTA's units and this CTA's slice of the active list.  With `ident` (the first BCD pass and the final pass) every
// block-column is active.  Otherwise the active ones are those whose scales
// changed in pass t - 1 (p.chg of pass t - 1, complete after the grid barrier
// that ended it): a block-column with no change is at a fixed point, and its
// residual total is carried into this pass's buffer.  `s_scan` holds 17 ints.
__device__ void pass_schedule(const Problem& p, int t, bool ident, Sched* sc, int* s_act, int* s_scan) {
  const int nb = p.nb;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const unsigned* flags = p.chg + (int64_t)((t - 1) % 3) * nb;
  const int per = (nb + kConsumers - 1) / kConsumers;
  const int c0 = min(nb, tid * per), c1 = min(nb, c0 + per);
  int nact = nb, excl = 0;
  uint32_t mask = 0u;  // this thread's flags (per <= 32)
  if (!ident) {
    int cnt = 0;
    for (int g = c0; g < c1; ++g) {
      const bool f = __ldcg(flags + g) != 0u;
      cnt += f;
      if (per <= 32) mask |= (uint32_t)f << (g - c0);
    }
    int incl = cnt;
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (lane == 31) s_scan[warp] = incl;
    consumer_sync(kConsumers);
    if (warp == 0) {
      const int x = lane < kConsumerWarps ? s_scan[lane] : 0;
      int xi = x;
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, xi, o);
        if (lane >= o) xi += y;
      }
      if (lane < kConsumerWarps) s_scan[lane] = xi - x;
      if (lane == 31) s_scan[16] = xi;
    }
    consumer_sync(kConsumers);
    excl = s_scan[warp] + incl - cnt;
    nact = s_scan[16];
  }
  const long long nv = ((long long)nact + kBcPerStrip - 1) / kBcPerStrip;
  const long long L = nv * p.M;
  const int Pt = pass_ctas(p.P, nv, L);
  const int k = blockIdx.x;
  const long long ub = k < Pt ? range_begin(k, Pt, L) : L;
  const long long ue = k < Pt ? range_begin(k + 1, Pt, L) : L;
  const int v_first = (int)(ub / p.M);
  if (!ident) {
    const long long lo = (long long)v_first * kBcPerStrip;
    const long long hi = lo + (long long)p.segmax * kBcPerStrip;
    double* cur = mse_bcs(p, t);
    const double* prev = mse_bcs(p, t - 1);
    int idx = excl;
    for (int g = c0; g < c1; ++g) {
      if (per <= 32 ? ((mask >> (g - c0)) & 1u) != 0u : __ldcg(flags + g) != 0u) {
        if (idx >= lo && idx < hi) s_act[idx - lo] = g;
        ++idx;
      } else if (g % (int)gridDim.x == k) {
        cur[g] = __ldcg(prev + g);  // at a fixed point: the same residual total
      }
    }
  }
  if (tid == 0) {
    sc->L = L;
    sc->u_begin = ub;
    sc->u_end = ue;
    sc->nact = nact;
    sc->Pt = Pt;
    sc->v_first = v_first;
    sc->ident = ident ? 1 : 0;
  }
  consumer_sync(kConsumers);
}

// Passes t = t_first .. t_last, in one persistent launch (cooperative: a grid
// barrier separates consecutive passes, so pass t + 1 reads the scales that
// pass t wrote).  PASS_ITER: BCD iteration t over the active block-columns
// (writes mse[t - 1], the MSE of the incoming iterate).  PASS_COUNT: the same,
// and the incoming iterate's codes replace those of the iterate before it in
// p.codes, the changed ones counted into changes[t - 1] (t >= 2; a
// block-column at a fixed point keeps its codes and adds nothing).
// PASS_FINAL: the final pass after T iterations over every block-column,
// called with t_first = t_last = T + 1: the codes of the final iterate, packed,
// and mse[T] (and changes[T] when counting, T >= 1).
template <int FMT, int WDT, int PASS>
__global__ void __launch_bounds__(kIterThreads, 1)
    k_iter(Problem p, int t_first, int t_last, const __grid_constant__ CUtensorMap wmap,
           const __grid_constant__ CUtensorMap wmap3) {
  constexpr int ES = WDT == DT_F32 ? 4 : 2;
  constexpr bool FIN = PASS == PASS_FINAL;
  const TileGeo geo = tile_geo(p.G, ES);
  const IterSmem lay = iter_smem(geo.lpb, p.P, p.segmax);
  const int S = geo.S;
  extern __shared__ __align__(128) unsigned char smem[];
  unsigned char* ring = smem;
  double2* acc = reinterpret_cast<double2*>(smem + lay.acc);
  double* racc = reinterpret_cast<double*>(smem + lay.racc);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + lay.bars);
  uint64_t* empty = full + kMaxStages;
  int* s_misc = reinterpret_cast<int*>(smem + lay.misc);  // [0] ticket result, [1] #ambiguous
  unsigned* s_cnt = reinterpret_cast<unsigned*>(s_misc + 2);  // [4] exact-path counters
  int* s_scan = s_misc + 40;   // [17] schedule scan
  Sched* s_sched = reinterpret_cast<Sched*>(smem + lay.sched);
  f2* ctab = reinterpret_cast<f2*>(smem + lay.ctab);
  int* s_sfirst = reinterpret_cast<int*>(smem + lay.sfirst);
  int* s_act = reinterpret_cast<int*>(smem + lay.act);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], kConsumerWarps);
    }
    mbar_fence_init();
    s_cnt[0] = s_cnt[1] = s_cnt[2] = s_cnt[3] = 0u;
  }
  if (threadIdx.x < kConsumers) racc[threadIdx.x] = 0.0;
  __syncthreads();
  // launched with programmatic stream serialization: what the kernels before
  // wrote (flags, scales, counters) is read only after this wait
  griddep_wait();
  griddep_launch_dependents();
  if (p.hdr->flags & kFlagAbort) return;

  if (warp == kConsumerWarps) {
    // ---------------- producer warp ----------------
    // Tile n of the CTA goes to stage n % S (use n / S of that stage).  The
    // producer stops issuing once some wait of the solve has given up, and
    // before it returns it waits (bounded) for the copy of the last use of
    // every stage, so no copy into this CTA's shared memory is in flight when
    // the CTA exits.
    int st = 0, issued = 0;
    unsigned par = 1u;
    bool stop = false;
    for (int t = t_first; t <= t_last; ++t) {
      cta_sync_all();  // the schedule of pass t is in shared memory
      const long long ub = s_sched->u_begin, ue = s_sched->u_end;
      const int nact = s_sched->nact, ident = s_sched->ident, v_first = s_sched->v_first;
      // this lane's block-column of the first segment (read now: the list is
      // rewritten once the consumers finish the pass)
      int pf_gl = -1;
      if (ub < ue) {
        const int i0 = (int)(ub / p.M) * kBcPerStrip;
        if (lane < min(kBcPerStrip, nact - i0)) pf_gl = ident ? i0 + lane : s_act[i0 - v_first * kBcPerStrip + lane];
      }
      for (long long u = ub; u < ue && !stop;) {
        const long long v = u / p.M;
        const long long r0 = u - v * p.M;
        const long long r1 = min((long long)p.M, r0 + (ue - u));
        const int i0 = (int)(v * kBcPerStrip);
        const int nbc = min(kBcPerStrip, nact - i0);
        const int* act = s_act - (long long)v_first * kBcPerStrip;
        const int gl = lane < nbc ? (ident ? i0 + lane : act[i0 + lane]) : 0;
        const int g_first = __shfl_sync(0xffffffffu, gl, 0), g_last = __shfl_sync(0xffffffffu, gl, nbc - 1);
        const bool wide = strip_contiguous(p, ident, g_first, g_last, nbc);
        for (long long tr = r0; tr < r1; tr += geo.RW) {
          if (ld_volatile(&p.hdr->flags) & kFlagTimeout) {
            stop = true;
            break;
          }
          if (!mbar_wait(&empty[st], par, &p.hdr->flags)) {
            stop = true;
            break;
          }
          unsigned char* slot = ring + st * geo.stage_bytes;
          if (wide) {  // the strip's block-columns are consecutive: one copy, [rows][15][G]
            if (lane == 0) {
              mbar_arrive_expect_tx(&full[st], (unsigned)(kBcPerStrip * geo.box_bytes));
              tma_load_3d(slot, &wmap3, 0, g_first, (int)tr, &full[st]);
            }
          } else if (p.use_tmap) {  // one copy per block-column, [15][rows][G]
            if (lane == 0) mbar_arrive_expect_tx(&full[st], (unsigned)(nbc * geo.box_bytes));
            __syncwarp();
            if (lane < nbc) tma_load_2d(slot + lane * geo.box_stride, &wmap, gl * p.G, (int)tr, &full[st]);
          } else {
            // one bulk copy per (block-column, row) of the tile inside the segment
            const int nr = (int)min((long long)geo.RW, r1 - tr);
            const unsigned row_bytes = (unsigned)(p.G * ES);
            if (lane == 0) mbar_arrive_expect_tx(&full[st], (unsigned)(nbc * nr) * row_bytes);
            __syncwarp();
            for (int it = lane; it < nbc * nr; it += 32) {
              const int w = it / nr, rr = it - w * nr;
              const long long gw = ident ? i0 + w : act[i0 + w];
              const unsigned char* src =
                  reinterpret_cast<const unsigned char*>(p.W) + ((tr + rr) * p.N + gw * p.G) * (long long)ES;
              bulk_g2s(slot + w * geo.box_stride + rr * (int)row_bytes, src, row_bytes, &full[st]);
            }
          }
          ++issued;
          if (++st == S) {
            st = 0;
            par ^= 1u;
          }
        }
        u = (v + 1) * p.M;
      }
      // Late passes usually keep the active list of the pass before, and with
      // it this CTA's range: the first tiles of that range are brought into
      // L2 now, while the consumers finish this pass, so the next pass's first
      // copies hit L2 (a hint only: nothing waits on it).
      if (t < t_last && p.use_tmap && !stop && pf_gl >= 0) {
        const long long r0 = ub - (ub / p.M) * p.M;
        const long long r1 = min((long long)p.M, r0 + (ue - ub));
        for (long long tr = r0, k = 0; tr < r1 && k < S; tr += geo.RW, ++k) tma_prefetch_2d(&wmap, pf_gl * p.G, (int)tr);
      }
    }
    if (lane == 0) {
      for (int s = 0; s < S && s < issued; ++s) mbar_drain(&full[s], (unsigned)(((issued - 1 - s) / S) & 1));
    }
    __syncwarp();
    return;
  }

  // ---------------- consumer warps ----------------
  const int lpb = geo.lpb, rl = geo.rl, RW = geo.RW;
  const int lg = __ffs(lpb) - 1;  // lpb is a power of two
  const int rho = lane >> lg, oct = lane & (lpb - 1);
  const bool leader = oct == 0;
  // residuals are squared as they are when max |W| lies in [2^-8, 2^41) (no
  // square of a residual can overflow, and none that underflows matters at the
  // MSE's tolerance), otherwise after scaling by rscale = 2^-floor(log2 amax),
  // which keeps every square inside the fp32 range whatever the magnitude of W
  const uint32_t amax_bits = p.hdr->amax_bits;
  const int amax_exp = (amax_bits == 0u) ? 0 : (int)((amax_bits >> 23) & 0xFFu) - 127;
  const bool scaled = amax_exp < -8 || amax_exp > 40;
  const float rscale = scaled ? __uint_as_float((uint32_t)(127 - max(-126, min(126, amax_exp))) << 23) : 1.f;
  const f2 rscale2 = splat(rscale);
  const double rscale_d = (double)rscale;
  const float sT = p.hdr->sT;
  const double sTd = (double)sT;
  const float isT = FMT == FMT_NVFP4 ? __frcp_rn(sT) : 1.f;
  const bool sT_ok = FMT != FMT_NVFP4 || in_range(isT);
  const int sT_bits = sig_bits(sT);
  int st = 0;
  unsigned par = 0u;
  const int64_t code_step = (int64_t)rl * (p.N >> 3);  // code groups between a lane's two rows
  unsigned tcnt = 0u;  // lane-rows settled as certified exact ties
  const f2* wtab = ctab + warp * 8 * lpb;  // this warp's column table

  for (int t = t_first; t <= t_last; ++t) {
  if (FIN && blockIdx.x == 0) {
    // the MSE of the passes that no grid barrier of the iteration launch summed
    for (int tp = max(1, t - 2); tp <= t - 1; ++tp)
      mse_total(p, mse_bcs(p, tp), p.nb, p.mse + (tp - 1), rscale_d, reinterpret_cast<double*>(acc));
  }
  if (!FIN && blockIdx.x == 0) {
    // the change flags of pass t + 1 were last read when pass t - 1 began, and
    // the strip counters of pass t + 1 were last waited on in pass t - 1
    unsigned* nxt = p.chg + (int64_t)((t + 1) % 3) * p.nb;
    for (int g = threadIdx.x; g < p.nb; g += kConsumers) nxt[g] = 0u;
    // (four counters per strip and pass parity: arrivals, ambiguous columns,
    // finalizers done, exact shares done)
    for (int v = threadIdx.x; v < p.n_strips; v += kConsumers)
      for (int c = 0; c < 4; ++c) p.strip_counter[(int64_t)(2 * c + ((t + 1) & 1)) * p.n_strips + v] = 0u;
  }
  pass_schedule(p, t, FIN || t == t_first || p.full_passes, s_sched, s_act, s_scan);
  const long long ub = s_sched->u_begin, ue = s_sched->u_end, L = s_sched->L;
  const int nact = s_sched->nact, Pt = s_sched->Pt, v_first = s_sched->v_first;
  const bool ident = s_sched->ident != 0;
  if (!FIN && blockIdx.x == 0 && threadIdx.x == 0) atomicAdd(&p.hdr->n_active_bc, (unsigned long long)nact);
  cta_sync_all();  // hand the schedule to the producer
  const int* act = s_act - (long long)v_first * kBcPerStrip;
  if (FIN) racc[threadIdx.x] = 0.0;
  // compare with the previous iterate's codes (kept in p.codes by the pass before)
  const bool cmp = (PASS == PASS_COUNT || (FIN && p.changes != nullptr)) && t > 1;
  unsigned nchg = 0u;

  for (long long u = ub; u < ue;) {
    const long long v = u / p.M;
    const long long r0 = u - v * p.M;
    const long long r1 = min((long long)p.M, r0 + (ue - u));
    const int i0 = (int)(v * kBcPerStrip);
    const int nbc = min(kBcPerStrip, nact - i0);
    const bool has = warp < nbc;  // warp-uniform: this warp owns a block-column of the strip
    const int g = has ? (ident ? i0 + warp : act[i0 + warp]) : 0;
    const int64_t col = (int64_t)g * p.G + 8 * oct;

    consumer_sync(kConsumers);  // the previous segment's readers of acc and the tables are done
    ColState cs;
    cs.tb = wtab + oct * 4;
    cs.tcb = wtab + 4 * lpb + oct * 4;
    cs.lane = lane;
    cs.ok = sT_ok;
    cs.res2 = 0ull;
    int b_bits = 1;  // longest odd significand among the lane's column scales
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float bj[2] = {1.f, 1.f}, cb[2] = {1.f, 1.f};
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int c = 2 * i + h;
        cs.thr[c] = 0.5f - kGuard;
        if (has) {
          bj[h] = b_decode_cg(p.b_store, p.col_dt, col + c);
          cb[h] = __frcp_rn(bj[h]) * isT;
          cs.ok = cs.ok && in_range(cb[h]);
          b_bits = max(b_bits, sig_bits(bj[h]));
          // MXINT4/MXINT8: a = 2^k, so a power-of-two b makes the candidate exact
          // (for bf16/fp16 W the tie certificate covers these columns as well)
          if (fmt_mxint(FMT) && WDT == DT_F32 && (__float_as_uint(bj[h]) & 0x007FFFFFu) == 0u) cs.thr[c] = 2.f;
        }
        acc[(warp * 8 + c) * 32 + lane] = make_double2(0.0, 0.0);
      }
      if (rho == 0) {
        ctab[warp * 8 * lpb + oct * 4 + i] = pk(bj[0], bj[1]);
        ctab[warp * 8 * lpb + 4 * lpb + oct * 4 + i] = pk(cb[0], cb[1]);
      }
      cs.cn2[i] = cs.cd2[i] = 0ull;
    }
    // odd part of a b: E4M3 e has at most 4 significant bits, 2^k has 1
    cs.tie_ok = tie_certified<FMT, WDT>(FMT == FMT_NVFP4 ? sT_bits + 4 + b_bits : b_bits);
    if (!FIN) racc[threadIdx.x] = 0.0;
    __syncwarp();  // the warp's column table is written
    bool achg = false;
    int run = 0;
    // block scales of this lane's rows (the block-column-major working copy:
    // a warp's rows are contiguous), one tile ahead
    const int64_t a_step = RW;
    int64_t aidx = (int64_t)g * p.M + r0 + rho;
    const int64_t y_off = rl;  // block-scale offset of the lane's second row
    // rows relative to the segment start, in 32 bits (a segment has fewer than 2^31 rows)
    const int nrows = (int)(r1 - r0);
    uint32_t an0 = a_raw_one<FMT>(), an1 = a_raw_one<FMT>();
    if (has && rho < nrows) an0 = a_fetch<FMT>(p.a_work, aidx);
    if (has && rho + rl < nrows) an1 = a_fetch<FMT>(p.a_work, aidx + y_off);
    // the tile's layout: [rows][15][G] (one copy of a strip of consecutive
    // block-columns) or [15][rows][G] (one copy per block-column)
    const bool wide = strip_contiguous(p, ident, ident ? i0 : act[i0], ident ? i0 + nbc - 1 : act[i0 + nbc - 1], nbc);
    const int row_stride = (wide ? kBcPerStrip : 1) * p.G * ES;
    const int slot_stride = wide ? p.G * ES : geo.box_stride;
    const unsigned char* wbase = ring + warp * slot_stride + rho * row_stride + 8 * oct * ES;
    const int y_bytes = rl * row_stride;

    for (int tr = 0; tr < nrows; tr += RW, aidx += a_step) {
      const int ra = tr + rho, rb = ra + rl;
      const bool vx = has && ra < nrows, vy = has && rb < nrows;  // per lane
      const uint32_t ra_raw = an0, rb_raw = an1;
      if (has && ra + RW < nrows) an0 = a_fetch<FMT>(p.a_work, aidx + a_step);
      if (has && rb + RW < nrows) an1 = a_fetch<FMT>(p.a_work, aidx + a_step + y_off);
      const int64_t cix = ((r0 + ra) * p.N + col) >> 3;  // code group of row ra, this lane's 8 columns
      uint2 oldx = make_uint2(0u, 0u), oldy = make_uint2(0u, 0u);
      if (PASS != PASS_ITER && cmp) {  // issued before the wait: the latency hides behind it
        if (vx) oldx = load_codes<FMT>(p.codes, cix);
        if (vy) oldy = load_codes<FMT>(p.codes, cix + code_step);
      }
      mbar_wait(&full[st], par, &p.hdr->flags);
      f2 wa[4], wb[4];
      const unsigned char* base = wbase + st * geo.stage_bytes;
      smem_row<WDT>(base, wa);
      smem_row<WDT>(base + y_bytes, wb);
      // the slot's loads are performed before its release lets a copy refill it
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[st]);
      if (++st == S) {
        st = 0;
        par ^= 1u;
      }
      if (has) {
        if (tr + RW > nrows) {  // warp-uniform: the segment's last tile
          // rows outside the segment (the next CTA's, or the zero fill past
          // the matrix) hold zeros: they add nothing and write nothing
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            if (!vx) wa[i] = 0ull;
            if (!vy) wb[i] = 0ull;
          }
        }
        const float aa = a_dec<FMT>(ra_raw), ab = a_dec<FMT>(rb_raw);  // fetched a tile ago
        if (FIN) {
          final_pair<FMT>(p, wa, aa, wb, ab, vx, vy, cs, sT, sTd, scaled, rscale2, s_cnt, tcnt, cix, code_step, oldx,
                          oldy, cmp, nchg);
          // the final block scales, in the output's row-major layout
          if (leader) {
            if (vx) a_put_raw<FMT>(p.a_store, (r0 + ra) * p.nb + g, ra_raw);
            if (vy) a_put_raw<FMT>(p.a_store, (r0 + rb) * p.nb + g, rb_raw);
          }
        } else {
          row_pair<FMT, PASS>(p, wa, aa, aidx, wb, ab, aidx + y_off, vx, vy, leader, lpb, cs, sT, isT, sTd, scaled,
                              rscale2, s_cnt, tcnt, cix, code_step, oldx, oldy, cmp, nchg, achg);
        }
      }
      run += 2;
      if (run >= run_rows<FMT>()) {
        run = 0;
        flush_runs(cs, acc, racc, warp, lane, has);
      }
    }
    flush_runs(cs, acc, racc, warp, lane, has);
    const int64_t slot = (int64_t)blockIdx.x * p.segmax + (v - v_first);
    if (!FIN) {
      // this segment's residual total of the warp's block-column (fixed xor
      // order over the lanes), and whether any of its block scales changed
      double r = racc[threadIdx.x];
      for (int o = 16; o > 0; o >>= 1) r += __shfl_xor_sync(0xffffffffu, r, o);
      if (has && lane == 0) p.mse_seg[slot * kBcPerStrip + warp] = r;
      if (__any_sync(0xffffffffu, achg) && has && lane == 0) p.chg[(int64_t)(t % 3) * p.nb + g] = 1u;
    }
    if (FIN) {  // no column update in the final pass
      u = (v + 1) * p.M;
      continue;
    }

    // CTA totals of the column sums: column (w, o, c) of the strip, i.e. column
    // 8 o + c of slot w's block-column, adds its row-lanes in order.
    consumer_sync(kConsumers);
    const int width = nbc * p.G;
    for (int vc = threadIdx.x; vc < width; vc += kConsumers) {
      const int w = vc / p.G, rem = vc - w * p.G, oo = rem >> 3, c = rem & 7;
      const double2* src = acc + (w * 8 + c) * 32 + oo;
      double2 tot = src[0];
      for (int rr = 1; rr < rl; ++rr) {
        const double2 x = src[rr * lpb];
        tot.x += x.x;
        tot.y += x.y;
      }
      p.col_part[slot * p.TSv + vc] = tot;
    }
    __threadfence();
    consumer_sync(kConsumers);
    // The strip's K CTAs have written their partial sums once its first
    // counter reaches K.  The nfin CTAs whose range ends in this strip (all but
    // a last one that runs on into the next strip; a lone CTA always) then
    // share its finalization: each waits (bounded) for the counter, finalizes
    // its block-columns w = q, q + nfin, ... and counts itself on the second
    // counter; once that reaches nfin the columns listed as ambiguous are
    // settled exactly, each finalizer taking a share of the rows.  A CTA that
    // runs on does not wait here.
    const int64_t k_first = cta_of(v * p.M, Pt, L);
    const int64_t k_last = cta_of((v + 1) * p.M - 1, Pt, L);
    const int K = (int)(k_last - k_first + 1);
    const int64_t par_off = (int64_t)(t & 1) * p.n_strips + v;
    unsigned* cnt = p.strip_counter + par_off;
    if (threadIdx.x == 0) atomicAdd(cnt, 1u);
    const bool ends_here = (v + 1) * p.M >= ue;
    const bool last_ends = range_begin(k_last + 1, Pt, L) <= (v + 1) * p.M;
    const int nfin = (K == 1 || last_ends) ? K : K - 1;
    const int q = (int)(blockIdx.x - k_first);
    if ((ends_here || K == 1) && q < nfin) {
      int* amb_list = p.amb_list + v * (int64_t)p.TSv;
      unsigned* amb_cnt = p.strip_counter + 2 * (int64_t)p.n_strips + par_off;
      unsigned* cnt2 = p.strip_counter + 4 * (int64_t)p.n_strips + par_off;
      // the first strip of each of the strip's CTAs (their partial slots are
      // indexed by it)
      for (int e = threadIdx.x; e < K; e += kConsumers)
        s_sfirst[k_first + e] = (int)(range_begin(k_first + e, Pt, L) / p.M);
      wait_count(cnt, (unsigned)K, &p.hdr->flags);
      consumer_sync(kConsumers);
      __threadfence();
      finalize_slots<FMT>(p, t, v, q, nfin, nbc, act, ident, i0, k_first, K, s_sfirst, sTd,
                          reinterpret_cast<double*>(acc), ctab, amb_list, amb_cnt, &s_misc[8]);
      if (threadIdx.x == 0) {
        __threadfence();
        atomicAdd(cnt2, 1u);
      }
      wait_count(cnt2, (unsigned)nfin, &p.hdr->flags);
      if (threadIdx.x == 0) s_misc[1] = (int)ld_acquire_gpu(amb_cnt);
      consumer_sync(kConsumers);
      const int n = s_misc[1];
      if (n > 0)
        exact_columns<FMT, WDT>(p, v, act, ident, i0, q, nfin, k_first, slot, s_sfirst, amb_list, n,
                                p.strip_counter + 6 * (int64_t)p.n_strips + par_off, sTd, isT,
                                reinterpret_cast<double*>(acc), &s_misc[0], s_cnt);
    }
    consumer_sync(kConsumers);
    u = (v + 1) * p.M;
  }

  if (PASS != PASS_ITER && cmp) {  // changed codes of this warp, one atomic per warp
    for (int o = 16; o > 0; o >>= 1) nchg += __shfl_xor_sync(0xffffffffu, nchg, o);
    if (lane == 0 && nchg) atomicAdd(&p.changes[t - 1], (unsigned long long)nchg);
  }

  if (FIN) {
    // MSE of the final iterate: per-thread residual sums, CTA tree, then the
    // CTA-ordered total by the last CTA to finish (no barrier follows)
    consumer_sync(kConsumers);
    double* mred = reinterpret_cast<double*>(acc);
    mred[threadIdx.x] = racc[threadIdx.x];
    consumer_sync(kConsumers);
    for (int o = kConsumerTreeTop; o > 0; o >>= 1) {
      if (threadIdx.x < o && threadIdx.x + o < kConsumers) mred[threadIdx.x] += mred[threadIdx.x + o];
      consumer_sync(kConsumers);
    }
    if (threadIdx.x == 0) {
      mse_part(p, t)[blockIdx.x] = mred[0];
      __threadfence();
      const unsigned prev = atomicAdd(&p.hdr->cta_counter, 1u);
      s_misc[0] = prev == (unsigned)p.P - 1u ? 1 : 0;
    }
    consumer_sync(kConsumers);
    if (s_misc[0]) {
      __threadfence();
      mse_total(p, mse_part(p, t), p.P, p.mse + (t - 1), rscale_d, mred);
      if (threadIdx.x == 0) p.hdr->cta_counter = 0u;
    }
  }
  // the scales of pass t (except the listed columns) are final before pass
  // t + 1 reads them
  if (t < t_last) grid_sync(p, t, rscale_d, reinterpret_cast<double*>(acc), &s_misc[0]);
  }  // passes

  for (int o = 16; o > 0; o >>= 1) tcnt += __shfl_xor_sync(0xffffffffu, tcnt, o);
  if (lane == 0 && tcnt) atomicAdd(&s_cnt[3], tcnt);
  consumer_sync(kConsumers);
  if (threadIdx.x == 0) {
    if (s_cnt[0]) atomicAdd(&p.hdr->n_quant_exact, (unsigned long long)s_cnt[0]);
    if (s_cnt[1]) atomicAdd(&p.hdr->n_block_exact, (unsigned long long)s_cnt[1]);
    if (s_cnt[2]) atomicAdd(&p.hdr->n_col_exact, (unsigned long long)s_cnt[2]);
    if (s_cnt[3]) atomicAdd(&p.hdr->n_quant_tie, (unsigned long long)s_cnt[3]);
  }
}

}  // namespace dq
