// dq_device.cuh -- device-side format helpers of the B200 DualQuant solver:
// grid quantizers Q (INT4 [-8,7], INT8 [-128,127], E2M1 and E4M3), projections of inverse scales onto
// the admissible sets (fp16, bf16, E4M3, E8M0 power of two), and storage
// decode/encode of block and column scales.
//
// Definitions followed (DualQuant reproduction README, "Core equations" and
// "Local reproduction"; DualQuant arXiv 2610.13767 summary, §3):
//  * Q(x): nearest grid value, an exact tie goes to the even neighbour (even
//    integer; even E2M1 mantissa bit), values past the ends clip.
//  * Projection: nearest admissible positive value in linear distance; ties go
//    to the even mantissa (fp16/bf16/E4M3) or to the larger power of two
//    (E8M0); beyond the ends the extreme admissible value.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>
#include <cuda_fp8.h>

namespace dq {

enum : int { FMT_INT4 = 0, FMT_MXINT4 = 1, FMT_NVFP4 = 2, FMT_MXFP4 = 3, FMT_MXINT8 = 4, FMT_MXFP8 = 5 };
// formats on the E2M1 grid, and formats with power-of-two (E8M0) block scales
__host__ __device__ constexpr bool fmt_e2m1(int f) { return f == FMT_NVFP4 || f == FMT_MXFP4; }
__host__ __device__ constexpr bool fmt_pow2(int f) {
  return f == FMT_MXINT4 || f == FMT_MXFP4 || f == FMT_MXINT8 || f == FMT_MXFP8;
}
// the FP8 E4M3 grid (MXFP8)
__host__ __device__ constexpr bool fmt_e4m3(int f) { return f == FMT_MXFP8; }
// integer grids with power-of-two block scales (MXINT4, MXINT8)
__host__ __device__ constexpr bool fmt_mxint(int f) { return f == FMT_MXINT4 || f == FMT_MXINT8; }
// one byte per code (INT8 and E4M3 grids) instead of two nibbles per byte
__host__ __device__ constexpr bool fmt_byte_codes(int f) { return f == FMT_MXINT8 || f == FMT_MXFP8; }
// ends of the integer grids, and qmax of the absmax initialization
__host__ __device__ constexpr float grid_lo(int f) { return f == FMT_MXINT8 ? -128.f : -8.f; }
__host__ __device__ constexpr float grid_hi(int f) { return f == FMT_MXINT8 ? 127.f : 7.f; }
__host__ __device__ constexpr double grid_qmax(int f) {
  return fmt_e2m1(f) ? 6.0 : (f == FMT_MXINT8 ? 127.0 : (f == FMT_MXFP8 ? 448.0 : 7.0));
}
enum : int { DT_F32 = 0, DT_BF16 = 1, DT_F16 = 2 };

// Distance (in grid units) from a rounding boundary inside which the fast fp32
// candidate x~ = (W * (1/b)) * (1/a) is not trusted and the decision is taken
// exactly.  The candidate's relative error is below 6 * 2^-24 (at most six
// correctly rounded fp32 operations), i.e. below 3.1e-6 grid units for
// |x| <= 8.5, far inside this guard, and below 4.6e-5 grid units for
// |x| <= 128.5 (INT8 grid; boundaries further out separate two values that
// clip to the same grid end), still inside it.
constexpr float kGuard = 0x1p-14f;

// ---------------------------------------------------------------------------
// Projection of a positive real inverse scale onto an admissible set.

// Nearest positive value of a binary float format with `mb` explicit mantissa
// bits, smallest normal exponent `emin` and largest finite value `vmax`.
__device__ __forceinline__ double proj_float(double v, int mb, int emin, double vmax) {
  const double minsub = scalbn(1.0, emin - mb);
  if (!(v > minsub)) return minsub;
  if (v >= vmax) return vmax;
  if (ilogb(v) < emin) {
    // subnormal range of the target: fixed quantum 2^(emin-mb); rint = half-even
    double r = scalbn(rint(scalbn(v, mb - emin)), emin - mb);
    return r < minsub ? minsub : r;
  }
  // normal range: round the fp64 significand to mb bits, half to even, in the
  // bit pattern (a carry into the exponent is the correct result)
  unsigned long long bits = (unsigned long long)__double_as_longlong(v);
  const int sh = 52 - mb;
  const unsigned long long lsb = (bits >> sh) & 1ull;
  bits += (1ull << (sh - 1)) - 1ull + lsb;
  bits &= ~((1ull << sh) - 1ull);
  double r = __longlong_as_double((long long)bits);
  return r > vmax ? vmax : r;
}

__device__ __forceinline__ double proj_f16(double v) { return proj_float(v, 10, -14, 65504.0); }
__device__ __forceinline__ double proj_bf16(double v) { return proj_float(v, 7, -126, 0x1.FEp127); }
__device__ __forceinline__ double proj_e4m3(double v) { return proj_float(v, 3, -6, 448.0); }

// Powers of two 2^k, k in [-126, 126]; a tie (1.5 * 2^k) goes up.
__device__ __forceinline__ double proj_pow2(double v) {
  const double lo = 0x1p-126, hi = 0x1p126;
  if (!(v > lo)) return lo;
  if (v >= hi) return hi;
  unsigned long long bits = (unsigned long long)__double_as_longlong(v);
  unsigned long long e = bits & 0x7FF0000000000000ull;
  if (bits & 0x0008000000000000ull) e += 0x0010000000000000ull;  // significand >= 1.5
  double r = __longlong_as_double((long long)e);
  return r > hi ? hi : r;
}

// ---------------------------------------------------------------------------
// Storage formats of the scales.

__device__ __forceinline__ float e4m3_value(uint32_t v) {
  const uint32_t e = (v >> 3) & 15u, m = v & 7u;
  return e == 0 ? (float)m * 0x1p-9f : __uint_as_float(((e + 120u) << 23) | (m << 20));
}

__device__ __forceinline__ uint8_t e4m3_bits(double v) {  // v admissible (exactly representable)
  return (uint8_t)__nv_cvt_double_to_fp8(v, __NV_SATFINITE, __NV_E4M3);
}

// Block scale stored factor as float (exact): fp16 value, 2^k, or E4M3 value e.
template <int FMT>
__device__ __forceinline__ float a_decode(const void* store, int64_t idx) {
  if (FMT == FMT_INT4) {
    return __half2float(reinterpret_cast<const __half*>(store)[idx]);
  } else if (fmt_pow2(FMT)) {
    return __uint_as_float((uint32_t)reinterpret_cast<const uint8_t*>(store)[idx] << 23);
  } else {
    return e4m3_value(reinterpret_cast<const uint8_t*>(store)[idx]);
  }
}

template <int FMT>
__device__ __forceinline__ void a_encode(void* store, int64_t idx, double v) {
  if (FMT == FMT_INT4) {
    reinterpret_cast<__half*>(store)[idx] = __double2half(v);
  } else if (fmt_pow2(FMT)) {
    reinterpret_cast<uint8_t*>(store)[idx] = (uint8_t)(ilogb(v) + 127);
  } else {
    reinterpret_cast<uint8_t*>(store)[idx] = e4m3_bits(v);
  }
}

// Projection of a least-squares block inverse scale value onto F_a; returns the
// stored factor (NVFP4: e with a = s_T * e, nearest s_T*e to v).
template <int FMT>
__device__ __forceinline__ double a_project(double v, double sT) {
  if (FMT == FMT_INT4) return proj_f16(v);
  if (fmt_pow2(FMT)) return proj_pow2(v);
  return proj_e4m3(v / sT);
}

__device__ __forceinline__ float b_decode(const void* store, int col_dt, int64_t j) {
  const uint16_t h = reinterpret_cast<const uint16_t*>(store)[j];
  return col_dt == DT_F16 ? __half2float(__ushort_as_half(h)) : __uint_as_float((uint32_t)h << 16);
}

__device__ __forceinline__ void b_encode(void* store, int col_dt, int64_t j, double v) {
  uint16_t h;
  if (col_dt == DT_F16) {
    h = __half_as_ushort(__double2half(v));
  } else {
    h = (uint16_t)(__float_as_uint((float)v) >> 16);  // v is an exact bf16 value
  }
  reinterpret_cast<uint16_t*>(store)[j] = h;
}

__device__ __forceinline__ double b_project(double v, int col_dt) {
  return col_dt == DT_F16 ? proj_f16(v) : proj_bf16(v);
}

// ---------------------------------------------------------------------------
// Grid quantizers.  `xt` is the fp32 candidate for x = W/(a b), `w` the exact
// weight, `ab` the exact product a*b in fp64.  Near a rounding boundary h the
// side is decided by the sign of fma(-h, ab, w) = w - h*a*b, whose single
// rounding cannot change the sign of the exact difference.

// exact a*b in fp64 (a = s_T * e for NVFP4): at most 36 significant bits
template <int FMT>
__device__ __forceinline__ double ab_exact(float astored, float b, double sTd) {
  return FMT == FMT_NVFP4 ? (sTd * (double)astored) * (double)b : (double)astored * (double)b;
}

template <int FMT>
__device__ __forceinline__ float q_int4(float xt, float w, float a, float b, double sTd) {
  const float c = fminf(fmaxf(xt, grid_lo(FMT)), grid_hi(FMT));
  float q = __fsub_rn(__fadd_rn(c, 12582912.f), 12582912.f);  // round half even
  const float r = c - q;
  if (fabsf(r) > 0.5f - kGuard) {
    const float h = q + copysignf(0.5f, r);
    const double d = fma(-(double)h, ab_exact<FMT>(a, b, sTd), (double)w);
    const float lo = h - 0.5f, hi = h + 0.5f;
    q = d > 0.0 ? hi : (d < 0.0 ? lo : (fmodf(lo, 2.f) == 0.f ? lo : hi));
    q = fminf(fmaxf(q, grid_lo(FMT)), grid_hi(FMT));
  }
  return q;
}

// E2M1 magnitudes {0,.5,1,1.5,2,3,4,6}: spacing 0.5 below 2, 1 in [2,4], 2 in
// [4,6]; rounding to a multiple of the local spacing with half-even gives the
// even-mantissa tie rule.
template <int FMT>
__device__ __forceinline__ float q_e2m1(float xt, float w, float a, float b, double sTd) {
  const float ax = fminf(fabsf(xt), 6.f);
  const float p2 = __uint_as_float(max(__float_as_uint(ax) & 0x7F800000u, 0x3F800000u));  // 1, 2 or 4
  const float magic = p2 * 6291456.f;  // 1.5 * 2^23 * (p2 / 2)
  float qm = __fsub_rn(__fadd_rn(ax, magic), magic);
  const float r = ax - qm;
  if (fabsf(r) > 0.25f * p2 - kGuard) {
    const float h = qm + copysignf(0.25f * p2, r);
    const float half = h < 2.f ? 0.25f : (h < 4.f ? 0.5f : 1.f);
    const float lo = h - half, hi = h + half;
    const double d = fma(-(double)h, ab_exact<FMT>(a, b, sTd), fabs((double)w));
    const bool lo_even = (lo == 0.f || lo == 1.f || lo == 2.f || lo == 4.f);
    qm = d > 0.0 ? hi : (d < 0.0 ? lo : (lo_even ? lo : hi));
    qm = fminf(qm, 6.f);
  }
  return copysignf(qm, xt);
}

// FP8 E4M3 magnitudes: binade [2^E, 2^(E+1)) with E >= -6 has spacing 2^(E-3),
// below 2^-6 the subnormal spacing 2^-9; 448 is the largest value and larger
// magnitudes clip to it.  Rounding to a multiple of the local spacing with
// half-even gives the even-mantissa tie rule (the spacing's multiples
// alternate mantissa parity, across binade ends too).  Near a boundary h the
// side is the sign of |w| - h*a*b, formed in fp64 (h has 5 significant bits).
template <int FMT>
__device__ __forceinline__ float q_e4m3(float xt, float w, float a, float b, double sTd) {
  const float ax = fminf(fabsf(xt), 448.f);
  const float p2 = __uint_as_float(max(__float_as_uint(ax) & 0x7F800000u, 0x3C800000u));  // binade base, >= 2^-6
  const float magic = p2 * 1572864.f;  // 1.5 * 2^23 * (p2 / 8)
  float qm = __fsub_rn(__fadd_rn(ax, magic), magic);
  const float half = p2 * 0.0625f;
  const float r = ax - qm;
  if (fabsf(r) > half - p2 * 0x1p-14f) {
    const float h = qm + copysignf(half, r);
    const float lo = h - half, hi = h + half;
    const double d = fma(-(double)h, ab_exact<FMT>(a, b, sTd), fabs((double)w));
    const bool lo_even = fmodf(lo / (2.f * half), 2.f) == 0.f;
    qm = d > 0.0 ? hi : (d < 0.0 ? lo : (lo_even ? lo : hi));
    qm = fminf(qm, 448.f);
  }
  return copysignf(qm, xt);
}

// Q(W/(a b)) for one element.  u = W * cb is the weight times the column
// factor (1/b, and 1/s_T for NVFP4), ia = 1/a (1/e for NVFP4); `ok` says the
// fast fp32 candidate u*ia is trustworthy, otherwise it comes from an fp64
// quotient.  Comments of the fast paths (grid units, guard) are above.
template <int FMT>
__device__ __forceinline__ float quant(float w, float u, float ia, bool ok, float a, float b, double sTd) {
  float xt;
  if (ok) {
    xt = u * ia;
  } else {
    xt = (float)((double)w / ab_exact<FMT>(a, b, sTd));
  }
  if (fmt_e2m1(FMT)) return q_e2m1<FMT>(xt, w, a, b, sTd);
  if (fmt_e4m3(FMT)) return q_e4m3<FMT>(xt, w, a, b, sTd);
  return q_int4<FMT>(xt, w, a, b, sTd);
}

// 4-bit code of a grid value (zero is always the 0x0 nibble).
template <int FMT>
__device__ __forceinline__ uint32_t nibble(float q) {
  if (!fmt_e2m1(FMT)) return (uint32_t)((int)q) & 15u;
  const float m = fabsf(q);
  if (m == 0.f) return 0u;
  // magnitude code: 0.5->1, 1->2, 1.5->3, 2->4, 3->5, 4->6, 6->7
  const uint32_t c = m < 2.f ? (uint32_t)(m * 2.f) : (m == 2.f ? 4u : (m == 3.f ? 5u : (m == 4.f ? 6u : 7u)));
  return (q < 0.f ? 8u : 0u) | c;
}

// ---------------------------------------------------------------------------
// Vector loads of 8 consecutive weights (exact conversion to fp32).

template <int WDT>
__device__ __forceinline__ void load8(const void* W, int64_t off, float w[8]) {
  if (WDT == DT_F32) {
    const float4* p = reinterpret_cast<const float4*>(reinterpret_cast<const float*>(W) + off);
    const float4 x = __ldg(p), y = __ldg(p + 1);
    w[0] = x.x; w[1] = x.y; w[2] = x.z; w[3] = x.w;
    w[4] = y.x; w[5] = y.y; w[6] = y.z; w[7] = y.w;
  } else {
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(W) + off));
    const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      if (WDT == DT_BF16) {
        w[2 * i] = __uint_as_float(u[i] << 16);
        w[2 * i + 1] = __uint_as_float(u[i] & 0xFFFF0000u);
      } else {
        const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&u[i]));
        w[2 * i] = f.x;
        w[2 * i + 1] = f.y;
      }
    }
  }
}

}  // namespace dq
