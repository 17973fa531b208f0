// dq_init.cuh -- initial iterates other than absmax RTN with b = 1 (included by
// dq_solver.cu): per-column L1-norm column scales, and a warm start from given
// scales.
//
// Per-column L1-norm init (DualQuant summary §5.3: the initialization uses
// format-native row absmax scales and per-column L1-norm scales).  The pages
// name the norm only; the reading taken:
//   c_j = sum_i |W_ij|,  mu = (sum_ij |W_ij|) / N      (each sum exact, then
//                                                      rounded once to fp64)
//   b_j = Proj_Fb(c_j / mu), 1 for an all-zero column
//   a   = Proj_Fa(max_{j in block} (|W_ij| / b_j) / qmax), 1 for a zero block
//   s_T = fp32(max_ij (|W_ij| / b_j) / 2688)            (NVFP4)
// every quotient one correctly rounded fp64 division.  The sums are exact, so
// no summation order enters the result: every |W_ij| (an fp32, bf16 or fp16
// value) is an integer m * 2^sh in units of 2^-149 with m < 2^24 and
// sh <= 253, and is added as 32-bit digits into 64-bit counters that never
// overflow (carry-save; carries are propagated only when partial sums merge).
#pragma once

#include "dq_device.cuh"
#include "dq_internal.h"

namespace dq {

// |w| of a finite float as m * 2^sh units of 2^-149.
__device__ __forceinline__ void units_of(float w, uint32_t& m, int& sh) {
  const uint32_t u = __float_as_uint(w) & 0x7FFFFFFFu;
  const uint32_t e = u >> 23;
  m = (u & 0x7FFFFFu) | (e ? 0x800000u : 0u);
  sh = e ? (int)e - 1 : 0;
}

// Propagate carries: digits 0..8 below 2^32, digit 9 takes the rest.  Each
// counter must be below 2^64 - 2^32.
__device__ __forceinline__ void xnorm(unsigned long long d[kXDigits]) {
  unsigned long long c = 0;
#pragma unroll
  for (int i = 0; i < kXDigits - 1; ++i) {
    const unsigned long long v = d[i] + c;
    d[i] = v & 0xFFFFFFFFull;
    c = v >> 32;
  }
  d[kXDigits - 1] += c;
}

// The exact value of normalized digits, rounded to fp64 (nearest, ties to
// even).  Works on the integer as 11 32-bit words, most significant first.
__device__ double xround(const unsigned long long d[kXDigits]) {
  uint32_t w[kXDigits + 1];
  for (int i = 0; i < kXDigits; ++i) w[i] = (uint32_t)d[i];
  w[kXDigits] = (uint32_t)(d[kXDigits - 1] >> 32);
  int hw = kXDigits;  // highest nonzero word
  while (hw >= 0 && w[hw] == 0u) --hw;
  if (hw < 0) return 0.0;
  const int top = 32 * hw + 31 - __clz(w[hw]);  // highest set bit
  if (top < 53) return scalbn((double)(((unsigned long long)w[1] << 32) | w[0]), -149);
  // the 53 bits top-52..top, and what lies below them
  const int low = top - 52;
  unsigned long long win = 0;  // bits low .. low+63 (zeros above the top)
  for (int k = 0; k < 3; ++k) {
    const int wi = (low >> 5) + k;
    const int pos = 32 * k - (low & 31);  // where word wi's bit 0 lands in the window
    if (wi <= kXDigits && pos < 64) {
      const unsigned long long v = w[wi];
      win |= pos >= 0 ? v << pos : v >> -pos;
    }
  }
  unsigned long long mant = win & ((1ull << 53) - 1ull);
  // round bit (low - 1) and sticky bits (below low - 1)
  const int rpos = low - 1;
  const bool rbit = (w[rpos >> 5] >> (rpos & 31)) & 1u;
  bool sticky = (w[rpos >> 5] & ((1u << (rpos & 31)) - 1u)) != 0u;
  for (int i = 0; i < (rpos >> 5); ++i) sticky = sticky || w[i] != 0u;
  if (rbit && (sticky || (mant & 1ull))) ++mant;  // 2^53 stays exact
  return scalbn((double)mant, low - 149);
}

// One weight as an exact float.
template <int WDT>
__device__ __forceinline__ float load1(const void* W, int64_t idx) {
  if (WDT == DT_F32) return __ldg(reinterpret_cast<const float*>(W) + idx);
  const unsigned short h = __ldg(reinterpret_cast<const unsigned short*>(W) + idx);
  return WDT == DT_BF16 ? __uint_as_float((uint32_t)h << 16) : __half2float(__ushort_as_half(h));
}

// Exact per-column magnitude sums.  CTA (x, y) takes columns 32x..32x+31 and
// rows [y R, (y+1) R); thread (warp, lane) adds column 32x + lane over every
// 8th row of the range into its own digit counters in shared memory; then the
// CTA merges the 8 warps' counters of each column, normalizes them and adds
// them into dig[j][0..9] in the workspace (zeroed before the launch).
template <int WDT>
__global__ void __launch_bounds__(kThreads) k_l1_sums(Problem p, int64_t rows_per_cta) {
  __shared__ unsigned long long dig[kXDigits][kThreads];
  if (p.hdr->flags & kFlagAbort) return;
#pragma unroll
  for (int d = 0; d < kXDigits; ++d) dig[d][threadIdx.x] = 0ull;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t j = (int64_t)blockIdx.x * 32 + lane;
  const int64_t r0 = (int64_t)blockIdx.y * rows_per_cta, r1 = min(p.M, r0 + rows_per_cta);
  if (j < p.N) {
#pragma unroll 4
    for (int64_t i = r0 + warp; i < r1; i += kWarps) {
      uint32_t m;
      int sh;
      units_of(load1<WDT>(p.W, i * p.N + j), m, sh);
      const unsigned long long v = (unsigned long long)m << (sh & 31);
      dig[sh >> 5][threadIdx.x] += v & 0xFFFFFFFFull;
      dig[(sh >> 5) + 1][threadIdx.x] += v >> 32;
    }
  }
  __syncthreads();
  const int64_t jc = (int64_t)blockIdx.x * 32 + threadIdx.x;
  if (threadIdx.x < 32 && jc < p.N) {
    unsigned long long s[kXDigits];
#pragma unroll
    for (int d = 0; d < kXDigits; ++d) {
      s[d] = 0ull;
      for (int wi = 0; wi < kWarps; ++wi) s[d] += dig[d][wi * 32 + threadIdx.x];
    }
    xnorm(s);
#pragma unroll
    for (int d = 0; d < kXDigits; ++d)
      if (s[d]) atomicAdd(&p.l1_dig[jc * kXDigits + d], s[d]);
  }
}

// Column norms c_j rounded to fp64, and the total over all columns (each
// column's normalized digits, so the total's counters stay below N * 2^33).
__global__ void __launch_bounds__(kThreads) k_l1_cols(Problem p) {
  if (p.hdr->flags & kFlagAbort) return;
  const int64_t j = (int64_t)blockIdx.x * kThreads + threadIdx.x;
  unsigned long long d[kXDigits];
#pragma unroll
  for (int k = 0; k < kXDigits; ++k) d[k] = j < p.N ? p.l1_dig[j * kXDigits + k] : 0ull;
  xnorm(d);
  if (j < p.N) p.l1_norm[j] = xround(d);
#pragma unroll
  for (int k = 0; k < kXDigits; ++k) {
    unsigned long long v = d[k];
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if ((threadIdx.x & 31) == 0 && v) atomicAdd(&p.l1_tot[k], v);
  }
}

// b_j = Proj_Fb(c_j / mu), mu = total / N; 1 for an all-zero column.
__global__ void __launch_bounds__(kThreads) k_l1_b(Problem p) {
  __shared__ double s_mu;
  if (p.hdr->flags & kFlagAbort) return;
  if (threadIdx.x == 0) {
    unsigned long long t[kXDigits];
    for (int k = 0; k < kXDigits; ++k) t[k] = p.l1_tot[k];
    xnorm(t);
    s_mu = xround(t) / (double)p.N;
  }
  __syncthreads();
  const double mu = s_mu;
  for (int64_t j = (int64_t)blockIdx.x * kThreads + threadIdx.x; j < p.N; j += (int64_t)gridDim.x * kThreads) {
    const double c = p.l1_norm[j];
    b_encode(p.b_store, p.col_dt, j, (c == 0.0 || mu == 0.0) ? 1.0 : b_project(c / mu, p.col_dt));
  }
}

// NVFP4 with column scales: max_ij |W_ij| / b_j (fp64 quotients) into the
// header, as the bits of a non-negative double (ordered like the values).
template <int WDT>
__global__ void __launch_bounds__(kThreads) k_amax_scaled(Problem p) {
  if (p.hdr->flags & kFlagAbort) return;
  const int64_t nchunks = p.M * p.N / 8;
  double m = 0.0;
  for (int64_t c = (int64_t)blockIdx.x * kThreads + threadIdx.x; c < nchunks; c += (int64_t)gridDim.x * kThreads) {
    float w[8];
    load8<WDT>(p.W, c * 8, w);
    const int64_t j0 = (c * 8) % p.N;
#pragma unroll
    for (int k = 0; k < 8; ++k) m = fmax(m, (double)fabsf(w[k]) / (double)b_decode(p.b_store, p.col_dt, j0 + k));
  }
  for (int o = 16; o > 0; o >>= 1) m = fmax(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0)
    atomicMax(&p.hdr->amax_scaled, (unsigned long long)__double_as_longlong(m));
}

// Warm start: every given scale must be admissible in its storage format
// (positive, finite, not NaN; E8M0 bytes 1..253 = 2^-126..2^126); the NVFP4
// tensor scale a positive finite float.  A violation sets kFlagBadInit and the
// later kernels do nothing.  Also fixes s_T in the header.
template <int FMT>
__global__ void __launch_bounds__(kThreads) k_check_given(Problem p) {
  if (p.hdr->flags & kFlagAbort) return;
  const int64_t stride = (int64_t)gridDim.x * kThreads;
  const int64_t tid = (int64_t)blockIdx.x * kThreads + threadIdx.x;
  bool bad = false;
  if (tid == 0) {
    float s = 1.f;
    if (FMT == FMT_NVFP4) {
      const uint32_t bits = __float_as_uint(*p.sT_out);
      bad = bits == 0u || bits >= 0x7F800000u;  // zero, negative, infinite or NaN
      s = __uint_as_float(bits);
    } else if (p.sT_out) {
      *p.sT_out = 1.f;
    }
    p.hdr->sT = s;
  }
  // the given block scales, checked and copied into the block-column-major
  // working copy the iterations use
  for (int64_t k = tid; k < p.M * p.nb; k += stride) {
    const int64_t i = k / p.nb, g = k - i * p.nb;
    if (FMT == FMT_INT4) {
      const unsigned short h = reinterpret_cast<const unsigned short*>(p.a_store)[k];
      bad = bad || h == 0u || h > 0x7BFFu;
      reinterpret_cast<unsigned short*>(p.a_work)[g * p.M + i] = h;
    } else {
      const uint8_t v = reinterpret_cast<const uint8_t*>(p.a_store)[k];
      bad = bad || v == 0u || v > (fmt_pow2(FMT) ? 253u : 0x7Eu);
      reinterpret_cast<uint8_t*>(p.a_work)[g * p.M + i] = v;
    }
  }
  for (int64_t j = tid; j < p.N; j += stride) {
    const uint32_t h = reinterpret_cast<const unsigned short*>(p.b_store)[j];
    bad = bad || h == 0u || h > (p.col_dt == DT_F16 ? 0x7BFFu : 0x7F7Fu);
  }
  if (bad) atomicOr(&p.hdr->flags, kFlagBadInit);
}

}  // namespace dq
