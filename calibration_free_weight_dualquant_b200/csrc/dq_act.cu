// dq_act.cu -- the beta-folded activation quantizer: X' = X diag(b) followed by
// the format's own row-wise absmax round-to-nearest, in one pass over X (NVFP4:
// an amax pass first, in the same launch, for the tensor scale).
//
// Method (DualQuant arXiv 2610.13767 summary, §4.4 "Inference-time procedure
// and overhead", and the reproduction README flowchart, last two boxes): with
// W ~ D_a Q D_b, a product X W^T equals (X D_b) Q^T D_a, so at inference the
// column inverse scales b multiply the activation channels before the
// format-native row-wise quantization, inside the quantization kernel; the row
// scales a fold into the weight dequantization.
//
// Exactness: X is bf16 or fp16 and b is bf16 or fp16, so x' = x b has at most
// 22 significant bits and is exact in fp32.  Group scales follow the solver's
// RTN initialization (absmax / qmax projected onto the format's scale set, 1
// for an all-zero group; NVFP4 tensor scale fp32(amax / 2688)), with the same
// certified fp32 projection and exact grid decisions as the solver.
#include "dq.h"
#include "dq_device.cuh"
#include "dq_fast.cuh"
#include "dq_internal.h"

namespace dq {

constexpr int kActThreads = 256;  // 8 warps
constexpr int kActWarps = kActThreads / 32;
// CTAs per SM of the one-pass kernels: 85 registers for E = 8, 128 for E = 16 and 32
__host__ __device__ constexpr int act_ctas_per_sm(int E) { return E >= 16 ? 2 : 3; }
constexpr int kActNvCtasPerSm = 2;  // the fused NVFP4 kernel: 128 registers
constexpr int kActEntry = 2048;     // bytes of one ring entry of a warp (one work item)
constexpr int kActStages = 4;       // ring entries per warp (a power of two)
constexpr int kActMinItems = 4;     // fewest items per warp before the grid shrinks
constexpr int kActSmem = kActWarps * kActStages * kActEntry;  // 64 KB

// Layout for E elements per lane (E = min(G, 32): 8, 16 or 32).  A warp
// covers a slab of 32 E columns of a row; lane l holds columns E l .. E l +
// E - 1, so a group of G columns lies in G / E consecutive lanes (one lane for
// G <= 32).  A work item is the slab piece of kRows consecutive rows (one
// ring entry).  In shared memory lane l's E/8 16-byte chunks of a row sit at
// l * 2E bytes, chunk c in place c ^ ((l / (64/E)) mod (E/8)), so the eight
// lanes of a 128-bit access phase hit eight different 16-byte bank groups.
template <int E>
struct ActGeo {
  static constexpr int kChunks = E / 8;
  static constexpr int kRowBytes = 64 * E;
  static constexpr int kRows = kActEntry / kRowBytes;  // 4, 2, 1
  static constexpr int kSlab = 32 * E;
  __device__ static int chunk_off(int lane, int c) {
    return lane * 2 * E + 16 * (c ^ ((lane / (64 / E)) & (kChunks - 1)));
  }
};

struct ActProblem {
  const void* X;
  const void* b_store;
  int col_dt, G;
  int lgG;          // log2 G
  int64_t M, K;
  int nb;           // groups per row
  int n_slabs;      // ceil(K / (32 E))
  void* codes;
  void* a_store;
  float* sT_out;
  WsHeader* hdr;
  int codes_vec;    // codes pointer aligned for one vector store per lane and row
};

// 16-byte asynchronous copy global -> shared (L1 bypassed); zero-fills the
// destination when `pred` is false (nothing is read then).
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool pred) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(pred ? 16 : 0) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// x' = x b of two elements, exact in fp32: the 16-bit halves of word u times
// those of bw in one mixed-precision fma each (X and b of one type, XDT), or
// the exact fp32 value of x times the fp32 b (types differ).
template <int XDT>
__device__ __forceinline__ f2 xb_same(uint32_t u, uint32_t bw) {
  float lo, hi;
  if (XDT == DT_BF16)
    asm("{\n.reg .b16 x0, x1, b0, b1;\nmov.b32 {x0, x1}, %2;\nmov.b32 {b0, b1}, %3;\n"
        "fma.rn.f32.bf16 %0, x0, b0, 0f80000000;\nfma.rn.f32.bf16 %1, x1, b1, 0f80000000;\n}"
        : "=f"(lo), "=f"(hi)
        : "r"(u), "r"(bw));
  else
    asm("{\n.reg .b16 x0, x1, b0, b1;\nmov.b32 {x0, x1}, %2;\nmov.b32 {b0, b1}, %3;\n"
        "fma.rn.f32.f16 %0, x0, b0, 0f80000000;\nfma.rn.f32.f16 %1, x1, b1, 0f80000000;\n}"
        : "=f"(lo), "=f"(hi)
        : "r"(u), "r"(bw));
  return pk(lo, hi);
}
template <int XDT>
__device__ __forceinline__ f2 xb_mixed(uint32_t u, f2 b2) {
  float lo, hi;
  if (XDT == DT_BF16)
    asm("{\n.reg .b16 h0, h1;\nmov.b32 {h0, h1}, %2;\nadd.rn.f32.bf16 %0, h0, 0f80000000;\n"
        "add.rn.f32.bf16 %1, h1, 0f80000000;\n}"
        : "=f"(lo), "=f"(hi)
        : "r"(u));
  else
    asm("{\n.reg .b16 h0, h1;\nmov.b32 {h0, h1}, %2;\nadd.rn.f32.f16 %0, h0, 0f80000000;\n"
        "add.rn.f32.f16 %1, h1, 0f80000000;\n}"
        : "=f"(lo), "=f"(hi)
        : "r"(u));
  return mul2(pk(lo, hi), b2);
}

// Three-input max that propagates NaN.
__device__ __forceinline__ float max3_nan(float a, float b, float c) {
  float d;
  asm("max.NaN.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// max |v| over P packed pairs (NaN if any is NaN).
template <int P>
__device__ __forceinline__ float absmax_pairs(const f2* v) {
  float m = max3_nan(fabsf(lo_of(v[0])), fabsf(hi_of(v[0])), 0.f);
#pragma unroll
  for (int i = 1; i < P; ++i) m = max3_nan(m, fabsf(lo_of(v[i])), fabsf(hi_of(v[i])));
  return m;
}

// The lane's column scales for the E columns starting at col (zeros past K):
// raw 16-bit pairs (BSAME) or fp32 pairs.
template <int E, bool BSAME>
struct ActCols {
  uint32_t w[BSAME ? E / 2 : 1];
  f2 f[BSAME ? 1 : E / 2];
  __device__ void load(const ActProblem& p, int64_t col) {
    const bool on = col < p.K;
    const uint16_t* bs = reinterpret_cast<const uint16_t*>(p.b_store);
#pragma unroll
    for (int i = 0; i < E / 2; ++i) {
      if (BSAME)
        w[i] = on ? (uint32_t)bs[col + 2 * i] | ((uint32_t)bs[col + 2 * i + 1] << 16) : 0u;
      else
        f[i] = on ? pk(b_decode(p.b_store, p.col_dt, col + 2 * i), b_decode(p.b_store, p.col_dt, col + 2 * i + 1))
                  : 0ull;
    }
  }
};

// The lane's E values of X' in one row of a ring entry, as packed pairs.
template <int E, int XDT, bool BSAME>
__device__ __forceinline__ void act_row(const unsigned char* row, int lane, const ActCols<E, BSAME>& bc, f2* x) {
#pragma unroll
  for (int c = 0; c < E / 8; ++c) {
    const uint4 v = *reinterpret_cast<const uint4*>(row + ActGeo<E>::chunk_off(lane, c));
    const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i)
      x[4 * c + i] = BSAME ? xb_same<XDT>(u[i], bc.w[4 * c + i]) : xb_mixed<XDT>(u[i], bc.f[4 * c + i]);
  }
}

// Work items of a grid: (row block q, slab s) pairs, rows kRows q .. kRows q
// + kRows - 1, numbered row-major, i = q n_slabs + s.  The grid's U warps
// (U rounded down to a multiple of the slab count where there are fewer slabs
// than warps) take them grid-stride, warp w items w, w + U, w + 2U, ...: the
// warps of the grid read one contiguous span of X at a time, and a warp keeps
// one slab (and its column scales) throughout.  REV walks a warp's items in
// the opposite order.  Each warp streams its items through a ring of
// kActStages entries in shared memory, filled by 16-byte asynchronous copies
// kActStages - 1 items ahead of the arithmetic: the copies in flight hold no
// registers.  A lane reads back only the bytes its own copies wrote, so
// completing its own copy groups is all the ordering it needs; an entry is
// refilled one iteration after it was read, when the values taken from it
// have been used.  `f(row, k, s, col, active, entry_row)` runs for every row
// of an item (k = 0 .. kRows - 1, rows below M only).
struct ActCursor {
  int64_t q, s;  // row block and slab of the current item
};
template <int E, bool REV, class F>
__device__ __forceinline__ void act_stream(const ActProblem& p, F&& f) {
  using Geo = ActGeo<E>;
  constexpr int R = Geo::kRows;
  extern __shared__ __align__(16) unsigned char act_ring[];
  const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
  const int64_t nw = (int64_t)gridDim.x * kActWarps;
  const int64_t ns = p.n_slabs;
  const int64_t U = ns <= nw ? nw / ns * ns : nw;  // warps that take items
  const int64_t w = (int64_t)blockIdx.x * kActWarps + wib;
  const int64_t MQ = (p.M + R - 1) / R;  // row blocks
  const int64_t T = MQ * ns;
  if (w >= U || w >= T) return;
  const int64_t n = (T - w + U - 1) / U;  // this warp's items
  // the stride U as a (row block, slab) step
  const int64_t dq_ = U / ns, ds = U - dq_ * ns;
  auto step = [&](ActCursor& c) {
    if (!REV) {
      c.q += dq_;
      c.s += ds;
      if (c.s >= ns) {
        c.s -= ns;
        ++c.q;
      }
    } else {
      c.q -= dq_;
      c.s -= ds;
      if (c.s < 0) {
        c.s += ns;
        --c.q;
      }
    }
  };
  const int64_t ifirst = REV ? w + (n - 1) * U : w;
  ActCursor cc{ifirst / ns, ifirst % ns};  // copy cursor
  ActCursor ac = cc;                       // arithmetic cursor
  unsigned char* wring = act_ring + wib * kActStages * kActEntry;
  const uint32_t wring_s = smem_u32(wring);
  int dst[Geo::kChunks];
#pragma unroll
  for (int c = 0; c < Geo::kChunks; ++c) dst[c] = Geo::chunk_off(lane, c);
  const uint16_t* X = reinterpret_cast<const uint16_t*>(p.X);
  auto fetch = [&](int slot, bool has) {
    const int64_t r0 = cc.q * R, col = cc.s * Geo::kSlab + lane * E;
    const bool on = has && col < p.K;
    const uint16_t* src = X + r0 * p.K + col;  // dereferenced only where a copy is predicated on
#pragma unroll
    for (int k = 0; k < R; ++k) {
      const bool pr = on && r0 + k < p.M;
#pragma unroll
      for (int c = 0; c < Geo::kChunks; ++c)
        cp_async16(wring_s + slot * kActEntry + k * Geo::kRowBytes + dst[c],
                   pr ? static_cast<const void*>(src + k * p.K + 8 * c) : p.X, pr);
    }
    cp_async_commit();  // one group per item, empty or not, so group counts stay uniform
    if (has) step(cc);
  };
#pragma unroll
  for (int k = 0; k < kActStages - 1; ++k) fetch(k, k < n);
#pragma unroll 1
  for (int64_t j = 0; j < n; ++j) {
    // refill the entry read in the previous iteration with item j + S - 1
    fetch((int)((j + kActStages - 1) & (kActStages - 1)), j + kActStages - 1 < n);
    cp_async_wait<kActStages - 1>();  // item j's group is complete
    const unsigned char* e = wring + (j & (kActStages - 1)) * kActEntry;
    const int64_t r = ac.q * R, col = ac.s * Geo::kSlab + lane * E;
    const int nr = (int)min((int64_t)R, p.M - r);
#pragma unroll
    for (int k = 0; k < R; ++k)
      if (k < nr) f(r + k, k, ac.s, col, col < p.K, e + k * Geo::kRowBytes);  // warp-uniform
    step(ac);
  }
  cp_async_wait<0>();
}

// Packed max of magnitudes of two 16-bit pairs (NaN propagates; the sign
// bits of the result are cleared by the caller).
template <int XDT>
__device__ __forceinline__ uint32_t hmax_abs(uint32_t a, uint32_t b) {
  uint32_t d;
  if (XDT == DT_BF16)
    asm("max.NaN.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  else
    asm("max.NaN.xorsign.abs.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// Pass 1 (NVFP4 only): amax = max |x b| over the grid's items into the
// header, and the non-finite check.  max_ij |x_ij b_j| = max_j |b_j| max_i
// |x_ij|, so a lane keeps the running max magnitude of each of its columns in
// the 16-bit input format (exact) and multiplies by b once per slab.
template <int E, int XDT, bool BSAME>
__device__ __forceinline__ void act_amax(const ActProblem& p) {
  const int lane = threadIdx.x & 31;
  float amax = 0.f;
  ActCols<E, BSAME> bc;
  uint32_t acc[E / 2];
#pragma unroll
  for (int i = 0; i < E / 2; ++i) acc[i] = 0u;
  int64_t s_have = -1, col_have = 0;
  auto fold = [&]() {  // the columns' maxima times b into amax
    bc.load(p, col_have);
    f2 v[E / 2];
#pragma unroll
    for (int i = 0; i < E / 2; ++i) {
      const uint32_t m = acc[i] & 0x7FFF7FFFu;
      v[i] = BSAME ? xb_same<XDT>(m, bc.w[i]) : xb_mixed<XDT>(m, bc.f[i]);
      acc[i] = 0u;
    }
    amax = max3_nan(amax, absmax_pairs<E / 2>(v), 0.f);
  };
  act_stream<E, false>(p, [&](int64_t, int, int64_t s, int64_t col, bool, const unsigned char* row) {
    if (s != s_have) {  // warp-uniform
      if (s_have >= 0) fold();
      s_have = s;
      col_have = col;
    }
#pragma unroll
    for (int c = 0; c < E / 8; ++c) {
      const uint4 v = *reinterpret_cast<const uint4*>(row + ActGeo<E>::chunk_off(lane, c));
      acc[4 * c + 0] = hmax_abs<XDT>(acc[4 * c + 0], v.x);
      acc[4 * c + 1] = hmax_abs<XDT>(acc[4 * c + 1], v.y);
      acc[4 * c + 2] = hmax_abs<XDT>(acc[4 * c + 2], v.z);
      acc[4 * c + 3] = hmax_abs<XDT>(acc[4 * c + 3], v.w);
    }
  });
  if (s_have >= 0) fold();
  for (int o = 16; o > 0; o >>= 1) amax = max3_nan(amax, __shfl_xor_sync(0xffffffffu, amax, o), 0.f);
  if (lane == 0) {
    if (amax <= 3.402823466e38f)
      atomicMax(&p.hdr->amax_bits, __float_as_uint(amax));
    else
      atomicOr(&p.hdr->flags, kFlagNonFinite);  // an infinity or a NaN
  }
}

// Exact decisions for the lane's E elements of one row (the fast path flagged
// one of them, or its factors are out of the trusted range): x' recomputed
// from the ring and b, each element through the solver's certified quantizer.
template <int FMT, int E, int XDT>
static __device__ __noinline__ void act_exact(const unsigned char* row, const ActProblem& p, int lane, int64_t col,
                                              float isT, float ia, bool ok, float a, double sTd, uint32_t* cw) {
#pragma unroll 1
  for (int c = 0; c < E / 8; ++c) {
    const uint4 v = *reinterpret_cast<const uint4*>(row + ActGeo<E>::chunk_off(lane, c));
    const uint32_t u[4] = {v.x, v.y, v.z, v.w};
    uint32_t word = 0;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const uint32_t h = (u[e >> 1] >> (16 * (e & 1))) & 0xFFFFu;
      const float xv = XDT == DT_BF16 ? __uint_as_float(h << 16) : __half2float(__ushort_as_half((unsigned short)h));
      const float x = xv * b_decode(p.b_store, p.col_dt, col + 8 * c + e);  // exact
      const float q = quant<FMT>(x, x * isT, ia, ok, a, 1.f, sTd);
      word |= nibble<FMT>(q) << (4 * e);
    }
    cw[c] = word;
  }
}

// Four E2M1 code pairs of packed values, as one word (element c in bits
// 4c .. 4c+3; hardware round-to-nearest-even with saturation at 6).
__device__ __forceinline__ uint32_t e2m1_word(const f2* v) {
  uint32_t w;
  asm("{\n.reg .b8 c0, c1, c2, c3;\n"
      "cvt.rn.satfinite.e2m1x2.f32 c0, %2, %1;\n"
      "cvt.rn.satfinite.e2m1x2.f32 c1, %4, %3;\n"
      "cvt.rn.satfinite.e2m1x2.f32 c2, %6, %5;\n"
      "cvt.rn.satfinite.e2m1x2.f32 c3, %8, %7;\n"
      "mov.b32 %0, {c0, c1, c2, c3};\n}"
      : "=r"(w)
      : "f"(lo_of(v[0])), "f"(hi_of(v[0])), "f"(lo_of(v[1])), "f"(hi_of(v[1])), "f"(lo_of(v[2])), "f"(hi_of(v[2])),
        "f"(lo_of(v[3])), "f"(hi_of(v[3])));
  return w;
}

// A zero E2M1 magnitude is always the 0x0 nibble (no "-0"): bit 3 of a nibble
// survives only where one of its bits 0..2 is set.
__device__ __forceinline__ uint32_t e2m1_no_negzero(uint32_t w) {
  return w & (0x77777777u | (w << 1) | (w << 2) | (w << 3));
}

// Two's-complement nibbles of four integer pairs, saturated to [-8, 7]; t
// holds q + 1.5 * 2^23 as fp32, whose bit pattern is 0x4B400000 + q.
__device__ __forceinline__ uint32_t int4_word(const f2* t) {
  int q[8];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    q[2 * i] = (int)__float_as_uint(lo_of(t[i])) - 0x4B400000;
    q[2 * i + 1] = (int)__float_as_uint(hi_of(t[i])) - 0x4B400000;
  }
  uint32_t w;
  asm("cvt.pack.sat.s4.s32.b32 %0, %1, %2, 0;" : "=r"(w) : "r"(q[7]), "r"(q[6]));
  asm("cvt.pack.sat.s4.s32.b32 %0, %1, %2, %0;" : "+r"(w) : "r"(q[5]), "r"(q[4]));
  asm("cvt.pack.sat.s4.s32.b32 %0, %1, %2, %0;" : "+r"(w) : "r"(q[3]), "r"(q[2]));
  asm("cvt.pack.sat.s4.s32.b32 %0, %1, %2, %0;" : "+r"(w) : "r"(q[1]), "r"(q[0]));
  return w;
}

// Exact INT-grid codes of a flagged lane, in fp32.  The candidate x (1/a)
// picks the boundary h nearest x/a; the side is the sign of fma(-h, a, x) =
// x - h a, which the fma's single rounding cannot change: x is exact, h a is a
// half-integer of at most 5 significant bits times an fp16 value, and a
// nonzero difference is a multiple of 2^-149.  Zero is a tie, to the even
// integer.  The pack saturates to [-8, 7].
template <int P>
__device__ __forceinline__ void int_exact_lane(const f2* x, float ia, float a, uint32_t* cw) {
#pragma unroll
  for (int c = 0; c < P / 4; ++c) {
    f2 t[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float qs[2];
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const float xv = e ? hi_of(x[4 * c + i]) : lo_of(x[4 * c + i]);
        const float xt = xv * ia;
        float q = __fsub_rn(__fadd_rn(xt, 12582912.f), 12582912.f);
        const float r = xt - q;
        if (fabsf(r) > 0.5f - kGuard) {
          const float h = q + copysignf(0.5f, r);
          const float d = fmaf(-h, a, xv);
          q = d > 0.f ? h + 0.5f : (d < 0.f ? h - 0.5f : __fsub_rn(__fadd_rn(h, 12582912.f), 12582912.f));
        }
        qs[e] = q + 12582912.f;
      }
      t[i] = pk(qs[0], qs[1]);
    }
    cw[c] = int4_word(t);
  }
}

// Exact E2M1 codes of a flagged NVFP4 lane, in fp32 (a = s_T e): the
// candidate picks the boundary h nearest |x|/(s_T e); the side is the sign of
// fma(-(h e), s_T, |x|), exact as h e has at most 7 significant bits.  Zero is
// a tie, to the even mantissa.
template <int P>
__device__ __forceinline__ void e2m1_exact_lane(const f2* x, float isT, float ia, float e, float sT, uint32_t* cw) {
#pragma unroll
  for (int c = 0; c < P / 4; ++c) {
    f2 v[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float qs[2];
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const float xv = k ? hi_of(x[4 * c + i]) : lo_of(x[4 * c + i]);
        const float ax = fminf(fabsf((xv * isT) * ia), 6.f);
        const float p2 = __uint_as_float(max(__float_as_uint(ax) & 0x7F800000u, 0x3F800000u));  // 1, 2 or 4
        const float magic = p2 * 6291456.f;
        const float qm = __fsub_rn(__fadd_rn(ax, magic), magic);
        const float h = qm + copysignf(0.25f * p2, ax - qm);
        const float half = h < 2.f ? 0.25f : (h < 4.f ? 0.5f : 1.f);
        const float lo = h - half, hi = h + half;
        const float d = fmaf(-(h * e), sT, fabsf(xv));
        const bool lo_even = lo == 0.f || lo == 1.f || lo == 2.f || lo == 4.f;
        qs[k] = copysignf(fminf(d > 0.f ? hi : (d < 0.f ? lo : (lo_even ? lo : hi)), 6.f), xv);
      }
      v[i] = pk(qs[0], qs[1]);
    }
    cw[c] = e2m1_no_negzero(e2m1_word(v));
  }
}

// Pass 2: group scales and codes of the grid's items.
template <int FMT, int E, int XDT, bool BSAME, bool REV>
__device__ __forceinline__ void act_quant(const ActProblem& p) {
  const int lane = threadIdx.x & 31;
  float sT = 1.f;
  if (FMT == FMT_NVFP4) {
    const float amax = __uint_as_float(ld_volatile(&p.hdr->amax_bits));
    sT = amax == 0.f ? 1.f : __double2float_rn((double)amax / 2688.0);
    if (sT == 0.f) sT = 0x1p-149f;
  }
  if (blockIdx.x == 0 && threadIdx.x == 0 && p.sT_out) *p.sT_out = sT;
  const double sTd = (double)sT;
  const float isT = FMT == FMT_NVFP4 ? __frcp_rn(sT) : 1.f;
  const bool sT_ok = FMT != FMT_NVFP4 || in_range(isT);
  const float qmax = fmt_e2m1(FMT) ? 6.f : 7.f;
  const int lpg = p.G > E ? p.G / E : 1;  // lanes per group
  const bool leader = (lane & (lpg - 1)) == 0;
  const int asz = FMT == FMT_INT4 ? 2 : 1;
  uint32_t* codes = reinterpret_cast<uint32_t*>(p.codes);
  unsigned char* astore = reinterpret_cast<unsigned char*>(p.a_store);
  bool bad = false;
  ActCols<E, BSAME> bc;
  int64_t s_have = -1;
  act_stream<E, REV>(p, [&](int64_t r, int, int64_t s, int64_t col, bool active, const unsigned char* row) {
    if (s != s_have) {  // warp-uniform
      bc.load(p, col);
      s_have = s;
    }
    f2 x[E / 2];
    act_row<E, XDT, BSAME>(row, lane, bc, x);
    float m = absmax_pairs<E / 2>(x);
    if (FMT != FMT_NVFP4) bad |= !(m <= 3.402823466e38f);  // NVFP4 checked in the amax pass
    if (FMT == FMT_INT4 && E == 32) {
#pragma unroll
      for (int o = 1; o < 8; o <<= 1)
        if (o < lpg) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    }
    if (!active) return;  // whole groups are inactive together (K is a multiple of G)
    // a = Proj(m / qmax): certified fp32 value, fp64 when ambiguous; 1 for a zero group
    bool amb = false;
    float a = a_fast<FMT>(m, qmax, isT, amb);
    if (amb) a = m == 0.f ? 1.f : (float)a_project<FMT>((double)m / (double)qmax, sTd);
    // 1/a: exact for a power of two
    const float ia = fmt_pow2(FMT) ? __uint_as_float(0x7F000000u - __float_as_uint(a)) : __frcp_rn(a);
    const bool ok = sT_ok && in_range(ia);
    uint32_t cw[E / 8];
    bool near = !ok;
    if (FMT == FMT_MXFP4) {
      // x / a is exact: the hardware conversion is the grid decision
      const f2 ia2 = splat(ia);
#pragma unroll
      for (int i = 0; i < E / 2; ++i) x[i] = mul2(x[i], ia2);
#pragma unroll
      for (int c = 0; c < E / 8; ++c) cw[c] = e2m1_no_negzero(e2m1_word(x + 4 * c));
    } else if (FMT == FMT_NVFP4) {
      // codes of a +-2^-20 relative bracket of the candidate x (1/s_T)(1/a);
      // the decision is certified where both ends agree
      const f2 cl = splat(isT * ia * (1.f - 0x1p-20f)), chh = splat(isT * ia * (1.f + 0x1p-20f));
#pragma unroll
      for (int c = 0; c < E / 8; ++c) {
        f2 lo[4], hi[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          lo[i] = mul2(x[4 * c + i], cl);
          hi[i] = mul2(x[4 * c + i], chh);
        }
        const uint32_t wl = e2m1_word(lo);
        near |= wl != e2m1_word(hi);
        cw[c] = e2m1_no_negzero(wl);
      }
    } else {
      // round half to even by adding 1.5 * 2^23 (exact for a power-of-two a;
      // guarded against the rounding of 1/a otherwise)
      const f2 ia2 = splat(ia), m2 = splat(12582912.f);
      float rmax = 0.f;
#pragma unroll
      for (int c = 0; c < E / 8; ++c) {
        f2 t[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          t[i] = fma2(x[4 * c + i], ia2, m2);
          if (FMT == FMT_INT4) {
            const f2 rr = fma2(x[4 * c + i], splat(-ia), add2(t[i], splat(-12582912.f)));  // q - x/a
            rmax = max3_nan(rmax, fabsf(lo_of(rr)), fabsf(hi_of(rr)));
          }
        }
        cw[c] = int4_word(t);
      }
      if (FMT == FMT_INT4) near |= rmax > 0.5f - kGuard;
    }
    if (near) {
      if (ok && FMT == FMT_INT4)
        int_exact_lane<E / 2>(x, ia, a, cw);
      else if (ok && FMT == FMT_NVFP4)
        e2m1_exact_lane<E / 2>(x, isT, ia, a, sT, cw);
      else
        act_exact<FMT, E, XDT>(row, p, lane, col, isT, ia, ok, a, sTd, cw);
    }
    // codes: E/2 bytes of the lane at (r K + col) / 2
    uint32_t* cp = codes + ((r * p.K + col) >> 3);
    if (E == 32 && p.codes_vec)
      *reinterpret_cast<uint4*>(cp) = make_uint4(cw[0], cw[E > 8 ? 1 : 0], cw[E > 16 ? 2 : 0], cw[E > 16 ? 3 : 0]);
    else if (E == 16 && p.codes_vec)
      *reinterpret_cast<uint2*>(cp) = make_uint2(cw[0], cw[E > 8 ? 1 : 0]);
    else {
#pragma unroll
      for (int c = 0; c < E / 8; ++c) cp[c] = cw[c];
    }
    if (leader) a_store_f<FMT>(astore + (r * p.nb + (col >> p.lgG)) * asz, 0, a);
  });
  if (FMT != FMT_NVFP4 && __any_sync(0xffffffffu, bad) && (threadIdx.x & 31) == 0)
    atomicOr(&p.hdr->flags, kFlagNonFinite);
}

// INT4, MXINT4, MXFP4: one pass.
template <int FMT, int E, int XDT, bool BSAME>
__global__ void __launch_bounds__(kActThreads, act_ctas_per_sm(E)) k_act(ActProblem p) {
  act_quant<FMT, E, XDT, BSAME, false>(p);
}

// NVFP4: the amax pass, a grid-wide barrier (the grid is co-resident: a
// cooperative launch), then the quantization pass over the same items in
// reverse order, so that the rows this warp read last, the likeliest to be
// still in L2, come first.  The barrier's wait is bounded (kFlagTimeout).
template <int XDT, bool BSAME>
__global__ void __launch_bounds__(kActThreads, kActNvCtasPerSm) k_act_nv(ActProblem p) {
  act_amax<16, XDT, BSAME>(p);
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    atomicAdd(&p.hdr->gbar, 1u);
    const unsigned long long t0 = global_ns();
    while (ld_acquire_gpu(&p.hdr->gbar) < gridDim.x)
      if (wait_expired(&p.hdr->flags, t0)) break;
  }
  __syncthreads();
  if (ld_volatile(&p.hdr->flags) & (kFlagNonFinite | kFlagTimeout)) return;
  act_quant<FMT_NVFP4, 16, XDT, BSAME, true>(p);
}

template <int FMT, int E, int XDT, bool BSAME>
static cudaError_t act_launch(const ActProblem& p, int sms, cudaStream_t st) {
  void (*kern)(ActProblem);
  if constexpr (FMT == FMT_NVFP4)
    kern = k_act_nv<XDT, BSAME>;
  else
    kern = k_act<FMT, E, XDT, BSAME>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kActSmem);
  if (e != cudaSuccess) return e;
  int per_sm = 0;
  if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kActThreads, kActSmem)) != cudaSuccess)
    return e;
  if (per_sm < 1) return cudaErrorInvalidConfiguration;
  // one resident wave: every CTA runs at once and takes equal ranges of the
  // items, so no second wave leaves SMs idle at the tail; small inputs get
  // fewer CTAs (kActMinItems items per warp at least)
  const int64_t items = (int64_t)p.n_slabs * ((p.M + ActGeo<E>::kRows - 1) / ActGeo<E>::kRows);
  const int64_t per_cta = (int64_t)kActWarps * kActMinItems;
  const int64_t want = (int64_t)sms * per_sm;
  const int grid = (int)((items + per_cta - 1) / per_cta < want ? (items + per_cta - 1) / per_cta : want);
  if (FMT != FMT_NVFP4) {
    kern<<<grid, kActThreads, kActSmem, st>>>(p);
    return cudaGetLastError();
  }
  ActProblem arg = p;
  void* args[] = {&arg};
  return cudaLaunchCooperativeKernel(reinterpret_cast<const void*>(kern), dim3(grid), dim3(kActThreads), args,
                                     (size_t)kActSmem, st);
}

template <int FMT, int E>
static cudaError_t act_fmt(ActProblem p, int xdt, int sms, cudaStream_t st) {
  p.n_slabs = (int)((p.K + ActGeo<E>::kSlab - 1) / ActGeo<E>::kSlab);
  p.codes_vec = ((uintptr_t)p.codes % (E / 2)) == 0;
  const bool same = p.col_dt == xdt;
  if (xdt == DT_BF16)
    return same ? act_launch<FMT, E, DT_BF16, true>(p, sms, st) : act_launch<FMT, E, DT_BF16, false>(p, sms, st);
  return same ? act_launch<FMT, E, DT_F16, true>(p, sms, st) : act_launch<FMT, E, DT_F16, false>(p, sms, st);
}

}  // namespace dq

extern "C" int dq_act_quant(const void* X, int x_dtype, int64_t rows, int64_t cols, const void* col_scales,
                            int col_dtype, int format, int group, const dq_outputs* out, void* workspace,
                            size_t workspace_bytes, void* stream) {
  if (rows <= 0 || cols <= 0 || group <= 0 || cols % group != 0) return DQ_EINVAL;
  if (format < DQ_INT4 || format > DQ_MXFP8) return DQ_EINVAL;
  if (format == DQ_MXINT8 || format == DQ_MXFP8) return DQ_EUNSUPPORTED;  // 4-bit codes only
  if ((format == DQ_MXINT4 || format == DQ_MXFP4) && group != 32) return DQ_EUNSUPPORTED;
  if (format == DQ_NVFP4 && group != 16) return DQ_EUNSUPPORTED;
  if (group < 8 || group > 256 || (group & (group - 1)) != 0) return DQ_EUNSUPPORTED;
  if (x_dtype != DQ_BF16 && x_dtype != DQ_F16) return DQ_EUNSUPPORTED;  // x b exact in fp32 needs <= 11-bit x
  if (col_dtype != DQ_BF16 && col_dtype != DQ_F16) return DQ_EUNSUPPORTED;
  if (rows > ((int64_t)1 << 40) / cols) return DQ_EUNSUPPORTED;
  if (!X || ((uintptr_t)X % 16) != 0 || !col_scales || ((uintptr_t)col_scales % 2) != 0) return DQ_EINVAL;
  if (!out || !out->codes || !out->block_scales || ((uintptr_t)out->codes % 4) != 0 ||
      ((uintptr_t)out->block_scales % 2) != 0 || (format == DQ_NVFP4 && !out->tensor_scale))
    return DQ_EINVAL;
  if (!workspace || ((uintptr_t)workspace % 256) != 0) return DQ_EINVAL;
  if (workspace_bytes < DQ_ACT_WORKSPACE_BYTES) return DQ_EWORKSPACE;
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return DQ_ECUDA;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return DQ_ECUDA;
  dq::ActProblem p;
  p.X = X;
  p.b_store = col_scales;
  p.col_dt = col_dtype;
  p.G = group;
  p.lgG = __builtin_ctz((unsigned)group);
  p.M = rows;
  p.K = cols;
  p.nb = (int)(cols / group);
  p.codes = out->codes;
  p.a_store = out->block_scales;
  p.sT_out = out->tensor_scale;
  p.hdr = static_cast<dq::WsHeader*>(workspace);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(workspace, 0, sizeof(dq::WsHeader), st) != cudaSuccess) return DQ_ECUDA;
  cudaError_t e;
  switch (format) {
    case DQ_INT4:
      e = group == 8 ? dq::act_fmt<dq::FMT_INT4, 8>(p, x_dtype, sms, st)
                     : (group == 16 ? dq::act_fmt<dq::FMT_INT4, 16>(p, x_dtype, sms, st)
                                    : dq::act_fmt<dq::FMT_INT4, 32>(p, x_dtype, sms, st));
      break;
    case DQ_MXINT4: e = dq::act_fmt<dq::FMT_MXINT4, 32>(p, x_dtype, sms, st); break;
    case DQ_MXFP4: e = dq::act_fmt<dq::FMT_MXFP4, 32>(p, x_dtype, sms, st); break;
    default: e = dq::act_fmt<dq::FMT_NVFP4, 16>(p, x_dtype, sms, st); break;
  }
  return e == cudaSuccess ? DQ_OK : DQ_ECUDA;
}
