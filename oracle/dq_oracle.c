/*
 * dq_oracle.c -- plain fp64 CPU reference of the DualQuant dual-scale
 * block-coordinate-descent (BCD) weight-quantization solver.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the oracle that the CUDA path is
 * checked against.  Only the tests, the smoke check and the CPU-baseline leg of
 * the benchmark load it; the product path never does.  It shares no code, header
 * or table with the CUDA library.
 *
 * Sources (web pages on the method; cited by title and section):
 *  [R5] "DualQuant: Calibration-Free Dual-Scale Weight and Activation
 *       Quantization" reproduction README (daiwk.github.io): "Original paper"
 *       flowchart, "Core equations", "Local reproduction".
 *  [P2] "DualQuant: Dual-scale Calibration-free Weight-and-Activation
 *       Quantization for LLMs" (arXiv 2610.13767) summary (paperlayer.ai):
 *       §3 Quantization preliminaries, §4.3 MSE optimization via BCD,
 *       App. A.1 variable splitting, App. B closed-form solutions.
 *  [L1] SQuant lesson, "Chapter 2: Quantization from Scratch" (uniform
 *       quantizer, worked int8 example).
 *  [T4] "Round-to-Nearest & basic weight quantization" tutorial, sections
 *       "Round-to-Nearest (RTN)" and "Absmax (Symmetric) Quantization".
 *
 * Everything here is written as the plain definition: loops in natural order
 * (j ascending inside a block, i ascending inside a column), fp64 arithmetic,
 * no blocking or fusion.  Readings of points the pages leave open:
 *  - Q rounds to the nearest grid value, ties to the "even" neighbour (even
 *    integer on the INT4 and INT8 grids; even mantissa bit for E2M1 and
 *    E4M3), values past the ends clip.
 *    The decision compares W with boundary*(a*b), which is exact in fp64
 *    because a*b and boundary*(a*b) have few significant bits.
 *  - Projection onto admissible inverse scales = nearest admissible value in
 *    linear distance (the minimiser of the 1-D quadratic); fp16/bf16/E4M3 ties
 *    go to the even mantissa, E8M0 ties go to the larger power of two.
 *  - NVFP4: one fp32 tensor scale s_T = fp32(amax / (6*448)) fixed at init;
 *    block inverse scale a = s_T * e with e a positive finite E4M3 value.
 *  - "Scale 1 for an all-zero code slice": a = 1 (INT4, MXINT4), e = 1 (NVFP4),
 *    b = 1.
 *  - Init: b = 1 and a = Proj(absmax(block) / qmax), qmax = 7 (INT4 grid
 *    [-8,7]), 127 (INT8 grid [-128,127]) or 6 (E2M1); an all-zero block gets
 *    scale 1.  Variants: the per-column L1-norm init (init_l1) and a warm
 *    start from given scales.
 *  - MXINT8 ([P2] App. G.2, 8-bit W+A quantization with MXINT8 and MXFP8): the INT8
 *    codebook [-128,127] with E8M0 power-of-two block scales, group 32, one
 *    byte per code; the OCP element's fixed 2^-6 factor is a power of two and
 *    is absorbed into the block scale.
 *  - MXFP8 (the same passage): the FP8 E4M3 codebook (1 sign, 4 exponent bits
 *    with bias 7, 3 mantissa bits, subnormals, largest finite value 448, no
 *    infinities) with E8M0 power-of-two block scales, group 32, absmax qmax
 *    448, ties to the value with an even mantissa bit, one byte per code (the
 *    E4M3 bit pattern; zero is always 0x00).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define DQO_OK 0
#define DQO_EINVAL 1
#define DQO_ENONFINITE 4
#define DQO_ENOMEM 6

/* formats (numbering mirrors the library's public enum by value only) */
#define DQO_INT4 0
#define DQO_MXINT4 1
#define DQO_NVFP4 2
#define DQO_MXFP4 3 /* E2M1 grid with E8M0 block scales (the MX family's FP4 member) */
#define DQO_MXINT8 4 /* INT8 grid [-128,127] with E8M0 block scales (the MX family's INT8 member) */
#define DQO_MXFP8 5  /* FP8 E4M3 grid with E8M0 block scales (the MX family's FP8 E4M3 member) */
/* element dtypes */
#define DQO_F32 0
#define DQO_BF16 1
#define DQO_F16 2
/* projection kinds for dqo_project() */
#define DQO_PROJ_F16 0
#define DQO_PROJ_BF16 1
#define DQO_PROJ_E4M3 2
#define DQO_PROJ_E8M0 3

/* ------------------------------------------------------------------------ */
/* Format grids Q ([P2] §3; [R5] "Local reproduction": INT4 codebook [-8,7]). */

static const double INT4_GRID[16] = {-8, -7, -6, -5, -4, -3, -2, -1, 0, 1, 2, 3, 4, 5, 6, 7};
static const unsigned char INT4_EVEN[16] = {1, 0, 1, 0, 1, 0, 1, 0, 1, 0, 1, 0, 1, 0, 1, 0};
/* E2M1 values and, per value, whether its mantissa bit is 0 ("even").
 * magnitudes 0,0.5,1,1.5,2,3,4,6 have encodings 000,001,010,011,100,101,110,111 */
static const double E2M1_GRID[15] = {-6, -4, -3, -2, -1.5, -1, -0.5, 0, 0.5, 1, 1.5, 2, 3, 4, 6};
static const unsigned char E2M1_EVEN[15] = {0, 1, 0, 1, 0, 1, 0, 1, 0, 1, 0, 1, 0, 1, 0};
/* INT8 codebook -128..127 and its even flags (filled by grids_init(), with the E4M3 table) */
static double INT8_GRID[256];
static unsigned char INT8_EVEN[256];
/* E4M3 values in ascending order (253: +-126 nonzero magnitudes and zero) and
 * whether each has mantissa bit 0; the magnitude with exponent field e and
 * mantissa m is m * 2^-9 for e = 0 and (1 + m/8) * 2^(e-7) otherwise, the
 * pattern e = 15, m = 7 being NaN. */
static double E4M3_GRID[253];
static unsigned char E4M3_EVEN[253];
static void grids_init(void) {
  for (int k = 0; k < 256; ++k) {
    INT8_GRID[k] = (double)(k - 128);
    INT8_EVEN[k] = (unsigned char)((k - 128) % 2 == 0);
  }
  double mag[127];
  unsigned char ev[127];
  int n = 0;
  for (int e = 0; e < 16; ++e)
    for (int m = 0; m < 8; ++m) {
      if (e == 15 && m == 7) continue;
      mag[n] = (e == 0) ? ldexp((double)m, -9) : ldexp(1.0 + m / 8.0, e - 7);
      ev[n] = (unsigned char)(m % 2 == 0);
      ++n;
    }
  /* mag[] ascends with the bit pattern; mirror it for the negative half */
  for (int k = 0; k < 126; ++k) {
    E4M3_GRID[k] = -mag[126 - k];
    E4M3_EVEN[k] = ev[126 - k];
  }
  for (int k = 0; k < 127; ++k) {
    E4M3_GRID[126 + k] = mag[k];
    E4M3_EVEN[126 + k] = ev[k];
  }
}

/*
 * Nearest grid value to w/scale ([L1] Ch. 2 round-to-nearest then clip;
 * [P2] §3 "nearest representable value").  grid[] is sorted ascending; the
 * boundary between grid[k] and grid[k+1] is their midpoint h_k.  For scale > 0,
 * w/scale > h_k exactly when w > h_k*scale, so the decision is a scan of
 * comparisons.  An exact tie (w == h_k*scale) picks the neighbour flagged even.
 * Values below the first / above the last boundary land on the end values
 * (clip).  Returns the grid index.
 */
int dqo_quant_index(double w, double scale, const double* grid, const unsigned char* even, int n) {
  int idx = 0;
  for (int k = 0; k + 1 < n; ++k) {
    double h = 0.5 * (grid[k] + grid[k + 1]);
    double t = h * scale;
    if (w > t) {
      idx = k + 1;
    } else if (w == t) {
      idx = even[k] ? k : k + 1;
      break;
    } else {
      break;
    }
  }
  return idx;
}

/* Symmetric absmax scale max|w|/qmax ([T4] "Absmax (Symmetric) Quantization";
 * [P2] §3 "Δ = max(|W|)/qmax"). */
double dqo_absmax_scale(const double* w, int64_t n, double qmax) {
  double m = 0.0;
  for (int64_t i = 0; i < n; ++i) {
    double v = fabs(w[i]);
    if (v > m) m = v;
  }
  return m / qmax;
}

/* ------------------------------------------------------------------------ */
/* Projection onto admissible (hardware-legal) positive inverse scales
 * ([R5] "Core equations": "Projection is on inverse scales"; [P2] App. B
 * "projecting to the nearest representable value").                       */

/*
 * Nearest positive finite value of a binary float format with `mbits`
 * explicit mantissa bits, smallest normal exponent `emin` (subnormals below
 * it) and largest finite value `vmax`.  Ties go to the value whose last
 * mantissa bit is 0.  Anything at or below the smallest positive value maps to
 * it (zero is not admissible); anything at or above vmax maps to vmax.
 */
static double project_float(double v, int mbits, int emin, double vmax) {
  double minsub = ldexp(1.0, emin - mbits);
  if (!(v > minsub)) return minsub;
  if (v >= vmax) return vmax;
  int e;
  frexp(v, &e);           /* v = f * 2^e, f in [0.5, 1) -> binade exponent e-1 */
  int E = e - 1;
  if (E < emin) E = emin; /* subnormal range: fixed spacing */
  double ulp = ldexp(1.0, E - mbits);
  double k = floor(v / ulp); /* v/ulp is an exact power-of-two scaling */
  double lo = k * ulp, hi = (k + 1.0) * ulp, mid = (k + 0.5) * ulp;
  double r;
  if (v < mid)
    r = lo;
  else if (v > mid)
    r = hi;
  else
    r = (fmod(k, 2.0) == 0.0) ? lo : hi;
  if (r < minsub) r = minsub;
  if (r > vmax) r = vmax;
  return r;
}

/* E8M0 power-of-two scales with exponent in [-126, 126] ([R5] "Local
 * reproduction"); nearest in linear distance, a tie (1.5 * 2^k) goes up. */
static double project_pow2(double v) {
  if (!(v > ldexp(1.0, -126))) return ldexp(1.0, -126);
  if (v >= ldexp(1.0, 126)) return ldexp(1.0, 126);
  int e;
  frexp(v, &e);
  double lo = ldexp(1.0, e - 1), hi = ldexp(1.0, e);
  double mid = 1.5 * lo;
  double r = (v < mid) ? lo : hi;
  if (r > ldexp(1.0, 126)) r = ldexp(1.0, 126);
  return r;
}

double dqo_project(int kind, double v) {
  switch (kind) {
    case DQO_PROJ_F16: return project_float(v, 10, -14, 65504.0);
    case DQO_PROJ_BF16: return project_float(v, 7, -126, ldexp(255.0, 120)); /* (2-2^-7)*2^127 */
    case DQO_PROJ_E4M3: return project_float(v, 3, -6, 448.0);
    case DQO_PROJ_E8M0: return project_pow2(v);
  }
  return NAN;
}

/* ------------------------------------------------------------------------ */
/* Storage encodings of admissible values (all inputs are exactly
 * representable; these only rewrite them as bit patterns).                 */

static uint16_t encode_float_bits(double v, int mbits, int emin, int ebits) {
  /* v > 0 and exactly representable */
  int e;
  frexp(v, &e);
  int E = e - 1;
  int bias = 1 - emin;
  uint32_t expfield, mant;
  if (E < emin) {
    expfield = 0;
    mant = (uint32_t)ldexp(v, mbits - emin);
  } else {
    expfield = (uint32_t)(E + bias);
    mant = (uint32_t)(ldexp(v, mbits - E) - ldexp(1.0, mbits));
  }
  (void)ebits;
  return (uint16_t)((expfield << mbits) | mant);
}

static uint8_t e2m1_nibble(double q) {
  double m = fabs(q);
  uint8_t code;
  if (m == 0.0) return 0; /* zero is always the +0 encoding */
  if (m == 0.5) code = 1;
  else if (m == 1.0) code = 2;
  else if (m == 1.5) code = 3;
  else if (m == 2.0) code = 4;
  else if (m == 3.0) code = 5;
  else if (m == 4.0) code = 6;
  else code = 7; /* 6.0 */
  return (uint8_t)((q < 0 ? 8 : 0) | code);
}

/* ------------------------------------------------------------------------ */
/* Solver state and steps                                                    */

typedef struct {
  int64_t M, N;
  int fmt, G, nb;
  int col_kind;  /* projection kind for b */
  double sT;     /* NVFP4 tensor scale (1 otherwise) */
  const double* W;
} problem;

/* the formats on the E2M1 grid */
static int e2m1_grid(int fmt) { return fmt == DQO_NVFP4 || fmt == DQO_MXFP4; }

static double qmax_of(int fmt) {
  if (e2m1_grid(fmt)) return 6.0;
  if (fmt == DQO_MXINT8) return 127.0;
  if (fmt == DQO_MXFP8) return 448.0;
  return 7.0;
}

/* formats with 8-bit codes (one byte per element) */
static int byte_codes(int fmt) { return fmt == DQO_MXINT8 || fmt == DQO_MXFP8; }

/* block inverse scale value a from its stored factor (NVFP4 stores e, a = s_T*e) */
static double a_value(const problem* p, double stored) { return p->fmt == DQO_NVFP4 ? p->sT * stored : stored; }

/* projection of an LS inverse-scale value onto F_a; returns the stored factor */
static double project_a(const problem* p, double v) {
  if (p->fmt == DQO_INT4) return dqo_project(DQO_PROJ_F16, v);
  if (p->fmt == DQO_MXINT4 || p->fmt == DQO_MXFP4 || p->fmt == DQO_MXINT8 || p->fmt == DQO_MXFP8)
    return dqo_project(DQO_PROJ_E8M0, v);
  return dqo_project(DQO_PROJ_E4M3, v / p->sT); /* nearest s_T*e to v */
}

/* Q(W/(a b)) -> grid value ([R5] flowchart "Black-box format grid Q") */
static double quant_value(const problem* p, double w, double a, double b) {
  double ab = a * b;
  if (e2m1_grid(p->fmt)) return E2M1_GRID[dqo_quant_index(w, ab, E2M1_GRID, E2M1_EVEN, 15)];
  if (p->fmt == DQO_MXINT8) return INT8_GRID[dqo_quant_index(w, ab, INT8_GRID, INT8_EVEN, 256)];
  if (p->fmt == DQO_MXFP8) return E4M3_GRID[dqo_quant_index(w, ab, E4M3_GRID, E4M3_EVEN, 253)];
  return INT4_GRID[dqo_quant_index(w, ab, INT4_GRID, INT4_EVEN, 16)];
}

/* requantize every element with the current (a, b)  ([R5] "Core equations":
 * requantize after each update).  q is [M][N]. */
void dqo_requant_impl(const problem* p, const double* astored, const double* b, double* q) {
  int64_t M = p->M, N = p->N;
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < M; ++i)
    for (int64_t j = 0; j < N; ++j) {
      double a = a_value(p, astored[i * p->nb + j / p->G]);
      q[i * N + j] = quant_value(p, p->W[i * N + j], a, b[j]);
    }
}

/*
 * Row/block update with codes fixed ([R5] "Core equations": with R = Q̂ D_b,
 * a_i <- Proj_Fa( sum_j W_ij R_ij / sum_j R_ij^2 ), scale 1 for an all-zero
 * code slice).  `raw` (optional) receives the unprojected least-squares value
 * (NaN for an all-zero slice).
 */
void dqo_row_update_impl(const problem* p, const double* q, const double* b, double* astored, double* raw) {
  int64_t M = p->M, N = p->N;
  int G = p->G, nb = p->nb;
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < M; ++i)
    for (int g = 0; g < nb; ++g) {
      double num = 0.0, den = 0.0;
      for (int jj = 0; jj < G; ++jj) {
        int64_t j = (int64_t)g * G + jj;
        double R = q[i * N + j] * b[j];
        num += p->W[i * N + j] * R;
        den += R * R;
      }
      double v = (den == 0.0) ? NAN : num / den;
      if (raw) raw[i * nb + g] = v;
      astored[i * nb + g] = (den == 0.0) ? 1.0 : project_a(p, v);
    }
}

/*
 * Column update with codes fixed ([R5] "Core equations": with S = D_a Q̂,
 * b_j <- Proj_Fb( sum_i W_ij S_ij / sum_i S_ij^2 ), scale 1 for an all-zero
 * code slice).  Column sums run over i ascending; the loop nest walks rows in
 * the outer loop so memory is read row by row, which does not change the
 * per-column summation order.
 */
void dqo_col_update_impl(const problem* p, const double* q, const double* astored, double* b, double* raw) {
  int64_t M = p->M, N = p->N;
  const int64_t CH = 256;
  int64_t nch = (N + CH - 1) / CH;
#pragma omp parallel for schedule(static)
  for (int64_t c = 0; c < nch; ++c) {
    double num[256], den[256];
    int64_t j0 = c * CH, j1 = j0 + CH < N ? j0 + CH : N;
    for (int64_t j = j0; j < j1; ++j) num[j - j0] = den[j - j0] = 0.0;
    for (int64_t i = 0; i < M; ++i)
      for (int64_t j = j0; j < j1; ++j) {
        double S = a_value(p, astored[i * p->nb + j / p->G]) * q[i * N + j];
        num[j - j0] += p->W[i * N + j] * S;
        den[j - j0] += S * S;
      }
    for (int64_t j = j0; j < j1; ++j) {
      double d = den[j - j0];
      double v = (d == 0.0) ? NAN : num[j - j0] / d;
      if (raw) raw[j] = v;
      b[j] = (d == 0.0) ? 1.0 : dqo_project(p->col_kind, v);
    }
  }
}

/* reconstruction MSE (1/MN) sum (W - a q b)^2: rows summed in order, each row
 * summed over j ascending. */
double dqo_mse_impl(const problem* p, const double* q, const double* astored, const double* b) {
  int64_t M = p->M, N = p->N;
  double* rows = (double*)malloc(sizeof(double) * (size_t)M);
  if (!rows) return NAN;
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < M; ++i) {
    double s = 0.0;
    for (int64_t j = 0; j < N; ++j) {
      double r = p->W[i * N + j] - a_value(p, astored[i * p->nb + j / p->G]) * q[i * N + j] * b[j];
      s += r * r;
    }
    rows[i] = s;
  }
  double tot = 0.0;
  for (int64_t i = 0; i < M; ++i) tot += rows[i];
  free(rows);
  return tot / ((double)M * (double)N);
}

/* NVFP4 tensor scale from the largest magnitude the block scales must cover:
 * s_T = fp32(amax / (6*448)), 1 when amax = 0, the least positive fp32 when it
 * rounds to zero.  1 for the other formats. */
static void set_tensor_scale(problem* p, double amax) {
  if (p->fmt != DQO_NVFP4 || amax == 0.0) {
    p->sT = 1.0;
    return;
  }
  float s = (float)(amax / 2688.0);
  if (s == 0.0f) s = ldexpf(1.0f, -149); /* nearest positive fp32 */
  p->sT = (double)s;
}

/* Absmax RTN init ([T4] absmax; [P2] §3 symmetric scale; spec config:
 * beta = 1).  NVFP4 first fixes s_T = fp32(amax / (6*448)). */
static void init_scales(problem* p, double* astored, double* b) {
  int64_t M = p->M, N = p->N;
  double amax = 0.0;
  for (int64_t k = 0; k < M * N; ++k)
    if (fabs(p->W[k]) > amax) amax = fabs(p->W[k]);
  set_tensor_scale(p, amax);
  double qmax = qmax_of(p->fmt);
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < M; ++i)
    for (int g = 0; g < p->nb; ++g) {
      double m = dqo_absmax_scale(p->W + i * N + (int64_t)g * p->G, p->G, 1.0);
      astored[i * p->nb + g] = (m == 0.0) ? 1.0 : project_a(p, m / qmax);
    }
  for (int64_t j = 0; j < N; ++j) b[j] = 1.0;
}

/* ------------------------------------------------------------------------ */
/* Exact sums of magnitudes.  Every input value (fp32, bf16 or fp16) is an
 * integer multiple of 2^-149 below 2^128, so a sum of fewer than 2^63 of them
 * is an integer below 2^340 in units of 2^-149.  It is held exactly in a
 * 384-bit unsigned integer and rounded once to fp64, to nearest with ties to
 * even. */
#define XS_LIMBS 6
typedef struct {
  uint64_t limb[XS_LIMBS]; /* little-endian 64-bit limbs, units of 2^-149 */
} xsum;

static void xsum_add(xsum* s, double v) { /* v >= 0, a multiple of 2^-149 below 2^128 */
  if (v == 0.0) return;
  int e;
  double f = frexp(v, &e);             /* v = f * 2^e with 0.5 <= f < 1 */
  uint64_t m = (uint64_t)ldexp(f, 53); /* v = m * 2^(e-53), m < 2^53 */
  int sh = e - 53 + 149;               /* v = m * 2^sh units */
  if (sh < 0) {                        /* m has at least -sh trailing zero bits */
    m >>= -sh;
    sh = 0;
  }
  int li = sh / 64, bo = sh % 64;
  uint64_t lo = m << bo, hi = bo ? m >> (64 - bo) : 0;
  uint64_t old = s->limb[li];
  s->limb[li] += lo;
  uint64_t carry = s->limb[li] < old;
  for (int k = li + 1; k < XS_LIMBS && (hi || carry); ++k) {
    old = s->limb[k];
    s->limb[k] += hi + carry; /* hi < 2^53: no overflow of the addend */
    carry = s->limb[k] < old;
    hi = 0;
  }
}

static int xsum_bit(const xsum* s, int i) { return (int)((s->limb[i / 64] >> (i % 64)) & 1u); }

static double xsum_round(const xsum* s) {
  int top = -1;
  for (int i = 64 * XS_LIMBS - 1; i >= 0; --i)
    if (xsum_bit(s, i)) {
      top = i;
      break;
    }
  if (top < 0) return 0.0;
  if (top < 53) return ldexp((double)s->limb[0], -149); /* fewer than 54 bits: exact */
  int low = top - 52; /* keep bits low..top */
  uint64_t mant = 0;
  for (int i = 0; i < 53; ++i) mant |= (uint64_t)xsum_bit(s, low + i) << i;
  int rbit = xsum_bit(s, low - 1), sticky = 0;
  for (int i = 0; i < low - 1; ++i) sticky |= xsum_bit(s, i);
  if (rbit && (sticky || (mant & 1u))) mant += 1; /* 2^53 is still exact */
  return ldexp((double)mant, low - 149);
}

/* sum of |x_k| over n values, exact then rounded once to fp64 (x_k must be
 * fp32-representable) */
double dqo_exact_abs_sum(const double* x, int64_t n) {
  xsum s;
  memset(&s, 0, sizeof s);
  for (int64_t k = 0; k < n; ++k) xsum_add(&s, fabs(x[k]));
  return xsum_round(&s);
}

/*
 * Per-column L1-norm init ([P2] §5.3: format-native row absmax scales and
 * per-column L1-norm scales).  The pages name the norm only; readings taken:
 *  - the column scale is the column's L1 norm relative to the mean column L1
 *    norm: b_j = Proj_Fb(c_j / mu), c_j = sum_i |W_ij|, mu = (sum_ij |W_ij|) / N,
 *    each sum exact and rounded once to fp64; b_j = 1 for an all-zero column;
 *  - the block scales are the absmax RTN scales of the column-scaled matrix
 *    W D_b^-1: a = Proj_Fa(max_j (|W_ij| / b_j) / qmax), 1 for an all-zero block;
 *  - NVFP4: s_T is taken from the same matrix, fp32(max_ij (|W_ij| / b_j) / 2688).
 * Every quotient is one correctly rounded fp64 division.  With all b_j = 1 this
 * is exactly the absmax RTN init.
 */
static void init_l1(problem* p, double* astored, double* b) {
  int64_t M = p->M, N = p->N;
  double mu = dqo_exact_abs_sum(p->W, M * N) / (double)N;
#pragma omp parallel for schedule(static)
  for (int64_t j = 0; j < N; ++j) {
    xsum c;
    memset(&c, 0, sizeof c);
    for (int64_t i = 0; i < M; ++i) xsum_add(&c, fabs(p->W[i * N + j]));
    double cj = xsum_round(&c);
    b[j] = (cj == 0.0 || mu == 0.0) ? 1.0 : dqo_project(p->col_kind, cj / mu);
  }
  double amax = 0.0;
  for (int64_t k = 0; k < M * N; ++k) {
    double v = fabs(p->W[k]) / b[k % N];
    if (v > amax) amax = v;
  }
  set_tensor_scale(p, amax);
  double qmax = qmax_of(p->fmt);
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < M; ++i)
    for (int g = 0; g < p->nb; ++g) {
      double m = 0.0;
      for (int jj = 0; jj < p->G; ++jj) {
        int64_t j = (int64_t)g * p->G + jj;
        double v = fabs(p->W[i * N + j]) / b[j];
        if (v > m) m = v;
      }
      astored[i * p->nb + g] = (m == 0.0) ? 1.0 : project_a(p, m / qmax);
    }
}

/* Warm start: the caller's scales are the initial iterate.  Each must be
 * admissible (an element of its set, so projection leaves it unchanged), and
 * the NVFP4 tensor scale a positive finite fp32 value. */
static int init_given(problem* p, const double* a0, const double* b0, double sT0, double* astored, double* b) {
  if (!a0 || !b0) return DQO_EINVAL;
  if (p->fmt == DQO_NVFP4) {
    if (!(sT0 > 0.0) || !isfinite(sT0) || (double)(float)sT0 != sT0) return DQO_EINVAL;
    p->sT = sT0;
  } else {
    p->sT = 1.0;
  }
  int akind = p->fmt == DQO_INT4 ? DQO_PROJ_F16 : (p->fmt == DQO_NVFP4 ? DQO_PROJ_E4M3 : DQO_PROJ_E8M0);
  for (int64_t k = 0; k < p->M * p->nb; ++k) {
    if (!(a0[k] > 0.0) || dqo_project(akind, a0[k]) != a0[k]) return DQO_EINVAL;
    astored[k] = a0[k];
  }
  for (int64_t j = 0; j < p->N; ++j) {
    if (!(b0[j] > 0.0) || dqo_project(p->col_kind, b0[j]) != b0[j]) return DQO_EINVAL;
    b[j] = b0[j];
  }
  return DQO_OK;
}

/* ------------------------------------------------------------------------ */
/* Public oracle entry points                                                */

static int load_problem(problem* p, const void* W, int wdt, int64_t M, int64_t N, int fmt, int G, int col_dt,
                        double** Wd_out) {
  if (!W || M <= 0 || N <= 0 || G <= 0 || N % G != 0 || N % 2 != 0) return DQO_EINVAL;
  if (fmt < 0 || fmt > 5 || (col_dt != DQO_F16 && col_dt != DQO_BF16)) return DQO_EINVAL;
  grids_init();
  double* Wd = (double*)malloc(sizeof(double) * (size_t)(M * N));
  if (!Wd) return DQO_ENOMEM;
  int bad = 0;
  for (int64_t k = 0; k < M * N; ++k) {
    double v;
    if (wdt == DQO_F32) {
      v = ((const float*)W)[k];
    } else if (wdt == DQO_BF16) {
      uint32_t u = (uint32_t)((const uint16_t*)W)[k] << 16;
      float f;
      memcpy(&f, &u, 4);
      v = f;
    } else {
      uint16_t h = ((const uint16_t*)W)[k];
      int s = h >> 15, e = (h >> 10) & 31, m = h & 1023;
      if (e == 31) v = m ? NAN : INFINITY;
      else if (e == 0) v = ldexp((double)m, -24);
      else v = ldexp((double)(m + 1024), e - 25);
      if (s) v = -v;
    }
    if (!isfinite(v)) bad = 1;
    Wd[k] = v;
  }
  if (bad) {
    free(Wd);
    return DQO_ENONFINITE;
  }
  p->M = M;
  p->N = N;
  p->fmt = fmt;
  p->G = G;
  p->nb = (int)(N / G);
  p->col_kind = (col_dt == DQO_F16) ? DQO_PROJ_F16 : DQO_PROJ_BF16;
  p->sT = 1.0;
  p->W = Wd;
  *Wd_out = Wd;
  return DQO_OK;
}

static void pack_codes(const problem* p, const double* q, uint8_t* codes) {
  int64_t M = p->M, N = p->N;
  if (p->fmt == DQO_MXINT8) { /* one two's-complement byte per element */
    for (int64_t k = 0; k < M * N; ++k) codes[k] = (uint8_t)((int)q[k] & 0xFF);
    return;
  }
  if (p->fmt == DQO_MXFP8) { /* one E4M3 bit pattern per element, zero as 0x00 */
    for (int64_t k = 0; k < M * N; ++k)
      codes[k] = (q[k] == 0.0) ? 0 : (uint8_t)((q[k] < 0 ? 0x80 : 0) | encode_float_bits(fabs(q[k]), 3, -6, 4));
    return;
  }
  for (int64_t i = 0; i < M; ++i)
    for (int64_t j = 0; j < N; j += 2) {
      uint8_t lo, hi;
      if (e2m1_grid(p->fmt)) {
        lo = e2m1_nibble(q[i * N + j]);
        hi = e2m1_nibble(q[i * N + j + 1]);
      } else {
        lo = (uint8_t)((int)q[i * N + j] & 0xF);
        hi = (uint8_t)((int)q[i * N + j + 1] & 0xF);
      }
      codes[(i * N + j) / 2] = (uint8_t)(lo | (hi << 4));
    }
}

/*
 * The whole solver ([R5] flowchart and "Core equations"; [P2] §4.3, §5.3):
 *   init (absmax RTN, b = 1); q = Q(W/(a b)); mse[0]
 *   for t = 1..iters:
 *     row update (codes fixed) -> project -> requantize
 *     column update (codes fixed) -> project -> requantize; mse[t]
 * Outputs (any may be NULL except mse when iters >= 0 is wanted):
 *   codes      [M][N/2] packed nibbles, even column in the low nibble (MXINT8:
 *              [M][N], one two's-complement byte per element; MXFP8: [M][N],
 *              one E4M3 bit pattern per element)
 *   a_out      [M][N/G] stored block scale values (fp16 value / 2^k / E4M3 e)
 *   b_out      [N] column inverse scales
 *   sT_out     NVFP4 tensor scale (1 for the other formats)
 *   mse        [iters+1]
 *   q_out      [M][N] final grid values
 *   trace_a    [(iters+1)][M][N/G] block scales after init and each iteration
 *   trace_b    [(iters+1)][N]
 */
/*
 * The solver.  mode 0: the dual-scale BCD iteration (row update, requantize,
 * column update, requantize).  The ablation modes of the DualQuant summary
 * (§5.3, Table 4: row scaling alone, column scaling alone) keep the other
 * scale at its initial value:  mode 1 = row (block) scales only, b keeps its
 * initial value (row update, requantize);  mode 2 = column scales only, a
 * keeps its initial value (column update, requantize).
 * init 0: absmax RTN with b = 1; init 1: per-column L1-norm column scales
 * (init_l1); init 2: warm start from the stored scales a0 [M][N/G], b0 [N] and
 * (NVFP4) sT0.
 * changes (optional, [iters+1]): changes[0] = 0 and changes[t] = the number of
 * elements whose grid value differs between the iterates after iterations t-1
 * and t ([P2] §4.3, App. B: the quantized matrix stabilizes; the relative
 * change of Q is changes[t] / (M N)).
 */
int dqo_solve_ex(const void* W, int wdt, int64_t M, int64_t N, int fmt, int G, int iters, int col_dt, int mode,
                 int init, const double* a0, const double* b0, double sT0, uint8_t* codes, double* a_out,
                 double* b_out, double* sT_out, double* mse, double* q_out, double* trace_a, double* trace_b,
                 uint64_t* changes) {
  if (iters < 0 || mode < 0 || mode > 2 || init < 0 || init > 2) return DQO_EINVAL;
  problem p;
  double* Wd = NULL;
  int st = load_problem(&p, W, wdt, M, N, fmt, G, col_dt, &Wd);
  if (st != DQO_OK) return st;
  int64_t nA = M * p.nb;
  double* a = (double*)malloc(sizeof(double) * (size_t)nA);
  double* b = (double*)malloc(sizeof(double) * (size_t)N);
  double* q = (double*)malloc(sizeof(double) * (size_t)(M * N));
  double* qprev = changes ? (double*)malloc(sizeof(double) * (size_t)(M * N)) : NULL;
  if (!a || !b || !q || (changes && !qprev)) {
    free(a);
    free(b);
    free(q);
    free(qprev);
    free(Wd);
    return DQO_ENOMEM;
  }
  if (init == 0) {
    init_scales(&p, a, b);
  } else if (init == 1) {
    init_l1(&p, a, b);
  } else {
    st = init_given(&p, a0, b0, sT0, a, b);
  }
  if (st == DQO_OK) {
    dqo_requant_impl(&p, a, b, q);
    if (mse) mse[0] = dqo_mse_impl(&p, q, a, b);
    if (changes) changes[0] = 0;
    if (trace_a) memcpy(trace_a, a, sizeof(double) * (size_t)nA);
    if (trace_b) memcpy(trace_b, b, sizeof(double) * (size_t)N);
    for (int t = 1; t <= iters; ++t) {
      if (changes) memcpy(qprev, q, sizeof(double) * (size_t)(M * N));
      if (mode != 2) {
        dqo_row_update_impl(&p, q, b, a, NULL);
        dqo_requant_impl(&p, a, b, q);
      }
      if (mode != 1) {
        dqo_col_update_impl(&p, q, a, b, NULL);
        dqo_requant_impl(&p, a, b, q);
      }
      if (mse) mse[t] = dqo_mse_impl(&p, q, a, b);
      if (changes) {
        uint64_t n = 0;
        for (int64_t k = 0; k < M * N; ++k) n += q[k] != qprev[k];
        changes[t] = n;
      }
      if (trace_a) memcpy(trace_a + (size_t)t * nA, a, sizeof(double) * (size_t)nA);
      if (trace_b) memcpy(trace_b + (size_t)t * N, b, sizeof(double) * (size_t)N);
    }
    if (codes) pack_codes(&p, q, codes);
    if (a_out) memcpy(a_out, a, sizeof(double) * (size_t)nA);
    if (b_out) memcpy(b_out, b, sizeof(double) * (size_t)N);
    if (sT_out) *sT_out = p.sT;
    if (q_out) memcpy(q_out, q, sizeof(double) * (size_t)(M * N));
  }
  free(a);
  free(b);
  free(q);
  free(qprev);
  free(Wd);
  return st;
}

int dqo_solve_mode(const void* W, int wdt, int64_t M, int64_t N, int fmt, int G, int iters, int col_dt, int mode,
                   uint8_t* codes, double* a_out, double* b_out, double* sT_out, double* mse, double* q_out,
                   double* trace_a, double* trace_b) {
  return dqo_solve_ex(W, wdt, M, N, fmt, G, iters, col_dt, mode, 0, NULL, NULL, 1.0, codes, a_out, b_out, sT_out, mse,
                      q_out, trace_a, trace_b, NULL);
}

int dqo_solve(const void* W, int wdt, int64_t M, int64_t N, int fmt, int G, int iters, int col_dt, uint8_t* codes,
              double* a_out, double* b_out, double* sT_out, double* mse, double* q_out, double* trace_a,
              double* trace_b) {
  return dqo_solve_mode(W, wdt, M, N, fmt, G, iters, col_dt, 0, codes, a_out, b_out, sT_out, mse, q_out, trace_a,
                        trace_b);
}

/* RTN = the solver's initial iterate ([R5]: RTN with beta = 1 is the start). */
int dqo_rtn(const void* W, int wdt, int64_t M, int64_t N, int fmt, int G, int col_dt, uint8_t* codes, double* a_out,
            double* b_out, double* sT_out, double* mse0) {
  return dqo_solve(W, wdt, M, N, fmt, G, 0, col_dt, codes, a_out, b_out, sT_out, mse0, NULL, NULL, NULL);
}

/*
 * Single steps from a given state, for pinning each step on its own and for
 * checking a GPU iterate against one oracle iteration.  astored holds stored
 * block-scale values (E4M3 e for NVFP4), sT the NVFP4 tensor scale.
 * mode: 0 = requantize -> q_out
 *       1 = row update from q_in  -> astored (in place), raw_out
 *       2 = column update from q_in -> b (in place), raw_out
 *       3 = one full BCD iteration from (astored, b): row update, requantize,
 *           column update, requantize -> astored, b, q_out (the codes q is
 *           recomputed from the given state first)
 *       4 = reconstruction MSE of (q_in, astored, b) -> *mse_out
 */
int dqo_step(const void* W, int wdt, int64_t M, int64_t N, int fmt, int G, int col_dt, double sT, int mode,
             double* astored, double* b, const double* q_in, double* q_out, double* raw_out, double* mse_out) {
  problem p;
  double* Wd = NULL;
  int st = load_problem(&p, W, wdt, M, N, fmt, G, col_dt, &Wd);
  if (st != DQO_OK) return st;
  p.sT = (fmt == DQO_NVFP4) ? sT : 1.0;
  st = DQO_OK;
  if (mode == 0) {
    dqo_requant_impl(&p, astored, b, q_out);
  } else if (mode == 1) {
    dqo_row_update_impl(&p, q_in, b, astored, raw_out);
  } else if (mode == 2) {
    dqo_col_update_impl(&p, q_in, astored, b, raw_out);
  } else if (mode == 3) {
    double* q = (double*)malloc(sizeof(double) * (size_t)(M * N));
    if (!q) {
      free(Wd);
      return DQO_ENOMEM;
    }
    dqo_requant_impl(&p, astored, b, q);
    dqo_row_update_impl(&p, q, b, astored, NULL);
    dqo_requant_impl(&p, astored, b, q);
    dqo_col_update_impl(&p, q, astored, b, NULL);
    dqo_requant_impl(&p, astored, b, q);
    if (q_out) memcpy(q_out, q, sizeof(double) * (size_t)(M * N));
    free(q);
  } else if (mode == 4) {
    *mse_out = dqo_mse_impl(&p, q_in, astored, b);
  } else {
    st = DQO_EINVAL;
  }
  free(Wd);
  return st;
}

/* Storage bit patterns of admissible values: fp16 / bf16 (16-bit), E4M3 and
 * E8M0 (8-bit).  v must be admissible (checked by the caller). */
uint32_t dqo_encode(int kind, double v) {
  if (kind == DQO_PROJ_F16) return encode_float_bits(v, 10, -14, 5);
  if (kind == DQO_PROJ_BF16) return encode_float_bits(v, 7, -126, 8);
  if (kind == DQO_PROJ_E4M3) return encode_float_bits(v, 3, -6, 4);
  int e;
  frexp(v, &e);
  return (uint32_t)(e - 1 + 127);
}

/* grid quantizer of a format on one value (for pins) -> grid value */
double dqo_quant_value(int fmt, double w, double ab) {
  if (e2m1_grid(fmt)) return E2M1_GRID[dqo_quant_index(w, ab, E2M1_GRID, E2M1_EVEN, 15)];
  if (fmt == DQO_MXINT8) {
    grids_init();
    return INT8_GRID[dqo_quant_index(w, ab, INT8_GRID, INT8_EVEN, 256)];
  }
  if (fmt == DQO_MXFP8) {
    grids_init();
    return E4M3_GRID[dqo_quant_index(w, ab, E4M3_GRID, E4M3_EVEN, 253)];
  }
  return INT4_GRID[dqo_quant_index(w, ab, INT4_GRID, INT4_EVEN, 16)];
}

int dqo_num_threads(void) {
#ifdef _OPENMP
  extern int omp_get_max_threads(void);
  return omp_get_max_threads();
#else
  return 1;
#endif
}

/* threads of later parallel loops (timing the oracle on one core) */
void dqo_set_num_threads(int n) {
#ifdef _OPENMP
  extern void omp_set_num_threads(int);
  omp_set_num_threads(n);
#else
  (void)n;
#endif
}
