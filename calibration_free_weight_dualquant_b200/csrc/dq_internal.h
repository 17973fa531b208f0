// dq_internal.h -- types shared by the C ABI layer and the kernels.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "dq.h"

namespace dq {

constexpr int kThreads = 256;   // 8 warps per CTA
constexpr int kWarps = kThreads / 32;
constexpr int kStripMax = 256;  // columns per strip (8 per lane, 32 lanes)
constexpr int kCtasPerSm = 1;        // per-iteration pass: one 512-thread CTA per SM
constexpr int kMaxGrid = 1024;       // CTAs of the per-iteration pass at most
constexpr int kFinalCtasPerSm = 4;   // one-time passes
constexpr int64_t kMinRowsPerCta = 64;
// 32-bit digits of an exact magnitude sum in units of 2^-149 (L1 init): one
// value reaches bit 277, a sum of up to 2^31 values bit 308
constexpr int kXDigits = 10;
constexpr int64_t kXPartCap = 32768;  // entries of the exact-update partial buffer
constexpr unsigned kFlagNonFinite = 1u;
constexpr unsigned kFlagTimeout = 2u;  // a bounded pipeline wait gave up (results invalid)
constexpr unsigned kFlagBadInit = 4u;  // a warm start was given an inadmissible scale
constexpr unsigned kFlagAbort = kFlagNonFinite | kFlagBadInit;  // later kernels do nothing

// Device workspace header (first 256 bytes of the workspace).
struct WsHeader {
  unsigned flags;        // kFlagNonFinite, kFlagTimeout, kFlagBadInit
  unsigned amax_bits;    // max |W| as fp32 bits
  unsigned cta_counter;  // arrival ticket for CTA-ordered totals
  unsigned amb_n[3];     // columns listed for the exact column update, by pass mod 3
  unsigned gbar;         // arrivals at k_iter's grid-wide barrier
  float sT;              // NVFP4 tensor scale (1 otherwise)
  unsigned long long n_quant_tie;    // lane-rows with a certified exact tie settled on the fast path
  // diagnostics: how often the exact paths ran in the per-iteration passes
  unsigned long long n_quant_exact;  // lane-rows (8 elements) decided on the exact path
  unsigned long long n_block_exact;  // block updates taken in fp64
  unsigned long long n_col_exact;    // column updates recomputed exactly over all rows
  unsigned long long amax_scaled;    // L1 init, NVFP4: max |W_ij| / b_j as the bits of a double
};

// Everything a kernel needs, passed by value.
struct Problem {
  const void* W;
  int wdt, fmt, G, col_dt;
  int64_t M, N;
  int nb;        // blocks per row = N / G
  int TS;        // strip width (columns), multiple of G and of 8, <= kStripMax
  int n_strips;  // ceil(N / TS)
  int P;         // CTAs of the per-iteration pass
  int segmax;    // max (CTA, strip) segments per CTA of that pass
  int P_final;   // CTAs of the one-time passes (stats, init, final)
  int segmax_final;
  int64_t L;     // n_strips * M (strip-major row units)
  void* codes;
  void* a_store;
  void* b_store;
  float* sT_out;
  double* mse;
  WsHeader* hdr;
  unsigned* strip_counter;  // [n_strips]
  double2* col_part;        // [P * segmax][TS] (sum W a q, sum (a q)^2)
  double* cta_part;         // [max(P, P_final)]
  int* amb_list;            // [3][N] columns whose certified projection was ambiguous, by pass mod 3
  unsigned* amb_tick;       // [N] arrival counters of their row chunks (zeroed)
  unsigned* sx_left;        // [n_strips] listed columns of a strip still awaiting their exact update (zeroed)
  double2* xpart;           // [kXPartCap] per-CTA exact partial sums of the listed columns
  int use_tmap;             // W streamed by 2-D tensor copies (else one bulk copy per row)
  int mode;                 // DQ_MODE_DUAL, DQ_MODE_ROW (b keeps its initial value) or DQ_MODE_COL
  int init;                 // DQ_INIT_RTN, DQ_INIT_L1 or DQ_INIT_GIVEN
  // L1 init scratch (overlays col_part, which the init kernels do not use)
  unsigned long long* l1_dig;   // [N][10] digit counters of the column magnitude sums (zeroed)
  unsigned long long* l1_tot;   // [10] digit counters of the total (zeroed)
  double* l1_norm;              // [N] column L1 norms rounded to fp64
  unsigned long long* changes;  // NULL, or [iters + 1] changed-code counts
};

cudaError_t launch_solve(const Problem& p, int iters, int stats_ctas, cudaStream_t st);
// Runs the bounded-wait self-test on `workspace` (>= 512 bytes).
cudaError_t launch_wait_selftest(void* workspace, cudaStream_t st);

// Host-side validation, workspace layout and enqueue of a whole solve (the body
// of dq_solve; `workspace` is a device address of at least the planned size).
// `opt` NULL means the defaults (dual mode, RTN init, no change counts).
int solve_impl(const void* W, int w_dtype, int64_t rows, int64_t cols, int format, int group, int iters,
               int col_dtype, const dq_outputs* out, void* workspace, size_t workspace_bytes,
               cudaStream_t stream, const dq_options* opt = nullptr);

}  // namespace dq
