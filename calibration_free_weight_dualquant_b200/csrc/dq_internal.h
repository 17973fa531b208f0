// dq_internal.h -- types shared by the C ABI layer and the kernels.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "dq.h"

namespace dq {

constexpr int kThreads = 256;   // 8 warps per CTA
constexpr int kWarps = kThreads / 32;
constexpr int kGroupMax = 256;  // largest block size (a block row spans at most one warp)
constexpr int kCtasPerSm = 1;        // per-iteration pass: one 512-thread CTA per SM
constexpr int kMaxGrid = 1024;       // CTAs of the per-iteration pass at most
constexpr int kFinalCtasPerSm = 4;   // one-time passes
constexpr int64_t kMinRowsPerCta = 64;
// 32-bit digits of an exact magnitude sum in units of 2^-149 (L1 init): one
// value reaches bit 277, a sum of up to 2^31 values bit 308
constexpr int kXDigits = 10;
constexpr unsigned kFlagNonFinite = 1u;
constexpr unsigned kFlagTimeout = 2u;  // a bounded pipeline wait gave up (results invalid)
constexpr unsigned kFlagBadInit = 4u;  // a warm start was given an inadmissible scale
constexpr unsigned kFlagAbort = kFlagNonFinite | kFlagBadInit;  // later kernels do nothing

// ---------------------------------------------------------------------------
// Geometry of the per-iteration pass k_iter (host and device).
constexpr int kConsumerWarps = 15;
constexpr int kConsumers = kConsumerWarps * 32;
constexpr int kIterThreads = kConsumers + 32;
// block-columns per strip: one per consumer warp
constexpr int kBcPerStrip = kConsumerWarps;
constexpr int kRingBytes = 96 * 1024;
constexpr int kMaxStages = 8;
// Tile geometry for block size G (a multiple of 8 dividing 256) and W element
// size es: lanes per block row, row-lanes per warp, rows per tile, bytes of
// one block-column's box and its slot in the ring (16-byte multiple, rounded
// to 128 bytes for the tensor copy's destination), stage bytes, ring stages.
struct TileGeo {
  int lpb, rl, RW, box_bytes, box_stride, stage_bytes, S;
};
__host__ __device__ inline TileGeo tile_geo(int G, int es) {
  TileGeo g;
  g.lpb = G / 8;
  g.rl = 32 / g.lpb;
  g.RW = 2 * g.rl;
  g.box_bytes = g.RW * G * es;
  g.box_stride = (g.box_bytes + 127) / 128 * 128;
  g.stage_bytes = kBcPerStrip * g.box_stride;
  g.S = kRingBytes / g.stage_bytes < kMaxStages ? kRingBytes / g.stage_bytes : kMaxStages;
  return g;
}

// Dynamic shared memory of k_iter (byte offsets): the tile ring; fp64 column
// accumulators (per consumer warp: 8 columns x 32 lanes of (sum W a q,
// sum (a q)^2)); one fp64 residual sum per consumer thread; ring barriers;
// small ints ([0] flag, [2..5] exact-path counters, [40..56] schedule scan);
// the pass schedule; the column tables (per warp: b pairs [lpb][4], then 1/b
// pairs [lpb][4]); the first strip of each CTA's range; this CTA's slice of
// the active list.
struct IterSmem {
  int acc, racc, bars, misc, sched, ctab, sfirst, act, total;
};
__host__ __device__ inline IterSmem iter_smem(int lpb, int P, int segmax) {
  IterSmem s;
  int off = kRingBytes;
  s.acc = off;
  off += kConsumerWarps * 8 * 32 * 16;
  s.racc = off;
  off += kConsumers * 8;
  s.bars = off;
  off += 2 * kMaxStages * 8;
  s.misc = off;
  off += 64 * 4;
  s.sched = off;
  off += 64;
  s.ctab = off;
  off += kConsumerWarps * 2 * 4 * lpb * 8;
  s.sfirst = off;
  off += (P * 4 + 15) / 16 * 16;
  s.act = off;
  off += (segmax * kBcPerStrip * 4 + 15) / 16 * 16;
  s.total = off;
  return s;
}
// CTAs that get units in a pass of nv strips (L = nv M units): a multiple of
// nv (every CTA within one strip) when that keeps at least 90% of the grid,
// else the grid; and at most one CTA per kMinRowsPerCta units, so every CTA
// that gets units gets at least one (the strip tickets count every CTA from
// the first to the last owner of a strip)
__host__ __device__ inline int pass_ctas(int P, long long nv, long long L) {
  int c = P;
  if (nv >= 1 && nv <= P) {
    const long long a = (long long)P / nv * nv;
    if (10 * a >= 9LL * P) c = (int)a;
  }
  const long long cap = L / kMinRowsPerCta;
  return cap < c ? (cap < 1 ? 1 : (int)cap) : c;
}

// Device workspace header (first 256 bytes of the workspace).
struct WsHeader {
  unsigned flags;        // kFlagNonFinite, kFlagTimeout, kFlagBadInit
  unsigned amax_bits;    // max |W| as fp32 bits
  unsigned cta_counter;  // arrival ticket for CTA-ordered totals
  unsigned gbar;         // arrivals at k_iter's grid-wide barrier
  float sT;              // NVFP4 tensor scale (1 otherwise)
  unsigned long long n_quant_tie;    // lane-rows with a certified exact tie settled on the fast path
  // diagnostics: how often the exact paths ran in the per-iteration passes
  unsigned long long n_quant_exact;  // lane-rows (8 elements) decided on the exact path
  unsigned long long n_block_exact;  // block updates taken in fp64
  unsigned long long n_col_exact;    // column updates recomputed exactly over all rows
  unsigned long long amax_scaled;    // L1 init, NVFP4: max |W_ij| / b_j as the bits of a double
  unsigned long long n_active_bc;    // block-columns processed, summed over the BCD passes
};
static_assert(sizeof(WsHeader) <= 256, "workspace header");

// Everything a kernel needs, passed by value.
struct Problem {
  const void* W;
  int wdt, fmt, G, col_dt;
  int64_t M, N;
  int nb;        // blocks per row = N / G (= block-columns)
  int TSv;       // columns of a strip of k_iter: 15 block-columns, 15 G
  int n_strips;  // strips of a pass over every block-column: ceil(nb / 15)
  int P;         // CTAs of the per-iteration pass
  int segmax;    // max (CTA, strip) segments per CTA in any pass
  int P_final;   // CTAs of the one-time passes (stats, init)
  int segmax_final;
  int64_t L;     // n_strips * M (strip-major row units of a full pass)
  void* codes;
  void* a_store;   // output block scales [M][nb] (storage format), written by the final pass
  void* a_work;    // working block scales [nb][M] (storage format): a block-column's rows contiguous
  void* b_store;
  float* sT_out;
  double* mse;
  WsHeader* hdr;
  unsigned* strip_counter;  // [4][2][n_strips] per strip and pass parity: arrivals, ambiguous columns,
                            // finalizers done, exact shares done (zeroed)
  int* amb_list;            // [n_strips][TSv] strip columns listed for the exact update
  double2* col_part;        // [P * segmax][TSv] (sum W a q, sum (a q)^2)
  double* cta_part;         // [3][max(P, P_final)] per-CTA residual totals of the final pass
  double* mse_seg;          // [P * segmax][15] residual total per (CTA segment, block-column slot)
  double* mse_bc;           // [3][nb] residual total per block-column, by pass mod 3
  unsigned* chg;            // [3][nb] a scale of the block-column changed (or was listed), by pass mod 3 (zeroed)
  int use_tmap;             // W streamed by 2-D tensor copies (else one bulk copy per row)
  int use_tmap3;            // a strip of consecutive block-columns streamed by one 3-D tensor copy per tile
  int mode;                 // DQ_MODE_DUAL, DQ_MODE_ROW (b keeps its initial value) or DQ_MODE_COL
  int init;                 // DQ_INIT_RTN, DQ_INIT_L1 or DQ_INIT_GIVEN
  int full_passes;          // every BCD pass takes every block-column (no skipping at fixed points)
  // L1 init scratch (overlays col_part, which the init kernels do not use)
  unsigned long long* l1_dig;   // [N][10] digit counters of the column magnitude sums (zeroed)
  unsigned long long* l1_tot;   // [10] digit counters of the total (zeroed)
  double* l1_norm;              // [N] column L1 norms rounded to fp64
  unsigned long long* changes;  // NULL, or [iters + 1] changed-code counts
};

cudaError_t launch_solve(const Problem& p, int iters, int stats_ctas, cudaStream_t st);
// Runs a bounded-wait self-test on `workspace` (>= 512 bytes): `which` 0 waits
// on a count in global memory, 1 on a shared-memory ring barrier.
cudaError_t launch_wait_selftest(void* workspace, int which, cudaStream_t st);

// Host-side validation, workspace layout and enqueue of a whole solve (the body
// of dq_solve; `workspace` is a device address of at least the planned size).
// `opt` NULL means the defaults (dual mode, RTN init, no change counts).
int solve_impl(const void* W, int w_dtype, int64_t rows, int64_t cols, int format, int group, int iters,
               int col_dtype, const dq_outputs* out, void* workspace, size_t workspace_bytes,
               cudaStream_t stream, const dq_options* opt = nullptr);

}  // namespace dq
