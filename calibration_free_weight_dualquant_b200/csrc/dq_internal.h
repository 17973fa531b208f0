// dq_internal.h -- types shared by the C ABI layer and the kernels.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace dq {

constexpr int kThreads = 256;   // 8 warps per CTA
constexpr int kWarps = kThreads / 32;
constexpr int kStripMax = 256;  // columns per strip (8 per lane, 32 lanes)
constexpr int kCtasPerSm = 2;
constexpr int64_t kMinRowsPerCta = 64;
constexpr unsigned kFlagNonFinite = 1u;

// Device workspace header (first 256 bytes of the workspace).
struct WsHeader {
  unsigned flags;        // kFlagNonFinite
  unsigned amax_bits;    // max |W| as fp32 bits
  unsigned cta_counter;  // arrival ticket for CTA-ordered totals
  float sT;              // NVFP4 tensor scale (1 otherwise)
  double sumW2;          // sum of W^2 (fp64)
};

// Everything a kernel needs, passed by value.
struct Problem {
  const void* W;
  int wdt, fmt, G, col_dt;
  int64_t M, N;
  int nb;        // blocks per row = N / G
  int TS;        // strip width (columns), multiple of G and of 8, <= kStripMax
  int n_strips;  // ceil(N / TS)
  int P;         // CTAs of the persistent passes
  int segmax;    // max (CTA, strip) segments per CTA
  int64_t L;     // n_strips * M (strip-major row units)
  void* codes;
  void* a_store;
  void* b_store;
  float* sT_out;
  double* mse;
  WsHeader* hdr;
  unsigned* strip_counter;  // [n_strips]
  double2* col_part;        // [P * segmax][TS] (sum W a q, sum (a q)^2)
  double* cta_part;         // [P]
};

cudaError_t launch_solve(const Problem& p, int iters, int stats_ctas, cudaStream_t st);

}  // namespace dq
