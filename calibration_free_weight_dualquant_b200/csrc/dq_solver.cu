// dq_solver.cu -- CUDA kernels (sm_100a) of the DualQuant dual-scale BCD solver.
//
// Method (DualQuant reproduction README, flowchart and "Core equations";
// DualQuant arXiv 2610.13767 summary, §4.3 and App. B):
//   init  : b = 1, a = Proj_Fa(absmax(block)/qmax)  (absmax round-to-nearest)
//   iterate t = 1..T:
//     q  = Q(W/(a b))                 codes of the current iterate
//     a <- Proj_Fa(sum W q b / sum (q b)^2)   per block, codes fixed
//     q' = Q(W/(a b))                 requantize after the block update
//     b <- Proj_Fb(sum W a q' / sum (a q')^2) per column, codes fixed
//   scale 1 for an all-zero code slice; codes are a function of (W, a, b).
//
// Launches per solve: k_stats (non-finite check, max |W|), k_init (scales of
// the initial iterate), one k_iter running all T BCD iterations (one read of W
// each, a grid barrier between them), and k_iter in its final mode (codes of
// the final iterate and the last MSE, one more read of W).  k_iter
// (dq_iter.cuh) runs one CTA per SM over contiguous ranges of strip-major
// (strip, row) units, so every CTA streams the same number of rows; the column
// totals and the MSE are summed in CTA order by the last CTA to arrive (an
// atomic ticket), so every result is deterministic.
#include <cudaTypedefs.h>  // PFN_cuTensorMapEncodeTiled

#include <algorithm>
#include <climits>
#include <cstring>

#include "dq_device.cuh"
#include "dq_fast.cuh"
#include "dq_init.cuh"
#include "dq_internal.h"
#include "dq_iter.cuh"

namespace dq {


// Last-arriving CTA election for a counter: every thread has already issued its
// writes; returns true in all threads of the CTA that arrived last.
__device__ __forceinline__ bool arrive_last(unsigned* counter, unsigned expected, int* s_flag) {
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    const unsigned prev = atomicAdd(counter, 1u);
    *s_flag = (prev == expected - 1u) ? 1 : 0;
  }
  __syncthreads();
  const bool last = *s_flag != 0;
  if (last) __threadfence();
  return last;
}

// ---------------------------------------------------------------------------
// Statistics pass: non-finite check and max |W| (for the NVFP4 tensor scale).
template <int WDT>
__global__ void __launch_bounds__(kThreads) k_stats(Problem p) {
  const int64_t nchunks = p.M * p.N / 8;
  float amax = 0.f;
  bool bad = false;
  for (int64_t c = (int64_t)blockIdx.x * kThreads + threadIdx.x; c < nchunks; c += (int64_t)gridDim.x * kThreads) {
    float w[8];
    load8<WDT>(p.W, c * 8, w);
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      bad |= !isfinite(w[k]);
      amax = fmaxf(amax, fabsf(w[k]));
    }
  }
  if (bad) atomicOr(&p.hdr->flags, kFlagNonFinite);
  // max of non-negative floats = max of their bit patterns (order independent)
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if ((threadIdx.x & 31) == 0 && isfinite(amax)) atomicMax(&p.hdr->amax_bits, __float_as_uint(amax));
}

// ---------------------------------------------------------------------------
// Init: s_T (NVFP4), a = Proj(absmax/qmax) per block (1 for an all-zero
// block), b = 1.  With the L1-norm init (dq_init.cuh) the column scales are
// already set and the absmax is taken of |W_ij| / b_j (fp64 quotients).
template <int FMT, int WDT>
__global__ void __launch_bounds__(kThreads) k_init(Problem p) {
  if (p.hdr->flags & kFlagAbort) return;
  const bool l1 = p.init == DQ_INIT_L1;
  double sTd = 1.0;
  if (FMT == FMT_NVFP4) {
    const double amax = l1 ? __longlong_as_double((long long)p.hdr->amax_scaled)
                           : (double)__uint_as_float(p.hdr->amax_bits);
    float s = amax == 0.0 ? 1.f : __double2float_rn(amax / 2688.0);
    if (s == 0.f) s = 0x1p-149f;
    sTd = (double)s;
    if (blockIdx.x == 0 && threadIdx.x == 0) {
      p.hdr->sT = s;
      if (p.sT_out) *p.sT_out = s;
    }
  } else if (blockIdx.x == 0 && threadIdx.x == 0) {
    p.hdr->sT = 1.f;
    if (p.sT_out) *p.sT_out = 1.f;
  }
  const double qmax = grid_qmax(FMT);
  const float isT = FMT == FMT_NVFP4 ? __frcp_rn((float)sTd) : 1.f;
  // A warp takes 32 consecutive rows of one block-column (lane = row): each
  // lane reads its block's G contiguous elements (whole sectors), and the
  // warp's 32 block scales land contiguously in the block-column-major a_work.
  const int lane = threadIdx.x & 31;
  const int64_t MT = (p.M + 31) / 32;
  const int64_t ntiles = MT * p.nb;
  const int64_t nwarps = (int64_t)gridDim.x * (kThreads / 32);
  for (int64_t t = (int64_t)blockIdx.x * (kThreads / 32) + (threadIdx.x >> 5); t < ntiles; t += nwarps) {
    const int64_t g = t / MT, i = (t - g * MT) * 32 + lane;
    if (i >= p.M) continue;
    const int64_t off = i * p.N + g * p.G;
    double a;
    if (l1) {
      double m = 0.0;
      for (int c = 0; c < p.G; c += 8) {
        float w[8];
        load8<WDT>(p.W, off + c, w);
#pragma unroll
        for (int k = 0; k < 8; ++k)
          m = fmax(m, (double)fabsf(w[k]) / (double)b_decode(p.b_store, p.col_dt, g * p.G + c + k));
      }
      a = (m == 0.0) ? 1.0 : a_project<FMT>(m / qmax, sTd);
    } else {
      float mf = 0.f;
      for (int c = 0; c < p.G; c += 8) {
        float w[8];
        load8<WDT>(p.W, off + c, w);
#pragma unroll
        for (int k = 0; k < 8; ++k) mf = fmaxf(mf, fabsf(w[k]));
      }
      // certified fp32 projection of absmax / qmax, fp64 where it is ambiguous
      bool amb = false;
      const float af = a_fast<FMT>(mf, (float)qmax, isT, amb);
      a = !amb ? (double)af : (mf == 0.f ? 1.0 : a_project<FMT>((double)mf / qmax, sTd));
    }
    a_encode<FMT>(p.a_work, g * p.M + i, a);
  }
  const int64_t stride = (int64_t)gridDim.x * kThreads;
  if (!l1)
    for (int64_t j = (int64_t)blockIdx.x * kThreads + threadIdx.x; j < p.N; j += stride)
      b_encode(p.b_store, p.col_dt, j, 1.0);
}

// ---------------------------------------------------------------------------
// Host-side launch of the whole solve on one stream.

// The driver's tensor-map encoder, looked up once through the runtime.
static PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static const PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return (PFN_cuTensorMapEncodeTiled_v12000) nullptr;
    return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  }();
  return fn;
}

// 2-D tensor map of W (columns innermost) whose box is one block-column's
// share of a ring tile: G columns x 2 * 32/(G/8) rows.  Returns false when W
// cannot be described (then k_iter copies one block row at a time).
template <int WDT>
static bool encode_w_map(const Problem& p, CUtensorMap* map) {
  constexpr int ES = WDT == DT_F32 ? 4 : 2;
  std::memset(map, 0, sizeof(*map));
  if (p.M > INT_MAX || p.N > INT_MAX || (p.N * ES) % 16 != 0 || (p.G * ES) % 16 != 0) return false;
  const PFN_cuTensorMapEncodeTiled_v12000 fn = tensor_map_encoder();
  if (fn == nullptr) return false;
  const TileGeo geo = tile_geo(p.G, ES);
  const cuuint64_t dims[2] = {(cuuint64_t)p.N, (cuuint64_t)p.M};
  const cuuint64_t strides[1] = {(cuuint64_t)p.N * ES};
  const cuuint32_t box[2] = {(cuuint32_t)p.G, (cuuint32_t)geo.RW};
  const cuuint32_t elem_strides[2] = {1, 1};
  const CUtensorMapDataType dt = WDT == DT_F32    ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
                                 : WDT == DT_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                                  : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  return fn(map, dt, 2, const_cast<void*>(p.W), dims, strides, box, elem_strides, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D view of W, (G columns, nb block-columns, M rows) with strides (1, G, N)
// elements, whose box is a whole strip's share of a ring tile: G x 15 x
// 2 * 32/(G/8).  It lands as [rows][15][G], row-major over the strip, when the
// strip's block-columns are consecutive.  Returns false when W cannot be
// described (then every tile takes one copy per block-column).
template <int WDT>
static bool encode_w_map3(const Problem& p, CUtensorMap* map) {
  constexpr int ES = WDT == DT_F32 ? 4 : 2;
  std::memset(map, 0, sizeof(*map));
  if (p.M > INT_MAX || p.nb > INT_MAX || (p.N * ES) % 16 != 0 || (p.G * ES) % 16 != 0) return false;
  const TileGeo geo = tile_geo(p.G, ES);
  if (geo.box_stride != geo.box_bytes) return false;  // the slot layout must be dense
  const PFN_cuTensorMapEncodeTiled_v12000 fn = tensor_map_encoder();
  if (fn == nullptr) return false;
  const cuuint64_t dims[3] = {(cuuint64_t)p.G, (cuuint64_t)p.nb, (cuuint64_t)p.M};
  const cuuint64_t strides[2] = {(cuuint64_t)p.G * ES, (cuuint64_t)p.N * ES};
  const cuuint32_t box[3] = {(cuuint32_t)p.G, (cuuint32_t)kBcPerStrip, (cuuint32_t)geo.RW};
  const cuuint32_t elem_strides[3] = {1, 1, 1};
  const CUtensorMapDataType dt = WDT == DT_F32    ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
                                 : WDT == DT_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                                  : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  return fn(map, dt, 3, const_cast<void*>(p.W), dims, strides, box, elem_strides, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Launch of k_iter: cooperative (all CTAs resident at once, for its grid
// barrier) and with programmatic stream serialization (the grid may start while
// the one before it in the stream finishes; the kernel waits, griddep_wait,
// before it reads earlier results).  Where the runtime refuses the two
// attributes together, the launch is cooperative alone.
template <typename... KArgs, typename... Args>
static cudaError_t launch_coop(void (*kernel)(KArgs...), unsigned grid, unsigned block, size_t smem, cudaStream_t st,
                               Args... args) {
  cudaLaunchConfig_t cfg;
  std::memset(&cfg, 0, sizeof(cfg));
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(block);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, args...);
  if (e == cudaErrorInvalidValue || e == cudaErrorNotSupported) {
    (void)cudaGetLastError();  // a refused configuration is not a sticky error
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, kernel, args...);
  }
  return e;
}

template <int FMT, int WDT>
static cudaError_t run_typed(const Problem& p, int iters, int stats_ctas, cudaStream_t st) {
  const size_t smem = (size_t)iter_smem(p.G / 8, p.P, p.segmax).total;
  const auto iter_kernel = p.changes ? k_iter<FMT, WDT, PASS_COUNT> : k_iter<FMT, WDT, PASS_ITER>;
  cudaError_t e = cudaFuncSetAttribute(iter_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(k_iter<FMT, WDT, PASS_FINAL>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  CUtensorMap wmap, wmap3;
  Problem pi = p;
  pi.use_tmap = encode_w_map<WDT>(p, &wmap) ? 1 : 0;
  pi.use_tmap3 = pi.use_tmap && encode_w_map3<WDT>(p, &wmap3) ? 1 : 0;
  Problem pf = p;
  pf.P = p.P_final;
  pf.segmax = p.segmax_final;
  k_stats<WDT><<<stats_ctas, kThreads, 0, st>>>(pf);
  if (p.init == DQ_INIT_GIVEN) {
    k_check_given<FMT><<<stats_ctas, kThreads, 0, st>>>(pf);
  } else {
    if (p.init == DQ_INIT_L1) {
      // exact column sums: 32 columns per CTA, rows split so the grid fills the GPU
      const int64_t gx = (p.N + 31) / 32;
      int64_t gy = std::max<int64_t>(1, std::min<int64_t>((8 * (int64_t)stats_ctas + gx - 1) / gx,
                                                          (p.M + kMinRowsPerCta - 1) / kMinRowsPerCta));
      const int64_t rows_per_cta = (p.M + gy - 1) / gy;
      gy = (p.M + rows_per_cta - 1) / rows_per_cta;
      k_l1_sums<WDT><<<dim3((unsigned)gx, (unsigned)gy), kThreads, 0, st>>>(pf, rows_per_cta);
      k_l1_cols<<<(unsigned)((p.N + kThreads - 1) / kThreads), kThreads, 0, st>>>(pf);
      k_l1_b<<<(unsigned)std::min<int64_t>(stats_ctas, (p.N + kThreads - 1) / kThreads), kThreads, 0, st>>>(pf);
      if (FMT == FMT_NVFP4) k_amax_scaled<WDT><<<stats_ctas, kThreads, 0, st>>>(pf);
    }
    k_init<FMT, WDT><<<stats_ctas, kThreads, 0, st>>>(pf);
  }
  // all BCD iterations in one persistent launch, then the final pass
  if (iters > 0) {
    e = launch_coop(iter_kernel, (unsigned)p.P, kIterThreads, smem, st, pi, 1, iters, wmap, wmap3);
    if (e != cudaSuccess) return e;
  }
  e = launch_coop(k_iter<FMT, WDT, PASS_FINAL>, (unsigned)p.P, kIterThreads, smem, st, pi, iters + 1, iters + 1, wmap,
                  wmap3);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <int FMT>
static cudaError_t run_fmt(const Problem& p, int iters, int stats_ctas, cudaStream_t st) {
  switch (p.wdt) {
    case DT_F32: return run_typed<FMT, DT_F32>(p, iters, stats_ctas, st);
    case DT_BF16: return run_typed<FMT, DT_BF16>(p, iters, stats_ctas, st);
    default: return run_typed<FMT, DT_F16>(p, iters, stats_ctas, st);
  }
}

cudaError_t launch_solve(const Problem& p, int iters, int stats_ctas, cudaStream_t st) {
  switch (p.fmt) {
    case FMT_INT4: return run_fmt<FMT_INT4>(p, iters, stats_ctas, st);
    case FMT_MXINT4: return run_fmt<FMT_MXINT4>(p, iters, stats_ctas, st);
    case FMT_MXFP4: return run_fmt<FMT_MXFP4>(p, iters, stats_ctas, st);
    case FMT_MXINT8: return run_fmt<FMT_MXINT8>(p, iters, stats_ctas, st);
    case FMT_MXFP8: return run_fmt<FMT_MXFP8>(p, iters, stats_ctas, st);
    default: return run_fmt<FMT_NVFP4>(p, iters, stats_ctas, st);
  }
}

// Self-tests of the bounded waits; nothing faults and the context stays
// usable.  which == 0: a strip counter that never reaches its target, so
// wait_count gives up after its time limit.  which == 1: a ring barrier in
// shared memory that nothing arrives at and no copy completes, so mbar_wait
// gives up after its time limit.  Both record kFlagTimeout.
__global__ void k_wait_selftest(Problem p, int which) {
  __shared__ uint64_t bar;
  if (which == 0) {
    if (threadIdx.x == 0) {
      p.hdr->flags = 0u;
      p.strip_counter[0] = 0u;
      __threadfence();
    }
    __syncwarp();
    wait_count(p.strip_counter, 1u, &p.hdr->flags);
  } else {
    if (threadIdx.x == 0) {
      p.hdr->flags = 0u;
      mbar_init(&bar, 1);
      mbar_fence_init();
    }
    __syncwarp();
    if (threadIdx.x == 0) mbar_wait(&bar, 0u, &p.hdr->flags);
    __syncwarp();
  }
}

cudaError_t launch_wait_selftest(void* workspace, int which, cudaStream_t st) {
  Problem p;
  std::memset(&p, 0, sizeof(p));
  p.hdr = reinterpret_cast<WsHeader*>(workspace);
  p.strip_counter = reinterpret_cast<unsigned*>(static_cast<char*>(workspace) + 256);
  k_wait_selftest<<<1, 32, 0, st>>>(p, which);
  return cudaGetLastError();
}

}  // namespace dq
