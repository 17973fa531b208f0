// dq_act.cu -- the beta-folded activation quantizer: X' = X diag(b) followed by
// the format's own row-wise absmax round-to-nearest, in one pass over X (plus
// an amax pass for the NVFP4 tensor scale).
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

constexpr int kActThreads = 256;      // 8 warps; a warp covers 256 columns of a row
constexpr int kActCtasPerSm = 4;

struct ActProblem {
  const void* X;
  const void* b_store;
  int col_dt, G;
  int64_t M, K;
  int nb;          // groups per row
  int n_slabs;     // ceil(K / 256)
  void* codes;
  void* a_store;
  float* sT_out;
  WsHeader* hdr;
};

// One row segment of 8 columns of a lane, times its column scales (exact).
template <int XDT>
__device__ __forceinline__ void act_load8(const ActProblem& p, int64_t r, int64_t col, const float bcol[8],
                                          float x[8]) {
  load8<XDT>(p.X, r * p.K + col, x);
#pragma unroll
  for (int c = 0; c < 8; ++c) x[c] *= bcol[c];
}

template <int XDT>
__device__ __forceinline__ void act_cols(const ActProblem& p, int64_t col, bool active, float bcol[8]) {
#pragma unroll
  for (int c = 0; c < 8; ++c) bcol[c] = active ? b_decode(p.b_store, p.col_dt, col + c) : 0.f;
}

// Pass 1 (NVFP4, and the non-finite check for every format): max |x b|.
template <int XDT>
__global__ void __launch_bounds__(kActThreads) k_act_amax(ActProblem p) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t units = (int64_t)p.n_slabs * p.M;  // (slab, row) pairs, slab-major
  float amax = 0.f;
  bool bad = false;
  int64_t cur_slab = -1;
  float bcol[8];
  bool active = false;
  int64_t col = 0;
  for (int64_t u = (int64_t)blockIdx.x * (kActThreads / 32) + warp; u < units;
       u += (int64_t)gridDim.x * (kActThreads / 32)) {
    const int64_t s = u / p.M, r = u - s * p.M;
    if (s != cur_slab) {
      cur_slab = s;
      col = s * 256 + lane * 8;
      active = col < p.K;
      act_cols<XDT>(p, col, active, bcol);
    }
    if (active) {
      float x[8];
      act_load8<XDT>(p, r, col, bcol, x);
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        bad |= !isfinite(x[c]);
        amax = fmaxf(amax, fabsf(x[c]));
      }
    }
  }
  if (bad) atomicOr(&p.hdr->flags, kFlagNonFinite);
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if (lane == 0 && isfinite(amax)) atomicMax(&p.hdr->amax_bits, __float_as_uint(amax));
}

// Pass 2: group scales and codes.  A warp takes one (slab, row) unit at a time;
// lane l holds columns 8l .. 8l+7 of the slab, a group spans G/8 lanes.
template <int FMT, int XDT>
__global__ void __launch_bounds__(kActThreads) k_act(ActProblem p) {
  if (p.hdr->flags & kFlagNonFinite) return;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  float sT = 1.f;
  if (FMT == FMT_NVFP4) {
    const float amax = __uint_as_float(p.hdr->amax_bits);
    sT = amax == 0.f ? 1.f : __double2float_rn((double)amax / 2688.0);
    if (sT == 0.f) sT = 0x1p-149f;
  }
  if (blockIdx.x == 0 && threadIdx.x == 0 && p.sT_out) *p.sT_out = sT;
  const double sTd = (double)sT;
  const float isT = FMT == FMT_NVFP4 ? __frcp_rn(sT) : 1.f;
  const bool sT_ok = FMT != FMT_NVFP4 || in_range(isT);
  const float qmax = FMT == FMT_NVFP4 ? 6.f : 7.f;
  const int lpg = p.G / 8;  // lanes per group
  const bool leader = (lane & (lpg - 1)) == 0;
  const int64_t units = (int64_t)p.n_slabs * p.M;
  int64_t cur_slab = -1;
  float bcol[8];
  bool active = false;
  int64_t col = 0;
  for (int64_t u = (int64_t)blockIdx.x * (kActThreads / 32) + warp; u < units;
       u += (int64_t)gridDim.x * (kActThreads / 32)) {
    const int64_t s = u / p.M, r = u - s * p.M;
    if (s != cur_slab) {
      cur_slab = s;
      col = s * 256 + lane * 8;
      active = col < p.K;
      act_cols<XDT>(p, col, active, bcol);
    }
    float x[8];
    float m = 0.f;
    if (active) {
      act_load8<XDT>(p, r, col, bcol, x);
#pragma unroll
      for (int c = 0; c < 8; ++c) m = fmaxf(m, fabsf(x[c]));
    }
    for (int o = 1; o < lpg; o <<= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (!active) continue;  // whole groups are inactive together (K is a multiple of G)
    // a = Proj(m / qmax): certified fp32 value, fp64 when ambiguous; 1 for a zero group
    bool amb = false;
    float a = a_fast<FMT>(m, qmax, isT, amb);
    if (amb) a = m == 0.f ? 1.f : (float)a_project<FMT>((double)m / (double)qmax, sTd);
    const float ia = __frcp_rn(a);
    const bool ok = sT_ok && in_range(ia) && in_range(isT);
    uint32_t packed = 0;
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const float q = quant<FMT>(x[c], x[c] * isT, ia, ok, a, 1.f, sTd);
      packed |= nibble<FMT>(q) << (4 * c);
    }
    reinterpret_cast<uint32_t*>(p.codes)[(r * p.K + col) / 8] = packed;
    if (leader) a_store_f<FMT>(p.a_store, r * p.nb + col / p.G, a);
  }
}

template <int FMT>
static cudaError_t act_fmt(const ActProblem& p, int xdt, int ctas, cudaStream_t st) {
  if (xdt == DT_BF16) {
    k_act_amax<DT_BF16><<<ctas, kActThreads, 0, st>>>(p);
    k_act<FMT, DT_BF16><<<ctas, kActThreads, 0, st>>>(p);
  } else {
    k_act_amax<DT_F16><<<ctas, kActThreads, 0, st>>>(p);
    k_act<FMT, DT_F16><<<ctas, kActThreads, 0, st>>>(p);
  }
  return cudaGetLastError();
}

}  // namespace dq

extern "C" int dq_act_quant(const void* X, int x_dtype, int64_t rows, int64_t cols, const void* col_scales,
                            int col_dtype, int format, int group, const dq_outputs* out, void* workspace,
                            size_t workspace_bytes, void* stream) {
  if (rows <= 0 || cols <= 0 || group <= 0 || cols % group != 0) return DQ_EINVAL;
  if (format < DQ_INT4 || format > DQ_NVFP4) return DQ_EINVAL;
  if (format == DQ_MXINT4 && group != 32) return DQ_EUNSUPPORTED;
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
  p.M = rows;
  p.K = cols;
  p.nb = (int)(cols / group);
  p.n_slabs = (int)((cols + 255) / 256);
  p.codes = out->codes;
  p.a_store = out->block_scales;
  p.sT_out = out->tensor_scale;
  p.hdr = static_cast<dq::WsHeader*>(workspace);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(workspace, 0, sizeof(dq::WsHeader), st) != cudaSuccess) return DQ_ECUDA;
  const int64_t units = (int64_t)p.n_slabs * rows;
  const int64_t want = (int64_t)sms * dq::kActCtasPerSm;
  const int ctas = (int)((units + 7) / 8 < want ? (units + 7) / 8 : want);
  cudaError_t e;
  switch (format) {
    case DQ_INT4: e = dq::act_fmt<dq::FMT_INT4>(p, x_dtype, ctas, st); break;
    case DQ_MXINT4: e = dq::act_fmt<dq::FMT_MXINT4>(p, x_dtype, ctas, st); break;
    default: e = dq::act_fmt<dq::FMT_NVFP4>(p, x_dtype, ctas, st); break;
  }
  return e == cudaSuccess ? DQ_OK : DQ_ECUDA;
}
