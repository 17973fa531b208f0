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
constexpr int kActCtasPerSm = 2;  // 96 registers: two 256-thread CTAs per SM

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

constexpr int kActChunk = 16;  // rows of a (slab, chunk) unit: several units per resident warp
constexpr int kActDepth = 4;   // rows whose loads are in flight ahead of the arithmetic (quantization pass)
constexpr int kAmaxDepth = 16; // the same for the amax pass, whose arithmetic is short

// Raw 16 bytes (8 elements) of row r at column col.
__device__ __forceinline__ uint4 act_raw(const ActProblem& p, int64_t r, int64_t col) {
  return __ldg(reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(p.X) + r * p.K + col));
}

template <int XDT>
__device__ __forceinline__ void act_unpack(uint4 v, const float bcol[8], float x[8]) {
  const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    if (XDT == DT_BF16) {
      x[2 * i] = __uint_as_float(u[i] << 16);
      x[2 * i + 1] = __uint_as_float(u[i] & 0xFFFF0000u);
    } else {
      const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&u[i]));
      x[2 * i] = f.x;
      x[2 * i + 1] = f.y;
    }
  }
#pragma unroll
  for (int c = 0; c < 8; ++c) x[c] *= bcol[c];  // exact: at most 22 significant bits
}

__device__ __forceinline__ void act_cols(const ActProblem& p, int64_t col, bool active, float bcol[8]) {
#pragma unroll
  for (int c = 0; c < 8; ++c) bcol[c] = active ? b_decode(p.b_store, p.col_dt, col + c) : 0.f;
}

// The (slab, chunk) units of a grid: a warp owns 256 columns of kActChunk
// consecutive rows at a time; lane l holds columns 8l .. 8l+7.  `f(r, x)` is
// called for every row with the lane's eight values of X' (active lanes only
// load; inactive lanes see zeros).  Rows are loaded DEPTH ahead.
template <int XDT, int DEPTH, class F>
__device__ __forceinline__ void act_rows(const ActProblem& p, F&& f) {
  const int lane = threadIdx.x & 31;
  const int64_t n_chunks = (p.M + kActChunk - 1) / kActChunk;
  const int64_t units = (int64_t)p.n_slabs * n_chunks;
  const int64_t nwarps = (int64_t)gridDim.x * (blockDim.x / 32);
  for (int64_t u = (int64_t)blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5); u < units; u += nwarps) {
    const int64_t s = u / n_chunks, ch = u - s * n_chunks;
    const int64_t rb = ch * kActChunk, re = min(p.M, rb + kActChunk);
    const int64_t col = s * 256 + lane * 8;
    const bool active = col < p.K;
    const int64_t blk = col / p.G;  // the lane's group within a row
    float bcol[8];
    act_cols(p, col, active, bcol);
    uint4 buf[DEPTH];
#pragma unroll
    for (int k = 0; k < DEPTH; ++k) buf[k] = (active && rb + k < re) ? act_raw(p, rb + k, col) : make_uint4(0, 0, 0, 0);
    for (int64_t r = rb; r < re; r += DEPTH) {
#pragma unroll
      for (int k = 0; k < DEPTH; ++k) {
        if (r + k >= re) break;  // warp-uniform
        const uint4 v = buf[k];
        const int64_t rn = r + k + DEPTH;
        if (active && rn < re) buf[k] = act_raw(p, rn, col);
        float x[8];
        act_unpack<XDT>(v, bcol, x);
        f(r + k, col, blk, active, x);
      }
    }
  }
}

// Pass 1 (NVFP4, and the non-finite check for every format): max |x b|.
template <int XDT>
__global__ void __launch_bounds__(kActThreads, kActCtasPerSm) k_act_amax(ActProblem p) {
  const int lane = threadIdx.x & 31;
  float amax = 0.f;
  bool bad = false;
  act_rows<XDT, kAmaxDepth>(p, [&](int64_t, int64_t, int64_t, bool, const float x[8]) {
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      bad |= !isfinite(x[c]);
      amax = fmaxf(amax, fabsf(x[c]));
    }
  });
  if (bad) atomicOr(&p.hdr->flags, kFlagNonFinite);
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if (lane == 0 && isfinite(amax)) atomicMax(&p.hdr->amax_bits, __float_as_uint(amax));
}

// Pass 2: group scales and codes; a group spans G/8 lanes of a warp.
template <int FMT, int XDT>
__global__ void __launch_bounds__(kActThreads, kActCtasPerSm) k_act(ActProblem p) {
  if (p.hdr->flags & kFlagNonFinite) return;
  const int lane = threadIdx.x & 31;
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
  const float qmax = fmt_e2m1(FMT) ? 6.f : 7.f;
  const int lpg = p.G / 8;  // lanes per group
  const bool leader = (lane & (lpg - 1)) == 0;
  bool bad = false;
  act_rows<XDT, kActDepth>(p, [&](int64_t r, int64_t col, int64_t blk, bool active, const float x[8]) {
    float m = 0.f;
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      if (FMT != FMT_NVFP4) bad |= !isfinite(x[c]);  // NVFP4 checked in the amax pass
      m = fmaxf(m, fabsf(x[c]));
    }
    for (int o = 1; o < lpg; o <<= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (!active) return;  // whole groups are inactive together (K is a multiple of G)
    // a = Proj(m / qmax): certified fp32 value, fp64 when ambiguous; 1 for a zero group
    bool amb = false;
    float a = a_fast<FMT>(m, qmax, isT, amb);
    if (amb) a = m == 0.f ? 1.f : (float)a_project<FMT>((double)m / (double)qmax, sTd);
    const float ia = __frcp_rn(a);
    const bool ok = sT_ok && in_range(ia) && in_range(isT);
    uint32_t packed = 0;
    bool near = !ok;
    if (fmt_e2m1(FMT)) {
      // hardware E2M1 codes of a +-2^-20 relative bracket of the candidate; the
      // lower bracket's code word is already the packed nibbles (element 2i in
      // the low nibble of byte i)
      const float ilo = ia * (1.f - 0x1p-20f), ihi = ia * (1.f + 0x1p-20f);
      uint32_t clo = 0, chi = 0;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float u0 = x[2 * i] * isT, u1 = x[2 * i + 1] * isT;
        uint32_t l, h;
        asm("{\n.reg .b8 t;\ncvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\ncvt.u32.u8 %0, t;\n}"
            : "=r"(l) : "f"(u1 * ilo), "f"(u0 * ilo));
        asm("{\n.reg .b8 t;\ncvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\ncvt.u32.u8 %0, t;\n}"
            : "=r"(h) : "f"(u1 * ihi), "f"(u0 * ihi));
        clo |= l << (8 * i);
        chi |= h << (8 * i);
      }
      near |= clo != chi;
      // a zero magnitude is always the 0x0 nibble (no E2M1 "-0")
      const uint32_t mag = (clo | (clo >> 1) | (clo >> 2)) & 0x11111111u;
      packed = clo & (0x77777777u | (mag << 3));
    } else {
      // round half to even by the 1.5 * 2^23 trick; the clamped sum's low four
      // bits are the two's-complement nibble of q in [-8, 7]
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const float t = fmaf(x[c], ia, 12582912.f);
        const float r = fmaf(x[c], ia, -(t - 12582912.f));
        near |= fabsf(r) > 0.5f - kGuard;
        const float tc = fminf(fmaxf(t, 12582904.f), 12582919.f);
        packed |= (__float_as_uint(tc) & 15u) << (4 * c);
      }
    }
    if (near) {  // exact decisions for this lane's eight elements
      packed = 0;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const float q = quant<FMT>(x[c], x[c] * isT, ia, ok, a, 1.f, sTd);
        packed |= nibble<FMT>(q) << (4 * c);
      }
    }
    reinterpret_cast<uint32_t*>(p.codes)[(r * p.K + col) / 8] = packed;
    if (leader) a_store_f<FMT>(p.a_store, r * p.nb + blk, a);
  });
  if (FMT != FMT_NVFP4 && __any_sync(0xffffffffu, bad) && (threadIdx.x & 31) == 0)
    atomicOr(&p.hdr->flags, kFlagNonFinite);
}

template <int FMT>
static cudaError_t act_fmt(const ActProblem& p, int xdt, int ctas, cudaStream_t st) {
  // the amax pass is needed for the NVFP4 tensor scale only; the other formats
  // check for non-finite values in the quantization pass itself
  if (xdt == DT_BF16) {
    if (FMT == FMT_NVFP4) k_act_amax<DT_BF16><<<ctas, kActThreads, 0, st>>>(p);
    k_act<FMT, DT_BF16><<<ctas, kActThreads, 0, st>>>(p);
  } else {
    if (FMT == FMT_NVFP4) k_act_amax<DT_F16><<<ctas, kActThreads, 0, st>>>(p);
    k_act<FMT, DT_F16><<<ctas, kActThreads, 0, st>>>(p);
  }
  return cudaGetLastError();
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
  // one resident wave: every CTA of the grid runs at once and loops over the
  // (slab, chunk) units, so no second wave leaves SMs idle at the tail
  const int64_t units = (int64_t)p.n_slabs * ((rows + dq::kActChunk - 1) / dq::kActChunk);
  const int64_t want = (int64_t)sms * dq::kActCtasPerSm;
  const int ctas = (int)((units + 7) / 8 < want ? (units + 7) / 8 : want);  // one unit per warp at least
  cudaError_t e;
  switch (format) {
    case DQ_INT4: e = dq::act_fmt<dq::FMT_INT4>(p, x_dtype, ctas, st); break;
    case DQ_MXINT4: e = dq::act_fmt<dq::FMT_MXINT4>(p, x_dtype, ctas, st); break;
    case DQ_MXFP4: e = dq::act_fmt<dq::FMT_MXFP4>(p, x_dtype, ctas, st); break;
    default: e = dq::act_fmt<dq::FMT_NVFP4>(p, x_dtype, ctas, st); break;
  }
  return e == cudaSuccess ? DQ_OK : DQ_ECUDA;
}
