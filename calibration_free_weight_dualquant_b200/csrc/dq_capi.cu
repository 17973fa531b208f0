// dq_capi.cu -- the C ABI of libdq.so (declared in include/dq.h): host-side
// validation, workspace layout and the stream-ordered launch of the solver.
#include "dq.h"
#include "dq_internal.h"

#include <algorithm>
#include <cstring>

namespace {

using dq::Problem;

constexpr size_t kAlign = 256;
size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

struct Plan {
  int TSv, n_strips, P, segmax, P_final, segmax_final, nb;
  int64_t L;
  size_t smem;  // dynamic shared memory of k_iter
  size_t off_counters, off_chg, off_col_part, off_cta_part, off_mse_seg, off_mse_bc, off_amb_list, off_a_work, total;
  size_t l1_zero_bytes;  // L1 init: digit counters to zero (start of the col_part region)
  size_t off_l1_tot, off_l1_norm;
};

// Argument checks that do not touch memory.  Returns DQ_OK or an error code.
int check_shape(int64_t rows, int64_t cols, int format, int group) {
  if (rows <= 0 || cols <= 0 || (cols & 1) || group <= 0) return DQ_EINVAL;
  if (format < DQ_INT4 || format > DQ_MXFP8) return DQ_EINVAL;
  if (cols % group != 0) return DQ_EINVAL;
  if ((format == DQ_MXINT4 || format == DQ_MXFP4 || format == DQ_MXINT8 || format == DQ_MXFP8) && group != 32)
    return DQ_EUNSUPPORTED;
  if (format == DQ_NVFP4 && group != 16) return DQ_EUNSUPPORTED;
  // a block row spans group/8 lanes of a warp: a power of two from 1 to 32
  if (group < 8 || group > dq::kGroupMax || (group & (group - 1)) != 0) return DQ_EUNSUPPORTED;
  if (rows > ((int64_t)1 << 40) / cols) return DQ_EUNSUPPORTED;  // keeps all index products in int64 range
  if (cols / group > INT32_MAX / 2) return DQ_EUNSUPPORTED;
  return DQ_OK;
}

int device_sms(int* sms) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return DQ_ECUDA;
  if (cudaDeviceGetAttribute(sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return DQ_ECUDA;
  return DQ_OK;
}

// Schedule and workspace layout for the current device.
int make_plan(int64_t M, int64_t N, int format, int group, int init, Plan* pl) {
  const int a_bytes = format == DQ_INT4 ? 2 : 1;  // a stored block scale
  int sms = 0;
  int st = device_sms(&sms);
  if (st != DQ_OK) return st;
  pl->nb = (int)(N / group);
  pl->TSv = dq::kBcPerStrip * group;
  pl->n_strips = (pl->nb + dq::kBcPerStrip - 1) / dq::kBcPerStrip;
  pl->L = (int64_t)pl->n_strips * M;
  const int64_t byrows = pl->L / dq::kMinRowsPerCta;
  auto ctas = [&](int64_t want) { return (int)(byrows < want ? (byrows < 1 ? 1 : byrows) : want); };
  // a grid that is a multiple of the strip count (when that keeps at least
  // 90% of the SMs) gives every CTA rows of a single strip in a full pass: no
  // CTA pays a second column-table setup and strip end inside a pass
  int64_t want = (int64_t)sms * dq::kCtasPerSm;
  if (want > dq::kMaxGrid) want = dq::kMaxGrid;
  if (pl->n_strips <= want) {
    const int64_t aligned = want / pl->n_strips * pl->n_strips;
    if (10 * aligned >= 9 * want) want = aligned;
  }
  pl->P = ctas(want);
  // A pass over nv <= n_strips strips splits L = nv M units over
  // pass_ctas(P, nv, L) CTAs; a CTA's contiguous range of len units touches at
  // most ceil(len / M) + 1 strips.  When that count is the aligned one or the
  // grid, len <= ceil(L_full / pmin) (pmin: the fewest such CTAs over every
  // nv); when it is capped at one CTA per kMinRowsPerCta units, len stays
  // below 2 kMinRowsPerCta.
  int pmin = pl->P;
  for (int nv = 1; nv <= pl->n_strips && nv <= pl->P; ++nv)
    pmin = std::min(pmin, dq::pass_ctas(pl->P, nv, INT64_MAX));
  const int64_t len = std::max((pl->L + pmin - 1) / pmin, 2 * dq::kMinRowsPerCta);
  pl->segmax = (int)((len + M - 1) / M + 1);
  pl->P_final = ctas((int64_t)sms * dq::kFinalCtasPerSm);
  pl->segmax_final = pl->segmax;
  pl->smem = (size_t)dq::iter_smem(group / 8, pl->P, pl->segmax).total;
  if (pl->smem > (size_t)227 * 1024) return DQ_EUNSUPPORTED;  // more strips per CTA than shared memory holds
  size_t off = align_up(sizeof(dq::WsHeader));
  // zeroed at the start of a solve: arrival counters, change flags
  pl->off_counters = off;
  off += align_up(sizeof(unsigned) * 8 * (size_t)pl->n_strips);
  pl->off_chg = off;
  off += align_up(sizeof(unsigned) * 3 * (size_t)pl->nb);
  pl->off_col_part = off;
  // the L1-init scratch overlays the column partials (the init kernels run
  // before the first iteration): per-column digits, the total's digits, norms;
  // only the L1 init asks for it
  const size_t dig_bytes = align_up(sizeof(unsigned long long) * dq::kXDigits * (size_t)N);
  const size_t tot_bytes = align_up(sizeof(unsigned long long) * dq::kXDigits);
  pl->off_l1_tot = off + dig_bytes;
  pl->off_l1_norm = pl->off_l1_tot + tot_bytes;
  pl->l1_zero_bytes = dig_bytes + tot_bytes;
  const size_t l1_bytes = dig_bytes + tot_bytes + align_up(sizeof(double) * (size_t)N);
  const size_t part_bytes = align_up(sizeof(double2) * (size_t)pl->P * (size_t)pl->segmax * (size_t)pl->TSv);
  off += (init == DQ_INIT_L1 && l1_bytes > part_bytes) ? l1_bytes : part_bytes;
  pl->off_cta_part = off;
  off += align_up(sizeof(double) * 3 * (size_t)(pl->P > pl->P_final ? pl->P : pl->P_final));
  pl->off_mse_seg = off;
  off += align_up(sizeof(double) * (size_t)pl->P * (size_t)pl->segmax * dq::kBcPerStrip);
  pl->off_mse_bc = off;
  off += align_up(sizeof(double) * 3 * (size_t)pl->nb);
  pl->off_amb_list = off;
  off += align_up(sizeof(int) * (size_t)pl->n_strips * (size_t)pl->TSv);
  pl->off_a_work = off;
  off += align_up((size_t)a_bytes * (size_t)pl->nb * (size_t)M);
  pl->total = off;
  return DQ_OK;
}

bool aligned(const void* p, size_t a) { return ((uintptr_t)p % a) == 0; }

// formats with one byte per code
bool byte_code_format(int format) { return format == DQ_MXINT8 || format == DQ_MXFP8; }

int check_outputs(const dq_outputs* out, int format, int col_dtype) {
  if (!out || !out->codes || !out->block_scales || !out->col_scales || !out->mse) return DQ_EINVAL;
  if (format == DQ_NVFP4 && !out->tensor_scale) return DQ_EINVAL;
  if (!aligned(out->codes, byte_code_format(format) ? 8 : 4) || !aligned(out->block_scales, 2) || !aligned(out->col_scales, 2) ||
      !aligned(out->mse, 8) || (out->tensor_scale && !aligned(out->tensor_scale, 4)))
    return DQ_EINVAL;
  (void)col_dtype;
  return DQ_OK;
}

}  // namespace

namespace dq {

int solve_impl(const void* W, int w_dtype, int64_t rows, int64_t cols, int format, int group, int iters,
               int col_dtype, const dq_outputs* out, void* workspace, size_t workspace_bytes, cudaStream_t stream,
               const dq_options* opt) {
  int st = check_shape(rows, cols, format, group);
  if (st != DQ_OK) return st;
  const int mode = opt ? opt->mode : DQ_MODE_DUAL;
  const int init = opt ? opt->init : DQ_INIT_RTN;
  unsigned long long* changes = opt ? reinterpret_cast<unsigned long long*>(opt->code_changes) : nullptr;
  if (mode < DQ_MODE_DUAL || mode > DQ_MODE_COL) return DQ_EINVAL;
  if (init < DQ_INIT_RTN || init > DQ_INIT_GIVEN) return DQ_EINVAL;
  if (changes != nullptr && !aligned(changes, 8)) return DQ_EINVAL;
  if (w_dtype < DQ_F32 || w_dtype > DQ_F16) return DQ_EINVAL;
  if (col_dtype != DQ_F16 && col_dtype != DQ_BF16) return DQ_EUNSUPPORTED;
  if (iters < 0) return DQ_EINVAL;
  if (!W || !aligned(W, 16)) return DQ_EINVAL;
  st = check_outputs(out, format, col_dtype);
  if (st != DQ_OK) return st;
  if (!workspace || !aligned(workspace, kAlign)) return DQ_EINVAL;
  Plan pl;
  st = make_plan(rows, cols, format, group, init, &pl);
  if (st != DQ_OK) return st;
  if (workspace_bytes < pl.total) return DQ_EWORKSPACE;

  char* ws = static_cast<char*>(workspace);
  dq::Problem p;
  std::memset(&p, 0, sizeof(p));
  p.W = W;
  p.wdt = w_dtype;
  p.fmt = format;
  p.G = group;
  p.col_dt = col_dtype;
  p.M = rows;
  p.N = cols;
  p.nb = pl.nb;
  p.TSv = pl.TSv;
  p.n_strips = pl.n_strips;
  p.P = pl.P;
  p.segmax = pl.segmax;
  p.P_final = pl.P_final;
  p.segmax_final = pl.segmax_final;
  p.L = pl.L;
  p.mode = mode;
  p.init = init;
  p.full_passes = opt ? (opt->full_passes != 0) : 0;
  p.changes = changes;
  p.l1_dig = reinterpret_cast<unsigned long long*>(ws + pl.off_col_part);
  p.l1_tot = reinterpret_cast<unsigned long long*>(ws + pl.off_l1_tot);
  p.l1_norm = reinterpret_cast<double*>(ws + pl.off_l1_norm);
  p.codes = out->codes;
  p.a_store = out->block_scales;
  p.b_store = out->col_scales;
  p.sT_out = out->tensor_scale;
  p.mse = out->mse;
  p.hdr = reinterpret_cast<dq::WsHeader*>(ws);
  p.strip_counter = reinterpret_cast<unsigned*>(ws + pl.off_counters);
  p.col_part = reinterpret_cast<double2*>(ws + pl.off_col_part);
  p.cta_part = reinterpret_cast<double*>(ws + pl.off_cta_part);
  p.chg = reinterpret_cast<unsigned*>(ws + pl.off_chg);
  p.mse_seg = reinterpret_cast<double*>(ws + pl.off_mse_seg);
  p.mse_bc = reinterpret_cast<double*>(ws + pl.off_mse_bc);
  p.amb_list = reinterpret_cast<int*>(ws + pl.off_amb_list);
  p.a_work = ws + pl.off_a_work;

  // header, strip arrival counters and change flags start at zero; the
  // partial buffers need no init
  if (cudaMemsetAsync(ws, 0, pl.off_col_part, stream) != cudaSuccess) return DQ_ECUDA;
  if (init == DQ_INIT_L1 && cudaMemsetAsync(ws + pl.off_col_part, 0, pl.l1_zero_bytes, stream) != cudaSuccess)
    return DQ_ECUDA;
  if (changes && cudaMemsetAsync(changes, 0, sizeof(unsigned long long) * (size_t)(iters + 1), stream) != cudaSuccess)
    return DQ_ECUDA;
  if (dq::launch_solve(p, iters, pl.P_final, stream) != cudaSuccess) return DQ_ECUDA;
  return DQ_OK;
}

// Device-side status of the solve that used `ws`, as a dq_status.
__global__ void k_ws_status(const WsHeader* ws, int* status) {
  const unsigned f = ws->flags;
  *status = (f & kFlagNonFinite) ? DQ_ENONFINITE
           : (f & kFlagBadInit)  ? DQ_EINVAL
           : (f & kFlagTimeout)  ? DQ_ECUDA
                                 : DQ_OK;
}

}  // namespace dq

extern "C" {

size_t dq_workspace_bytes(int64_t rows, int64_t cols, int format, int group) {
  if (check_shape(rows, cols, format, group) != DQ_OK) return 0;
  Plan pl;
  if (make_plan(rows, cols, format, group, DQ_INIT_RTN, &pl) != DQ_OK) return 0;
  return pl.total;
}

size_t dq_workspace_bytes_ex(int64_t rows, int64_t cols, int format, int group, const dq_options* options) {
  if (check_shape(rows, cols, format, group) != DQ_OK) return 0;
  Plan pl;
  if (make_plan(rows, cols, format, group, options ? options->init : DQ_INIT_RTN, &pl) != DQ_OK) return 0;
  return pl.total;
}

int dq_solve(const void* W, int w_dtype, int64_t rows, int64_t cols, int format, int group, int iters, int col_dtype,
             const dq_outputs* out, void* workspace, size_t workspace_bytes, void* stream) {
  return dq::solve_impl(W, w_dtype, rows, cols, format, group, iters, col_dtype, out, workspace, workspace_bytes,
                    static_cast<cudaStream_t>(stream));
}

int dq_solve_mode(const void* W, int w_dtype, int64_t rows, int64_t cols, int format, int group, int iters,
                  int col_dtype, int mode, const dq_outputs* out, void* workspace, size_t workspace_bytes,
                  void* stream) {
  dq_options opt;
  std::memset(&opt, 0, sizeof(opt));
  opt.mode = mode;
  return dq::solve_impl(W, w_dtype, rows, cols, format, group, iters, col_dtype, out, workspace, workspace_bytes,
                        static_cast<cudaStream_t>(stream), &opt);
}

int dq_solve_ex(const void* W, int w_dtype, int64_t rows, int64_t cols, int format, int group, int iters,
                int col_dtype, const dq_options* options, const dq_outputs* out, void* workspace,
                size_t workspace_bytes, void* stream) {
  return dq::solve_impl(W, w_dtype, rows, cols, format, group, iters, col_dtype, out, workspace, workspace_bytes,
                        static_cast<cudaStream_t>(stream), options);
}

int dq_rtn(const void* W, int w_dtype, int64_t rows, int64_t cols, int format, int group, int col_dtype,
           const dq_outputs* out, void* workspace, size_t workspace_bytes, void* stream) {
  return dq::solve_impl(W, w_dtype, rows, cols, format, group, 0, col_dtype, out, workspace, workspace_bytes,
                    static_cast<cudaStream_t>(stream));
}

int dq_sync_status(const void* workspace, void* stream) {
  if (!workspace) return DQ_EINVAL;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return DQ_ECUDA;
  unsigned flags = 0;
  if (cudaMemcpy(&flags, workspace, sizeof(flags), cudaMemcpyDeviceToHost) != cudaSuccess) return DQ_ECUDA;
  if (flags & dq::kFlagNonFinite) return DQ_ENONFINITE;
  if (flags & dq::kFlagBadInit) return DQ_EINVAL;
  return (flags & dq::kFlagTimeout) ? DQ_ECUDA : DQ_OK;
}

int dq_wait_selftest(void* workspace, size_t workspace_bytes, int which, void* stream) {
  if (!workspace || !aligned(workspace, kAlign)) return DQ_EINVAL;
  if (which != 0 && which != 1) return DQ_EINVAL;
  if (workspace_bytes < 512) return DQ_EWORKSPACE;
  if (dq::launch_wait_selftest(workspace, which, static_cast<cudaStream_t>(stream)) != cudaSuccess) return DQ_ECUDA;
  return DQ_OK;
}

int dq_diagnostics(const void* workspace, void* stream, uint64_t out[4]) {
  if (!workspace || !out) return DQ_EINVAL;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return DQ_ECUDA;
  dq::WsHeader h;
  if (cudaMemcpy(&h, workspace, sizeof(h), cudaMemcpyDeviceToHost) != cudaSuccess) return DQ_ECUDA;
  out[0] = h.n_quant_exact;
  out[1] = h.n_block_exact;
  out[2] = h.n_col_exact;
  out[3] = h.n_quant_tie;
  return DQ_OK;
}

int dq_active_block_columns(const void* workspace, void* stream, uint64_t* out) {
  if (!workspace || !out) return DQ_EINVAL;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return DQ_ECUDA;
  dq::WsHeader h;
  if (cudaMemcpy(&h, workspace, sizeof(h), cudaMemcpyDeviceToHost) != cudaSuccess) return DQ_ECUDA;
  *out = h.n_active_bc;
  return DQ_OK;
}

static size_t wsize(int dt) { return dt == DQ_F32 ? 4 : 2; }
// bytes of the codes: one per element on the INT8 and E4M3 grids, else two per byte
static size_t code_bytes(int64_t rows, int64_t cols, int format) {
  return byte_code_format(format) ? (size_t)rows * cols : (size_t)rows * cols / 2;
}

size_t dq_host_workspace_bytes(int64_t rows, int64_t cols, int w_dtype, int format, int group, int iters) {
  if (w_dtype < DQ_F32 || w_dtype > DQ_F16 || iters < 0) return 0;
  size_t solver = dq_workspace_bytes(rows, cols, format, group);
  if (solver == 0) return 0;
  const size_t nb = (size_t)(cols / group);
  size_t tot = align_up((size_t)rows * cols * wsize(w_dtype));
  tot += align_up(code_bytes(rows, cols, format));
  tot += align_up((size_t)rows * nb * (format == DQ_INT4 ? 2 : 1));
  tot += kAlign;  // tensor scale
  tot += align_up((size_t)cols * 2);
  tot += align_up((size_t)(iters + 1) * sizeof(double));
  return tot + solver;
}

int dq_solve_host(const void* W_host, int w_dtype, int64_t rows, int64_t cols, int format, int group, int iters,
                  int col_dtype, const dq_outputs* out_host, void* device_workspace, size_t device_workspace_bytes,
                  void* stream) {
  int st = check_shape(rows, cols, format, group);
  if (st != DQ_OK) return st;
  if (!W_host || w_dtype < DQ_F32 || w_dtype > DQ_F16 || iters < 0) return DQ_EINVAL;
  if (!out_host || !device_workspace || !aligned(device_workspace, kAlign)) return DQ_EINVAL;
  const size_t need = dq_host_workspace_bytes(rows, cols, w_dtype, format, group, iters);
  if (need == 0) return DQ_ECUDA;
  if (device_workspace_bytes < need) return DQ_EWORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  char* base = static_cast<char*>(device_workspace);
  const size_t nb = (size_t)(cols / group);
  const size_t bytes_w = (size_t)rows * cols * wsize(w_dtype);
  const size_t bytes_codes = code_bytes(rows, cols, format);
  const size_t bytes_a = (size_t)rows * nb * (format == DQ_INT4 ? 2 : 1);
  const size_t bytes_b = (size_t)cols * 2;
  const size_t bytes_mse = (size_t)(iters + 1) * sizeof(double);
  char* dW = base;
  base += align_up(bytes_w);
  dq_outputs dout;
  dout.codes = base;
  base += align_up(bytes_codes);
  dout.block_scales = base;
  base += align_up(bytes_a);
  dout.tensor_scale = reinterpret_cast<float*>(base);
  base += kAlign;
  dout.col_scales = base;
  base += align_up(bytes_b);
  dout.mse = reinterpret_cast<double*>(base);
  base += align_up(bytes_mse);
  void* ws = base;
  const size_t ws_bytes = device_workspace_bytes - (size_t)(base - static_cast<char*>(device_workspace));

  if (cudaMemcpyAsync(dW, W_host, bytes_w, cudaMemcpyHostToDevice, s) != cudaSuccess) return DQ_ECUDA;
  st = dq::solve_impl(dW, w_dtype, rows, cols, format, group, iters, col_dtype, &dout, ws, ws_bytes, s);
  if (st != DQ_OK) return st;
  if (out_host->codes && cudaMemcpyAsync(out_host->codes, dout.codes, bytes_codes, cudaMemcpyDeviceToHost, s))
    return DQ_ECUDA;
  if (out_host->block_scales &&
      cudaMemcpyAsync(out_host->block_scales, dout.block_scales, bytes_a, cudaMemcpyDeviceToHost, s))
    return DQ_ECUDA;
  if (out_host->tensor_scale &&
      cudaMemcpyAsync(out_host->tensor_scale, dout.tensor_scale, sizeof(float), cudaMemcpyDeviceToHost, s))
    return DQ_ECUDA;
  if (out_host->col_scales &&
      cudaMemcpyAsync(out_host->col_scales, dout.col_scales, bytes_b, cudaMemcpyDeviceToHost, s))
    return DQ_ECUDA;
  if (out_host->mse && cudaMemcpyAsync(out_host->mse, dout.mse, bytes_mse, cudaMemcpyDeviceToHost, s))
    return DQ_ECUDA;
  return dq_sync_status(ws, stream);
}

int dq_solve_batched(const dq_matrix* mats, int count, int format, int group, int iters, int col_dtype, int* status,
                     void* workspace, size_t workspace_bytes, int* bad_index, void* stream) {
  if (count < 0 || (count > 0 && !mats)) return DQ_EINVAL;
  if (status && !aligned(status, sizeof(int))) return DQ_EINVAL;
  if (!workspace || !aligned(workspace, kAlign)) return DQ_EINVAL;
  if (iters < 0) return DQ_EINVAL;
  if (col_dtype != DQ_F16 && col_dtype != DQ_BF16) return DQ_EUNSUPPORTED;
  // validate everything first: nothing is enqueued unless every matrix is valid
  for (int i = 0; i < count; ++i) {
    const dq_matrix& m = mats[i];
    int st = check_shape(m.rows, m.cols, format, group);
    if (st == DQ_OK && (m.w_dtype < DQ_F32 || m.w_dtype > DQ_F16 || !m.W || !aligned(m.W, 16))) st = DQ_EINVAL;
    if (st == DQ_OK) st = check_outputs(&m.out, format, col_dtype);
    if (st == DQ_OK) {
      Plan pl;
      st = make_plan(m.rows, m.cols, format, group, DQ_INIT_RTN, &pl);
      if (st == DQ_OK && workspace_bytes < pl.total) st = DQ_EWORKSPACE;
    }
    if (st != DQ_OK) {
      if (bad_index) *bad_index = i;
      return st;
    }
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  for (int i = 0; i < count; ++i) {
    const dq_matrix& m = mats[i];
    const int st = dq::solve_impl(m.W, m.w_dtype, m.rows, m.cols, format, group, iters, col_dtype, &m.out, workspace,
                                  workspace_bytes, s);
    if (st != DQ_OK) {
      if (bad_index) *bad_index = i;
      return st;
    }
    if (status) {
      dq::k_ws_status<<<1, 1, 0, s>>>(static_cast<const dq::WsHeader*>(workspace), status + i);
      if (cudaGetLastError() != cudaSuccess) return DQ_ECUDA;
    }
  }
  return DQ_OK;
}

const char* dq_status_str(int status) {
  switch (status) {
    case DQ_OK: return "DQ_OK";
    case DQ_EINVAL: return "DQ_EINVAL: invalid argument";
    case DQ_EUNSUPPORTED: return "DQ_EUNSUPPORTED: unsupported format/group/dtype combination";
    case DQ_EWORKSPACE: return "DQ_EWORKSPACE: workspace too small";
    case DQ_ENONFINITE: return "DQ_ENONFINITE: W holds Inf or NaN";
    case DQ_ECUDA: return "DQ_ECUDA: CUDA runtime error";
  }
  return "unknown dq_status";
}

}  // extern "C"
