/*
 * dq.h -- C ABI of the B200 DualQuant solver library (libdq.so).
 *
 * The library computes the DualQuant dual-scale block-coordinate-descent (BCD)
 * weight quantization of one matrix on one GPU:
 *
 *     W  ~  D_a . Q( W / (a b) ) . D_b           (a: block inverse scales,
 *                                                 b: column inverse scales)
 *
 * as defined by the DualQuant reproduction README ("Core equations": the
 * dual-scale model, the closed-form row and column inverse-scale updates with
 * codes fixed, projection onto representable inverse scales, requantization
 * after each update, scale 1 for an all-zero code slice) and by the DualQuant
 * (arXiv 2610.13767) summary (§3 formats, §4.3 BCD, App. B closed forms).
 *
 * Conventions shared by every entry point
 *  - All tensor pointers are DEVICE pointers unless the name says host; the
 *    caller owns every buffer.  The library allocates no memory and keeps no
 *    global state between calls (dq_solve_static excepted: its scratch is one
 *    static device array); calls on different streams with different
 *    workspaces are independent.
 *  - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *    stream) and is asynchronous: a DQ_OK return means the arguments were
 *    valid and the kernels were enqueued.  Conditions detected on the device
 *    (non-finite W) are reported by dq_sync_status().
 *  - Matrices are row-major, `rows` x `cols`, densely packed.
 *  - W is never modified.
 *  - Errors found on the host (bad sizes, NULL pointers, short workspace) are
 *    returned before anything is enqueued; nothing is written then.
 */
#ifndef DQ_H
#define DQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  DQ_OK = 0,
  DQ_EINVAL = 1,        /* NULL pointer, non-positive size, cols not a multiple of group, ... */
  DQ_EUNSUPPORTED = 2,  /* valid but unsupported combination (e.g. group size for the format) */
  DQ_EWORKSPACE = 3,    /* workspace smaller than dq_workspace_bytes() */
  DQ_ENONFINITE = 4,    /* W holds Inf or NaN (reported by dq_sync_status / dq_solve_host) */
  DQ_ECUDA = 5          /* a CUDA runtime call failed */
} dq_status;

/* Formats (DualQuant §3; reproduction README "Local reproduction"):
 *  DQ_INT4   grid [-8,7], block inverse scales fp16, group 8, 16, 32, 64, 128
 *            or 256; column inverse scales fp16 or bf16.  Only powers of two:
 *            a block row spans group/8 lanes of a warp, so group/8 must
 *            divide 32; an even divisor of cols that is not a power of two
 *            (24, 48, 96, ...) returns DQ_EUNSUPPORTED.  The pages' INT4
 *            results and storage figures use groups of 64 and 128.
 *  DQ_MXINT4 grid [-8,7], group 32, block inverse scales 2^k with k in
 *            [-126,126] stored as E8M0 bytes (k+127).
 *  DQ_NVFP4  E2M1 grid {0,+-0.5,+-1,+-1.5,+-2,+-3,+-4,+-6}, group 16, block
 *            inverse scale a = s_T * e with e an FP8 E4M3 value (stored as the
 *            E4M3 byte) and one fp32 tensor scale s_T = fp32(amax|W| / 2688).
 *  DQ_MXFP4  E2M1 grid, group 32, block inverse scales 2^k stored as E8M0 bytes
 *            (the MX family's FP4 member; no tensor scale).
 *  DQ_MXINT8 grid [-128,127], group 32, block inverse scales 2^k stored as
 *            E8M0 bytes (the MX family's INT8 member; the 8-bit weight format
 *            of DualQuant App. G.2).  Absmax initialization with qmax 127.
 *  DQ_MXFP8  FP8 E4M3 grid (3 mantissa bits, subnormals down to 2^-9, largest
 *            value 448, ties to the even mantissa bit, larger magnitudes clip),
 *            group 32, E8M0 block scales (the MX family's FP8 E4M3 member,
 *            App. G.2).  Absmax initialization with qmax 448. */
typedef enum { DQ_INT4 = 0, DQ_MXINT4 = 1, DQ_NVFP4 = 2, DQ_MXFP4 = 3, DQ_MXINT8 = 4, DQ_MXFP8 = 5 } dq_format;

typedef enum { DQ_F32 = 0, DQ_BF16 = 1, DQ_F16 = 2 } dq_dtype;

/* Outputs (device pointers, caller-owned).
 *  codes         uint8 [rows][cols/2]: two 4-bit codes per byte, the even
 *                column in the low nibble.  INT4/MXINT4: two's-complement
 *                nibble of q in [-8,7].  NVFP4/MXFP4: E2M1 nibble s|ee|m; a
 *                zero code is always 0x0.  MXINT8: int8 [rows][cols], one
 *                two's-complement byte of q in [-128,127] per element (8-byte
 *                aligned).  MXFP8: uint8 [rows][cols], the E4M3 bit pattern of
 *                q per element, zero always 0x00 (8-byte aligned).
 *  block_scales  [rows][cols/group]: fp16 (INT4), E8M0 byte (MXINT4, MXFP4,
 *                MXINT8, MXFP8), E4M3 byte (NVFP4).
 *  tensor_scale  one float: s_T for NVFP4, 1.0 for the other formats (which
 *                accept NULL here).
 *  col_scales    [cols] inverse column scales, fp16 or bf16 (col_dtype).
 *  mse           double [iters+1]: mse[0] is the RTN reconstruction MSE,
 *                mse[t] the MSE after BCD iteration t, each
 *                (1/(rows*cols)) * sum (W - a*q*b)^2.
 * The solver uses block_scales and col_scales as its working state, so they
 * must not alias W or the workspace. */
typedef struct {
  void* codes;
  void* block_scales;
  float* tensor_scale;
  void* col_scales;
  double* mse;
} dq_outputs;

/* Device workspace bytes dq_rtn / dq_solve need for this shape (0 on invalid
 * arguments).  The workspace is scratch: its contents on entry do not matter,
 * and it must stay untouched by the caller until the enqueued work finishes
 * (or until dq_sync_status returns).  Alignment: 256 bytes. */
size_t dq_workspace_bytes(int64_t rows, int64_t cols, int format, int group);

/* Absmax round-to-nearest with column scales 1: the solver's initial iterate
 * and its comparison point (DualQuant §3 "symmetric scale max|W|/qmax", qmax 7
 * for INT4/MXINT4, 127 for MXINT8, 448 for MXFP8 and 6 for E2M1, projected onto the admissible set; an
 * all-zero block gets scale 1).  Bit-identical to dq_solve(..., iters = 0).
 * Writes codes, block_scales, tensor_scale, col_scales (all 1) and mse[0]. */
int dq_rtn(const void* W, int w_dtype, int64_t rows, int64_t cols, int format, int group, int col_dtype,
           const dq_outputs* out, void* workspace, size_t workspace_bytes, void* stream);

/* The BCD solver (reproduction README flowchart and "Core equations"):
 * RTN init, then `iters` iterations of
 *   block update with codes fixed   a <- Proj_Fa( sum W q b / sum (q b)^2 )
 *   requantize                      q <- Q( W / (a b) )
 *   column update with codes fixed  b <- Proj_Fb( sum W a q / sum (a q)^2 )
 *   requantize
 * with scale 1 for an all-zero code slice.  iters >= 0; mse has iters+1
 * entries. */
int dq_solve(const void* W, int w_dtype, int64_t rows, int64_t cols, int format, int group, int iters, int col_dtype,
             const dq_outputs* out, void* workspace, size_t workspace_bytes, void* stream);

/* Ablation modes of the solver (DualQuant summary §5.3, Table 4: row scaling
 * alone, column scaling alone). */
typedef enum {
  DQ_MODE_DUAL = 0,  /* the dual-scale BCD iteration (dq_solve) */
  DQ_MODE_ROW = 1,   /* block scales only: row update and requantize; b keeps its initial value */
  DQ_MODE_COL = 2    /* column scales only: column update and requantize; a keeps its initial value */
} dq_mode;

/* dq_solve with an ablation mode (dq_mode); DQ_MODE_DUAL is dq_solve. */
int dq_solve_mode(const void* W, int w_dtype, int64_t rows, int64_t cols, int format, int group, int iters,
                  int col_dtype, int mode, const dq_outputs* out, void* workspace, size_t workspace_bytes,
                  void* stream);

/* Initial iterate of the solver.
 *  DQ_INIT_RTN    absmax RTN block scales, column scales 1 (what dq_solve uses).
 *  DQ_INIT_L1     per-column L1-norm column scales (DualQuant summary §5.3: the
 *                 initialization uses format-native row absmax scales and
 *                 per-column L1-norm scales).  The pages name the norm only; the
 *                 reading implemented: b_j = Proj_Fb(c_j / mu) with
 *                 c_j = sum_i |W_ij| and mu = (sum_ij |W_ij|) / cols, each sum
 *                 exact and rounded once to fp64, b_j = 1 for an all-zero column;
 *                 then the absmax RTN scales of W D_b^-1:
 *                 a = Proj_Fa(max_j (|W_ij| / b_j) / qmax) (1 for a zero block) and,
 *                 for NVFP4, s_T = fp32(max_ij (|W_ij| / b_j) / 2688).  With every
 *                 b_j = 1 this is DQ_INIT_RTN.
 *  DQ_INIT_GIVEN  warm start: the scales already in out->block_scales,
 *                 out->col_scales and (NVFP4) out->tensor_scale, in their storage
 *                 formats, are the initial iterate.  Each must be admissible:
 *                 positive and finite (E8M0 bytes 1..253, E4M3 bytes 0x01..0x7E,
 *                 fp16 0x0001..0x7BFF, bf16 0x0001..0x7F7F, s_T a positive finite
 *                 float).  A violation is found on the device: dq_sync_status then
 *                 returns DQ_EINVAL and nothing but the given scales is written.
 *                 T1 iterations followed by a warm start of T2 more give exactly the
 *                 outputs of T1 + T2 iterations (mse[0] of the second call is mse[T1]
 *                 of the whole). */
typedef enum { DQ_INIT_RTN = 0, DQ_INIT_L1 = 1, DQ_INIT_GIVEN = 2 } dq_init;

/* Options of dq_solve_ex.  A NULL options pointer means all defaults. */
typedef struct {
  int mode;                /* dq_mode (default DQ_MODE_DUAL = 0) */
  int init;                /* dq_init (default DQ_INIT_RTN = 0) */
  uint64_t* code_changes;  /* NULL, or a device array of iters+1 counters: code_changes[0] = 0 and
                            * code_changes[t] = the number of elements whose code differs between
                            * the iterates after iterations t-1 and t (DualQuant summary §4.3 and
                            * App. B: the quantized matrix stabilizes; the relative change of Q is
                            * code_changes[t] / (rows*cols)).  The solver keeps the codes of the
                            * previous iterate in out->codes meanwhile. */
  int full_passes;         /* 0 (default): a block-column (the rows x group slab under one column of
                            * blocks) whose scales come out of an iteration unchanged is at a fixed
                            * point of the iteration and later iterations skip it.  Nonzero: every
                            * iteration processes every block-column.  The outputs are the same. */
} dq_options;

/* Device workspace bytes dq_solve_ex needs with these options (0 on invalid
 * arguments).  Equal to dq_workspace_bytes except for DQ_INIT_L1, whose exact
 * column sums need 88 bytes per column of scratch, and more for very wide
 * matrices. */
size_t dq_workspace_bytes_ex(int64_t rows, int64_t cols, int format, int group, const dq_options* options);

/* The solver with options: ablation mode, initial iterate, changed-code
 * counts.  dq_solve is dq_solve_ex with NULL options.  DQ_EINVAL for an
 * unknown mode or init; DQ_EWORKSPACE below dq_workspace_bytes_ex. */
int dq_solve_ex(const void* W, int w_dtype, int64_t rows, int64_t cols, int format, int group, int iters,
                int col_dtype, const dq_options* options, const dq_outputs* out, void* workspace,
                size_t workspace_bytes, void* stream);

/* Waits for `stream`, then reports what the device recorded in `workspace`
 * during the last dq_rtn / dq_solve that used it: DQ_OK, DQ_ENONFINITE,
 * DQ_EINVAL (a warm start with an inadmissible scale), or DQ_ECUDA if the
 * wait itself failed or a bounded pipeline wait gave up. */
int dq_sync_status(const void* workspace, void* stream);

/* Device bytes dq_solve_host needs: room for a device copy of W, the outputs
 * and the solver workspace (0 on invalid arguments). */
size_t dq_host_workspace_bytes(int64_t rows, int64_t cols, int w_dtype, int format, int group, int iters);

/* dq_solve with HOST input and outputs: copies W (host, ideally pinned) into
 * `device_workspace`, solves there, copies the outputs back into the host
 * buffers of `out_host`, and waits for the stream.  Returns the final status
 * (including DQ_ENONFINITE).  Same argument rules as dq_solve. */
int dq_solve_host(const void* W_host, int w_dtype, int64_t rows, int64_t cols, int format, int group, int iters,
                  int col_dtype, const dq_outputs* out_host, void* device_workspace, size_t device_workspace_bytes,
                  void* stream);

/* Diagnostics of the last solve that used `workspace` (waits for `stream`):
 *   out[0]  lane-rows (8 consecutive elements) whose grid decisions took the
 *           exact path (an fp32 candidate within the guard band of a rounding
 *           boundary, or a scale outside the fast path's range),
 *   out[1]  block inverse-scale updates taken in fp64 (fp32 value too close to
 *           a projection midpoint, a zero or out-of-range sum),
 *   out[2]  column inverse-scale updates recomputed exactly over all rows,
 *   out[3]  lane-rows holding an element that lies exactly on a rounding
 *           boundary (a tie) and that the fast path settled as a certified tie
 *           (the scale product has so few significant bits that a flagged
 *           element can only be an exact tie).
 * Counts cover the BCD iterations only (not init or the final pass). */
int dq_diagnostics(const void* workspace, void* stream, uint64_t out[4]);

/* Work done by the BCD iterations of the last solve that used `workspace`
 * (waits for `stream`): *out = the number of block-columns (the rows x group
 * slab under one column of blocks) processed, summed over the iterations.
 * A block-column whose scales come out of an iteration unchanged is at a fixed
 * point of the BCD map (its block and column updates read only its own
 * scales), so later iterations skip it; the full count is iters * cols/group.
 * No counterpart in the method; a work statistic. */
int dq_active_block_columns(const void* workspace, void* stream, uint64_t* out);

/* Self-test of the solver's bounded device waits (no counterpart in the
 * method; failure detection).  Every wait of the per-iteration kernel (the
 * tile pipeline's ring barriers, the grid barrier between BCD passes, the wait
 * for a block-column's exactly updated column scales) gives up after a time
 * limit (about 1 s), records a timeout in the workspace header and lets the
 * kernel finish, so a lost arrival ends in a status instead of a hung GPU.
 * This call enqueues one such wait that nothing releases: which = 0 waits on a
 * pending count in global memory, which = 1 on a shared-memory ring barrier
 * that no copy completes.  Afterwards dq_sync_status on the same workspace
 * returns DQ_ECUDA, and the context stays usable (the next dq_solve clears the
 * header).  `workspace`: device, 256-byte aligned, at least 512 bytes,
 * overwritten.  Returns DQ_EINVAL / DQ_EWORKSPACE / DQ_ECUDA on bad arguments
 * or a failed launch. */
int dq_wait_selftest(void* workspace, size_t workspace_bytes, int which, void* stream);

/* One matrix of a batched solve: W (device, row-major rows x cols, w_dtype)
 * and its outputs (as for dq_solve, mse with iters+1 entries). */
typedef struct {
  const void* W;
  int w_dtype;
  int64_t rows;
  int64_t cols;
  dq_outputs out;
} dq_matrix;

/* dq_solve for `count` matrices with the same format, group, iteration count
 * and column-scale dtype, enqueued one after another on `stream` and sharing
 * one workspace (stream order keeps them apart).  This is how a whole model's
 * linear layers are quantized in one call (the DualQuant summary, App. I and
 * Table 12: the 224 linear layers of Llama-3.1-8B, each quantized on its
 * own).  The workspace must hold
 * dq_workspace_bytes() of the largest matrix.  Every matrix is validated
 * before anything is enqueued; an invalid one returns its error and
 * `*bad_index` (if non-NULL) receives its index.
 *  status  optional device int[count]: after each matrix a stream-ordered
 *          kernel stores its device-side status (DQ_OK, DQ_ENONFINITE or
 *          DQ_ECUDA), so one non-finite matrix does not hide the others. */
int dq_solve_batched(const dq_matrix* mats, int count, int format, int group, int iters, int col_dtype, int* status,
                     void* workspace, size_t workspace_bytes, int* bad_index, void* stream);

/* Workspace bytes of dq_act_quant (header: flags and the NVFP4 amax). */
#define DQ_ACT_WORKSPACE_BYTES 256u

/* The beta-folded activation quantizer (DualQuant summary §4.4 "Inference-time
 * procedure and overhead"; reproduction README flowchart, "Scale X by column
 * inverse scales, then quantize"): with W ~ D_a Q D_b, X W^T = (X D_b) Q^T D_a,
 * so the activations X [rows][cols] (rows = tokens, cols = input features) are
 * multiplied per channel by the solver's column inverse scales b [cols] and
 * quantized row-wise in the format's own way, in one kernel:
 *   x'   = x * b[col]                      exact in fp32 (bf16/fp16 x and b)
 *   a    = Proj_Fa(max|x'| over the group / qmax), 1 for an all-zero group
 *          (NVFP4: a = s_T * e with s_T = fp32(amax|X'| / 2688), one per call)
 *   q    = Q(x' / a)                       nearest grid value, ties to even
 * Outputs as for dq_solve: out->codes [rows][cols/2], out->block_scales
 * [rows][cols/group], out->tensor_scale (NVFP4; 1.0 otherwise, may be NULL
 * then); col_scales and mse of `out` are not used.  x_dtype is DQ_BF16 or
 * DQ_F16, col_dtype the dtype of `col_scales` (DQ_BF16 or DQ_F16).  The
 * workspace (DQ_ACT_WORKSPACE_BYTES, 256-byte aligned) reports a non-finite
 * X * b through dq_sync_status.  The 4-bit formats only: DQ_MXINT8 and
 * DQ_MXFP8 return DQ_EUNSUPPORTED.  X must be 16-byte aligned, codes 4-byte
 * aligned (16-byte alignment lets a lane store its codes in one vector store).
 * NVFP4 runs its amax pass and quantization pass in one cooperative launch
 * with a grid-wide barrier whose wait is bounded (a wait that runs out is
 * reported as DQ_ECUDA by dq_sync_status); the other formats are one pass. */
int dq_act_quant(const void* X, int x_dtype, int64_t rows, int64_t cols, const void* col_scales, int col_dtype,
                 int format, int group, const dq_outputs* out, void* workspace, size_t workspace_bytes,
                 void* stream);

/* Size of the library-owned device scratch that dq_solve_static uses: 8 MiB.
 * A shape fits when dq_workspace_bytes(rows, cols, format, group) is at most
 * this.  The workspace holds the working block scales (rows x cols/group
 * stored values) and per-CTA column partials that grow with the group; on a
 * 148-SM B200 the four matrix shapes of a Llama-3.1-8B layer (4096 x 4096,
 * 1024 x 4096, 14336 x 4096, 4096 x 14336) fit in NVFP4, the MX formats and
 * INT4 with group 32 or 64 (at most 6.1 MiB), while larger matrices (8192 x
 * 28672 and up) and INT4 groups of 8, 16, 128 or 256 on the 14336 x 4096
 * shape do not: those take dq_solve with a caller's workspace. */
#define DQ_STATIC_SCRATCH_BYTES (8u << 20)

/* dq_solve without a workspace argument, for callers that cannot allocate
 * device memory.  The paper has no counterpart; this is a library-usage entry
 * point.  It serves code that is not allowed to call cudaMalloc: a plugin or
 * extension whose host application owns all device memory through its own
 * pool, or a path on which an allocation would synchronise the device or
 * could fail mid-run.  Such a caller still passes W and the outputs (its own
 * buffers) but no workspace: the solver's scratch is a fixed array of
 * DQ_STATIC_SCRATCH_BYTES defined in the library's device code, which every
 * GPU that loads the library holds until the process exits.
 *
 * Arguments, layouts and results are those of dq_solve (bit-identical
 * outputs); nothing is allocated: no cudaMalloc, cudaFree or allocating
 * library routine.  Returns DQ_EWORKSPACE, before enqueueing anything, when
 * the shape needs more scratch than DQ_STATIC_SCRATCH_BYTES.
 *  status  optional (may be NULL) pointer the GPU can write, 4-byte aligned
 *          (device memory or mapped host memory): after the solve, a stream-
 *          ordered kernel stores DQ_OK, DQ_ENONFINITE or DQ_ECUDA there, the
 *          device-side outcome that dq_sync_status reports for dq_solve.
 * Set-up: every call looks up the scratch array's device address on the
 * current device (cudaGetSymbolAddress; nothing is cached, so a context torn
 * down and created again is handled).  The first call on a device also loads
 * the library's device code there; make that first call before any stream
 * capture on the device.
 * Sharing: all calls on one device share the same scratch, and each call
 * clears the parts that must start at zero.  Calls whose work overlaps on the
 * GPU (different streams, or several host threads, without ordering between
 * them) race on that scratch and give wrong results; order them on one stream
 * or wait between them. */
int dq_solve_static(const void* W, int w_dtype, int64_t rows, int64_t cols, int format, int group, int iters,
                    int col_dtype, const dq_outputs* out, int* status, void* stream);

/* Static string for a status code. */
const char* dq_status_str(int status);

#ifdef __cplusplus
}
#endif

#endif /* DQ_H */
