// dq_static.cu -- dq_solve_static: the solver for callers that cannot allocate
// device memory.
//
// Some callers have no way to obtain a device workspace: code that runs inside
// a host framework which owns every byte of device memory through its own
// pool and forbids raw cudaMalloc, or code on a path where an allocation would
// synchronise the device or may fail at a bad moment.  For them the solver's
// scratch (header, arrival counters, per-CTA partial sums) lives in a fixed
// array that the library itself defines in device memory.  The array belongs
// to the module, so each GPU that loads the library's device code holds
// DQ_STATIC_SCRATCH_BYTES of it until the process exits.
//
// The kernels are the ones dq_solve runs; only the scratch differs.
#include "dq.h"
#include "dq_internal.h"

// Scratch of dq_solve_static, shared by every call on a device.  Host code
// must not pass this name to a kernel: on the host it denotes a stand-in
// object, not the device array.  The device address comes from
// cudaGetSymbolAddress (static_scratch_address below).
static __device__ __align__(256) unsigned char g_static_scratch[DQ_STATIC_SCRATCH_BYTES];

namespace {

// Device address of the scratch array on the current device, looked up on
// every call: a cached address would go stale if the caller tore the context
// down (cudaDeviceReset) and the module were loaded again at another address.
// The lookup is cheap once the module is loaded; the first one on a device
// loads it there.
int static_scratch_address(void** addr) {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || p == nullptr) return DQ_ECUDA;
  *addr = p;
  return DQ_OK;
}

// Turns the flags the solve left in the scratch header into a dq_status.
// Device code names the array directly.
__global__ void k_static_status(int* status) {
  const unsigned f = reinterpret_cast<const dq::WsHeader*>(g_static_scratch)->flags;
  *status = (f & dq::kFlagNonFinite) ? DQ_ENONFINITE : ((f & dq::kFlagTimeout) ? DQ_ECUDA : DQ_OK);
}

}  // namespace

extern "C" int dq_solve_static(const void* W, int w_dtype, int64_t rows, int64_t cols, int format, int group,
                               int iters, int col_dtype, const dq_outputs* out, int* status, void* stream) {
  if (status != nullptr && ((uintptr_t)status % alignof(int)) != 0) return DQ_EINVAL;
  void* scratch = nullptr;
  int st = static_scratch_address(&scratch);
  if (st != DQ_OK) return st;
  // dq::solve_impl validates the arguments, returns DQ_EWORKSPACE when the
  // shape needs more than DQ_STATIC_SCRATCH_BYTES, clears the header and the
  // arrival counters (what must start at zero) and enqueues the kernels.
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  st = dq::solve_impl(W, w_dtype, rows, cols, format, group, iters, col_dtype, out, scratch,
                      (size_t)DQ_STATIC_SCRATCH_BYTES, s);
  if (st != DQ_OK) return st;
  if (status != nullptr) {
    k_static_status<<<1, 1, 0, s>>>(status);
    if (cudaGetLastError() != cudaSuccess) return DQ_ECUDA;
  }
  return DQ_OK;
}
