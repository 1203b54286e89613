// dq_noalloc.cu -- a variant of dq_solve_scales for callers that cannot
// allocate device memory.
//
// Some callers cannot obtain a scratch buffer: a serving process that has
// already handed every free byte of device memory to its own pool (KV cache,
// caching allocator) and must not go around it with cudaMalloc, or a
// latency-critical path that must never block in the driver's allocator.
// For them the solver's small scratch (a per-tensor maximum, ||W||^2 and the
// error trace accumulators) lives in a fixed array compiled into this
// library; the caller still owns and passes every input and output.
//
// The array occupies DQ_NOALLOC_SCRATCH_BYTES on every GPU that loads the
// library, until the process exits.  Its name is a host-side stand-in in
// host code, so the device address is looked up once per device (with that
// device current) and that address is what the kernels receive.
#include <cuda_runtime.h>

#include <mutex>

#include "dq_internal.h"

namespace {

__device__ __align__(256) unsigned char g_solve_scratch[DQ_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 128;
void* g_scratch_addr[kMaxDevices];
int g_setup_status[kMaxDevices];
std::once_flag g_setup_once[kMaxDevices];

}  // namespace

extern "C" int dq_solve_scales_noalloc(const void* W, dq_dtype wt, int64_t m, int64_t n,
                                       dq_format f, int group, int T, float* r, float* c,
                                       float* s_tensor, double* mse_trace, void* stream) {
  if (T < 0) return DQ_ERR_ARG;
  if (T > DQ_NOALLOC_MAX_ROUNDS || dq::solve_workspace_bytes(T) > DQ_NOALLOC_SCRATCH_BYTES)
    return DQ_ERR_WORKSPACE;  // the fixed scratch holds the trace of at most this many rounds
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return DQ_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return DQ_ERR_UNSUPPORTED;
  // The scratch address belongs to the current device, so the stream must be
  // one of that device's streams (the legacy / per-thread default streams,
  // passed as null, always are).
  if (stream) {
    int sdev = -1;
    if (cudaStreamGetDevice((cudaStream_t)stream, &sdev) != cudaSuccess) return DQ_ERR_CUDA;
    if (sdev != dev) return DQ_ERR_ARG;
  }
  // First call on this device: resolve the array's device address with the
  // device current.  Later calls reuse it.
  std::call_once(g_setup_once[dev], [dev]() {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_solve_scratch);
    g_scratch_addr[dev] = (e == cudaSuccess) ? p : nullptr;
    g_setup_status[dev] = (e == cudaSuccess && p) ? DQ_OK : DQ_ERR_CUDA;
  });
  if (g_setup_status[dev] != DQ_OK) return g_setup_status[dev];
  // The solver clears the part of the scratch it uses at the start of the
  // call (stream-ordered), so leftovers from the previous call do not matter.
  return dq_solve_scales(W, wt, m, n, f, group, T, r, c, s_tensor, mse_trace,
                         g_scratch_addr[dev], DQ_NOALLOC_SCRATCH_BYTES, stream);
}
