// dq_internal.h -- launchers shared between the entry points (dq_api.cu) and
// the kernel files.  Not part of the public C ABI (include/dq.h).
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

#include "../../include/dq.h"

namespace dq {

size_t solve_workspace_bytes(int T);
int solve_scales(const void* W, int wt, int64_t m, int64_t n, int f, int G, int T,
                 unsigned flags, const float* r0, const float* c0, float* r, float* c, float* sT,
                 double* trace, void* ws, cudaStream_t st);
int quantize_act(const void* X, int xt, int64_t M, int64_t K, const float* c, int f, int G,
                 uint8_t* codes, void* scales, float* s_tok, cudaStream_t st);
int solve_scales_batched(int nw, const void* const* W, int wt, const int64_t* m,
                         const int64_t* n, int f, int G, int T, unsigned flags, float* const* r,
                         float* const* c, float* const* sT, double* const* trace, void* ws,
                         cudaStream_t st);
int w4a4_linear_fused(const void* X, const float* c, const uint8_t* B, const uint8_t* sB,
                      const float* s_w, const float* r_row, void* Y, int yt, int64_t M,
                      int64_t N, int64_t K, cudaStream_t st);
int act_quant_error(const void* X, int xt, int64_t M, int64_t K, const float* c, int f, int G,
                    const uint8_t* codes, const void* scales, const float* s_tok, double* sums,
                    cudaStream_t st);
int quantize_weight(const void* W, int wt, int64_t m, int64_t n, int f, int G, const float* r,
                    const float* c, const float* sT, uint8_t* codes, void* scales,
                    cudaStream_t st);
int w4a4_linear(const uint8_t* A, const uint8_t* sA, const float* s_tok, const uint8_t* B,
                const uint8_t* sB, const float* s_w, const float* r_row, void* Y, int yt,
                int64_t M, int64_t N, int64_t K, int f, cudaStream_t st);
// The linear for at most GEMV_MAX_TOKENS tokens on the CUDA cores (NVFP4,
// MXFP4, K % 1024 == 0); DQ_ERR_UNSUPPORTED when it does not apply, and the
// caller takes the tensor-core kernels.
constexpr int GEMV_MAX_TOKENS = 1;
int w4a4_gemv(const uint8_t* A, const uint8_t* sA, const float* s_tok, const uint8_t* B,
              const uint8_t* sB, const float* s_w, const float* r_row, void* Y, int yt, int64_t M,
              int64_t N, int64_t K, int f, cudaStream_t st);

// Set the function attributes a launch needs (dynamic shared memory bytes,
// the all-shared L1 carveout, and optionally non-portable cluster sizes)
// once per kernel, device and size: they persist, and setting them on every call costs host time
// comparable to a small kernel.  Keyed by the kernel's address.
bool ensure_kernel_attrs(const void* kernel, int smem_bytes, bool big_cluster);

// Programmatic dependent launch for the inference kernels (activation
// quantiser, GEMMs).  Launched with programmatic stream serialisation, a
// kernel may begin while the previous kernel of the stream is still
// finishing; each such kernel therefore runs only its prologue (barrier
// set-up, tensor-memory allocation, descriptor prefetch) before pdl_wait(),
// which returns once the previous kernel has completed and its memory is
// visible, and calls pdl_trigger() right after so that the next kernel's
// launch overlaps its own work.  Without the launch attribute both are no-ops.
// Setting DQ_PDL=0 in the environment launches without the attribute.
bool pdl_enabled();

template <typename... KArgs, typename... Args>
cudaError_t launch_ex(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                      cudaStream_t st, unsigned cluster_x, Args&&... args) {
  cudaLaunchAttribute attr[2];
  unsigned n = 0;
  if (cluster_x > 1) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = cluster_x;
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = 1;
    ++n;
  }
  if (pdl_enabled()) {
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Device-side error words written by kernels whose bounded waits expire
// (one per translation unit); read_device_error combines them.
int read_device_error(int clear);
int read_quant_error(int clear);
// Time limits of the bounded waits (ns) of the GEMM and quantiser kernels.
int set_gemm_wait_limit(unsigned long long ns);
int set_quant_wait_limit(unsigned long long ns);

}  // namespace dq
