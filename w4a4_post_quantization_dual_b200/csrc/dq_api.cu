// dq_api.cu -- extern "C" entry points of include/dq.h: argument validation
// and dispatch.  Nothing here computes; every step runs in the kernels.
#include <cuda_runtime.h>
#include <stdint.h>

#include <stdlib.h>

#include <mutex>
#include <vector>

#include "dq_internal.h"

namespace dq {

bool ensure_kernel_attrs(const void* kernel, int smem_bytes, bool big_cluster) {
  struct Done {
    const void* k;
    int dev, smem;
    bool cluster;
  };
  static std::mutex mu;
  static std::vector<Done> done;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  {
    std::lock_guard<std::mutex> g(mu);
    for (const Done& d : done)
      if (d.k == kernel && d.dev == dev && d.smem >= smem_bytes && (d.cluster || !big_cluster))
        return true;
  }
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes) !=
      cudaSuccess)
    return false;
  // Every kernel of the library asks for the same L1 / shared-memory split
  // (all shared), so consecutive kernels (act quant -> GEMM -> ...) never
  // make the SMs re-partition their on-chip memory between launches.
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                           cudaSharedmemCarveoutMaxShared) != cudaSuccess)
    return false;
  if (big_cluster &&
      cudaFuncSetAttribute(kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) !=
          cudaSuccess)
    return false;
  std::lock_guard<std::mutex> g(mu);
  done.push_back({kernel, dev, smem_bytes, big_cluster});
  return true;
}

bool pdl_enabled() {
  static const bool on = [] {
    const char* e = getenv("DQ_PDL");
    return !(e && e[0] == '0');
  }();
  return on;
}

}  // namespace dq

namespace {

inline bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

inline bool valid_group(int f, int G) {
  switch (f) {
    case DQ_NVFP4: return G == 16;
    case DQ_MXFP4:
    case DQ_MXINT4: return G == 32;
    case DQ_INT4: return G == 32 || G == 64 || G == 128;
    case DQ_MXINT8:
    case DQ_MXFP8: return G == 32;
    case DQ_INT8: return G == 32 || G == 64 || G == 128;
  }
  return false;
}

// 8-bit variants (MXFP8 has a tensor-core linear; INT8 / MXINT8 do not:
// sm_100a's block-scaled MMA takes FP8/FP6/FP4 operands only)
inline bool is_8bit(int f) { return f == DQ_INT8 || f == DQ_MXINT8 || f == DQ_MXFP8; }

inline int resolve_group(int f, int group) { return group > 0 ? group : dq_native_group((dq_format)f); }

inline bool valid_dtype(int t) { return t == DQ_F32 || t == DQ_BF16; }

}  // namespace

extern "C" {

const char* dq_status_string(int s) {
  switch (s) {
    case DQ_OK: return "DQ_OK";
    case DQ_ERR_ARG: return "DQ_ERR_ARG: invalid argument";
    case DQ_ERR_UNSUPPORTED: return "DQ_ERR_UNSUPPORTED: not implemented for these arguments";
    case DQ_ERR_CUDA: return "DQ_ERR_CUDA: CUDA launch or runtime error";
    case DQ_ERR_DEVICE_TIMEOUT: return "DQ_ERR_DEVICE_TIMEOUT: a bounded device wait expired";
    case DQ_ERR_WORKSPACE: return "DQ_ERR_WORKSPACE: workspace missing or too small";
  }
  return "unknown dq status";
}

int dq_version(void) { return 200; }

int dq_native_group(dq_format f) {
  switch (f) {
    case DQ_INT4: return 64;
    case DQ_MXINT4:
    case DQ_MXFP4: return 32;
    case DQ_NVFP4: return 16;
    case DQ_INT8: return 128;
    case DQ_MXINT8:
    case DQ_MXFP8: return 32;
  }
  return 0;
}

size_t dq_scales_bytes(int64_t rows, int64_t k, dq_format f, int group) {
  const int G = resolve_group(f, group);
  if (rows < 0 || k <= 0 || !valid_group(f, G) || k % G) return 0;
  const int64_t S = k / G;
  if (f == DQ_INT4 || f == DQ_INT8) return (size_t)(rows * S * 2);
  return (size_t)(((rows + 127) / 128) * ((S + 3) / 4) * 512);
}

size_t dq_solve_workspace_size(int T) { return T < 0 ? 0 : dq::solve_workspace_bytes(T); }

int dq_solve_scales_ex(const void* W, dq_dtype wt, int64_t m, int64_t n, dq_format f, int group,
                       int T, unsigned flags, const float* r0, const float* c0, float* r,
                       float* c, float* s_tensor, double* mse_trace, void* workspace,
                       size_t ws_bytes, void* stream) {
  const int G = resolve_group(f, group);
  const unsigned known = DQ_SOLVE_ALPHA_ONLY | DQ_SOLVE_BETA_ONLY | DQ_SOLVE_KEEP_TENSOR_SCALE |
                         DQ_SOLVE_TRACE_CODES;
  if (((flags & DQ_SOLVE_TRACE_CODES) && !mse_trace) ||
      !W || !r || !c || !s_tensor || m <= 0 || n <= 0 || T < 0 || !valid_dtype(wt) ||
      !valid_group(f, G) || n % G || !aligned(W, 16) || !aligned(r, 4) || !aligned(c, 4) ||
      !aligned(r0, 4) || !aligned(c0, 4) || (flags & ~known) ||
      ((flags & DQ_SOLVE_ALPHA_ONLY) && (flags & DQ_SOLVE_BETA_ONLY)) ||
      m > (int64_t)1 << 30 || n > (int64_t)1 << 30)
    return DQ_ERR_ARG;
  if (!workspace || ws_bytes < dq::solve_workspace_bytes(T) || !aligned(workspace, 16))
    return DQ_ERR_WORKSPACE;
  return dq::solve_scales(W, wt, m, n, f, G, T, flags, r0, c0, r, c, s_tensor, mse_trace,
                          workspace, (cudaStream_t)stream);
}

size_t dq_solve_batched_workspace_size(int nw, int T) {
  return (T < 0 || nw <= 0) ? 0 : (size_t)nw * dq::solve_workspace_bytes(T);
}

int dq_solve_scales_batched(int nw, const void* const* W, dq_dtype wt, const int64_t* m,
                            const int64_t* n, dq_format f, int group, int T, unsigned flags,
                            float* const* r, float* const* c, float* const* s_tensor,
                            double* const* mse_trace, void* workspace, size_t ws_bytes,
                            void* stream) {
  const int G = resolve_group(f, group);
  const unsigned known = DQ_SOLVE_ALPHA_ONLY | DQ_SOLVE_BETA_ONLY | DQ_SOLVE_KEEP_TENSOR_SCALE |
                         DQ_SOLVE_TRACE_CODES;
  if (((flags & DQ_SOLVE_TRACE_CODES) && !mse_trace) ||
      nw <= 0 || !W || !m || !n || !r || !c || !s_tensor || T < 0 || !valid_dtype(wt) ||
      !valid_group(f, G) || (flags & ~known) ||
      ((flags & DQ_SOLVE_ALPHA_ONLY) && (flags & DQ_SOLVE_BETA_ONLY)))
    return DQ_ERR_ARG;
  for (int i = 0; i < nw; ++i) {
    if (!W[i] || !r[i] || !c[i] || !s_tensor[i] || m[i] <= 0 || n[i] <= 0 || n[i] % G ||
        !aligned(W[i], 16) || !aligned(r[i], 4) || !aligned(c[i], 4) ||
        m[i] > (int64_t)1 << 30 || n[i] > (int64_t)1 << 30)
      return DQ_ERR_ARG;
  }
  if (!workspace || ws_bytes < dq_solve_batched_workspace_size(nw, T) || !aligned(workspace, 16))
    return DQ_ERR_WORKSPACE;
  return dq::solve_scales_batched(nw, W, wt, m, n, f, G, T, flags, r, c, s_tensor, mse_trace,
                                  workspace, (cudaStream_t)stream);
}

int dq_solve_scales(const void* W, dq_dtype wt, int64_t m, int64_t n, dq_format f, int group,
                    int T, float* r, float* c, float* s_tensor, double* mse_trace,
                    void* workspace, size_t ws_bytes, void* stream) {
  return dq_solve_scales_ex(W, wt, m, n, f, group, T, 0u, nullptr, nullptr, r, c, s_tensor,
                            mse_trace, workspace, ws_bytes, stream);
}

int dq_quantize_weight(const void* W, dq_dtype wt, int64_t m, int64_t n, dq_format f, int group,
                       const float* r, const float* c, const float* s_tensor, uint8_t* codes,
                       void* scales, void* stream) {
  const int G = resolve_group(f, group);
  if (!W || !r || !c || !codes || !scales || m <= 0 || n <= 0 || !valid_dtype(wt) ||
      !valid_group(f, G) || n % G || !aligned(W, 16) || !aligned(codes, 16) ||
      !aligned(scales, 16) || (f == DQ_NVFP4 && !s_tensor))
    return DQ_ERR_ARG;
  return dq::quantize_weight(W, wt, m, n, f, G, r, c, s_tensor, codes, scales,
                             (cudaStream_t)stream);
}

int dq_quantize_act(const void* X, dq_dtype xt, int64_t M, int64_t K, const float* c,
                    dq_format f, int group, uint8_t* codes, void* scales, float* s_tok,
                    void* stream) {
  const int G = resolve_group(f, group);
  if (!X || !codes || !scales || M <= 0 || K <= 0 || !valid_dtype(xt) || !valid_group(f, G) ||
      K % G || !aligned(X, 16) || !aligned(codes, 16) || !aligned(scales, 16) ||
      (f == DQ_NVFP4 && !s_tok) || (f != DQ_INT4 && f != DQ_INT8 && K % (4 * G)) ||
      K / G > 4096)
    return DQ_ERR_ARG;
  return dq::quantize_act(X, xt, M, K, c, f, G, codes, scales, s_tok, (cudaStream_t)stream);
}

int dq_act_quant_error(const void* X, dq_dtype xt, int64_t M, int64_t K, const float* c,
                       dq_format f, int group, const uint8_t* codes, const void* scales,
                       const float* s_tok, double* sums, void* stream) {
  const int G = resolve_group(f, group);
  if (!X || !codes || !scales || !sums || M <= 0 || K <= 0 || !valid_dtype(xt) ||
      !valid_group(f, G) || K % G || K % 8 || !aligned(X, 16) ||
      !aligned(codes, is_8bit(f) ? 8 : 4) ||
      !aligned(scales, 2) || !aligned(sums, 8) || !aligned(c, 4) || (f == DQ_NVFP4 && !s_tok))
    return DQ_ERR_ARG;
  return dq::act_quant_error(X, xt, M, K, c, f, G, codes, scales, s_tok, sums,
                             (cudaStream_t)stream);
}

int dq_w4a4_linear_fused(const void* X, dq_dtype xt, const float* c, const uint8_t* B,
                         const uint8_t* sB, const float* s_w, const float* r_row, void* Y,
                         dq_dtype yt, int64_t M, int64_t N, int64_t K, dq_format f,
                         void* stream) {
  if (f != DQ_NVFP4 || xt != DQ_BF16) return DQ_ERR_UNSUPPORTED;
  if (!X || !B || !sB || !s_w || !Y || M <= 0 || N <= 0 || K <= 0 || !valid_dtype(yt) ||
      N % 128 || K % 256 || !aligned(X, 16) || !aligned(B, 16) || !aligned(sB, 16) ||
      !aligned(Y, 16) || !aligned(c, 4) || M > ((int64_t)1 << 31) - 128 ||
      N > ((int64_t)1 << 31) - 128 || K > ((int64_t)1 << 20))
    return DQ_ERR_ARG;
  return dq::w4a4_linear_fused(X, c, B, sB, s_w, r_row, Y, yt, M, N, K, (cudaStream_t)stream);
}

int dq_w4a4_linear(const uint8_t* A, const uint8_t* sA, const float* s_tok, const uint8_t* B,
                   const uint8_t* sB, const float* s_w, const float* r_row, void* Y,
                   dq_dtype yt, int64_t M, int64_t N, int64_t K, dq_format f, void* stream) {
  if (f == DQ_INT8) return DQ_ERR_UNSUPPORTED;
  if (f == DQ_INT4) return DQ_ERR_UNSUPPORTED;
  if (f != DQ_NVFP4 && f != DQ_MXFP4 && f != DQ_MXINT4 && f != DQ_MXFP8 && f != DQ_MXINT8)
    return DQ_ERR_ARG;
  if (!A || !sA || !B || !sB || !Y || M <= 0 || N <= 0 || K <= 0 || !valid_dtype(yt) ||
      N % 128 || K % 256 || !aligned(A, 16) || !aligned(B, 16) || !aligned(sA, 16) ||
      !aligned(sB, 16) || !aligned(Y, 16) || (f == DQ_NVFP4 && !s_tok) ||
      M > ((int64_t)1 << 31) - 128 || N > ((int64_t)1 << 31) - 128 || K > ((int64_t)1 << 20))
    return DQ_ERR_ARG;
  return dq::w4a4_linear(A, sA, s_tok, B, sB, s_w, r_row, Y, yt, M, N, K, f,
                         (cudaStream_t)stream);
}

int dq_device_error(int clear) { return dq::read_device_error(clear); }

int dq_set_wait_limit(uint64_t ns) {
  const unsigned long long v = ns ? (unsigned long long)ns : 2000000000ull;
  if (cudaDeviceSynchronize() != cudaSuccess) return DQ_ERR_CUDA;
  const int a = dq::set_gemm_wait_limit(v), b = dq::set_quant_wait_limit(v);
  return a != DQ_OK ? a : b;
}

}  // extern "C"
