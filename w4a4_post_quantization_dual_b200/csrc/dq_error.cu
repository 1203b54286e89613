// dq_error.cu -- quantisation error of the activation path, measured on the
// device from the stored codes: the activation SQNR with and without the
// column scales c = beta^-1 ("DualQuant: Dual-scale Calibration-free
// Weight-and-Activation Quantization for LLMs", Appendix E, Table 6).
//
// For every element the dequantised rescaled activation
//   x~^_ij = q_ij * s_blk (* s_tok_i for NVFP4)      (exact in fp64)
// is mapped back to the activation's own space, x^_ij = x~^_ij / c_j (fp64),
// and the kernel accumulates sum x^2 and sum (x - x^)^2 in fp64.
#include <cuda_runtime.h>
#include <stdint.h>

#include "dq_device.cuh"
#include "dq_internal.h"

namespace dq {

namespace {

__device__ __forceinline__ double e2m1_value_f64(uint32_t code) {
  const double mag[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};
  const double v = mag[code & 7u];
  return (code & 8u) ? -v : v;
}

template <int F, int G, typename XT>
__global__ void __launch_bounds__(256)
act_error_kernel(const XT* __restrict__ X, int64_t M, int64_t K, const float* __restrict__ c,
                 const uint8_t* __restrict__ codes, const uint8_t* __restrict__ scales,
                 const float* __restrict__ s_tok, double* sums) {
  const int64_t n8 = M * (K / 8), S = K / G;
  double sx = 0.0, se = 0.0;
  for (int64_t p = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; p < n8;
       p += (int64_t)gridDim.x * blockDim.x) {
    const int64_t row = p / (K / 8), col = (p % (K / 8)) * 8;
    float x[8];
    if constexpr (sizeof(XT) == 2) {
      bf16x8_to_f32(*reinterpret_cast<const uint4*>(X + row * K + col), x);
    } else {
      const float4 a = reinterpret_cast<const float4*>(X + row * K + col)[0];
      const float4 b = reinterpret_cast<const float4*>(X + row * K + col)[1];
      x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
      x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
    }
    uint32_t w = 0, w2 = 0;   // 8-bit formats: eight bytes in w (0-3), w2 (4-7)
    if constexpr (is_8bit(F)) {
      const uint2 v = *reinterpret_cast<const uint2*>(codes + row * K + col);
      w = v.x;
      w2 = v.y;
    } else {
      w = *reinterpret_cast<const uint32_t*>(codes + row * (K / 2) + col / 2);
    }
    const int64_t s = col / G;
    double scale;
    if constexpr (F == INT4 || F == INT8) {
      const uint16_t h = reinterpret_cast<const uint16_t*>(scales)[row * S + s];
      scale = (double)__uint_as_float((uint32_t)h << 16);
    } else {
      const uint32_t byte = scales[sf_offset(row, s, S)];
      if constexpr (F == NVFP4) scale = (double)ue4m3_value(byte) * (double)s_tok[row];
      else scale = (double)pow2f((int)byte - 127);
    }
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      double q;
      if constexpr (is_8bit(F)) {
        const uint32_t code = ((k < 4 ? w : w2) >> (8 * (k & 3))) & 0xFFu;
        if constexpr (F == MXFP8) {
          const float mag = ue4m3_value(code & 0x7Fu);
          q = (code & 0x80u) ? -(double)mag : (double)mag;
        } else {
          q = (double)((int)(code << 24) >> 24);
        }
      } else {
        const uint32_t code = (w >> (4 * k)) & 0xFu;
        q = is_int_grid(F) ? (double)((int)(code << 28) >> 28) : e2m1_value_f64(code);
      }
      double xh = q * scale;
      if (c != nullptr) xh = xh / (double)c[col + k];
      const double xv = (double)x[k], e = xv - xh;
      sx += xv * xv;
      se += e * e;
    }
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) {
    sx += __shfl_xor_sync(0xffffffffu, sx, o);
    se += __shfl_xor_sync(0xffffffffu, se, o);
  }
  if ((threadIdx.x & 31) == 0) {
    atomicAdd(&sums[0], sx);
    atomicAdd(&sums[1], se);
  }
}

template <int F, int G>
int launch_error(const void* X, int xt, int64_t M, int64_t K, const float* c,
                 const uint8_t* codes, const void* scales, const float* s_tok, double* sums,
                 cudaStream_t st) {
  const int64_t n8 = M * (K / 8);
  const int threads = 256;
  int64_t blocks = (n8 + threads - 1) / threads;
  if (blocks > 148 * 8) blocks = 148 * 8;
  const uint8_t* sc = reinterpret_cast<const uint8_t*>(scales);
  if (xt == 1)
    act_error_kernel<F, G, __nv_bfloat16><<<(unsigned)blocks, threads, 0, st>>>(
        reinterpret_cast<const __nv_bfloat16*>(X), M, K, c, codes, sc, s_tok, sums);
  else
    act_error_kernel<F, G, float><<<(unsigned)blocks, threads, 0, st>>>(
        reinterpret_cast<const float*>(X), M, K, c, codes, sc, s_tok, sums);
  return cudaGetLastError() == cudaSuccess ? DQ_OK : DQ_ERR_CUDA;
}

}  // namespace

int act_quant_error(const void* X, int xt, int64_t M, int64_t K, const float* c, int f, int G,
                    const uint8_t* codes, const void* scales, const float* s_tok, double* sums,
                    cudaStream_t st) {
  if (cudaMemsetAsync(sums, 0, 2 * sizeof(double), st) != cudaSuccess) return DQ_ERR_CUDA;
  switch (f) {
    case NVFP4: return launch_error<NVFP4, 16>(X, xt, M, K, c, codes, scales, s_tok, sums, st);
    case MXFP4: return launch_error<MXFP4, 32>(X, xt, M, K, c, codes, scales, s_tok, sums, st);
    case MXINT4: return launch_error<MXINT4, 32>(X, xt, M, K, c, codes, scales, s_tok, sums, st);
    case INT4:
      if (G == 32) return launch_error<INT4, 32>(X, xt, M, K, c, codes, scales, s_tok, sums, st);
      if (G == 64) return launch_error<INT4, 64>(X, xt, M, K, c, codes, scales, s_tok, sums, st);
      return launch_error<INT4, 128>(X, xt, M, K, c, codes, scales, s_tok, sums, st);
    case MXINT8: return launch_error<MXINT8, 32>(X, xt, M, K, c, codes, scales, s_tok, sums, st);
    case MXFP8: return launch_error<MXFP8, 32>(X, xt, M, K, c, codes, scales, s_tok, sums, st);
    case INT8:
      if (G == 32) return launch_error<INT8, 32>(X, xt, M, K, c, codes, scales, s_tok, sums, st);
      if (G == 64) return launch_error<INT8, 64>(X, xt, M, K, c, codes, scales, s_tok, sums, st);
      return launch_error<INT8, 128>(X, xt, M, K, c, codes, scales, s_tok, sums, st);
  }
  return DQ_ERR_ARG;
}

}  // namespace dq
