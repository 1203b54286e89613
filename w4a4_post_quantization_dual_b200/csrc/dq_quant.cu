// dq_quant.cu -- fused activation rescale+quantise and weight packing (sm_100a).
//
// Activations ("DualQuant", Eq. 3 and Section 4.4): X~ = X diag(c), then the
// format-native quantiser computes its own per-row scale on X~.  The column
// scale is applied inside this kernel, so the rescale costs no extra pass
// over X (Section 5.2, "Inference and memory overhead").
//
// Weights (Algorithm 1's returned Q(Diag(alpha) W Diag(beta)), packed as in
// Section 4.4 / Appendix I): codes and encoded row-block scales in the
// layout the block-scaled tensor-core GEMM reads.
//
// Both kernels are HBM-bound streaming passes: one thread owns one block of
// G contiguous elements (16-byte vector loads), CTAs stride over rows.
#include <cuda_runtime.h>
#include <stdint.h>

#include "dq_device.cuh"
#include "dq_internal.h"

namespace dq {

template <typename XT, int G>
__device__ __forceinline__ void load_block(const XT* __restrict__ p, float* x) {
  if constexpr (sizeof(XT) == 2) {
#pragma unroll
    for (int u = 0; u < G / 8; ++u) {
      uint4 v = __ldcs(reinterpret_cast<const uint4*>(p) + u);  // streamed once
      bf16x8_to_f32(v, x + 8 * u);
    }
  } else {
#pragma unroll
    for (int u = 0; u < G / 4; ++u) {
      float4 v = __ldcs(reinterpret_cast<const float4*>(p) + u);
      x[4 * u] = v.x; x[4 * u + 1] = v.y; x[4 * u + 2] = v.z; x[4 * u + 3] = v.w;
    }
  }
}

// Codes of G grid arguments z -> G/2 bytes written to dst (16-byte aligned for G >= 32).
template <int F, int G>
__device__ __forceinline__ void store_codes(uint8_t* dst, const float* z) {
  uint32_t w[G / 8];
#pragma unroll
  for (int u = 0; u < G / 8; ++u) {
    if constexpr (is_int_grid(F)) {
      uint32_t v = 0;
#pragma unroll
      for (int k = 0; k < 8; ++k) v |= int4_code(int4_value_rn(z[8 * u + k])) << (4 * k);
      w[u] = v;
    } else {
      w[u] = e2m1x8(z + 8 * u);
    }
  }
  if constexpr (G == 16) {
    *reinterpret_cast<uint2*>(dst) = make_uint2(w[0], w[1]);
  } else {
#pragma unroll
    for (int u = 0; u < G / 32; ++u)
      reinterpret_cast<uint4*>(dst)[u] = make_uint4(w[4 * u], w[4 * u + 1], w[4 * u + 2], w[4 * u + 3]);
  }
}

// ---------------------------------------------------------------------------
// Activation quantiser.  NT threads per CTA, BPT blocks per thread per row.
// ---------------------------------------------------------------------------
template <int F, int G, typename XT, int BPT>
__global__ void __launch_bounds__(1024)
quantize_act_kernel(const XT* __restrict__ X, int64_t M, int64_t Mpad, int64_t K,
                    const float* __restrict__ c, uint8_t* __restrict__ codes,
                    uint8_t* __restrict__ scales, float* __restrict__ s_tok) {
  __shared__ float red[32];
  const int tid = threadIdx.x, NT = blockDim.x;
  const int64_t S = K / G;
  for (int64_t t = blockIdx.x; t < Mpad; t += gridDim.x) {
    if (t >= M) {  // padding rows of the tensor-core scale layout
      if constexpr (F != INT4) {
        for (int j = 0; j < BPT; ++j) {
          int64_t s = tid + (int64_t)j * NT;
          if (s < S) scales[sf_offset(t, s, S)] = 0;
        }
      }
      continue;
    }
    float xt[BPT][G];
    float ab[BPT];
    float amax = 0.0f;
#pragma unroll
    for (int j = 0; j < BPT; ++j) {
      int64_t s = tid + (int64_t)j * NT;
      ab[j] = 0.0f;
      if (s < S) {
        load_block<XT, G>(X + t * K + s * G, xt[j]);
#pragma unroll
        for (int k = 0; k < G; ++k) {
          float cv = c ? __ldg(c + s * G + k) : 1.0f;
          xt[j][k] = __fmul_rn(xt[j][k], cv);
          ab[j] = fmaxf(ab[j], fabsf(xt[j][k]));
        }
        amax = fmaxf(amax, ab[j]);
      }
    }
    float st = 0.0f;
    if constexpr (F == NVFP4) {
#pragma unroll
      for (int o = 16; o; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
      if ((tid & 31) == 0) red[tid >> 5] = amax;
      __syncthreads();
      if (tid < 32) {
        float v = (tid < (NT + 31) / 32) ? red[tid] : 0.0f;
#pragma unroll
        for (int o = 16; o; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
        if (tid == 0) red[0] = v;
      }
      __syncthreads();
      amax = red[0];
      __syncthreads();  // red[] is rewritten for the next row
      st = __fdiv_rn(amax, 2688.0f);
      if (tid == 0) s_tok[t] = st;
    }
#pragma unroll
    for (int j = 0; j < BPT; ++j) {
      int64_t s = tid + (int64_t)j * NT;
      if (s >= S) continue;
      float inv = 0.0f;
      bool zero = false;
      if constexpr (F == NVFP4) {
        uint32_t byte = 0;
        if (st > 0.0f) byte = ue4m3_rn(__fdiv_rn(ab[j], __fmul_rn(6.0f, st)));
        scales[sf_offset(t, s, S)] = (uint8_t)byte;
        float sblk = __fmul_rn(ue4m3_value(byte), st);
        zero = (sblk == 0.0f);
        inv = zero ? 0.0f : __frcp_rn(sblk);
      } else if constexpr (F == MXFP4 || F == MXINT4) {
        int e = -127;
        if (ab[j] > 0.0f) {
          e = ilog2f(ab[j]) - 2;
          e = e < -127 ? -127 : (e > 127 ? 127 : e);
        } else {
          zero = true;
        }
        scales[sf_offset(t, s, S)] = (uint8_t)(e + 127);
        inv = pow2f(-e);
      } else {
        __nv_bfloat16 h = __float2bfloat16_rn(__fdiv_rn(ab[j], 7.0f));
        reinterpret_cast<__nv_bfloat16*>(scales)[t * S + s] = h;
        float sc = __bfloat162float(h);
        zero = (sc == 0.0f);
        inv = zero ? 0.0f : __frcp_rn(sc);
      }
      float z[G];
#pragma unroll
      for (int k = 0; k < G; ++k) z[k] = zero ? 0.0f : __fmul_rn(xt[j][k], inv);
      store_codes<F, G>(codes + t * (K / 2) + s * (G / 2), z);
    }
  }
}

// ---------------------------------------------------------------------------
// Activation quantiser for the tensor-core formats (G <= 32).  Each thread
// owns BPT column blocks for the whole launch (their column scales c stay in
// registers); a CTA iteration covers R rows, so R rows of loads are in flight
// per thread and the per-token reduction costs one barrier per R rows.
// ---------------------------------------------------------------------------
template <int F, int G, typename XT, int BPT, int R>
__global__ void __launch_bounds__(512)
quantize_act_rows_kernel(const XT* __restrict__ X, int64_t M, int64_t Mpad, int64_t K,
                         const float* __restrict__ c, uint8_t* __restrict__ codes,
                         uint8_t* __restrict__ scales, float* __restrict__ s_tok) {
  constexpr int PIECES = G * (int)sizeof(XT) / 16;   // 16-byte loads per block
  __shared__ float red[2][R][16];
  const int tid = threadIdx.x, NT = blockDim.x, lane = tid & 31, warp = tid >> 5;
  const int NWARP = (NT + 31) >> 5;
  const int64_t S = K / G;
  float cv[BPT][G];
#pragma unroll
  for (int j = 0; j < BPT; ++j) {
    const int64_t s = tid + (int64_t)j * NT;
#pragma unroll
    for (int k = 0; k < G; k += 4) {
      float4 v = (c && s < S) ? __ldg(reinterpret_cast<const float4*>(c + s * G + k))
                              : make_float4(1.f, 1.f, 1.f, 1.f);
      cv[j][k] = v.x; cv[j][k + 1] = v.y; cv[j][k + 2] = v.z; cv[j][k + 3] = v.w;
    }
  }
  // element k of a block held as raw 16-byte pieces
  auto elem = [&](const uint4 (&raw)[PIECES], int k) -> float {
    if constexpr (sizeof(XT) == 2) {
      const uint4& v = raw[k / 8];
      const int w = (k % 8) / 2;
      const uint32_t u = w == 0 ? v.x : (w == 1 ? v.y : (w == 2 ? v.z : v.w));
      return (k & 1) ? __uint_as_float(u & 0xFFFF0000u) : __uint_as_float(u << 16);
    } else {
      const uint4& v = raw[k / 4];
      const int w = k % 4;
      return __uint_as_float(w == 0 ? v.x : (w == 1 ? v.y : (w == 2 ? v.z : v.w)));
    }
  };
  int it = 0;
  for (int64_t t0 = (int64_t)blockIdx.x * R; t0 < Mpad; t0 += (int64_t)gridDim.x * R, ++it) {
    uint4 raw[R][BPT][PIECES];
    float ab[R][BPT];
    float amax[R];
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const int64_t t = t0 + r;
#pragma unroll
      for (int j = 0; j < BPT; ++j) {
        const int64_t s = tid + (int64_t)j * NT;
#pragma unroll
        for (int u = 0; u < PIECES; ++u)
          raw[r][j][u] = (t < M && s < S)
                             ? __ldcs(reinterpret_cast<const uint4*>(X + t * K + s * G) + u)
                             : make_uint4(0, 0, 0, 0);
      }
    }
#pragma unroll
    for (int r = 0; r < R; ++r) {
      amax[r] = 0.0f;
#pragma unroll
      for (int j = 0; j < BPT; ++j) {
        float a = 0.0f;
#pragma unroll
        for (int k = 0; k < G; ++k) a = fmaxf(a, fabsf(__fmul_rn(elem(raw[r][j], k), cv[j][k])));
        ab[r][j] = a;
        amax[r] = fmaxf(amax[r], a);
      }
    }
    float st[R];
    if constexpr (F == NVFP4) {
      const int par = it & 1;  // double-buffered: one barrier per iteration
#pragma unroll
      for (int r = 0; r < R; ++r) {
        float v = amax[r];
#pragma unroll
        for (int o = 16; o; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
        if (lane == 0) red[par][r][warp] = v;
      }
      __syncthreads();
#pragma unroll
      for (int r = 0; r < R; ++r) {
        float v = 0.0f;
        for (int w = 0; w < NWARP; ++w) v = fmaxf(v, red[par][r][w]);
        st[r] = __fdiv_rn(v, 2688.0f);
        if (tid == 0 && t0 + r < M) s_tok[t0 + r] = st[r];
      }
    }
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const int64_t t = t0 + r;
#pragma unroll
      for (int j = 0; j < BPT; ++j) {
        const int64_t s = tid + (int64_t)j * NT;
        uint32_t byte = 0;
        if (t < M && s < S) {
          float inv = 0.0f;
          bool zero = true;
          if constexpr (F == NVFP4) {
            if (st[r] > 0.0f) byte = ue4m3_rn(__fdiv_rn(ab[r][j], __fmul_rn(6.0f, st[r])));
            const float sblk = __fmul_rn(ue4m3_value(byte), st[r]);
            zero = (sblk == 0.0f);
            inv = zero ? 0.0f : __frcp_rn(sblk);
          } else {
            int e = -127;
            if (ab[r][j] > 0.0f) {
              e = ilog2f(ab[r][j]) - 2;
              e = e < -127 ? -127 : (e > 127 ? 127 : e);
              zero = false;
            }
            byte = (uint32_t)(e + 127);
            inv = pow2f(-e);
          }
          float z[G];
#pragma unroll
          for (int k = 0; k < G; ++k)
            z[k] = zero ? 0.0f : __fmul_rn(__fmul_rn(elem(raw[r][j], k), cv[j][k]), inv);
          store_codes<F, G>(codes + t * (K / 2) + s * (G / 2), z);
        }
        // scale bytes of 4 consecutive blocks share one 32-bit word of the
        // layout: gather them in the lane whose block index is a multiple of 4
        const uint32_t b1 = __shfl_down_sync(0xffffffffu, byte, 1);
        const uint32_t b2 = __shfl_down_sync(0xffffffffu, byte, 2);
        const uint32_t b3 = __shfl_down_sync(0xffffffffu, byte, 3);
        if ((s & 3) == 0 && s < S && t < Mpad)
          *reinterpret_cast<uint32_t*>(scales + sf_offset(t, s, S)) =
              byte | (b1 << 8) | (b2 << 16) | (b3 << 24);
      }
    }
  }
}

// ---------------------------------------------------------------------------
// Weight packer: one thread per (row, block).
// ---------------------------------------------------------------------------
template <int F, int G, typename WT>
__global__ void __launch_bounds__(256)
pack_weight_kernel(const WT* __restrict__ W, int64_t m, int64_t n, const float* __restrict__ r,
                   const float* __restrict__ c, const float* __restrict__ sTp,
                   uint8_t* __restrict__ codes, uint8_t* __restrict__ scales) {
  const int64_t nb = n / G;
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= m * nb) return;
  const int64_t i = idx / nb, b = idx % nb;
  const float rr = r[idx];
  const float alpha = __frcp_rn(rr);
  float x[G], z[G];
  if constexpr (sizeof(WT) == 2) {
#pragma unroll
    for (int u = 0; u < G / 8; ++u)
      bf16x8_to_f32(__ldcs(reinterpret_cast<const uint4*>(W + i * n + b * G) + u), x + 8 * u);
  } else {
#pragma unroll
    for (int u = 0; u < G / 4; ++u) {
      float4 v = __ldcs(reinterpret_cast<const float4*>(W + i * n + b * G) + u);
      x[4 * u] = v.x; x[4 * u + 1] = v.y; x[4 * u + 2] = v.z; x[4 * u + 3] = v.w;
    }
  }
#pragma unroll
  for (int k = 0; k < G; ++k)
    z[k] = __fmul_rn(__fmul_rn(x[k], __frcp_rn(__ldg(c + b * G + k))), alpha);
  store_codes<F, G>(codes + i * (n / 2) + b * (G / 2), z);
  if constexpr (F == NVFP4) {
    scales[sf_offset(i, b, nb)] = (uint8_t)ue4m3_rn(__fdiv_rn(rr, *sTp));
  } else if constexpr (F == MXFP4 || F == MXINT4) {
    uint32_t e = (__float_as_uint(rr) >> 23) & 0xFFu;  // exponent of a power of two
    scales[sf_offset(i, b, nb)] = (uint8_t)(e > 254u ? 254u : e);
  } else {
    reinterpret_cast<__nv_bfloat16*>(scales)[idx] = __float2bfloat16_rn(rr);
  }
}

// Zero the padding of a tensor-core scale buffer (rows m..Mpad-1 and the
// scale columns beyond n/G inside the last atom column).
__global__ void zero_bytes_kernel(uint8_t* p, int64_t nbytes) {
  int64_t i = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) * 16;
  if (i + 16 <= nbytes) *reinterpret_cast<uint4*>(p + i) = make_uint4(0, 0, 0, 0);
  else for (int64_t k = i; k < nbytes; ++k) p[k] = 0;
}

// ---------------------------------------------------------------------------
// Host launchers
// ---------------------------------------------------------------------------
static int num_sms() {
  static int n = 0;
  if (!n) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}

template <int F, int G, typename XT>
static int launch_act(const void* X, int64_t M, int64_t K, const float* c, uint8_t* codes,
                      uint8_t* scales, float* s_tok, cudaStream_t st) {
  const int64_t S = K / G;
  int NT = (int)((S < 1024 ? S : 1024) + 31) / 32 * 32;
  const int bpt = (int)((S + NT - 1) / NT);
  const int64_t Mpad = (F == INT4) ? M : ((M + 127) / 128) * 128;
  const XT* Xp = reinterpret_cast<const XT*>(X);
  if constexpr (F != INT4) {
    // rows kernel: R rows per CTA iteration, BPT blocks per thread
    constexpr int R = (G == 16) ? 4 : 2;
    NT = (int)((S < 512 ? S : 512) + 31) / 32 * 32;
    const int bpt = (int)((S + NT - 1) / NT);
    int64_t grid = (int64_t)num_sms() * (2048 / NT);
    const int64_t groups = (Mpad + R - 1) / R;
    if (grid > groups) grid = groups;
    if (bpt == 1) {
      auto k = quantize_act_rows_kernel<F, G, XT, 1, R>;
      if (!ensure_kernel_attrs((const void*)k, 0, false)) return DQ_ERR_CUDA;
      k<<<(unsigned)grid, NT, 0, st>>>(Xp, M, Mpad, K, c, codes, scales, s_tok);
    } else if (bpt == 2) {
      auto k = quantize_act_rows_kernel<F, G, XT, 2, R / 2>;
      if (!ensure_kernel_attrs((const void*)k, 0, false)) return DQ_ERR_CUDA;
      k<<<(unsigned)grid, NT, 0, st>>>(Xp, M, Mpad, K, c, codes, scales, s_tok);
    } else if (bpt <= 4) {
      auto k = quantize_act_rows_kernel<F, G, XT, 4, 1>;
      if (!ensure_kernel_attrs((const void*)k, 0, false)) return DQ_ERR_CUDA;
      k<<<(unsigned)grid, NT, 0, st>>>(Xp, M, Mpad, K, c, codes, scales, s_tok);
    } else {
      return DQ_ERR_UNSUPPORTED;
    }
    return cudaGetLastError() == cudaSuccess ? DQ_OK : DQ_ERR_CUDA;
  }
  int64_t grid = (int64_t)num_sms() * (2048 / NT);
  if (grid > Mpad) grid = Mpad;
  switch (bpt) {
    case 1: quantize_act_kernel<F, G, XT, 1><<<(unsigned)grid, NT, 0, st>>>(Xp, M, Mpad, K, c, codes, scales, s_tok); break;
    case 2: quantize_act_kernel<F, G, XT, 2><<<(unsigned)grid, NT, 0, st>>>(Xp, M, Mpad, K, c, codes, scales, s_tok); break;
    case 3:
    case 4: quantize_act_kernel<F, G, XT, 4><<<(unsigned)grid, NT, 0, st>>>(Xp, M, Mpad, K, c, codes, scales, s_tok); break;
    default: return DQ_ERR_UNSUPPORTED;
  }
  return cudaGetLastError() == cudaSuccess ? DQ_OK : DQ_ERR_CUDA;
}

int quantize_act(const void* X, int xt, int64_t M, int64_t K, const float* c, int f, int G,
                 uint8_t* codes, void* scales, float* s_tok, cudaStream_t st) {
  uint8_t* sc = reinterpret_cast<uint8_t*>(scales);
#define DQ_ACT(FF, GG)                                                                     \
  return xt == 1 ? launch_act<FF, GG, __nv_bfloat16>(X, M, K, c, codes, sc, s_tok, st)   \
                 : launch_act<FF, GG, float>(X, M, K, c, codes, sc, s_tok, st)
  switch (f) {
    case NVFP4: DQ_ACT(NVFP4, 16);
    case MXFP4: DQ_ACT(MXFP4, 32);
    case MXINT4: DQ_ACT(MXINT4, 32);
    case INT4:
      if (G == 32) { DQ_ACT(INT4, 32); }
      if (G == 64) { DQ_ACT(INT4, 64); }
      DQ_ACT(INT4, 128);
  }
#undef DQ_ACT
  return DQ_ERR_ARG;
}

template <int F, int G, typename WT>
static int launch_pack(const void* W, int64_t m, int64_t n, const float* r, const float* c,
                       const float* sT, uint8_t* codes, uint8_t* scales, cudaStream_t st) {
  const int64_t nb = n / G;
  if (F != INT4) {
    // padding rows / scale columns of the tensor-core layout are zeroed first
    int64_t bytes = (int64_t)(((m + 127) / 128) * ((nb + 3) / 4) * 512);
    if ((m & 127) || (nb & 3)) {
      zero_bytes_kernel<<<(unsigned)((bytes / 16 + 255) / 256 + 1), 256, 0, st>>>(scales, bytes);
    }
  }
  int64_t total = m * nb;
  if (!ensure_kernel_attrs((const void*)pack_weight_kernel<F, G, WT>, 0, false)) return DQ_ERR_CUDA;
  pack_weight_kernel<F, G, WT><<<(unsigned)((total + 255) / 256), 256, 0, st>>>(
      reinterpret_cast<const WT*>(W), m, n, r, c, sT, codes, scales);
  return cudaGetLastError() == cudaSuccess ? DQ_OK : DQ_ERR_CUDA;
}

int quantize_weight(const void* W, int wt, int64_t m, int64_t n, int f, int G, const float* r,
                    const float* c, const float* sT, uint8_t* codes, void* scales,
                    cudaStream_t st) {
  uint8_t* sc = reinterpret_cast<uint8_t*>(scales);
#define DQ_PACK(FF, GG)                                                                       \
  return wt == 1 ? launch_pack<FF, GG, __nv_bfloat16>(W, m, n, r, c, sT, codes, sc, st)     \
                 : launch_pack<FF, GG, float>(W, m, n, r, c, sT, codes, sc, st)
  switch (f) {
    case NVFP4: DQ_PACK(NVFP4, 16);
    case MXFP4: DQ_PACK(MXFP4, 32);
    case MXINT4: DQ_PACK(MXINT4, 32);
    case INT4:
      if (G == 32) { DQ_PACK(INT4, 32); }
      if (G == 64) { DQ_PACK(INT4, 64); }
      DQ_PACK(INT4, 128);
  }
#undef DQ_PACK
  return DQ_ERR_ARG;
}

}  // namespace dq
