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

template <typename XT, int G>
__device__ __forceinline__ void load_block_smem(const XT* p, float* x) {
  if constexpr (sizeof(XT) == 2) {
#pragma unroll
    for (int u = 0; u < G / 8; ++u) bf16x8_to_f32(reinterpret_cast<const uint4*>(p)[u], x + 8 * u);
  } else {
#pragma unroll
    for (int u = 0; u < G / 4; ++u) {
      float4 v = reinterpret_cast<const float4*>(p)[u];
      x[4 * u] = v.x; x[4 * u + 1] = v.y; x[4 * u + 2] = v.z; x[4 * u + 3] = v.w;
    }
  }
}

// 8-bit codes of G grid arguments z -> G bytes written to dst (16-byte
// aligned): INT8 two's-complement bytes (nearest even, clipped), FP8 E4M3
// bytes (nearest even, saturating).
template <int F, int G>
__device__ __forceinline__ void store_codes8(uint8_t* dst, const float* z) {
  uint32_t w[G / 4];
#pragma unroll
  for (int u = 0; u < G / 4; ++u) {
    if constexpr (F == MXFP8) {
      uint16_t lo, hi;   // element 2k in the low byte of each pair
      asm("cvt.rn.satfinite.e4m3x2.f32 %0, %2, %1;" : "=h"(lo) : "f"(z[4 * u]), "f"(z[4 * u + 1]));
      asm("cvt.rn.satfinite.e4m3x2.f32 %0, %2, %1;" : "=h"(hi)
          : "f"(z[4 * u + 2]), "f"(z[4 * u + 3]));
      w[u] = (uint32_t)lo | ((uint32_t)hi << 16);
    } else {
      uint32_t v = 0;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int q = (int)rintf(fminf(fmaxf(z[4 * u + k], -128.0f), 127.0f));
        v |= ((uint32_t)q & 0xFFu) << (8 * k);
      }
      w[u] = v;
    }
  }
#pragma unroll
  for (int u = 0; u < G / 16; ++u)
    reinterpret_cast<uint4*>(dst)[u] = make_uint4(w[4 * u], w[4 * u + 1], w[4 * u + 2], w[4 * u + 3]);
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
  pdl_wait();
  pdl_trigger();
  const int tid = threadIdx.x, NT = blockDim.x;
  const int64_t S = K / G;
  for (int64_t t = blockIdx.x; t < Mpad; t += gridDim.x) {
    if (t >= M) {  // padding rows of the tensor-core scale layout
      if constexpr (F != INT4 && F != INT8) {
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
      } else if constexpr (is_mx(F)) {
        int e = -127;
        if (ab[j] > 0.0f) {
          e = ilog2f(ab[j]) - mx_emax(F);
          e = e < -127 ? -127 : (e > 127 ? 127 : e);
        } else {
          zero = true;
        }
        scales[sf_offset(t, s, S)] = (uint8_t)(e + 127);
        inv = pow2f(-e);
      } else {
        __nv_bfloat16 h = __float2bfloat16_rn(__fdiv_rn(ab[j], F == INT8 ? 127.0f : 7.0f));
        reinterpret_cast<__nv_bfloat16*>(scales)[t * S + s] = h;
        float sc = __bfloat162float(h);
        zero = (sc == 0.0f);
        inv = zero ? 0.0f : __frcp_rn(sc);
      }
      float z[G];
#pragma unroll
      for (int k = 0; k < G; ++k) z[k] = zero ? 0.0f : __fmul_rn(xt[j][k], inv);
      if constexpr (is_8bit(F)) store_codes8<F, G>(codes + t * K + s * G, z);
      else store_codes<F, G>(codes + t * (K / 2) + s * (G / 2), z);
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
  pdl_trigger();
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
  pdl_wait();   // c was read ahead of the dependency wait, X and the outputs after it
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
// Ring-buffered activation quantiser for the tensor-core formats, bf16 input.
//
// Rows of X are contiguous, so a group of RT rows is one bulk copy
// (cp.async.bulk) into a ring of NST shared-memory stages that thread 0 keeps
// in flight.  Row slot rt of a stage is handled by NTS threads; thread tl owns
// blocks tl + j*NTS (j < BPT) of that row and keeps their column scales c and
// the rescaled values x~ = x*c (Eq. 3) in registers.  A stage is therefore
// read from shared memory exactly once, and is refilled right after the
// barrier of the per-token reduction, while the codes are still being made.
//
// Conflict-free reads: a block is P = G/8 pieces of 16 bytes and lanes own
// consecutive blocks; lane l starts at piece (l / (8/P)) mod P, so the 8 lanes
// of each 128-byte shared-memory wavefront touch 8 distinct bank groups.  The
// values stay in that rotated order (block maximum and scaling do not depend
// on it) and the packed code words are rotated back before the store.
// ---------------------------------------------------------------------------
__device__ int g_dq_quant_error = 0;
// Time limit of the ring's bounded waits, in ns (2 s by default, far beyond
// any legitimate wait; dq_set_wait_limit changes it for testing).  The waits
// that unwind a CTA after an expiry keep the fixed 2 s.
__device__ unsigned long long g_dq_quant_wait_limit_ns = 2000000000ull;

namespace aq {
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ bool wait_parity(uint64_t* bar, uint32_t parity,
                                            bool fixed_limit = false) {
  uint32_t ok;
  // usual case: the stage landed while the previous ones were processed
  asm volatile(
      "{\n\t.reg .pred p;\n\tmbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity) : "memory");
  if (ok) return true;
  const uint64_t limit =
      fixed_limit ? 2000000000ull
                  : *reinterpret_cast<volatile unsigned long long*>(&g_dq_quant_wait_limit_ns);
  // elapsed time: the larger of the global timer (coarse ticks) and the SM
  // cycle counter at two cycles per ns (resolution for very small limits)
  uint64_t t0, c0, t, cyc;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t0));
  c0 = clock64();
  while (true) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity) : "memory");
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    cyc = (clock64() - c0) >> 1;
    const uint64_t el = (t - t0) > cyc ? (t - t0) : cyc;
    // a pipeline wait that outlasted its limit counts as expired even if the
    // phase completed meanwhile (try_wait may suspend until it does); an
    // unwinding wait only needs the phase
    if (ok && (fixed_limit || el <= limit)) return true;
    if (el > limit) {
      atomicExch(&g_dq_quant_error, DQ_ERR_DEVICE_TIMEOUT);
      return false;
    }
  }
}
__device__ __forceinline__ float2 bf16pair(uint32_t w) {
  return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
}
__device__ __forceinline__ float absmax2(float2 v) { return fmaxf(fabsf(v.x), fabsf(v.y)); }
// Eight values (four pairs) -> 32 bits of E2M1 codes, element k in nibble k.
__device__ __forceinline__ uint32_t e2m1x8_pairs(const float2* z) {
  uint32_t out;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
      : "=r"(out)
      : "f"(z[0].x), "f"(z[0].y), "f"(z[1].x), "f"(z[1].y), "f"(z[2].x), "f"(z[2].y),
        "f"(z[3].x), "f"(z[3].y));
  return out;
}
// Eight values -> 32 bits of INT4 codes (round to nearest even, clip to
// [-8, 7]), element k in nibble k.  |z| < 2^22 here, so adding 1.5 * 2^23
// rounds to the nearest integer (ties to even) and leaves it in the low
// mantissa bits; cvt.pack.sat.s4 clips and packs two integers per step.
__device__ __forceinline__ uint32_t int4x8_pairs(const float2* z) {
  const float2 magic = make_float2(12582912.0f, 12582912.0f);
  int n[8];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 t = __fadd2_rn(z[i], magic);
    n[2 * i] = (int)__float_as_uint(t.x) - 0x4B400000;
    n[2 * i + 1] = (int)__float_as_uint(t.y) - 0x4B400000;
  }
  uint32_t d = 0;
#pragma unroll
  for (int i = 3; i >= 0; --i)  // d = (d << 8) | sat(n[2i+1]) << 4 | sat(n[2i])
    asm("cvt.pack.sat.s4.s32.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(n[2 * i + 1]), "r"(n[2 * i]), "r"(d));
  return d;
}
}  // namespace aq

// Block scale (byte of the layout) and reciprocal for one block of
// block maximum ab; st is the per-token scale (NVFP4 only).
template <int F>
__device__ __forceinline__ void act_block_scale(float ab, float st, float d6, uint32_t& byte,
                                                float& inv, bool& zero) {
  if constexpr (F == NVFP4) {
    byte = st > 0.0f ? ue4m3_rn(__fdiv_rn(ab, d6)) : 0u;
    const float sblk = __fmul_rn(ue4m3_value(byte), st);
    zero = (sblk == 0.0f);
    inv = zero ? 0.0f : __frcp_rn(sblk);
  } else {  // OCP MX rule: 2^(floor(log2 amax) - emax), E8M0 byte e + 127
    int e = -127;
    zero = !(ab > 0.0f);
    if (!zero) {
      e = ilog2f(ab) - mx_emax(F);
      e = e < -127 ? -127 : (e > 127 ? 127 : e);
    }
    byte = (uint32_t)(e + 127);
    inv = pow2f(-e);
  }
}

// Codes of one block (values xt in the rotated piece order), rotated back
// and stored; all-zero codes when the block scale is zero.
template <int F, int G>
__device__ __forceinline__ void act_block_codes(const float2* xt, float inv, bool zero, int rot,
                                                uint8_t* dst) {
  constexpr int P = G / 8;
  const float2 inv2 = make_float2(inv, inv);
  uint32_t wv[P];
#pragma unroll
  for (int p = 0; p < P; ++p) {
    float2 z[4];
#pragma unroll
    for (int h = 0; h < 4; ++h) z[h] = __fmul2_rn(xt[4 * p + h], inv2);
    if constexpr (F == MXINT4) wv[p] = aq::int4x8_pairs(z);
    else wv[p] = aq::e2m1x8_pairs(z);
    if (zero) wv[p] = 0u;
  }
  // undo the piece rotation: code word q comes from wv[(q - rot) mod P]
  if (rot & 1) {
    const uint32_t last = wv[P - 1];
#pragma unroll
    for (int q = P - 1; q > 0; --q) wv[q] = wv[q - 1];
    wv[0] = last;
  }
  if constexpr (P == 4) {
    if (rot & 2) {
      const uint32_t a0 = wv[0], a1 = wv[1];
      wv[0] = wv[2]; wv[1] = wv[3]; wv[2] = a0; wv[3] = a1;
    }
  }
  if constexpr (P == 2) *reinterpret_cast<uint2*>(dst) = make_uint2(wv[0], wv[1]);
  else *reinterpret_cast<uint4*>(dst) = make_uint4(wv[0], wv[1], wv[2], wv[3]);
}

// One-byte codes of one block (values xt in the rotated piece order): MXFP8
// E4M3 (nearest even, saturating, sign kept) or MXINT8 integers (nearest
// even, clipped to [-128, 127]); rotated back and stored (G bytes, 16-byte
// aligned); all-zero codes when the block scale is zero.
template <int F, int G>
__device__ __forceinline__ void act_block_codes8(const float2* xt, float inv, bool zero, int rot,
                                                 uint8_t* dst) {
  constexpr int P = G / 8;
  static_assert(P == 4, "one-byte codes: 32-element blocks");
  const float2 inv2 = make_float2(inv, inv);
  uint2 wv[P];   // 8 codes per piece
#pragma unroll
  for (int p = 0; p < P; ++p) {
    uint32_t w[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const float2 z0 = __fmul2_rn(xt[4 * p + 2 * h], inv2), z1 = __fmul2_rn(xt[4 * p + 2 * h + 1], inv2);
      if constexpr (F == MXFP8) {
        uint16_t lo, hi;   // element 2k in the low byte of each pair
        asm("cvt.rn.satfinite.e4m3x2.f32 %0, %2, %1;" : "=h"(lo) : "f"(z0.x), "f"(z0.y));
        asm("cvt.rn.satfinite.e4m3x2.f32 %0, %2, %1;" : "=h"(hi) : "f"(z1.x), "f"(z1.y));
        w[h] = (uint32_t)lo | ((uint32_t)hi << 16);
      } else {
        const float v[4] = {z0.x, z0.y, z1.x, z1.y};
        uint32_t b = 0;
#pragma unroll
        for (int k = 0; k < 4; ++k)
          b |= ((uint32_t)(int)rintf(fminf(fmaxf(v[k], -128.0f), 127.0f)) & 0xFFu) << (8 * k);
        w[h] = b;
      }
    }
    wv[p] = zero ? make_uint2(0u, 0u) : make_uint2(w[0], w[1]);
  }
  // undo the piece rotation: output piece q comes from wv[(q - rot) mod P]
  uint2 o[P];
#pragma unroll
  for (int q = 0; q < P; ++q) {
    const uint2 a0 = wv[q], a1 = wv[(q + 3) & 3], a2 = wv[(q + 2) & 3], a3 = wv[(q + 1) & 3];
    o[q] = rot == 0 ? a0 : (rot == 1 ? a1 : (rot == 2 ? a2 : a3));
  }
  reinterpret_cast<uint4*>(dst)[0] = make_uint4(o[0].x, o[0].y, o[1].x, o[1].y);
  reinterpret_cast<uint4*>(dst)[1] = make_uint4(o[2].x, o[2].y, o[3].x, o[3].y);
}

// x~ = x*c for one block read from shared memory, and its absolute maximum.
template <int G>
__device__ __forceinline__ float act_block_load(const unsigned char* bp, const float2* cv, int rot,
                                                float2* xt) {
  constexpr int P = G / 8, H = G / 2;
#pragma unroll
  for (int p = 0; p < P; ++p) {
    const uint4 v = *reinterpret_cast<const uint4*>(bp + 16 * ((p + rot) & (P - 1)));
    xt[4 * p + 0] = __fmul2_rn(aq::bf16pair(v.x), cv[4 * p + 0]);
    xt[4 * p + 1] = __fmul2_rn(aq::bf16pair(v.y), cv[4 * p + 1]);
    xt[4 * p + 2] = __fmul2_rn(aq::bf16pair(v.z), cv[4 * p + 2]);
    xt[4 * p + 3] = __fmul2_rn(aq::bf16pair(v.w), cv[4 * p + 3]);
  }
  float m[H / 2];
#pragma unroll
  for (int h = 0; h < H / 2; ++h) m[h] = fmaxf(aq::absmax2(xt[2 * h]), aq::absmax2(xt[2 * h + 1]));
#pragma unroll
  for (int w = H / 4; w >= 1; w >>= 1)
#pragma unroll
    for (int h = 0; h < w; ++h) m[h] = fmaxf(m[h], m[h + w]);
  return m[0];
}

// x~ = x*c for one block, the column scales from the shared-memory copy cT:
// piece q (4 floats) of block s at float4 index q * S + s, so that the lanes
// of a wavefront (consecutive blocks, in the rotated piece order of x) read
// disjoint banks.
template <int G>
__device__ __forceinline__ float act_block_load_cs(const unsigned char* bp, const float4* cT,
                                                   int S, int s, int rot, float2* xt) {
  constexpr int P = G / 8, H = G / 2;
#pragma unroll
  for (int p = 0; p < P; ++p) {
    const int q = (p + rot) & (P - 1);
    const uint4 v = *reinterpret_cast<const uint4*>(bp + 16 * q);
    const float4 c0 = cT[(2 * q) * S + s], c1 = cT[(2 * q + 1) * S + s];
    xt[4 * p + 0] = __fmul2_rn(aq::bf16pair(v.x), make_float2(c0.x, c0.y));
    xt[4 * p + 1] = __fmul2_rn(aq::bf16pair(v.y), make_float2(c0.z, c0.w));
    xt[4 * p + 2] = __fmul2_rn(aq::bf16pair(v.z), make_float2(c1.x, c1.y));
    xt[4 * p + 3] = __fmul2_rn(aq::bf16pair(v.w), make_float2(c1.z, c1.w));
  }
  float m[H / 2];
#pragma unroll
  for (int h = 0; h < H / 2; ++h) m[h] = fmaxf(aq::absmax2(xt[2 * h]), aq::absmax2(xt[2 * h + 1]));
#pragma unroll
  for (int w = H / 4; w >= 1; w >>= 1)
#pragma unroll
    for (int h = 0; h < w; ++h) m[h] = fmaxf(m[h], m[h + w]);
  return m[0];
}

// CSM: the column scales live in shared memory (loaded once per CTA) instead
// of registers, so that rows of more blocks keep their rescaled values in
// registers: long rows (K up to ~28K), one row per stage.
template <int F, int G, int BPT, int MAXT, int MINB, bool CSM = false>
__global__ void __launch_bounds__(MAXT, MINB)
quantize_act_ring_kernel(const __nv_bfloat16* __restrict__ X, int64_t M, int64_t Mpad, int64_t K,
                         const float* __restrict__ c, uint8_t* __restrict__ codes,
                         uint8_t* __restrict__ scales, float* __restrict__ s_tok, int NTS, int RT,
                         int NST) {
  constexpr int P = G / 8;   // 16-byte pieces per block
  constexpr int LG = 8 / P;  // consecutive lanes sharing one piece rotation
  constexpr int H = G / 2;   // value pairs per block
  extern __shared__ __align__(128) unsigned char smem_raw[];
  const uint32_t row_bytes = (uint32_t)K * 2;
  const uint32_t stage_bytes = row_bytes * (uint32_t)RT;
  // CSM: [column scales, K floats][stages]; else [stages]
  const float4* cT = reinterpret_cast<const float4*>(smem_raw);
  unsigned char* stages = smem_raw + (CSM ? (size_t)K * 4 : 0);
  uint64_t* full = reinterpret_cast<uint64_t*>(stages + (size_t)stage_bytes * NST);
  uint32_t* rowmax = reinterpret_cast<uint32_t*>(full + NST);  // [3][16] fp32 bits, >= 0
  volatile int* abort_flag = reinterpret_cast<volatile int*>(rowmax + 48);

  const int tid = threadIdx.x, lane = tid & 31;
  const int rt = tid / NTS, tl = tid - rt * NTS;
  const int rot = (lane / LG) % P;
  const int S = (int)(K / G), S4 = S >> 2;

  // per-thread constants of the owned blocks s = tl + j * NTS
  bool own[BPT];
  uint32_t boff[BPT], coff[BPT], sfo[BPT];
#pragma unroll
  for (int j = 0; j < BPT; ++j) {
    const int s = tl + j * NTS;
    own[j] = s < S;
    boff[j] = (uint32_t)rt * row_bytes + (uint32_t)s * (G * 2);
    coff[j] = (uint32_t)s * (is_8bit(F) ? G : G / 2);
    sfo[j] = ((uint32_t)(s >> 2) << 9) | (uint32_t)(s & 3);
  }
  if (tid < 48) rowmax[tid] = 0u;
  if (tid == 0) {
    for (int i = 0; i < NST; ++i)
      asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(aq::smem_u32(&full[i])));
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  pdl_trigger();
  // column scales of the owned blocks, in the rotated piece order: c comes
  // from the solver, never from the kernel launched just before this one, so
  // it is read ahead of the dependency wait (X and the outputs after it)
  float2 cv[CSM ? 1 : BPT][H];
  if constexpr (CSM) {
    // column scales into shared memory, piece-transposed (see act_block_load_cs)
    float4* cw = reinterpret_cast<float4*>(smem_raw);
    for (int i = tid; i < S * (G / 4); i += blockDim.x) {
      const int sb = i / (G / 4), q = i % (G / 4);
      cw[q * S + sb] = c ? __ldg(reinterpret_cast<const float4*>(c) + i)
                         : make_float4(1.f, 1.f, 1.f, 1.f);
    }
  } else {
#pragma unroll
    for (int j = 0; j < BPT; ++j) {
      const int s = tl + j * NTS;
#pragma unroll
      for (int p = 0; p < P; ++p) {
        const int q = (p + rot) & (P - 1);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const float4 v = (c && own[j])
                               ? __ldg(reinterpret_cast<const float4*>(c + (int64_t)s * G + q * 8) + h)
                               : make_float4(1.f, 1.f, 1.f, 1.f);
          cv[j][4 * p + 2 * h] = make_float2(v.x, v.y);
          cv[j][4 * p + 2 * h + 1] = make_float2(v.z, v.w);
        }
      }
    }
  }
  pdl_wait();
  __syncthreads();

  const int64_t step = (int64_t)gridDim.x * RT;  // rows between consecutive groups of a CTA
  auto issue = [&](int64_t t0, int stg) {         // rows t0.. -> stage stg
    uint64_t* bar = &full[stg];
    if (t0 < M) {
      const int64_t rows = (M - t0) < RT ? (M - t0) : RT;
      const uint32_t bytes = (uint32_t)rows * row_bytes;
      asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(
                       aq::smem_u32(bar)), "r"(bytes) : "memory");
      asm volatile(
          "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
              "r"(aq::smem_u32(stages + (size_t)stg * stage_bytes)),
          "l"(X + t0 * K), "r"(bytes), "r"(aq::smem_u32(bar))
          : "memory");
    } else {  // padding rows only: nothing to load
      asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(aq::smem_u32(bar)) : "memory");
    }
  };
  const int64_t first = (int64_t)blockIdx.x * RT;
  if (tid == 0)
    for (int k = 0; k < NST; ++k) issue(first + k * step, k);

  int stg = 0, rb = 0;
  uint32_t phase = 0;
  int64_t t0 = first;
  for (; t0 < Mpad; t0 += step) {
    const int64_t t = t0 + rt;
    const bool rowv = t < M, rowp = t < Mpad;  // both uniform over a warp
    if (!aq::wait_parity(&full[stg], phase)) *abort_flag = 1;
    const unsigned char* sp = stages + (size_t)stg * stage_bytes;
    uint8_t* crow = codes + t * (is_8bit(F) ? K : K / 2);
    uint8_t* sfrow = scales + ((((t >> 7) * S4) << 9) + ((t & 31) << 4) + (((t & 127) >> 5) << 2));

    if constexpr (F == NVFP4) {
      // pass 1: x~ into registers, block maxima, per-token maximum
      float2 xt[BPT][H];
      float ab[BPT];
      float amax = 0.0f;
#pragma unroll
      for (int j = 0; j < BPT; ++j) {
        ab[j] = 0.0f;
        if (rowv && own[j]) {
          if constexpr (CSM) ab[j] = act_block_load_cs<G>(sp + boff[j], cT, S, tl + j * NTS, rot, xt[j]);
          else ab[j] = act_block_load<G>(sp + boff[j], cv[j], rot, xt[j]);
        }
        amax = fmaxf(amax, ab[j]);
      }
      // maxima are >= 0, so their bit patterns order like the values
      const uint32_t wmax = __reduce_max_sync(0xffffffffu, __float_as_uint(amax));
      if (lane == 0) atomicMax(&rowmax[rb * 16 + rt], wmax);
      __syncthreads();  // the stage is consumed; per-token maxima are complete
      if (*abort_flag) break;
      if (tid == 0) issue(t0 + NST * step, stg);
      const int rz = rb == 0 ? 2 : rb - 1;  // buffer last read one iteration ago
      if (tid < 16) rowmax[rz * 16 + tid] = 0u;
      // pass 2: block scales and codes
      if (rowp) {
        const float st = __fdiv_rn(__uint_as_float(rowmax[rb * 16 + rt]), 2688.0f);
        const float d6 = __fmul_rn(6.0f, st);
        if (tl == 0 && rowv) s_tok[t] = st;  // s_tok = amax / (6 * 448)
#pragma unroll
        for (int j = 0; j < BPT; ++j) {
          uint32_t byte = 0;
          if (rowv && own[j]) {
            float inv;
            bool zero;
            act_block_scale<F>(ab[j], st, d6, byte, inv, zero);
            act_block_codes<F, G>(xt[j], inv, zero, rot, crow + coff[j]);
          }
          // one scale byte per block: the 4 bytes of a layout word come from
          // 4 consecutive lanes of the same store instruction
          if (own[j]) sfrow[sfo[j]] = (uint8_t)byte;
        }
      }
      rb = rb == 2 ? 0 : rb + 1;
    } else {
      // MX: blocks are independent, one pass
      if (rowp) {
#pragma unroll
        for (int j = 0; j < BPT; ++j) {
          uint32_t byte = 0;
          if (rowv && own[j]) {
            float2 xt[H];
            float ab;
            if constexpr (CSM) ab = act_block_load_cs<G>(sp + boff[j], cT, S, tl + j * NTS, rot, xt);
            else ab = act_block_load<G>(sp + boff[j], cv[j], rot, xt);
            float inv;
            bool zero;
            act_block_scale<F>(ab, 0.0f, 0.0f, byte, inv, zero);
            if constexpr (is_8bit(F)) act_block_codes8<F, G>(xt, inv, zero, rot, crow + coff[j]);
            else act_block_codes<F, G>(xt, inv, zero, rot, crow + coff[j]);
          }
          if (own[j]) sfrow[sfo[j]] = (uint8_t)byte;
        }
      }
      __syncthreads();  // the stage is consumed
      if (*abort_flag) break;
      if (tid == 0) issue(t0 + NST * step, stg);
    }
    if (++stg == NST) {
      stg = 0;
      phase ^= 1u;
    }
  }
  if (*abort_flag && tid == 0) {
    // a bounded wait expired: the group being processed and the NST - 1
    // after it may still have copies in flight; let each land (each wait is
    // bounded as well) before the CTA exits
    for (int k = 0; k < NST; ++k) {
      const int sk = stg + k < NST ? stg + k : stg + k - NST;
      const uint32_t pk = stg + k < NST ? phase : phase ^ 1u;
      if (t0 + k * step < M) aq::wait_parity(&full[sk], pk, true);
    }
  }
}

// ---------------------------------------------------------------------------
// Weight packer: one CTA per tile of 128 rows x 32 row-blocks (eight 512-byte
// scale atoms of the tensor-core layout).  Lane l of each warp takes block l
// of the tile, so a warp reads and writes one row's 32 consecutive blocks
// contiguously; the 8 warps step through the 128 rows.  beta = fl(1/c) of
// the tile's columns is computed once into shared memory (transposed:
// element k of every lane's block side by side, so the lanes read distinct
// banks); the quantiser argument is fl(fl(w * beta) * alpha), alpha =
// fl(1/r).  The scale atoms are assembled in shared memory and stored
// whole; rows past m and blocks past n/G get zero scale bytes (the layout's
// padding) and no codes.  INT4 / INT8 scales are bf16, row-major.
// ---------------------------------------------------------------------------
template <int F, int G, typename WT>
__global__ void __launch_bounds__(256)
pack_weight_kernel(const WT* __restrict__ W, int64_t m, int64_t n, const float* __restrict__ r,
                   const float* __restrict__ c, const float* __restrict__ sTp,
                   uint8_t* __restrict__ codes, uint8_t* __restrict__ scales) {
  constexpr int TB = 32;                  // blocks per tile, one per lane
  constexpr int CH = G < 32 ? G : 32;     // elements per chunk of a block
  constexpr bool LAYOUT = F != INT4 && F != INT8;
  __shared__ float beta_t[G * TB];        // [element k of a block][lane]
  __shared__ __align__(16) uint8_t atoms[LAYOUT ? 8 * 512 : 16];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t nb = n / G;
  const int64_t r0 = (int64_t)blockIdx.x * 128, b0 = (int64_t)blockIdx.y * TB;
  for (int k = tid; k < TB * G; k += 256) {   // k = block-in-tile * G + element
    const int64_t col = b0 * G + k;
    beta_t[(k % G) * TB + k / G] = col < n ? __frcp_rn(__ldg(c + col)) : 0.0f;
  }
  const float sT = (F == NVFP4) ? *sTp : 1.0f;
  __syncthreads();
  const int64_t b = b0 + lane;
#pragma unroll 1
  for (int rr = warp; rr < 128; rr += 8) {
    const int64_t i = r0 + rr;
    uint32_t byte = 0;
    if (i < m && b < nb) {
      const float rv = r[i * nb + b];
      const float alpha = __frcp_rn(rv);
#pragma unroll
      for (int h = 0; h < G / CH; ++h) {
        float x[CH], z[CH];
        load_block<WT, CH>(W + i * n + b * G + h * CH, x);
#pragma unroll
        for (int k = 0; k < CH; ++k)
          z[k] = __fmul_rn(__fmul_rn(x[k], beta_t[(h * CH + k) * TB + lane]), alpha);
        if constexpr (is_8bit(F)) store_codes8<F, CH>(codes + i * n + b * G + h * CH, z);
        else store_codes<F, CH>(codes + i * (n / 2) + b * (G / 2) + h * (CH / 2), z);
      }
      if constexpr (F == NVFP4) {
        byte = ue4m3_rn(__fdiv_rn(rv, sT));
      } else if constexpr (is_mx(F)) {
        const uint32_t e = (__float_as_uint(rv) >> 23) & 0xFFu;  // exponent of a power of two
        byte = e > 254u ? 254u : e;
      } else {
        reinterpret_cast<__nv_bfloat16*>(scales)[i * nb + b] = __float2bfloat16_rn(rv);
      }
    }
    // byte (row % 32) * 16 + ((row % 128) / 32) * 4 + (block % 4) of atom block / 4
    if constexpr (LAYOUT) atoms[(lane >> 2) * 512 + (rr & 31) * 16 + (rr >> 5) * 4 + (lane & 3)] = (uint8_t)byte;
  }
  if constexpr (LAYOUT) {
    __syncthreads();
    const int64_t S4 = (nb + 3) / 4, a = b0 / 4 + (tid >> 5);
    if (a < S4)
      reinterpret_cast<uint4*>(scales + ((int64_t)blockIdx.x * S4 + a) * 512)[lane] =
          reinterpret_cast<const uint4*>(atoms + (tid >> 5) * 512)[lane];
  }
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
  const int64_t Mpad = (F == INT4 || F == INT8) ? M : ((M + 127) / 128) * 128;
  const XT* Xp = reinterpret_cast<const XT*>(X);
  if constexpr (F == NVFP4 || is_mx(F)) {
    if constexpr (sizeof(XT) == 2) {
      // ring kernel: NTS threads per row, BPT blocks per thread, at most MAXT
      // threads and MINB CTAs per SM (the register budget of each variant)
      auto ring = [&](auto kern, int bpt2, int maxt, int minb) -> int {
        const int NTS = (int)((S + bpt2 - 1) / bpt2 + 31) / 32 * 32;
        int RT = maxt / NTS;
        RT = RT > 16 ? 16 : RT;
        const size_t stage = (size_t)K * sizeof(XT) * RT;
        int NST = (int)((minb == 2 ? 100 * 1024 : 200 * 1024) / stage);
        NST = NST > 8 ? 8 : NST;
        if (RT < 1 || NST < 2) return -1;
        const size_t smem = stage * NST + 8 * NST + 48 * 4 + 16;
        int64_t grid = (Mpad + RT - 1) / RT;
        if (grid > (int64_t)num_sms() * minb) grid = (int64_t)num_sms() * minb;
        if (!ensure_kernel_attrs((const void*)kern, (int)smem, false)) return (int)DQ_ERR_CUDA;
        const cudaError_t e =
            launch_ex(kern, dim3((unsigned)grid), dim3(NTS * RT), smem, st, 1,
                      reinterpret_cast<const __nv_bfloat16*>(X), M, Mpad, K, c, codes, scales,
                      s_tok, NTS, RT, NST);
        return e == cudaSuccess ? (int)DQ_OK : (int)DQ_ERR_CUDA;
      };
      // long rows: column scales in shared memory, one row per stage, up to
      // BPT2 blocks per thread in registers (at most 512 threads)
      auto ring_long = [&](auto kern, int bpt2) -> int {
        const int NTS = (int)((S + bpt2 - 1) / bpt2 + 31) / 32 * 32;
        const size_t stage = (size_t)K * sizeof(XT), cbytes = (size_t)K * 4;
        if (NTS > 512 || cbytes + 2 * stage + 8 * 8 + 48 * 4 + 16 > 227 * 1024) return -1;
        int NST = (int)((227 * 1024 - cbytes - 8 * 8 - 48 * 4 - 16) / stage);
        NST = NST > 8 ? 8 : NST;
        const size_t smem = cbytes + stage * NST + 8 * NST + 48 * 4 + 16;
        int64_t grid = Mpad;
        if (grid > (int64_t)num_sms()) grid = num_sms();
        if (!ensure_kernel_attrs((const void*)kern, (int)smem, false)) return (int)DQ_ERR_CUDA;
        const cudaError_t e =
            launch_ex(kern, dim3((unsigned)grid), dim3(NTS), smem, st, 1,
                      reinterpret_cast<const __nv_bfloat16*>(X), M, Mpad, K, c, codes, scales,
                      s_tok, NTS, 1, NST);
        return e == cudaSuccess ? (int)DQ_OK : (int)DQ_ERR_CUDA;
      };
      int rc = -1;
      if constexpr (F == NVFP4) {
        // two blocks per thread halve the per-row overhead per element once
        // a row has enough blocks to keep 128+ threads busy
        if (S >= 256 && S <= 1024) rc = ring(quantize_act_ring_kernel<F, G, 2, 512, 1>, 2, 512, 1);
        else if (S <= 512) rc = ring(quantize_act_ring_kernel<F, G, 1, 512, 2>, 1, 512, 2);
        else rc = ring_long(quantize_act_ring_kernel<F, G, 4, 512, 1, true>, 4);
      } else {
        if (S <= 384) rc = ring(quantize_act_ring_kernel<F, G, 1, 384, 2>, 1, 384, 2);
        else if (S <= 512) rc = ring(quantize_act_ring_kernel<F, G, 1, 512, 1>, 1, 512, 1);
        else rc = ring_long(quantize_act_ring_kernel<F, G, 2, 512, 1, true>, 2);
      }
      if (rc >= 0) return rc;
    }
  }
  if constexpr (F == NVFP4 || (is_mx(F) && !is_8bit(F))) {
    // rows kernel (fp32 input, or rows too long for the register-resident ring):
    // R rows per CTA iteration, BPT blocks per thread
    constexpr int R = (G == 16) ? 4 : 2;
    NT = (int)((S < 512 ? S : 512) + 31) / 32 * 32;
    const int bpt = (int)((S + NT - 1) / NT);
    int64_t grid = (int64_t)num_sms() * (2048 / NT);
    const int64_t groups = (Mpad + R - 1) / R;
    if (grid > groups) grid = groups;
    if (bpt == 1) {
      auto k = quantize_act_rows_kernel<F, G, XT, 1, R>;
      if (!ensure_kernel_attrs((const void*)k, 0, false)) return DQ_ERR_CUDA;
      if (launch_ex(k, dim3((unsigned)grid), dim3(NT), 0, st, 1, Xp, M, Mpad, K, c, codes, scales,
                    s_tok) != cudaSuccess)
        return DQ_ERR_CUDA;
    } else if (bpt == 2) {
      auto k = quantize_act_rows_kernel<F, G, XT, 2, R / 2>;
      if (!ensure_kernel_attrs((const void*)k, 0, false)) return DQ_ERR_CUDA;
      if (launch_ex(k, dim3((unsigned)grid), dim3(NT), 0, st, 1, Xp, M, Mpad, K, c, codes, scales,
                    s_tok) != cudaSuccess)
        return DQ_ERR_CUDA;
    } else if (bpt <= 4) {
      auto k = quantize_act_rows_kernel<F, G, XT, 4, 1>;
      if (!ensure_kernel_attrs((const void*)k, 0, false)) return DQ_ERR_CUDA;
      if (launch_ex(k, dim3((unsigned)grid), dim3(NT), 0, st, 1, Xp, M, Mpad, K, c, codes, scales,
                    s_tok) != cudaSuccess)
        return DQ_ERR_CUDA;
    } else {
      return DQ_ERR_UNSUPPORTED;
    }
    return cudaGetLastError() == cudaSuccess ? DQ_OK : DQ_ERR_CUDA;
  }
  int64_t grid = (int64_t)num_sms() * (2048 / NT);
  if (grid > Mpad) grid = Mpad;
  cudaError_t e;
  switch (bpt) {
    case 1:
      e = launch_ex(quantize_act_kernel<F, G, XT, 1>, dim3((unsigned)grid), dim3(NT), 0, st, 1, Xp,
                    M, Mpad, K, c, codes, scales, s_tok);
      break;
    case 2:
      e = launch_ex(quantize_act_kernel<F, G, XT, 2>, dim3((unsigned)grid), dim3(NT), 0, st, 1, Xp,
                    M, Mpad, K, c, codes, scales, s_tok);
      break;
    case 3:
    case 4:
      e = launch_ex(quantize_act_kernel<F, G, XT, 4>, dim3((unsigned)grid), dim3(NT), 0, st, 1, Xp,
                    M, Mpad, K, c, codes, scales, s_tok);
      break;
    default: return DQ_ERR_UNSUPPORTED;
  }
  return e == cudaSuccess ? DQ_OK : DQ_ERR_CUDA;
}

int read_quant_error(int clear) {
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_dq_quant_error, sizeof(int)) != cudaSuccess) return DQ_ERR_CUDA;
  if (clear) {
    int z = 0;
    cudaMemcpyToSymbol(g_dq_quant_error, &z, sizeof(int));
  }
  return v;
}

int set_quant_wait_limit(unsigned long long ns) {
  return cudaMemcpyToSymbol(g_dq_quant_wait_limit_ns, &ns, sizeof(ns)) == cudaSuccess ? DQ_OK
                                                                                       : DQ_ERR_CUDA;
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
    case MXINT8: DQ_ACT(MXINT8, 32);
    case MXFP8: DQ_ACT(MXFP8, 32);
    case INT8:
      if (G == 32) { DQ_ACT(INT8, 32); }
      if (G == 64) { DQ_ACT(INT8, 64); }
      DQ_ACT(INT8, 128);
  }
#undef DQ_ACT
  return DQ_ERR_ARG;
}

template <int F, int G, typename WT>
static int launch_pack(const void* W, int64_t m, int64_t n, const float* r, const float* c,
                       const float* sT, uint8_t* codes, uint8_t* scales, cudaStream_t st) {
  const int64_t nb = n / G;
  const int64_t row_tiles = (m + 127) / 128, col_tiles = (nb + 31) / 32;
  if (row_tiles > 0x7FFFFFFF || col_tiles > 65535) return DQ_ERR_UNSUPPORTED;
  auto kern = pack_weight_kernel<F, G, WT>;
  if (!ensure_kernel_attrs((const void*)kern, 0, false)) return DQ_ERR_CUDA;
  kern<<<dim3((unsigned)row_tiles, (unsigned)col_tiles), 256, 0, st>>>(
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
    case MXINT8: DQ_PACK(MXINT8, 32);
    case MXFP8: DQ_PACK(MXFP8, 32);
    case INT8:
      if (G == 32) { DQ_PACK(INT8, 32); }
      if (G == 64) { DQ_PACK(INT8, 64); }
      DQ_PACK(INT8, 128);
  }
#undef DQ_PACK
  return DQ_ERR_ARG;
}

}  // namespace dq
