// dq_device.cuh -- device-side element / scale codecs for sm_100a.
//
// Element grids (DualQuant, Section 3): E2M1 {0,.5,1,1.5,2,3,4,6} for
// MXFP4 / NVFP4, integers -8..7 for INT4 / MXINT4.  Scale sets (Section
// 4.2): BF16, E8M0, UE4M3.  Every conversion rounds to nearest, ties to
// even, saturating, using the PTX cvt instructions whose rounding the PTX
// ISA defines (cvt.rn.satfinite.e2m1x2.f32, cvt.rn.satfinite.e4m3x2.f32,
// cvt.rn.bf16.f32).  All fp32 products / quotients that decide a code are
// single correctly-rounded operations (__fmul_rn / __fdiv_rn / __frcp_rn),
// never contracted into FMAs.
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

namespace dq {

enum Fmt : int { INT4 = 0, MXINT4 = 1, MXFP4 = 2, NVFP4 = 3, INT8 = 4, MXINT8 = 5, MXFP8 = 6 };

// 4-bit integer grid (-8..7)
__host__ __device__ constexpr bool is_int_grid(int f) { return f == INT4 || f == MXINT4; }
// 8-bit variants (INT8 / MXINT8: integers -128..127; MXFP8: FP8 E4M3)
__host__ __device__ constexpr bool is_int8_grid(int f) { return f == INT8 || f == MXINT8; }
__host__ __device__ constexpr bool is_8bit(int f) { return f == INT8 || f == MXINT8 || f == MXFP8; }
// E8M0 block scales
__host__ __device__ constexpr bool is_mx(int f) {
  return f == MXINT4 || f == MXFP4 || f == MXINT8 || f == MXFP8;
}
// OCP MX shared-exponent rule 2^(floor(log2 amax) - emax): exponent of the
// element grid's largest power of two (E2M1 / INT4 2, INT8 6, E4M3 8)
__host__ __device__ constexpr int mx_emax(int f) { return f == MXINT8 ? 6 : (f == MXFP8 ? 8 : 2); }

// ---------------------------------------------------------------- E2M1
// Two fp32 -> one byte: x0 in the low nibble, x1 in the high nibble.
__device__ __forceinline__ uint32_t e2m1x2(float x0, float x1) {
  uint32_t out;
  asm("{\n\t.reg .b8 t;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 t, %2, %1;\n\t"
      "cvt.u32.u8 %0, t;\n\t}"
      : "=r"(out) : "f"(x0), "f"(x1));
  return out;
}

// Eight fp32 -> 32 bits of packed codes (element k in nibble k).
__device__ __forceinline__ uint32_t e2m1x8(const float* x) {
  uint32_t out;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
      : "=r"(out)
      : "f"(x[0]), "f"(x[1]), "f"(x[2]), "f"(x[3]), "f"(x[4]), "f"(x[5]), "f"(x[6]), "f"(x[7]));
  return out;
}

// Byte of two E2M1 codes -> their values as half2 (.x = low nibble).
__device__ __forceinline__ __half2 e2m1x2_to_half2(uint32_t byte) {
  uint32_t h;
  asm("{\n\t.reg .b8 t;\n\t"
      "cvt.u8.u32 t, %1;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, t;\n\t}"
      : "=r"(h) : "r"(byte));
  return *reinterpret_cast<__half2*>(&h);
}

// ---------------------------------------------------------------- INT4
// Round to nearest even, clip to [-8, 7]; returned as the value.
__device__ __forceinline__ float int4_value_rn(float z) {
  float v = rintf(z);
  return fminf(fmaxf(v, -8.0f), 7.0f);
}
__device__ __forceinline__ uint32_t int4_code(float v) { return ((uint32_t)(int)v) & 0xFu; }

// ---------------------------------------------------------------- E4M3
// fp32 (>= 0) -> UE4M3 byte, RNE, saturating at 448 (0x7E).
__device__ __forceinline__ uint32_t ue4m3_rn(float x) {
  uint32_t out;
  asm("{\n\t.reg .b16 t;\n\t"
      "cvt.rn.satfinite.e4m3x2.f32 t, %2, %1;\n\t"
      "cvt.u32.u16 %0, t;\n\t}"
      : "=r"(out) : "f"(x), "f"(0.0f));
  return out & 0xFFu;
}
// Value of a UE4M3 byte (0..126): every E4M3 value is exact in fp16, so the
// hardware conversion e4m3 -> f16 followed by f16 -> f32 is exact.
__device__ __forceinline__ float ue4m3_value(uint32_t b) {
  float f;
  asm("{\n\t.reg .b16 t;\n\t.reg .b32 h;\n\t.reg .b16 lo, hi;\n\t"
      "cvt.u16.u32 t, %1;\n\t"
      "cvt.rn.f16x2.e4m3x2 h, t;\n\t"
      "mov.b32 {lo, hi}, h;\n\t"
      "cvt.f32.f16 %0, lo;\n\t}"
      : "=f"(f) : "r"(b & 0xFFu));
  return f;
}

// ---------------------------------------------------------------- E8M0
__device__ __forceinline__ float pow2f(int k) {  // 2^k, k in [-127, 127]
  return k >= -126 ? __uint_as_float((uint32_t)(k + 127) << 23) : __uint_as_float(0x00400000u);
}
// floor(log2 x) for finite x > 0 (handles fp32 subnormals).
__device__ __forceinline__ int ilog2f(float x) {
  uint32_t u = __float_as_uint(x);
  int e = (int)((u >> 23) & 0xFFu);
  if (e) return e - 127;
  return -127 - (__clz(u & 0x7FFFFFu) - 9);  // subnormal: 2^-149 * mantissa
}

// ---------------------------------------------------------------- projections
// Nearest positive value of each admissible set (DualQuant Section 4.3 /
// Appendix C Remark 1: project the updated inverse scale to the nearest
// representable value).  u > 0 finite.
__device__ __forceinline__ float proj_ue4m3(float u) {
  uint32_t b = ue4m3_rn(u);
  return ue4m3_value(b ? b : 1u);
}
__device__ __forceinline__ float proj_e8m0(float u) {
  uint32_t bits = __float_as_uint(u);
  int e = (int)((bits >> 23) & 0xFFu);
  int k;
  if (e) {
    k = e - 127 + ((bits & 0x7FFFFFu) >= 0x400000u ? 1 : 0);  // midpoint 1.5*2^k -> up
  } else {
    k = (u >= 1.5f * 5.877471754111438e-39f) ? -126 : -127;
  }
  k = k < -127 ? -127 : (k > 127 ? 127 : k);
  return pow2f(k);
}
__device__ __forceinline__ float proj_bf16(float u) {
  __nv_bfloat16 h = __float2bfloat16_rn(u);
  uint16_t b = *reinterpret_cast<uint16_t*>(&h);
  if (b == 0) b = 1;                     // never zero: smallest positive
  if ((b & 0x7F80u) == 0x7F80u) b = 0x7F7F;  // overflow -> largest finite
  return __uint_as_float((uint32_t)b << 16);
}

// Row-block scale set F_alpha.
template <int F>
__device__ __forceinline__ float proj_alpha(float u, float sT) {
  if constexpr (F == NVFP4) {
    float v = proj_ue4m3(__fdiv_rn(u, sT));
    return __fmul_rn(sT, v);
  } else if constexpr (is_mx(F)) {
    return proj_e8m0(u);
  } else {
    return proj_bf16(u);
  }
}
// Column scale set F_beta.
template <int F>
__device__ __forceinline__ float proj_beta(float u) {
  if constexpr (F == NVFP4) return proj_ue4m3(u);
  else if constexpr (is_mx(F)) return proj_e8m0(u);
  else return proj_bf16(u);
}

// Format-native RTN block scale for a block whose rescaled absmax is a
// (initialisation, Section 5.3; OCP MX rule 2^(floor(log2 amax) - 2)).
template <int F>
__device__ __forceinline__ float rtn_block_scale(float a, float sT) {
  if (a == 0.0f) return proj_alpha<F>(1.0f, sT);
  if constexpr (F == NVFP4) {
    return proj_alpha<F>(__fdiv_rn(a, 6.0f), sT);
  } else if constexpr (is_mx(F)) {
    int k = ilog2f(a) - mx_emax(F);
    k = k < -127 ? -127 : (k > 127 ? 127 : k);
    return pow2f(k);
  } else {
    return proj_bf16(__fdiv_rn(a, F == INT8 ? 127.0f : 7.0f));
  }
}

// ---------------------------------------------------------------- bf16 loads
__device__ __forceinline__ void bf16x8_to_f32(const uint4& v, float* x) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    x[2 * i] = __uint_as_float(w[i] << 16);
    x[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

// Programmatic dependent launch (see pdl_enabled in dq_internal.h): wait for
// the previous kernel of the stream to complete, and let the next one launch.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Block-scale layout of the block-scaled tensor-core MMA (see include/dq.h).
__host__ __device__ __forceinline__ int64_t sf_offset(int64_t row, int64_t s, int64_t S) {
  int64_t S4 = (S + 3) >> 2;
  return (((row >> 7) * S4 + (s >> 2)) << 9) + ((row & 31) << 4) + (((row & 127) >> 5) << 2) +
         (s & 3);
}

}  // namespace dq
