// dq_gemv.cu -- the W4A4 linear for a single token (decode), on the CUDA
// cores.
//
// "DualQuant", Section 4.4: the layer computes Q(X~) What^T Diag(alpha)^-1
// with the row-block scales as the weight's native block scales.  Same
// result contract as the tensor-core kernels of dq_gemm.cu:
//
//   Y[t, o] = s_tok[t] s_w r_row[o] sum_k a[t,k] sa[t,k/G] b[o,k] sb[o,k/G]
//
// With one token every weight byte is used once: the product is a stream of
// W through the SMs, bound by HBM, and a 128-row tensor-core tile would
// spend 127 of its rows on padding.  So:
//
// * Rows are taken in quad order: slot 4 d + x is row 128 (d / 32) + 32 x +
//   d % 32, so that the four rows of quad d (one per 32-row quarter of a
//   128-row group) share one 16-byte piece of every 512-byte scale atom, and
//   consecutive quads own consecutive pieces.  CTA c owns the slots
//   [c N / grid, (c+1) N / grid) and first copies its quads' pieces into
//   shared memory with coalesced 16-byte loads: every scale byte the CTA
//   needs, read once, instead of two bytes per lane scattered over sixteen
//   atoms for every 1024 elements of a row (that version ran at 28 % of HBM).
// * The CTA's units (one row x 1024 elements: 512 contiguous code bytes, 16
//   per lane) are split evenly over its 16 warps; each lane keeps 4 units of
//   16 bytes in flight (non-allocating loads).  The grid is the CTAs that
//   fit on the device at once (two per SM).
// * Exact block dot products in integers: the activations are staged once
//   per CTA in shared memory as int8 values 2a (E2M1 values times two are
//   the integers 0, +-1, +-2, +-3, +-4, +-6, +-8, +-12).  For a weight code
//   word, one byte permute over the table of doubled magnitudes gives |2b|
//   (sign bit masked off) and a second, with the sign bit left in the
//   selector, gives |2b| for positive codes and 0 for negative ones (the
//   permute's sign-replicate mode copies the table byte's zero sign bit).
//   Then sum 4ab = 2 dp4a(2a, pos) - dp4a(2a, |2b|) over a block, exactly,
//   and the block adds (sum) * (sa / 4) * sb to an fp32 accumulator (the
//   scale product is exact: UE4M3 x UE4M3 needs 8 significant bits, E8M0 is
//   a power of two).
// * When a warp moves to the next row it reduces its accumulator over the
//   lanes (a fixed butterfly) into a shared slot [row][warp]; at the end the
//   slots of each row are summed in warp order and the epilogue scales are
//   applied.  No atomics: the result is the same on every run.
// No waits other than CTA barriers; every access is bounded by the CTA's own
// slot range.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdlib.h>

#include <mutex>
#include <vector>

#include "dq_device.cuh"
#include "dq_internal.h"

namespace dq {
namespace gemv {

constexpr int WARPS = 16;
constexpr int THREADS = WARPS * 32;
// units in flight per lane: 4 with two CTAs per SM (one token), 8 with one
// CTA per SM (the larger register set of several tokens)
template <int MT> constexpr int U = MT == 1 ? 4 : 8;
template <int MT> constexpr int MIN_CTAS = MT == 1 ? 2 : 1;
constexpr int CHUNK_ELEMS = 1024;    // elements of one row per warp unit
// Doubled E2M1 magnitudes by magnitude index 0..7: 0, 1, 2, 3, 4, 6, 8, 12
// (bytes 0..3 in the first word, 4..7 in the second).
constexpr uint32_t MAG_LO = 0x03020100u, MAG_HI = 0x0C080604u;

__device__ __forceinline__ uint32_t mag_permute(uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(MAG_LO), "r"(MAG_HI), "r"(sel));
  return d;
}

// 16 bytes of weight codes, streamed (not kept in L1).
__device__ __forceinline__ uint4 ld_stream16(const uint8_t* p) {
  uint4 v;
  asm("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
      : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
      : "l"(p));
  return v;
}

// Value of an E8M0 byte, 2^(e - 127), exactly (e = 0 is the subnormal 2^-127).
__device__ __forceinline__ float e8m0_value(uint32_t e) {
  return e ? __uint_as_float(e << 23) : __uint_as_float(0x00400000u);
}

// Two UE4M3 bytes (low byte first) -> their values.
__device__ __forceinline__ float2 ue4m3x2_value(uint32_t two) {
  uint32_t h;
  asm("{\n\t.reg .b16 t;\n\tcvt.u16.u32 t, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, t;\n\t}"
      : "=r"(h)
      : "r"(two & 0xFFFFu));
  const __half2 hv = *reinterpret_cast<const __half2*>(&h);
  return __half22float2(hv);
}

// Row x (0..3) of quad d: 128 (d / 32) + 32 x + d % 32.
__device__ __forceinline__ int64_t quad_row(int64_t d, int x) {
  return ((d >> 5) << 7) + (x << 5) + (d & 31);
}

template <int FMT, int MT, int YT>
__global__ void __launch_bounds__(THREADS, MIN_CTAS<MT>)
w4a4_gemv_kernel(const uint8_t* __restrict__ A, const uint8_t* __restrict__ sA,
                 const float* __restrict__ s_tok, const uint8_t* __restrict__ B,
                 const uint8_t* __restrict__ sB, const float* __restrict__ s_w,
                 const float* __restrict__ r_row, void* __restrict__ Y, int M, int N, int K) {
  constexpr int G = FMT == NVFP4 ? 16 : 32;
  extern __shared__ __align__(16) unsigned char smem[];
  const int S = K / G, S4 = S >> 2, CPR = K / CHUNK_ELEMS;
  // row slots i = 4 d + x (row x of quad d); this CTA owns slots [i0, i1),
  // touching quads [q0, q0 + nq)
  const int64_t i0 = (int64_t)blockIdx.x * N / gridDim.x;
  const int rows = (int)((int64_t)(blockIdx.x + 1) * N / gridDim.x - i0);
  const int64_t q0 = i0 >> 2;
  const int nq = (int)(((i0 + rows - 1) >> 2) - q0 + 1);
  // [MT][K] activation values 2a (int8, chunk-permuted: a lane's 32 elements
  // are two 16-byte pieces 512 bytes apart); [MT][S] activation block scales
  // / 4; [nq][S4][16] the quads' scale pieces; [rows][WARPS][MT] row partials
  int8_t* a8 = reinterpret_cast<int8_t*>(smem);
  float* asc = reinterpret_cast<float*>(smem + (size_t)MT * K);
  uint8_t* scs = reinterpret_cast<uint8_t*>(asc + (size_t)MT * S);
  float* part = reinterpret_cast<float*>(scs + (size_t)nq * S4 * 16);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  // this warp's units: unit (slot, kc) = 1024 elements (512 contiguous code
  // bytes, 16 per lane) of one row
  const int64_t tot = (int64_t)rows * CPR;
  const int64_t s0 = tot * warp / WARPS, s1 = tot * (warp + 1) / WARPS;
  const int64_t K2 = K >> 1;
  auto code_ptr = [&](int rl) {   // rl: slot i0 + rl
    const int64_t i = i0 + rl;
    return B + (size_t)quad_row(i >> 2, (int)(i & 3)) * (size_t)K2 + lane * 16;
  };
  int rl = (int)(s0 / CPR), kc = (int)(s0 - (int64_t)rl * CPR);
  const uint8_t* bp = code_ptr(rl);
  // the weight is not written by the kernel this one may overlap with: start
  // its first bytes towards L2 before the dependency wait
  if (s0 < s1) asm volatile("prefetch.global.L2 [%0];" ::"l"(bp + (size_t)kc * 512));

  for (int i = tid; i < rows * WARPS * MT; i += THREADS) part[i] = 0.0f;
  // the quads' scale pieces: 16 bytes per (quad, atom) = the four quarters'
  // 4 scale bytes of row d % 32; consecutive quads are consecutive pieces
  for (int i = tid; i < nq * S4; i += THREADS) {
    const int ql = i % nq, at = i / nq;
    const int64_t d = q0 + ql;
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(
        sB + ((((d >> 5) * S4) + at) << 9) + ((d & 31) << 4)));
    *reinterpret_cast<uint4*>(scs + ((size_t)ql * S4 + at) * 16) = v;
  }

  pdl_wait();
  // ---- stage the activations (tokens >= M are zeros)
  const int W8 = K >> 3;   // code words (8 elements) per token
  for (int i = tid; i < MT * W8; i += THREADS) {
    const int t = i / W8, jw = i - t * W8;
    const uint32_t w =
        t < M ? __ldg(reinterpret_cast<const uint32_t*>(A + (size_t)t * (K >> 1)) + jw) : 0u;
    const uint32_t m = w & 0x77777777u;
    const uint32_t pl = mag_permute(w), ph = mag_permute(w >> 16);
    const uint32_t ml = mag_permute(m), mh = mag_permute(m >> 16);
    // per byte 2 pos - mag: +|2a| for positive codes, -|2a| for negative ones
    const uint32_t lo = __vsub4(pl + pl, ml), hi = __vsub4(ph + ph, mh);
    const int k = jw << 3;
    *reinterpret_cast<uint2*>(a8 + (size_t)t * K + ((k >> 10) << 10) + (((k >> 4) & 1) << 9) +
                              (((k >> 5) & 31) << 4) + (k & 8)) = make_uint2(lo, hi);
  }
  for (int i = tid; i < MT * S; i += THREADS) {
    const int t = i / S, sb = i - t * S;
    float v = 0.0f;
    if (t < M) {
      const uint32_t b = __ldg(sA + sf_offset(t, sb, S));
      v = __fmul_rn(FMT == NVFP4 ? ue4m3_value(b) : e8m0_value(b), 0.25f);
    }
    asc[i] = v;
  }
  __syncthreads();
  pdl_trigger();

  // this lane's scale byte(s) inside a piece: quarter x at 4 x; NVFP4 blocks
  // 64 kc + 2 lane (+1) (atom 16 kc + lane / 2), MX block 32 kc + lane (atom
  // 8 kc + lane / 4)
  const int sl = FMT == NVFP4 ? (((lane >> 1) << 4) + ((lane & 1) << 1))
                              : (((lane >> 2) << 4) + (lane & 3));
  constexpr int SC_STEP = FMT == NVFP4 ? 16 * 16 : 8 * 16;   // piece bytes per unit
  auto scale_ptr = [&](int rl) {
    const int64_t i = i0 + rl;
    return scs + (size_t)((i >> 2) - q0) * S4 * 16 + ((i & 3) << 2) + sl;
  };

  float acc[MT];
#pragma unroll
  for (int t = 0; t < MT; ++t) acc[t] = 0.0f;
  int cur = rl;
  const uint8_t* sp = scale_ptr(rl);

  auto flush = [&](int r) {
#pragma unroll
    for (int t = 0; t < MT; ++t) {
      float x = acc[t];
#pragma unroll
      for (int off = 16; off; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
      if (lane == 0) part[(r * WARPS + warp) * MT + t] = x;
      acc[t] = 0.0f;
    }
  };

  constexpr int UU = U<MT>;
  for (int64_t s = s0; s < s1; s += UU) {
    uint4 v[UU];
    uint32_t sb[UU];
    int rlc = rl, kcc = kc;   // position of unit s, advanced again below
#pragma unroll
    for (int u = 0; u < UU; ++u) {
      if (s + u < s1) {
        v[u] = ld_stream16(bp + (size_t)kc * 512);
        if constexpr (FMT == NVFP4)
          sb[u] = *reinterpret_cast<const unsigned short*>(sp + (size_t)kc * SC_STEP);
        else
          sb[u] = sp[(size_t)kc * SC_STEP];
      }
      if (++kc == CPR) {
        kc = 0;
        if (s + u + 1 < s1) {
          ++rl;
          bp = code_ptr(rl);
          sp = scale_ptr(rl);
        }
      }
    }
#pragma unroll
    for (int u = 0; u < UU; ++u) {
      if (s + u >= s1) break;
      if (rlc != cur) {
        flush(cur);
        cur = rlc;
      }
      const uint32_t wv[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
      uint32_t pos[8], mag[8];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint32_t m = wv[q] & 0x77777777u;
        pos[2 * q] = mag_permute(wv[q]);
        pos[2 * q + 1] = mag_permute(wv[q] >> 16);
        mag[2 * q] = mag_permute(m);
        mag[2 * q + 1] = mag_permute(m >> 16);
      }
      float bs0, bs1 = 0.0f;
      if constexpr (FMT == NVFP4) {
        const float2 b2 = ue4m3x2_value(sb[u]);
        bs0 = b2.x;
        bs1 = b2.y;
      } else {
        bs0 = e8m0_value(sb[u]);
      }
#pragma unroll
      for (int t = 0; t < MT; ++t) {
        const int8_t* ap = a8 + (size_t)t * K + kcc * CHUNK_ELEMS + lane * 16;
        const uint4 a0 = *reinterpret_cast<const uint4*>(ap);
        const uint4 a1 = *reinterpret_cast<const uint4*>(ap + 512);
        const uint32_t av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
        if constexpr (FMT == NVFP4) {
          const float2 as =
              *reinterpret_cast<const float2*>(asc + (size_t)t * S + kcc * 64 + 2 * lane);
          int p0 = 0, q0 = 0, p1 = 0, q1 = 0;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            p0 = __dp4a((int)av[q], (int)pos[q], p0);
            q0 = __dp4a((int)av[q], (int)mag[q], q0);
            p1 = __dp4a((int)av[4 + q], (int)pos[4 + q], p1);
            q1 = __dp4a((int)av[4 + q], (int)mag[4 + q], q1);
          }
          acc[t] = fmaf((float)(2 * p0 - q0), __fmul_rn(as.x, bs0), acc[t]);
          acc[t] = fmaf((float)(2 * p1 - q1), __fmul_rn(as.y, bs1), acc[t]);
        } else {
          const float as = asc[(size_t)t * S + kcc * 32 + lane];
          int pp = 0, qq = 0;
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            pp = __dp4a((int)av[q], (int)pos[q], pp);
            qq = __dp4a((int)av[q], (int)mag[q], qq);
          }
          acc[t] = fmaf((float)(2 * pp - qq), __fmul_rn(as, bs0), acc[t]);
        }
      }
      if (++kcc == CPR) {
        kcc = 0;
        ++rlc;
      }
    }
  }
  if (s0 < s1) flush(cur);
  __syncthreads();

  // ---- sum each row's warp partials (warp order); epilogue scales
  const float sw = (FMT == NVFP4 && s_w) ? __ldg(s_w) : 1.0f;
  for (int i = tid; i < M * rows; i += THREADS) {
    const int t = i / rows, r = i - t * rows;
    float sum = 0.0f;
#pragma unroll
    for (int w = 0; w < WARPS; ++w) sum += part[(r * WARPS + w) * MT + t];
    const int64_t slot = i0 + r;
    const int64_t n = quad_row(slot >> 2, (int)(slot & 3));
    float rs = sw;
    if (FMT == NVFP4) rs = __fmul_rn(__ldg(s_tok + t), sw);
    float y = __fmul_rn(sum, rs);
    if (r_row) y = __fmul_rn(y, __ldg(r_row + n));
    if constexpr (YT == 1)
      reinterpret_cast<__nv_bfloat16*>(Y)[(size_t)t * N + n] = __float2bfloat16_rn(y);
    else
      reinterpret_cast<float*>(Y)[(size_t)t * N + n] = y;
  }
}

static int num_sms() {
  static int n = 0;
  if (!n) {
    int dev = 0, v = 0;
    if (cudaGetDevice(&dev) == cudaSuccess &&
        cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess)
      n = v;
  }
  return n;
}

// CTAs of `kernel` with `smem` dynamic bytes that one SM holds (cached).
static int resident_ctas(const void* kernel, int smem) {
  struct Entry {
    const void* k;
    int dev, smem, occ;
  };
  static std::mutex mu;
  static std::vector<Entry> cache;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  {
    std::lock_guard<std::mutex> g(mu);
    for (const Entry& e : cache)
      if (e.k == kernel && e.dev == dev && e.smem == smem) return e.occ;
  }
  int occ = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kernel, THREADS, smem) != cudaSuccess) {
    cudaGetLastError();
    occ = 0;
  }
  std::lock_guard<std::mutex> g(mu);
  cache.push_back({kernel, dev, smem, occ});
  return occ;
}

template <int FMT, int YT>
static int launch(const uint8_t* A, const uint8_t* sA, const float* s_tok, const uint8_t* B,
                  const uint8_t* sB, const float* s_w, const float* r_row, void* Y, int64_t M,
                  int64_t N, int64_t K, cudaStream_t st) {
  constexpr int G = FMT == NVFP4 ? 16 : 32;
  constexpr int MT = 1;
  auto kern = w4a4_gemv_kernel<FMT, MT, YT>;
  const int sms = num_sms();
  if (sms <= 0) return DQ_ERR_CUDA;
  const size_t fixed = (size_t)MT * K + (size_t)MT * (K / G) * 4;
  // as many CTAs per SM as the registers allow (MIN_CTAS), fewer if the
  // shared memory does not
  for (int want = MIN_CTAS<MT>; want >= 1; --want) {
    const int64_t grid = (int64_t)want * sms < N ? (int64_t)want * sms : N;
    const int64_t rows_max = (N + grid - 1) / grid;
    const int64_t quads_max = rows_max / 4 + 2;
    const size_t smem = fixed + (size_t)quads_max * (K / G / 4) * 16 +
                        (size_t)rows_max * WARPS * MT * 4;
    if (smem > 227 * 1024) continue;
    if (!ensure_kernel_attrs((const void*)kern, (int)smem, false)) return DQ_ERR_CUDA;
    if (resident_ctas((const void*)kern, (int)smem) < want) continue;
    const cudaError_t e = launch_ex(kern, dim3((unsigned)grid), dim3(THREADS), smem, st, 1, A, sA,
                                    s_tok, B, sB, s_w, r_row, Y, (int)M, (int)N, (int)K);
    return e == cudaSuccess ? DQ_OK : DQ_ERR_CUDA;
  }
  return DQ_ERR_UNSUPPORTED;
}

static bool enabled() {
  static const bool on = [] {
    const char* e = getenv("DQ_GEMV");
    return !(e && e[0] == '0');
  }();
  return on;
}

}  // namespace gemv

int w4a4_gemv(const uint8_t* A, const uint8_t* sA, const float* s_tok, const uint8_t* B,
              const uint8_t* sB, const float* s_w, const float* r_row, void* Y, int yt, int64_t M,
              int64_t N, int64_t K, int f, cudaStream_t st) {
  if (!gemv::enabled() || M < 1 || M > GEMV_MAX_TOKENS || K % gemv::CHUNK_ELEMS ||
      (f != NVFP4 && f != MXFP4))
    return DQ_ERR_UNSUPPORTED;
  if (f == NVFP4)
    return yt == 1 ? gemv::launch<NVFP4, 1>(A, sA, s_tok, B, sB, s_w, r_row, Y, M, N, K, st)
                   : gemv::launch<NVFP4, 0>(A, sA, s_tok, B, sB, s_w, r_row, Y, M, N, K, st);
  return yt == 1 ? gemv::launch<MXFP4, 1>(A, sA, s_tok, B, sB, s_w, r_row, Y, M, N, K, st)
                 : gemv::launch<MXFP4, 0>(A, sA, s_tok, B, sB, s_w, r_row, Y, M, N, K, st);
}

}  // namespace dq
