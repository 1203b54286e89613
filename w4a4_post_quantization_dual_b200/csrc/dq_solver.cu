// dq_solver.cu -- DualQuant's block-coordinate-descent scale solver on sm_100a.
//
// "DualQuant: Dual-scale Calibration-free Weight-and-Activation Quantization
// for LLMs", Algorithm 1 / Section 4.3 (closed-form updates Eqs. 10 and 14,
// Appendix B), initialisation of Section 5.3.
//
// With the row scale alpha being the format's native block scale, every
// m x G column-block tile of W is an independent problem: r_ib touches only
// tile b and every column lies in one tile.  One thread-block CLUSTER owns
// one tile; its C CTAs split the tile's rows.  The whole iteration loop runs
// on the device:
//   row half-step   : each thread owns 8 contiguous columns of a row; the
//                     G/8 threads of a row-block combine <W,R> and ||R||^2
//                     with warp shuffles; the projected update is written to
//                     shared memory.
//   column half-step: per-thread column partials -> transposed shared-memory
//                     reduction in fp64 -> per-CTA sums in cluster-visible
//                     shared memory -> every CTA reads all C partial sums
//                     over DSMEM in rank order (identical c in every CTA).
// Each CTA stages its rows of the tile in shared memory once, converted to
// fp32 (clusters of up to 16 CTAs keep the share <= 96 KB), and reads them
// from there in every pass; tiles too tall for that stream their rows through the read-only
// global path (L1 / L2 hits after the first round).  HBM sees W about once.
#include <cuda_runtime.h>
#include <stdint.h>

#include <type_traits>
#include <vector>

#include "dq_device.cuh"
#include "dq_internal.h"

namespace dq {

template <int G>
struct SolverShape {
  static constexpr int OPB = G / 8;            // 8-column octets per row-block
  static constexpr int NT = (G >= 64) ? 512 : 256;
  static constexpr int NW = NT / 32;
  static constexpr int RPW = 32 / OPB;         // rows per warp per step
  static constexpr int RPS = NW * RPW;         // rows per CTA per step
};

// Workspace layout (bytes): [0] u32 amax bits, [8] f64 ||W||^2, [16..] f64
// err[T+1], then f64 qnum[T+1] and qden[T+1] (code-change trace sums).
struct SolverWs {
  uint32_t amax_bits;
  uint32_t pad;
  double w2;
  double err[1];
};

// Ablation mode and warm start (DualQuant, Table 4 scale ablation; the
// initialisation (alpha_0, beta_0) of Section 5.3 given by the caller).
// Flag values are those of dq_solve_flags in include/dq.h.
struct SolveOpts {
  unsigned flags;
  const float* r0;   // nullable, m x (n/G)
  const float* c0;   // nullable, n
};
constexpr unsigned SOLVE_ALPHA_ONLY = 1u, SOLVE_BETA_ONLY = 2u, SOLVE_KEEP_S = 4u,
                   SOLVE_TRACE_CODES = 8u;

// The weights of one launch (all with the same row count m): launch z-index
// i solves weight i.  Passed by value (kernel parameter space).
constexpr int SOLVE_BATCH_MAX = 16;
struct SolveItem {
  const void* W;      // m x n
  float* r;           // m x n/G
  float* c;           // n
  float* sT;          // 1
  SolverWs* ws;       // this weight's workspace
  int64_t n;
};
struct SolveBatch {
  SolveItem item[SOLVE_BATCH_MAX];
};

template <typename WT>
__device__ __forceinline__ void load8(const WT* __restrict__ W, int64_t off, float* x);
template <>
__device__ __forceinline__ void load8<__nv_bfloat16>(const __nv_bfloat16* __restrict__ W,
                                                     int64_t off, float* x) {
  uint4 v = __ldg(reinterpret_cast<const uint4*>(W + off));
  bf16x8_to_f32(v, x);
}
template <>
__device__ __forceinline__ void load8<float>(const float* __restrict__ W, int64_t off, float* x) {
  float4 a = __ldg(reinterpret_cast<const float4*>(W + off));
  float4 b = __ldg(reinterpret_cast<const float4*>(W + off) + 1);
  x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
  x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
}

__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;"
               ::: "memory");
}
// A double of CTA `rank`'s shared memory.  No memory clobber: the loads of
// all CTAs are issued back to back before they are summed; the cluster
// barrier before them orders them after the peers' writes.
__device__ __forceinline__ double ld_dsmem_f64(const double* local, uint32_t rank) {
  uint32_t a = (uint32_t)__cvta_generic_to_shared(local), ra;
  double v;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"(a), "r"(rank));
  asm volatile("ld.shared::cluster.f64 %0, [%1];" : "=d"(v) : "r"(ra));
  return v;
}

// Reduce V fp32 partials per thread over the CTA's threads that share an
// octet.  Thread (oct, rslot) contributes acc[v] to value gv = oct*V + v.
// out[gv] (shared, fp64) receives the CTA total, summed in a fixed order.
template <int G, int V>
__device__ __forceinline__ void cta_octet_reduce(const float* acc, float* scr, double* part,
                                                 double* out) {
  using S = SolverShape<G>;
  constexpr int NV = S::OPB * V;           // values per CTA
  constexpr int P = S::NT / NV;            // parts per value
  constexpr int SPP = S::RPS / P;          // slots per part
  static_assert(S::NT % NV == 0 && S::RPS % P == 0, "reduction shape");
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int oct = lane % S::OPB, rslot = warp * S::RPW + lane / S::OPB;
#pragma unroll
  for (int v = 0; v < V; ++v) scr[(oct * V + v) * (S::RPS + 1) + rslot] = acc[v];
  __syncthreads();
  {
    const int gv = tid % NV, p = tid / NV;
    double s = 0.0;
    const float* src = scr + gv * (S::RPS + 1) + p * SPP;
#pragma unroll 4
    for (int i = 0; i < SPP; ++i) s += (double)src[i];
    part[gv * P + p] = s;
  }
  __syncthreads();
  if (tid < NV) {
    double s = 0.0;
    for (int p = 0; p < P; ++p) s += part[tid * P + p];
    out[tid] = s;
  }
  __syncthreads();
}

// Same reduction for V fp64 partials per thread; scr (the float scratch of
// SolverSmem) is reused as OPB * V * (RPS + 1) doubles, V <= 8.
template <int G, int V>
__device__ __forceinline__ void cta_octet_reduce_f64(const double* acc, double* scr,
                                                     double* part, double* out) {
  using S = SolverShape<G>;
  constexpr int NV = S::OPB * V;
  constexpr int P = S::NT / NV;
  constexpr int SPP = S::RPS / P;
  static_assert(V <= 8 && S::NT % NV == 0 && S::RPS % P == 0, "reduction shape");
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int oct = lane % S::OPB, rslot = warp * S::RPW + lane / S::OPB;
#pragma unroll
  for (int v = 0; v < V; ++v) scr[(oct * V + v) * (S::RPS + 1) + rslot] = acc[v];
  __syncthreads();
  {
    const int gv = tid % NV, p = tid / NV;
    double s = 0.0;
    const double* src = scr + gv * (S::RPS + 1) + p * SPP;
    for (int i = 0; i < SPP; ++i) s += src[i];
    part[gv * P + p] = s;
  }
  __syncthreads();
  if (tid < NV) {
    double s = 0.0;
    for (int p = 0; p < P; ++p) s += part[tid * P + p];
    out[tid] = s;
  }
  __syncthreads();
}

// Closeness of an fp32 scale update to a rounding boundary of its
// projection.  The fast passes sum positive terms in fp32 (row: a tree of
// depth at most 9 per row-block; column: a chain of at most `steps` terms
// per thread, then fp64), so num and den are each within (depth) * 2^-24
// relative of their exact values and the quotient within 2 * depth + 4 fp32
// ulps.  An update whose distance to a boundary is inside that window is
// recomputed from exact fp64 sums, so that every projected scale is the one
// the exact quotient selects.  win = half-width of the window in ulps.
__device__ __forceinline__ bool near_half(uint32_t bits, int drop, uint32_t win) {
  const uint32_t mask = (1u << drop) - 1u, half = 1u << (drop - 1);
  return ((bits - half + win) & mask) <= 2u * win;   // |low bits - half| <= win
}
template <int F>
__device__ __forceinline__ bool near_tie_beta(float u, uint32_t win) {
  if constexpr (F == NVFP4) {
    // UE4M3: 3 mantissa bits above 2^-6; below it (subnormal steps of 2^-9,
    // a rare range) every update takes the exact path
    return u < 0.015625f || near_half(__float_as_uint(u), 20, win);
  } else if constexpr (is_mx(F)) {
    return near_half(__float_as_uint(u), 23, win);      // E8M0: midpoint 1.5 * 2^k
  } else {
    return near_half(__float_as_uint(u), 16, win);      // bf16
  }
}
template <int F>
__device__ __forceinline__ bool near_tie_alpha(float u, float inv_sT, uint32_t win) {
  if constexpr (F == NVFP4) return near_tie_beta<F>(u * inv_sT, win + 2);  // + fl(1/s_T)
  else return near_tie_beta<F>(u, win);
}
constexpr uint32_t ROW_TIE_WIN = 24;   // 2 * 9 + 4, rounded up

template <int G>
struct SolverSmem {
  using S = SolverShape<G>;
  float scr[S::OPB * 16 * (S::RPS + 1)];
  double part[S::NT];                       // NV * P == NT
  double cpart[2][2 * G];                   // cluster-visible, double-buffered
  float c_s[G], b_s[G];
  float b_old[G];                           // beta before the column update
  double l1[G];                             // init: column l1; main: exact-pass totals
};

// ---------------------------------------------------------------------------
// Initialisation kernel: c0 (Section 5.3, read as the inverse column scale
// proportional to the column l1 norm, normalised to mean 1 per tile and
// projected onto F_beta; or the projection of the caller's c0, or of 1 for
// alpha-only), the NVFP4 per-tensor amax of W diag(c0)^-1 (unless the
// caller's tensor scale is kept), and ||W||_F^2 for the trace.
// ---------------------------------------------------------------------------
template <int F, int G, typename WT>
__global__ void __launch_bounds__(SolverShape<G>::NT)
solve_init_kernel(SolveBatch bt, int64_t m, int steps, SolveOpts o) {
  using S = SolverShape<G>;
  const int64_t n = bt.item[blockIdx.z].n;
  if ((int64_t)blockIdx.y >= n / G) return;   // whole clusters (they span x only)
  const WT* __restrict__ W = reinterpret_cast<const WT*>(bt.item[blockIdx.z].W);
  float* c = bt.item[blockIdx.z].c;
  SolverWs* ws = bt.item[blockIdx.z].ws;
  extern __shared__ __align__(16) unsigned char smem_raw[];
  SolverSmem<G>& sm = *reinterpret_cast<SolverSmem<G>*>(smem_raw);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int oct = lane % S::OPB, rslot = warp * S::RPW + lane / S::OPB;
  const uint32_t rank = cluster_ctarank(), C = gridDim.x;
  const int64_t b = blockIdx.y;
  const int64_t col0 = b * G + oct * 8;
  const int64_t row0 = (int64_t)rank * steps * S::RPS;
  // the caller's c0 is read before the cluster barrier below, after which
  // rank 0 writes c (c0 may alias c)
  const bool given_c = o.c0 != nullptr || (o.flags & SOLVE_ALPHA_ONLY);
  const float c0v = (o.c0 != nullptr && tid < G) ? o.c0[b * G + tid] : 1.0f;

  // column l1 norms in fp64 (exact for bf16 weights: the same sums as a
  // sequential fp64 loop), so c0's projection decisions are the exact ones
  double acc[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) acc[k] = 0.0;
  float w2 = 0.0f;
  for (int s = 0; s < steps; ++s) {
    int64_t i = row0 + (int64_t)s * S::RPS + rslot;
    if (i < m) {
      float x[8];
      load8<WT>(W, i * n + col0, x);
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        acc[k] += (double)fabsf(x[k]);
        w2 = fmaf(x[k], x[k], w2);
      }
    }
  }
  // ||W||^2: warp sum then one fp64 atomic per warp
#pragma unroll
  for (int o = 16; o; o >>= 1) w2 += __shfl_xor_sync(0xffffffffu, w2, o);
  if (lane == 0) atomicAdd(&ws->w2, (double)w2);

  cta_octet_reduce_f64<G, 8>(acc, reinterpret_cast<double*>(sm.scr), sm.part,
                             sm.cpart[0]);  // cpart[0][j] = CTA l1 of col j
  cluster_sync_all();
  if (tid < G) {
    double s = 0.0;
    for (uint32_t q = 0; q < C; ++q) s += ld_dsmem_f64(&sm.cpart[0][tid], q);
    sm.l1[tid] = s;
  }
  __syncthreads();
  if (tid < G) {
    double mean = 0.0;
    for (int j = 0; j < G; ++j) mean += sm.l1[j];
    mean /= (double)G;
    double v = sm.l1[tid];
    float cj = given_c                  ? proj_beta<F>(c0v)
               : (mean > 0.0 && v > 0.0) ? proj_beta<F>((float)(v / mean))
                                         : proj_beta<F>(1.0f);
    sm.c_s[tid] = cj;
    sm.b_s[tid] = __frcp_rn(cj);
    if (rank == 0) c[b * G + tid] = cj;
  }
  __syncthreads();
  if (F == NVFP4 && !(o.flags & SOLVE_KEEP_S)) {
    float beta[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) beta[k] = sm.b_s[oct * 8 + k];
    float a = 0.0f;
    for (int s = 0; s < steps; ++s) {
      int64_t i = row0 + (int64_t)s * S::RPS + rslot;
      if (i < m) {
        float x[8];
        load8<WT>(W, i * n + col0, x);
#pragma unroll
        for (int k = 0; k < 8; ++k) a = fmaxf(a, fabsf(__fmul_rn(x[k], beta[k])));
      }
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
    if (lane == 0) atomicMax(&ws->amax_bits, __float_as_uint(a));
  }
  cluster_sync_all();  // keep this CTA's shared memory alive for DSMEM readers
}

// ---------------------------------------------------------------------------
// Main kernel: r0 and T rounds of Algorithm 1, final error, outputs.
//
// WSMEM: the CTA's rows of the tile are staged once in shared memory and
// every pass reads them from there; otherwise they are re-read through the
// read-only global path (L1 / L2).  Element arithmetic uses the packed
// fp32x2 instructions of sm_100 (each lane of a pair is an ordinary
// correctly-rounded fp32 operation, so the quantiser argument
// (w * beta) * alpha is bit-identical to the scalar definition).
// TRACE: accumulate the reconstruction error for the MSE trace.
// ---------------------------------------------------------------------------
template <int F>
struct RowProj {
  // projected row scale r in F_alpha and alpha = fl(1/r) for an update u
  __device__ __forceinline__ static void apply(float u, float inv_sT, const float* rtab,
                                               const float* atab, float sT, float& r, float& a) {
    if constexpr (F == NVFP4) {
      uint32_t b = ue4m3_rn(u * inv_sT);
      b = b ? b : 1u;
      r = rtab[b];
      a = atab[b];
    } else if constexpr (is_mx(F)) {
      uint32_t bits = __float_as_uint(u);
      int e = (int)((bits >> 23) & 0xFFu);
      int k = e ? e - 127 + ((bits & 0x7FFFFFu) >= 0x400000u ? 1 : 0)
                : ((u >= 8.816207631167156e-39f) ? -126 : -127);
      k = k < -127 ? -127 : (k > 127 ? 127 : k);
      r = pow2f(k);
      a = pow2f(-k);
    } else {
      r = proj_bf16(u);
      a = __frcp_rn(r);
    }
  }
};

// Grid values of one pair of quantiser arguments: nearest grid point (ties
// to even), saturating.  E2M1 / E4M3 pairs go through the hardware
// conversion to their code bytes and straight back to an exact f16x2.
template <int F>
__device__ __forceinline__ float2 grid2_packed(float2 z) {
  if constexpr (is_int_grid(F)) {
    return make_float2(rintf(fminf(fmaxf(z.x, -8.0f), 7.0f)), rintf(fminf(fmaxf(z.y, -8.0f), 7.0f)));
  } else if constexpr (is_int8_grid(F)) {
    return make_float2(rintf(fminf(fmaxf(z.x, -128.0f), 127.0f)),
                       rintf(fminf(fmaxf(z.y, -128.0f), 127.0f)));
  } else if constexpr (F == MXFP8) {
    uint32_t h;
    asm("{\n\t.reg .b16 t;\n\t"
        "cvt.rn.satfinite.e4m3x2.f32 t, %2, %1;\n\t"
        "cvt.rn.f16x2.e4m3x2 %0, t;\n\t}"
        : "=r"(h) : "f"(z.x), "f"(z.y));
    return __half22float2(*reinterpret_cast<__half2*>(&h));
  } else {
    uint32_t h;
    asm("{\n\t.reg .b8 t;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 t, %2, %1;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, t;\n\t}"
        : "=r"(h) : "f"(z.x), "f"(z.y));
    return __half22float2(*reinterpret_cast<__half2*>(&h));
  }
}

template <int F>
__device__ __forceinline__ void grid8_packed(const float2* z, float2* q) {
#pragma unroll
  for (int k = 0; k < 4; ++k) q[k] = grid2_packed<F>(z[k]);
}

template <typename WT>
__device__ __forceinline__ void unpack8(const WT* p, float2* x);
template <>
__device__ __forceinline__ void unpack8<__nv_bfloat16>(const __nv_bfloat16* p, float2* x) {
  uint4 v = *reinterpret_cast<const uint4*>(p);
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) x[i] = make_float2(__uint_as_float(w[i] << 16), __uint_as_float(w[i] & 0xFFFF0000u));
}
template <>
__device__ __forceinline__ void unpack8<float>(const float* p, float2* x) {
  float4 a = reinterpret_cast<const float4*>(p)[0];
  float4 b = reinterpret_cast<const float4*>(p)[1];
  x[0] = make_float2(a.x, a.y); x[1] = make_float2(a.z, a.w);
  x[2] = make_float2(b.x, b.y); x[3] = make_float2(b.z, b.w);
}
template <typename WT>
__device__ __forceinline__ void unpack8_global(const WT* __restrict__ p, float2* x) {
  if constexpr (sizeof(WT) == 2) {
    uint4 v = __ldg(reinterpret_cast<const uint4*>(p));
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) x[i] = make_float2(__uint_as_float(w[i] << 16), __uint_as_float(w[i] & 0xFFFF0000u));
  } else {
    float4 a = __ldg(reinterpret_cast<const float4*>(p));
    float4 b = __ldg(reinterpret_cast<const float4*>(p) + 1);
    x[0] = make_float2(a.x, a.y); x[1] = make_float2(a.z, a.w);
    x[2] = make_float2(b.x, b.y); x[3] = make_float2(b.z, b.w);
  }
}

// Columns 2k, 2k+1 of an 8-column piece, as fp32.
template <typename T>
__device__ __forceinline__ float2 load_pair(const T* p, int k) {
  if constexpr (sizeof(T) == 2) {
    const uint32_t w = *reinterpret_cast<const uint32_t*>(p + 2 * k);
    return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
  } else {
    return *reinterpret_cast<const float2*>(p + 2 * k);
  }
}

// STG: 0 rows stream through the read-only global path, 1 rows staged in
// shared memory as WT, 2 rows staged as fp32 (no unpacking in the passes).
template <int F, int G, typename WT, int STG, bool TRACE>
__global__ void __launch_bounds__(SolverShape<G>::NT, 2048 / SolverShape<G>::NT / 2)
solve_bcd_kernel(SolveBatch bt, int64_t m, int steps, int T, SolveOpts o) {
  using S = SolverShape<G>;
  const int64_t n = bt.item[blockIdx.z].n;
  if ((int64_t)blockIdx.y >= n / G) return;   // whole clusters (they span x only)
  const WT* __restrict__ W = reinterpret_cast<const WT*>(bt.item[blockIdx.z].W);
  float* r_out = bt.item[blockIdx.z].r;
  float* __restrict__ c_io = bt.item[blockIdx.z].c;
  float* sT_io = bt.item[blockIdx.z].sT;
  SolverWs* ws = bt.item[blockIdx.z].ws;
  extern __shared__ __align__(16) unsigned char smem_raw[];
  SolverSmem<G>& sm = *reinterpret_cast<SolverSmem<G>*>(smem_raw);
  float* r_s = reinterpret_cast<float*>(smem_raw + sizeof(SolverSmem<G>));
  float* a_s = r_s + (size_t)steps * S::RPS;
  float* rtab = a_s + (size_t)steps * S::RPS;       // NVFP4: r and alpha of every scale byte
  float* atab = rtab + 128;
  constexpr bool WSMEM = STG != 0;
  using ST = typename std::conditional<STG == 2, float, WT>::type;  // staged element type
  ST* wch = reinterpret_cast<ST*>(atab + 128);      // staged rows
  // TRACE: alpha of the previous round per row-step (code-change trace)
  float* ap_s = reinterpret_cast<float*>(wch + (WSMEM ? (size_t)steps * S::RPS * G : 0));

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int oct = lane % S::OPB, rslot = warp * S::RPW + lane / S::OPB;
  const uint32_t rank = cluster_ctarank(), C = gridDim.x;
  const int64_t b = blockIdx.y, nb = n / G;
  const int64_t col0 = b * G + oct * 8;
  const int64_t row0 = (int64_t)rank * steps * S::RPS;
  const int rows_cta = steps * S::RPS;

  const bool alpha_only = o.flags & SOLVE_ALPHA_ONLY, beta_only = o.flags & SOLVE_BETA_ONLY;
  const bool keep_s = F == NVFP4 && (o.flags & SOLVE_KEEP_S);
  float sT = 1.0f;
  if constexpr (F == NVFP4) {
    if (keep_s) {
      sT = *sT_io;
    } else {
      float amax = __uint_as_float(*(volatile uint32_t*)&ws->amax_bits);
      sT = (amax > 0.0f) ? __fdiv_rn(amax, 2688.0f) : 1.0f;
    }
    if (tid < 128) {
      float rv = __fmul_rn(sT, ue4m3_value(tid ? (uint32_t)tid : 1u));
      rtab[tid] = rv;
      atab[tid] = __frcp_rn(rv);
    }
  }
  if (rank == 0 && b == 0 && tid == 0 && !keep_s) *sT_io = sT;
  const float inv_sT = __frcp_rn(sT);

  if constexpr (STG == 2) {
    // stage rows [row0, row0 + rows_cta) x columns [b*G, b*G+G) (zeros past
    // m) as fp32, so the passes below read values without unpacking
    constexpr int PPR = G / 8;                        // 8-element pieces per row
    for (int p = tid; p < rows_cta * PPR; p += S::NT) {
      const int lr = p / PPR, pc = p % PPR;
      const int64_t i = row0 + lr;
      float2 v[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                     make_float2(0.f, 0.f)};
      if (i < m) unpack8_global<WT>(W + i * n + b * G + pc * 8, v);
      float4* dst = reinterpret_cast<float4*>(wch + (size_t)lr * G + pc * 8);
      dst[0] = make_float4(v[0].x, v[0].y, v[1].x, v[1].y);
      dst[1] = make_float4(v[2].x, v[2].y, v[3].x, v[3].y);
    }
    __syncthreads();
  } else if constexpr (STG == 1) {
    // stage the rows in their own type (16-byte pieces, zeros past m)
    constexpr int V = 16 / sizeof(WT);
    constexpr int PPR = G / V;
    for (int p = tid; p < rows_cta * PPR; p += S::NT) {
      const int lr = p / PPR, pc = p % PPR;
      const int64_t i = row0 + lr;
      uint4 v = make_uint4(0, 0, 0, 0);
      if (i < m) v = __ldg(reinterpret_cast<const uint4*>(W + i * n + b * G) + pc);
      reinterpret_cast<uint4*>(wch + (size_t)lr * G)[pc] = v;
    }
    __syncthreads();
  }
  // this thread's row-steps s cover rows row0 + s*RPS + rslot; those below m
  // are s < s_end.  Per-thread bases and constant strides for the hot loops.
  const int64_t first_row = row0 + rslot;
  const int s_end = first_row >= m ? 0
                    : (int)((m - first_row + S::RPS - 1) / S::RPS) < steps
                          ? (int)((m - first_row + S::RPS - 1) / S::RPS)
                          : steps;
  const ST* xsm = WSMEM ? wch + (size_t)rslot * G + oct * 8 : nullptr;
  const WT* xgl = WSMEM ? nullptr : W + first_row * n + col0;
  constexpr int XSM_STEP = S::RPS * G;
  const int64_t xgl_step = (int64_t)S::RPS * n;
  float* rsl = r_s + rslot;
  float* asl = a_s + rslot;
  float* apl = ap_s + rslot;
  const bool trace_codes = TRACE && (o.flags & SOLVE_TRACE_CODES);
  float2 beta_prev[4];   // TRACE: beta of the previous round
  auto load_x = [&](int s, float2* x) {
    if constexpr (WSMEM) unpack8<ST>(xsm + s * XSM_STEP, x);
    else unpack8_global<WT>(xgl + s * xgl_step, x);
  };

  float2 cc[4], beta[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    cc[k] = make_float2(c_io[col0 + 2 * k], c_io[col0 + 2 * k + 1]);
    beta[k] = make_float2(__frcp_rn(cc[k].x), __frcp_rn(cc[k].y));
  }
  if (tid < G) {   // the current beta also in shared memory (exact column pass)
    sm.c_s[tid] = c_io[b * G + tid];
    sm.b_s[tid] = __frcp_rn(sm.c_s[tid]);
  }

  // r0: the caller's scales projected onto F_alpha (rows past m take the
  // projection of 1), or else the format-native absmax scale of
  // W diag(c0)^-1 per row-block (IEEE arithmetic: the same fp32 decisions
  // as the oracle's initialisation).  Each r0 entry is read by the thread
  // that writes the same entry of r at the end (r0 may alias r).
  if (o.r0 != nullptr) {
    if (oct == 0)
      for (int s = 0; s < steps; ++s) {
        const float u = s < s_end ? o.r0[(first_row + (int64_t)s * S::RPS) * nb + b] : 1.0f;
        const float rv = proj_alpha<F>(u, sT);
        rsl[s * S::RPS] = rv;
        asl[s * S::RPS] = __frcp_rn(rv);
      }
  } else
  for (int s = 0; s < steps; ++s) {
    float a = 0.0f;
    if (s < s_end) {
      float2 x[4];
      load_x(s, x);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        float2 p = __fmul2_rn(x[k], beta[k]);
        a = fmaxf(a, fmaxf(fabsf(p.x), fabsf(p.y)));
      }
    }
#pragma unroll
    for (int o = 1; o < S::OPB; o <<= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
    if (oct == 0) {
      float r0 = rtn_block_scale<F>(a, sT);
      rsl[s * S::RPS] = r0;
      asl[s * S::RPS] = __frcp_rn(r0);
    }
  }
  __syncwarp();

  int xb = 0;  // exchange buffer of the next column exchange
  // column window: 2 * steps + 4 ulps, + 4 for S = r q rounded to fp32
  const uint32_t col_win = 2u * (uint32_t)steps + 8u;
  for (int t = 0; t <= T; ++t) {
    // ---- row half-step (t < T) / error at the current scales ----
    float e_acc = 0.0f;
    float2 qn2 = make_float2(0.f, 0.f), qd2 = qn2;   // TRACE: code-change sums
    bool any_tie = false;
    if ((t < T && !beta_only) || TRACE) {
      for (int s = 0; s < steps; ++s) {
        const bool valid = s < s_end;
        float2 num2 = make_float2(0.f, 0.f), den2 = num2, err2 = num2;
        const float rr = rsl[s * S::RPS], alpha = asl[s * S::RPS];
        const float alpha_prev = (TRACE && t > 0) ? apl[s * S::RPS] : 0.0f;
        if (valid) {
          float2 x[4], z[4], q[4];
          load_x(s, x);
          const float2 a2 = make_float2(alpha, alpha);
#pragma unroll
          for (int k = 0; k < 4; ++k) z[k] = __fmul2_rn(__fmul2_rn(x[k], beta[k]), a2);
          grid8_packed<F>(z, q);
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            float2 R = __fmul2_rn(q[k], cc[k]);
            num2 = __ffma2_rn(x[k], R, num2);
            den2 = __ffma2_rn(R, R, den2);
            if constexpr (TRACE) {
              float2 d = __ffma2_rn(make_float2(-rr, -rr), R, x[k]);
              err2 = __ffma2_rn(d, d, err2);
            }
          }
          if constexpr (TRACE) {
            // Qhat(t) - Qhat(t-1): the codes at the previous round's scales
            if (trace_codes && t > 0) {
              const float2 ap2 = make_float2(alpha_prev, alpha_prev);
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                const float2 qp = grid2_packed<F>(__fmul2_rn(__fmul2_rn(x[k], beta_prev[k]), ap2));
                const float2 d = make_float2(q[k].x - qp.x, q[k].y - qp.y);
                qn2 = __ffma2_rn(d, d, qn2);
                qd2 = __ffma2_rn(qp, qp, qd2);
              }
            }
          }
        }
        float num = num2.x + num2.y, den = den2.x + den2.y, err = err2.x + err2.y;
#pragma unroll
        for (int o = 1; o < S::OPB; o <<= 1) {
          num += __shfl_xor_sync(0xffffffffu, num, o);
          den += __shfl_xor_sync(0xffffffffu, den, o);
          if constexpr (TRACE) err += __shfl_xor_sync(0xffffffffu, err, o);
        }
        if (TRACE && oct == 0) e_acc += err;
        // the alpha these codes were taken with serves the next round's trace
        if (TRACE && trace_codes && oct == 0) apl[s * S::RPS] = alpha;
        if (t < T && !beta_only) {
          const float u = den > 0.0f ? __fdividef(num, den) : 1.0f;
          // all lanes of a row-block hold the same sums, hence the same flag
          const bool tie = den > 0.0f && near_tie_alpha<F>(u, inv_sT, ROW_TIE_WIN);  // den = 0 past m
          any_tie |= tie;
          if (oct == 0 && valid) {
            float rn, an;
            RowProj<F>::apply(u, inv_sT, rtab, atab, sT, rn, an);
            // exact update pending: r holds -alpha (the alpha it needs)
            rsl[s * S::RPS] = tie ? -alpha : rn;
            asl[s * S::RPS] = an;
          }
        }
      }
      // rare: row-blocks whose update lies near a projection boundary get it
      // from exact sums -- <W_i, R_i> and ||R_i||^2 in fp64 (x * R is exact
      // in fp64, R = q * c exact in fp32), the quotient rounded once to fp32
      if (t < T && !beta_only && __any_sync(0xffffffffu, any_tie)) {
        __syncwarp();
        for (int s = 0; s < steps; ++s) {
          const bool need = rsl[s * S::RPS] < 0.0f;   // the same word for the whole row-block
          if (!__any_sync(0xffffffffu, need)) continue;
          double dn = 0.0, dd = 0.0;
          if (need) {   // one column pair at a time (few live registers)
            const float alpha = -rsl[s * S::RPS];
            const float2 a2 = make_float2(alpha, alpha);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              float2 xp;
              if constexpr (WSMEM) xp = load_pair<ST>(xsm + s * XSM_STEP, k);
              else xp = load_pair<WT>(xgl + s * xgl_step, k);
              const float2 q = grid2_packed<F>(__fmul2_rn(__fmul2_rn(xp, beta[k]), a2));
              const float2 R = __fmul2_rn(q, cc[k]);
              dn = fma((double)xp.x, (double)R.x, dn);
              dn = fma((double)xp.y, (double)R.y, dn);
              dd = fma((double)R.x, (double)R.x, dd);
              dd = fma((double)R.y, (double)R.y, dd);
            }
          }
#pragma unroll
          for (int o = 1; o < S::OPB; o <<= 1) {
            dn += __shfl_xor_sync(0xffffffffu, dn, o);
            dd += __shfl_xor_sync(0xffffffffu, dd, o);
          }
          __syncwarp();
          if (need && oct == 0) {
            const float rn = proj_alpha<F>((float)(dn / dd), sT);
            rsl[s * S::RPS] = rn;
            asl[s * S::RPS] = __frcp_rn(rn);
          }
        }
      }
    }
    if constexpr (TRACE) {
#pragma unroll
      for (int o = 16; o; o >>= 1) e_acc += __shfl_xor_sync(0xffffffffu, e_acc, o);
      if (lane == 0) atomicAdd(&ws->err[t], (double)e_acc);
      if (trace_codes) {
        // sums of this warp; qnum / qden follow err[T+1] in the workspace
        float qn = qn2.x + qn2.y, qd = qd2.x + qd2.y;
#pragma unroll
        for (int o = 16; o; o >>= 1) {
          qn += __shfl_xor_sync(0xffffffffu, qn, o);
          qd += __shfl_xor_sync(0xffffffffu, qd, o);
        }
        if (lane == 0 && t > 0) {
          atomicAdd(&ws->err[(T + 1) + t], (double)qn);
          atomicAdd(&ws->err[2 * (T + 1) + t], (double)qd);
        }
#pragma unroll
        for (int k = 0; k < 4; ++k) beta_prev[k] = beta[k];
      }
    }
    if (t == T) break;
    __syncwarp();
    if (alpha_only) continue;

    // ---- column half-step: re-quantise with the new r, update c ----
    float2 acc[8];
#pragma unroll
    for (int v = 0; v < 8; ++v) acc[v] = make_float2(0.f, 0.f);
    for (int s = 0; s < s_end; ++s) {
      {
        const float rr = rsl[s * S::RPS], alpha = asl[s * S::RPS];
        float2 x[4], z[4], q[4];
        load_x(s, x);
        const float2 a2 = make_float2(alpha, alpha), r2 = make_float2(rr, rr);
#pragma unroll
        for (int k = 0; k < 4; ++k) z[k] = __fmul2_rn(__fmul2_rn(x[k], beta[k]), a2);
        grid8_packed<F>(z, q);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          float2 Sv = __fmul2_rn(r2, q[k]);
          acc[2 * k] = __ffma2_rn(Sv, x[k], acc[2 * k]);        // (num_j, num_j+1)
          acc[2 * k + 1] = __ffma2_rn(Sv, Sv, acc[2 * k + 1]);  // (den_j, den_j+1)
        }
      }
    }
    // reorder to [column][num, den] for the reduction
    float accv[16];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      accv[4 * k + 0] = acc[2 * k].x;       // num of column 2k
      accv[4 * k + 1] = acc[2 * k + 1].x;   // den of column 2k
      accv[4 * k + 2] = acc[2 * k].y;       // num of column 2k+1
      accv[4 * k + 3] = acc[2 * k + 1].y;   // den of column 2k+1
    }
    // the exchange buffer alternates with every exchange: a CTA writes
    // buffer xb only after all peers passed the barrier that follows their
    // last reads of it
    cta_octet_reduce<G, 16>(accv, sm.scr, sm.part, sm.cpart[xb]);
    cluster_sync_all();
    // column j's total (num, den) over the cluster, summed in rank order;
    // four CTAs' partials in flight at a time
    auto cluster_sum = [&](int j, double& sn, double& sd) {
      const int o = j >> 3, k = j & 7;
      sn = 0.0;
      sd = 0.0;
      for (int q0 = 0; q0 < (int)C; q0 += 4) {
        double pn[4], pd[4];
#pragma unroll
        for (int u = 0; u < 4; ++u)
          if (q0 + u < (int)C) {
            pn[u] = ld_dsmem_f64(&sm.cpart[xb][o * 16 + 2 * k], (uint32_t)(q0 + u));
            pd[u] = ld_dsmem_f64(&sm.cpart[xb][o * 16 + 2 * k + 1], (uint32_t)(q0 + u));
          }
#pragma unroll
        for (int u = 0; u < 4; ++u)
          if (q0 + u < (int)C) {
            sn += pn[u];
            sd += pd[u];
          }
      }
    };
    // projected update, written at once; a column near a projection
    // boundary is redone below from exact sums
    bool ctie = false;
    if (tid < G) {
      double sn, sd;
      cluster_sum(tid, sn, sd);
      const float cu = (sd > 0.0) ? (float)(sn / sd) : 1.0f;
      ctie = sd > 0.0 && near_tie_beta<F>(cu, col_win);
      const float cn = proj_beta<F>(cu);
      sm.b_old[tid] = sm.b_s[tid];
      sm.c_s[tid] = cn;
      sm.b_s[tid] = __frcp_rn(cn);
    }
    xb ^= 1;
    // every CTA of the cluster sums the same partials in the same order, so
    // the flag is cluster-uniform and the exact pass below (with its cluster
    // barrier) runs in all of them or in none
    if (__syncthreads_or(ctie)) {
      // rare: exact fp64 column sums of the tile
      // -- per thread <S_j, W_j> and ||S_j||^2 for one column pair of its
      // octet at a time, S = r q formed in fp64 (exact) and S * S rounded
      // once as in a plain fp64 loop, reduced over the CTA in fp64 into the
      // exchange layout of the fast pass (the old beta from shared memory,
      // the pair loaded on its own: no register array is indexed by kp)
#pragma unroll 1
      for (int kp = 0; kp < 4; ++kp) {
        double a4[4] = {0.0, 0.0, 0.0, 0.0};
        const float2 bp = make_float2(sm.b_old[oct * 8 + 2 * kp], sm.b_old[oct * 8 + 2 * kp + 1]);
        for (int s = 0; s < s_end; ++s) {
          const float rr = rsl[s * S::RPS], alpha = asl[s * S::RPS];
          float2 xp;
          if constexpr (WSMEM) xp = load_pair<ST>(xsm + s * XSM_STEP, kp);
          else xp = load_pair<WT>(xgl + s * xgl_step, kp);
          const float2 q = grid2_packed<F>(__fmul2_rn(__fmul2_rn(xp, bp), make_float2(alpha, alpha)));
          const double s0 = (double)rr * (double)q.x, s1 = (double)rr * (double)q.y;
          a4[0] = __dadd_rn(a4[0], __dmul_rn(s0, (double)xp.x));
          a4[1] = __dadd_rn(a4[1], __dmul_rn(s0, s0));
          a4[2] = __dadd_rn(a4[2], __dmul_rn(s1, (double)xp.y));
          a4[3] = __dadd_rn(a4[3], __dmul_rn(s1, s1));
        }
        cta_octet_reduce_f64<G, 4>(a4, reinterpret_cast<double*>(sm.scr), sm.part, sm.l1);
        if (tid < S::OPB * 4) sm.cpart[xb][(tid >> 2) * 16 + 4 * kp + (tid & 3)] = sm.l1[tid];
        __syncthreads();
      }
      cluster_sync_all();
      if (ctie) {   // rank order, one CTA at a time (rare path)
        const int o = tid >> 3, k = tid & 7;
        double sn = 0.0, sd = 0.0;
        for (uint32_t q = 0; q < C; ++q) {
          sn += ld_dsmem_f64(&sm.cpart[xb][o * 16 + 2 * k], q);
          sd += ld_dsmem_f64(&sm.cpart[xb][o * 16 + 2 * k + 1], q);
        }
        const float cn = proj_beta<F>((float)(sn / sd));
        sm.c_s[tid] = cn;
        sm.b_s[tid] = __frcp_rn(cn);
      }
      xb ^= 1;
      __syncthreads();
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      cc[k] = make_float2(sm.c_s[oct * 8 + 2 * k], sm.c_s[oct * 8 + 2 * k + 1]);
      beta[k] = make_float2(sm.b_s[oct * 8 + 2 * k], sm.b_s[oct * 8 + 2 * k + 1]);
    }
  }

  // outputs
  for (int s = 0; s < s_end; ++s)
    if (oct == 0) r_out[(first_row + (int64_t)s * S::RPS) * nb + b] = rsl[s * S::RPS];
  if (rank == 0 && tid < G && T > 0 && !alpha_only) c_io[b * G + tid] = sm.c_s[tid];
  cluster_sync_all();  // no CTA leaves while a peer may still read its cpart
}

// mse_trace[t] = err[t] / ||W||^2; with the code-change trace also
// mse_trace[T + 1 + t] = sqrt(qnum[t] / qden[t]) for t >= 1 (NaN at t = 0).
__global__ void solve_finalize_kernel(const SolverWs* ws, int T, double* mse_trace, int codes) {
  int t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t <= T) {
    mse_trace[t] = ws->w2 > 0.0 ? ws->err[t] / ws->w2 : 0.0;
    if (codes) {
      const double qn = ws->err[(T + 1) + t], qd = ws->err[2 * (T + 1) + t];
      mse_trace[(T + 1) + t] = t == 0 ? __longlong_as_double(0x7FF8000000000000ll)
                                      : (qd > 0.0 ? sqrt(qn / qd) : 0.0);
    }
  }
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------
// trace: one more float per row-step (the previous round's alpha, for the
// code-change trace), after the staged rows.
template <int G>
static size_t solver_smem_bytes(int steps, size_t staged_elem_bytes, bool trace = false) {
  const size_t rows = (size_t)steps * SolverShape<G>::RPS;
  return sizeof(SolverSmem<G>) + 2 * sizeof(float) * rows + 2 * 128 * sizeof(float) +
         rows * G * staged_elem_bytes + (trace ? sizeof(float) * rows : 0);
}

// Launch geometry: the tile's rows are split over C CTAs of one cluster,
// `steps` row-steps of RPS rows per CTA.  Prefer clusters of 8, staging the
// CTA's rows in shared memory as fp32, else in the weight's own type
// (<= 96 KB of rows); otherwise, for G = 16 only, clusters of 16 with the
// same staging; otherwise stream the rows through the read-only global
// path with clusters of 8.  stg: 2 fp32, 1 own type, 0 global.
// Measured (B200, T = 50, bf16): 14336 x 4096 NVFP4 6.1 ms with fp32 rows
// in 16 CTAs, 4.1 ms with bf16 rows in 8; 14336 x 4096 MXFP4 5.0 ms staged
// in 16 CTAs, 4.0 ms streamed by 8; 27648 x 5120 NVFP4 12.0 ms staged in 16,
// 13.2 ms streamed by 8.  Larger staging at one CTA per SM was slower in
// every case.
template <int G, typename WT>
static void solver_geometry(int64_t m, int& steps, int& C, int& stg) {
  using S = SolverShape<G>;
  for (int cmax : {8, 16}) {
    if (cmax == 16 && G != 16) break;
    for (int s_try : {2, 1}) {
      const size_t row_bytes = (size_t)G * (s_try == 2 ? sizeof(float) : sizeof(WT));
      int st = (int)((m + (int64_t)S::RPS * cmax - 1) / ((int64_t)S::RPS * cmax));
      if (st < 1) st = 1;
      if ((size_t)st * S::RPS * row_bytes <= 96 * 1024) {
        steps = st;
        C = (int)((m + (int64_t)S::RPS * st - 1) / ((int64_t)S::RPS * st));
        stg = s_try;
        return;
      }
    }
  }
  steps = (int)((m + (int64_t)S::RPS * 8 - 1) / ((int64_t)S::RPS * 8));
  C = (int)((m + (int64_t)S::RPS * steps - 1) / ((int64_t)S::RPS * steps));
  stg = 0;
}

template <typename K>
static bool allow_big_cluster(K kern, size_t smem) {
  return ensure_kernel_attrs((const void*)kern, (int)smem, true);
}

// One launch pair (initialisation + BCD) for `count` weights of row count m;
// traces[i] may be null.
template <int F, int G, typename WT>
static int launch_solver(const SolveBatch& bt, int count, int64_t m, int T, const SolveOpts& o,
                         double* const* traces, cudaStream_t st) {
  using S = SolverShape<G>;
  int steps, C, stg;
  solver_geometry<G, WT>(m, steps, C, stg);
  int64_t tiles = 0;
  bool any_trace = false;
  for (int i = 0; i < count; ++i) {
    tiles = bt.item[i].n / G > tiles ? bt.item[i].n / G : tiles;
    any_trace = any_trace || (traces && traces[i]);
  }
  const size_t sm_init = sizeof(SolverSmem<G>),
               sm_main = solver_smem_bytes<G>(
                   steps, stg == 2 ? sizeof(float) : (stg == 1 ? sizeof(WT) : 0), any_trace);
  if (sm_main > 227 * 1024) return DQ_ERR_UNSUPPORTED;
  if (tiles > 65535) return DQ_ERR_UNSUPPORTED;

  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(C, (unsigned)tiles, (unsigned)count);
  cfg.blockDim = dim3(S::NT, 1, 1);
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;

  auto kinit = solve_init_kernel<F, G, WT>;
  if (!allow_big_cluster(kinit, sm_init)) return DQ_ERR_CUDA;
  cfg.dynamicSmemBytes = sm_init;
  if (cudaLaunchKernelEx(&cfg, kinit, bt, m, steps, o) != cudaSuccess) return DQ_ERR_CUDA;

  cfg.dynamicSmemBytes = sm_main;
  cudaError_t e;
#define DQ_MAIN(WS, TR)                                                                     \
  {                                                                                         \
    auto km = solve_bcd_kernel<F, G, WT, WS, TR>;                                          \
    if (!allow_big_cluster(km, sm_main)) return DQ_ERR_CUDA;                               \
    e = cudaLaunchKernelEx(&cfg, km, bt, m, steps, T, o);                                   \
  }
  if (stg == 2) {
    if (any_trace) DQ_MAIN(2, true) else DQ_MAIN(2, false)
  } else if (stg == 1) {
    if (any_trace) DQ_MAIN(1, true) else DQ_MAIN(1, false)
  } else {
    if (any_trace) DQ_MAIN(0, true) else DQ_MAIN(0, false)
  }
#undef DQ_MAIN
  if (e != cudaSuccess) return DQ_ERR_CUDA;
  for (int i = 0; i < count && any_trace; ++i) {
    if (!traces[i]) continue;
    solve_finalize_kernel<<<(T + 1 + 127) / 128, 128, 0, st>>>(
        bt.item[i].ws, T, traces[i], (o.flags & SOLVE_TRACE_CODES) ? 1 : 0);
    if (cudaGetLastError() != cudaSuccess) return DQ_ERR_CUDA;
  }
  return DQ_OK;
}

// Whether a launch of this shape is possible (grid and shared-memory
// limits), checked before anything is enqueued.
template <int G, typename WT>
static int solver_supported(int64_t m, int64_t n) {
  int steps, C, stg;
  solver_geometry<G, WT>(m, steps, C, stg);
  const size_t sm_main =   // with the trace array: the largest variant
      solver_smem_bytes<G>(steps, stg == 2 ? sizeof(float) : (stg == 1 ? sizeof(WT) : 0), true);
  return (sm_main > 227 * 1024 || n / G > 65535) ? DQ_ERR_UNSUPPORTED : DQ_OK;
}

template <typename WT>
static int check_solver(int f, int G, int64_t m, int64_t n) {
  switch (f) {
    case NVFP4: return solver_supported<16, WT>(m, n);
    case MXFP4:
    case MXINT4:
    case MXINT8:
    case MXFP8: return solver_supported<32, WT>(m, n);
    case INT8:
    case INT4:
      if (G == 32) return solver_supported<32, WT>(m, n);
      if (G == 64) return solver_supported<64, WT>(m, n);
      return solver_supported<128, WT>(m, n);
  }
  return DQ_ERR_ARG;
}

template <typename WT>
static int dispatch_solver(int f, int G, const SolveBatch& bt, int count, int64_t m, int T,
                           const SolveOpts& o, double* const* traces, cudaStream_t st) {
  switch (f) {
    case NVFP4: return launch_solver<NVFP4, 16, WT>(bt, count, m, T, o, traces, st);
    case MXFP4: return launch_solver<MXFP4, 32, WT>(bt, count, m, T, o, traces, st);
    case MXINT4: return launch_solver<MXINT4, 32, WT>(bt, count, m, T, o, traces, st);
    case INT4:
      if (G == 32) return launch_solver<INT4, 32, WT>(bt, count, m, T, o, traces, st);
      if (G == 64) return launch_solver<INT4, 64, WT>(bt, count, m, T, o, traces, st);
      return launch_solver<INT4, 128, WT>(bt, count, m, T, o, traces, st);
    case MXINT8: return launch_solver<MXINT8, 32, WT>(bt, count, m, T, o, traces, st);
    case MXFP8: return launch_solver<MXFP8, 32, WT>(bt, count, m, T, o, traces, st);
    case INT8:
      if (G == 32) return launch_solver<INT8, 32, WT>(bt, count, m, T, o, traces, st);
      if (G == 64) return launch_solver<INT8, 64, WT>(bt, count, m, T, o, traces, st);
      return launch_solver<INT8, 128, WT>(bt, count, m, T, o, traces, st);
  }
  return DQ_ERR_ARG;
}

size_t solve_workspace_bytes(int T) {
  size_t b = 16 + 3 * 8 * (size_t)(T + 1);
  return (b + 255) & ~(size_t)255;
}

int solve_scales(const void* W, int wt, int64_t m, int64_t n, int f, int G, int T,
                 unsigned flags, const float* r0, const float* c0, float* r, float* c, float* sT,
                 double* trace, void* ws, cudaStream_t st) {
  const int ok = wt == 1 ? check_solver<__nv_bfloat16>(f, G, m, n) : check_solver<float>(f, G, m, n);
  if (ok != DQ_OK) return ok;
  if (cudaMemsetAsync(ws, 0, solve_workspace_bytes(T), st) != cudaSuccess) return DQ_ERR_CUDA;
  SolveBatch bt = {};
  bt.item[0] = SolveItem{W, r, c, sT, reinterpret_cast<SolverWs*>(ws), n};
  const SolveOpts o{flags, r0, c0};
  double* traces[1] = {trace};
  if (wt == 1) return dispatch_solver<__nv_bfloat16>(f, G, bt, 1, m, T, o, traces, st);
  return dispatch_solver<float>(f, G, bt, 1, m, T, o, traces, st);
}

// Weights are grouped by row count (one geometry per launch), in order of
// first appearance, up to SOLVE_BATCH_MAX per launch; a row count with more
// weights than that is picked up again by the later, not yet done weights.
int solve_scales_batched(int nw, const void* const* W, int wt, const int64_t* m,
                         const int64_t* n, int f, int G, int T, unsigned flags, float* const* r,
                         float* const* c, float* const* sT, double* const* trace, void* ws,
                         cudaStream_t st) {
  for (int i = 0; i < nw; ++i) {   // every launch possible before any is enqueued
    const int ok = wt == 1 ? check_solver<__nv_bfloat16>(f, G, m[i], n[i])
                           : check_solver<float>(f, G, m[i], n[i]);
    if (ok != DQ_OK) return ok;
  }
  const size_t per = solve_workspace_bytes(T);
  if (cudaMemsetAsync(ws, 0, per * (size_t)nw, st) != cudaSuccess) return DQ_ERR_CUDA;
  const SolveOpts o{flags, nullptr, nullptr};
  std::vector<char> done((size_t)nw, 0);
  for (int i = 0; i < nw; ++i) {
    if (done[i]) continue;
    SolveBatch bt = {};
    double* traces[SOLVE_BATCH_MAX] = {};
    int count = 0;
    for (int j = i; j < nw && count < SOLVE_BATCH_MAX; ++j) {
      if (done[j] || m[j] != m[i]) continue;
      bt.item[count] = SolveItem{W[j], r[j], c[j], sT[j],
                                 reinterpret_cast<SolverWs*>((char*)ws + per * (size_t)j), n[j]};
      traces[count] = trace ? trace[j] : nullptr;
      done[j] = 1;
      ++count;
    }
    const int rc = wt == 1 ? dispatch_solver<__nv_bfloat16>(f, G, bt, count, m[i], T, o, traces, st)
                           : dispatch_solver<float>(f, G, bt, count, m[i], T, o, traces, st);
    if (rc != DQ_OK) return rc;
  }
  return DQ_OK;
}

}  // namespace dq
