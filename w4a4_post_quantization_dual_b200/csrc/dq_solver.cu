// dq_solver.cu -- DualQuant's block-coordinate-descent scale solver on sm_100a.
//
// "DualQuant: Dual-scale Calibration-free Weight-and-Activation Quantization
// for LLMs", Algorithm 1 / Section 4.3 (closed-form updates Eqs. 10 and 14,
// Appendix B), initialisation of Section 5.3.
//
// With the row scale alpha being the format's native block scale, every
// m x G column-block tile of W is an independent problem: r_ib touches only
// tile b and every column lies in one tile.  One CTA (or, for tiles taller
// than one SM's shared memory holds, one thread-block cluster) owns one tile;
// the whole iteration loop runs on the device with the tile resident in
// shared memory.  Each thread owns 8 contiguous columns of a row per
// row-step; the G/8 threads of a row-block are lanes of one warp.  A round
// is one pass over the tile: per row-block the row update (warp shuffles
// over the row-block's lanes) and, at the new row scale, the thread's column
// partials; then the column update from the partials (warp reduce-scatter,
// fp64 over warps, DSMEM over the cluster in rank order).
#include <cuda_runtime.h>
#include <stdint.h>

#include <type_traits>
#include <vector>

#include "dq_device.cuh"
#include "dq_internal.h"

namespace dq {

template <int G>
struct SolverShape {
  static constexpr int OPB = G / 8;            // 8-column octets per row-block (lanes per row-block)
  static constexpr int NT = 512;
  static constexpr int NW = NT / 32;
  static constexpr int RPW = 32 / OPB;         // rows per warp per step
  static constexpr int RPS = NW * RPW;         // rows per CTA per step
  // column reduce-scatter over the RPW lanes that share an octet: LV shuffle
  // levels, after which each lane holds VPL of the octet's 16 (num, den) sums
  static constexpr int LV = RPW == 16 ? 4 : RPW == 8 ? 3 : RPW == 4 ? 2 : RPW == 2 ? 1 : 0;
  static constexpr int VPL = 16 / RPW;
  static_assert((1 << LV) == RPW && RPW <= 16, "reduce-scatter shape");
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
// Two doubles into CTA `rank`'s shared memory (made visible to it by the
// release / acquire of the next cluster barrier).
__device__ __forceinline__ void st_dsmem_f64x2(const double* local, uint32_t rank, double a,
                                               double b) {
  uint32_t la = (uint32_t)__cvta_generic_to_shared(local), ra;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"(la), "r"(rank));
  asm volatile("st.shared::cluster.v2.f64 [%0], {%1, %2};" ::"r"(ra), "d"(a), "d"(b) : "memory");
}

// Reduce V fp64 partials per thread over the CTA's threads that share an
// octet (initialisation: column l1 norms); scr (the float scratch of
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
// One pass over the tile per round.  A row's update depends only on that
// row, and the column update needs every row's new scale, so each row-block
// is taken through the whole round at once: x -> y = x beta (used by both
// half-steps of the round) -> codes at the old alpha -> <W_i, R_i>,
// ||R_i||^2 over the row-block's lanes -> projected row scale -> codes at
// the new alpha -> the thread's column partials <S_j, W_j>, ||S_j||^2.
// After the pass the column partials are reduce-scattered over the lanes of
// each warp that share an octet (shuffles), summed over the warps in fp64
// and, when the tile spans a cluster, over its CTAs in rank order (DSMEM).
//
// Each CTA keeps its rows of the tile in shared memory in the weight's own
// type for all T rounds (tiles too tall for that stream their rows through
// the read-only global path); rows past m are zeros, so every loop runs the
// same number of steps in every lane.  Element arithmetic uses the packed
// fp32x2 instructions of sm_100 (each lane of a pair is an ordinary
// correctly-rounded fp32 operation, so the quantiser argument
// (w * beta) * alpha is bit-identical to the scalar definition).
// TRACE: accumulate the reconstruction error for the MSE trace (and, with
// DQ_SOLVE_TRACE_CODES, the code change between rounds).
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

__device__ __forceinline__ void bf16x8_to_f2(const uint4& v, float2* x) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i)
    x[i] = make_float2(__uint_as_float(w[i] << 16), __uint_as_float(w[i] & 0xFFFF0000u));
}

// Fixed part of the main kernel's shared memory; the row-block scales of
// the CTA's rows (r, alpha), the trace's previous alphas and the staged rows
// follow it.
template <int G>
struct BcdSmem {
  using S = SolverShape<G>;
  float part[S::NW * 2 * G];   // per-warp column partials [warp][octet][16]; the exact
                               // column pass reuses it as doubles [warp][octet][4]
  double cpart[2][2 * G];      // this CTA's column totals, cluster-visible, double-buffered
  float c_s[G], b_s[G];        // current c and beta = fl(1/c)
  float b_old[G];              // beta before the column update (exact column pass)
  float rtab[128], atab[128];  // NVFP4: r and alpha of every scale byte
};

template <int F, int G, typename WT, bool STAGED, bool TRACE>
__global__ void __launch_bounds__(SolverShape<G>::NT, 1)
solve_bcd_kernel(SolveBatch bt, int64_t m, int steps, int T, SolveOpts o) {
  using S = SolverShape<G>;
  constexpr uint32_t FULL = 0xffffffffu;
  const int64_t n = bt.item[blockIdx.z].n;
  if ((int64_t)blockIdx.y >= n / G) return;   // whole clusters (they span x only)
  const WT* __restrict__ W = reinterpret_cast<const WT*>(bt.item[blockIdx.z].W);
  float* r_out = bt.item[blockIdx.z].r;
  float* __restrict__ c_io = bt.item[blockIdx.z].c;
  float* sT_io = bt.item[blockIdx.z].sT;
  SolverWs* ws = bt.item[blockIdx.z].ws;
  extern __shared__ __align__(16) unsigned char smem_raw[];
  BcdSmem<G>& sm = *reinterpret_cast<BcdSmem<G>*>(smem_raw);
  const int rows_cta = steps * S::RPS;
  const uint32_t C = gridDim.x;
  // cluster receive buffers [2][C][2G] of column totals (C > 1), then
  // (r, alpha) per row, the trace's previous alphas and the staged rows
  double* recv = reinterpret_cast<double*>(smem_raw + ((sizeof(BcdSmem<G>) + 15) & ~(size_t)15));
  float2* ra_s = reinterpret_cast<float2*>(recv + (C > 1 ? 4 * (size_t)C * G : 0));
  float* ap_s = reinterpret_cast<float*>(ra_s + rows_cta);        // TRACE only
  WT* wch = reinterpret_cast<WT*>(ap_s + (TRACE ? rows_cta : 0));  // staged rows

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int oct = lane % S::OPB, rr = lane / S::OPB, rslot = warp * S::RPW + rr;
  const uint32_t rank = cluster_ctarank();
  const int64_t b = blockIdx.y, nb = n / G;
  const int64_t col0 = b * G + oct * 8;
  const int64_t row0 = (int64_t)rank * rows_cta;

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
      sm.rtab[tid] = rv;
      sm.atab[tid] = __frcp_rn(rv);
    }
  }
  if (rank == 0 && b == 0 && tid == 0 && !keep_s) *sT_io = sT;
  const float inv_sT = __frcp_rn(sT);

  if constexpr (STAGED) {
    // rows [row0, row0 + rows_cta) x columns [b*G, b*G + G), zeros past m,
    // in 16-byte pieces.  bf16: row-major.  fp32: two planes (elements 0-3
    // and 4-7 of every octet), so that a warp's 16-byte reads are contiguous.
    constexpr int PPR = G * (int)sizeof(WT) / 16;     // pieces per row
    for (int p = tid; p < rows_cta * PPR; p += S::NT) {
      const int lr = p / PPR, pc = p % PPR;
      const int64_t i = row0 + lr;
      uint4 v = make_uint4(0u, 0u, 0u, 0u);
      if (i < m) v = __ldg(reinterpret_cast<const uint4*>(W + i * n + b * G) + pc);
      if constexpr (sizeof(WT) == 2)
        reinterpret_cast<uint4*>(wch)[p] = v;
      else
        reinterpret_cast<uint4*>(wch)[(pc & 1) * rows_cta * S::OPB + lr * S::OPB + (pc >> 1)] = v;
    }
  }
  // elements 8 oct .. 8 oct + 7 of CTA row lr, as fp32 pairs
  auto load_x = [&](int lr, float2* x) {
    if constexpr (STAGED) {
      if constexpr (sizeof(WT) == 2) {
        bf16x8_to_f2(reinterpret_cast<const uint4*>(wch)[lr * S::OPB + oct], x);
      } else {
        const float4 a = reinterpret_cast<const float4*>(wch)[lr * S::OPB + oct];
        const float4 c = reinterpret_cast<const float4*>(wch)[rows_cta * S::OPB + lr * S::OPB + oct];
        x[0] = make_float2(a.x, a.y); x[1] = make_float2(a.z, a.w);
        x[2] = make_float2(c.x, c.y); x[3] = make_float2(c.z, c.w);
      }
    } else {
      const int64_t i = row0 + lr;
      if (i < m) {
        if constexpr (sizeof(WT) == 2) {
          bf16x8_to_f2(__ldg(reinterpret_cast<const uint4*>(W + i * n + col0)), x);
        } else {
          const float4 a = __ldg(reinterpret_cast<const float4*>(W + i * n + col0));
          const float4 c = __ldg(reinterpret_cast<const float4*>(W + i * n + col0) + 1);
          x[0] = make_float2(a.x, a.y); x[1] = make_float2(a.z, a.w);
          x[2] = make_float2(c.x, c.y); x[3] = make_float2(c.z, c.w);
        }
      } else {
#pragma unroll
        for (int k = 0; k < 4; ++k) x[k] = make_float2(0.f, 0.f);
      }
    }
  };

  float2 cc[4], beta[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    cc[k] = make_float2(c_io[col0 + 2 * k], c_io[col0 + 2 * k + 1]);
    beta[k] = make_float2(__frcp_rn(cc[k].x), __frcp_rn(cc[k].y));
  }
  if (tid < G) {
    sm.c_s[tid] = c_io[b * G + tid];
    sm.b_s[tid] = __frcp_rn(sm.c_s[tid]);
  }
  __syncthreads();   // staged rows, scale tables

  // r0: the caller's scales projected onto F_alpha (rows past m take the
  // projection of 1), or else the format-native absmax scale of
  // W diag(c0)^-1 per row-block (the same fp32 decisions as the oracle's
  // initialisation).  Each r0 entry is read by the lane that writes the same
  // entry of r at the end (r0 may alias r).
  for (int s = 0; s < steps; ++s) {
    const int lr = s * S::RPS + rslot;
    const int64_t i = row0 + lr;
    float rv;
    if (o.r0 != nullptr) {
      rv = proj_alpha<F>((oct == 0 && i < m) ? o.r0[i * nb + b] : 1.0f, sT);
    } else {
      float2 x[4];
      load_x(lr, x);
      float a = 0.0f;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float2 p = __fmul2_rn(x[k], beta[k]);
        a = fmaxf(a, fmaxf(fabsf(p.x), fabsf(p.y)));
      }
#pragma unroll
      for (int d = 1; d < S::OPB; d <<= 1) a = fmaxf(a, __shfl_xor_sync(FULL, a, d));
      rv = rtn_block_scale<F>(a, sT);
    }
    if (oct == 0) ra_s[lr] = make_float2(rv, __frcp_rn(rv));
  }
  __syncwarp();

  int xb = 0;   // buffer of the next exact-pass exchange
  int xr = 0;   // index of the next column-total exchange (receive buffer xr & 1)
  // column window: the per-thread fp32 chain (steps terms) and the fp32
  // reduce-scatter levels, 2 * depth + 4 ulps, + 4 for S = r q in fp32
  const uint32_t col_win = 2u * (uint32_t)(steps + S::LV) + 8u;
  const bool trace_codes = TRACE && (o.flags & SOLVE_TRACE_CODES);
  float2 beta_prev[4];   // TRACE: beta of the previous round
#pragma unroll
  for (int k = 0; k < 4; ++k) beta_prev[k] = beta[k];
  for (int t = 0; t <= T; ++t) {
    const bool do_row = t < T && !beta_only;
    const bool do_col = t < T && !alpha_only;
    if (!do_row && !do_col && !TRACE) break;
    float e_acc = 0.0f;
    float2 qn2 = make_float2(0.f, 0.f), qd2 = qn2;   // TRACE: code-change sums
    float2 accn[4], accd[4];                          // column partials (num, den) per pair
#pragma unroll
    for (int k = 0; k < 4; ++k) accn[k] = accd[k] = make_float2(0.f, 0.f);

    for (int s = 0; s < steps; ++s) {
      const int lr = s * S::RPS + rslot;
      float2 x[4], q[4];
      load_x(lr, x);
      const float2 ra = ra_s[lr];
      float rn = ra.x, an = ra.y;
      {
        // codes at the current scales: the row half-step's, and the column
        // half-step's too wherever the row scale does not move
        const float2 a2 = make_float2(ra.y, ra.y);
#pragma unroll
        for (int k = 0; k < 4; ++k) q[k] = grid2_packed<F>(__fmul2_rn(__fmul2_rn(x[k], beta[k]), a2));
      }
      if (do_row || TRACE) {
        // ---- row half-step at the current scales (and the error there) ----
        const float2 a2 = make_float2(ra.y, ra.y);
        float2 num2 = make_float2(0.f, 0.f), den2 = num2, err2 = num2;
        float2 R[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) R[k] = __fmul2_rn(q[k], cc[k]);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          num2 = __ffma2_rn(x[k], R[k], num2);
          den2 = __ffma2_rn(R[k], R[k], den2);
          if constexpr (TRACE) {
            const float2 d = __ffma2_rn(make_float2(-ra.x, -ra.x), R[k], x[k]);
            err2 = __ffma2_rn(d, d, err2);
          }
        }
        if constexpr (TRACE) {
          // Qhat(t) - Qhat(t-1): the codes at the previous round's scales
          if (trace_codes && t > 0) {
            const float ap = ap_s[lr];
            const float2 ap2 = make_float2(ap, ap);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const float2 qp = grid2_packed<F>(__fmul2_rn(__fmul2_rn(x[k], beta_prev[k]), ap2));
              const float2 d = make_float2(q[k].x - qp.x, q[k].y - qp.y);
              qn2 = __ffma2_rn(d, d, qn2);
              qd2 = __ffma2_rn(qp, qp, qd2);
            }
          }
        }
        float num = num2.x + num2.y, den = den2.x + den2.y, err = err2.x + err2.y;
#pragma unroll
        for (int d = 1; d < S::OPB; d <<= 1) {
          num += __shfl_xor_sync(FULL, num, d);
          den += __shfl_xor_sync(FULL, den, d);
          if constexpr (TRACE) err += __shfl_xor_sync(FULL, err, d);
        }
        if constexpr (TRACE) {
          if (oct == 0) e_acc += err;
          if (trace_codes) {   // the alpha these codes were taken with serves the next round
            __syncwarp();
            if (oct == 0) ap_s[lr] = ra.y;
          }
        }
        if (do_row) {
          const float u = den > 0.0f ? __fdividef(num, den) : 1.0f;
          // all lanes of a row-block hold the same sums, hence the same flag
          const bool tie = den > 0.0f && near_tie_alpha<F>(u, inv_sT, ROW_TIE_WIN);
          RowProj<F>::apply(u, inv_sT, sm.rtab, sm.atab, sT, rn, an);
          if (__any_sync(FULL, tie)) {
            // rare: the update lies near a projection boundary -- take it from
            // exact sums, <W_i, R_i> and ||R_i||^2 in fp64 (x R is exact in
            // fp64, R = q c exact in fp32), the quotient rounded once to fp32
            double dn = 0.0, dd = 0.0;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const float2 Rk = __fmul2_rn(q[k], cc[k]);
              dn = fma((double)x[k].x, (double)Rk.x, dn);
              dn = fma((double)x[k].y, (double)Rk.y, dn);
              dd = fma((double)Rk.x, (double)Rk.x, dd);
              dd = fma((double)Rk.y, (double)Rk.y, dd);
            }
#pragma unroll
            for (int d = 1; d < S::OPB; d <<= 1) {
              dn += __shfl_xor_sync(FULL, dn, d);
              dd += __shfl_xor_sync(FULL, dd, d);
            }
            if (tie) {
              rn = proj_alpha<F>((float)(dn / dd), sT);
              an = __frcp_rn(rn);
            }
          }
          if (oct == 0) ra_s[lr] = make_float2(rn, an);
        }
      }
      if (do_col) {
        // ---- column partials with the new row scale ----
        // a row-block whose scale did not move keeps its codes (the same
        // fp32 products as above); the warp re-quantises only if one moved
        if (!__all_sync(FULL, an == ra.y)) {
          const float2 a2 = make_float2(an, an);
#pragma unroll
          for (int k = 0; k < 4; ++k) q[k] = grid2_packed<F>(__fmul2_rn(__fmul2_rn(x[k], beta[k]), a2));
        }
        const float2 r2 = make_float2(rn, rn);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float2 Sv = __fmul2_rn(r2, q[k]);
          accn[k] = __ffma2_rn(Sv, x[k], accn[k]);
          accd[k] = __ffma2_rn(Sv, Sv, accd[k]);
        }
      }
    }
    if constexpr (TRACE) {
#pragma unroll
      for (int d = 16; d; d >>= 1) e_acc += __shfl_xor_sync(FULL, e_acc, d);
      if (lane == 0) atomicAdd(&ws->err[t], (double)e_acc);
      if (trace_codes) {
        // sums of this warp; qnum / qden follow err[T+1] in the workspace
        float qn = qn2.x + qn2.y, qd = qd2.x + qd2.y;
#pragma unroll
        for (int d = 16; d; d >>= 1) {
          qn += __shfl_xor_sync(FULL, qn, d);
          qd += __shfl_xor_sync(FULL, qd, d);
        }
        if (lane == 0 && t > 0) {
          atomicAdd(&ws->err[(T + 1) + t], (double)qn);
          atomicAdd(&ws->err[2 * (T + 1) + t], (double)qd);
        }
#pragma unroll
        for (int k = 0; k < 4; ++k) beta_prev[k] = beta[k];
      }
    }
    if (!do_col) continue;

    // ---- column half-step: c_j <- Pi(<S_j, W_j> / ||S_j||^2) ----
    // v[2c], v[2c+1] = (num, den) of column c of the octet; reduce-scatter
    // over the RPW lanes sharing the octet: after LV levels each lane holds
    // the warp's sums of VPL of the 16 values, starting at `base`
    float v[16];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      v[4 * k + 0] = accn[k].x;
      v[4 * k + 1] = accd[k].x;
      v[4 * k + 2] = accn[k].y;
      v[4 * k + 3] = accd[k].y;
    }
    int base = 0;
#pragma unroll
    for (int l = 0; l < S::LV; ++l) {
      const int half = 16 >> (l + 1);
      const bool up = (lane & (S::OPB << l)) != 0;
#pragma unroll
      for (int i = 0; i < half; ++i) {
        const float send = up ? v[i] : v[i + half];
        const float keep = up ? v[i + half] : v[i];
        v[i] = keep + __shfl_xor_sync(FULL, send, S::OPB << l);
      }
      base += up ? half : 0;
    }
#pragma unroll
    for (int i = 0; i < S::VPL; ++i) sm.part[(warp * S::OPB + oct) * 16 + base + i] = v[i];
    __syncthreads();
    double sn = 0.0, sd = 0.0;
    if (tid < G) {   // column tid: its warps' sums in fp64, warp order
      const float* p = sm.part + (tid >> 3) * 16 + 2 * (tid & 7);
      float pn[S::NW], pd[S::NW];
#pragma unroll
      for (int w = 0; w < S::NW; ++w) {
        pn[w] = p[w * 2 * G];
        pd[w] = p[w * 2 * G + 1];
      }
#pragma unroll
      for (int w = 0; w < S::NW; ++w) {
        sn += (double)pn[w];
        sd += (double)pd[w];
      }
    }
    if (C > 1) {
      // the CTA totals go to the cluster; every CTA sums all of them in rank
      // order (identical c in every CTA).  The buffer alternates with every
      // exchange: a CTA writes buffer xb only after all peers passed the
      // barrier that follows their last reads of it.
      // pushed into slot `rank` of every CTA's receive buffer before the
      // barrier, read locally after it
      double* rb = recv + (size_t)(xr & 1) * C * 2 * G;
      if (tid < G)
        for (uint32_t q = 0; q < C; ++q) st_dsmem_f64x2(rb + rank * 2 * G + 2 * tid, q, sn, sd);
      cluster_sync_all();
      if (tid < G) {
        sn = 0.0;
        sd = 0.0;
        for (uint32_t q = 0; q < C; ++q) {
          sn += rb[q * 2 * G + 2 * tid];
          sd += rb[q * 2 * G + 2 * tid + 1];
        }
      }
      ++xr;
    }
    // projected update; a column near a projection boundary is redone below
    // from exact sums
    bool ctie = false;
    if (tid < G) {
      const float cu = (sd > 0.0) ? (float)(sn / sd) : 1.0f;
      ctie = sd > 0.0 && near_tie_beta<F>(cu, col_win);
      const float cn = proj_beta<F>(cu);
      sm.b_old[tid] = sm.b_s[tid];
      sm.c_s[tid] = cn;
      sm.b_s[tid] = __frcp_rn(cn);
    }
    // every CTA of the cluster sums the same totals in the same order, so the
    // flag is cluster-uniform and the exact pass below (with its cluster
    // barrier) runs in all of them or in none
    if (__syncthreads_or(ctie)) {
      // rare: exact fp64 column sums of the tile -- per thread <S_j, W_j> and
      // ||S_j||^2 for one column pair of its octet at a time, S = r q formed
      // in fp64 (exact) and S * S rounded once as in a plain fp64 loop, then
      // over the octet's lanes, the warps (warp order) and the CTAs (rank order)
      double* xpart = reinterpret_cast<double*>(sm.part);   // [warp][octet][4]
#pragma unroll 1
      for (int kp = 0; kp < 4; ++kp) {
        double a4[4] = {0.0, 0.0, 0.0, 0.0};
        const float2 bp = make_float2(sm.b_old[oct * 8 + 2 * kp], sm.b_old[oct * 8 + 2 * kp + 1]);
        for (int s = 0; s < steps; ++s) {
          const int lr = s * S::RPS + rslot;
          const float2 ra = ra_s[lr];
          float2 x[4];
          load_x(lr, x);
          float2 xp = x[0];
#pragma unroll
          for (int k = 1; k < 4; ++k) xp = (k == kp) ? x[k] : xp;
          const float2 q = grid2_packed<F>(__fmul2_rn(__fmul2_rn(xp, bp), make_float2(ra.y, ra.y)));
          const double s0 = (double)ra.x * (double)q.x, s1 = (double)ra.x * (double)q.y;
          a4[0] = __dadd_rn(a4[0], __dmul_rn(s0, (double)xp.x));
          a4[1] = __dadd_rn(a4[1], __dmul_rn(s0, s0));
          a4[2] = __dadd_rn(a4[2], __dmul_rn(s1, (double)xp.y));
          a4[3] = __dadd_rn(a4[3], __dmul_rn(s1, s1));
        }
#pragma unroll
        for (int l = 0; l < S::LV; ++l)
#pragma unroll
          for (int i = 0; i < 4; ++i) a4[i] += __shfl_xor_sync(FULL, a4[i], S::OPB << l);
        if (rr == 0)
#pragma unroll
          for (int i = 0; i < 4; ++i) xpart[(warp * S::OPB + oct) * 4 + i] = a4[i];
        __syncthreads();
        if (tid < S::OPB * 4) {
          double acc = 0.0;
          for (int w = 0; w < S::NW; ++w) acc += xpart[(w * S::OPB + (tid >> 2)) * 4 + (tid & 3)];
          // value i of the pair: (num, den) of column 2 kp, then of 2 kp + 1
          const int j = (tid >> 2) * 8 + 2 * kp + ((tid & 3) >> 1);
          sm.cpart[xb][2 * j + (tid & 1)] = acc;
        }
        __syncthreads();
      }
      if (C > 1) cluster_sync_all();
      if (ctie) {   // rank order, one CTA at a time (rare path)
        double en = 0.0, ed = 0.0;
        for (uint32_t q = 0; q < C; ++q) {
          en += ld_dsmem_f64(&sm.cpart[xb][2 * tid], q);
          ed += ld_dsmem_f64(&sm.cpart[xb][2 * tid + 1], q);
        }
        const float cn = proj_beta<F>((float)(en / ed));
        sm.c_s[tid] = cn;
        sm.b_s[tid] = __frcp_rn(cn);
      }
      if (C > 1) xb ^= 1;
      __syncthreads();
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      cc[k] = make_float2(sm.c_s[oct * 8 + 2 * k], sm.c_s[oct * 8 + 2 * k + 1]);
      beta[k] = make_float2(sm.b_s[oct * 8 + 2 * k], sm.b_s[oct * 8 + 2 * k + 1]);
    }
  }

  // outputs
  for (int s = 0; s < steps; ++s) {
    const int lr = s * S::RPS + rslot;
    if (oct == 0 && row0 + lr < m) r_out[(row0 + lr) * nb + b] = ra_s[lr].x;
  }
  if (rank == 0 && tid < G && T > 0 && !alpha_only) c_io[b * G + tid] = sm.c_s[tid];
  if (C > 1) cluster_sync_all();  // no CTA leaves while a peer may still read its cpart
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
constexpr size_t SOLVER_SMEM_MAX = 227 * 1024;

// Dynamic shared memory of the main kernel: the fixed part, (r, alpha) per
// row, the previous alpha per row (trace), and the staged rows
// (elem_bytes = 0: streamed).
template <int G>
static size_t solver_smem_bytes(int steps, size_t elem_bytes, bool trace, int C) {
  const size_t rows = (size_t)steps * SolverShape<G>::RPS;
  return ((sizeof(BcdSmem<G>) + 15) & ~(size_t)15) + (C > 1 ? 32 * (size_t)C * G : 0) +
         rows * 8 + (trace ? rows * 4 : 0) + rows * G * elem_bytes;
}

// Launch geometry: the tile's rows are split over C CTAs of one cluster,
// `steps` row-steps of RPS rows per CTA.  The fewest CTAs whose rows fit in
// shared memory in the weight's own type (one CTA per SM, so a tile that fits
// one SM needs no cluster exchange); tiles taller than 16 CTAs hold stream
// their rows through the read-only global path with clusters of up to 8.
// The sizes are those of the traced variant, so that a trace never changes
// the geometry.
template <int G, typename WT>
static void solver_geometry(int64_t m, int& steps, int& C, int& stg) {
  using S = SolverShape<G>;
  for (int c = 1; c <= 16; ++c) {
    const int64_t rows = (m + c - 1) / c;
    const int st = (int)((rows + S::RPS - 1) / S::RPS);
    const int cc = (int)((m + (int64_t)S::RPS * st - 1) / ((int64_t)S::RPS * st));
    if (solver_smem_bytes<G>(st, sizeof(WT), true, cc) <= SOLVER_SMEM_MAX) {
      steps = st;
      C = cc;
      stg = 1;
      return;
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
               sm_main = solver_smem_bytes<G>(steps, stg ? sizeof(WT) : 0, any_trace, C);
  if (sm_main > SOLVER_SMEM_MAX) return DQ_ERR_UNSUPPORTED;
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
#define DQ_MAIN(STAGED, TR)                                                                 \
  {                                                                                         \
    auto km = solve_bcd_kernel<F, G, WT, STAGED, TR>;                                      \
    if (!allow_big_cluster(km, sm_main)) return DQ_ERR_CUDA;                               \
    e = cudaLaunchKernelEx(&cfg, km, bt, m, steps, T, o);                                   \
  }
  if (stg) {
    if (any_trace) DQ_MAIN(true, true) else DQ_MAIN(true, false)
  } else {
    if (any_trace) DQ_MAIN(false, true) else DQ_MAIN(false, false)
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
  const size_t sm_main = solver_smem_bytes<G>(steps, stg ? sizeof(WT) : 0, true, C);
  return (sm_main > SOLVER_SMEM_MAX || n / G > 65535) ? DQ_ERR_UNSUPPORTED : DQ_OK;
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
