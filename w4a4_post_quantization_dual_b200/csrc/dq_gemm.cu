// dq_gemm.cu -- block-scaled FP4 GEMM with the DualQuant epilogue (sm_100a).
//
// "DualQuant", Section 4.4: at inference the layer computes
// Q(X~) What^T Diag(alpha)^-1.  The row-block scales r = alpha^-1 are the
// weight's native block scales, so they are applied inside the tensor-core
// MMA together with the activation block scales; the per-token (NVFP4)
// and per-tensor scales, and an optional per-output-row factor, are applied
// in the epilogue.
//
//   Y[t, o] = s_tok[t] s_w r_row[o] sum_k a[t,k] sa[t,k/G] b[o,k] sb[o,k/G]
//
// Design (one CTA per SM, persistent over 128 x BN output tiles):
//   warp 0      TMA producer: A / B code tiles (128-byte swizzled K-major,
//               BK = 256 four-bit elements) and the matching 512-byte
//               block-scale atoms (bulk copies), into a STAGES-deep ring.
//   warp 1      allocates tensor memory; one thread issues
//               tcgen05.mma.kind::mxf4nvf4 / kind::mxf4 .block_scale, fp32
//               accumulation in tensor memory; commits free the ring slots.
//   warps 2..5  epilogue: tcgen05.ld the accumulator (each warp its 32-lane
//               quadrant), release it to the MMA warp, scale, convert, store.
//   warps 6..9  copy each stage's scale atoms into that stage's own slot of
//               tensor memory (tcgen05.cp 32x128b.warpx4), a quarter each,
//               and signal the MMA warp: a thread's copies run one after
//               another at about an MMA's duration each, but the copies of
//               different warps overlap each other and the MMAs.
// Every mbarrier wait is bounded (globaltimer); on expiry the kernel records
// DQ_ERR_DEVICE_TIMEOUT in the device error word and unwinds.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdlib.h>

#include "dq_device.cuh"
#include "dq_internal.h"

namespace dq {

__device__ int g_dq_device_error = 0;
// Time limit of the bounded mbarrier waits of the pipelines, in ns: 2 s by
// default, far beyond any legitimate wait.  dq_set_wait_limit changes it
// (a test makes the waits expire to exercise the unwinding below).
__device__ unsigned long long g_dq_wait_limit_ns = 2000000000ull;

namespace gemm {

constexpr int BM = 128;
constexpr int BK = 256;             // four-bit elements per k-tile (128 bytes per row)
constexpr int BKB = BK / 2;         // bytes per row per k-tile
constexpr int NUM_THREADS = 320;
// Scale-factor copies: one tcgen05.cp occupies its issuing thread's queue for
// roughly an MMA's time, while copies issued by different warps run
// concurrently with each other and with the MMAs.  Four copier warps
// (6..9) therefore share each stage's scale atoms round-robin.
constexpr int COPIERS = 4;
constexpr int FIRST_COPIER = 6;
// Limit of the waits that unwind a CTA after an expiry: fixed, whatever the
// pipeline limit, because they only wait for work that was issued and will
// complete on its own.
constexpr uint64_t DRAIN_LIMIT_NS = 2000000000ull;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity) : "memory");
  return ok != 0;
}
// Bounded wait: returns false (and raises the abort flag) if the phase does
// not complete within the pipeline limit or another role already aborted.
__device__ __noinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  const uint64_t lim = *reinterpret_cast<volatile unsigned long long*>(&g_dq_wait_limit_ns);
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (globaltimer() - t0 > lim) {
      *abort_flag = 1;
      atomicExch(&g_dq_device_error, DQ_ERR_DEVICE_TIMEOUT);
      return false;
    }
  }
}
// Bounded wait with the fixed limit that ignores the abort flag: a role
// whose progress must not depend on another role's abort (the producers of
// the paired-SM kernel, whose loads are counted on one CTA's barrier).
__device__ __noinline__ bool mbar_wait_fixed(uint64_t* bar, uint32_t parity,
                                             volatile int* abort_flag) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (globaltimer() - t0 > DRAIN_LIMIT_NS) {
      *abort_flag = 1;
      atomicExch(&g_dq_device_error, DQ_ERR_DEVICE_TIMEOUT);
      return false;
    }
  }
}
// Unwinding wait: for a phase that work already issued will complete (loads
// that landed or are in flight, a commit after issued tensor-core work).
// Ignores the abort flag; bounded by the fixed limit.
__device__ __noinline__ bool mbar_drain(uint64_t* bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (globaltimer() - t0 > DRAIN_LIMIT_NS) {
      atomicExch(&g_dq_device_error, DQ_ERR_DEVICE_TIMEOUT);
      return false;
    }
  }
}
// A producer's unwinding: wait until the loads of the last `issued` stages
// (at most STAGES) before ring position (stage, phase) -- the next slot it
// would have filled -- have landed, on `full` (and `full2`, nullable).  A
// stage filled at phase p completes its barrier's phase of parity p, and no
// later fill of the stage was issued, so the wait is unambiguous.
template <int STAGES>
__device__ __forceinline__ void drain_loads(uint64_t* full, uint64_t* full2, int stage,
                                            uint32_t phase, int issued) {
  for (int i = 0; i < issued && i < STAGES; ++i) {
    if (stage == 0) {
      stage = STAGES - 1;
      phase ^= 1u;
    } else {
      --stage;
    }
    mbar_drain(&full[stage], phase);
    if (full2) mbar_drain(&full2[stage], phase);
  }
}

// Fetch a tensor map's descriptor ahead of its first use.
__device__ __forceinline__ void prefetch_tmap(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)map) : "memory");
}
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
      "l"((uint64_t)map), "r"(smem_u32(bar)), "r"(x), "r"(y)
      : "memory");
}
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes,
                                          uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(smem_u32(dst)), "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// Shared-memory matrix descriptor (tcgen05): start, leading / stride byte
// offsets (>> 4), version 1, layout type in bits 61-63.
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo,
                                              uint32_t layout) {
  uint64_t d = 0;
  d |= (uint64_t)((addr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)(layout & 7u) << 61;
  return d;
}
constexpr uint32_t LAYOUT_SW128 = 2, LAYOUT_NONE = 0;

// Instruction descriptor for kind::mxf4 / kind::mxf4nvf4 with E2M1 A and B,
// K-major operands, M = 128.
__host__ __device__ constexpr uint32_t idesc_fp4(int N, bool e8m0_scales) {
  return (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((e8m0_scales ? 1u : 0u) << 23) |
         ((uint32_t)(BM >> 4) << 24);
}

template <int FMT>
__device__ __forceinline__ void mma_fp4(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                        uint32_t idesc, uint32_t accumulate, uint32_t tsfa,
                                        uint32_t tsfb) {
  if constexpr (FMT == NVFP4) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t}"
        ::"r"(tmem_d), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(tsfa), "r"(tsfb)
        : "memory");
  } else {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf4.block_scale.block32 [%0], %1, %2, %3, [%5], [%6], p;\n\t}"
        ::"r"(tmem_d), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(tsfa), "r"(tsfb)
        : "memory");
  }
}
__device__ __forceinline__ void tmem_cp_32x128b_x4(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc)
               : "memory");
}
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}
__device__ __forceinline__ void fence_after_sync() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void fence_before_sync() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t* v) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
        "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]),
        "=r"(v[14]), "=r"(v[15]), "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]),
        "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]), "=r"(v[24]), "=r"(v[25]),
        "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// AR: rows of A staged per k-tile.  The MMA always computes 128 rows; with
// AR < 128 (every token fits in AR rows) it reads the rows past AR from the
// shared memory that follows the stage, which only feeds accumulator rows
// that are never stored, and each stage is smaller, so more of the weight
// stream is in flight.
template <int FMT, int BN, int RESERVE = 0, int AR = BM>
struct Cfg {
  static constexpr int G = (FMT == NVFP4) ? 16 : 32;
  static constexpr int SF_PER_ROW = BK / G;                   // scales per row per k-tile
  static constexpr int SF_ATOMS = SF_PER_ROW / 4;             // 512-byte atoms per 128 rows
  static constexpr int A_BYTES = AR * BKB;                    // 16 KB for 128 rows
  static constexpr int B_BYTES = BN * BKB;
  static constexpr int SFA_BYTES = SF_ATOMS * 512;
  static constexpr int SFB_BYTES = (BN / 128) * SF_ATOMS * 512;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES;
  static constexpr int STAGES = (227 * 1024 - 1024 - 512 - RESERVE) / STAGE_BYTES;
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 /*align*/ + 512 /*barriers*/ + RESERVE;
  static_assert(AR % 32 == 0 && AR <= BM, "staged A rows");
  static_assert(4 * STAGES * 8 + 40 <= 512, "barrier area");
  // the MMA's 128-row read of the last A stage stays inside the B stages
  static_assert((BM - AR) * BKB <= STAGES * B_BYTES, "A read window");
  // tensor-memory columns: accumulator, then one scale slot per stage
  // (SFA: 4 columns per atom; SFB: 4 columns per atom and 128-row group)
  static constexpr int SF_COLS = 4 * SF_ATOMS * (1 + BN / 128);
  static constexpr int SF_BASE = BN;
  static constexpr int TMEM_USED = SF_BASE + STAGES * SF_COLS;
  static constexpr int TMEM_COLS = TMEM_USED <= 128 ? 128 : (TMEM_USED <= 256 ? 256 : 512);
  static constexpr int K_STEPS = BK / 64;                     // MMAs per k-tile (K = 64 each)
  static_assert(STAGES >= 2, "pipeline depth");
  static_assert(TMEM_USED <= 512, "tensor memory budget");
};

// Output tile `tile` of the persistent loop -> (tm, tn).  The tiles the SMs
// run at the same time are consecutive: with M <= N they share N columns and
// the whole of A (the smaller operand) stays in L2 while B streams; with
// M > N they share M rows and B stays in L2 instead (8192 x 5120 x 27648 in
// M-fastest order read 1.25 GB from DRAM for 0.2 GB of operands).
__device__ __forceinline__ int2 tile_mn(int tile, int tiles_m, int tiles_n, bool nfast) {
  return nfast ? make_int2(tile / tiles_n, tile % tiles_n) : make_int2(tile % tiles_m, tile / tiles_m);
}

// bf16 epilogue of one 128 x BN tile for one thread (one accumulator row):
// drain the whole row from tensor memory into packed bf16 registers, hand the
// accumulator back to the MMA warp, then store.
template <int BN, bool ROWF>
__device__ __forceinline__ void epilogue_bf16(uint32_t tmem, int quad, int lane, int row, int M,
                                              int N, int n0, float rs,
                                              const float* __restrict__ r_row, void* Y,
                                              uint64_t* acc_empty) {
  uint32_t pk[BN / 2];
#pragma unroll
  for (int c0 = 0; c0 < BN; c0 += 32) {
    uint32_t v[32];
    tmem_ld32(tmem + ((uint32_t)(quad * 32) << 16) + c0, v);
#pragma unroll
    for (int k = 0; k < 32; k += 2) {
      float f0 = __fmul_rn(__uint_as_float(v[k]), rs);
      float f1 = __fmul_rn(__uint_as_float(v[k + 1]), rs);
      if constexpr (ROWF) {
        f0 = __fmul_rn(f0, __ldg(r_row + n0 + c0 + k));
        f1 = __fmul_rn(f1, __ldg(r_row + n0 + c0 + k + 1));
      }
      __nv_bfloat162 p2 = __floats2bfloat162_rn(f0, f1);
      pk[(c0 + k) / 2] = *reinterpret_cast<uint32_t*>(&p2);
    }
  }
  fence_before_sync();
  __syncwarp();
  if (lane == 0) mbar_arrive(acc_empty);
  if (row < M) {
    uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(Y) + (size_t)row * N + n0);
#pragma unroll
    for (int q = 0; q < BN / 8; ++q)
      dst[q] = make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
  }
}

template <int FMT, int BN, int YT, int AR = BM>
__global__ void __launch_bounds__(NUM_THREADS, 1)
w4a4_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                 const uint8_t* __restrict__ sfA, const uint8_t* __restrict__ sfB,
                 const float* __restrict__ s_tok, const float* __restrict__ s_w,
                 const float* __restrict__ r_row, void* __restrict__ Y, int M, int N, int K) {
  using C = Cfg<FMT, BN, 0, AR>;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  // 1024-byte alignment for the 128-byte swizzle atoms
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  unsigned char* sA = smem;
  unsigned char* sB = sA + C::STAGES * C::A_BYTES;
  unsigned char* sSFA = sB + C::STAGES * C::B_BYTES;
  unsigned char* sSFB = sSFA + C::STAGES * C::SFA_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(sSFB + C::STAGES * C::SFB_BYTES);
  uint64_t* empty = full + C::STAGES;
  uint64_t* sfready = empty + C::STAGES;
  uint64_t* sffull = sfready + C::STAGES;   // scale atoms of the stage landed
  uint64_t* acc_full = sffull + C::STAGES;
  uint64_t* acc_empty = acc_full + 1;
  uint32_t* tmem_base_slot = reinterpret_cast<uint32_t*>(acc_empty + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_base_slot + 1);
  uint64_t* drain = acc_empty + 2;   // tensor-core work of the MMA and copier threads done

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
  }
  const int tiles_m = (M + BM - 1) / BM, tiles_n = N / BN;
  const int num_tiles = tiles_m * tiles_n;
  const bool nfast = M > N;   // tile order (tile_mn)
  const int KT = K / BK;
  const int S4 = (K / C::G) / 4;  // scale atoms along K per 128-row block

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
      mbar_init(&sfready[s], COPIERS);
      mbar_init(&sffull[s], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, 4);
    mbar_init(drain, 1 + COPIERS);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_base_slot)),
                 "r"((uint32_t)C::TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tmem = *tmem_base_slot;
  // Programmatic dependent launch: the weight operand (B and its scales) is
  // never written by the kernel launched just before a GEMM (the activation
  // quantiser), so the producer fetches the first stages' weights before the
  // dependency wait; the activations, the per-token scales and the output
  // are touched only after it (producer and epilogue roles).
  pdl_trigger();

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      // the scale atoms of a stage complete on sffull (issued first, so the
      // copier warps move them into tensor memory while the A / B tiles are
      // still landing), the code tiles on full
      constexpr uint32_t TX_AB = C::A_BYTES + C::B_BYTES, TX_SF = C::SFA_BYTES + C::SFB_BYTES;
      auto load_b = [&](int stage, int n0, int kt) {
#pragma unroll
        for (int g = 0; g < BN / 128; ++g)
          bulk_load(sSFB + stage * C::SFB_BYTES + g * C::SF_ATOMS * 512,
                    sfB + ((size_t)(n0 / 128 + g) * S4 + (size_t)kt * C::SF_ATOMS) * 512,
                    C::SF_ATOMS * 512, &sffull[stage]);
        tma_load_2d(sB + stage * C::B_BYTES, &tmB, &full[stage], kt * BKB, n0);
      };
      // weights of the first stages ahead of the dependency wait
      const int pre = (blockIdx.x < num_tiles) ? (KT < C::STAGES ? KT : C::STAGES) : 0;
      for (int kt = 0; kt < pre; ++kt) {
        mbar_expect_tx(&sffull[kt], TX_SF);
        mbar_expect_tx(&full[kt], TX_AB);
        load_b(kt, tile_mn(blockIdx.x, tiles_m, tiles_n, nfast).y * BN, kt);
      }
      pdl_wait();
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      bool first = true;
      int issued = 0;   // stages whose loads were all issued
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x, first = false) {
        const int2 tt = tile_mn(tile, tiles_m, tiles_n, nfast);
        const int tm = tt.x, tn = tt.y;
        const int m0 = tm * BM, n0 = tn * BN;
        for (int kt = 0; kt < KT; ++kt) {
          if (!(first && kt < pre)) {
            if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag)) { ok = false; break; }
            mbar_expect_tx(&sffull[stage], TX_SF);
            mbar_expect_tx(&full[stage], TX_AB);
            load_b(stage, n0, kt);
          }
          bulk_load(sSFA + stage * C::SFA_BYTES,
                    sfA + ((size_t)(m0 / 128) * S4 + (size_t)kt * C::SF_ATOMS) * 512,
                    C::SFA_BYTES, &sffull[stage]);
          tma_load_2d(sA + stage * C::A_BYTES, &tmA, &full[stage], kt * BKB, m0);
          ++issued;
          if (++stage == C::STAGES) { stage = 0; phase ^= 1; }
        }
      }
      // every stage consumed by the MMAs (normal end) ...
      const int stage_end = stage;
      const uint32_t phase_end = phase;
      if (ok) {
        for (int s = 0; s < C::STAGES; ++s) {
          if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag)) break;
          if (++stage == C::STAGES) { stage = 0; phase ^= 1; }
        }
      }
      // ... and, whatever happened, every issued load landed before the CTA
      // may exit (an expired wait leaves stages unconsumed)
      drain_loads<C::STAGES>(full, sffull, stage_end, phase_end, issued);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      bool ok = true;
      const uint32_t idesc0 = idesc_fp4(BN, FMT != NVFP4);
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x, ++it) {
        if (!mbar_wait(acc_empty, (it & 1) ^ 1, abort_flag)) break;
        fence_after_sync();
        for (int kt = 0; kt < KT; ++kt) {
          if (!mbar_wait(&full[stage], phase, abort_flag) ||
              !mbar_wait(&sfready[stage], phase, abort_flag)) { ok = false; break; }
          fence_after_sync();
          const uint32_t a_base = smem_u32(sA + stage * C::A_BYTES);
          const uint32_t b_base = smem_u32(sB + stage * C::B_BYTES);
          const uint32_t sfa0 = C::SF_BASE + stage * C::SF_COLS;
          const uint32_t sfb0 = sfa0 + 4 * C::SF_ATOMS;
#pragma unroll
          for (int kk = 0; kk < C::K_STEPS; ++kk) {
            // K = 64 four-bit elements = 32 bytes inside the 128-byte swizzle row
            const uint64_t ad = smem_desc(a_base + kk * 32, 16, 1024, LAYOUT_SW128);
            const uint64_t bd = smem_desc(b_base + kk * 32, 16, 1024, LAYOUT_SW128);
            uint32_t sf_id, sfa_col, sfb_col;
            if constexpr (FMT == NVFP4) {  // 4 scales per row per MMA: one column each
              sf_id = 0;
              sfa_col = sfa0 + 4 * kk;
              sfb_col = sfb0 + 4 * (BN / 128) * kk;
            } else {                        // 2 scales per row per MMA: half a column
              sf_id = 2 * (kk & 1);
              sfa_col = sfa0 + 4 * (kk >> 1);
              sfb_col = sfb0 + 4 * (BN / 128) * (kk >> 1);
            }
            const uint32_t idesc = idesc0 | (sf_id << 29) | (sf_id << 4);
            mma_fp4<FMT>(tmem, ad, bd, idesc, (kt > 0 || kk > 0) ? 1u : 0u,
                         (tmem + sfa_col) | (sf_id << 30), (tmem + sfb_col) | (sf_id << 30));
          }
          mma_commit(&empty[stage]);
          if (++stage == C::STAGES) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
        mma_commit(acc_full);
      }
      // the MMAs issued so far have completed before the CTA may exit
      mma_commit(drain);
      mbar_drain(drain, 0);
    }
  } else if (warp >= FIRST_COPIER && warp < FIRST_COPIER + COPIERS) {
    // ------------------------------------------------------------ scale copiers
    // atom a of a stage (SFA atoms first, then the SFB groups) goes to copier
    // a % COPIERS; each copier commits to the stage's sfready barrier
    if (lane == 0) {
      const int me = warp - FIRST_COPIER;
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        for (int kt = 0; kt < KT; ++kt) {
          if (!mbar_wait(&sffull[stage], phase, abort_flag)) { ok = false; break; }
          fence_after_sync();
          const uint32_t sfa_base = smem_u32(sSFA + stage * C::SFA_BYTES);
          const uint32_t sfb_base = smem_u32(sSFB + stage * C::SFB_BYTES);
          const uint32_t sfa0 = C::SF_BASE + stage * C::SF_COLS;
          const uint32_t sfb0 = sfa0 + 4 * C::SF_ATOMS;
          for (int a = me; a < C::SF_ATOMS * (1 + BN / 128); a += COPIERS) {
            if (a < C::SF_ATOMS) {
              tmem_cp_32x128b_x4(tmem + sfa0 + 4 * a, smem_desc(sfa_base + a * 512, 0, 128, LAYOUT_NONE));
            } else {
              const int g = (a - C::SF_ATOMS) / C::SF_ATOMS, j = (a - C::SF_ATOMS) % C::SF_ATOMS;
              tmem_cp_32x128b_x4(tmem + sfb0 + 4 * (BN / 128) * j + 4 * g,
                                 smem_desc(sfb_base + (g * C::SF_ATOMS + j) * 512, 0, 128,
                                           LAYOUT_NONE));
            }
          }
          mma_commit(&sfready[stage]);
          if (++stage == C::STAGES) { stage = 0; phase ^= 1; }
        }
      }
      mma_commit(drain);   // this copier's scale copies have completed
      mbar_drain(drain, 0);
    }
  } else if (warp >= 2 && warp <= 5) {
    // ------------------------------------------------------------ epilogue
    const int quad = warp & 3;                 // tensor-memory lane quadrant of this warp
    pdl_wait();
    const float sw = (FMT == NVFP4 && s_w) ? *s_w : 1.0f;
    int it = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++it) {
      const int2 tt = tile_mn(tile, tiles_m, tiles_n, nfast);
        const int tm = tt.x, tn = tt.y;
      const int row = tm * BM + quad * 32 + lane;
      const int n0 = tn * BN;
      // this row's scale is loaded before the accumulator wait, off the
      // critical path of the hand-off back to the MMA warp
      float rs = sw;
      if (FMT == NVFP4 && s_tok && row < M) rs = __fmul_rn(s_tok[row], sw);
      // one lane waits, the warp follows (the tensor-memory loads below are
      // warp-collective and must never run in a partial warp)
      int ok = 1;
      if (lane == 0) ok = mbar_wait(acc_full, it & 1, abort_flag) ? 1 : 0;
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      fence_after_sync();
      if constexpr (YT == 1) {
        if (r_row)
          epilogue_bf16<BN, true>(tmem, quad, lane, row, M, N, n0, rs, r_row, Y, acc_empty);
        else
          epilogue_bf16<BN, false>(tmem, quad, lane, row, M, N, n0, rs, r_row, Y, acc_empty);
      } else {
#pragma unroll 1
        for (int c0 = 0; c0 < BN; c0 += 32) {
          uint32_t v[32];
          tmem_ld32(tmem + ((uint32_t)(quad * 32) << 16) + c0, v);
          if (c0 + 32 == BN) {  // accumulator fully read: hand it back to the MMA warp
            fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(acc_empty);
          }
          if (row < M) {
            float f[32];
#pragma unroll
            for (int k = 0; k < 32; ++k) {
              f[k] = __fmul_rn(__uint_as_float(v[k]), rs);
              if (r_row) f[k] = __fmul_rn(f[k], __ldg(r_row + n0 + c0 + k));
            }
            float4* dst = reinterpret_cast<float4*>(reinterpret_cast<float*>(Y) +
                                                    (size_t)row * N + n0 + c0);
#pragma unroll
            for (int q = 0; q < 8; ++q)
              dst[q] = make_float4(f[4 * q], f[4 * q + 1], f[4 * q + 2], f[4 * q + 3]);
          }
        }
      }
    }
  }

  fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    fence_after_sync();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"((uint32_t)C::TMEM_COLS)
                 : "memory");
  }
}

// ---------------------------------------------------------------------------
// Split-K variant for problems with few output tiles (small M): the S CTAs
// of a thread-block cluster compute K-slices of the same 128 x 128 tile with
// the same TMA / scale-copy / tcgen05 pipeline.  Each CTA owns one column
// slice of the tile: while draining its fp32 partial tile from tensor memory
// it stores every slice straight into the owner's shared memory (DSMEM);
// after one cluster barrier each CTA sums its S partial slices from local
// shared memory (in rank order), applies the epilogue scales and stores.
// No global workspace.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_barrier() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;"
               ::: "memory");
}
// Store four floats at a shared-memory offset of CTA `rank` of the cluster
// (16-byte aligned).  Ordered before the peers' reads by the cluster barrier
// (release / acquire).
__device__ __forceinline__ void st_dsmem_f32x4(uint32_t local_addr, uint32_t rank, uint32_t a,
                                               uint32_t b, uint32_t c, uint32_t d) {
  uint32_t ra;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"(local_addr), "r"(rank));
  asm volatile("st.shared::cluster.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(ra), "r"(a), "r"(b),
               "r"(c), "r"(d)
               : "memory");
}

// A float of CTA `rank`'s shared memory (ordered after the peer's write by a
// cluster barrier).
__device__ __forceinline__ float ld_dsmem_f32(const float* local, uint32_t rank) {
  uint32_t a = (uint32_t)__cvta_generic_to_shared(local), ra;
  float v;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"(a), "r"(rank));
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(ra) : "memory");
  return v;
}

constexpr int SK_BN = 128;
// partial slices received from the S CTAs of the cluster: [S][BM][BN / S] floats
constexpr int SK_PART_BYTES = BM * SK_BN * 4;

// FUSED (NVFP4, bf16 activations): the activation rescale and quantisation
// run inside the kernel.  Each CTA takes the per-token maximum of |x c| over
// its K slice, the cluster combines them over DSMEM into s_tok, and warps
// 2..5 write the A operand tiles (128-byte swizzled E2M1 codes) and the A
// scale atoms (UE4M3) of every k-tile of the slice straight into the stage
// buffers, with the arithmetic of the standalone activation quantiser; TMA
// brings only the weights.  Requires kt_per_slice <= STAGES.
template <int FMT, int YT, bool FUSED, int AR = BM>
__global__ void __launch_bounds__(NUM_THREADS, 1)
w4a4_gemm_splitk_kernel(const __grid_constant__ CUtensorMap tmA,
                        const __grid_constant__ CUtensorMap tmB, const uint8_t* __restrict__ sfA,
                        const uint8_t* __restrict__ sfB, const float* __restrict__ s_tok,
                        const float* __restrict__ s_w, const float* __restrict__ r_row,
                        void* __restrict__ Y, int M, int N, int K, int kt_per_slice,
                        int a_rows, const __nv_bfloat16* __restrict__ X,
                        const float* __restrict__ cvec) {
  constexpr int BN = SK_BN;
  using C = Cfg<FMT, BN, SK_PART_BYTES, AR>;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  unsigned char* sA = smem;
  unsigned char* sB = sA + C::STAGES * C::A_BYTES;
  unsigned char* sSFA = sB + C::STAGES * C::B_BYTES;
  unsigned char* sSFB = sSFA + C::STAGES * C::SFA_BYTES;
  float* part = reinterpret_cast<float*>(sSFB + C::STAGES * C::SFB_BYTES);
  uint64_t* full = reinterpret_cast<uint64_t*>(reinterpret_cast<unsigned char*>(part) + SK_PART_BYTES);
  uint64_t* empty = full + C::STAGES;
  uint64_t* sfready = empty + C::STAGES;
  uint64_t* acc_full = sfready + C::STAGES;
  uint32_t* tmem_base_slot = reinterpret_cast<uint32_t*>(acc_full + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_base_slot + 1);
  uint64_t* drain = acc_full + 2;  // tensor-core work of the MMA and copier threads done
  __shared__ float s_rs[BM];       // per-row output scale
  __shared__ float s_rr[SK_BN];    // per-output-column factor of this tile
  __shared__ float s_pamax[FUSED ? BM : 1];   // FUSED: this CTA's row maxima of |x c|
  __shared__ float s_stok[FUSED ? BM : 1];    // FUSED: per-token scale of the m-tile

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
  }
  const uint32_t rank = cluster_rank(), S = gridDim.x;
  const int n0 = blockIdx.y * BN, m0 = blockIdx.z * BM;
  const int kt0 = (int)rank * kt_per_slice;
  const int S4 = (K / C::G) / 4;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      // FUSED: the weights' TMA plus one arrival per A-producer warp
      mbar_init(&full[s], FUSED ? 5 : 1);
      mbar_init(&empty[s], 1);
      mbar_init(&sfready[s], COPIERS);
    }
    mbar_init(acc_full, 1);
    mbar_init(drain, 1 + COPIERS);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_base_slot)),
                 "r"((uint32_t)C::TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tmem = *tmem_base_slot;
  pdl_trigger();   // weights are fetched before the dependency wait (see the 1-CTA kernel)

  if constexpr (FUSED) {
    // weights of every k-tile of the slice first (they do not depend on X)
    if (warp == 0 && lane == 0) {
      for (int kt = 0; kt < kt_per_slice; ++kt) {
        mbar_expect_tx(&full[kt], C::B_BYTES + C::SFB_BYTES);
        tma_load_2d(sB + kt * C::B_BYTES, &tmB, &full[kt], (kt0 + kt) * BKB, n0);
        bulk_load(sSFB + kt * C::SFB_BYTES,
                  sfB + ((size_t)(n0 / 128) * S4 + (size_t)(kt0 + kt) * C::SF_ATOMS) * 512,
                  C::SFB_BYTES, &full[kt]);
      }
    }
    pdl_wait();   // X and c may come from the kernel launched just before
    // row maxima of |x c| over this CTA's K slice: one warp per row, lanes
    // over 8-element pieces
    const int rows_here = (M - m0) < a_rows ? (M - m0) : a_rows;
    const int64_t k_lo = (int64_t)kt0 * BK, k_n = (int64_t)kt_per_slice * BK;
    for (int r = warp; r < a_rows; r += NUM_THREADS / 32) {
      float a = 0.0f;
      if (r < rows_here) {
        const __nv_bfloat16* xr = X + (size_t)(m0 + r) * K + k_lo;
        for (int64_t p = lane * 8; p < k_n; p += 256) {
          float x[8];
          bf16x8_to_f32(*reinterpret_cast<const uint4*>(xr + p), x);
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const float cv = cvec ? __ldg(cvec + k_lo + p + k) : 1.0f;
            a = fmaxf(a, fabsf(__fmul_rn(x[k], cv)));
          }
        }
      }
#pragma unroll
      for (int o = 16; o; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
      if (lane == 0) s_pamax[r] = a;
    }
    cluster_barrier();   // every CTA's partial maxima are visible to the cluster
    if ((int)threadIdx.x < a_rows) {
      float a = 0.0f;
      for (uint32_t q = 0; q < S; ++q) a = fmaxf(a, ld_dsmem_f32(&s_pamax[threadIdx.x], q));
      s_stok[threadIdx.x] = __fdiv_rn(a, 2688.0f);
    }
    __syncthreads();
  }

  if (warp == 0) {
    if (lane == 0 && !FUSED) {
      // A tiles carry only the a_rows rows that exist (rounded up to 16): the
      // MMA's other rows feed accumulator rows that are never stored
      const uint32_t tx = C::STAGE_BYTES - (AR - a_rows) * BKB;
      auto load_b = [&](int stage, int kt) {
        tma_load_2d(sB + stage * C::B_BYTES, &tmB, &full[stage], (kt0 + kt) * BKB, n0);
        bulk_load(sSFB + stage * C::SFB_BYTES,
                  sfB + ((size_t)(n0 / 128) * S4 + (size_t)(kt0 + kt) * C::SF_ATOMS) * 512,
                  C::SFB_BYTES, &full[stage]);
      };
      const int pre = kt_per_slice < C::STAGES ? kt_per_slice : C::STAGES;
      for (int kt = 0; kt < pre; ++kt) {   // weights ahead of the dependency wait
        mbar_expect_tx(&full[kt], tx);
        load_b(kt, kt);
      }
      pdl_wait();
      int stage = 0;
      uint32_t phase = 0;
      int issued = 0;
      for (int kt = 0; kt < kt_per_slice; ++kt) {
        if (kt >= pre) {
          if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag)) break;
          mbar_expect_tx(&full[stage], tx);
          load_b(stage, kt);
        }
        tma_load_2d(sA + stage * C::A_BYTES, &tmA, &full[stage], (kt0 + kt) * BKB, m0);
        bulk_load(sSFA + stage * C::SFA_BYTES,
                  sfA + ((size_t)(m0 / 128) * S4 + (size_t)(kt0 + kt) * C::SF_ATOMS) * 512,
                  C::SFA_BYTES, &full[stage]);
        ++issued;
        if (++stage == C::STAGES) { stage = 0; phase ^= 1; }
      }
      const int stage_end = stage;
      const uint32_t phase_end = phase;
      for (int s = 0; s < C::STAGES; ++s) {  // every issued stage consumed (normal end)
        if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag)) break;
        if (++stage == C::STAGES) { stage = 0; phase ^= 1; }
      }
      // every issued load landed before the CTA may exit
      drain_loads<C::STAGES>(full, nullptr, stage_end, phase_end, issued);
    }
    if (FUSED && lane == 0) {
      // the weights of every k-tile were issued up front; full[kt] also
      // counts the A-producer warps, which never wait on a limit
      for (int kt = 0; kt < kt_per_slice; ++kt) mbar_drain(&full[kt], 0);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      const uint32_t idesc0 = idesc_fp4(BN, FMT != NVFP4);
      for (int kt = 0; kt < kt_per_slice; ++kt) {
        if (!mbar_wait(&full[stage], phase, abort_flag) ||
            !mbar_wait(&sfready[stage], phase, abort_flag)) { ok = false; break; }
        fence_after_sync();
        const uint32_t a_base = smem_u32(sA + stage * C::A_BYTES);
        const uint32_t b_base = smem_u32(sB + stage * C::B_BYTES);
        const uint32_t sfa0 = C::SF_BASE + stage * C::SF_COLS;
        const uint32_t sfb0 = sfa0 + 4 * C::SF_ATOMS;
#pragma unroll
        for (int kk = 0; kk < C::K_STEPS; ++kk) {
          const uint64_t ad = smem_desc(a_base + kk * 32, 16, 1024, LAYOUT_SW128);
          const uint64_t bd = smem_desc(b_base + kk * 32, 16, 1024, LAYOUT_SW128);
          uint32_t sf_id, sfa_col, sfb_col;
          if constexpr (FMT == NVFP4) {
            sf_id = 0;
            sfa_col = sfa0 + 4 * kk;
            sfb_col = sfb0 + 4 * kk;
          } else {
            sf_id = 2 * (kk & 1);
            sfa_col = sfa0 + 4 * (kk >> 1);
            sfb_col = sfb0 + 4 * (kk >> 1);
          }
          const uint32_t idesc = idesc0 | (sf_id << 29) | (sf_id << 4);
          mma_fp4<FMT>(tmem, ad, bd, idesc, (kt > 0 || kk > 0) ? 1u : 0u,
                       (tmem + sfa_col) | (sf_id << 30), (tmem + sfb_col) | (sf_id << 30));
        }
        mma_commit(&empty[stage]);
        if (++stage == C::STAGES) { stage = 0; phase ^= 1; }
      }
      if (ok) mma_commit(acc_full);
      mma_commit(drain);   // the MMAs issued so far have completed before exit
      mbar_drain(drain, 0);
    }
  } else {
    // warps 2..5 and the copier warps 6..9 drain the partial tile after the
    // mainloop, each pair of warps one TMEM lane quadrant, half the columns each
    const bool copier = warp >= FIRST_COPIER;
    if (copier && lane == 0) {
      const int me = warp - FIRST_COPIER;
      int stage = 0;
      uint32_t phase = 0;
      for (int kt = 0; kt < kt_per_slice; ++kt) {
        if (!mbar_wait(&full[stage], phase, abort_flag)) break;
        fence_after_sync();
        const uint32_t sfa_base = smem_u32(sSFA + stage * C::SFA_BYTES);
        const uint32_t sfb_base = smem_u32(sSFB + stage * C::SFB_BYTES);
        const uint32_t sfa0 = C::SF_BASE + stage * C::SF_COLS;
        const uint32_t sfb0 = sfa0 + 4 * C::SF_ATOMS;
        for (int a = me; a < 2 * C::SF_ATOMS; a += COPIERS) {
          if (a < C::SF_ATOMS)
            tmem_cp_32x128b_x4(tmem + sfa0 + 4 * a, smem_desc(sfa_base + a * 512, 0, 128, LAYOUT_NONE));
          else
            tmem_cp_32x128b_x4(tmem + sfb0 + 4 * (a - C::SF_ATOMS),
                               smem_desc(sfb_base + (a - C::SF_ATOMS) * 512, 0, 128, LAYOUT_NONE));
        }
        mma_commit(&sfready[stage]);
        if (++stage == C::STAGES) { stage = 0; phase ^= 1; }
      }
      mma_commit(drain);   // this copier's scale copies have completed
      mbar_drain(drain, 0);
    }
    __syncwarp();
    const int quad = warp & 3;
    if (FUSED && !copier) {
      // A producers: codes and scale bytes of every (row, 16-block) of every
      // k-tile of the slice, rows past M as zeros
      const int pt = (warp - 2) * 32 + lane;            // 0..127
      const int rows_here = (M - m0) < a_rows ? (M - m0) : a_rows;
      for (int kt = 0; kt < kt_per_slice; ++kt) {
        unsigned char* tA = sA + kt * C::A_BYTES;
        unsigned char* tS = sSFA + kt * C::SFA_BYTES;
        const int64_t kb = (int64_t)(kt0 + kt) * BK;
        for (int idx = pt; idx < a_rows * (BK / 16); idx += 128) {
          const int r = idx / (BK / 16), j = idx % (BK / 16);
          uint32_t byte = 0u;
          uint2 codes = make_uint2(0u, 0u);
          if (r < rows_here) {
            const float st = s_stok[r];
            const __nv_bfloat16* xr = X + (size_t)(m0 + r) * K + kb + j * 16;
            float xt[16];
            bf16x8_to_f32(reinterpret_cast<const uint4*>(xr)[0], xt);
            bf16x8_to_f32(reinterpret_cast<const uint4*>(xr)[1], xt + 8);
            float ab = 0.0f;
#pragma unroll
            for (int k = 0; k < 16; ++k) {
              const float cv = cvec ? __ldg(cvec + kb + j * 16 + k) : 1.0f;
              xt[k] = __fmul_rn(xt[k], cv);
              ab = fmaxf(ab, fabsf(xt[k]));
            }
            byte = st > 0.0f ? ue4m3_rn(__fdiv_rn(ab, __fmul_rn(6.0f, st))) : 0u;
            const float sblk = __fmul_rn(ue4m3_value(byte), st);
            if (sblk != 0.0f) {
              const float inv = __frcp_rn(sblk);
#pragma unroll
              for (int k = 0; k < 16; ++k) xt[k] = __fmul_rn(xt[k], inv);
              codes = make_uint2(e2m1x8(xt), e2m1x8(xt + 8));
            }
          }
          // 8 code bytes at byte j * 8 of the row, 16-byte chunks swizzled by row
          *reinterpret_cast<uint2*>(tA + r * 128 + ((((j >> 1) ^ (r & 7))) << 4) + (j & 1) * 8) =
              codes;
          tS[(j >> 2) * 512 + (r & 31) * 16 + ((r & 127) >> 5) * 4 + (j & 3)] = (uint8_t)byte;
        }
        // generic-proxy writes -> visible to the tensor core and tcgen05.cp
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncwarp();
        if (lane == 0) mbar_arrive(&full[kt]);
      }
    }
    if (!copier) {
      // per-row scale and the tile's output-row factors, staged before the
      // accumulator wait so the reduction below reads shared memory only
      // (these warps pass the dependency wait before the output is written
      // by anyone: every thread writes it only after the cluster barrier)
      pdl_wait();
      const int rr = quad * 32 + lane;
      float rs = (FMT == NVFP4 && s_w) ? *s_w : 1.0f;
      if constexpr (FUSED) {
        if (m0 + rr < M && rr < a_rows) rs = __fmul_rn(s_stok[rr], rs);
      } else {
        if (FMT == NVFP4 && s_tok && m0 + rr < M) rs = __fmul_rn(s_tok[m0 + rr], rs);
      }
      s_rs[rr] = rs;
      s_rr[rr] = r_row ? __ldg(r_row + n0 + rr) : 1.0f;
    }
    // drain this CTA's partial tile (rows that exist) straight into the
    // shared memory of the CTA that reduces each column slice: owner q keeps
    // slice [q * cols, (q + 1) * cols) of every rank, at part[rank][row][.]
    const int cols = BN / (int)S;
    const int c_lo = copier ? BN / 2 : 0;
    int ok = 1;
    if (lane == 0) ok = mbar_wait(acc_full, 0, abort_flag) ? 1 : 0;
    ok = __shfl_sync(0xffffffffu, ok, 0);
    if (ok && m0 + quad * 32 < M) {
      fence_after_sync();
      const int row = quad * 32 + lane;
      const uint32_t mine = smem_u32(part + ((size_t)rank * BM + row) * cols);
#pragma unroll 1
      for (int c0 = c_lo; c0 < c_lo + BN / 2; c0 += 32) {
        uint32_t v[32];
        tmem_ld32(tmem + ((uint32_t)(quad * 32) << 16) + c0, v);
#pragma unroll
        for (int kk = 0; kk < 32; kk += 4) {
          const int c = c0 + kk, q = c / cols;
          st_dsmem_f32x4(mine + (uint32_t)(c - q * cols) * 4, (uint32_t)q, v[kk], v[kk + 1],
                         v[kk + 2], v[kk + 3]);
        }
      }
    }
  }

  fence_before_sync();
  cluster_barrier();   // every partial slice has landed in its owner's shared memory
  {
    // this CTA owns columns [rank * cols, (rank + 1) * cols) of the tile:
    // sum the S partial slices (local shared memory, rank order), scale, store
    const int cols = BN / (int)S, c4 = cols / 4, c_begin = (int)rank * cols;
    const int rows = (M - m0) < BM ? (M - m0) : BM;
    const int total = rows * c4;
    for (int idx = threadIdx.x; idx < total; idx += NUM_THREADS) {
      const int r = idx / c4, cc = (idx % c4) * 4, c = c_begin + cc;
      float4 acc = *reinterpret_cast<const float4*>(part + (size_t)r * cols + cc);
      for (uint32_t q = 1; q < S; ++q) {
        const float4 p = *reinterpret_cast<const float4*>(part + ((size_t)q * BM + r) * cols + cc);
        acc.x += p.x; acc.y += p.y; acc.z += p.z; acc.w += p.w;
      }
      const float rs = s_rs[r];
      float f[4] = {__fmul_rn(acc.x, rs), __fmul_rn(acc.y, rs), __fmul_rn(acc.z, rs),
                    __fmul_rn(acc.w, rs)};
      if (r_row) {
#pragma unroll
        for (int q = 0; q < 4; ++q) f[q] = __fmul_rn(f[q], s_rr[c + q]);
      }
      const size_t o = (size_t)(m0 + r) * N + n0 + c;
      if constexpr (YT == 1) {
        __nv_bfloat162 lo = __floats2bfloat162_rn(f[0], f[1]), hi = __floats2bfloat162_rn(f[2], f[3]);
        *reinterpret_cast<uint2*>(reinterpret_cast<__nv_bfloat16*>(Y) + o) =
            make_uint2(*reinterpret_cast<uint32_t*>(&lo), *reinterpret_cast<uint32_t*>(&hi));
      } else {
        *reinterpret_cast<float4*>(reinterpret_cast<float*>(Y) + o) = make_float4(f[0], f[1], f[2], f[3]);
      }
    }
  }
  // no peer touches this CTA's shared memory after the barrier above
  __syncthreads();
  if (warp == 1) {
    fence_after_sync();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"((uint32_t)C::TMEM_COLS)
                 : "memory");
  }
}

// ---------------------------------------------------------------------------
// Paired-SM variant for large problems: one 256 x 256 output tile per
// cluster of two CTAs (one per SM), tcgen05.mma.cta_group::2.  Each CTA
// loads its own 128 rows of A, its own 128 columns of B, the block scales
// of its A rows and all 256 B scale rows; the even CTA ("leader") issues the
// scale copies and the MMAs for both, which read A and the scale copies from
// each CTA's own shared memory, B from both, and accumulate 128 x 256 in each
// CTA's tensor memory.  Per 256 x 256 tile the pair reads 512 operand rows
// from L2 instead of the 768 that two 128 x 256 tiles need.
//   warp 0      TMA producer (both CTAs; completions counted on the leader's
//               barrier, the cta_group::2 form of the tensor copy, no multicast)
//   warp 1      tensor-memory allocation (both); MMA issuer (leader)
//   warps 2..5  epilogue (both), each CTA its own 128 rows
//   warps 6..9  scale copiers (leader): tcgen05.cp.cta_group::2, each a
//               quarter of every stage's atoms
// ---------------------------------------------------------------------------
namespace pair {
constexpr int BN = 256;                             // output columns per tile
template <int FMT>
struct Cfg2 {
  static constexpr int G = (FMT == NVFP4) ? 16 : 32;
  static constexpr int SF_ATOMS = (BK / G) / 4;     // 512-byte atoms per 128 rows per k-tile
  static constexpr int A_BYTES = BM * BKB;          // own 128 rows
  static constexpr int B_BYTES = 128 * BKB;         // own 128 columns
  static constexpr int SFA_BYTES = SF_ATOMS * 512;
  static constexpr int SFB_BYTES = 2 * SF_ATOMS * 512;  // all 256 scale rows
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES;
  static constexpr int STAGES = (227 * 1024 - 1024 - 256) / STAGE_BYTES;
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 + 256;
  static constexpr int SF_COLS = 4 * SF_ATOMS * 3;  // SFA (one group) + SFB (two groups)
  static constexpr int SF_BASE = BN;
  static constexpr int TMEM_COLS = 512;
  static constexpr int K_STEPS = BK / 64;
  static_assert(SF_BASE + STAGES * SF_COLS <= TMEM_COLS, "tensor memory budget");
  static_assert(4 * STAGES * 8 + 40 <= 256, "barrier area");
  static_assert(STAGES >= 3, "pipeline depth");
};

__device__ __forceinline__ uint32_t mapa(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}
// Tensor copy into this CTA's shared memory whose completion is counted on
// the pair leader's barrier (cluster address `bar`).
__device__ __forceinline__ void tma_load_2d_pair(void* dst, const CUtensorMap* map, uint32_t bar,
                                                 int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
      "l"((uint64_t)map), "r"(bar), "r"(x), "r"(y)
      : "memory");
}
__device__ __forceinline__ void tmem_cp_pair(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::2.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc)
               : "memory");
}
template <int FMT>
__device__ __forceinline__ void mma_pair(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                         uint32_t idesc, uint32_t accumulate, uint32_t tsfa,
                                         uint32_t tsfb) {
  if constexpr (FMT == NVFP4) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t}"
        ::"r"(tmem_d), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(tsfa), "r"(tsfb)
        : "memory");
  } else {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::mxf4.block_scale.block32 [%0], %1, %2, %3, [%5], [%6], p;\n\t}"
        ::"r"(tmem_d), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(tsfa), "r"(tsfb)
        : "memory");
  }
}
// Arrive on the barrier at the same offset in both CTAs of the pair once the
// leader's earlier tcgen05 operations have completed.
__device__ __forceinline__ void commit_both(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;"
      ::"r"(smem_u32(bar)), "h"((uint16_t)0x3)
      : "memory");
}
// Arrive on the leader's own barrier once its earlier tcgen05 operations completed.
__device__ __forceinline__ void commit_leader(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}
__device__ __forceinline__ void arrive_remote(uint32_t cluster_bar) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_bar)
               : "memory");
}
__device__ __forceinline__ bool try_wait_cluster(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity) : "memory");
  return ok != 0;
}
// Bounded wait with cluster-scope acquire (barriers that receive arrivals
// from the other CTA of the pair).
__device__ __noinline__ bool wait_cluster(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
  if (try_wait_cluster(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  const uint64_t lim = *reinterpret_cast<volatile unsigned long long*>(&g_dq_wait_limit_ns);
  while (true) {
    if (try_wait_cluster(bar, parity)) return true;
    if (*abort_flag) return false;
    if (globaltimer() - t0 > lim) {
      *abort_flag = 1;
      atomicExch(&g_dq_device_error, DQ_ERR_DEVICE_TIMEOUT);
      return false;
    }
  }
}
// Instruction descriptor: E2M1 A and B, K-major, M = 256 (the pair), N = 256.
__host__ __device__ constexpr uint32_t idesc_pair(bool e8m0_scales) {
  return (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) | ((e8m0_scales ? 1u : 0u) << 23) |
         ((uint32_t)(256 >> 4) << 24);
}
}  // namespace pair

template <int FMT, int YT>
__global__ void __launch_bounds__(NUM_THREADS, 1)
w4a4_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                      const __grid_constant__ CUtensorMap tmSFA,
                      const __grid_constant__ CUtensorMap tmSFB, const float* __restrict__ s_tok,
                      const float* __restrict__ s_w, const float* __restrict__ r_row,
                      void* __restrict__ Y, int M, int N, int K) {
  using C = pair::Cfg2<FMT>;
  constexpr int BN = pair::BN;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  unsigned char* sA = smem;
  unsigned char* sB = sA + C::STAGES * C::A_BYTES;
  unsigned char* sSFA = sB + C::STAGES * C::B_BYTES;
  unsigned char* sSFB = sSFA + C::STAGES * C::SFA_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(sSFB + C::STAGES * C::SFB_BYTES);
  uint64_t* empty = full + C::STAGES;
  uint64_t* sfready = empty + C::STAGES;
  uint64_t* acc_full = sfready + C::STAGES;
  uint64_t* acc_empty = acc_full + 1;
  uint32_t* tmem_base_slot = reinterpret_cast<uint32_t*>(acc_empty + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_base_slot + 1);
  uint64_t* drain = acc_empty + 2;   // leader: its tensor-core work done

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();            // 0: leader, 1: peer
  const bool leader = rank == 0;
  const int pair_id = blockIdx.x >> 1, num_pairs = gridDim.x >> 1;
  const int tiles_m = (M + 255) / 256, tiles_n = N / BN;
  const int num_tiles = tiles_m * tiles_n;
  const bool nfast = M > N;   // tile order (tile_mn)
  const int KT = K / BK;
  const int S4 = (K / C::G) / 4;                   // scale atoms along K per 128-row block
  constexpr uint32_t TX = 2u * C::STAGE_BYTES;     // both CTAs' bytes per stage

  if (threadIdx.x == 0) {
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
    prefetch_tmap(&tmSFA);
    prefetch_tmap(&tmSFB);
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
      mbar_init(&sfready[s], COPIERS);
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, 8);                       // 4 epilogue warps in each CTA
    mbar_init(drain, 1 + COPIERS);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_base_slot)),
                 "r"((uint32_t)C::TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  fence_before_sync();
  __syncthreads();
  cluster_barrier();   // both CTAs' barriers are initialised before any remote use
  fence_after_sync();
  const uint32_t tmem = *tmem_base_slot;
  pdl_trigger();   // weights are fetched before the dependency wait (see the 1-CTA kernel)

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      auto load_b = [&](int stage, int tn, int kt) {
        const uint32_t bar = pair::mapa(smem_u32(&full[stage]), 0);
        pair::tma_load_2d_pair(sB + stage * C::B_BYTES, &tmB, bar, kt * BKB, tn * BN + (int)rank * 128);
#pragma unroll
        for (int g = 0; g < 2; ++g)
          pair::tma_load_2d_pair(sSFB + stage * C::SFB_BYTES + g * C::SF_ATOMS * 512, &tmSFB, bar,
                                 0, 2 * ((tn * 2 + g) * S4 + kt * C::SF_ATOMS));
      };
      // weights of the first stages ahead of the dependency wait
      const int pre = (pair_id < num_tiles) ? (KT < C::STAGES ? KT : C::STAGES) : 0;
      for (int kt = 0; kt < pre; ++kt) {
        if (leader) mbar_expect_tx(&full[kt], TX);
        load_b(kt, tile_mn(pair_id, tiles_m, tiles_n, nfast).y, kt);
      }
      pdl_wait();
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      bool first = true;
      int issued = 0;
      for (int tile = pair_id; tile < num_tiles && ok; tile += num_pairs, first = false) {
        const int2 tt = tile_mn(tile, tiles_m, tiles_n, nfast);
        const int tm = tt.x, tn = tt.y;
        const int m_own = tm * 256 + (int)rank * 128;
        for (int kt = 0; kt < KT; ++kt) {
          const uint32_t bar = pair::mapa(smem_u32(&full[stage]), 0);
          if (!(first && kt < pre)) {
            // both producers see the same phases of their empty barriers (the
            // leader's commits arrive on both at once) and give up only on the
            // fixed limit, never on an abort flag: so the two CTAs always fill
            // the same stages, and the leader's barrier, which counts both
            // CTAs' bytes, completes for every stage either of them filled
            if (!mbar_wait_fixed(&empty[stage], phase ^ 1, abort_flag)) { ok = false; break; }
            if (leader) mbar_expect_tx(&full[stage], TX);
            load_b(stage, tn, kt);
          }
          pair::tma_load_2d_pair(sA + stage * C::A_BYTES, &tmA, bar, kt * BKB, m_own);
          // scale atoms as rows of 256 bytes: atom a of row block rb is rows 2a, 2a + 1
          pair::tma_load_2d_pair(sSFA + stage * C::SFA_BYTES, &tmSFA, bar, 0,
                                 2 * ((m_own / 128) * S4 + kt * C::SF_ATOMS));
          ++issued;
          if (++stage == C::STAGES) { stage = 0; phase ^= 1; }
        }
      }
      // the leader waits until both CTAs' loads of every filled stage have
      // landed; the peer leaves only after the cluster barrier at the end
      if (leader) drain_loads<C::STAGES>(full, nullptr, stage, phase, issued);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (leader)
    if (leader && lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      bool ok = true;
      const uint32_t idesc0 = pair::idesc_pair(FMT != NVFP4);
      for (int tile = pair_id; tile < num_tiles && ok; tile += num_pairs, ++it) {
        if (!pair::wait_cluster(acc_empty, (it & 1) ^ 1, abort_flag)) break;
        fence_after_sync();
        for (int kt = 0; kt < KT; ++kt) {
          if (!mbar_wait(&full[stage], phase, abort_flag) ||
              !mbar_wait(&sfready[stage], phase, abort_flag)) { ok = false; break; }
          fence_after_sync();
          const uint32_t a_base = smem_u32(sA + stage * C::A_BYTES);
          const uint32_t b_base = smem_u32(sB + stage * C::B_BYTES);
          const uint32_t sfa0 = C::SF_BASE + stage * C::SF_COLS;
          const uint32_t sfb0 = sfa0 + 4 * C::SF_ATOMS;
#pragma unroll
          for (int kk = 0; kk < C::K_STEPS; ++kk) {
            const uint64_t ad = smem_desc(a_base + kk * 32, 16, 1024, LAYOUT_SW128);
            const uint64_t bd = smem_desc(b_base + kk * 32, 16, 1024, LAYOUT_SW128);
            uint32_t sf_id, sfa_col, sfb_col;
            if constexpr (FMT == NVFP4) {
              sf_id = 0;
              sfa_col = sfa0 + 4 * kk;
              sfb_col = sfb0 + 8 * kk;
            } else {
              sf_id = 2 * (kk & 1);
              sfa_col = sfa0 + 4 * (kk >> 1);
              sfb_col = sfb0 + 8 * (kk >> 1);
            }
            const uint32_t idesc = idesc0 | (sf_id << 29) | (sf_id << 4);
            pair::mma_pair<FMT>(tmem, ad, bd, idesc, (kt > 0 || kk > 0) ? 1u : 0u,
                                (tmem + sfa_col) | (sf_id << 30), (tmem + sfb_col) | (sf_id << 30));
          }
          pair::commit_both(&empty[stage]);
          if (++stage == C::STAGES) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
        pair::commit_both(acc_full);
      }
      // the MMAs issued into both CTAs' tensor memory have completed before
      // either CTA leaves (the peer waits at the cluster barrier)
      pair::commit_leader(drain);
      mbar_drain(drain, 0);
    }
  } else if (warp >= FIRST_COPIER && warp < FIRST_COPIER + COPIERS) {
    // ------------------------------------------------------------ scale copiers (leader)
    if (leader && lane == 0) {
      const int me = warp - FIRST_COPIER;
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int tile = pair_id; tile < num_tiles && ok; tile += num_pairs) {
        for (int kt = 0; kt < KT; ++kt) {
          if (!mbar_wait(&full[stage], phase, abort_flag)) { ok = false; break; }
          fence_after_sync();
          const uint32_t sfa_base = smem_u32(sSFA + stage * C::SFA_BYTES);
          const uint32_t sfb_base = smem_u32(sSFB + stage * C::SFB_BYTES);
          const uint32_t sfa0 = C::SF_BASE + stage * C::SF_COLS;
          const uint32_t sfb0 = sfa0 + 4 * C::SF_ATOMS;
          for (int a = me; a < 3 * C::SF_ATOMS; a += COPIERS) {
            if (a < C::SF_ATOMS) {
              pair::tmem_cp_pair(tmem + sfa0 + 4 * a, smem_desc(sfa_base + a * 512, 0, 128, LAYOUT_NONE));
            } else {
              const int g = (a - C::SF_ATOMS) / C::SF_ATOMS, j = (a - C::SF_ATOMS) % C::SF_ATOMS;
              pair::tmem_cp_pair(tmem + sfb0 + 8 * j + 4 * g,
                                 smem_desc(sfb_base + (g * C::SF_ATOMS + j) * 512, 0, 128,
                                           LAYOUT_NONE));
            }
          }
          pair::commit_leader(&sfready[stage]);
          if (++stage == C::STAGES) { stage = 0; phase ^= 1; }
        }
      }
      pair::commit_leader(drain);   // this copier's scale copies have completed
      mbar_drain(drain, 0);
    }
  } else if (warp >= 2 && warp <= 5) {
    // ------------------------------------------------------------ epilogue (both)
    const int quad = warp & 3;
    pdl_wait();
    const float sw = (FMT == NVFP4 && s_w) ? *s_w : 1.0f;
    const uint32_t acc_empty_leader = pair::mapa(smem_u32(acc_empty), 0);
    int it = 0;
    for (int tile = pair_id; tile < num_tiles; tile += num_pairs, ++it) {
      const int2 tt = tile_mn(tile, tiles_m, tiles_n, nfast);
        const int tm = tt.x, tn = tt.y;
      const int row = tm * 256 + (int)rank * 128 + quad * 32 + lane;
      const int n0 = tn * BN;
      float rs = sw;   // loaded before the accumulator wait
      if (FMT == NVFP4 && s_tok && row < M) rs = __fmul_rn(s_tok[row], sw);
      int ok = 1;
      if (lane == 0) ok = mbar_wait(acc_full, it & 1, abort_flag) ? 1 : 0;
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      fence_after_sync();
      // drain the 128 x 256 accumulator slice of this warp into registers,
      // release it to the leader's MMA warp, then scale, convert and store
      uint32_t pk[BN / 2];
#pragma unroll
      for (int c0 = 0; c0 < BN; c0 += 32) {
        uint32_t v[32];
        tmem_ld32(tmem + ((uint32_t)(quad * 32) << 16) + c0, v);
#pragma unroll
        for (int k = 0; k < 32; k += 2) {
          float f0 = __fmul_rn(__uint_as_float(v[k]), rs);
          float f1 = __fmul_rn(__uint_as_float(v[k + 1]), rs);
          if (r_row) {
            f0 = __fmul_rn(f0, __ldg(r_row + n0 + c0 + k));
            f1 = __fmul_rn(f1, __ldg(r_row + n0 + c0 + k + 1));
          }
          if constexpr (YT == 1) {
            __nv_bfloat162 p2 = __floats2bfloat162_rn(f0, f1);
            pk[(c0 + k) / 2] = *reinterpret_cast<uint32_t*>(&p2);
          } else {
            v[k] = __float_as_uint(f0);
            v[k + 1] = __float_as_uint(f1);
          }
        }
        if constexpr (YT != 1) {   // fp32 output: store this 32-column chunk now
          if (row < M) {
            float4* dst = reinterpret_cast<float4*>(reinterpret_cast<float*>(Y) + (size_t)row * N + n0 + c0);
#pragma unroll
            for (int q = 0; q < 8; ++q)
              dst[q] = make_float4(__uint_as_float(v[4 * q]), __uint_as_float(v[4 * q + 1]),
                                   __uint_as_float(v[4 * q + 2]), __uint_as_float(v[4 * q + 3]));
          }
        }
      }
      fence_before_sync();
      __syncwarp();
      if (lane == 0) pair::arrive_remote(acc_empty_leader);
      if constexpr (YT == 1) {
        if (row < M) {
          uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(Y) + (size_t)row * N + n0);
#pragma unroll
          for (int q = 0; q < BN / 8; ++q)
            dst[q] = make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
        }
      }
    }
  }

  fence_before_sync();
  __syncthreads();
  cluster_barrier();   // the leader's last MMAs into this CTA's tensor memory are done
  if (warp == 1) {
    fence_after_sync();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"((uint32_t)C::TMEM_COLS)
                 : "memory");
  }
}

// ---------------------------------------------------------------------------
// MXINT4 linear.  sm_100a has no 4-bit integer tensor-core MMA, so the
// integer codes (-8..7, exact in E4M3) are widened on chip: TMA stages the
// packed codes, four converter warps turn each two's-complement nibble into
// its E4M3 byte (byte-permute table lookups) and write the 128-byte-swizzled
// K-major operand tiles, and tcgen05.mma.kind::mxf8f6f4 with E8M0 scales per
// 32 elements (one scale byte per MMA, K = 32) accumulates in tensor memory.
// Tiles 128 x 128, BK = 128 elements per stage, persistent.
//   warp 0 TMA, warp 1 MMA, warps 2..5 epilogue, warp 6 scale copies,
//   warps 7..14 converters.
// ---------------------------------------------------------------------------
namespace i4 {
constexpr int BN = 128, BKE = 128;                   // elements per k-tile
constexpr int CONVERTERS = 8;                  // converter warps (7 .. 14)
constexpr int THREADS = (7 + CONVERTERS) * 32;
constexpr int STG_A = BM * BKE / 2, STG_B = BN * BKE / 2;      // packed staging (8 KB each)
constexpr int OP_A = BM * BKE, OP_B = BN * BKE;                // E4M3 operands (16 KB each)
constexpr int SF_A = 512, SF_B = 512;                          // one 128 x 4 atom each
constexpr int STAGE = STG_A + STG_B + OP_A + OP_B + SF_A + SF_B;
constexpr int STAGES = 4;
constexpr int SMEM = STAGES * STAGE + 1024 + 256;
constexpr int SF_COLS = 8;                                     // 4 (A) + 4 (B) columns per slot
constexpr int TMEM_COLS = 256;
static_assert(BN + STAGES * SF_COLS <= TMEM_COLS, "tensor memory budget");
static_assert(SMEM <= 227 * 1024, "shared memory budget");

// Eight two's-complement INT4 codes (one 32-bit word, element k in nibble k)
// -> eight E4M3 bytes (two words, element k in byte k).
__device__ __forceinline__ uint2 widen8(uint32_t w) {
  // E4M3 of 0..7 and of -8..-1 (indexed by the low three bits of the code)
  constexpr uint32_t POS_LO = 0x44403800u, POS_HI = 0x4E4C4A48u;
  constexpr uint32_t NEG_LO = 0xCACCCED0u, NEG_HI = 0xB8C0C4C8u;
  uint32_t out[2];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const uint32_t sel = (w >> (16 * h)) & 0xFFFFu;
    const uint32_t pos = __byte_perm(POS_LO, POS_HI, sel);
    const uint32_t neg = __byte_perm(NEG_LO, NEG_HI, sel);
    // byte i from pos (selector i) or neg (selector 4 + i) by bit 3 of code i
    const uint32_t pick = ((sel >> 1) & 0x4444u) | 0x3210u;
    out[h] = __byte_perm(pos, neg, pick);
  }
  return make_uint2(out[0], out[1]);
}

// kind::f16 MMA (bf16 A and B from shared memory, fp32 accumulator), K = 16.
__device__ __forceinline__ void mma_bf16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                         uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
      ::"r"(tmem_d), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Sixteen int8 codes (a 16-byte chunk) times the block's power of two ->
// sixteen bf16 values, exact (8 significant bits), packed two per word.
__device__ __forceinline__ void dequant16_bf16(uint4 v, float scale, uint32_t* out) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int lo = (int)(w[i] << (24 - 16 * h)) >> 24;       // byte 2h of the word
      const int hi = (int)(w[i] << (16 - 16 * h)) >> 24;       // byte 2h + 1
      const uint32_t blo = __float_as_uint(__fmul_rn((float)lo, scale)) >> 16;
      const uint32_t bhi = __float_as_uint(__fmul_rn((float)hi, scale)) >> 16;
      out[2 * i + h] = blo | (bhi << 16);
    }
}

__device__ __forceinline__ void mma_f8(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                       uint32_t idesc, uint32_t accumulate, uint32_t tsfa,
                                       uint32_t tsfb) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}"
      ::"r"(tmem_d), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(tsfa), "r"(tsfb)
      : "memory");
}
}  // namespace i4

// MODE 0: MXINT4 (as described above).
// MODE 1: MXFP8 operands (E4M3 codes in global memory): TMA places them
//         straight into the swizzled operand tiles and the converter warps idle.
// MODE 2: MXINT8 operands: an int8 code times its block's power of two is a
//         bf16 value exactly, so the converters dequantise each 64-element
//         k-tile (int8 staging, scale bytes read from global memory) into
//         128-byte-swizzled bf16 operand tiles, and kind::f16 MMAs with fp32
//         accumulation compute the block-scaled product exactly; no scale
//         copies into tensor memory.
template <int YT, int MODE>
__global__ void __launch_bounds__(i4::THREADS, 1)
w4a4_gemm_mxint4_kernel(const __grid_constant__ CUtensorMap tmA,
                        const __grid_constant__ CUtensorMap tmB, const uint8_t* __restrict__ sfA,
                        const uint8_t* __restrict__ sfB, const float* __restrict__ r_row,
                        void* __restrict__ Y, int M, int N, int K) {
  using namespace i4;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  unsigned char* opA = smem;                              // 1024-aligned operand tiles
  unsigned char* opB = opA + STAGES * OP_A;
  unsigned char* stA = opB + STAGES * OP_B;
  unsigned char* stB = stA + STAGES * STG_A;
  unsigned char* sSFA = stB + STAGES * STG_B;
  unsigned char* sSFB = sSFA + STAGES * SF_A;
  uint64_t* full = reinterpret_cast<uint64_t*>(sSFB + STAGES * SF_B);
  uint64_t* empty = full + STAGES;
  uint64_t* sfready = empty + STAGES;
  uint64_t* conv = sfready + STAGES;
  uint64_t* acc_full = conv + STAGES;
  uint64_t* acc_empty = acc_full + 1;
  uint32_t* tmem_base_slot = reinterpret_cast<uint32_t*>(acc_empty + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_base_slot + 1);
  uint64_t* drain = acc_empty + 2;   // tensor-core work of the MMA and copier threads done

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tiles_m = (M + BM - 1) / BM, tiles_n = N / BN, num_tiles = tiles_m * tiles_n;
  constexpr bool FP8 = MODE == 1, I8 = MODE == 2;
  constexpr int KTE = I8 ? 64 : BKE;                 // elements per k-tile
  const int KT = K / KTE;
  const int S4 = (K / 32) / 4;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
      mbar_init(&sfready[s], 1);
      mbar_init(&conv[s], CONVERTERS);
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, 4);
    mbar_init(drain, 2);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_base_slot)), "r"((uint32_t)TMEM_COLS) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tmem = *tmem_base_slot;
  pdl_wait();     // operands and output may belong to the previous kernel of the stream
  pdl_trigger();

  if (warp == 0) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      int issued = 0;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        const int m0 = (tile % tiles_m) * BM, n0 = (tile / tiles_m) * BN;
        for (int kt = 0; kt < KT; ++kt) {
          if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag)) { ok = false; break; }
          ++issued;   // every load of the stage is issued below, with no wait in between
          if constexpr (I8) {          // int8 staging, 64 bytes per row; no scale copies
            mbar_expect_tx(&full[stage], STG_A + STG_B);
            tma_load_2d(stA + stage * STG_A, &tmA, &full[stage], kt * KTE, m0);
            tma_load_2d(stB + stage * STG_B, &tmB, &full[stage], kt * KTE, n0);
            if (++stage == STAGES) { stage = 0; phase ^= 1; }
            continue;
          } else if constexpr (FP8) {
            mbar_expect_tx(&full[stage], OP_A + OP_B + SF_A + SF_B);
            tma_load_2d(opA + stage * OP_A, &tmA, &full[stage], kt * BKE, m0);
            tma_load_2d(opB + stage * OP_B, &tmB, &full[stage], kt * BKE, n0);
          } else {
            mbar_expect_tx(&full[stage], STG_A + STG_B + SF_A + SF_B);
            tma_load_2d(stA + stage * STG_A, &tmA, &full[stage], kt * (BKE / 2), m0);
            tma_load_2d(stB + stage * STG_B, &tmB, &full[stage], kt * (BKE / 2), n0);
          }
          bulk_load(sSFA + stage * SF_A, sfA + ((size_t)(m0 / 128) * S4 + kt) * 512, SF_A,
                    &full[stage]);
          bulk_load(sSFB + stage * SF_B, sfB + ((size_t)(n0 / 128) * S4 + kt) * 512, SF_B,
                    &full[stage]);
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
      }
      const int stage_end = stage;
      const uint32_t phase_end = phase;
      if (ok)
        for (int s = 0; s < STAGES; ++s) {
          if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag)) break;
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
      // every issued load landed before the CTA may exit
      drain_loads<STAGES>(full, nullptr, stage_end, phase_end, issued);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      int stage = 0, it = 0;
      uint32_t phase = 0;
      bool ok = true;
      // kind::mxf8f6f4: E4M3 A and B (format 0), E8M0 scales, K-major, M = 128
      const uint32_t idesc0 = ((uint32_t)(BN >> 3) << 17) | (1u << 23) | ((uint32_t)(BM >> 4) << 24);
      // kind::f16: fp32 accumulator (c_format 1), bf16 A and B (format 1), K-major
      const uint32_t idesc_bf16 = (1u << 4) | (1u << 7) | (1u << 10) |
                                  ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x, ++it) {
        if (!mbar_wait(acc_empty, (it & 1) ^ 1, abort_flag)) break;
        fence_after_sync();
        for (int kt = 0; kt < KT; ++kt) {
          if constexpr (I8) {
            if (!mbar_wait(&conv[stage], phase, abort_flag)) { ok = false; break; }
            fence_after_sync();
            const uint32_t a_base = smem_u32(opA + stage * OP_A);
            const uint32_t b_base = smem_u32(opB + stage * OP_B);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {    // K = 16 bf16 (32 bytes) per MMA
              const uint64_t ad = smem_desc(a_base + kk * 32, 16, 1024, LAYOUT_SW128);
              const uint64_t bd = smem_desc(b_base + kk * 32, 16, 1024, LAYOUT_SW128);
              mma_bf16(tmem, ad, bd, idesc_bf16, (kt > 0 || kk > 0) ? 1u : 0u);
            }
            mma_commit(&empty[stage]);
            if (++stage == STAGES) { stage = 0; phase ^= 1; }
            continue;
          }
          if (!mbar_wait(FP8 ? &full[stage] : &conv[stage], phase, abort_flag) ||
              !mbar_wait(&sfready[stage], phase, abort_flag)) { ok = false; break; }
          fence_after_sync();
          const uint32_t a_base = smem_u32(opA + stage * OP_A);
          const uint32_t b_base = smem_u32(opB + stage * OP_B);
          const uint32_t sfa_col = BN + stage * SF_COLS, sfb_col = sfa_col + 4;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {      // K = 32 bytes per MMA in the 128-byte row
            const uint64_t ad = smem_desc(a_base + kk * 32, 16, 1024, LAYOUT_SW128);
            const uint64_t bd = smem_desc(b_base + kk * 32, 16, 1024, LAYOUT_SW128);
            const uint32_t sf_id = (uint32_t)kk;  // scale byte kk of the 32-bit column
            const uint32_t idesc = idesc0 | (sf_id << 29) | (sf_id << 4);
            mma_f8(tmem, ad, bd, idesc, (kt > 0 || kk > 0) ? 1u : 0u,
                   (tmem + sfa_col) | (sf_id << 30), (tmem + sfb_col) | (sf_id << 30));
          }
          mma_commit(&empty[stage]);
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
        mma_commit(acc_full);
      }
      mma_commit(drain);   // the MMAs issued so far have completed before exit
      mbar_drain(drain, 0);
    }
  } else if (warp == 6) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      for (int tile = blockIdx.x; tile < num_tiles && !I8; tile += gridDim.x) {
        bool ok = true;
        for (int kt = 0; kt < KT; ++kt) {
          if (!mbar_wait(&full[stage], phase, abort_flag)) { ok = false; break; }
          fence_after_sync();
          const uint32_t sfa_col = BN + stage * SF_COLS;
          tmem_cp_32x128b_x4(tmem + sfa_col, smem_desc(smem_u32(sSFA + stage * SF_A), 0, 128, LAYOUT_NONE));
          tmem_cp_32x128b_x4(tmem + sfa_col + 4, smem_desc(smem_u32(sSFB + stage * SF_B), 0, 128, LAYOUT_NONE));
          mma_commit(&sfready[stage]);
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
      }
      mma_commit(drain);   // the scale copies have completed (none for MXINT8)
      mbar_drain(drain, 0);
    }
  } else if (warp >= 7) {
    if constexpr (I8) {
    // converters: int8 staging x block power of two -> swizzled bf16 operand tiles
    const int ct = threadIdx.x - 7 * 32;        // 0 .. 32 * CONVERTERS - 1
    const int64_t S = K / 32;
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
      const int m0 = (tile % tiles_m) * BM, n0 = (tile / tiles_m) * BN;
      for (int kt = 0; kt < KT; ++kt) {
        int got = 1;
        if (lane == 0) got = mbar_wait(&full[stage], phase, abort_flag) ? 1 : 0;
        got = __shfl_sync(0xffffffffu, got, 0);
        if (!got) { ok = false; break; }
        // 16-byte int8 chunks: A rows 0..127 (4 chunks each), then B rows
#pragma unroll 2
        for (int c = ct; c < (BM + BN) * 4; c += 32 * CONVERTERS) {
          const bool isB = c >= BM * 4;
          const int cc = isB ? c - BM * 4 : c;
          const int r = cc >> 2, kc = cc & 3;
          const uint4 v = *reinterpret_cast<const uint4*>(
              (isB ? stB + stage * STG_B : stA + stage * STG_A) + r * 64 + kc * 16);
          // chunks 0-1 hold block 2kt of the row, chunks 2-3 block 2kt + 1; rows
          // past M read the zero scale bytes of the padded layout
          const int64_t grow = (isB ? n0 : m0) + r;
          const uint32_t e = __ldg((isB ? sfB : sfA) + sf_offset(grow, 2 * kt + (kc >> 1), S));
          uint32_t o[8];
          dequant16_bf16(v, pow2f((int)e - 127), o);
          unsigned char* rowp = (isB ? opB + stage * OP_B : opA + stage * OP_A) + r * 128;
          const int sw = r & 7;
          *reinterpret_cast<uint4*>(rowp + (((2 * kc) ^ sw) << 4)) = make_uint4(o[0], o[1], o[2], o[3]);
          *reinterpret_cast<uint4*>(rowp + (((2 * kc + 1) ^ sw) << 4)) = make_uint4(o[4], o[5], o[6], o[7]);
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncwarp();
        if (lane == 0) mbar_arrive(&conv[stage]);
        if (++stage == STAGES) { stage = 0; phase ^= 1; }
      }
    }
    } else if constexpr (!FP8) {
    // converters: packed INT4 staging -> swizzled E4M3 operand tiles
    const int ct = threadIdx.x - 7 * 32;        // 0 .. 32 * CONVERTERS - 1
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
      for (int kt = 0; kt < KT; ++kt) {
        int got = 1;
        if (lane == 0) got = mbar_wait(&full[stage], phase, abort_flag) ? 1 : 0;
        got = __shfl_sync(0xffffffffu, got, 0);
        if (!got) { ok = false; break; }
        // 16-byte packed chunks: A rows 0..127 (4 chunks each), then B rows
#pragma unroll 2
        for (int c = ct; c < (BM + BN) * 4; c += 32 * CONVERTERS) {
          const bool isB = c >= BM * 4;
          const int cc = isB ? c - BM * 4 : c;
          const int r = cc >> 2, kc = cc & 3;
          const uint4 v = *reinterpret_cast<const uint4*>(
              (isB ? stB + stage * STG_B : stA + stage * STG_A) + r * 64 + kc * 16);
          const uint2 w0 = widen8(v.x), w1 = widen8(v.y), w2 = widen8(v.z), w3 = widen8(v.w);
          unsigned char* rowp = (isB ? opB + stage * OP_B : opA + stage * OP_A) + r * 128;
          const int sw = r & 7;
          *reinterpret_cast<uint4*>(rowp + (((2 * kc) ^ sw) << 4)) = make_uint4(w0.x, w0.y, w1.x, w1.y);
          *reinterpret_cast<uint4*>(rowp + (((2 * kc + 1) ^ sw) << 4)) = make_uint4(w2.x, w2.y, w3.x, w3.y);
        }
        // make the generic-proxy writes visible to the tensor core (async proxy)
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncwarp();
        if (lane == 0) mbar_arrive(&conv[stage]);
        if (++stage == STAGES) { stage = 0; phase ^= 1; }
      }
    }
    }
  } else {
    // epilogue (warps 2..5)
    const int quad = warp & 3;
    int it = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++it) {
      const int row = (tile % tiles_m) * BM + quad * 32 + lane, n0 = (tile / tiles_m) * BN;
      int ok = 1;
      if (lane == 0) ok = mbar_wait(acc_full, it & 1, abort_flag) ? 1 : 0;
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      fence_after_sync();
      if constexpr (YT == 1) {
        if (r_row)
          epilogue_bf16<BN, true>(tmem, quad, lane, row, M, N, n0, 1.0f, r_row, Y, acc_empty);
        else
          epilogue_bf16<BN, false>(tmem, quad, lane, row, M, N, n0, 1.0f, r_row, Y, acc_empty);
      } else {
#pragma unroll 1
        for (int c0 = 0; c0 < BN; c0 += 32) {
          uint32_t v[32];
          tmem_ld32(tmem + ((uint32_t)(quad * 32) << 16) + c0, v);
          if (c0 + 32 == BN) {
            fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(acc_empty);
          }
          if (row < M) {
            float* dst = reinterpret_cast<float*>(Y) + (size_t)row * N + n0 + c0;
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              float4 f = make_float4(__uint_as_float(v[4 * q]), __uint_as_float(v[4 * q + 1]),
                                     __uint_as_float(v[4 * q + 2]), __uint_as_float(v[4 * q + 3]));
              if (r_row) {
                f.x = __fmul_rn(f.x, __ldg(r_row + n0 + c0 + 4 * q));
                f.y = __fmul_rn(f.y, __ldg(r_row + n0 + c0 + 4 * q + 1));
                f.z = __fmul_rn(f.z, __ldg(r_row + n0 + c0 + 4 * q + 2));
                f.w = __fmul_rn(f.w, __ldg(r_row + n0 + c0 + 4 * q + 3));
              }
              reinterpret_cast<float4*>(dst)[q] = f;
            }
          }
        }
      }
    }
  }

  fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    fence_after_sync();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"((uint32_t)TMEM_COLS) : "memory");
  }
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------
typedef CUresult (*PFN_encodeTiled)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                    const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                    const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                    CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static PFN_encodeTiled get_encode() {
  static PFN_encodeTiled fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_encodeTiled>(p);
  }
  return fn;
}

// 2-D map over a rows x (K/2) byte matrix, box = box_rows x 128 bytes, 128-byte swizzle.
// Encoding a map is host work comparable to a small kernel, so the maps of
// recent operands are kept in a small per-thread cache (a map only encodes
// the base pointer, sizes and strides, so a hit is always valid).
struct MapEntry {
  const void* base;
  int64_t rows, kbytes;
  int box_rows, box_bytes;
  CUtensorMap map;
};
static bool make_map(CUtensorMap* map, const void* base, int64_t rows, int64_t kbytes,
                     int box_rows, int box_bytes = BKB) {
  constexpr int kEntries = 16;
  thread_local MapEntry cache[kEntries];
  thread_local int used = 0, next = 0;
  for (int i = 0; i < used; ++i)
    if (cache[i].base == base && cache[i].rows == rows && cache[i].kbytes == kbytes &&
        cache[i].box_rows == box_rows && cache[i].box_bytes == box_bytes) {
      *map = cache[i].map;
      return true;
    }
  PFN_encodeTiled enc = get_encode();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)kbytes, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)kbytes};
  cuuint32_t box[2] = {(cuuint32_t)box_bytes, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  const CUtensorMapSwizzle sw =
      box_bytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE;
  if (enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box,
          estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return false;
  MapEntry& e = cache[next];
  e.base = base; e.rows = rows; e.kbytes = kbytes; e.box_rows = box_rows;
  e.box_bytes = box_bytes; e.map = *map;
  next = (next + 1) % kEntries;
  if (used < kEntries) ++used;
  return true;
}

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

template <int FMT, int BN, int YT, int AR = BM>
static int launch(const uint8_t* A, const uint8_t* sA, const float* s_tok, const uint8_t* B,
                  const uint8_t* sB, const float* s_w, const float* r_row, void* Y, int64_t M,
                  int64_t N, int64_t K, cudaStream_t st) {
  using C = Cfg<FMT, BN, 0, AR>;
  if (AR < BM && M > AR) return DQ_ERR_UNSUPPORTED;
  CUtensorMap ta, tb;
  if (!make_map(&ta, A, M, K / 2, AR) || !make_map(&tb, B, N, K / 2, BN)) return DQ_ERR_CUDA;
  auto kern = w4a4_gemm_kernel<FMT, BN, YT, AR>;
  if (!ensure_kernel_attrs((const void*)kern, C::SMEM_BYTES, false)) return DQ_ERR_CUDA;
  const int64_t tiles = ((M + BM - 1) / BM) * (N / BN);
  const int grid = (int)(tiles < num_sms() ? tiles : num_sms());
  const cudaError_t e = launch_ex(kern, dim3(grid), dim3(NUM_THREADS), C::SMEM_BYTES, st, 1, ta, tb,
                                  sA, sB, s_tok, s_w, r_row, Y, (int)M, (int)N, (int)K);
  return e == cudaSuccess ? DQ_OK : DQ_ERR_CUDA;
}

template <int FMT, int YT, int AR = BM>
static int launch_splitk(const uint8_t* A, const uint8_t* sA, const float* s_tok, const uint8_t* B,
                         const uint8_t* sB, const float* s_w, const float* r_row, void* Y,
                         int64_t M, int64_t N, int64_t K, int S, cudaStream_t st) {
  using C = Cfg<FMT, SK_BN, SK_PART_BYTES, AR>;
  // each CTA owns a column slice of SK_BN / S columns, moved as float4
  if (S < 1 || S > 8 || SK_BN % (4 * S)) return DQ_ERR_UNSUPPORTED;
  const int a_rows = M < BM ? (int)((M + 15) / 16 * 16) : BM;
  if (a_rows > AR) return DQ_ERR_UNSUPPORTED;
  CUtensorMap ta, tb;
  if (!make_map(&ta, A, M, K / 2, a_rows) || !make_map(&tb, B, N, K / 2, SK_BN)) return DQ_ERR_CUDA;
  auto kern = w4a4_gemm_splitk_kernel<FMT, YT, false, AR>;
  if (!ensure_kernel_attrs((const void*)kern, C::SMEM_BYTES, false)) return DQ_ERR_CUDA;
  const int kt_per_slice = (int)(K / BK) / S;
  if (launch_ex(kern, dim3(S, (unsigned)(N / SK_BN), (unsigned)((M + BM - 1) / BM)),
                dim3(NUM_THREADS), C::SMEM_BYTES, st, (unsigned)S, ta, tb, sA, sB, s_tok, s_w,
                r_row, Y, (int)M, (int)N, (int)K, kt_per_slice, a_rows,
                (const __nv_bfloat16*)nullptr, (const float*)nullptr) != cudaSuccess)
    return DQ_ERR_CUDA;
  return DQ_OK;
}

// Fused activation quantisation + split-K GEMM (NVFP4, bf16 X): the A tensor
// map is not used (a placeholder on the weights keeps the parameter valid).
template <int YT>
static int launch_splitk_fused(const __nv_bfloat16* X, const float* c, const uint8_t* B,
                               const uint8_t* sB, const float* s_w, const float* r_row, void* Y,
                               int64_t M, int64_t N, int64_t K, int S, cudaStream_t st) {
  using C = Cfg<NVFP4, SK_BN, SK_PART_BYTES>;
  if (S < 1 || S > 8 || SK_BN % (4 * S)) return DQ_ERR_UNSUPPORTED;
  const int a_rows = M < BM ? (int)((M + 15) / 16 * 16) : BM;
  const int kt_per_slice = (int)(K / BK) / S;
  if (kt_per_slice > C::STAGES) return DQ_ERR_UNSUPPORTED;
  CUtensorMap tb;
  if (!make_map(&tb, B, N, K / 2, SK_BN)) return DQ_ERR_CUDA;
  auto kern = w4a4_gemm_splitk_kernel<NVFP4, YT, true>;
  if (!ensure_kernel_attrs((const void*)kern, C::SMEM_BYTES, false)) return DQ_ERR_CUDA;
  if (launch_ex(kern, dim3(S, (unsigned)(N / SK_BN), (unsigned)((M + BM - 1) / BM)),
                dim3(NUM_THREADS), C::SMEM_BYTES, st, (unsigned)S, tb, tb,
                (const uint8_t*)nullptr, sB, (const float*)nullptr, s_w, r_row, Y, (int)M,
                (int)N, (int)K, kt_per_slice, a_rows, X, c) != cudaSuccess)
    return DQ_ERR_CUDA;
  return DQ_OK;
}

// Paired-SM launch: 2 CTAs per cluster, persistent over 256 x 256 tiles.
template <int FMT, int YT>
static int pair_max_clusters() {
  static int cache[16];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 16) return 0;
  if (cache[dev]) return cache[dev] > 0 ? cache[dev] : 0;
  using C = pair::Cfg2<FMT>;
  auto kern = w4a4_gemm_pair_kernel<FMT, YT>;
  int n = 0;
  if (ensure_kernel_attrs((const void*)kern, C::SMEM_BYTES, false)) {
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2, 1, 1);
    cfg.blockDim = dim3(NUM_THREADS, 1, 1);
    cfg.dynamicSmemBytes = C::SMEM_BYTES;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaOccupancyMaxActiveClusters(&n, (const void*)kern, &cfg) != cudaSuccess) {
      cudaGetLastError();
      n = 0;
    }
  }
  cache[dev] = n > 0 ? n : -1;
  return n > 0 ? n : 0;
}

template <int FMT, int YT>
static int launch_pair(const uint8_t* A, const uint8_t* sA, const float* s_tok, const uint8_t* B,
                       const uint8_t* sB, const float* s_w, const float* r_row, void* Y,
                       int64_t M, int64_t N, int64_t K, int max_pairs, cudaStream_t st) {
  using C = pair::Cfg2<FMT>;
  const int64_t S4 = (K / C::G) / 4;
  const int64_t sfa_rows = ((M + 127) / 128) * S4 * 2;  // scale atoms as 256-byte rows
  const int64_t sfb_rows = (N / 128) * S4 * 2;
  CUtensorMap ta, tb, tsa, tsb;
  if (!make_map(&ta, A, M, K / 2, BM) || !make_map(&tb, B, N, K / 2, 128) ||
      !make_map(&tsa, sA, sfa_rows, 256, 2 * C::SF_ATOMS, 256) ||
      !make_map(&tsb, sB, sfb_rows, 256, 2 * C::SF_ATOMS, 256))
    return DQ_ERR_CUDA;
  auto kern = w4a4_gemm_pair_kernel<FMT, YT>;
  if (!ensure_kernel_attrs((const void*)kern, C::SMEM_BYTES, false)) return DQ_ERR_CUDA;
  const int64_t tiles = ((M + 255) / 256) * (N / pair::BN);
  const int pairs = (int)(tiles < max_pairs ? tiles : max_pairs);
  const cudaError_t e = launch_ex(kern, dim3(2 * pairs), dim3(NUM_THREADS), C::SMEM_BYTES, st, 2,
                                  ta, tb, tsa, tsb, s_tok, s_w, r_row, Y, (int)M, (int)N, (int)K);
  return e == cudaSuccess ? DQ_OK : DQ_ERR_CUDA;
}

// DQ_GEMM_PAIR: 0 never uses the paired-SM kernel, 2 prefers it whenever N
// is a multiple of 256, anything else (default) lets the tile policy decide.
static int pair_mode() {
  static const int mode = [] {
    const char* e = getenv("DQ_GEMM_PAIR");
    return (e && e[0] == '0') ? 0 : ((e && e[0] == '2') ? 2 : 1);
  }();
  return mode;
}

// How many clusters of S split-K CTAs the device runs at once (each CTA
// takes one SM's shared memory; a cluster must fit inside one GPC).
template <int FMT, int YT>
static int splitk_max_clusters(int S) {
  static int cache[16][9];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 16 || S < 1 || S > 8) return 0;
  if (cache[dev][S]) return cache[dev][S] > 0 ? cache[dev][S] : 0;
  using C = Cfg<FMT, SK_BN, SK_PART_BYTES>;
  auto kern = w4a4_gemm_splitk_kernel<FMT, YT, false>;
  int n = 0;
  if (ensure_kernel_attrs((const void*)kern, C::SMEM_BYTES, false)) {
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = S;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(S, 1, 1);
    cfg.blockDim = dim3(NUM_THREADS, 1, 1);
    cfg.dynamicSmemBytes = C::SMEM_BYTES;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaOccupancyMaxActiveClusters(&n, (const void*)kern, &cfg) != cudaSuccess) {
      cudaGetLastError();
      n = 0;
    }
  }
  cache[dev][S] = n > 0 ? n : -1;
  return n > 0 ? n : 0;
}

// Tile-shape policy: up to four tokens on the CUDA cores (dq_gemv.cu); 128 x
// 256 persistent tiles when they fill the machine, else 128 x 128 persistent
// tiles, else split-K over a cluster of S CTAs.
template <int FMT, int YT>
static int dispatch(const uint8_t* A, const uint8_t* sA, const float* s_tok, const uint8_t* B,
                    const uint8_t* sB, const float* s_w, const float* r_row, void* Y, int64_t M,
                    int64_t N, int64_t K, cudaStream_t st) {
  if (M <= GEMV_MAX_TOKENS) {   // a weight stream: the CUDA-core kernel of dq_gemv.cu
    const int rc = w4a4_gemv(A, sA, s_tok, B, sB, s_w, r_row, Y, YT, M, N, K, FMT, st);
    if (rc != DQ_ERR_UNSUPPORTED) return rc;
  }
  const int64_t tm = (M + BM - 1) / BM, sms = num_sms();
  // long K with plenty of 256 x 256 tiles: the paired-SM kernel reads 30 %
  // fewer operand bytes per SM (measured 8192 x 5120 x 27648: 3.88 vs 3.60
  // PFLOP/s); at K of a few thousand both tile shapes run alike
  if (N % 256 == 0 && (pair_mode() == 2 || (pair_mode() == 1 && K >= 16384 &&
                                             ((M + 255) / 256) * (N / 256) >= 2 * sms))) {
    const int max_pairs = pair_max_clusters<FMT, YT>();
    if (max_pairs > 0)
      return launch_pair<FMT, YT>(A, sA, s_tok, B, sB, s_w, r_row, Y, M, N, K, max_pairs, st);
  }
  if (N % 256 == 0 && tm * (N / 256) >= sms)
    return launch<FMT, 256, YT>(A, sA, s_tok, B, sB, s_w, r_row, Y, M, N, K, st);
  if (N % 256 == 0 && pair_mode() != 0 && (tm > 1 || pair_mode() == 2)) {
    // too few 128 x 256 tiles to fill the SMs: paired-SM 256 x 256 tiles
    // once they occupy at least half of the SM pairs (not when one 128-row
    // tile holds every token: the weight-streaming 128-wide tiles measured
    // faster there, M = 1 x 27648 x 5120: 30.3 vs 34.9 us)
    const int max_pairs = pair_max_clusters<FMT, YT>();
    const int64_t tiles2 = ((M + 255) / 256) * (N / 256);
    if (max_pairs > 0 && 2 * tiles2 >= max_pairs)
      return launch_pair<FMT, YT>(A, sA, s_tok, B, sB, s_w, r_row, Y, M, N, K, max_pairs, st);
  }
  const int64_t t128 = tm * (N / 128);
  const int KT = (int)(K / BK);
  // largest split whose clusters (one per output tile) all run in one wave
  int S = 1;
  for (int cand : {8, 4, 2})   // the column slice 128 / S must stay a multiple of 4
    if (S == 1 && KT % cand == 0 && t128 * cand <= sms &&
        t128 <= splitk_max_clusters<FMT, YT>(cand))
      S = cand;
  const bool few = M <= 32;   // every token in 32 staged rows
  if (S > 1)
    return few ? launch_splitk<FMT, YT, 32>(A, sA, s_tok, B, sB, s_w, r_row, Y, M, N, K, S, st)
               : launch_splitk<FMT, YT>(A, sA, s_tok, B, sB, s_w, r_row, Y, M, N, K, S, st);
  if (N % 256 == 0 && tm * (N / 256) * 2 > t128)  // few tiles either way: keep the wide tile
    return few ? launch<FMT, 256, YT, 32>(A, sA, s_tok, B, sB, s_w, r_row, Y, M, N, K, st)
               : launch<FMT, 256, YT>(A, sA, s_tok, B, sB, s_w, r_row, Y, M, N, K, st);
  return few ? launch<FMT, 128, YT, 32>(A, sA, s_tok, B, sB, s_w, r_row, Y, M, N, K, st)
             : launch<FMT, 128, YT>(A, sA, s_tok, B, sB, s_w, r_row, Y, M, N, K, st);
}

// MODE 1: MXFP8 codes (one byte per element, 128-byte swizzled TMA boxes);
// MODE 2: MXINT8 codes (one byte per element, 64-byte boxes of 64 elements
// into the staging buffers); MODE 0: packed MXINT4 codes (64-byte boxes of
// 128 elements into the staging buffers).
template <int YT, int MODE>
static int launch_mxint4(const uint8_t* A, const uint8_t* sA, const uint8_t* B, const uint8_t* sB,
                         const float* r_row, void* Y, int64_t M, int64_t N, int64_t K,
                         cudaStream_t st) {
  CUtensorMap ta, tb;
  const int64_t kb = MODE == 0 ? K / 2 : K;
  const int box = MODE == 1 ? i4::BKE : i4::BKE / 2;
  if (!make_map(&ta, A, M, kb, BM, box) || !make_map(&tb, B, N, kb, i4::BN, box))
    return DQ_ERR_CUDA;
  auto kern = w4a4_gemm_mxint4_kernel<YT, MODE>;
  if (!ensure_kernel_attrs((const void*)kern, i4::SMEM, false)) return DQ_ERR_CUDA;
  const int64_t tiles = ((M + BM - 1) / BM) * (N / i4::BN);
  const int grid = (int)(tiles < num_sms() ? tiles : num_sms());
  const cudaError_t e = launch_ex(kern, dim3(grid), dim3(i4::THREADS), i4::SMEM, st, 1, ta, tb, sA,
                                  sB, r_row, Y, (int)M, (int)N, (int)K);
  return e == cudaSuccess ? DQ_OK : DQ_ERR_CUDA;
}

}  // namespace gemm

int w4a4_linear(const uint8_t* A, const uint8_t* sA, const float* s_tok, const uint8_t* B,
                const uint8_t* sB, const float* s_w, const float* r_row, void* Y, int yt,
                int64_t M, int64_t N, int64_t K, int f, cudaStream_t st) {
  if (f == NVFP4)
    return yt == 1 ? gemm::dispatch<NVFP4, 1>(A, sA, s_tok, B, sB, s_w, r_row, Y, M, N, K, st)
                   : gemm::dispatch<NVFP4, 0>(A, sA, s_tok, B, sB, s_w, r_row, Y, M, N, K, st);
  if (f == MXFP4)
    return yt == 1 ? gemm::dispatch<MXFP4, 1>(A, sA, s_tok, B, sB, s_w, r_row, Y, M, N, K, st)
                   : gemm::dispatch<MXFP4, 0>(A, sA, s_tok, B, sB, s_w, r_row, Y, M, N, K, st);
  if (f == MXINT4)
    return yt == 1 ? gemm::launch_mxint4<1, 0>(A, sA, B, sB, r_row, Y, M, N, K, st)
                   : gemm::launch_mxint4<0, 0>(A, sA, B, sB, r_row, Y, M, N, K, st);
  if (f == MXFP8)
    return yt == 1 ? gemm::launch_mxint4<1, 1>(A, sA, B, sB, r_row, Y, M, N, K, st)
                   : gemm::launch_mxint4<0, 1>(A, sA, B, sB, r_row, Y, M, N, K, st);
  if (f == MXINT8)
    return yt == 1 ? gemm::launch_mxint4<1, 2>(A, sA, B, sB, r_row, Y, M, N, K, st)
                   : gemm::launch_mxint4<0, 2>(A, sA, B, sB, r_row, Y, M, N, K, st);
  return DQ_ERR_UNSUPPORTED;
}

// Fused activation rescale + quantise + linear for small M (NVFP4, bf16 X):
// the split of K is chosen as for the split-K GEMM, and must leave at most
// STAGES k-tiles per CTA.
int w4a4_linear_fused(const void* X, const float* c, const uint8_t* B, const uint8_t* sB,
                      const float* s_w, const float* r_row, void* Y, int yt, int64_t M,
                      int64_t N, int64_t K, cudaStream_t st) {
  using C = gemm::Cfg<NVFP4, gemm::SK_BN, gemm::SK_PART_BYTES>;
  const int sms = gemm::num_sms();
  const int64_t tm = (M + gemm::BM - 1) / gemm::BM;
  const int64_t t128 = tm * (N / gemm::SK_BN);
  const int KT = (int)(K / gemm::BK);
  int S = 0;
  for (int cand : {8, 4, 2})
    if (S == 0 && KT % cand == 0 && KT / cand <= C::STAGES && t128 * cand <= sms &&
        t128 <= gemm::splitk_max_clusters<NVFP4, 1>(cand))
      S = cand;
  if (S == 0) return DQ_ERR_UNSUPPORTED;
  const __nv_bfloat16* Xb = reinterpret_cast<const __nv_bfloat16*>(X);
  return yt == 1 ? gemm::launch_splitk_fused<1>(Xb, c, B, sB, s_w, r_row, Y, M, N, K, S, st)
                 : gemm::launch_splitk_fused<0>(Xb, c, B, sB, s_w, r_row, Y, M, N, K, S, st);
}

int set_gemm_wait_limit(unsigned long long ns) {
  return cudaMemcpyToSymbol(g_dq_wait_limit_ns, &ns, sizeof(ns)) == cudaSuccess ? DQ_OK
                                                                                 : DQ_ERR_CUDA;
}

int read_device_error(int clear) {
  int v = 0;
  if (cudaDeviceSynchronize() != cudaSuccess) return DQ_ERR_CUDA;
  if (cudaMemcpyFromSymbol(&v, g_dq_device_error, sizeof(int)) != cudaSuccess) return DQ_ERR_CUDA;
  if (clear) {
    int z = 0;
    cudaMemcpyToSymbol(g_dq_device_error, &z, sizeof(int));
  }
  const int q = read_quant_error(clear);
  return v ? v : q;
}

}  // namespace dq
