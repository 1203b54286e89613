/*
 * dq.h -- C ABI of the DualQuant dual-scale W4A4 library for NVIDIA B200
 * (sm_100a).  Library: w4a4_post_quantization_dual_b200/lib/libdq.so.
 *
 * Method: "DualQuant: Dual-scale Calibration-free Weight-and-Activation
 * Quantization for LLMs" (Salmani, Sharify, Mostafa; arXiv 2610.13767).
 * A weight W (m x n, out-features x in-features) is approximated as
 *     W ~= diag_blk(r) * What * diag(c)                      (Section 4.2, Eq. 2)
 * with r = alpha^-1 one scale per row and block of G columns (the format's
 * native block scale), c = beta^-1 one scale per column, and What on the
 * format's 4-bit grid.  At inference the activations are rescaled by c and
 * quantised in the same block format, so that
 *     Y = X W^T ~= Q(X diag(c)) What^T diag_blk(r)             (Eq. 3, Section 4.4).
 *
 * Conventions for every entry point
 *  - Pointers are DEVICE pointers owned by the caller unless stated.  The
 *    library never allocates device or host memory and never synchronises
 *    the stream; every call is stream-ordered and asynchronous on `stream`
 *    (a cudaStream_t; NULL = legacy default stream).
 *  - Matrices are row-major and dense (leading dimension = row length).
 *  - 4-bit codes are packed two per byte, element 2k in the low nibble of
 *    byte k.  E2M1 codes: bit 3 sign, bits 0-2 magnitude index of
 *    {0, .5, 1, 1.5, 2, 3, 4, 6}.  INT4 / MXINT4 codes: two's complement
 *    nibble, values -8..7.  8-bit codes are one byte per element: INT8 /
 *    MXINT8 two's complement (-128..127), MXFP8 FP8 E4M3 (OCP), rows K
 *    bytes long.
 *  - Block scales for NVFP4 and the MX formats are one byte per
 *    (row, block) (UE4M3 for NVFP4, E8M0 for MX) stored in the layout the
 *    block-scaled tensor-core MMA reads: 512-byte atoms of 128 rows x 4
 *    scales, atoms ordered row-block-major then along K; inside an atom the
 *    scale (row, s) sits at byte (row%32)*16 + ((row%128)/32)*4 + s%4.
 *    Rows are padded to a multiple of 128 and scale columns to a multiple
 *    of 4; dq_scales_bytes() gives the size.  INT4 and INT8 block scales
 *    are bf16, row-major rows x (k/G).
 *  - Inputs must be finite.  For NVFP4 and INT4 activations a row (NVFP4)
 *    or block (INT4) whose absmax is below about 1e-30 is outside the
 *    supported range: its fp32 reciprocal block scale overflows.  Arguments are validated before any launch; a
 *    non-DQ_OK return means nothing was enqueued (except DQ_ERR_CUDA, which
 *    reports a failed launch).
 */
#ifndef DQ_H
#define DQ_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define DQ_API __attribute__((visibility("default")))
#else
#define DQ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  DQ_INT4 = 0,   /* integers -8..7, bf16 block scale, G in {32, 64, 128}   */
  DQ_MXINT4 = 1, /* integers -8..7, E8M0 block scale, G = 32               */
  DQ_MXFP4 = 2,  /* E2M1, E8M0 block scale, G = 32 (OCP MX)                */
  DQ_NVFP4 = 3   /* E2M1, UE4M3 block scale, G = 16, plus an fp32 per-tensor
                    (weights) or per-token (activations) scale             */,
  /* 8-bit variants (Appendix G.2, Table 9): the solver, packer, activation
     quantiser and error measure take all three; dq_w4a4_linear takes
     MXFP8 and MXINT8 and returns DQ_ERR_UNSUPPORTED for INT8             */
  DQ_INT8 = 4,   /* integers -128..127, bf16 block scale, G in {32, 64, 128} */
  DQ_MXINT8 = 5, /* integers -128..127, E8M0 block scale, G = 32           */
  DQ_MXFP8 = 6   /* FP8 E4M3, E8M0 block scale, G = 32 (OCP MX)            */
} dq_format;

typedef enum { DQ_F32 = 0, DQ_BF16 = 1 } dq_dtype;

typedef enum {
  DQ_OK = 0,
  DQ_ERR_ARG = 1,            /* null pointer, bad size, alignment, G, dtype */
  DQ_ERR_UNSUPPORTED = 2,    /* valid request the library does not implement */
  DQ_ERR_CUDA = 3,           /* a launch or CUDA runtime call failed        */
  DQ_ERR_DEVICE_TIMEOUT = 4, /* a kernel's bounded wait expired (see
                                dq_device_error)                           */
  DQ_ERR_WORKSPACE = 5       /* workspace missing or too small              */
} dq_status;

/* Human-readable name of a status code (static string). */
DQ_API const char* dq_status_string(int status);

/* Native block size of a format: 64 for INT4 (the paper's setting, Section
 * 5), 32 for MXINT4 / MXFP4, 16 for NVFP4 (Section 3). */
DQ_API int dq_native_group(dq_format f);

/* Bytes of the block-scale buffer for a rows x k operand quantised with
 * block size G: the padded tensor-core layout above for NVFP4 / MX, or
 * rows*(k/G)*2 for INT4.  Returns 0 for invalid arguments. */
DQ_API size_t dq_scales_bytes(int64_t rows, int64_t k, dq_format f, int group);

/* ------------------------------------------------------------------------
 * dq_solve_scales -- Algorithm 1 (dual-scale quantisation via block
 * coordinate descent, Section 4.3; closed-form updates Eqs. 10 and 14,
 * Appendix B), run independently on every m x G column-block tile of W.
 *
 *  W        m x n, dtype wt (DQ_BF16 or DQ_F32).  n % G == 0; n / G <= 65535
 *           (one launch grid), else DQ_ERR_UNSUPPORTED before anything is
 *           enqueued.
 *  f, group format and block size G (see dq_format).
 *  T        number of BCD rounds (>= 0).  Each round: quantise, update and
 *           project the row-block scales r, re-quantise, update and project
 *           the column scales c (Section 4.3, cycle (i)-(iv)).
 *  r        out, m x (n/G) fp32: row-block scales alpha^-1, each in F_alpha
 *           (BF16 for INT4, E8M0 for MX, s_tensor * UE4M3 for NVFP4).
 *  c        out, n fp32: column scales beta^-1, each in F_beta (BF16,
 *           E8M0, UE4M3).
 *  s_tensor out, 1 fp32: NVFP4 per-tensor scale amax(W diag(c0)^-1)/2688,
 *           fixed at initialisation; 1.0 for the other formats.
 *  mse_trace out (nullable), T+1 doubles: normalised reconstruction error
 *           ||W - diag_blk(r) What diag(c)||_F^2 / ||W||_F^2 at the scales
 *           after round t (t = 0: initial scales), What re-quantised at
 *           those scales (the quantity of Fig. 2(b)).
 *  workspace, ws_bytes: caller-owned device scratch of at least
 *           dq_solve_workspace_size(T) bytes, 16-byte aligned; contents on
 *           entry are ignored (the call clears what it uses).
 * Initialisation (Section 5.3): c0 proportional to the column l1 norm,
 * normalised to mean 1 per tile and projected; r0 = the format-native
 * absmax (RTN) block scale of W diag(c0)^-1.  Degenerate rows / columns
 * (all codes zero) take the projection of 1 (Section 4.3, after
 * Assumption 1).  Accumulation: fp32 per thread, fp64 across threads; the
 * quantiser argument is fp32: (W * fl(1/c)) * fl(1/r).
 * ---------------------------------------------------------------------- */
DQ_API size_t dq_solve_workspace_size(int T);
DQ_API int dq_solve_scales(const void* W, dq_dtype wt, int64_t m, int64_t n, dq_format f, int group,
                    int T, float* r, float* c, float* s_tensor, double* mse_trace,
                    void* workspace, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------
 * dq_solve_scales_ex -- dq_solve_scales with an ablation mode and a warm
 * start.  dq_solve_scales(...) is dq_solve_scales_ex with flags 0 and no
 * r0 / c0.
 *
 * flags (dq_solve_flags, OR-ed; ALPHA_ONLY and BETA_ONLY exclude each other):
 *  DQ_SOLVE_ALPHA_ONLY  the "alpha-only" arm of the scale ablation
 *           (Table 4): beta stays fixed -- at 1 (c = 1), or at the
 *           projection of c0 when given -- and each round is the row
 *           half-step only (Eq. 10 / Eq. 11).  With T = 0 and no c0 this is
 *           the single-scale RTN quantiser (Appendix F baseline).
 *  DQ_SOLVE_BETA_ONLY   the "beta-only" arm: alpha stays at its initial
 *           value (RTN of W diag(c0)^-1, or the projection of r0 when
 *           given) and each round is the column half-step only (Eq. 14 /
 *           Eq. 15).
 *  DQ_SOLVE_KEEP_TENSOR_SCALE  NVFP4: *s_tensor is an INPUT (device fp32,
 *           positive, finite) and is used as the per-tensor scale instead
 *           of amax(W diag(c0)^-1)/2688; it is not written.  Resuming from
 *           an earlier result (r, c, s_tensor) with this flag continues
 *           that solve exactly: T1 rounds then T2 resumed rounds give the
 *           scales and trace tail of T1 + T2 rounds.  Ignored (s_tensor
 *           receives 1.0) for the other formats.
 *  DQ_SOLVE_TRACE_CODES  mse_trace (then required) holds 2 (T+1) doubles:
 *           the MSE trace, then the relative code change of Fig. 2(a) /
 *           Fig. 3(a), ||Qhat(t) - Qhat(t-1)||_F / ||Qhat(t-1)||_F with
 *           Qhat(t) the codes at the scales after round t (entry 0 NaN).
 *  r0       nullable, device, m x (n/G) fp32, positive and finite: initial
 *           row-block scales (the initialisation (alpha_0, beta_0) of
 *           Section 5.3 given by the caller), each projected onto F_alpha
 *           (nearest admissible value; NVFP4 with the tensor scale in use).
 *           May alias r (in-place resume).
 *  c0       nullable, device, n fp32, positive and finite: initial column
 *           scales, each projected onto F_beta; replaces the l1
 *           initialisation.  May alias c.
 * The other arguments and the error behaviour are those of dq_solve_scales;
 * unknown flag bits or both ablation flags return DQ_ERR_ARG.
 * ---------------------------------------------------------------------- */
typedef enum {
  DQ_SOLVE_ALPHA_ONLY = 1,
  DQ_SOLVE_BETA_ONLY = 2,
  DQ_SOLVE_KEEP_TENSOR_SCALE = 4,
  DQ_SOLVE_TRACE_CODES = 8
} dq_solve_flags;
DQ_API int dq_solve_scales_ex(const void* W, dq_dtype wt, int64_t m, int64_t n, dq_format f,
                              int group, int T, unsigned flags, const float* r0, const float* c0,
                              float* r, float* c, float* s_tensor, double* mse_trace,
                              void* workspace, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------
 * dq_quantize_weight -- the stored low-precision weight of Algorithm 1's
 * result, What = Q(Diag(alpha) W Diag(beta)), packed for the GEMM
 * (Section 4.4 artefacts; Appendix I, packed offline).
 *
 *  W        m x n (dtype wt), r m x (n/G), c n, as produced by
 *           dq_solve_scales (r must lie in F_alpha: a power of two for MX,
 *           s_tensor * UE4M3 for NVFP4, a bf16 value for INT4).
 *  s_tensor device pointer to the NVFP4 per-tensor scale (ignored, may be
 *           NULL, for other formats).
 *  codes    out, m x n/2 bytes (m x n for the 8-bit formats).
 *  scales   out, dq_scales_bytes(m, n, f, G) bytes: the row-block scales
 *           encoded (UE4M3 of r/s_tensor, E8M0 exponent of r, bf16 of r).
 * Element code = grid(fl(fl(W_ij * fl(1/c_j)) * fl(1/r_ib))), round to
 * nearest, ties to even, saturating.  Bit-exact with the oracle.
 * ---------------------------------------------------------------------- */
DQ_API int dq_quantize_weight(const void* W, dq_dtype wt, int64_t m, int64_t n, dq_format f, int group,
                       const float* r, const float* c, const float* s_tensor, uint8_t* codes,
                       void* scales, void* stream);

/* ------------------------------------------------------------------------
 * dq_quantize_act -- fused activation rescale + quantise: X~ = X diag(c)
 * (Eq. 3, X~ = X Diag(beta)^-1) followed by the format-native quantiser
 * with its own per-row scale on X~ (Section 4.4; Section 5.2: the column
 * scale is applied inside the activation-quantisation kernel).
 *
 *  X        M x K (dtype xt: DQ_BF16 or DQ_F32); K % G == 0.
 *  c        K fp32 column scales (NULL = all ones).
 *  codes    out, M x K/2 bytes (M x K for the 8-bit formats).
 *  scales   out, dq_scales_bytes(M, K, f, G) bytes; padding rows of the
 *           tensor-core layout are written as zero.
 *  s_tok    out, M fp32 (NVFP4 only, else may be NULL): per-token scale
 *           amax_t(X~)/2688.
 * NVFP4 block byte = UE4M3(amax_blk / (6 s_tok)); MX block byte =
 * floor(log2 amax_blk) - 2 + 127 (OCP rule, E2M1 / INT4 emax = 2); INT4
 * block scale = bf16(amax_blk / 7).  Codes: grid(x~ * fl(1/scale)), round
 * to nearest even, saturating; an all-zero block gives zero codes.
 * Bit-exact with the oracle.
 * Ordering: stream-ordered; launched with programmatic dependent launch,
 * the kernel reads c before waiting for the kernel launched just before it,
 * so c must not be written by such a kernel when it triggers its
 * dependents early (the solver, memory copies and ordinary kernels do not).
 * ---------------------------------------------------------------------- */
DQ_API int dq_quantize_act(const void* X, dq_dtype xt, int64_t M, int64_t K, const float* c,
                    dq_format f, int group, uint8_t* codes, void* scales, float* s_tok,
                    void* stream);

/* ------------------------------------------------------------------------
 * dq_w4a4_linear -- Y = Q(X~) What^T with the block scales applied inside
 * the tensor-core MMA and the remaining scales in the epilogue
 * (Section 4.4: "Q(X~) What^T Diag(alpha)^-1"):
 *   Y[t, o] = s_tok[t] * s_w * r_row[o] * sum_k a[t,k] sa[t,k/G] b[o,k] sb[o,k/G]
 *
 *  A, sA    activation codes (M x K/2; M x K for MXFP8) and scales from
 *           dq_quantize_act.
 *  s_tok    M fp32 per-token scales (NVFP4; ignored for MX, may be NULL).
 *  B, sB    weight codes (N x K/2) and scales from dq_quantize_weight.
 *  s_w      device pointer to the weight's per-tensor scale (NVFP4; may be
 *           NULL = 1).
 *  r_row    N fp32 extra per-output scale (nullable): lets a caller keep
 *           a per-row alpha outside the block scales.
 *  Y        out, M x N, dtype yt (DQ_BF16: round to nearest even; DQ_F32).
 * Formats: DQ_NVFP4 (kind::mxf4nvf4, UE4M3 scales, 16-blocks), DQ_MXFP4
 * (kind::mxf4, E8M0, 32-blocks), DQ_MXINT4 (integer codes widened on chip to
 * E4M3, exact for -8..7, kind::mxf8f6f4 with E8M0 32-block scales);
 * DQ_INT4 returns DQ_ERR_UNSUPPORTED (bf16 group scales have no
 * block-scaled tensor-core form on sm_100a).
 * Sizes: M >= 1, N % 128 == 0, K % 256 == 0; A, B, sA, sB 16-byte aligned.
 * FP32 accumulation in tensor memory.  With M == 1 (NVFP4, MXFP4, K a
 * multiple of 1024) the call runs on the CUDA cores instead: a weight
 * stream with exact integer block dot products and fp32 accumulation,
 * summed in a fixed order (the same bits on every call).
 * Ordering: stream-ordered.  The inference kernels use programmatic
 * dependent launch and read the weight operand (B, sB) before waiting for
 * the kernel launched just before them in the stream; B and sB must
 * therefore not be written by such a kernel when it triggers its
 * dependents early (dq_quantize_weight's packer, memory copies and ordinary
 * kernels do not).  A, sA, s_tok and Y are accessed only after that wait.
 * ---------------------------------------------------------------------- */
DQ_API int dq_w4a4_linear(const uint8_t* A, const uint8_t* sA, const float* s_tok, const uint8_t* B,
                   const uint8_t* sB, const float* s_w, const float* r_row, void* Y,
                   dq_dtype yt, int64_t M, int64_t N, int64_t K, dq_format f, void* stream);

/* ------------------------------------------------------------------------
 * dq_solve_scales_batched -- dq_solve_scales on nw weights of one format and
 * dtype in few launches: weights with the same row count m share one
 * initialisation and one BCD launch (up to 16 weights per launch), so a
 * model's many projections fill the GPU together instead of one after the
 * other.  Every tile is still an independent problem (Algorithm 1 per m x G
 * tile), so each weight's r, c, s_tensor are exactly those of a separate
 * dq_solve_scales call; traces agree up to the order of fp64 atomic adds.
 *
 *  nw       number of weights (> 0).
 *  W, m, n  HOST arrays of nw entries: device pointer to weight i (m[i] x
 *           n[i], dtype wt, 16-byte aligned) and its sizes.
 *  r, c, s_tensor  HOST arrays of nw device pointers (the outputs of
 *           dq_solve_scales for weight i).
 *  mse_trace nullable HOST array of nw nullable device pointers (T+1
 *           doubles each).
 *  flags    as dq_solve_scales_ex (warm starts are single-weight only).
 *  workspace dq_solve_batched_workspace_size(nw, T) bytes, 16-byte aligned.
 * Errors as dq_solve_scales; nothing is enqueued when an argument is invalid.
 * ---------------------------------------------------------------------- */
DQ_API size_t dq_solve_batched_workspace_size(int nw, int T);
DQ_API int dq_solve_scales_batched(int nw, const void* const* W, dq_dtype wt, const int64_t* m,
                                   const int64_t* n, dq_format f, int group, int T,
                                   unsigned flags, float* const* r, float* const* c,
                                   float* const* s_tensor, double* const* mse_trace,
                                   void* workspace, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------
 * dq_act_quant_error -- quantisation error of the activation path, for the
 * activation SQNR with and without the column scales (Appendix E, Table 6:
 * the quantised weights held fixed, only the presence of the beta
 * pre-scaling varies).
 *
 *  X        M x K (dtype xt), the activations before rescaling.
 *  c        K fp32 column scales that dq_quantize_act used (NULL = none,
 *           i.e. the path without beta).
 *  codes, scales, s_tok  as written by dq_quantize_act(X, c, f, group).
 *  sums     out, device, 2 doubles (the call zeroes them first):
 *           sums[0] = sum x^2, sums[1] = sum (x - x^)^2, where
 *           x^_ij = (q_ij * s_blk (* s_tok_i for NVFP4)) / c_j in fp64.
 *           SQNR (dB) = 10 log10(sums[0] / sums[1]).
 * K % 8 == 0.  Stream-ordered; the fp64 sums are accumulated with atomics
 * (summation order unspecified).  Not part of the inference path.
 * ---------------------------------------------------------------------- */
DQ_API int dq_act_quant_error(const void* X, dq_dtype xt, int64_t M, int64_t K, const float* c,
                              dq_format f, int group, const uint8_t* codes, const void* scales,
                              const float* s_tok, double* sums, void* stream);

/* ------------------------------------------------------------------------
 * dq_w4a4_linear_fused -- dq_quantize_act followed by dq_w4a4_linear in one
 * kernel, for small token counts (decode): the activation rescale by c and
 * the NVFP4 quantisation (per-token scale over the whole row, UE4M3 block
 * scales, E2M1 codes, the arithmetic of dq_quantize_act) run in the GEMM's
 * producer warps, so no activation codes travel through memory.  Y equals
 * the unfused pair's output bit for bit.
 *
 *  X        M x K bf16 activations (xt must be DQ_BF16); c K fp32 or NULL.
 *  B, sB, s_w, r_row, Y, yt, N, K   as dq_w4a4_linear (NVFP4 only).
 * Returns DQ_ERR_UNSUPPORTED when no split of K across a cluster leaves each
 * CTA at most its pipeline depth of k-tiles within one wave of the GPU (use
 * the unfused pair then), or for a format other than NVFP4.
 * ---------------------------------------------------------------------- */
DQ_API int dq_w4a4_linear_fused(const void* X, dq_dtype xt, const float* c, const uint8_t* B,
                                const uint8_t* sB, const float* s_w, const float* r_row, void* Y,
                                dq_dtype yt, int64_t M, int64_t N, int64_t K, dq_format f,
                                void* stream);

/* ------------------------------------------------------------------------
 * dq_solve_scales_noalloc -- dq_solve_scales for callers that cannot
 * allocate device memory (the paper has no counterpart: this is a library
 * convenience).  Some callers have no way to provide the workspace: a
 * serving process that has handed all free device memory to its own pool
 * and may not call cudaMalloc around it, or a latency-critical path that
 * must never wait in the driver's allocator.  This entry point takes the
 * same inputs and outputs but no workspace: its scratch is a fixed array of
 * DQ_NOALLOC_SCRATCH_BYTES compiled into the library, present on every GPU
 * that loads the library until the process exits.  It never calls
 * cudaMalloc, cudaFree or any allocating routine.
 *  - T may be at most DQ_NOALLOC_MAX_ROUNDS; larger T returns
 *    DQ_ERR_WORKSPACE before anything is enqueued.
 *  - The first call on each device looks up the array's device address with
 *    that device current (a host-side step); make that first call before any
 *    stream capture.
 *  - The scratch used is the current device's: a non-null stream must belong
 *    to the current device, else DQ_ERR_ARG before anything is enqueued.
 *  - Every call on a device shares the one array, which keeps the contents
 *    of the last call (each call clears what it uses first).  Calls whose
 *    execution overlaps on the GPU (different streams, no ordering between
 *    them) race on the array and may corrupt each other's trace and NVFP4
 *    tensor scale; serialise them.
 * ---------------------------------------------------------------------- */
#define DQ_NOALLOC_SCRATCH_BYTES 49152
#define DQ_NOALLOC_MAX_ROUNDS 2045
DQ_API int dq_solve_scales_noalloc(const void* W, dq_dtype wt, int64_t m, int64_t n, dq_format f,
                                   int group, int T, float* r, float* c, float* s_tensor,
                                   double* mse_trace, void* stream);

/* Device-side error word set by a kernel whose bounded wait expired
 * (0 = none).  Synchronises the current device; clear != 0 resets it. */
DQ_API int dq_device_error(int clear);

/* Time limit, in nanoseconds, of the bounded waits inside the GEMM and
 * activation-quantiser pipelines on the current device (default 2 s; ns = 0
 * restores the default).  Diagnostic: the paper has no counterpart.  A wait
 * that runs out sets the device error word to DQ_ERR_DEVICE_TIMEOUT and the
 * kernel unwinds -- every role first waits, with a fixed 2 s limit, for the
 * copies and tensor-core work it has already issued, then the CTA releases
 * its tensor memory and exits; the outputs of that call are undefined.  A
 * very small limit makes the waits of a normal call expire, which is how the
 * unwinding is tested.  Synchronises the device; do not call it while
 * another thread has work of this library in flight. */
DQ_API int dq_set_wait_limit(uint64_t ns);

/* Library version, major * 10000 + minor * 100 + patch. */
DQ_API int dq_version(void);

#ifdef __cplusplus
}
#endif
#endif /* DQ_H */
