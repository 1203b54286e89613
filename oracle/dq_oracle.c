/*
 * dq_oracle.c -- plain, slow CPU oracle for the DualQuant dual-scale W4A4 path.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
 * cpu_baseline / reference legs of bench.py may load this file's library.
 * It shares no code, header, table or constant generator with the CUDA
 * library under w4a4_post_quantization_dual_b200/csrc, and neither side
 * includes or imports the other.
 *
 * Source: "DualQuant: Dual-scale Calibration-free Weight-and-Activation
 * Quantization for LLMs" (Salmani, Sharify, Mostafa; arXiv 2610.13767).
 * Each function cites the section / equation it follows.  Element formats
 * (E2M1, E4M3, E8M0, BF16) are not defined in the paper; their value sets
 * follow the OCP Microscaling Formats (MX) v1.0 specification and the
 * IEEE-754-style bfloat16 definition.
 *
 * Precision policy: every accumulation is fp64.  Where floating point
 * decides a quantised code, the decision is taken in fp32 exactly as
 * specified below (both this oracle and the CUDA path use the same fp32
 * expression), because the paper does not fix that precision.
 *
 * Notation: r = alpha^-1 (per row and block of G columns), c = beta^-1
 * (per column).  W ~= diag_blk(r) * Q * diag(c)  (Eq. 2 written with the
 * inverse scales).  Q = proj_G(W .* beta .* alpha), Section 3 / Eq. 2.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

enum { F_INT4 = 0, F_MXINT4 = 1, F_MXFP4 = 2, F_NVFP4 = 3,
       F_INT8 = 4, F_MXINT8 = 5, F_MXFP8 = 6 };

/* Format families.  The 8-bit variants (Appendix G.2, Table 9: INT8 with
 * G = 128, MXINT8 and MXFP8 with G = 32) reuse Algorithm 1 unchanged with
 * their own element grids: INT8 integers -128..127 (Section 3's integer grid
 * with B = 8), FP8 E4M3 (OCP MX v1.0 MXFP8 element type). */
static int is_mx(int fmt) {
  return fmt == F_MXINT4 || fmt == F_MXFP4 || fmt == F_MXINT8 || fmt == F_MXFP8;
}
static int is_8bit(int fmt) { return fmt == F_INT8 || fmt == F_MXINT8 || fmt == F_MXFP8; }
/* OCP MX shared-exponent rule X = 2^(floor(log2 amax) - emax_elem):
 * emax_elem = exponent of the element grid's largest power of two
 * (E2M1 6 -> 2, INT4 7 -> 2, INT8 127 -> 6, E4M3 448 -> 8). */
static int mx_emax(int fmt) { return fmt == F_MXINT8 ? 6 : (fmt == F_MXFP8 ? 8 : 2); }

/* ------------------------------------------------------------------ */
/* Element grids (Section 3: "canonical, unit-scale grid")            */
/* ------------------------------------------------------------------ */

/* E2M1 magnitudes for codes 0..7 (OCP MX v1.0, FP4 E2M1). Bit 3 = sign. */
static const double E2M1_MAG[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

double oracle_e2m1_value(int code) {
  double m = E2M1_MAG[code & 7];
  return (code & 8) ? -m : m;
}

/* proj_G for E2M1: nearest grid magnitude by exhaustive search, ties to
 * the even code, saturating at 6 (the nearest point for |t| > 6), sign
 * kept from t (so a negative t that rounds to 0 gives code 8). */
int oracle_e2m1_encode(float t) {
  double a = fabs((double)t);
  int best = 0;
  double bd = INFINITY;
  for (int k = 0; k < 8; ++k) {
    double d = fabs(a - E2M1_MAG[k]);
    if (d < bd || (d == bd && (k % 2) == 0)) { bd = d; best = k; }
  }
  return (signbit(t) ? 8 : 0) | best;
}

/* INT4 grid: integers -8..7 (Section 3, -2^(B-1) .. 2^(B-1)-1, B = 4).
 * Code = two's-complement nibble. */
double oracle_int4_value(int code) {
  int v = code & 0xF;
  return (double)(v >= 8 ? v - 16 : v);
}

/* proj_G for INT4: nearest integer in [-8, 7] by exhaustive search, ties
 * to the even integer ("rounds and clips", Section 3). */
int oracle_int4_encode(float t) {
  double a = (double)t;
  int best = 0;
  double bd = INFINITY;
  for (int v = -8; v <= 7; ++v) {
    double d = fabs(a - (double)v);
    if (d < bd || (d == bd && (v % 2) == 0)) { bd = d; best = v; }
  }
  return best & 0xF;
}

/* INT8 grid: integers -128..127 (Section 3 with B = 8); code = the
 * two's-complement byte. */
double oracle_int8_value(int code) {
  int v = code & 0xFF;
  return (double)(v >= 128 ? v - 256 : v);
}

/* proj_G for INT8: nearest integer, ties to even (the IEEE default
 * rounding of nearbyint), clipped to [-128, 127]. */
int oracle_int8_encode(float t) {
  double v = nearbyint((double)t);
  if (v < -128.0) v = -128.0;
  if (v > 127.0) v = 127.0;
  return ((int)v) & 0xFF;
}

static int elem_encode_e4m3(float t);
static double elem_value_e4m3(int code);

static int elem_encode(int fmt, float t) {
  switch (fmt) {
    case F_INT4:
    case F_MXINT4: return oracle_int4_encode(t);
    case F_INT8:
    case F_MXINT8: return oracle_int8_encode(t);
    case F_MXFP8: return elem_encode_e4m3(t);
    default: return oracle_e2m1_encode(t);
  }
}
static double elem_value(int fmt, int code) {
  switch (fmt) {
    case F_INT4:
    case F_MXINT4: return oracle_int4_value(code);
    case F_INT8:
    case F_MXINT8: return oracle_int8_value(code);
    case F_MXFP8: return elem_value_e4m3(code);
    default: return oracle_e2m1_value(code);
  }
}

/* ------------------------------------------------------------------ */
/* Scale formats (Section 4.2: admissible sets F_alpha, F_beta)        */
/* ------------------------------------------------------------------ */

/* Unsigned E4M3 (bias 7, no infinities, 0x7F = NaN): value of byte b. */
double oracle_e4m3_value(int b) {
  int e = (b >> 3) & 0xF, m = b & 7;
  if ((b & 0x7F) == 0x7F) return NAN;
  double v = (e == 0) ? ldexp((double)m, -9) : ldexp(1.0 + m / 8.0, e - 7);
  return (b & 0x80) ? -v : v;
}

/* Nearest finite non-negative E4M3 byte to x >= 0 (0 allowed), ties to
 * the even byte, saturating at 448: exhaustive search. */
int oracle_ue4m3_rne(double x) {
  int best = 0;
  double bd = INFINITY;
  for (int b = 0; b <= 126; ++b) {
    double d = fabs(x - oracle_e4m3_value(b));
    if (d < bd || (d == bd && (b % 2) == 0)) { bd = d; best = b; }
  }
  return best;
}

/* Nearest POSITIVE E4M3 byte to u > 0 (projection onto F = UE4M3 \ {0}). */
int oracle_ue4m3_proj(double u) {
  int best = 1;
  double bd = INFINITY;
  for (int b = 1; b <= 126; ++b) {
    double d = fabs(u - oracle_e4m3_value(b));
    if (d < bd || (d == bd && (b % 2) == 0)) { bd = d; best = b; }
  }
  return best;
}

/* FP8 E4M3 element (MXFP8): value of the byte (sign bit 7), and the nearest
 * finite value to t, ties to the even byte, saturating at +-448, the sign
 * kept from t (a negative t that rounds to 0 gives 0x80). */
static double elem_value_e4m3(int code) { return oracle_e4m3_value(code & 0xFF); }
static int elem_encode_e4m3(float t) {
  return oracle_ue4m3_rne(fabs((double)t)) | (signbit(t) ? 0x80 : 0);
}
double oracle_e4m3_elem_value(int code) { return elem_value_e4m3(code); }
int oracle_e4m3_elem_encode(float t) { return elem_encode_e4m3(t); }

/* E8M0: 2^(b-127), b in 0..254. */
double oracle_e8m0_value(int b) { return ldexp(1.0, b - 127); }

/* Nearest power of two to u > 0 in linear distance; an exact midpoint
 * 1.5*2^k goes to the larger power; clamped to [2^-127, 2^127]. */
int oracle_e8m0_proj(double u) {
  int E;
  frexp(u, &E);             /* u = f * 2^E, f in [0.5, 1) */
  int k = E - 1;            /* 2^k <= u < 2^(k+1) */
  double lo = ldexp(1.0, k), hi = ldexp(1.0, k + 1);
  int kk = (u - lo < hi - u) ? k : k + 1;
  if (kk < -127) kk = -127;
  if (kk > 127) kk = 127;
  return kk + 127;
}

/* bfloat16 helpers.  Value of 16-bit pattern h. */
double oracle_bf16_value(int h) {
  uint32_t u = ((uint32_t)(h & 0xFFFF)) << 16;
  float f;
  memcpy(&f, &u, 4);
  return (double)f;
}

/* Round a finite double x to the nearest bfloat16 (ties to even
 * mantissa), saturating at the largest finite value.  Works directly from
 * the exact value (no intermediate fp32 rounding). */
int oracle_bf16_rne(double x) {
  const double maxv = oracle_bf16_value(0x7F7F);
  int neg = signbit(x) ? 1 : 0;
  double a = fabs(x);
  int h;
  if (a >= maxv) {
    h = 0x7F7F;
  } else if (a == 0.0) {
    h = 0;
  } else {
    int E;
    frexp(a, &E);
    int k = E - 1;                                     /* 2^k <= a */
    double spacing = (k < -126) ? ldexp(1.0, -133) : ldexp(1.0, k - 7);
    double m = floor(a / spacing);                     /* exact: a / 2^p */
    double lo = m * spacing, hi = (m + 1.0) * spacing;
    double pick;
    if (a - lo < hi - a) pick = lo;
    else if (a - lo > hi - a) pick = hi;
    else pick = (fmod(m, 2.0) == 0.0) ? lo : hi;
    float f = (float)pick;                              /* exact */
    uint32_t u;
    memcpy(&u, &f, 4);
    h = (int)(u >> 16);
  }
  return h | (neg ? 0x8000 : 0);
}

/* Nearest POSITIVE bfloat16 to u > 0 (never 0), as a double value. */
double oracle_bf16_proj(double u) {
  double v = oracle_bf16_value(oracle_bf16_rne(u));
  if (v == 0.0) v = ldexp(1.0, -133);
  return v;
}

/* ------------------------------------------------------------------ */
/* Projections Pi_F (Section 4.3 "projected onto the admissible set";  */
/* Appendix C, Remark 1: nearest value of the scale's inverse).        */
/* F_alpha / F_beta per format (Section 4.2): BF16 for INT4 / INT8,     */
/* E8M0 for the MX formats, UE4M3 for NVFP4 (F_alpha = s_T * UE4M3 with the */
/* per-tensor fp32 scale s_T fixed at initialisation).                 */
/* ------------------------------------------------------------------ */

/* Decision precision.  The paper fixes no precision for the projection
 * step, so the scale decision is taken on the fp32 value of the updated
 * inverse scale (the kernel's precision): u is rounded once to fp32, and for
 * NVFP4 the ratio u / s_T is one fp32 division.  Accumulations that produce
 * u stay fp64. */

/* Row-scale projection: returns r in F_alpha (as float; exactly
 * representable for every format). */
static float proj_alpha(int fmt, double u, float s_T) {
  float u32 = (float)u;
  switch (fmt) {
    case F_NVFP4: {
      volatile float x = u32 / s_T;
      double v = oracle_e4m3_value(oracle_ue4m3_proj((double)x));
      return (float)((double)s_T * v); /* one fp32 rounding of s_T * v */
    }
    case F_MXFP4:
    case F_MXINT4:
    case F_MXINT8:
    case F_MXFP8: return (float)oracle_e8m0_value(u32 > 0.0f ? oracle_e8m0_proj((double)u32) : 0);
    default: return (float)oracle_bf16_proj((double)u32);
  }
}

/* Column-scale projection: c in F_beta (decision on the fp32 value of u). */
static float proj_beta(int fmt, double u) {
  float u32 = (float)u;
  switch (fmt) {
    case F_NVFP4: return (float)oracle_e4m3_value(oracle_ue4m3_proj((double)u32));
    case F_MXFP4:
    case F_MXINT4:
    case F_MXINT8:
    case F_MXFP8: return (float)oracle_e8m0_value(u32 > 0.0f ? oracle_e8m0_proj((double)u32) : 0);
    default: return (float)oracle_bf16_proj((double)u32);
  }
}

double oracle_proj_alpha(int fmt, double u, float s_T) { return proj_alpha(fmt, u, s_T); }
double oracle_proj_beta(int fmt, double u) { return proj_beta(fmt, u); }

/* Quantiser argument in fp32: z = (w * beta_j) * alpha_ib with
 * beta = 1/c and alpha = 1/r each rounded to fp32 (Algorithm 1 forms
 * Diag(alpha) W Diag(beta) from the inverses of the stored scales). */
static inline float quant_arg(float w, float beta, float alpha) {
  volatile float p = w * beta;     /* volatile: forbid contraction/reassociation */
  volatile float z = p * alpha;
  return z;
}

static inline float inv32(float x) {
  volatile float y = 1.0f / x;
  return y;
}

/* ------------------------------------------------------------------ */
/* Initialisation (Section 5.3, "Hyperparameter selection").           */
/* The printed formulas give the inverse scales: c0_j proportional to  */
/* the column l1 norm, r0 = the format-native absmax (RTN) block scale. */
/* c0 is normalised to mean 1 over each G-column block (scale ambiguity */
/* (alpha, beta) ~ (k alpha, beta / k), Appendix C footnote) and        */
/* projected onto F_beta.                                               */
/* ------------------------------------------------------------------ */

/* Column scales c0 for all n columns. */
void oracle_init_c(const float* W, int64_t m, int64_t n, int fmt, int G, float* c) {
  double* l1 = (double*)calloc((size_t)n, sizeof(double));
  for (int64_t i = 0; i < m; ++i)
    for (int64_t j = 0; j < n; ++j) l1[j] += fabs((double)W[i * n + j]);
  for (int64_t b = 0; b < n / G; ++b) {
    double mean = 0.0;
    for (int j = 0; j < G; ++j) mean += l1[b * G + j];
    mean /= (double)G;
    for (int j = 0; j < G; ++j) {
      double v = l1[b * G + j];
      c[b * G + j] = (mean > 0.0 && v > 0.0) ? proj_beta(fmt, v / mean) : proj_beta(fmt, 1.0);
    }
  }
  free(l1);
}

/* NVFP4 per-tensor scale s_T = amax(W * beta0) / (6 * 448), in fp32.
 * Not in the paper (NVFP4's second-level scale); fixed for all rounds. */
float oracle_tensor_scale(const float* W, int64_t m, int64_t n, const float* c) {
  float amax = 0.0f;
  for (int64_t j = 0; j < n; ++j) {
    float beta = inv32(c[j]);
    for (int64_t i = 0; i < m; ++i) {
      volatile float p = W[i * n + j] * beta;
      float a = fabsf(p);
      if (a > amax) amax = a;
    }
  }
  if (amax == 0.0f) return 1.0f;
  volatile float s = amax / 2688.0f;
  return s;
}

/* Format-native RTN block scale of a block whose rescaled absmax is a. */
static float rtn_block_scale(int fmt, float a, float s_T) {
  if (a == 0.0f) return proj_alpha(fmt, 1.0, s_T);  /* degenerate convention */
  switch (fmt) {
    case F_NVFP4: {
      volatile float q = a / 6.0f;
      return proj_alpha(fmt, (double)q, s_T);
    }
    case F_MXFP4:
    case F_MXINT4:
    case F_MXINT8:
    case F_MXFP8: {
      /* OCP MX: X = 2^(floor(log2 amax) - emax_elem). */
      int E;
      frexp((double)a, &E);
      int k = (E - 1) - mx_emax(fmt);
      if (k < -127) k = -127;
      if (k > 127) k = 127;
      return (float)ldexp(1.0, k);
    }
    case F_INT8: {
      volatile float q = a / 127.0f;
      return proj_alpha(fmt, (double)q, s_T);
    }
    default: {
      volatile float q = a / 7.0f;
      return proj_alpha(fmt, (double)q, s_T);
    }
  }
}

/* r0 for the row-blocks of the given tiles. */
static void init_r_tile(const float* W, int64_t m, int64_t n, int fmt, int G, int64_t b,
                        const float* c, float s_T, float* r) {
  int64_t nb = n / G;
  for (int64_t i = 0; i < m; ++i) {
    float a = 0.0f;
    for (int j = 0; j < G; ++j) {
      int64_t col = b * G + j;
      volatile float p = W[i * n + col] * inv32(c[col]);
      float v = fabsf(p);
      if (v > a) a = v;
    }
    r[i * nb + b] = rtn_block_scale(fmt, a, s_T);
  }
}

/* r0 for every row-block (format-native RTN scales of W * diag(c)^-1).
 * With c = 1 this is the single-scale RTN baseline (Appendix F, "RTN"). */
void oracle_init_r(const float* W, int64_t m, int64_t n, int fmt, int G, const float* c,
                   float s_T, float* r) {
  for (int64_t b = 0; b < n / G; ++b) init_r_tile(W, m, n, fmt, G, b, c, s_T, r);
}

/* ------------------------------------------------------------------ */
/* Reconstruction error of one tile at (r, c), Q re-quantised at those */
/* scales: sum (W - r Q c)^2 (Eq. 4 objective, unnormalised).          */
/* ------------------------------------------------------------------ */
static double tile_error(const float* W, int64_t m, int64_t n, int fmt, int G, int64_t b,
                         const float* r, const float* c) {
  int64_t nb = n / G;
  double e = 0.0;
  for (int64_t i = 0; i < m; ++i) {
    float alpha = inv32(r[i * nb + b]);
    for (int j = 0; j < G; ++j) {
      int64_t col = b * G + j;
      float w = W[i * n + col];
      int q = elem_encode(fmt, quant_arg(w, inv32(c[col]), alpha));
      double rec = (double)r[i * nb + b] * elem_value(fmt, q) * (double)c[col];
      double d = (double)w - rec;
      e += d * d;
    }
  }
  return e;
}

/* Ablation flags (Table 4, scale ablation): ALPHA_ONLY keeps the column
 * scales fixed and runs only the row half-steps; BETA_ONLY keeps the
 * row-block scales fixed and runs only the column half-steps. */
#define ORACLE_ALPHA_ONLY 1
#define ORACLE_BETA_ONLY 2
/* Warm start with a given NVFP4 tensor scale: *s_T is read, not computed. */
#define ORACLE_KEEP_S 4

/* ------------------------------------------------------------------ */
/* Algorithm 1 on one m x G tile (columns b*G .. b*G+G-1).             */
/* Per round (Section 4.3, cycle (i)-(iv); Appendix A.2):              */
/*   Q <- Q(Diag(alpha) W Diag(beta));  R = Q Diag(beta)^-1            */
/*   r_i <- Pi(<W_i, R_i> / ||R_i||^2)   (Eq. 10 / Eq. 11)             */
/*   Q <- Q(Diag(alpha) W Diag(beta));  S = Diag(alpha)^-1 Q           */
/*   c_j <- Pi(<S_j, W_j> / ||S_j||^2)   (Eq. 14 / Eq. 15)             */
/* Degenerate rows / columns (all codes zero) take Pi(1) (Section 4.3, */
/* Assumption 1 and the convention that follows it).                   */
/* err_trace[t] (t = 0..T, may be NULL) accumulates the tile's squared */
/* error at the scales after round t (t = 0: initialisation).          */
/* flags skip the row (BETA_ONLY) or column (ALPHA_ONLY) half-step.    */
/* ------------------------------------------------------------------ */
/* Grid values of the tile's codes at the current scales, into q (m x G). */
static void tile_codes(const float* W, int64_t m, int64_t n, int fmt, int G, int64_t b,
                       const float* r, const float* c, double* q) {
  int64_t nb = n / G;
  for (int64_t i = 0; i < m; ++i)
    for (int j = 0; j < G; ++j) {
      int64_t col = b * G + j;
      q[i * G + j] = elem_value(fmt, elem_encode(fmt, quant_arg(W[i * n + col], inv32(c[col]),
                                                                  inv32(r[i * nb + b]))));
    }
}

/* qnum / qden (T+1 entries, nullable): for t >= 1 they accumulate
 * ||Qhat(t) - Qhat(t-1)||_F^2 and ||Qhat(t-1)||_F^2, Qhat(t) being the code
 * values at the scales after round t (the relative change of Fig. 2(a) /
 * Fig. 3(a) is sqrt(qnum / qden)). */
static void solve_tile_flags(const float* W, int64_t m, int64_t n, int fmt, int G, int T,
                             int64_t b, float s_T, float* r, float* c, double* err_trace,
                             int flags, double* qnum, double* qden) {
  int64_t nb = n / G;
  double* num = (double*)malloc(sizeof(double) * (size_t)G);
  double* den = (double*)malloc(sizeof(double) * (size_t)G);
  double* qprev = NULL;
  double* qcur = NULL;
  if (qnum && qden) {
    qprev = (double*)malloc(sizeof(double) * (size_t)(m * G));
    qcur = (double*)malloc(sizeof(double) * (size_t)(m * G));
    tile_codes(W, m, n, fmt, G, b, r, c, qprev);
  }
  if (err_trace) err_trace[0] += tile_error(W, m, n, fmt, G, b, r, c);
  for (int t = 1; t <= T; ++t) {
    /* row half-step */
    for (int64_t i = 0; i < m && !(flags & ORACLE_BETA_ONLY); ++i) {
      float alpha = inv32(r[i * nb + b]);
      double sn = 0.0, sd = 0.0;
      for (int j = 0; j < G; ++j) {
        int64_t col = b * G + j;
        float w = W[i * n + col];
        int q = elem_encode(fmt, quant_arg(w, inv32(c[col]), alpha));
        double R = elem_value(fmt, q) * (double)c[col];
        sn += (double)w * R;
        sd += R * R;
      }
      r[i * nb + b] = (sd > 0.0) ? proj_alpha(fmt, sn / sd, s_T) : proj_alpha(fmt, 1.0, s_T);
    }
    /* re-quantise, column half-step */
    for (int j = 0; j < G; ++j) { num[j] = 0.0; den[j] = 0.0; }
    for (int64_t i = 0; i < m && !(flags & ORACLE_ALPHA_ONLY); ++i) {
      float rr = r[i * nb + b];
      float alpha = inv32(rr);
      for (int j = 0; j < G; ++j) {
        int64_t col = b * G + j;
        float w = W[i * n + col];
        int q = elem_encode(fmt, quant_arg(w, inv32(c[col]), alpha));
        double S = (double)rr * elem_value(fmt, q);
        num[j] += S * (double)w;
        den[j] += S * S;
      }
    }
    for (int j = 0; j < G && !(flags & ORACLE_ALPHA_ONLY); ++j)
      c[b * G + j] = (den[j] > 0.0) ? proj_beta(fmt, num[j] / den[j]) : proj_beta(fmt, 1.0);
    if (err_trace) err_trace[t] += tile_error(W, m, n, fmt, G, b, r, c);
    if (qprev) {
      tile_codes(W, m, n, fmt, G, b, r, c, qcur);
      for (int64_t k = 0; k < m * G; ++k) {
        double d = qcur[k] - qprev[k];
        qnum[t] += d * d;
        qden[t] += qprev[k] * qprev[k];
      }
      double* tmp = qprev;
      qprev = qcur;
      qcur = tmp;
    }
  }
  free(num);
  free(den);
  free(qprev);
  free(qcur);
}

static void solve_tile(const float* W, int64_t m, int64_t n, int fmt, int G, int T, int64_t b,
                       float s_T, float* r, float* c, double* err_trace) {
  solve_tile_flags(W, m, n, fmt, G, T, b, s_T, r, c, err_trace, 0, NULL, NULL);
}

/* Full solve of the listed tiles (all tiles when tiles == NULL).
 * W: m x n fp32 row-major.  Outputs r (m x n/G), c (n), *s_T (NVFP4; 1
 * otherwise).  c and s_T are initialised from the WHOLE matrix (the
 * per-tensor scale needs every column); r and c are then refined only on
 * the listed tiles; other entries hold their initial values.
 * err_trace (T+1 entries, may be NULL) receives the squared error summed
 * over the listed tiles; w2 (may be NULL) receives their ||W||_F^2. */
void oracle_solve(const float* W, int64_t m, int64_t n, int fmt, int G, int T,
                  const int64_t* tiles, int64_t ntiles, float* r, float* c, float* s_T,
                  double* err_trace, double* w2) {
  int64_t nb = n / G;
  oracle_init_c(W, m, n, fmt, G, c);
  float sT = (fmt == F_NVFP4) ? oracle_tensor_scale(W, m, n, c) : 1.0f;
  *s_T = sT;
  int64_t cnt = tiles ? ntiles : nb;
  if (err_trace) for (int t = 0; t <= T; ++t) err_trace[t] = 0.0;
  double ww = 0.0;
  for (int64_t k = 0; k < cnt; ++k) {
    int64_t b = tiles ? tiles[k] : k;
    for (int64_t i = 0; i < m; ++i)
      for (int j = 0; j < G; ++j) { double v = W[i * n + b * G + j]; ww += v * v; }
  }
  if (w2) *w2 = ww;
  for (int64_t b = 0; b < nb; ++b) init_r_tile(W, m, n, fmt, G, b, c, sT, r);
  for (int64_t k = 0; k < cnt; ++k) {
    int64_t b = tiles ? tiles[k] : k;
    solve_tile(W, m, n, fmt, G, T, b, sT, r, c, err_trace);
  }
}

/* Algorithm 1 with an ablation mode and an optional warm start.
 * flags: 0 both scales (as oracle_solve), ORACLE_ALPHA_ONLY (Table 4
 * "alpha-only": beta fixed, at 1 unless c0 is given), ORACLE_BETA_ONLY
 * (Table 4 "beta-only": alpha fixed at its initial value, the format-native
 * RTN scale of W diag(c)^-1 unless r0 is given).
 * c0 (n, nullable): initial column scales, projected onto F_beta (Section
 * 4.3 projection); replaces the l1 initialisation.  The NVFP4 tensor scale
 * is then taken with these c, unless ORACLE_KEEP_S is set: then *s_T is
 * an input (NVFP4) and kept, so that a solve resumed from an earlier
 * result (r, c, s_T) continues it exactly.  r0 (m x n/G, nullable): initial
 * row-block scales, projected onto F_alpha; replaces the RTN
 * initialisation. */
static void solve_ex_impl(const float* W, int64_t m, int64_t n, int fmt, int G, int T, int flags,
                          const float* r0, const float* c0, const int64_t* tiles, int64_t ntiles,
                          float* r, float* c, float* s_T, double* err_trace, double* w2,
                          double* qnum, double* qden);

void oracle_solve_ex(const float* W, int64_t m, int64_t n, int fmt, int G, int T, int flags,
                     const float* r0, const float* c0, const int64_t* tiles, int64_t ntiles,
                     float* r, float* c, float* s_T, double* err_trace, double* w2) {
  solve_ex_impl(W, m, n, fmt, G, T, flags, r0, c0, tiles, ntiles, r, c, s_T, err_trace, w2, NULL,
                NULL);
}

/* oracle_solve_ex plus the code-change trace of Fig. 2(a): qnum[t], qden[t]
 * (T+1 entries each, entry 0 unused) as described at solve_tile_flags, summed
 * over the solved tiles. */
void oracle_solve_qtrace(const float* W, int64_t m, int64_t n, int fmt, int G, int T, int flags,
                         const float* r0, const float* c0, const int64_t* tiles, int64_t ntiles,
                         float* r, float* c, float* s_T, double* err_trace, double* w2,
                         double* qnum, double* qden) {
  for (int t = 0; t <= T; ++t) { qnum[t] = 0.0; qden[t] = 0.0; }
  solve_ex_impl(W, m, n, fmt, G, T, flags, r0, c0, tiles, ntiles, r, c, s_T, err_trace, w2, qnum,
                qden);
}

static void solve_ex_impl(const float* W, int64_t m, int64_t n, int fmt, int G, int T, int flags,
                          const float* r0, const float* c0, const int64_t* tiles, int64_t ntiles,
                          float* r, float* c, float* s_T, double* err_trace, double* w2,
                          double* qnum, double* qden) {
  int64_t nb = n / G;
  if (c0) {
    for (int64_t j = 0; j < n; ++j) c[j] = proj_beta(fmt, (double)c0[j]);
  } else if (flags & ORACLE_ALPHA_ONLY) {
    for (int64_t j = 0; j < n; ++j) c[j] = proj_beta(fmt, 1.0);
  } else {
    oracle_init_c(W, m, n, fmt, G, c);
  }
  float sT = 1.0f;
  if (fmt == F_NVFP4) sT = (flags & ORACLE_KEEP_S) ? *s_T : oracle_tensor_scale(W, m, n, c);
  *s_T = sT;
  int64_t cnt = tiles ? ntiles : nb;
  if (err_trace) for (int t = 0; t <= T; ++t) err_trace[t] = 0.0;
  double ww = 0.0;
  for (int64_t k = 0; k < cnt; ++k) {
    int64_t b = tiles ? tiles[k] : k;
    for (int64_t i = 0; i < m; ++i)
      for (int j = 0; j < G; ++j) { double v = W[i * n + b * G + j]; ww += v * v; }
  }
  if (w2) *w2 = ww;
  if (r0) {
    for (int64_t i = 0; i < m * nb; ++i) r[i] = proj_alpha(fmt, (double)r0[i], sT);
  } else {
    for (int64_t b = 0; b < nb; ++b) init_r_tile(W, m, n, fmt, G, b, c, sT, r);
  }
  for (int64_t k = 0; k < cnt; ++k) {
    int64_t b = tiles ? tiles[k] : k;
    solve_tile_flags(W, m, n, fmt, G, T, b, sT, r, c, err_trace, flags, qnum, qden);
  }
}

/* Squared reconstruction error of a whole matrix at given (r, c). */
double oracle_error(const float* W, int64_t m, int64_t n, int fmt, int G, const float* r,
                    const float* c) {
  double e = 0.0;
  for (int64_t b = 0; b < n / G; ++b) e += tile_error(W, m, n, fmt, G, b, r, c);
  return e;
}

/* Error with a FIXED code matrix Q (int8 codes, m x n): sum (W - r Q c)^2.
 * This is g(alpha, beta) of Appendix C, Eq. (16). */
double oracle_error_fixed_q(const float* W, const uint8_t* Q, int64_t m, int64_t n, int fmt,
                            int G, const float* r, const float* c) {
  int64_t nb = n / G;
  double e = 0.0;
  for (int64_t i = 0; i < m; ++i)
    for (int64_t j = 0; j < n; ++j) {
      double rec = (double)r[i * nb + j / G] * elem_value(fmt, Q[i * n + j]) * (double)c[j];
      double d = (double)W[i * n + j] - rec;
      e += d * d;
    }
  return e;
}

/* Codes Q = proj_G(W .* beta .* alpha) (unpacked, one code per byte). */
void oracle_codes(const float* W, int64_t m, int64_t n, int fmt, int G, const float* r,
                  const float* c, uint8_t* Q) {
  int64_t nb = n / G;
  for (int64_t i = 0; i < m; ++i)
    for (int64_t j = 0; j < n; ++j)
      Q[i * n + j] = (uint8_t)elem_encode(fmt, quant_arg(W[i * n + j], inv32(c[j]),
                                                          inv32(r[i * nb + j / G])));
}

/* One closed-form half-step with Q fixed (for the pins of Eqs. 10/14 and
 * Remark 1): rows (which = 0) or columns (which = 1). */
void oracle_update_fixed_q(const float* W, const uint8_t* Q, int64_t m, int64_t n, int fmt,
                           int G, float s_T, float* r, float* c, int which) {
  int64_t nb = n / G;
  if (which == 0) {
    for (int64_t i = 0; i < m; ++i)
      for (int64_t b = 0; b < nb; ++b) {
        double sn = 0.0, sd = 0.0;
        for (int j = 0; j < G; ++j) {
          int64_t col = b * G + j;
          double R = elem_value(fmt, Q[i * n + col]) * (double)c[col];
          sn += (double)W[i * n + col] * R;
          sd += R * R;
        }
        r[i * nb + b] = (sd > 0.0) ? proj_alpha(fmt, sn / sd, s_T) : proj_alpha(fmt, 1.0, s_T);
      }
  } else {
    for (int64_t j = 0; j < n; ++j) {
      double sn = 0.0, sd = 0.0;
      for (int64_t i = 0; i < m; ++i) {
        double S = (double)r[i * nb + j / G] * elem_value(fmt, Q[i * n + j]);
        sn += S * (double)W[i * n + j];
        sd += S * S;
      }
      c[j] = (sd > 0.0) ? proj_beta(fmt, sn / sd) : proj_beta(fmt, 1.0);
    }
  }
}

/* ------------------------------------------------------------------ */
/* Block-scale storage layout consumed by the block-scaled tensor-core */
/* GEMM: 128-row x 4-scale atoms of 512 bytes, atom-major along K;     */
/* inside an atom byte (row%32)*16 + ((row%128)/32)*4 + (s%4).         */
/* ------------------------------------------------------------------ */
int64_t oracle_sf_offset(int64_t row, int64_t s, int64_t S) {
  int64_t S4 = (S + 3) / 4;
  return ((row / 128) * S4 + s / 4) * 512 + (row % 32) * 16 + ((row % 128) / 32) * 4 + (s % 4);
}

int64_t oracle_sf_bytes(int64_t rows, int64_t S) { return ((rows + 127) / 128) * ((S + 3) / 4) * 512; }

/* ------------------------------------------------------------------ */
/* Weight packing (Section 4.4 artefacts; Appendix I "packed offline") */
/* codes: m x n/2 bytes, element 2k in the low nibble of byte k        */
/*        (8-bit formats: m x n bytes, one per element).                */
/* scales: NVFP4/MX -> one byte per (row, block) in the GEMM layout;   */
/*         INT4 -> bf16 bits, row-major m x n/G (uint16).               */
/* ------------------------------------------------------------------ */
void oracle_pack_weight(const float* W, int64_t m, int64_t n, int fmt, int G, const float* r,
                        const float* c, float s_T, uint8_t* codes, uint8_t* scales) {
  int64_t nb = n / G;
  if (is_8bit(fmt)) {   /* one byte per element */
    for (int64_t i = 0; i < m; ++i)
      for (int64_t j = 0; j < n; ++j)
        codes[i * n + j] = (uint8_t)elem_encode(
            fmt, quant_arg(W[i * n + j], inv32(c[j]), inv32(r[i * nb + j / G])));
  } else
  for (int64_t i = 0; i < m; ++i)
    for (int64_t j = 0; j < n; j += 2) {
      int lo = elem_encode(fmt, quant_arg(W[i * n + j], inv32(c[j]), inv32(r[i * nb + j / G])));
      int hi = elem_encode(fmt, quant_arg(W[i * n + j + 1], inv32(c[j + 1]),
                                          inv32(r[i * nb + (j + 1) / G])));
      codes[i * (n / 2) + j / 2] = (uint8_t)(lo | (hi << 4));
    }
  if (fmt == F_INT4 || fmt == F_INT8) {
    uint16_t* s16 = (uint16_t*)scales;
    for (int64_t i = 0; i < m; ++i)
      for (int64_t b = 0; b < nb; ++b) s16[i * nb + b] = (uint16_t)oracle_bf16_rne(r[i * nb + b]);
    return;
  }
  memset(scales, 0, (size_t)oracle_sf_bytes(m, nb));
  for (int64_t i = 0; i < m; ++i)
    for (int64_t b = 0; b < nb; ++b) {
      float rv = r[i * nb + b];
      int byte;
      if (fmt == F_NVFP4) {
        volatile float v = rv / s_T;
        byte = oracle_ue4m3_rne((double)v);
      } else {
        int E;
        frexp((double)rv, &E);
        byte = (E - 1) + 127;          /* exponent of the power of two r */
        if (byte < 0) byte = 0;
        if (byte > 254) byte = 254;
      }
      scales[oracle_sf_offset(i, b, nb)] = (uint8_t)byte;
    }
}

/* ------------------------------------------------------------------ */
/* Activation rescale + quantise (Eq. 3: X~ = X Diag(beta)^-1 = X      */
/* diag(c); Section 4.4: Q computes its own format-native per-row      */
/* scale on X~).  X: M x K fp32 (bf16 values), c: K.                   */
/*   NVFP4: per-token fp32 s_tok = amax(X~_t) / 2688; block byte       */
/*          = E4M3_rne(amax_blk / (6 * s_tok)); element code           */
/*          = E2M1(x~ * (1 / (dec(byte) * s_tok))).                    */
/*   MXFP4 / MXINT4: block byte = floor(log2 amax_blk) - 2 + 127;      */
/*          code = grid(x~ * 2^-e).                                    */
/*   INT4:  block scale bf16(amax_blk / 7), code = INT4(x~ / scale).   */
/*   8-bit: MXINT8 / MXFP8 as MX with emax_elem 6 / 8, INT8 with         */
/*          bf16(amax_blk / 127); codes one byte per element.          */
/* All products / quotients are single fp32 operations.                */
/* ------------------------------------------------------------------ */
void oracle_quantize_act(const float* X, int64_t M, int64_t K, const float* c, int fmt, int G,
                         uint8_t* codes, uint8_t* scales, float* s_tok) {
  int64_t S = K / G;
  float* xt = (float*)malloc(sizeof(float) * (size_t)K);
  const int bf16_scales = fmt == F_INT4 || fmt == F_INT8;
  if (!bf16_scales) memset(scales, 0, (size_t)oracle_sf_bytes(M, S));
  for (int64_t t = 0; t < M; ++t) {
    float amax = 0.0f;
    for (int64_t j = 0; j < K; ++j) {
      volatile float v = X[t * K + j] * c[j];
      xt[j] = v;
      if (fabsf(v) > amax) amax = fabsf(v);
    }
    volatile float st = amax / 2688.0f;
    if (fmt == F_NVFP4) s_tok[t] = st;
    for (int64_t s = 0; s < S; ++s) {
      float ab = 0.0f;
      for (int j = 0; j < G; ++j) {
        float v = fabsf(xt[s * G + j]);
        if (v > ab) ab = v;
      }
      float inv = 0.0f;
      int zero = 0;
      if (fmt == F_NVFP4) {
        int byte = 0;
        if (st > 0.0f) {
          volatile float d = 6.0f * st;
          volatile float sb = ab / d;
          byte = oracle_ue4m3_rne((double)sb);
        }
        scales[oracle_sf_offset(t, s, S)] = (uint8_t)byte;
        volatile float sblk = (float)oracle_e4m3_value(byte) * st;
        if (sblk == 0.0f) zero = 1; else inv = inv32(sblk);
      } else if (is_mx(fmt)) {
        int e = -127;
        if (ab > 0.0f) {
          int E;
          frexp((double)ab, &E);
          e = (E - 1) - mx_emax(fmt);
          if (e < -127) e = -127;
          if (e > 127) e = 127;
        } else {
          zero = 1;
        }
        scales[oracle_sf_offset(t, s, S)] = (uint8_t)(e + 127);
        inv = (float)ldexp(1.0, -e);
      } else {
        volatile float q = ab / (fmt == F_INT8 ? 127.0f : 7.0f);
        int h = oracle_bf16_rne((double)q);
        ((uint16_t*)scales)[t * S + s] = (uint16_t)h;
        float sc = (float)oracle_bf16_value(h);
        if (sc == 0.0f) zero = 1; else inv = inv32(sc);
      }
      if (is_8bit(fmt)) {   /* one byte per element */
        for (int j = 0; j < G; ++j) {
          int q = 0;
          if (!zero) {
            volatile float a0 = xt[s * G + j] * inv;
            q = elem_encode(fmt, a0);
          }
          codes[t * K + s * G + j] = (uint8_t)q;
        }
        continue;
      }
      for (int j = 0; j < G; j += 2) {
        int lo = 0, hi = 0;
        if (!zero) {
          volatile float a0 = xt[s * G + j] * inv;
          volatile float a1 = xt[s * G + j + 1] * inv;
          lo = elem_encode(fmt, a0);
          hi = elem_encode(fmt, a1);
        }
        codes[t * (K / 2) + (s * G + j) / 2] = (uint8_t)(lo | (hi << 4));
      }
    }
  }
  free(xt);
}
