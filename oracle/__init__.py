"""CPU oracle for the DualQuant dual-scale W4A4 path -- TEST INFRASTRUCTURE.

Only tests/, __graft_entry__.smoke() and bench.py's cpu_baseline / reference
legs may import this package.  It shares no code with the CUDA library in
w4a4_post_quantization_dual_b200 and imports nothing from it.

Source: "DualQuant: Dual-scale Calibration-free Weight-and-Activation
Quantization for LLMs" (arXiv 2610.13767).  The element-level quantisers and
Algorithm 1 live in dq_oracle.c (fp64 accumulation, fp32 quantiser
arguments); this module adds ctypes marshalling and the dequantised
reference matmul of Eq. (3) / Section 4.4 in numpy fp64.

The block-scale storage layout (sf_offset) is a hardware convention of the
block-scaled tensor-core MMA, not a result of the paper: parity unpinned
(it is checked only against its own written definition).
"""
import ctypes
import os

import numpy as np

from . import build as _build

INT4, MXINT4, MXFP4, NVFP4 = 0, 1, 2, 3
INT8, MXINT8, MXFP8 = 4, 5, 6          # 8-bit variants (Appendix G.2, Table 9)
FORMAT_NAMES = {"int4": INT4, "mxint4": MXINT4, "mxfp4": MXFP4, "nvfp4": NVFP4,
                "int8": INT8, "mxint8": MXINT8, "mxfp8": MXFP8}
NATIVE_GROUP = {INT4: 64, MXINT4: 32, MXFP4: 32, NVFP4: 16, INT8: 128, MXINT8: 32, MXFP8: 32}
EIGHT_BIT = (INT8, MXINT8, MXFP8)
BF16_SCALED = (INT4, INT8)

_lib = None

_f32p = ctypes.POINTER(ctypes.c_float)
_f64p = ctypes.POINTER(ctypes.c_double)
_u8p = ctypes.POINTER(ctypes.c_uint8)
_i64p = ctypes.POINTER(ctypes.c_int64)
_i64 = ctypes.c_int64


def lib():
    """Load (building if needed) the C oracle."""
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        sig = {
            "oracle_e2m1_value": (ctypes.c_double, [ctypes.c_int]),
            "oracle_e2m1_encode": (ctypes.c_int, [ctypes.c_float]),
            "oracle_int4_value": (ctypes.c_double, [ctypes.c_int]),
            "oracle_int4_encode": (ctypes.c_int, [ctypes.c_float]),
            "oracle_e4m3_value": (ctypes.c_double, [ctypes.c_int]),
            "oracle_int8_value": (ctypes.c_double, [ctypes.c_int]),
            "oracle_int8_encode": (ctypes.c_int, [ctypes.c_float]),
            "oracle_e4m3_elem_value": (ctypes.c_double, [ctypes.c_int]),
            "oracle_e4m3_elem_encode": (ctypes.c_int, [ctypes.c_float]),
            "oracle_ue4m3_rne": (ctypes.c_int, [ctypes.c_double]),
            "oracle_ue4m3_proj": (ctypes.c_int, [ctypes.c_double]),
            "oracle_e8m0_value": (ctypes.c_double, [ctypes.c_int]),
            "oracle_e8m0_proj": (ctypes.c_int, [ctypes.c_double]),
            "oracle_bf16_value": (ctypes.c_double, [ctypes.c_int]),
            "oracle_bf16_rne": (ctypes.c_int, [ctypes.c_double]),
            "oracle_bf16_proj": (ctypes.c_double, [ctypes.c_double]),
            "oracle_proj_alpha": (ctypes.c_double, [ctypes.c_int, ctypes.c_double, ctypes.c_float]),
            "oracle_proj_beta": (ctypes.c_double, [ctypes.c_int, ctypes.c_double]),
            "oracle_init_c": (None, [_f32p, _i64, _i64, ctypes.c_int, ctypes.c_int, _f32p]),
            "oracle_tensor_scale": (ctypes.c_float, [_f32p, _i64, _i64, _f32p]),
            "oracle_init_r": (None, [_f32p, _i64, _i64, ctypes.c_int, ctypes.c_int, _f32p,
                                     ctypes.c_float, _f32p]),
            "oracle_solve": (None, [_f32p, _i64, _i64, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                    _i64p, _i64, _f32p, _f32p, _f32p, _f64p, _f64p]),
            "oracle_solve_ex": (None, [_f32p, _i64, _i64, ctypes.c_int, ctypes.c_int,
                                       ctypes.c_int, ctypes.c_int, _f32p, _f32p, _i64p, _i64,
                                       _f32p, _f32p, _f32p, _f64p, _f64p]),
            "oracle_solve_qtrace": (None, [_f32p, _i64, _i64, ctypes.c_int, ctypes.c_int,
                                           ctypes.c_int, ctypes.c_int, _f32p, _f32p, _i64p, _i64,
                                           _f32p, _f32p, _f32p, _f64p, _f64p, _f64p, _f64p]),
            "oracle_error": (ctypes.c_double, [_f32p, _i64, _i64, ctypes.c_int, ctypes.c_int,
                                               _f32p, _f32p]),
            "oracle_error_fixed_q": (ctypes.c_double, [_f32p, _u8p, _i64, _i64, ctypes.c_int,
                                                       ctypes.c_int, _f32p, _f32p]),
            "oracle_codes": (None, [_f32p, _i64, _i64, ctypes.c_int, ctypes.c_int, _f32p, _f32p,
                                    _u8p]),
            "oracle_update_fixed_q": (None, [_f32p, _u8p, _i64, _i64, ctypes.c_int, ctypes.c_int,
                                             ctypes.c_float, _f32p, _f32p, ctypes.c_int]),
            "oracle_sf_offset": (_i64, [_i64, _i64, _i64]),
            "oracle_sf_bytes": (_i64, [_i64, _i64]),
            "oracle_pack_weight": (None, [_f32p, _i64, _i64, ctypes.c_int, ctypes.c_int, _f32p,
                                          _f32p, ctypes.c_float, _u8p, _u8p]),
            "oracle_quantize_act": (None, [_f32p, _i64, _i64, _f32p, ctypes.c_int, ctypes.c_int,
                                           _u8p, _u8p, _f32p]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _p(a, t):
    return a.ctypes.data_as(t)


def _f32(a):
    return np.ascontiguousarray(a, dtype=np.float32)


# ---------------------------------------------------------------- formats
def e2m1_value(code):
    return lib().oracle_e2m1_value(int(code))


def e2m1_encode(t):
    return lib().oracle_e2m1_encode(float(np.float32(t)))


def int4_value(code):
    return lib().oracle_int4_value(int(code))


def int4_encode(t):
    return lib().oracle_int4_encode(float(np.float32(t)))


def e4m3_value(b):
    return lib().oracle_e4m3_value(int(b))


def ue4m3_rne(x):
    return lib().oracle_ue4m3_rne(float(x))


def ue4m3_proj(u):
    return lib().oracle_ue4m3_proj(float(u))


def e8m0_value(b):
    return lib().oracle_e8m0_value(int(b))


def e8m0_proj(u):
    return lib().oracle_e8m0_proj(float(u))


def bf16_value(h):
    return lib().oracle_bf16_value(int(h))


def bf16_rne(x):
    return lib().oracle_bf16_rne(float(x))


def bf16_proj(u):
    return lib().oracle_bf16_proj(float(u))


def proj_alpha(fmt, u, s_T=1.0):
    return lib().oracle_proj_alpha(fmt, float(u), float(s_T))


def proj_beta(fmt, u):
    return lib().oracle_proj_beta(fmt, float(u))


def int8_value(code):
    return lib().oracle_int8_value(int(code))


def int8_encode(t):
    return lib().oracle_int8_encode(float(np.float32(t)))


def e4m3_elem_value(code):
    return lib().oracle_e4m3_elem_value(int(code))


def e4m3_elem_encode(t):
    return lib().oracle_e4m3_elem_encode(float(np.float32(t)))


def elem_value_table(fmt):
    """Value of each element code (16 for the 4-bit grids, 256 for 8-bit)."""
    if fmt in (INT8, MXINT8):
        return np.array([int8_value(k) for k in range(256)], dtype=np.float64)
    if fmt == MXFP8:
        return np.array([e4m3_elem_value(k) for k in range(256)], dtype=np.float64)
    f = int4_value if fmt in (INT4, MXINT4) else e2m1_value
    return np.array([f(k) for k in range(16)], dtype=np.float64)


# ---------------------------------------------------------------- solver
def init_c(W, fmt, G):
    W = _f32(W)
    m, n = W.shape
    c = np.empty(n, np.float32)
    lib().oracle_init_c(_p(W, _f32p), m, n, fmt, G, _p(c, _f32p))
    return c


def tensor_scale(W, c):
    W = _f32(W)
    m, n = W.shape
    return float(lib().oracle_tensor_scale(_p(W, _f32p), m, n, _p(_f32(c), _f32p)))


def init_r(W, fmt, G, c, s_T=1.0):
    """Format-native RTN row-block scales of W * diag(c)^-1 (c = 1: plain RTN)."""
    W = _f32(W)
    m, n = W.shape
    r = np.empty((m, n // G), np.float32)
    lib().oracle_init_r(_p(W, _f32p), m, n, fmt, G, _p(_f32(c), _f32p), float(s_T), _p(r, _f32p))
    return r


def solve(W, fmt, G, T, tiles=None):
    """Algorithm 1 on every (or the listed) m x G tile.

    Returns dict(r (m, n/G) f32, c (n,) f32, s_T float, trace (T+1,) f64 =
    normalised MSE ||W - W_hat||^2 / ||W||^2 over the solved tiles).
    """
    W = _f32(W)
    m, n = W.shape
    nb = n // G
    r = np.empty((m, nb), np.float32)
    c = np.empty(n, np.float32)
    sT = np.zeros(1, np.float32)
    err = np.zeros(T + 1, np.float64)
    w2 = np.zeros(1, np.float64)
    if tiles is None:
        tp, nt = None, 0
    else:
        tarr = np.ascontiguousarray(tiles, dtype=np.int64)
        tp, nt = _p(tarr, _i64p), len(tarr)
    lib().oracle_solve(_p(W, _f32p), m, n, fmt, G, T, tp, nt, _p(r, _f32p), _p(c, _f32p),
                       _p(sT, _f32p), _p(err, _f64p), _p(w2, _f64p))
    trace = err / w2[0] if w2[0] > 0 else err
    return {"r": r, "c": c, "s_T": float(sT[0]), "trace": trace, "err": err, "w2": float(w2[0])}


ALPHA_ONLY, BETA_ONLY, KEEP_S = 1, 2, 4


def solve_ex(W, fmt, G, T, flags=0, r0=None, c0=None, s_T=None, tiles=None):
    """Algorithm 1 with an ablation mode (ALPHA_ONLY / BETA_ONLY, Table 4)
    and optional initial scales r0 (m, n/G) / c0 (n,), projected onto the
    admissible sets; with KEEP_S the NVFP4 tensor scale s_T is given rather
    than computed.  Same return value as solve()."""
    W = _f32(W)
    m, n = W.shape
    nb = n // G
    r = np.empty((m, nb), np.float32)
    c = np.empty(n, np.float32)
    sT = np.array([s_T if s_T is not None else 0.0], np.float32)
    if (flags & KEEP_S) and s_T is None:
        raise ValueError("KEEP_S needs s_T")
    err = np.zeros(T + 1, np.float64)
    w2 = np.zeros(1, np.float64)
    if tiles is None:
        tp, nt = None, 0
    else:
        tarr = np.ascontiguousarray(tiles, dtype=np.int64)
        tp, nt = _p(tarr, _i64p), len(tarr)
    r0p = _p(_f32(np.asarray(r0).reshape(m, nb)), _f32p) if r0 is not None else None
    c0p = _p(_f32(np.asarray(c0).reshape(n)), _f32p) if c0 is not None else None
    keep = (r0p, c0p)  # noqa: F841 (keep the arrays alive through the call)
    lib().oracle_solve_ex(_p(W, _f32p), m, n, fmt, G, T, flags, r0p, c0p, tp, nt,
                          _p(r, _f32p), _p(c, _f32p), _p(sT, _f32p), _p(err, _f64p),
                          _p(w2, _f64p))
    trace = err / w2[0] if w2[0] > 0 else err
    return {"r": r, "c": c, "s_T": float(sT[0]), "trace": trace, "err": err, "w2": float(w2[0])}


def solve_qtrace(W, fmt, G, T, flags=0, tiles=None):
    """solve_ex plus the relative code change of Fig. 2(a) / Fig. 3(a):
    result["qchange"][t] = ||Qhat(t) - Qhat(t-1)||_F / ||Qhat(t-1)||_F for
    t = 1..T (entry 0 is nan), Qhat(t) the code values at the scales after
    round t, over the solved tiles."""
    W = _f32(W)
    m, n = W.shape
    nb = n // G
    r = np.empty((m, nb), np.float32)
    c = np.empty(n, np.float32)
    sT = np.zeros(1, np.float32)
    err = np.zeros(T + 1, np.float64)
    w2 = np.zeros(1, np.float64)
    qn = np.zeros(T + 1, np.float64)
    qd = np.zeros(T + 1, np.float64)
    if tiles is None:
        tp, nt = None, 0
    else:
        tarr = np.ascontiguousarray(tiles, dtype=np.int64)
        tp, nt = _p(tarr, _i64p), len(tarr)
    lib().oracle_solve_qtrace(_p(W, _f32p), m, n, fmt, G, T, flags, None, None, tp, nt,
                              _p(r, _f32p), _p(c, _f32p), _p(sT, _f32p), _p(err, _f64p),
                              _p(w2, _f64p), _p(qn, _f64p), _p(qd, _f64p))
    qc = np.full(T + 1, np.nan)
    qc[1:] = np.sqrt(qn[1:] / np.where(qd[1:] > 0, qd[1:], np.nan))
    trace = err / w2[0] if w2[0] > 0 else err
    return {"r": r, "c": c, "s_T": float(sT[0]), "trace": trace, "err": err, "w2": float(w2[0]),
            "qchange": qc}


def error(W, fmt, G, r, c):
    W = _f32(W)
    m, n = W.shape
    return lib().oracle_error(_p(W, _f32p), m, n, fmt, G, _p(_f32(r), _f32p), _p(_f32(c), _f32p))


def error_fixed_q(W, Q, fmt, G, r, c):
    W = _f32(W)
    m, n = W.shape
    Q = np.ascontiguousarray(Q, np.uint8)
    return lib().oracle_error_fixed_q(_p(W, _f32p), _p(Q, _u8p), m, n, fmt, G,
                                      _p(_f32(r), _f32p), _p(_f32(c), _f32p))


def codes(W, fmt, G, r, c):
    W = _f32(W)
    m, n = W.shape
    Q = np.empty((m, n), np.uint8)
    lib().oracle_codes(_p(W, _f32p), m, n, fmt, G, _p(_f32(r), _f32p), _p(_f32(c), _f32p),
                       _p(Q, _u8p))
    return Q


def update_fixed_q(W, Q, fmt, G, r, c, which, s_T=1.0):
    """One projected closed-form half-step with Q held fixed (Eq. 10 rows, Eq. 14 columns)."""
    W = _f32(W)
    m, n = W.shape
    r = _f32(r).copy()
    c = _f32(c).copy()
    Q = np.ascontiguousarray(Q, np.uint8)
    lib().oracle_update_fixed_q(_p(W, _f32p), _p(Q, _u8p), m, n, fmt, G, float(s_T),
                                _p(r, _f32p), _p(c, _f32p), int(which))
    return r, c


# ---------------------------------------------------------------- packing
def sf_offset(row, s, S):
    return int(lib().oracle_sf_offset(int(row), int(s), int(S)))


def sf_bytes(rows, S):
    return int(lib().oracle_sf_bytes(int(rows), int(S)))


def pack_weight(W, fmt, G, r, c, s_T=1.0):
    """Packed codes (m, n/2) u8 ((m, n) for 8-bit formats) and scales (GEMM layout
    bytes, or (m, n/G) u16 bf16 for INT4 / INT8)."""
    W = _f32(W)
    m, n = W.shape
    cod = np.empty((m, n if fmt in EIGHT_BIT else n // 2), np.uint8)
    if fmt in BF16_SCALED:
        sc = np.empty((m, n // G), np.uint16)
    else:
        sc = np.empty(sf_bytes(m, n // G), np.uint8)
    lib().oracle_pack_weight(_p(W, _f32p), m, n, fmt, G, _p(_f32(r), _f32p), _p(_f32(c), _f32p),
                             float(s_T), _p(cod, _u8p), sc.ctypes.data_as(_u8p))
    return cod, sc


def quantize_act(X, c, fmt, G):
    """Rescale by c and quantise.  Returns (codes (M, K/2) u8 ((M, K) for 8-bit
    formats), scales, s_tok (M,) f32)."""
    X = _f32(X)
    M, K = X.shape
    cod = np.empty((M, K if fmt in EIGHT_BIT else K // 2), np.uint8)
    if fmt in BF16_SCALED:
        sc = np.empty((M, K // G), np.uint16)
    else:
        sc = np.empty(sf_bytes(M, K // G), np.uint8)
    st = np.zeros(M, np.float32)
    lib().oracle_quantize_act(_p(X, _f32p), M, K, _p(_f32(c), _f32p), fmt, G, _p(cod, _u8p),
                              sc.ctypes.data_as(_u8p), _p(st, _f32p))
    return cod, sc, st


# ---------------------------------------------------------------- reference GEMM
def unpack_codes(packed, K):
    """(R, K/2) bytes -> (R, K) codes, element 2k in the low nibble of byte k
    ((R, K) bytes of an 8-bit format are returned as they are)."""
    packed = np.asarray(packed, np.uint8)
    if packed.shape[1] == K:
        return packed.copy()
    out = np.empty((packed.shape[0], K), np.uint8)
    out[:, 0::2] = packed & 0xF
    out[:, 1::2] = packed >> 4
    return out


def scale_values(sf, rows, S, fmt):
    """Decode block scales stored in the GEMM layout -> (rows, S) float64."""
    sf = np.asarray(sf, np.uint8).reshape(-1)
    rr = np.arange(rows)[:, None]
    ss = np.arange(S)[None, :]
    S4 = (S + 3) // 4
    off = ((rr // 128) * S4 + ss // 4) * 512 + (rr % 32) * 16 + ((rr % 128) // 32) * 4 + (ss % 4)
    b = sf[off]
    if fmt == NVFP4:
        tab = np.array([e4m3_value(k) for k in range(256)], np.float64)
    else:
        tab = np.array([e8m0_value(k) if k < 255 else np.nan for k in range(256)], np.float64)
    return tab[b]


def dequant(packed, sf, rows, K, fmt, G, row_scale=None):
    """Dequantised operand (rows, K) fp64 = code value x block scale (x per-row scale)."""
    q = elem_value_table(fmt)[unpack_codes(packed, K)]
    if fmt in BF16_SCALED:
        s = np.vectorize(bf16_value)(np.asarray(sf).reshape(rows, K // G).astype(np.int64))
    else:
        s = scale_values(sf, rows, K // G, fmt)
    v = q * np.repeat(s, G, axis=1)
    if row_scale is not None:
        v = v * np.asarray(row_scale, np.float64)[:, None]
    return v


def linear(A, sA, s_tok, B, sB, s_W, M, N, K, fmt, r_row=None):
    """Y = dequant(A) dequant(B)^T * s_tok[t] * s_W (* r_row[n]) in fp64 (Eq. 3, Section 4.4)."""
    G = NATIVE_GROUP[fmt]
    a = dequant(A, sA, M, K, fmt, G, s_tok if fmt == NVFP4 else None)
    b = dequant(B, sB, N, K, fmt, G)
    Y = a @ b.T
    if fmt == NVFP4:
        Y = Y * float(s_W)
    if r_row is not None:
        Y = Y * np.asarray(r_row, np.float64)[None, :]
    return Y


def act_error_sums(X, c, fmt, G):
    """Quantisation error of the activation path (Appendix E, Table 6): X is
    rescaled by c (None: without beta, c = 1), quantised by quantize_act,
    dequantised and mapped back by 1/c, all in fp64.  Returns
    (sum x^2, sum (x - x^)^2) over all elements."""
    X = _f32(X)
    M, K = X.shape
    cc = np.ones(K, np.float32) if c is None else _f32(c)
    cod, sc, st = quantize_act(X, cc, fmt, G)
    if fmt in BF16_SCALED:
        q = elem_value_table(fmt)[unpack_codes(cod, K)]
        s = np.vectorize(bf16_value)(sc.astype(np.int64))
        xt = q * np.repeat(s, G, axis=1)
    else:
        xt = dequant(cod, sc, M, K, fmt, G, st if fmt == NVFP4 else None)
    xh = xt / cc.astype(np.float64)[None, :]
    x = X.astype(np.float64)
    return float(np.sum(x * x)), float(np.sum((x - xh) ** 2))


def act_sqnr_db(X, c, fmt, G):
    """10 log10(sum x^2 / sum (x - x^)^2) of act_error_sums."""
    sx, se = act_error_sums(X, c, fmt, G)
    return 10.0 * np.log10(sx / se) if se > 0 else np.inf


def dequant_rows(packed, sf, row_idx, K, fmt, G=None):
    """Dequantised rows `row_idx` (fp64, len(row_idx) x K) of an operand whose
    codes are (R, K/2) bytes and whose scales are in the GEMM layout."""
    G = G or NATIVE_GROUP[fmt]
    rows = np.asarray(row_idx)
    S = K // G
    P = np.asarray(packed, np.uint8).reshape(-1, K // 2)[rows]
    q = elem_value_table(fmt)[unpack_codes(P, K)]
    sfa = np.asarray(sf, np.uint8).reshape(-1)
    S4 = (S + 3) // 4
    rr = rows[:, None]
    ss = np.arange(S)[None, :]
    off = ((rr // 128) * S4 + ss // 4) * 512 + (rr % 32) * 16 + ((rr % 128) // 32) * 4 + (ss % 4)
    if fmt == NVFP4:
        tab = np.array([e4m3_value(k) for k in range(256)], np.float64)
    else:
        tab = np.array([e8m0_value(k) if k < 255 else np.nan for k in range(256)], np.float64)
    return q * np.repeat(tab[sfa[off]], G, axis=1)


def linear_rows(A, sA, s_tok, B, sB, s_W, rows, M, N, K, fmt, r_row=None, cols=None):
    """Output rows `rows` (and columns `cols`, default all) of linear(), for
    sampled checks at full size."""
    rows = np.asarray(rows)
    cols = np.arange(N) if cols is None else np.asarray(cols)
    a = dequant_rows(A, sA, rows, K, fmt)
    if fmt == NVFP4:
        a = a * np.asarray(s_tok, np.float64)[rows][:, None]
    b = dequant_rows(B, sB, cols, K, fmt)
    Y = a @ b.T
    if fmt == NVFP4:
        Y = Y * float(s_W)
    if r_row is not None:
        Y = Y * np.asarray(r_row, np.float64)[cols][None, :]
    return Y
