"""Pins for the oracle's Algorithm 1 (CPU only).

The objective is evaluated here independently of the oracle: numpy fp32
products for the quantiser argument, ml_dtypes (E2M1) or numpy rint+clip
(INT4) for the grid projection, numpy fp64 for the error.  Each closed-form
update is checked against exhaustive / random search over the admissible
scale set, the descent property of Theorem 1 / Remark 1 is checked at every
half-step, and special cases with a known answer are checked exactly.
"""
import ml_dtypes
import numpy as np
import pytest

import oracle as O
from w4a4_post_quantization_dual_b200 import synth

FMTS = [(O.NVFP4, 16), (O.MXFP4, 32), (O.MXINT4, 32), (O.INT4, 64)]


# ------------------------------------------------------------ independent evaluator
def grid_value(fmt, z):
    z = np.asarray(z, np.float32)
    if fmt in (O.INT4, O.MXINT4):
        return np.clip(np.rint(z), -8, 7).astype(np.float64)
    return z.astype(ml_dtypes.float4_e2m1fn).astype(np.float64)


def quant_values(W, r, c, fmt, G):
    """proj_G((W * (1/c)) * (1/r)) with fp32 products, as values."""
    W = np.asarray(W, np.float32)
    beta = (np.float32(1.0) / np.asarray(c, np.float32)).astype(np.float32)
    alpha = (np.float32(1.0) / np.asarray(r, np.float32)).astype(np.float32)
    z = (W * beta[None, :]).astype(np.float32)
    z = (z * np.repeat(alpha, G, axis=1)).astype(np.float32)
    return grid_value(fmt, z)


def err_true(W, r, c, fmt, G):
    q = quant_values(W, r, c, fmt, G)
    rec = np.repeat(np.asarray(r, np.float64), G, axis=1) * q * np.asarray(c, np.float64)[None, :]
    return float(np.sum((np.asarray(W, np.float64) - rec) ** 2))


def qvals_from_codes(Q, fmt):
    return O.elem_value_table(fmt)[Q]


def admissible_alpha(fmt, s_T, around=None):
    if fmt == O.NVFP4:
        return np.float32(s_T) * np.array([O.e4m3_value(b) for b in range(1, 127)], np.float32)
    if fmt in (O.MXFP4, O.MXINT4):
        return np.array([2.0 ** (b - 127) for b in range(255)], np.float64)
    h = O.bf16_rne(around)
    return np.array([O.bf16_value(k) for k in range(max(1, h - 300), min(0x7F7F, h + 300))])


def admissible_beta(fmt, around=None):
    if fmt == O.NVFP4:
        return np.array([O.e4m3_value(b) for b in range(1, 127)], np.float64)
    return admissible_alpha(fmt, 1.0, around)


def make_matrix(m, n, seed, outliers=4):
    W, _ = synth.student_t_weight(m, n, seed, std=0.02, unit_variance=False,
                                  outlier_cols=outliers, outlier_scale=20.0, bf16=False)
    return W


# ------------------------------------------------------------ objective agreement
@pytest.mark.parametrize("fmt,G", FMTS)
def test_oracle_objective_matches_independent_evaluator(fmt, G):
    W = make_matrix(32, 128, 11)
    res = O.solve(W, fmt, G, 5)
    assert O.error(W, fmt, G, res["r"], res["c"]) == pytest.approx(
        err_true(W, res["r"], res["c"], fmt, G), rel=1e-12)
    Q = O.codes(W, fmt, G, res["r"], res["c"])
    assert np.array_equal(qvals_from_codes(Q, fmt), quant_values(W, res["r"], res["c"], fmt, G))


# ------------------------------------------------------------ closed forms (Eqs. 10, 14) + Remark 1
@pytest.mark.parametrize("fmt,G", FMTS)
def test_row_update_is_argmin_over_admissible_set(fmt, G):
    W = make_matrix(8, 2 * G, 12)
    res = O.solve(W, fmt, G, 2)
    r, c, sT = res["r"], res["c"], res["s_T"]
    Q = O.codes(W, fmt, G, r, c)
    q = qvals_from_codes(Q, fmt)
    r2, _ = O.update_fixed_q(W, Q, fmt, G, r, c, 0, sT)
    Wd = W.astype(np.float64)
    for i in range(W.shape[0]):
        for b in range(W.shape[1] // G):
            sl = slice(b * G, (b + 1) * G)
            R = q[i, sl] * c[sl].astype(np.float64)
            cand = admissible_alpha(fmt, sT, r2[i, b]).astype(np.float64)
            errs = ((Wd[i, sl][None, :] - cand[:, None] * R[None, :]) ** 2).sum(1)
            mine = ((Wd[i, sl] - float(r2[i, b]) * R) ** 2).sum()
            assert mine <= errs.min() * (1 + 1e-12) + 1e-30


@pytest.mark.parametrize("fmt,G", FMTS)
def test_column_update_is_argmin_over_admissible_set(fmt, G):
    W = make_matrix(24, 2 * G, 13)
    res = O.solve(W, fmt, G, 2)
    r, c, sT = res["r"], res["c"], res["s_T"]
    Q = O.codes(W, fmt, G, r, c)
    q = qvals_from_codes(Q, fmt)
    _, c2 = O.update_fixed_q(W, Q, fmt, G, r, c, 1, sT)
    Wd = W.astype(np.float64)
    S = np.repeat(r.astype(np.float64), G, axis=1) * q
    for j in range(W.shape[1]):
        cand = admissible_beta(fmt, c2[j]).astype(np.float64)
        errs = ((Wd[:, j][None, :] - cand[:, None] * S[None, :, j]) ** 2).sum(1)
        mine = ((Wd[:, j] - float(c2[j]) * S[:, j]) ** 2).sum()
        assert mine <= errs.min() * (1 + 1e-12) + 1e-30


def test_update_beats_random_perturbations():
    """Each projected closed-form update beats >= 1000 random admissible
    perturbations of its coordinate with Q fixed (Eqs. 10/14, Remark 1)."""
    fmt, G = O.NVFP4, 16
    W = make_matrix(16, 64, 14)
    res = O.solve(W, fmt, G, 3)
    r, c, sT = res["r"], res["c"], res["s_T"]
    Q = O.codes(W, fmt, G, r, c)
    r2, c2 = O.update_fixed_q(W, Q, fmt, G, r, c, 0, sT)
    base = O.error_fixed_q(W, Q, fmt, G, r2, c)
    g = np.random.default_rng(0)
    cand = admissible_alpha(fmt, sT)
    for _ in range(1000):
        rp = r2.copy()
        i, b = g.integers(0, rp.shape[0]), g.integers(0, rp.shape[1])
        rp[i, b] = cand[g.integers(0, len(cand))]
        assert O.error_fixed_q(W, Q, fmt, G, rp, c) >= base * (1 - 1e-12)
    _, c3 = O.update_fixed_q(W, Q, fmt, G, r2, c, 1, sT)
    base = O.error_fixed_q(W, Q, fmt, G, r2, c3)
    candb = admissible_beta(fmt)
    for _ in range(1000):
        cp = c3.copy()
        cp[g.integers(0, len(cp))] = candb[g.integers(0, len(candb))]
        assert O.error_fixed_q(W, Q, fmt, G, r2, cp) >= base * (1 - 1e-12)


def test_closed_form_matches_scalar_minimiser():
    """Unconstrained optimum of ||W_i - u R_i||^2 found by a library 1-D
    minimiser lies within half a bf16 step of the projected update (INT4
    rows project onto BF16, so the update is that optimum rounded)."""
    from scipy.optimize import minimize_scalar
    fmt, G = O.INT4, 64
    W = make_matrix(6, 128, 15)
    res = O.solve(W, fmt, G, 1)
    r, c = res["r"], res["c"]
    Q = O.codes(W, fmt, G, r, c)
    q = qvals_from_codes(Q, fmt)
    r2, _ = O.update_fixed_q(W, Q, fmt, G, r, c, 0)
    for i in range(6):
        for b in range(2):
            sl = slice(b * G, (b + 1) * G)
            R = q[i, sl] * c[sl]
            f = lambda u: float(((W[i, sl].astype(np.float64) - u * R) ** 2).sum())
            u0 = float(r2[i, b])
            opt = minimize_scalar(f, bracket=(u0 * 0.9, u0 * 1.1), tol=1e-14)
            assert abs(opt.x - u0) <= u0 * 2.0 ** -8 * 1.01


# ------------------------------------------------------------ descent (Theorem 1(i), Remark 1)
@pytest.mark.parametrize("fmt,G", FMTS)
def test_mse_non_increasing_every_half_step(fmt, G):
    W = make_matrix(64, 4 * G, 16)
    T = 6
    res0 = O.solve(W, fmt, G, 0)
    r, c, sT = res0["r"].copy(), res0["c"].copy(), res0["s_T"]
    e_prev = err_true(W, r, c, fmt, G)
    for _ in range(T):
        Q = O.codes(W, fmt, G, r, c)
        r, _ = O.update_fixed_q(W, Q, fmt, G, r, c, 0, sT)
        e_fixed = O.error_fixed_q(W, Q, fmt, G, r, c)
        assert e_fixed <= e_prev * (1 + 1e-9)
        e_req = err_true(W, r, c, fmt, G)            # re-quantised at the new r
        assert e_req <= e_fixed * (1 + 1e-9)
        Q = O.codes(W, fmt, G, r, c)
        _, c = O.update_fixed_q(W, Q, fmt, G, r, c, 1, sT)
        e_fixed = O.error_fixed_q(W, Q, fmt, G, r, c)
        assert e_fixed <= e_req * (1 + 1e-9)
        e_prev = err_true(W, r, c, fmt, G)
        assert e_prev <= e_fixed * (1 + 1e-9)
    # the oracle's fused solver follows exactly the same half-steps
    res = O.solve(W, fmt, G, T)
    assert np.array_equal(res["r"], r) and np.array_equal(res["c"], c)
    assert res["err"][-1] == pytest.approx(e_prev, rel=1e-12)


@pytest.mark.parametrize("fmt,G", FMTS)
def test_trace_monotone_and_plateaus(fmt, G):
    """Normalised MSE decreases monotonically and flattens (Fig. 2(b))."""
    W = make_matrix(256, 256, 17)
    res = O.solve(W, fmt, G, 30)
    tr = res["trace"]
    assert np.all(np.diff(tr) <= tr[:-1] * 1e-9)
    assert tr[-1] < tr[0]
    assert (tr[20] - tr[30]) <= 0.02 * tr[20]


# ------------------------------------------------------------ special cases
@pytest.mark.parametrize("fmt,G", FMTS)
def test_exactly_representable_weight_is_a_fixed_point(fmt, G):
    """W = diag_blk(r*) Q* with the grid maximum in every row-block and equal
    column l1 norms inside each tile (magnitudes follow a cyclic Latin
    pattern, r* constant on groups of G rows), so c0 = 1 and RTN recovers
    (r*, Q*): the error is 0 (NVFP4: within fp32 rounding of its
    tensor-scaled row scale) and Algorithm 1 stays at that point."""
    g = np.random.default_rng(21)
    m, n = 2 * G, 2 * G
    if fmt in (O.MXFP4, O.NVFP4):
        mags = np.array([6.0, 4.0, 3.0, 2.0, 1.5, 1.0, 0.5, 0.0])
    else:
        mags = np.array([7.0, 6.0, 5.0, 4.0, 3.0, 2.0, 1.0, 0.0])  # never -8: keeps amax = 7 r*
    P = np.resize(mags, G)
    i = np.arange(m)[:, None]
    j = np.arange(n)[None, :]
    q = P[(i + j) % G] * np.where(g.random((m, n)) < 0.5, -1.0, 1.0)
    rstar = 2.0 ** g.integers(-12, -4, size=(m // G, n // G))
    rstar = np.repeat(rstar, G, axis=0)
    W = (np.repeat(rstar, G, axis=1) * q).astype(np.float32)
    res = O.solve(W, fmt, G, 10)
    assert np.all(res["c"] == 1.0)
    Qc = O.codes(W, fmt, G, res["r"], res["c"])
    assert np.array_equal(O.elem_value_table(fmt)[Qc], q)
    w2 = float(np.sum(W.astype(np.float64) ** 2))
    tol = 0.0 if fmt != O.NVFP4 else 1e-12 * w2
    assert np.all(res["err"] <= tol)
    if fmt != O.NVFP4:
        assert np.array_equal(res["r"], rstar.astype(np.float32))


def test_mx_scale_equivariance():
    """W -> 2^k W leaves the codes unchanged and multiplies r by 2^k (E8M0
    scales are powers of two)."""
    for fmt in (O.MXFP4, O.MXINT4):
        W = make_matrix(64, 128, 22)
        a = O.solve(W, fmt, 32, 8)
        b = O.solve(W * np.float32(2.0 ** 5), fmt, 32, 8)
        assert np.array_equal(b["r"], a["r"] * np.float32(32.0))
        assert np.array_equal(b["c"], a["c"])
        assert np.array_equal(O.codes(W, fmt, 32, a["r"], a["c"]),
                              O.codes(W * np.float32(32.0), fmt, 32, b["r"], b["c"]))


def test_degenerate_rows_columns_and_zero_matrix():
    fmt, G = O.MXFP4, 32
    W = make_matrix(8, 64, 23)
    W[3, 0:32] = 0.0        # an all-zero row-block
    W[:, 40] = 0.0          # an all-zero column
    res = O.solve(W, fmt, G, 4)
    assert res["r"][3, 0] == 1.0
    assert res["c"][40] == 1.0
    Z = np.zeros((8, 64), np.float32)
    z = O.solve(Z, O.NVFP4, 16, 3)
    assert np.all(z["c"] == 1.0) and z["s_T"] == 1.0
    assert np.all(z["r"] == np.float32(O.e4m3_value(O.ue4m3_proj(1.0))))
    assert np.all(z["err"] == 0.0)


def test_brute_force_window_on_4x8():
    """4 x 8 matrix, one block (G = 8, E8M0 scales): exhaustive search of the
    true objective (Eq. 4) over a 3-exponent window around every one of the
    12 scales (3^12 combinations).  BCD's value must equal the independent
    evaluation at its point, no window point may be better than the
    exhaustive minimum, and BCD must land within 10 % of that minimum."""
    fmt, G = O.MXFP4, 8
    W = make_matrix(4, 8, 24, outliers=1)
    res = O.solve(W, fmt, G, 20)
    r0, c0 = res["r"][:, 0].astype(np.float64), res["c"].astype(np.float64)
    e_bcd = err_true(W, res["r"], res["c"], fmt, G)
    assert e_bcd == pytest.approx(res["err"][-1], rel=1e-12)
    steps = np.array([0.5, 1.0, 2.0])
    import itertools
    rs = np.array(list(itertools.product(steps, repeat=4))) * r0[None, :]     # 81 x 4
    cs = np.array(list(itertools.product(steps, repeat=8))) * c0[None, :]     # 6561 x 8
    Wd = W.astype(np.float64)
    best = np.inf
    for rr in rs:
        alpha = (np.float32(1) / rr.astype(np.float32)).astype(np.float32)
        beta = (np.float32(1) / cs.astype(np.float32)).astype(np.float32)        # 6561 x 8
        z = (W[None, :, :] * beta[:, None, :]).astype(np.float32)
        z = (z * alpha[None, :, None]).astype(np.float32)
        q = grid_value(fmt, z)
        rec = rr[None, :, None] * q * cs[:, None, :]
        e = ((Wd[None] - rec) ** 2).sum(axis=(1, 2))
        best = min(best, float(e.min()))
    assert best <= e_bcd * (1 + 1e-12)
    assert e_bcd <= 1.10 * best


def test_dual_scale_vs_rtn_on_outlier_tile():
    """Qualitative (Fig. 1, Table 4).  With the fine scale sets (UE4M3 for
    NVFP4, BF16 for INT4) the dual-scale solution has a much lower weight
    MSE than single-scale RTN (c = 1, format-native absmax row-block scales).
    For every format Algorithm 1 never ends above its own initial point
    (Theorem 1(i)).  With E8M0's factor-2 steps the closed-form moves are
    local, so the MX formats are only required not to increase their own
    initial error."""
    W = make_matrix(256, 256, 0)
    for fmt, G in FMTS:
        res = O.solve(W, fmt, G, 20)
        assert res["err"][-1] <= res["err"][0]
        if fmt in (O.NVFP4, O.INT4):
            ones = np.ones(256, np.float32)
            sT = O.tensor_scale(W, ones) if fmt == O.NVFP4 else 1.0
            e_rtn = err_true(W, O.init_r(W, fmt, G, ones, sT), ones, fmt, G)
            assert res["err"][-1] * 1.5 < e_rtn
