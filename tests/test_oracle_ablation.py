"""Pins for the oracle's ablation modes and warm start (CPU only).

DualQuant, Table 4 (scale ablation): "alpha-only" keeps beta = 1 and
optimises the row-block scales alone; "beta-only" keeps alpha at its
initial value and optimises the column scales alone.  Section 5.3 names
the initialisation (alpha_0, beta_0) as a hyper-parameter; a warm start
replaces it by given scales, projected onto the admissible sets.

Independent evaluation: the RTN starting point, the projections and the
objective are recomputed here with numpy / ml_dtypes; the descent property
of Theorem 1 is checked on every trace; resuming from a stored result must
continue the iteration exactly (the state of Algorithm 1 between rounds is
(r, c) alone, and s_T is fixed at initialisation).
"""
import ml_dtypes
import numpy as np
import pytest

import oracle as O
from w4a4_post_quantization_dual_b200 import synth

FMTS = [(O.NVFP4, 16), (O.MXFP4, 32), (O.MXINT4, 32), (O.INT4, 64)]


def make_matrix(m, n, seed, outliers=4):
    W, _ = synth.student_t_weight(m, n, seed, std=0.02, unit_variance=False,
                                  outlier_cols=outliers, outlier_scale=20.0, bf16=False)
    return W


def grid_value(fmt, z):
    z = np.asarray(z, np.float32)
    if fmt in (O.INT4, O.MXINT4):
        return np.clip(np.rint(z), -8, 7).astype(np.float64)
    return z.astype(ml_dtypes.float4_e2m1fn).astype(np.float64)


def err_true(W, r, c, fmt, G):
    beta = (np.float32(1.0) / np.asarray(c, np.float32)).astype(np.float32)
    alpha = (np.float32(1.0) / np.asarray(r, np.float32)).astype(np.float32)
    z = (np.asarray(W, np.float32) * beta[None, :]).astype(np.float32)
    z = (z * np.repeat(alpha, G, axis=1)).astype(np.float32)
    q = grid_value(fmt, z)
    rec = np.repeat(np.asarray(r, np.float64), G, axis=1) * q * np.asarray(c, np.float64)[None, :]
    return float(np.sum((np.asarray(W, np.float64) - rec) ** 2))


def e4m3_rne(x):
    """UE4M3 value nearest to x > 0 (ties to even), at least the smallest
    subnormal 2^-9, at most 448."""
    v = np.asarray(x, np.float32).astype(ml_dtypes.float8_e4m3fn).astype(np.float64)
    return np.clip(np.where(v > 0, v, 2.0 ** -9), 2.0 ** -9, 448.0)


def pow2_nearest(x):
    """Nearest power of two (ties at 1.5 * 2^k go up), the E8M0 projection."""
    x = np.asarray(x, np.float64)
    k = np.floor(np.log2(x))
    return np.where(x >= 1.5 * 2.0 ** k, 2.0 ** (k + 1), 2.0 ** k)


def bf16_rne(x):
    return np.asarray(x, np.float32).astype(ml_dtypes.bfloat16).astype(np.float64)


def rtn_scales(W, fmt, G):
    """Single-scale RTN (Appendix F baseline): beta = 1, format-native
    absmax row-block scale; NVFP4 with the per-tensor scale amax/2688."""
    W = np.asarray(W, np.float32)
    m, n = W.shape
    a = np.abs(W).reshape(m, n // G, G).max(axis=2)
    sT = np.float32(1.0)
    if fmt == O.NVFP4:
        sT = np.float32(np.abs(W).max()) / np.float32(2688.0)
        u = (a / np.float32(6.0)).astype(np.float32) / sT
        r = (np.float64(sT) * e4m3_rne(u.astype(np.float32))).astype(np.float32)
    elif fmt in (O.MXFP4, O.MXINT4):
        r = (2.0 ** (np.floor(np.log2(a.astype(np.float64))) - 2)).astype(np.float32)
    else:
        r = bf16_rne((a / np.float32(7.0)).astype(np.float32)).astype(np.float32)
    return r, float(sT)


# ------------------------------------------------------------ default mode
@pytest.mark.parametrize("fmt,G", FMTS)
def test_no_flags_is_algorithm_1(fmt, G):
    W = make_matrix(64, 4 * G, 30)
    a = O.solve(W, fmt, G, 6)
    b = O.solve_ex(W, fmt, G, 6)
    assert np.array_equal(a["r"], b["r"]) and np.array_equal(a["c"], b["c"])
    assert a["s_T"] == b["s_T"] and np.array_equal(a["err"], b["err"])


# ------------------------------------------------------------ alpha-only
@pytest.mark.parametrize("fmt,G", FMTS)
def test_alpha_only_starts_at_rtn_and_keeps_beta_one(fmt, G):
    """T = 0 alpha-only is the single-scale RTN quantiser exactly; every
    round keeps c = 1 and never raises the error (Theorem 1 restricted to
    the row block)."""
    W = make_matrix(128, 8 * G, 31)
    r_rtn, sT = rtn_scales(W, fmt, G)
    z = O.solve_ex(W, fmt, G, 0, flags=O.ALPHA_ONLY)
    assert np.all(z["c"] == 1.0)
    assert z["s_T"] == sT
    assert np.array_equal(z["r"], r_rtn)
    assert z["err"][0] == pytest.approx(err_true(W, r_rtn, np.ones(W.shape[1]), fmt, G),
                                        rel=1e-12)
    res = O.solve_ex(W, fmt, G, 12, flags=O.ALPHA_ONLY)
    assert np.all(res["c"] == 1.0)
    assert np.all(np.diff(res["err"]) <= res["err"][:-1] * 1e-9)
    assert res["err"][-1] == pytest.approx(err_true(W, res["r"], res["c"], fmt, G), rel=1e-12)
    # the row update is a closed form in r alone: a second solve from the
    # result makes no further row move once the codes stop changing
    if np.array_equal(res["err"][-2:], res["err"][-1:].repeat(2)):
        again = O.solve_ex(W, fmt, G, 1, flags=O.ALPHA_ONLY | O.KEEP_S, r0=res["r"],
                           c0=res["c"], s_T=res["s_T"])
        assert np.array_equal(again["r"], res["r"])


@pytest.mark.parametrize("fmt,G", FMTS)
def test_alpha_only_rounds_are_row_half_steps(fmt, G):
    """Each alpha-only round is the row half-step of Algorithm 1 (Eq. 10 /
    Eq. 11 with its projection) at c = 1, nothing else."""
    W = make_matrix(64, 4 * G, 32)
    res = O.solve_ex(W, fmt, G, 0, flags=O.ALPHA_ONLY)
    r, c, sT = res["r"].copy(), res["c"].copy(), res["s_T"]
    for _ in range(5):
        Q = O.codes(W, fmt, G, r, c)
        r, _ = O.update_fixed_q(W, Q, fmt, G, r, c, 0, sT)
    five = O.solve_ex(W, fmt, G, 5, flags=O.ALPHA_ONLY)
    assert np.array_equal(five["r"], r)


# ------------------------------------------------------------ beta-only
@pytest.mark.parametrize("fmt,G", FMTS)
def test_beta_only_keeps_initial_row_scales(fmt, G):
    W = make_matrix(128, 8 * G, 33)
    init = O.solve_ex(W, fmt, G, 0)
    res = O.solve_ex(W, fmt, G, 12, flags=O.BETA_ONLY)
    assert np.array_equal(res["r"], init["r"])
    assert res["s_T"] == init["s_T"]
    assert np.all(np.diff(res["err"]) <= res["err"][:-1] * 1e-9)
    assert res["err"][-1] == pytest.approx(err_true(W, res["r"], res["c"], fmt, G), rel=1e-12)
    # each round is the column half-step (Eq. 14 / Eq. 15) at the fixed r
    r, c, sT = init["r"].copy(), init["c"].copy(), init["s_T"]
    for _ in range(12):
        Q = O.codes(W, fmt, G, r, c)
        _, c = O.update_fixed_q(W, Q, fmt, G, r, c, 1, sT)
    assert np.array_equal(res["c"], c)


# ------------------------------------------------------------ Table 4 ordering
def test_table4_weight_mse_ordering():
    """Weight MSE on outlier-heavy layers: optimising both scales is never
    worse than beta-only, and alpha-only (a descent from RTN) never worse
    than RTN.  With the fine scale sets (UE4M3, BF16) both beats alpha-only
    too, the order of Table 4's accuracy columns."""
    for seed in range(2):
        W = make_matrix(256, 512, 40 + seed)
        for fmt, G in FMTS:
            both = O.solve_ex(W, fmt, G, 15)["trace"][-1]
            beta = O.solve_ex(W, fmt, G, 15, flags=O.BETA_ONLY)["trace"][-1]
            alpha = O.solve_ex(W, fmt, G, 15, flags=O.ALPHA_ONLY)["trace"][-1]
            rtn = O.solve_ex(W, fmt, G, 0, flags=O.ALPHA_ONLY)["trace"][0]
            assert both <= beta
            assert alpha <= rtn
            if fmt in (O.NVFP4, O.INT4):
                assert both < alpha


# ------------------------------------------------------------ warm start
@pytest.mark.parametrize("fmt,G", FMTS)
def test_warm_start_projects_given_scales(fmt, G):
    """Given c0 / r0 are projected onto F_beta / F_alpha (nearest admissible
    value), and the NVFP4 tensor scale is taken from W diag(c0)^-1."""
    g = np.random.default_rng(34)
    W = make_matrix(64, 4 * G, 35)
    m, n = W.shape
    c0 = np.exp(g.uniform(-2, 2, n)).astype(np.float32)
    res = O.solve_ex(W, fmt, G, 0, c0=c0)
    if fmt == O.NVFP4:
        c_exp = e4m3_rne(c0)
        sT = np.float32(np.abs((W * (np.float32(1) / c_exp.astype(np.float32)))
                               .astype(np.float32)).max()) / np.float32(2688.0)
        assert res["s_T"] == float(sT)
    elif fmt in (O.MXFP4, O.MXINT4):
        c_exp = pow2_nearest(c0)
    else:
        c_exp = bf16_rne(c0)
    assert np.array_equal(res["c"].astype(np.float64), c_exp)
    fixed = O.solve_ex(W, fmt, G, 3, flags=O.ALPHA_ONLY, c0=c0)   # beta stays at Pi(c0)
    assert np.array_equal(fixed["c"].astype(np.float64), c_exp)
    r0 = (np.abs(W).reshape(m, n // G, G).max(axis=2) * g.uniform(0.05, 0.5, (m, n // G)))
    r0 = r0.astype(np.float32)
    res = O.solve_ex(W, fmt, G, 0, r0=r0, c0=c0)
    sT = np.float32(res["s_T"])
    if fmt == O.NVFP4:
        r_exp = (np.float64(sT) * e4m3_rne((r0 / sT).astype(np.float32))).astype(np.float32)
    elif fmt in (O.MXFP4, O.MXINT4):
        r_exp = pow2_nearest(r0).astype(np.float32)
    else:
        r_exp = bf16_rne(r0).astype(np.float32)
    assert np.array_equal(res["r"], r_exp)
    assert res["err"][0] == pytest.approx(err_true(W, res["r"], res["c"], fmt, G), rel=1e-12)


@pytest.mark.parametrize("fmt,G", FMTS)
@pytest.mark.parametrize("flags", [0, O.ALPHA_ONLY, O.BETA_ONLY])
def test_resume_continues_exactly(fmt, G, flags):
    """Solving T1 rounds, then resuming from (r, c, s_T) for T2 rounds, ends
    exactly where T1 + T2 rounds end, with the same error trace."""
    W = make_matrix(96, 4 * G, 36)
    full = O.solve_ex(W, fmt, G, 9, flags=flags)
    part = O.solve_ex(W, fmt, G, 4, flags=flags)
    rest = O.solve_ex(W, fmt, G, 5, flags=flags | O.KEEP_S, r0=part["r"], c0=part["c"],
                      s_T=part["s_T"])
    assert np.array_equal(rest["r"], full["r"]) and np.array_equal(rest["c"], full["c"])
    assert rest["s_T"] == full["s_T"]
    assert np.array_equal(rest["err"], full["err"][4:])


def test_keep_s_uses_the_given_tensor_scale():
    """NVFP4 warm start with KEEP_S: the given s_T is used for the row-scale
    set s_T * UE4M3 instead of amax(W diag(c)^-1) / 2688."""
    W = make_matrix(64, 64, 37)
    base = O.solve_ex(W, O.NVFP4, 16, 3)
    s_given = np.float32(base["s_T"] * 1.37)
    res = O.solve_ex(W, O.NVFP4, 16, 0, flags=O.KEEP_S, r0=base["r"], c0=base["c"],
                     s_T=float(s_given))
    assert res["s_T"] == float(s_given)
    r_exp = (np.float64(s_given) * e4m3_rne((base["r"] / s_given).astype(np.float32)))
    assert np.array_equal(res["r"], r_exp.astype(np.float32))
    assert np.array_equal(res["c"], base["c"])
