"""Pins for the oracle's 8-bit variants (CPU only): INT8 (G = 128, bf16
scales), MXINT8 and MXFP8 (G = 32, E8M0 scales) of DualQuant's Appendix
G.2 / Table 9, through the same Algorithm 1.

Element grids are checked against numpy (INT8: rint half-even + clip) and
ml_dtypes (FP8 E4M3); the objective is evaluated independently in numpy;
each closed-form update is the argmin over its admissible set with Q fixed;
the descent property of Theorem 1 holds at every half-step; exactly
representable weights are fixed points; MX solves are scale-equivariant;
the activation quantiser and the packer follow their rules with library
codecs."""
import ml_dtypes
import numpy as np
import pytest

import oracle as O
from w4a4_post_quantization_dual_b200 import synth

FMTS8 = [(O.INT8, 128), (O.MXINT8, 32), (O.MXFP8, 32)]
EMAX = {O.MXINT8: 6, O.MXFP8: 8}
QMAX = {O.INT8: 127.0, O.MXINT8: 127.0, O.MXFP8: 448.0}


def grid_value(fmt, z):
    z = np.asarray(z, np.float32)
    if fmt == O.MXFP8:
        return np.clip(z, -448, 448).astype(ml_dtypes.float8_e4m3fn).astype(np.float64)
    return np.clip(np.rint(z), -128, 127).astype(np.float64)


def err_true(W, r, c, fmt, G):
    beta = (np.float32(1.0) / np.asarray(c, np.float32)).astype(np.float32)
    alpha = (np.float32(1.0) / np.asarray(r, np.float32)).astype(np.float32)
    z = (np.asarray(W, np.float32) * beta[None, :]).astype(np.float32)
    z = (z * np.repeat(alpha, G, axis=1)).astype(np.float32)
    q = grid_value(fmt, z)
    rec = np.repeat(np.asarray(r, np.float64), G, axis=1) * q * np.asarray(c, np.float64)[None, :]
    return float(np.sum((np.asarray(W, np.float64) - rec) ** 2))


def make_matrix(m, n, seed, outliers=4):
    W, _ = synth.student_t_weight(m, n, seed, std=0.02, unit_variance=False,
                                  outlier_cols=outliers, outlier_scale=20.0, bf16=False)
    return W


def admissible(fmt, around):
    if fmt in (O.MXINT8, O.MXFP8):
        return np.array([2.0 ** (b - 127) for b in range(255)])
    h = O.bf16_rne(around)
    return np.array([O.bf16_value(k) for k in range(max(1, h - 300), min(0x7F7F, h + 300))])


# ------------------------------------------------------------ element grids
def test_int8_grid():
    assert [O.int8_value(k) for k in (0, 1, 127, 128, 255)] == [0, 1, 127, -128, -1]
    g = np.random.default_rng(0)
    t = np.concatenate([g.uniform(-140, 140, 20000), np.arange(-130, 130) + 0.5]).astype(np.float32)
    got = np.array([O.int8_value(O.int8_encode(x)) for x in t])
    assert np.array_equal(got, np.clip(np.rint(t), -128, 127))


def test_e4m3_element_grid():
    ref = np.arange(256, dtype=np.uint8).view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    got = np.array([O.e4m3_elem_value(k) for k in range(256)])
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    assert np.array_equal(got[~np.isnan(got)], ref[~np.isnan(ref)])
    fin = np.unique(np.abs(ref[np.isfinite(ref)]))
    mids = (fin[:-1] + fin[1:]) / 2
    g = np.random.default_rng(1)
    t = np.concatenate([g.uniform(-600, 600, 20000), g.uniform(-0.05, 0.05, 5000),
                        mids, -mids, np.nextafter(mids.astype(np.float32), np.float32(0)),
                        np.nextafter(mids.astype(np.float32), np.float32(1e9))]).astype(np.float32)
    want = np.clip(t, -448, 448).astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    got = np.array([O.e4m3_elem_encode(x) for x in t], dtype=np.uint8)
    assert np.array_equal(got, want)


# ------------------------------------------------------------ objective, updates, descent
@pytest.mark.parametrize("fmt,G", FMTS8)
def test_objective_matches_independent_evaluator(fmt, G):
    W = make_matrix(64, 2 * G, 2)
    res = O.solve(W, fmt, G, 3)
    assert O.error(W, fmt, G, res["r"], res["c"]) == pytest.approx(
        err_true(W, res["r"], res["c"], fmt, G), rel=1e-12)
    assert res["err"][-1] == pytest.approx(err_true(W, res["r"], res["c"], fmt, G), rel=1e-12)


@pytest.mark.parametrize("fmt,G", FMTS8)
def test_updates_are_argmin_over_admissible_set(fmt, G):
    W = make_matrix(16, 2 * G, 3)
    res = O.solve(W, fmt, G, 2)
    r, c, sT = res["r"], res["c"], res["s_T"]
    Q = O.codes(W, fmt, G, r, c)
    r2, _ = O.update_fixed_q(W, Q, fmt, G, r, c, 0, sT)
    for i in range(3):
        for b in range(2):
            best = None
            for a in admissible(fmt, float(r2[i, b])):
                rr = r2.copy()
                rr[i, b] = np.float32(a)
                e = O.error_fixed_q(W, Q, fmt, G, rr, c)
                best = e if best is None or e < best else best
            assert O.error_fixed_q(W, Q, fmt, G, r2, c) <= best * (1 + 1e-12)
    _, c2 = O.update_fixed_q(W, Q, fmt, G, r, c, 1, sT)
    for j in (0, 5, G + 3):
        best = None
        for a in admissible(fmt, float(c2[j])):
            cc = c2.copy()
            cc[j] = np.float32(a)
            e = O.error_fixed_q(W, Q, fmt, G, r, cc)
            best = e if best is None or e < best else best
        assert O.error_fixed_q(W, Q, fmt, G, r, c2) <= best * (1 + 1e-12)


@pytest.mark.parametrize("fmt,G", FMTS8)
def test_mse_non_increasing_every_half_step(fmt, G):
    W = make_matrix(64, 2 * G, 4)
    res0 = O.solve(W, fmt, G, 0)
    r, c, sT = res0["r"].copy(), res0["c"].copy(), res0["s_T"]
    e_prev = err_true(W, r, c, fmt, G)
    for _ in range(5):
        Q = O.codes(W, fmt, G, r, c)
        r, _ = O.update_fixed_q(W, Q, fmt, G, r, c, 0, sT)
        e_fixed = O.error_fixed_q(W, Q, fmt, G, r, c)
        assert e_fixed <= e_prev * (1 + 1e-9)
        e_req = err_true(W, r, c, fmt, G)
        assert e_req <= e_fixed * (1 + 1e-9)
        Q = O.codes(W, fmt, G, r, c)
        _, c = O.update_fixed_q(W, Q, fmt, G, r, c, 1, sT)
        e_fixed = O.error_fixed_q(W, Q, fmt, G, r, c)
        assert e_fixed <= e_req * (1 + 1e-9)
        e_prev = err_true(W, r, c, fmt, G)
        assert e_prev <= e_fixed * (1 + 1e-9)
    res = O.solve(W, fmt, G, 5)
    assert np.array_equal(res["r"], r) and np.array_equal(res["c"], c)


# ------------------------------------------------------------ initialisation and special cases
@pytest.mark.parametrize("fmt,G", FMTS8)
def test_rtn_start_rule(fmt, G):
    """alpha-only at T = 0 (c = 1) is the format-native RTN quantiser:
    OCP 2^(floor(log2 amax) - emax) with emax 6 (INT8 grid) / 8 (E4M3),
    bf16(amax / 127) for INT8."""
    W = make_matrix(32, 4 * G, 5)
    r = O.solve_ex(W, fmt, G, 0, flags=O.ALPHA_ONLY)["r"]
    a = np.abs(W).reshape(32, 4, G).max(axis=2)
    if fmt == O.INT8:
        want = (a / np.float32(127.0)).astype(np.float32).astype(ml_dtypes.bfloat16)
        want = want.astype(np.float32)
    else:
        want = (2.0 ** (np.floor(np.log2(a.astype(np.float64))) - EMAX[fmt])).astype(np.float32)
    assert np.array_equal(r, want)


@pytest.mark.parametrize("fmt,G", FMTS8)
def test_exactly_representable_weight_is_a_fixed_point(fmt, G):
    """W = diag_blk(r*) Q*, every row-block reaching the grid's top value and
    equal column l1 norms per tile (cyclic pattern): c0 = 1, the RTN start
    recovers (r*, Q*) (for INT8 r* = 2^k: amax/127 = 2^k exactly) and
    Algorithm 1 stays there with zero error."""
    g = np.random.default_rng(6)
    m = n = 2 * G
    top = QMAX[fmt]
    if fmt == O.MXFP8:
        mags = np.array([448.0, 320.0, 224.0, 96.0, 40.0, 13.0, 2.5, 0.0])
    else:
        mags = np.array([127.0, 100.0, 77.0, 50.0, 31.0, 12.0, 3.0, 0.0])
    P = np.resize(mags, G)
    i = np.arange(m)[:, None]
    j = np.arange(n)[None, :]
    q = P[(i + j) % G] * np.where(g.random((m, n)) < 0.5, -1.0, 1.0)
    rstar = np.repeat(2.0 ** g.integers(-14, -6, size=(m // G, n // G)), G, axis=0)
    if fmt == O.INT8:
        rstar = rstar  # amax / 127 = r* exactly since the top value is 127
    W = (np.repeat(rstar, G, axis=1) * q).astype(np.float32)
    assert top == mags[0]
    res = O.solve(W, fmt, G, 6)
    assert np.all(res["c"] == 1.0)
    assert np.array_equal(res["r"], rstar.astype(np.float32))
    assert np.all(res["err"] == 0.0)


@pytest.mark.parametrize("fmt", [O.MXINT8, O.MXFP8])
def test_mx_scale_equivariance(fmt):
    W = make_matrix(64, 64, 7)
    a = O.solve(W, fmt, 32, 5)
    b = O.solve(W * np.float32(2.0 ** 3), fmt, 32, 5)
    assert np.array_equal(b["r"], a["r"] * np.float32(8.0))
    assert np.array_equal(b["c"], a["c"])


def test_int8_dual_scale_beats_rtn_on_outlier_tile():
    """With the fine bf16 scale sets the dual-scale solution has a lower
    weight MSE than single-scale RTN (Table 9's setting, qualitatively)."""
    W = make_matrix(256, 256, 8)
    res = O.solve(W, O.INT8, 128, 15)
    rtn = O.solve_ex(W, O.INT8, 128, 0, flags=O.ALPHA_ONLY)["err"][0]
    assert res["err"][-1] <= res["err"][0]
    assert res["err"][-1] < rtn


# ------------------------------------------------------------ activations, packing, GEMM
@pytest.mark.parametrize("fmt,G", FMTS8)
def test_act_quant_follows_its_rule(fmt, G):
    X, _ = synth.activations(5, 256, 9, n_outliers=3, outlier_scale=40.0)
    c = np.exp(np.random.default_rng(10).uniform(-1, 1, 256)).astype(np.float32)
    cod, sc, st = O.quantize_act(X, c, fmt, G)
    assert cod.shape == (5, 256)
    xt = (X * c[None, :]).astype(np.float32)
    S = 256 // G
    for t in range(5):
        for s in range(S):
            blk = xt[t, s * G:(s + 1) * G]
            ab = np.abs(blk).max()
            if fmt == O.INT8:
                h = np.float32(ab / np.float32(127.0)).astype(ml_dtypes.bfloat16)
                assert sc[t, s] == h.view(np.uint16)
                inv = np.float32(np.float32(1.0) / np.float32(h.astype(np.float32)))
            else:
                e = int(np.frexp(ab)[1]) - 1 - EMAX[fmt]
                assert sc[O.sf_offset(t, s, S)] == e + 127
                inv = np.float32(2.0 ** -e)
            z = (blk * inv).astype(np.float32)
            if fmt == O.MXFP8:
                want = np.clip(z, -448, 448).astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
            else:
                want = (np.clip(np.rint(z), -128, 127).astype(np.int64) & 0xFF).astype(np.uint8)
            assert np.array_equal(cod[t, s * G:(s + 1) * G], want)


@pytest.mark.parametrize("fmt,G", FMTS8)
def test_pack_weight_codes_and_scales(fmt, G):
    W = make_matrix(130, 2 * G, 11)
    res = O.solve(W, fmt, G, 3)
    cod, sc = O.pack_weight(W, fmt, G, res["r"], res["c"], res["s_T"])
    assert np.array_equal(cod, O.codes(W, fmt, G, res["r"], res["c"]))
    if fmt == O.INT8:
        dec = np.vectorize(O.bf16_value)(sc.astype(np.int64))
    else:
        dec = O.scale_values(sc, 130, 2, fmt)
    assert np.array_equal(dec, res["r"].astype(np.float64))


def test_reference_gemm_mxint8_integer_case():
    """MXINT8 operands with unit scales: the fp64 reference GEMM is the
    integer matmul of the codes."""
    g = np.random.default_rng(12)
    M, N, K = 8, 16, 64
    qa = g.integers(-128, 128, (M, K))
    qb = g.integers(-128, 128, (N, K))
    A = (qa & 0xFF).astype(np.uint8)
    B = (qb & 0xFF).astype(np.uint8)
    sA = np.zeros(O.sf_bytes(M, K // 32), np.uint8)
    sB = np.zeros(O.sf_bytes(N, K // 32), np.uint8)
    for rows, sf in ((M, sA), (N, sB)):
        for r_ in range(rows):
            for s in range(K // 32):
                sf[O.sf_offset(r_, s, K // 32)] = 127
    Y = O.linear(A, sA, None, B, sB, 1.0, M, N, K, O.MXINT8)
    assert np.array_equal(Y, (qa @ qb.T).astype(np.float64))
