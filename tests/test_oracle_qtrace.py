"""Pins for the oracle's code-change trace (CPU only): the relative change
||Qhat(t) - Qhat(t-1)||_F / ||Qhat(t-1)||_F of Fig. 2(a) / Fig. 3(a) in
"DualQuant", Qhat(t) the code values at the scales after round t.

It is recomputed here from T + 1 separate solves (the scales after round t
are those of a T = t solve) and the oracle's pinned quantiser; an exactly
representable weight never changes its codes; and the change decays on an
outlier-heavy layer (Fig. 2(a), qualitatively)."""
import numpy as np
import pytest

import oracle as O
from w4a4_post_quantization_dual_b200 import synth

FMTS = [(O.NVFP4, 16), (O.MXFP4, 32), (O.MXINT4, 32), (O.INT4, 64), (O.MXFP8, 32), (O.INT8, 128)]


def make_matrix(m, n, seed):
    W, _ = synth.student_t_weight(m, n, seed, std=0.02, unit_variance=False, outlier_cols=4,
                                  outlier_scale=20.0, bf16=False)
    return W


@pytest.mark.parametrize("fmt,G", FMTS)
def test_qchange_equals_separate_solves(fmt, G):
    W = make_matrix(64, 2 * max(G, 64), 120)
    T = 6
    res = O.solve_qtrace(W, fmt, G, T)
    full = O.solve(W, fmt, G, T)
    assert np.array_equal(res["r"], full["r"]) and np.array_equal(res["c"], full["c"])
    vals = O.elem_value_table(fmt)
    Q = [vals[O.codes(W, fmt, G, O.solve(W, fmt, G, t)["r"], O.solve(W, fmt, G, t)["c"])]
         for t in range(T + 1)]
    for t in range(1, T + 1):
        den = np.sum(Q[t - 1] ** 2)
        want = np.sqrt(np.sum((Q[t] - Q[t - 1]) ** 2) / den)
        assert res["qchange"][t] == pytest.approx(want, rel=1e-12, abs=0)
    assert np.isnan(res["qchange"][0])


def test_fixed_point_has_no_code_change():
    """W = r* Q* with every row-block at the grid top and equal column l1
    norms: Algorithm 1 starts at its fixed point, so the codes never move."""
    g = np.random.default_rng(121)
    G = 32
    mags = np.resize(np.array([6.0, 4.0, 3.0, 2.0, 1.5, 1.0, 0.5, 0.0]), G)
    i = np.arange(2 * G)[:, None]
    j = np.arange(2 * G)[None, :]
    q = mags[(i + j) % G] * np.where(g.random((2 * G, 2 * G)) < 0.5, -1.0, 1.0)
    W = (q * 2.0 ** -6).astype(np.float32)
    res = O.solve_qtrace(W, O.MXFP4, G, 5)
    assert np.all(res["qchange"][1:] == 0.0)


def test_code_change_decays():
    """Fig. 2(a): the relative code change decays over the rounds."""
    W = make_matrix(256, 256, 122)
    for fmt, G in [(O.NVFP4, 16), (O.INT4, 64)]:
        qc = O.solve_qtrace(W, fmt, G, 20)["qchange"]
        assert qc[1] > 0
        assert qc[20] <= 0.25 * qc[1]
        assert qc[20] < 0.02
