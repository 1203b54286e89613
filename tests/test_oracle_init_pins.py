"""Pins for the oracle's initialisation and decision precision (CPU only).

DualQuant, Section 5.3 "Hyperparameter selection": the column scales start
from the column l1 norms and the row-block scales from the format-native
absmax (RTN) scale.  The oracle normalises the l1 norms to mean 1 over each
G-column tile before projecting them onto F_beta, and (NVFP4) takes the
per-tensor scale as amax(W diag(c)^-1) / (6 * 448).

These tests pin those functions against values worked out by hand, with no
call into the oracle's arithmetic on the expected side, so that a wrong norm
(l2, max), a wrong normaliser (the whole-matrix mean, no mean), c in place
of 1/c, or a fp64 projection decision each fails one of them.

Decision precision: every scale decision is taken on the fp32 value of the
closed-form update (Section 4.3's projection; Appendix C, Remark 1).  fp32
is the precision the scale formats are defined from (E8M0, E4M3 and bf16
scales are conversions of an fp32 quantity in the OCP MX and OFP8
specifications), and the paper fixes none.  The last tests build updates
whose fp32 and fp64 values project to different scales.
"""
import ml_dtypes
import numpy as np
import pytest

import oracle as O


def col_block(l1_pattern, scale=1.0):
    """4 rows whose columns have the given l1 norms (signs mixed, magnitudes
    unequal inside a column so that l1 and l2 disagree)."""
    cols = []
    for l1 in l1_pattern:
        # split l1 into magnitudes 0.5, 0.25, 0.125, 0.125 of it, alternating signs
        cols.append(np.array([0.5, -0.25, 0.125, -0.125]) * l1 * scale)
    return np.stack(cols, axis=1)


# ------------------------------------------------------------ c0 by hand
# l1 norms {1, 2, 3, 6} -> tile mean 3 -> ratios {1/3, 2/3, 1, 2}.
# Nearest admissible values worked out by hand:
#   E8M0 (powers of two, linear distance): 1/3 -> 1/4 (1/12 < 1/6); 2/3 -> 1/2 (1/6 < 1/3).
#   UE4M3: 1/3 lies in [1/4, 1/2) with step 1/32: neighbours 10/32 and 11/32,
#          distances 1/48 and 1/96 -> 11/32 = 0.34375; 2/3 in [1/2, 1) step 1/16:
#          neighbours 10/16, 11/16 at 1/24, 1/48 -> 11/16 = 0.6875.
#   bf16 (8 significant bits): 1/3 = (4/3) 2^-2, 4/3 * 128 = 170.67 -> 171 ->
#          171/512 = 0.333984375; 2/3 -> 171/256 = 0.66796875.
HAND_C = {
    O.MXFP4: [0.25, 0.5, 1.0, 2.0],
    O.MXINT4: [0.25, 0.5, 1.0, 2.0],
    O.NVFP4: [0.34375, 0.6875, 1.0, 2.0],
    O.INT4: [171 / 512, 171 / 256, 1.0, 2.0],
}


@pytest.mark.parametrize("fmt", [O.MXFP4, O.MXINT4, O.NVFP4, O.INT4])
def test_init_c_hand_values(fmt):
    # tile 0: l1 {1, 2, 3, 6}; tile 1: the same pattern x 10 (per-tile mean
    # gives the same c; a whole-matrix mean would not); tile 2: a zero column
    # (-> Pi(1) = 1) beside l1 {2, 2, 4} (mean 2 -> 1, 1, 2); tile 3: all zero.
    W = np.concatenate([col_block([1, 2, 3, 6]), col_block([1, 2, 3, 6], 10.0),
                        col_block([0, 2, 2, 4]), np.zeros((4, 4))], axis=1).astype(np.float32)
    # every value above is exact in fp32 (multiples of 1/128 times small integers)
    c = O.init_c(W, fmt, 4)
    expect = HAND_C[fmt] + HAND_C[fmt] + [1.0, 1.0, 1.0, 2.0] + [1.0] * 4
    assert c.tolist() == pytest.approx(expect, abs=0, rel=0)


def test_init_c_does_not_use_l2_or_max():
    # The same l1 norms reached with equal magnitudes in one column and a
    # single spike in another: l1 gives both ratio 1, l2 and max do not.
    W = np.zeros((4, 4), np.float32)
    W[:, 0] = 0.25           # l1 1, l2 0.5, max 0.25
    W[0, 1] = 1.0            # l1 1, l2 1,   max 1
    W[:, 2] = [0.5, 0.5, 0, 0]
    W[:, 3] = [-0.25, 0.25, -0.25, 0.25]
    for fmt in (O.NVFP4, O.MXFP4, O.INT4):
        assert O.init_c(W, fmt, 4).tolist() == [1.0, 1.0, 1.0, 1.0]


@pytest.mark.parametrize("fmt,G", [(O.NVFP4, 16), (O.MXFP4, 32), (O.INT4, 64)])
def test_init_c_invariances(fmt, G):
    rng = np.random.default_rng(11)
    W = (rng.standard_t(4, size=(48, 4 * G)) * 0.02).astype(np.float32)
    W[:, rng.choice(4 * G, 6, replace=False)] *= 15.0
    c = O.init_c(W, fmt, G)
    # a positive factor of 2 on the whole matrix is exact in fp32 and cancels in l1 / mean
    assert np.array_equal(O.init_c(W * np.float32(2.0), fmt, G), c)
    # row order and signs do not enter l1
    assert np.array_equal(O.init_c(-W[::-1].copy(), fmt, G), c)
    # a column permutation inside a tile permutes c the same way
    p = np.arange(4 * G)
    p[:G] = rng.permutation(G)
    assert np.array_equal(O.init_c(W[:, p].copy(), fmt, G), c[p])


def test_init_c_independent_recomputation():
    """l1 per column in fp64, divided by the tile mean, rounded to fp32, then
    the nearest admissible value by the library codecs (ml_dtypes E4M3 and
    bf16 casts are round-to-nearest-even; E8M0 by comparing the two powers of
    two that bracket the value)."""
    rng = np.random.default_rng(5)
    W = (rng.standard_t(4, size=(40, 128)) * 0.02).astype(np.float32)
    W[:, [3, 40, 77]] *= 30.0
    for fmt, G in [(O.NVFP4, 16), (O.MXFP4, 32), (O.INT4, 64)]:
        l1 = np.abs(W.astype(np.float64)).sum(axis=0)
        mean = l1.reshape(-1, G).mean(axis=1).repeat(G)
        u = (l1 / mean).astype(np.float32)
        if fmt == O.NVFP4:
            expect = u.astype(ml_dtypes.float8_e4m3fn).astype(np.float64)
        elif fmt == O.INT4:
            expect = u.astype(ml_dtypes.bfloat16).astype(np.float64)
        else:
            lo = 2.0 ** np.floor(np.log2(u.astype(np.float64)))
            expect = np.where(u - lo < 2 * lo - u, lo, 2 * lo)
        got = O.init_c(W, fmt, G).astype(np.float64)
        assert np.array_equal(got, expect), fmt


# ------------------------------------------------------------ s_T by hand
def test_tensor_scale_uses_the_inverse_column_scale():
    W = np.zeros((2, 4), np.float32)
    c = np.array([0.5, 4.0, 2.0, 1.0], np.float32)
    W[0, 0] = 3.0     # / 0.5 -> 6   (the maximum of W diag(c)^-1)
    W[1, 1] = 5.0     # / 4   -> 1.25 (the maximum of |W| and of W diag(c))
    W[0, 2] = -4.0    # / 2   -> 2
    W[1, 3] = 1.0
    s = O.tensor_scale(W, c)
    assert s == float(np.float32(6.0) / np.float32(2688.0))
    # sanity of the hand value against the wrong readings
    assert s != float(np.float32(20.0) / np.float32(2688.0))      # W diag(c)
    assert s != float(np.float32(5.0) / np.float32(2688.0))       # no c
    assert O.tensor_scale(np.zeros((3, 4), np.float32), c) == 1.0  # degenerate convention


def test_tensor_scale_maps_the_tensor_maximum_onto_the_largest_block_scale():
    """With s_T = amax / (6 * 448), the RTN scale of the block holding the
    tensor maximum is s_T * 448 (the largest UE4M3 value), and its largest
    element lands on the E2M1 maximum 6."""
    rng = np.random.default_rng(2)
    W = (rng.standard_t(4, size=(32, 64)) * 0.02).astype(np.float32)
    c = (2.0 ** rng.integers(-3, 4, size=64)).astype(np.float32)
    s = O.tensor_scale(W, c)
    z = np.abs(W / c[None, :])                  # power-of-two c: exact in fp32
    i, j = np.unravel_index(np.argmax(z), z.shape)
    assert s == float(np.float32(z[i, j]) / np.float32(2688.0))
    r = O.init_r(W, O.NVFP4, 16, c, s)
    assert r[i, j // 16] == np.float32(np.float64(s) * 448.0)
    Q = O.codes(W, O.NVFP4, 16, r, c)
    assert abs(O.e2m1_value(int(Q[i, j]))) == 6.0


# ------------------------------------------------------------ fp32 decisions
def test_projection_decides_on_the_fp32_value():
    eps = 2.0 ** -40
    # E8M0: 1.5 - eps is nearer 1 in exact arithmetic, but its fp32 value is
    # the midpoint 1.5, which goes to the larger power (R6).
    assert O.proj_beta(O.MXFP4, 1.5 - eps) == 2.0
    assert O.proj_beta(O.MXFP4, 1.5 - 2.0 ** -20) == 1.0      # fp32 keeps it below
    # UE4M3: 1.0625 is the midpoint of 1 (byte 0x38, even) and 1.125 (0x39):
    # 1.0625 + eps is nearer 1.125 exactly, its fp32 value is the tie -> 1.
    assert O.proj_beta(O.NVFP4, 1.0625 + eps) == 1.0
    assert O.proj_beta(O.NVFP4, 1.0625 + 2.0 ** -20) == 1.125
    # bf16: 1 + 2^-8 is the midpoint of 1 and 1 + 2^-7 (ties to the even mantissa 1).
    assert O.proj_beta(O.INT4, 1.0 + 2.0 ** -8 + eps) == 1.0
    assert O.proj_beta(O.INT4, 1.0 + 2.0 ** -8 + 2.0 ** -20) == 1.0 + 2.0 ** -7
    # NVFP4 row scale: the ratio u / s_T is one fp32 division of the fp32 u.
    assert O.proj_alpha(O.NVFP4, 0.53125 + eps, 0.5) == 0.5
    assert O.proj_alpha(O.NVFP4, 0.53125 + 2.0 ** -20, 0.5) == 0.5625


def test_closed_form_update_decides_on_the_fp32_quotient():
    """A row-block and a column whose closed-form update is 1.5 - 2^-25 in
    fp64: the fp32 quotient is the tie 1.5, so E8M0 takes 2 (fp64 would take 1)."""
    G = 32
    w = np.full(G, 1.5, np.float32)
    w[-1] = np.float32(1.5 - 2.0 ** -20)
    one = 2                                   # E2M1 code of the value 1.0
    assert O.e2m1_value(one) == 1.0
    u = float(np.sum(w.astype(np.float64))) / G
    assert u < 1.5 and np.float32(u) == np.float32(1.5)
    # row half-step (Eq. 10): Q = 1, c = 1 -> u = mean of the row-block
    W = w[None, :].copy()
    Q = np.full((1, G), one, np.uint8)
    r, _ = O.update_fixed_q(W, Q, O.MXFP4, G, np.ones((1, 1)), np.ones(G), 0)
    assert r[0, 0] == 2.0
    # column half-step (Eq. 14): Q = 1, r = 1 -> u = mean of the column
    Wc = np.tile(w[:, None], (1, G)).astype(np.float32)
    Qc = np.full((G, G), one, np.uint8)
    _, c = O.update_fixed_q(Wc, Qc, O.MXFP4, G, np.ones((G, 1)), np.ones(G), 1)
    assert np.all(c == 2.0)
