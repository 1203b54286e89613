"""Pins for the oracle's activation quantisation error (CPU only): the
measure behind the activation SQNR with and without beta (DualQuant,
Appendix E, Table 6).  The dequantisation is recomputed here with library
decoders (ml_dtypes E2M1, torch E4M3 / bfloat16), exact cases give zero
error, and the MX formats are scale-equivariant."""
import ml_dtypes
import numpy as np
import pytest
import torch

import oracle as O
from w4a4_post_quantization_dual_b200 import synth

FMTS = [(O.NVFP4, 16), (O.MXFP4, 32), (O.MXINT4, 32), (O.INT4, 64)]


def _independent_sums(X, c, fmt, G):
    """sum x^2 and sum (x - x^)^2 with the oracle's codes and scale bytes
    decoded by library codecs."""
    M, K = X.shape
    cc = np.ones(K, np.float32) if c is None else c
    cod, sc, st = O.quantize_act(X, cc, fmt, G)
    nib = np.empty((M, K), np.uint8)
    nib[:, 0::2] = cod & 0xF
    nib[:, 1::2] = cod >> 4
    if fmt in (O.NVFP4, O.MXFP4):
        q = nib.view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    else:
        q = ((nib.astype(np.int64) ^ 8) - 8).astype(np.float64)   # two's complement nibble
    S = K // G
    if fmt == O.INT4:
        s = torch.from_numpy(sc.astype(np.int16)).view(torch.bfloat16).double().numpy()
    else:
        idx = np.array([[O.sf_offset(r, b, S) for b in range(S)] for r in range(M)])
        b = sc[idx]
        if fmt == O.NVFP4:
            s = torch.from_numpy(b).view(torch.float8_e4m3fn).double().numpy()
            s = s * st.astype(np.float64)[:, None]
        else:
            s = np.ldexp(1.0, b.astype(np.int64) - 127)
    xh = q * np.repeat(s, G, axis=1) / cc.astype(np.float64)[None, :]
    x = X.astype(np.float64)
    return float(np.sum(x * x)), float(np.sum((x - xh) ** 2))


@pytest.mark.parametrize("fmt,G", FMTS)
@pytest.mark.parametrize("with_c", [False, True])
def test_error_sums_match_library_decode(fmt, G, with_c):
    X, _ = synth.activations(33, 256, 4, n_outliers=3, outlier_scale=40.0)
    c = None
    if with_c:
        c = np.exp(np.random.default_rng(3).uniform(-1.5, 1.5, 256)).astype(np.float32)
    got = O.act_error_sums(X, c, fmt, G)
    want = _independent_sums(X, c, fmt, G)
    assert got[0] == pytest.approx(want[0], rel=1e-12)
    assert got[1] == pytest.approx(want[1], rel=1e-12)
    assert got[1] > 0
    # Per-element error is at most half a grid step of its block (E2M1: the
    # top step 6 - 4 = 2 scale units, INT4: 1 unit), so the SQNR is bounded
    assert O.act_sqnr_db(X, c, fmt, G) > 5.0


def test_exactly_representable_activations_have_no_error():
    g = np.random.default_rng(4)
    q = np.array([O.e2m1_value(k) for k in range(16)])[g.integers(0, 16, (4, 128))]
    q[:, ::32] = 6.0                               # every MX block reaches the top of the grid
    X = (q * 2.0 ** -5).astype(np.float32)
    assert O.act_error_sums(X, None, O.MXFP4, 32)[1] == 0.0
    assert O.act_sqnr_db(X, None, O.MXFP4, 32) == np.inf
    # power-of-two column scales keep the rescaled rows on the grid (a whole
    # block shares one exponent shift)
    c = np.repeat(2.0 ** g.integers(-3, 4, 4), 32).astype(np.float32)
    assert O.act_error_sums(X / c, c, O.MXFP4, 32)[1] == 0.0


@pytest.mark.parametrize("fmt,G", [(O.MXFP4, 32), (O.MXINT4, 32)])
def test_mx_error_is_scale_equivariant(fmt, G):
    """X -> 2^k X: same codes, block exponents + k, both sums x 4^k."""
    X, _ = synth.activations(16, 128, 5, n_outliers=2, outlier_scale=30.0)
    a = O.act_error_sums(X, None, fmt, G)
    b = O.act_error_sums((X * np.float32(8.0)).astype(np.float32), None, fmt, G)
    assert b[0] == a[0] * 64.0 and b[1] == a[1] * 64.0
