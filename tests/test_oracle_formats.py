"""Pins for the oracle's element and scale codecs (CPU only).

Every check compares against something other than the oracle itself: the
OCP tables under tests/golden, an independent library conversion
(ml_dtypes / torch, both round-to-nearest-even), or a brute-force nearest
search over the golden value set.
"""
import math

import ml_dtypes
import numpy as np
import pytest
import torch

from conftest import golden

pytestmark = pytest.mark.filterwarnings("ignore")


def _val(s):
    return float("nan") if s == "nan" else float(s)


def test_e2m1_table_matches_ocp(orc):
    for code, v in golden("e2m1_values.txt"):
        got = orc.e2m1_value(int(code))
        assert got == _val(v) and math.copysign(1, got) == math.copysign(1, _val(v))


def test_e4m3_selected_values_match_ofp8(orc):
    for b, v in golden("e4m3_values.txt"):
        got, want = orc.e4m3_value(int(b, 16)), _val(v)
        assert (math.isnan(got) and math.isnan(want)) or got == want


def test_e8m0_selected_values_match_ocp(orc):
    for b, v in golden("e8m0_values.txt"):
        b = int(b)
        if b == 255:
            continue  # NaN code is never produced or decoded by the path
        assert orc.e8m0_value(b) == _val(v)


def test_e2m1_encode_matches_ml_dtypes_rne():
    import oracle
    g = np.random.default_rng(1)
    x = np.concatenate([g.standard_normal(20000).astype(np.float32) * 3,
                        # every midpoint of the grid and +-1 ulp around it
                        np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.5, 7.0, 100.0],
                                 np.float32)])
    x = np.concatenate([x, -x, np.nextafter(x, np.float32(np.inf)),
                        np.nextafter(x, np.float32(-np.inf))]).astype(np.float32)
    ref = x.astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 0xF
    got = np.array([oracle.e2m1_encode(v) for v in x], np.uint8)
    assert np.array_equal(got, ref)


def test_e2m1_encode_is_nearest_grid_point():
    import oracle
    table = np.array([_val(v) for _, v in golden("e2m1_values.txt")])
    g = np.random.default_rng(2)
    for t in g.uniform(-8, 8, 3000).astype(np.float32):
        code = oracle.e2m1_encode(t)
        assert abs(t - table[code]) <= np.min(np.abs(t - table)) + 0.0


def test_int4_encode_round_half_even_and_clip():
    import oracle
    g = np.random.default_rng(3)
    x = np.concatenate([g.uniform(-12, 12, 5000), np.arange(-10, 10.5, 0.5)]).astype(np.float32)
    ref = np.clip(np.rint(x), -8, 7).astype(np.int64) & 0xF     # numpy rint = half-to-even
    got = np.array([oracle.int4_encode(v) for v in x])
    assert np.array_equal(got, ref)
    assert [oracle.int4_value(k) for k in range(16)] == list(range(8)) + list(range(-8, 0))


def test_ue4m3_rne_matches_torch_float8():
    import oracle
    g = np.random.default_rng(4)
    x = np.concatenate([np.exp(g.uniform(np.log(1e-4), np.log(440.0), 4000)),
                        [oracle.e4m3_value(b) for b in range(127)]])
    mids = [(oracle.e4m3_value(b) + oracle.e4m3_value(b + 1)) / 2 for b in range(126)]
    x = np.concatenate([x, mids]).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([oracle.ue4m3_rne(float(v)) for v in x], np.uint8)
    assert np.array_equal(got, ref)
    assert oracle.ue4m3_rne(1e6) == 0x7E  # saturating


def test_ue4m3_projection_is_nearest_positive():
    import oracle
    vals = np.array([oracle.e4m3_value(b) for b in range(1, 127)])
    g = np.random.default_rng(5)
    for u in np.exp(g.uniform(np.log(1e-5), np.log(1e3), 2000)):
        b = oracle.ue4m3_proj(u)
        assert b >= 1
        assert abs(u - oracle.e4m3_value(b)) == np.min(np.abs(u - vals))


def test_e8m0_projection_nearest_with_ties_up():
    import oracle
    vals = np.array([2.0 ** (b - 127) for b in range(255)])
    g = np.random.default_rng(6)
    us = np.concatenate([np.exp(g.uniform(-60, 60, 3000)), [1.5 * 2.0 ** k for k in range(-20, 20)]])
    for u in us:
        b = oracle.e8m0_proj(u)
        d = np.abs(u - vals)
        assert d[b] == d.min()
        if u in [1.5 * 2.0 ** k for k in range(-20, 20)]:
            assert vals[b] > u  # exact midpoint goes to the larger power
    # ml_dtypes' float -> e8m0 rounding agrees on normal-range values
    x = np.exp(g.uniform(-40, 40, 2000)).astype(np.float32)
    ref = x.astype(ml_dtypes.float8_e8m0fnu).view(np.uint8)
    got = np.array([oracle.e8m0_proj(float(v)) for v in x], np.uint8)
    assert np.array_equal(got, ref)


def test_bf16_rne_matches_torch_and_brute_force():
    import oracle
    g = np.random.default_rng(7)
    x = (g.standard_normal(5000) * np.exp(g.uniform(-30, 30, 5000))).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().astype(np.int64) & 0xFFFF
    got = np.array([oracle.bf16_rne(float(v)) for v in x])
    assert np.array_equal(got, ref)
    # doubles (not fp32-representable): brute force over all positive bf16
    allv = np.array([oracle.bf16_value(h) for h in range(0x0001, 0x7F80)])
    for u in np.exp(g.uniform(-20, 20, 300)):
        h = oracle.bf16_rne(u)
        assert abs(u - oracle.bf16_value(h)) == np.min(np.abs(u - allv))
        assert oracle.bf16_proj(u) == oracle.bf16_value(h)


def test_alpha_projection_nvfp4_is_tensor_scaled_e4m3(orc):
    sT = 0.000123
    for u in [1e-6, 3e-4, 0.01, 0.05]:
        r = orc.proj_alpha(orc.NVFP4, u, sT)
        cands = np.float32(sT) * np.array([orc.e4m3_value(b) for b in range(1, 127)], np.float32)
        assert r in set(cands.tolist())
        assert abs(u - r) <= np.min(np.abs(u - cands.astype(np.float64))) * (1 + 1e-6) + 1e-12
