"""Pins for the oracle's activation quantiser, weight packer, block-scale
layout and dequantised reference matmul (CPU only).

Independent references: ml_dtypes (E2M1, RNE, saturating), torch's
float8_e4m3fn and bfloat16 casts (RNE), numpy frexp for the OCP MX shared
exponent, integer matmul in numpy for the GEMM, plus special cases with a
known answer.
"""
import ml_dtypes
import numpy as np
import pytest
import torch

import oracle as O
from w4a4_post_quantization_dual_b200 import synth


def _e2m1(z):
    return np.asarray(z, np.float32).astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 0xF


def _int4(z):
    return np.clip(np.rint(np.asarray(z, np.float32)), -8, 7).astype(np.int64) & 0xF


def _sf_index(rows, S):
    return np.array([[O.sf_offset(r, s, S) for s in range(S)] for r in range(rows)])


def test_sf_layout_is_a_bijection_into_the_buffer():
    for rows, S in [(1, 4), (130, 8), (256, 16), (300, 12)]:
        off = _sf_index(rows, S).ravel()
        assert len(np.unique(off)) == off.size
        assert off.min() >= 0 and off.max() < O.sf_bytes(rows, S)
        assert O.sf_bytes(rows, S) % 512 == 0


@pytest.mark.parametrize("fmt", [O.NVFP4, O.MXFP4, O.MXINT4, O.INT4])
def test_act_quant_follows_its_rule_with_library_codecs(fmt):
    G = O.NATIVE_GROUP[fmt]
    X, _ = synth.activations(5, 256, 3, n_outliers=3, outlier_scale=40.0)
    c = np.exp(np.random.default_rng(1).uniform(-1, 1, 256)).astype(np.float32)
    c = torch.from_numpy(c).to(torch.float8_e4m3fn).to(torch.float32).numpy()
    cod, sc, st = O.quantize_act(X, c, fmt, G)
    codes = O.unpack_codes(cod, 256)
    xt = (X * c[None, :]).astype(np.float32)
    S = 256 // G
    for t in range(5):
        amax = np.abs(xt[t]).max()
        s_tok = np.float32(amax / np.float32(2688.0))
        for s in range(S):
            blk = xt[t, s * G:(s + 1) * G]
            ab = np.abs(blk).max()
            if fmt == O.NVFP4:
                assert st[t] == s_tok
                sb = np.float32(ab / np.float32(np.float32(6.0) * s_tok))
                byte = torch.tensor([sb]).to(torch.float8_e4m3fn).view(torch.uint8).item()
                assert sc[O.sf_offset(t, s, S)] == byte
                sblk = np.float32(np.float32(O.e4m3_value(byte)) * s_tok)
                inv = np.float32(np.float32(1.0) / sblk)
                want = _e2m1((blk * inv).astype(np.float32))
            elif fmt in (O.MXFP4, O.MXINT4):
                e = int(np.frexp(ab)[1]) - 1 - 2
                assert sc[O.sf_offset(t, s, S)] == e + 127
                z = (blk * np.float32(2.0 ** -e)).astype(np.float32)
                want = _e2m1(z) if fmt == O.MXFP4 else _int4(z)
            else:
                h = torch.tensor([np.float32(ab / np.float32(7.0))]).to(torch.bfloat16)
                hb = h.view(torch.int16).item() & 0xFFFF
                assert sc[t, s] == hb
                inv = np.float32(np.float32(1.0) / np.float32(h.to(torch.float32).item()))
                want = _int4((blk * inv).astype(np.float32))
            assert np.array_equal(codes[t, s * G:(s + 1) * G], want)


def test_act_quant_special_cases():
    # zero rows -> zero codes, zero scales, s_tok 0
    X = np.zeros((3, 64), np.float32)
    c = np.ones(64, np.float32)
    for fmt in (O.NVFP4, O.MXFP4, O.MXINT4):
        cod, sc, st = O.quantize_act(X, c, fmt, O.NATIVE_GROUP[fmt])
        assert not cod.any() and not st.any()
    # NVFP4: the row maximum always lands on the top grid point 6 with block byte 448
    X, _ = synth.activations(4, 128, 9, n_outliers=2, outlier_scale=30.0)
    cod, sc, st = O.quantize_act(X, np.ones(128, np.float32), O.NVFP4, 16)
    codes = O.unpack_codes(cod, 128)
    for t in range(4):
        j = int(np.argmax(np.abs(X[t])))
        assert codes[t, j] & 7 == 7
        assert sc[O.sf_offset(t, j // 16, 8)] == 0x7E
    # a row that is exactly on the MXFP4 grid is reproduced exactly
    g = np.random.default_rng(2)
    q = np.array([O.e2m1_value(k) for k in range(16)])[g.integers(0, 16, (2, 64))]
    q[:, ::32] = 6.0
    X = (q * 2.0 ** -3).astype(np.float32)
    cod, sc, _ = O.quantize_act(X, np.ones(64, np.float32), O.MXFP4, 32)
    deq = O.dequant(cod, sc, 2, 64, O.MXFP4, 32)
    assert np.array_equal(deq, X.astype(np.float64))


@pytest.mark.parametrize("fmt", [O.NVFP4, O.MXFP4, O.MXINT4, O.INT4])
def test_pack_weight_codes_and_scales(fmt):
    G = O.NATIVE_GROUP[fmt]
    W = synth.student_t_weight(64, 128, 5)[0]
    res = O.solve(W, fmt, G, 3)
    cod, sc = O.pack_weight(W, fmt, G, res["r"], res["c"], res["s_T"])
    assert np.array_equal(O.unpack_codes(cod, 128), O.codes(W, fmt, G, res["r"], res["c"]))
    if fmt == O.INT4:
        assert np.array_equal(np.array([[O.bf16_value(h) for h in row] for row in sc], np.float32),
                              res["r"])
    else:
        vals = O.scale_values(sc, 64, 128 // G, fmt)
        if fmt == O.NVFP4:
            vals = (np.float32(res["s_T"]) * vals.astype(np.float32)).astype(np.float32)
        assert np.array_equal(vals.astype(np.float32), res["r"])


def test_reference_gemm_integer_case():
    """Unit block scales and integer codes: the reference equals an exact
    integer matmul."""
    g = np.random.default_rng(3)
    M, N, K = 5, 7, 64
    a = g.integers(-8, 8, (M, K))
    b = g.integers(-8, 8, (N, K))
    pack = lambda v: ((v[:, 0::2] & 0xF) | ((v[:, 1::2] & 0xF) << 4)).astype(np.uint8)
    S = K // 32
    sfa = np.zeros(O.sf_bytes(M, S), np.uint8)
    sfb = np.zeros(O.sf_bytes(N, S), np.uint8)
    for r in range(M):
        for s in range(S):
            sfa[O.sf_offset(r, s, S)] = 127
    for r in range(N):
        for s in range(S):
            sfb[O.sf_offset(r, s, S)] = 127
    Y = O.linear(pack(a), sfa, None, pack(b), sfb, 1.0, M, N, K, O.MXINT4)
    assert np.array_equal(Y, (a @ b.T).astype(np.float64))
    rows = np.array([0, 3])
    assert np.array_equal(O.linear_rows(pack(a), sfa, None, pack(b), sfb, 1.0, rows, M, N, K,
                                        O.MXINT4), Y[rows])


def test_reference_gemm_nvfp4_matches_library_decode():
    """NVFP4 reference = (ml_dtypes-decoded codes x torch-decoded E4M3 scales
    x s_tok) @ (... x s_W)^T."""
    X, _ = synth.activations(6, 128, 4, n_outliers=2, outlier_scale=20.0)
    W = synth.student_t_weight(9, 128, 6)[0]
    c = np.ones(128, np.float32)
    A, sA, st = O.quantize_act(X, c, O.NVFP4, 16)
    res = O.solve(W, O.NVFP4, 16, 2)
    B, sB = O.pack_weight(W, O.NVFP4, 16, res["r"], res["c"], res["s_T"])
    Y = O.linear(A, sA, st, B, sB, res["s_T"], 6, 9, 128, O.NVFP4)

    def dec(packed, sf, rows):
        codes = O.unpack_codes(packed, 128)
        vals = codes.astype(np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float64)
        off = _sf_index(rows, 8)
        sc = torch.from_numpy(sf[off].astype(np.uint8)).view(torch.float8_e4m3fn).to(
            torch.float64).numpy()
        return vals * np.repeat(sc, 16, axis=1)

    ref = (dec(A, sA, 6) * st[:, None].astype(np.float64)) @ dec(B, sB, 9).T * res["s_T"]
    assert np.allclose(Y, ref, rtol=1e-13, atol=0)
