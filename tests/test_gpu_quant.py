"""GPU parity: fused activation rescale+quantise and weight packing against
the oracle, element by element (bit-exact: codes, every scale byte including
layout padding, per-token scales)."""
import numpy as np
import pytest
import torch

import oracle as O
from gpu_helpers import gpu_act, gpu_pack
from w4a4_post_quantization_dual_b200 import synth

pytestmark = pytest.mark.gpu

FMTS = [(O.NVFP4, 16), (O.MXFP4, 32), (O.MXINT4, 32), (O.INT4, 64), (O.INT4, 128)]


def col_scales(fmt, G, K, seed):
    """Valid column scales (in F_beta) from the oracle's initialisation of a
    random Student-t weight with outlier columns."""
    W, _ = synth.student_t_weight(64, K, seed, outlier_cols=max(1, K // 100), outlier_scale=30.0)
    return O.init_c(W, fmt, G)


def _pad_expectation(sc_oracle, M, K, G, fmt):
    return sc_oracle  # oracle writes zeros in the padding (rows >= M)


@pytest.mark.parametrize("fmt,G", FMTS)
@pytest.mark.parametrize("M,K,xdt", [(16, 256, torch.float32), (1, 4096, torch.bfloat16),
                                     (17, 4096, torch.bfloat16), (300, 5120, torch.bfloat16),
                                     (129, 14336, torch.bfloat16), (40, 27648, torch.bfloat16),
                                     (4100, 4096, torch.bfloat16)])
def test_act_quant_bit_exact(fmt, G, M, K, xdt):
    X, _ = synth.activations(M, K, 100 + M, n_outliers=max(1, K // 100), outlier_scale=50.0,
                             bf16=(xdt == torch.bfloat16))
    c = col_scales(fmt, G, K, 7)
    cod, sc, st = gpu_act(X, c, fmt, G, xdt)
    ocod, osc, ost = O.quantize_act(X, c, fmt, G)
    assert np.array_equal(cod, ocod)
    assert np.array_equal(sc, osc)
    if fmt == O.NVFP4:
        assert np.array_equal(st.view(np.uint32), ost.view(np.uint32))


def test_act_quant_rounding_boundaries():
    """Values on every E2M1 / INT4 midpoint (and one ulp either side),
    saturation, tiny values that round to (signed) zero, and zero blocks."""
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.5, 7.0, 7.49, 7.5, 7.99, 0.0, 1e-30],
                    np.float32)
    vals = np.concatenate([mids, np.nextafter(mids, 10), np.nextafter(mids, -10)])
    row = np.concatenate([vals, -vals])
    K = 256
    X = np.zeros((4, K), np.float32)
    X[0, :row.size] = row
    X[0, 31] = 7.99          # pin the MX block exponent: floor(log2 7.99) - 2 = 0
    X[0, 63] = -7.99
    X[1, :row.size] = row * np.float32(2.0 ** -40)
    # row 3 stays zero
    for fmt, G in FMTS[:4]:
        # fp32-subnormal activations: only the power-of-two MX scales keep the
        # reciprocal block scale finite there (see include/dq.h, input range)
        X[2, 5] = 1e-38 if fmt in (O.MXFP4, O.MXINT4) else 3.0e-7
        cod, sc, st = gpu_act(X, np.ones(K, np.float32), fmt, G, torch.float32)
        ocod, osc, ost = O.quantize_act(X, np.ones(K, np.float32), fmt, G)
        assert np.array_equal(cod, ocod), fmt
        assert np.array_equal(sc, osc), fmt


@pytest.mark.parametrize("fmt,G", FMTS[:3])
def test_act_quant_rounding_boundaries_bf16(fmt, G):
    """The bf16 path: every E2M1 / INT4 midpoint in block-scale units (exact
    in bf16), one bf16 ulp either side, saturation, signed zeros, zero blocks
    and a block whose values all round to zero, in rows that span several
    32-lane groups of blocks."""
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.5, 7.0, 7.5, 0.0], np.float32)
    up = torch.from_numpy(mids).to(torch.bfloat16)
    nxt = lambda d: (up.view(torch.int16) + d).view(torch.bfloat16).float().numpy()
    vals = np.concatenate([mids, nxt(1), nxt(-1)[mids > 0]])
    row = np.concatenate([vals, -vals])
    K = 2048
    X = np.zeros((6, K), np.float32)
    for off in range(0, K, 512):
        X[0, off:off + row.size] = row
    X[0, 31::64] = 7.96875       # MX block exponent floor(log2 7.97) - 2 = 0: unit scale
    X[0, 63::64] = -7.96875
    X[1] = X[0] * np.float32(2.0 ** -40)
    X[2, 700:716] = np.float32(1e-3)  # a tiny block in a row whose token max is large
    X[2, 5] = 1000.0
    # rows 3..5 stay zero
    X = torch.from_numpy(X).to(torch.bfloat16).float().numpy()
    c = np.ones(K, np.float32)
    c[100:140] = 2.0
    cod, sc, st = gpu_act(X, c, fmt, G, torch.bfloat16)
    ocod, osc, ost = O.quantize_act(X, c, fmt, G)
    assert np.array_equal(cod, ocod)
    assert np.array_equal(sc, osc)
    if fmt == O.NVFP4:
        assert np.array_equal(st.view(np.uint32), ost.view(np.uint32))


@pytest.mark.parametrize("fmt,G", FMTS)
@pytest.mark.parametrize("m,n,wdt", [(256, 256, torch.float32), (300, 512, torch.bfloat16),
                                     (1024, 4096, torch.bfloat16)])
def test_weight_pack_bit_exact(fmt, G, m, n, wdt):
    W, _ = synth.student_t_weight(m, n, 3, outlier_cols=4, outlier_scale=20.0,
                                  bf16=(wdt == torch.bfloat16))
    res = O.solve(W, fmt, G, 0)  # initial (valid, admissible) scales
    cod, sc = gpu_pack(W, res["r"], res["c"], res["s_T"], fmt, G, wdt)
    ocod, osc = O.pack_weight(W, fmt, G, res["r"], res["c"], res["s_T"])
    assert np.array_equal(cod, ocod)
    assert np.array_equal(sc, osc)


@pytest.mark.parametrize("fmt,G", [(O.NVFP4, 16), (O.MXFP4, 32)])
def test_weight_pack_full_size(fmt, G):
    """Full Llama-3.1-8B-shaped q/o projection (4096 x 4096, bf16)."""
    W, _ = synth.weight("llama8b_attn_nvfp4", 0)
    res = O.solve(W, fmt, G, 0)
    cod, sc = gpu_pack(W, res["r"], res["c"], res["s_T"], fmt, G)
    ocod, osc = O.pack_weight(W, fmt, G, res["r"], res["c"], res["s_T"])
    assert np.array_equal(cod, ocod)
    assert np.array_equal(sc, osc)
