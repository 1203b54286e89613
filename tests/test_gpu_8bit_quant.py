"""GPU parity of the 8-bit packer and activation quantiser (INT8, MXINT8,
MXFP8; DualQuant Appendix G.2) against the oracle: codes and scale bytes
bit-exact, including the padding of the tensor-core scale layout; and the
activation error sums (Appendix E measure) within rtol 1e-9."""
import numpy as np
import pytest
import torch

import oracle as O
from gpu_helpers import gpu_act, gpu_pack, gpu_solve, to_dev, DEV
from w4a4_post_quantization_dual_b200 import dq, synth

pytestmark = pytest.mark.gpu

FMTS8 = [(O.INT8, 128), (O.INT8, 64), (O.MXINT8, 32), (O.MXFP8, 32)]


@pytest.mark.parametrize("fmt,G", FMTS8)
@pytest.mark.parametrize("M,K,xdtype", [(1, 4096, torch.bfloat16), (300, 1024, torch.bfloat16),
                                        (17, 512, torch.float32)])
def test_act_quant_8bit_bit_exact(fmt, G, M, K, xdtype):
    X, _ = synth.activations(M, K, 90, n_outliers=4, outlier_scale=50.0)
    if xdtype == torch.bfloat16:
        X = torch.from_numpy(X).to(torch.bfloat16).to(torch.float32).numpy()
    c = np.exp(np.random.default_rng(91).uniform(-1, 1, K)).astype(np.float32)
    cod, sc, _ = gpu_act(X, c, fmt, G, xdtype)
    wcod, wsc, _ = O.quantize_act(X, c, fmt, G)
    assert np.array_equal(cod, wcod)
    assert np.array_equal(np.asarray(sc).reshape(-1), np.asarray(wsc).reshape(-1))


@pytest.mark.parametrize("fmt,G", FMTS8)
def test_pack_weight_8bit_bit_exact(fmt, G):
    W, _ = synth.student_t_weight(300, 512, 92, outlier_cols=3, outlier_scale=20.0, bf16=True)
    r, c, sT, _ = gpu_solve(W, fmt, G, 6, trace=False)
    cod, sc = gpu_pack(W, r, c, sT, fmt, G)
    wcod, wsc = O.pack_weight(W, fmt, G, r, c, sT)
    assert np.array_equal(cod, wcod)
    assert np.array_equal(np.asarray(sc).reshape(-1), np.asarray(wsc).reshape(-1))


@pytest.mark.parametrize("fmt,G", FMTS8)
def test_act_error_8bit_parity(fmt, G):
    X, _ = synth.activations(64, 1024, 93, n_outliers=4, outlier_scale=50.0)
    X = torch.from_numpy(X).to(torch.bfloat16).to(torch.float32).numpy()
    c = np.exp(np.random.default_rng(94).uniform(-1, 1, 1024)).astype(np.float32)
    Xd, cd = to_dev(X, torch.bfloat16), to_dev(c)
    A = torch.empty((64, 1024), dtype=torch.uint8, device=DEV)
    sA = torch.empty(dq.scales_bytes(64, 1024, fmt, G), dtype=torch.uint8, device=DEV)
    sums = torch.empty(2, dtype=torch.float64, device=DEV)
    dq.dq_quantize_act(Xd, fmt, cd, A, sA, None, group=G)
    dq.dq_act_quant_error(Xd, fmt, cd, A, sA, None, sums, group=G)
    np.testing.assert_allclose(sums.cpu().numpy(), O.act_error_sums(X, c, fmt, G), rtol=1e-9)


@pytest.mark.parametrize("fmt", [O.MXFP8, O.MXINT8])
@pytest.mark.parametrize("M,N,K", [(1, 256, 512), (130, 256, 512), (300, 1024, 2048)])
@pytest.mark.parametrize("ydtype", [torch.float32, torch.bfloat16])
def test_mx8_linear_parity(fmt, M, N, K, ydtype):
    """MXFP8 linear (E4M3 codes, E8M0 32-blocks, tcgen05 kind::mxf8f6f4) and
    MXINT8 linear (int8 codes dequantised exactly to bf16 on chip, kind::f16)
    on the device's own codes vs the fp64 reference product: relative
    Frobenius error <= 1e-3 (fp32 output) / bf16 rounding of the reference."""
    X, _ = synth.activations(M, K, 95, n_outliers=4, outlier_scale=50.0)
    X = torch.from_numpy(X).to(torch.bfloat16).to(torch.float32).numpy()
    W, _ = synth.student_t_weight(N, K, 96, outlier_cols=3, outlier_scale=20.0, bf16=True)
    r, c, sT, _ = gpu_solve(W, fmt, 32, 5, trace=False)
    A, sA, _ = gpu_act(X, c, fmt, 32)
    B, sB = gpu_pack(W, r, c, sT, fmt, 32)
    Y = torch.empty((M, N), dtype=ydtype, device=DEV)
    dq.dq_w4a4_linear(to_dev(A), to_dev(sA), None, to_dev(B), to_dev(sB), None, Y, fmt)
    torch.cuda.synchronize()
    ref = O.linear(A, sA, None, B, sB, 1.0, M, N, K, fmt)
    got = Y.float().cpu().numpy().astype(np.float64)
    if ydtype == torch.float32:
        assert np.linalg.norm(got - ref) <= 1e-3 * np.linalg.norm(ref)
    else:
        refb = torch.from_numpy(ref).to(torch.bfloat16).double().numpy()
        assert np.linalg.norm(got - refb) <= 1e-3 * np.linalg.norm(refb)
