"""GPU parity of the block-scaled FP4 GEMM (tcgen05) against the oracle's
dequantised fp64 product.

Tolerance: relative Frobenius error <= 1e-3 with fp32 output (FP32
accumulation; expected ~1e-6).  With bf16 output the kernel's result is
compared with the bf16 rounding of the fp64 reference at the same 1e-3 bound,
and at least 99 % of the elements must round to the identical bf16 value
(a flip needs the fp32 accumulation error to straddle a bf16 rounding
boundary).  Full-size shapes are checked on sampled output rows/columns."""
import numpy as np
import pytest
import torch

import oracle as O
from gpu_helpers import bf16_round, gpu_linear, rel_fro
from w4a4_post_quantization_dual_b200 import synth

pytestmark = pytest.mark.gpu


def operands(M, N, K, fmt, seed=0, T=0, x_outliers=0.01, x_scale=50.0):
    G = O.NATIVE_GROUP[fmt]
    W, _ = synth.student_t_weight(N, K, seed, outlier_cols=max(1, K // 256), outlier_scale=10.0)
    res = O.solve(W, fmt, G, T, tiles=[0])  # T=0: admissible initial scales for every tile
    X, _ = synth.activations(M, K, 50 + seed, n_outliers=max(1, int(K * x_outliers)),
                             outlier_scale=x_scale)
    A, sA, st = O.quantize_act(X, res["c"], fmt, G)
    B, sB = O.pack_weight(W, fmt, G, res["r"], res["c"], res["s_T"])
    return A, sA, st, B, sB, res["s_T"]


@pytest.mark.parametrize("fmt", [O.NVFP4, O.MXFP4, O.MXINT4])
@pytest.mark.parametrize("M,N,K", [(16, 256, 256), (1, 512, 4096), (300, 512, 768),
                                   (128, 128, 256), (257, 384, 512), (1000, 1024, 1024),
                                   (64, 4096, 4096), (8, 1024, 5120)])
def test_gemm_small_parity(fmt, M, N, K):
    A, sA, st, B, sB, sW = operands(M, N, K, fmt, seed=M + N)
    ref = O.linear(A, sA, st, B, sB, sW, M, N, K, fmt)
    Y32 = gpu_linear(A, sA, st, B, sB, sW, M, N, K, fmt, torch.float32)
    assert rel_fro(Y32, ref) <= 1e-3
    Y16 = gpu_linear(A, sA, st, B, sB, sW, M, N, K, fmt, torch.bfloat16)
    ref16 = bf16_round(ref)
    assert rel_fro(Y16, ref16) <= 1e-3
    assert np.mean(Y16 == ref16) >= 0.99


@pytest.mark.parametrize("fmt,M,N,K", [(O.NVFP4, 300, 9216, 512), (O.MXFP4, 200, 9216, 768),
                                        (O.NVFP4, 512, 8960, 256)])
def test_gemm_paired_tiles_parity(fmt, M, N, K):
    """Shapes with enough 256 x 256 tiles for the paired-SM kernel, including
    a ragged last tile whose second CTA lies entirely beyond M, and the
    per-output-row factor in its epilogue."""
    A, sA, st, B, sB, sW = operands(M, N, K, fmt, seed=M + K)
    rr = np.exp(np.random.default_rng(1).uniform(-1, 1, N)).astype(np.float32)
    ref = O.linear(A, sA, st, B, sB, sW, M, N, K, fmt, r_row=rr)
    Y32 = gpu_linear(A, sA, st, B, sB, sW, M, N, K, fmt, torch.float32, r_row=rr)
    assert rel_fro(Y32, ref) <= 1e-3
    Y16 = gpu_linear(A, sA, st, B, sB, sW, M, N, K, fmt, torch.bfloat16, r_row=rr)
    ref16 = bf16_round(ref)
    assert rel_fro(Y16, ref16) <= 1e-3
    assert np.mean(Y16 == ref16) >= 0.99


def test_gemm_row_factor_epilogue():
    M, N, K = 64, 256, 512
    A, sA, st, B, sB, sW = operands(M, N, K, O.NVFP4, seed=3)
    rr = np.exp(np.random.default_rng(0).uniform(-2, 2, N)).astype(np.float32)
    ref = O.linear(A, sA, st, B, sB, sW, M, N, K, O.NVFP4, r_row=rr)
    Y = gpu_linear(A, sA, st, B, sB, sW, M, N, K, O.NVFP4, torch.float32, r_row=rr)
    assert rel_fro(Y, ref) <= 1e-3


@pytest.mark.parametrize("fmt,M,N,K", [
    (O.NVFP4, 4096, 4096, 4096),    # Llama-3.1-8B q/o projection, prefill
    (O.NVFP4, 1, 1024, 4096),       # k/v projection, decode (split-K over a cluster)
    (O.NVFP4, 8, 27648, 5120),      # Qwen-32B up projection, decode
    (O.MXFP4, 2048, 14336, 4096),   # gate/up, MX
    (O.MXINT4, 2048, 14336, 4096),  # gate/up, MXINT4 (widened on chip to E4M3)
    (O.MXINT4, 2048, 4096, 14336),  # down, MXINT4
    (O.NVFP4, 8192, 5120, 27648),   # Qwen-32B down projection, prefill
])
def test_gemm_full_size_sampled(fmt, M, N, K):
    A, sA, st, B, sB, sW = operands(M, N, K, fmt, seed=1)
    Y = gpu_linear(A, sA, st, B, sB, sW, M, N, K, fmt, torch.float32)
    g = np.random.default_rng(M)
    rows = np.unique(np.concatenate([[0, M - 1], g.integers(0, M, 30)]))
    cols = np.unique(np.concatenate([[0, N - 1], g.integers(0, N, 500)]))
    ref = O.linear_rows(A, sA, st, B, sB, sW, rows, M, N, K, fmt, cols=cols)
    assert rel_fro(Y[np.ix_(rows, cols)], ref) <= 1e-3
    assert np.all(np.isfinite(Y))


def test_gemm_zero_activation_rows():
    M, N, K = 40, 256, 512
    A, sA, st, B, sB, sW = operands(M, N, K, O.NVFP4, seed=9)
    A[5] = 0
    st[5] = 0.0
    Y = gpu_linear(A, sA, st, B, sB, sW, M, N, K, O.NVFP4, torch.float32)
    assert np.all(Y[5] == 0.0)
    ref = O.linear(A, sA, st, B, sB, sW, M, N, K, O.NVFP4)
    assert rel_fro(Y, ref) <= 1e-3


def test_no_device_error_recorded():
    from w4a4_post_quantization_dual_b200 import dq
    assert dq.dq_device_error(clear=True) == 0
