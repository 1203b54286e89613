"""GPU parity of the decode linear (one token: the CUDA-core weight-streaming
kernel that dq_w4a4_linear takes for NVFP4 / MXFP4 when M == 1 and
K % 1024 == 0; two tokens take the tensor-core path and are checked beside
it) against the oracle's dequantised fp64 product.

Same bar as the tensor-core GEMM: relative Frobenius error <= 1e-3 with fp32
output (the block dot products are exact integers, the accumulation fp32),
and with bf16 output against the bf16 rounding of the reference, 99 % of the
elements identical.  The shapes cover a single 128-row group (fewer rows
than the grid's CTAs: one row each), CTA row ranges that start and end
inside a quad of rows, rows split over several warps and warps spanning
several rows, K of one and of many 1024-element chunks, the per-output-row
factor, and repeatability (no atomics: two calls give the same bits)."""
import numpy as np
import pytest
import torch

import oracle as O
from gpu_helpers import bf16_round, gpu_linear, rel_fro, to_dev
from w4a4_post_quantization_dual_b200 import dq, synth

pytestmark = pytest.mark.gpu


def operands(M, N, K, fmt, seed=0):
    G = O.NATIVE_GROUP[fmt]
    W, _ = synth.student_t_weight(N, K, seed, outlier_cols=max(1, K // 256), outlier_scale=10.0)
    res = O.solve(W, fmt, G, 0, tiles=[0])
    X, _ = synth.activations(M, K, 70 + seed, n_outliers=max(1, K // 100), outlier_scale=50.0)
    A, sA, st = O.quantize_act(X, res["c"], fmt, G)
    B, sB = O.pack_weight(W, fmt, G, res["r"], res["c"], res["s_T"])
    return A, sA, st, B, sB, res["s_T"]


@pytest.mark.parametrize("fmt", [O.NVFP4, O.MXFP4])
@pytest.mark.parametrize("M", [1, 2])
@pytest.mark.parametrize("N,K", [(128, 1024), (384, 3072), (1152, 2048), (640, 5120)])
def test_gemv_parity(fmt, M, N, K):
    A, sA, st, B, sB, sW = operands(M, N, K, fmt, seed=M * 7 + N)
    ref = O.linear(A, sA, st, B, sB, sW, M, N, K, fmt)
    Y32 = gpu_linear(A, sA, st, B, sB, sW, M, N, K, fmt, torch.float32)
    assert rel_fro(Y32, ref) <= 1e-3
    Y16 = gpu_linear(A, sA, st, B, sB, sW, M, N, K, fmt, torch.bfloat16)
    ref16 = bf16_round(ref)
    assert rel_fro(Y16, ref16) <= 1e-3
    assert np.mean(Y16 == ref16) >= 0.99


@pytest.mark.parametrize("fmt", [O.NVFP4, O.MXFP4])
def test_gemv_row_factor_and_repeatability(fmt):
    M, N, K = 1, 768, 4096
    A, sA, st, B, sB, sW = operands(M, N, K, fmt, seed=11)
    rr = np.exp(np.random.default_rng(2).uniform(-2, 2, N)).astype(np.float32)
    ref = O.linear(A, sA, st, B, sB, sW, M, N, K, fmt, r_row=rr)
    Y = gpu_linear(A, sA, st, B, sB, sW, M, N, K, fmt, torch.float32, r_row=rr)
    assert rel_fro(Y, ref) <= 1e-3
    args = [to_dev(A), to_dev(sA), to_dev(st) if st is not None else None, to_dev(B), to_dev(sB),
            to_dev(np.array([sW], np.float32))]
    Y1 = torch.empty((M, N), dtype=torch.float32, device="cuda")
    Y2 = torch.empty((M, N), dtype=torch.float32, device="cuda")
    dq.dq_w4a4_linear(*args, Y1, fmt)
    dq.dq_w4a4_linear(*args, Y2, fmt)
    torch.cuda.synchronize()
    assert torch.equal(Y1, Y2)


def test_gemv_zero_token():
    M, N, K = 1, 512, 2048
    A, sA, st, B, sB, sW = operands(M, N, K, O.NVFP4, seed=5)
    A[0] = 0
    st[0] = 0.0
    Y = gpu_linear(A, sA, st, B, sB, sW, M, N, K, O.NVFP4, torch.float32)
    assert np.all(Y[0] == 0.0)
    ref = O.linear(A, sA, st, B, sB, sW, M, N, K, O.NVFP4)
    assert rel_fro(Y, ref) <= 1e-3


@pytest.mark.parametrize("fmt,M,N,K", [
    (O.NVFP4, 1, 27648, 5120),    # Qwen-32B up projection, one token
    (O.NVFP4, 1, 5120, 27648),    # Qwen-32B down projection, one token
    (O.MXFP4, 1, 14336, 4096),    # Llama-3.1-8B gate/up, MX
])
def test_gemv_full_size_sampled(fmt, M, N, K):
    A, sA, st, B, sB, sW = operands(M, N, K, fmt, seed=3)
    Y = gpu_linear(A, sA, st, B, sB, sW, M, N, K, fmt, torch.float32)
    g = np.random.default_rng(N)
    rows = np.arange(M)
    cols = np.unique(np.concatenate([[0, N - 1], g.integers(0, N, 600)]))
    ref = O.linear_rows(A, sA, st, B, sB, sW, rows, M, N, K, fmt, cols=cols)
    assert rel_fro(Y[np.ix_(rows, cols)], ref) <= 1e-3
    assert np.all(np.isfinite(Y))


def test_no_device_error_recorded():
    assert dq.dq_device_error(clear=True) == 0
