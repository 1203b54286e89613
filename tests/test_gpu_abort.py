"""The expiry path of the device-side bounded waits of the GEMMs, on the GPU.

Every mbarrier wait inside the GEMM pipelines has a time limit.  When one
runs out the kernel records DQ_ERR_DEVICE_TIMEOUT in the device error word
and unwinds: each role first waits (with a fixed 2 s
limit) for the copies and tensor-core work it already issued, then the CTA
releases its tensor memory and exits.  dq_set_wait_limit shortens the limit
so that the waits of an ordinary call run out; nothing here waits on a flag
that is never set and nothing faults.  Each test checks that the call
returns, that the error word reports the timeout, and that, with the limit
restored, the same call gives the result it gave before (and the GEMM its
oracle parity), so the context is intact."""
import numpy as np
import pytest
import torch

import oracle as O
from gpu_helpers import rel_fro
from w4a4_post_quantization_dual_b200 import dq, synth

pytestmark = pytest.mark.gpu
DEV = "cuda"
TINY_NS = 100          # a limit that the first wait of every CTA outlasts
DQ_ERR_DEVICE_TIMEOUT = 4


@pytest.fixture(autouse=True)
def restore_limit():
    dq.dq_device_error(clear=True)
    yield
    dq.dq_set_wait_limit(0)
    dq.dq_device_error(clear=True)


def _layer(N, K, fmt, seed):
    W, _ = synth.student_t_weight(N, K, seed, outlier_cols=3, outlier_scale=20.0)
    q, _, _ = dq.quantize_linear(torch.from_numpy(W).to(torch.bfloat16).to(DEV), fmt, 2)
    return q


def _acts(M, K, q, fmt, seed):
    X, _ = synth.activations(M, K, seed, n_outliers=4, outlier_scale=50.0)
    Xd = torch.from_numpy(X).to(torch.bfloat16).to(DEV)
    G = dq.native_group(fmt)
    A = torch.empty((M, K // 2), dtype=torch.uint8, device=DEV)
    sA = torch.empty(dq.scales_bytes(M, K, fmt, G), dtype=torch.uint8, device=DEV)
    st = torch.empty(M, dtype=torch.float32, device=DEV) if fmt == "nvfp4" else None
    dq.dq_quantize_act(Xd, fmt, q.c, A, sA, st, group=G)
    return Xd, A, sA, st


def _expire_then_recover(run):
    """run() enqueues the call and returns its output tensor."""
    ref = run().clone()
    torch.cuda.synchronize()
    assert dq.dq_device_error(clear=True) == 0
    dq.dq_set_wait_limit(TINY_NS)
    run()
    torch.cuda.synchronize()
    assert dq.dq_device_error(clear=True) == DQ_ERR_DEVICE_TIMEOUT
    dq.dq_set_wait_limit(0)
    again = run()
    torch.cuda.synchronize()
    assert dq.dq_device_error(clear=True) == 0
    assert torch.equal(again, ref)
    return again


# (M, N, K): the 128 x 256 persistent kernel, the paired-SM kernel, split-K
# (small M), and the 128 x 128 persistent kernel
@pytest.mark.parametrize("M,N,K", [(2048, 4096, 512), (4096, 1024, 1024), (8, 1024, 4096),
                                   (8192, 384, 256)])
def test_gemm_wait_expiry_unwinds(M, N, K):
    fmt = "nvfp4"
    q = _layer(N, K, fmt, 200 + M)
    _, A, sA, st = _acts(M, K, q, fmt, 201 + M)
    Y = torch.empty((M, N), dtype=torch.float32, device=DEV)

    def run():
        dq.dq_w4a4_linear(A, sA, st, q.codes, q.scales, q.s_tensor, Y, fmt)
        return Y

    Yd = _expire_then_recover(run)
    # the recovered call still matches the oracle's fp64 product
    rows = np.unique(np.linspace(0, M - 1, min(M, 24)).astype(int))
    ref = O.linear_rows(A.cpu().numpy(), sA.cpu().numpy(), st.cpu().numpy(), q.codes.cpu().numpy(),
                        q.scales.cpu().numpy(), float(q.s_tensor.cpu()[0]), rows, M, N, K, O.NVFP4)
    assert rel_fro(Yd.cpu().numpy()[rows], ref) <= 1e-3


def test_mxint4_gemm_wait_expiry_unwinds():
    fmt, M, N, K = "mxint4", 256, 512, 1024
    q = _layer(N, K, fmt, 210)
    _, A, sA, _ = _acts(M, K, q, fmt, 211)
    Y = torch.empty((M, N), dtype=torch.bfloat16, device=DEV)

    def run():
        dq.dq_w4a4_linear(A, sA, None, q.codes, q.scales, None, Y, fmt)
        return Y

    _expire_then_recover(run)


def test_fused_linear_wait_expiry_unwinds():
    fmt, M, N, K = "nvfp4", 1, 1024, 4096
    q = _layer(N, K, fmt, 220)
    Xd, _, _, _ = _acts(M, K, q, fmt, 221)
    Y = torch.empty((M, N), dtype=torch.bfloat16, device=DEV)

    def run():
        dq.dq_w4a4_linear_fused(Xd, q.c, q.codes, q.scales, q.s_tensor, Y, fmt)
        return Y

    _expire_then_recover(run)

