"""GPU tests of the fused activation-quantise + linear kernel
(dq_w4a4_linear_fused, NVFP4, small token counts): its output equals the
unfused pair dq_quantize_act -> dq_w4a4_linear bit for bit (same codes,
same scales, same MMAs), whose parity with the oracle is tested elsewhere."""
import numpy as np
import pytest
import torch

from w4a4_post_quantization_dual_b200 import dq, synth

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _layer(N, K, seed):
    W, _ = synth.student_t_weight(N, K, seed, outlier_cols=3, outlier_scale=20.0, bf16=True)
    q, _, _ = dq.quantize_linear(torch.from_numpy(W).to(torch.bfloat16).to(DEV), "nvfp4", 5)
    return q


@pytest.mark.parametrize("M,N,K", [(1, 4096, 4096), (16, 1024, 4096), (100, 1024, 2048),
                                   (16, 4096, 1024)])
@pytest.mark.parametrize("ydtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("with_c,with_r", [(True, False), (False, True)])
def test_fused_equals_unfused(M, N, K, ydtype, with_c, with_r):
    q = _layer(N, K, 110)
    X, _ = synth.activations(M, K, 111, n_outliers=4, outlier_scale=50.0)
    Xd = torch.from_numpy(X).to(torch.bfloat16).to(DEV)
    c = q.c if with_c else None
    r_row = (torch.rand(N, device=DEV) + 0.5) if with_r else None
    # unfused reference through the public pair
    A = torch.empty((M, K // 2), dtype=torch.uint8, device=DEV)
    sA = torch.empty(dq.scales_bytes(M, K, "nvfp4", 16), dtype=torch.uint8, device=DEV)
    st = torch.empty(M, dtype=torch.float32, device=DEV)
    dq.dq_quantize_act(Xd, "nvfp4", c, A, sA, st, group=16)
    Y1 = torch.empty((M, N), dtype=ydtype, device=DEV)
    dq.dq_w4a4_linear(A, sA, st, q.codes, q.scales, q.s_tensor, Y1, "nvfp4", r_row=r_row)
    Y2 = torch.full((M, N), 7.0, dtype=ydtype, device=DEV)
    dq.dq_w4a4_linear_fused(Xd, c, q.codes, q.scales, q.s_tensor, Y2, "nvfp4", r_row=r_row)
    torch.cuda.synchronize()
    assert dq.dq_device_error(clear=True) == 0
    assert torch.equal(Y1, Y2)


def test_fused_refuses_shapes_without_a_fitting_split():
    q = _layer(16384, 4096, 112)
    Xd = torch.zeros((1, 4096), dtype=torch.bfloat16, device=DEV)
    Y = torch.empty((1, 16384), dtype=torch.bfloat16, device=DEV)
    with pytest.raises(dq.DQError):
        dq.dq_w4a4_linear_fused(Xd, q.c, q.codes, q.scales, q.s_tensor, Y, "nvfp4")
