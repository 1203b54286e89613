"""GPU parity of the activation quantisation error measure (the activation
SQNR with and without beta, DualQuant Appendix E, Table 6) through
dq_act_quant_error: the device sums equal the oracle's fp64 sums (up to the
order of the fp64 atomic adds, rtol 1e-9), on the GPU's own codes and on
the oracle's codes fed to the device."""
import numpy as np
import pytest
import torch

import oracle as O
from gpu_helpers import DEV, to_dev
from w4a4_post_quantization_dual_b200 import dq, synth

pytestmark = pytest.mark.gpu

FMTS = [(O.NVFP4, 16), (O.MXFP4, 32), (O.MXINT4, 32), (O.INT4, 64), (O.INT4, 128)]


def _device_sums(X, c, fmt, G, xdtype, codes=None, scales=None, s_tok=None):
    M, K = X.shape
    Xd = to_dev(X.astype(np.float32), xdtype)
    cd = to_dev(np.asarray(c, np.float32)) if c is not None else None
    if codes is None:
        A = torch.empty((M, K // 2), dtype=torch.uint8, device=DEV)
        sA = torch.empty(dq.scales_bytes(M, K, fmt, G), dtype=torch.uint8, device=DEV)
        st = torch.empty(M, dtype=torch.float32, device=DEV) if fmt == O.NVFP4 else None
        dq.dq_quantize_act(Xd, fmt, cd, A, sA, st, group=G)
    else:
        A, sA = to_dev(codes), to_dev(np.ascontiguousarray(scales).view(np.uint8).reshape(-1))
        st = to_dev(s_tok) if fmt == O.NVFP4 else None
    sums = torch.full((2,), -1.0, dtype=torch.float64, device=DEV)
    dq.dq_act_quant_error(Xd, fmt, cd, A, sA, st, sums, group=G)
    torch.cuda.synchronize()
    return sums.cpu().numpy()


@pytest.mark.parametrize("fmt,G", FMTS)
@pytest.mark.parametrize("with_c", [False, True])
@pytest.mark.parametrize("M,K,xdtype", [(300, 4096, torch.bfloat16), (17, 1024, torch.float32)])
def test_act_error_parity(fmt, G, with_c, M, K, xdtype):
    X, _ = synth.activations(M, K, 7, n_outliers=4, outlier_scale=50.0)
    if xdtype == torch.bfloat16:
        X = torch.from_numpy(X).to(torch.bfloat16).to(torch.float32).numpy()
    c = None
    if with_c:
        c = np.exp(np.random.default_rng(8).uniform(-1.5, 1.5, K)).astype(np.float32)
    want = O.act_error_sums(X, c, fmt, G)
    got = _device_sums(X, c, fmt, G, xdtype)
    np.testing.assert_allclose(got, want, rtol=1e-9, atol=0)
    # the kernel alone, on the oracle's codes
    cod, sc, st = O.quantize_act(X, np.ones(K, np.float32) if c is None else c, fmt, G)
    got2 = _device_sums(X, c, fmt, G, xdtype, cod, sc, st)
    np.testing.assert_allclose(got2, want, rtol=1e-9, atol=0)


def test_act_sqnr_with_and_without_beta():
    """The convenience call returns the oracle's SQNR for both arms on the
    4096 x 4096 attention projection's solved column scales."""
    W, _ = synth.weight("llama8b_attn_nvfp4", 0)
    X, _ = synth.activations(256, 4096, 11, n_outliers=8, outlier_scale=50.0)
    X = torch.from_numpy(X).to(torch.bfloat16).to(torch.float32).numpy()
    from gpu_helpers import gpu_solve
    _, c, _, _ = gpu_solve(W, O.NVFP4, 16, 15, trace=False)
    Xd = to_dev(X, torch.bfloat16)
    cd = to_dev(c)
    with_b = dq.act_sqnr_db(Xd, dq.DQ_NVFP4, cd)
    without = dq.act_sqnr_db(Xd, dq.DQ_NVFP4, None)
    assert with_b == pytest.approx(O.act_sqnr_db(X, c, O.NVFP4, 16), abs=1e-7)
    assert without == pytest.approx(O.act_sqnr_db(X, None, O.NVFP4, 16), abs=1e-7)
