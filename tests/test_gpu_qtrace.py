"""GPU parity of the solver's code-change trace (DQ_SOLVE_TRACE_CODES): the
relative change ||Qhat(t) - Qhat(t-1)||_F / ||Qhat(t-1)||_F of Fig. 2(a) /
Fig. 3(a) in "DualQuant" equals the oracle's (the kernel's scales are the
oracle's bit for bit, so are its codes; the sums are exact), and the MSE
half of the trace is unchanged by the flag."""
import numpy as np
import pytest
import torch

import oracle as O
from gpu_helpers import DEV, to_dev
from w4a4_post_quantization_dual_b200 import dq, synth

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("fmt,G,m,n,wdt", [
    (O.NVFP4, 16, 384, 512, torch.bfloat16),
    (O.MXFP4, 32, 300, 512, torch.bfloat16),
    (O.INT4, 64, 256, 512, torch.float32),
    (O.MXFP8, 32, 256, 256, torch.bfloat16),
])
def test_code_change_trace_parity(fmt, G, m, n, wdt):
    W, _ = synth.student_t_weight(m, n, 130, outlier_cols=3, outlier_scale=20.0,
                                  bf16=(wdt == torch.bfloat16))
    T = 8
    Wd = to_dev(W.astype(np.float32), wdt)
    r = torch.empty((m, n // G), device=DEV)
    c = torch.empty(n, device=DEV)
    sT = torch.empty(1, device=DEV)
    tr = torch.full((2 * (T + 1),), -1.0, dtype=torch.float64, device=DEV)
    ws = torch.empty(dq.solve_workspace_size(T), dtype=torch.uint8, device=DEV)
    dq.dq_solve_scales_ex(Wd, fmt, T, r, c, sT, flags=dq.DQ_SOLVE_TRACE_CODES, mse_trace=tr,
                          workspace=ws, group=G)
    torch.cuda.synchronize()
    got = tr.cpu().numpy()
    res = O.solve_qtrace(W, fmt, G, T)
    assert np.array_equal(r.cpu().numpy(), res["r"]) and np.array_equal(c.cpu().numpy(), res["c"])
    np.testing.assert_allclose(got[:T + 1], res["trace"], rtol=1e-4, atol=0)
    assert np.isnan(got[T + 1])
    np.testing.assert_allclose(got[T + 2:], res["qchange"][1:], rtol=1e-12, atol=0)
