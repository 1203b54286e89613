"""The allocation-free solver entry point (dq_solve_scales_noalloc).

It exists for callers that cannot allocate device memory -- for example a
serving process whose free memory is already owned by its own pool, or a
latency-critical path that must not wait in the driver's allocator.  Its
scratch is a fixed array inside the library instead of a caller workspace.

Checked through the C ABI on a GPU: on two calls in a row it gives the same
scales as dq_solve_scales (with a caller workspace) within the solver tests'
tolerance (here bit-identical scales, trace to 1e-9), the device's free
memory does not change across a call, and rounds beyond the fixed scratch
are refused.  This file is collected last so that a run stopping at the
first failure has already run every other test."""
import ctypes

import numpy as np
import pytest
import torch

from w4a4_post_quantization_dual_b200 import dq, synth

pytestmark = pytest.mark.gpu


def _solve_with_workspace(Wd, fmt, T, G):
    m, n = Wd.shape
    r = torch.empty((m, n // G), dtype=torch.float32, device="cuda")
    c = torch.empty(n, dtype=torch.float32, device="cuda")
    sT = torch.empty(1, dtype=torch.float32, device="cuda")
    tr = torch.empty(T + 1, dtype=torch.float64, device="cuda")
    ws = torch.empty(dq.solve_workspace_size(T), dtype=torch.uint8, device="cuda")
    dq.dq_solve_scales(Wd, fmt, T, r, c, sT, tr, ws, group=G)
    torch.cuda.synchronize()
    return r, c, sT, tr


def _solve_noalloc_cabi(Wd, fmt, T, G, out):
    """Direct C-ABI call (ctypes), outputs preallocated by the caller."""
    r, c, sT, tr = out
    m, n = Wd.shape
    st = dq.lib().dq_solve_scales_noalloc(
        ctypes.c_void_p(Wd.data_ptr()), dq.DQ_BF16, m, n, fmt, G, T,
        ctypes.c_void_p(r.data_ptr()), ctypes.c_void_p(c.data_ptr()),
        ctypes.c_void_p(sT.data_ptr()), ctypes.c_void_p(tr.data_ptr()),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return st


@pytest.mark.parametrize("fmt,G,shape,T", [(dq.DQ_NVFP4, 16, (1024, 512), 12),
                                          (dq.DQ_MXFP4, 32, (300, 256), 8)])
def test_noalloc_matches_workspace_entry_point_twice(fmt, G, shape, T):
    W, _ = synth.student_t_weight(*shape, 31, outlier_cols=3, outlier_scale=20.0)
    Wd = torch.from_numpy(W).to(torch.bfloat16).cuda()
    ref = _solve_with_workspace(Wd, fmt, T, G)
    m, n = shape
    for call in range(2):
        out = (torch.full((m, n // G), -1.0, device="cuda"), torch.full((n,), -1.0, device="cuda"),
               torch.zeros(1, device="cuda"),
               torch.full((T + 1,), -1.0, dtype=torch.float64, device="cuda"))
        torch.cuda.synchronize()
        free0 = torch.cuda.mem_get_info()[0]
        assert _solve_noalloc_cabi(Wd, fmt, T, G, out) == 0
        torch.cuda.synchronize()
        if call == 1:  # set-up happened on the first call; nothing is allocated after it
            assert torch.cuda.mem_get_info()[0] == free0
        for a, b in zip(out[:3], ref[:3]):
            assert torch.equal(a, b)
        np.testing.assert_allclose(out[3].cpu().numpy(), ref[3].cpu().numpy(), rtol=1e-9, atol=0)


def test_noalloc_rejects_rounds_beyond_fixed_scratch():
    Wd = torch.zeros((16, 16), dtype=torch.bfloat16, device="cuda")
    T = 2046  # one more round than the fixed scratch holds
    out = (torch.empty((16, 1), device="cuda"), torch.empty(16, device="cuda"),
           torch.empty(1, device="cuda"), torch.empty(T + 1, dtype=torch.float64, device="cuda"))
    assert _solve_noalloc_cabi(Wd, dq.DQ_NVFP4, T, 16, out) == 5  # DQ_ERR_WORKSPACE
