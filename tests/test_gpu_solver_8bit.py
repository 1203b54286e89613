"""GPU parity of the solver on the 8-bit variants (DualQuant Appendix G.2,
Table 9: INT8 with G = 128 and bf16 scales, MXINT8 / MXFP8 with G = 32 and
E8M0 scales) against the oracle: the scales are the oracle's bit for bit
(the kernel recomputes updates near a projection boundary exactly), final
error and trace within 1e-4 relative."""
import numpy as np
import pytest
import torch

import oracle as O
from gpu_helpers import gpu_solve, gpu_solve_ex
from w4a4_post_quantization_dual_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("fmt,G,m,n,T,wdt", [
    (O.INT8, 128, 256, 512, 10, torch.bfloat16),
    (O.INT8, 64, 300, 256, 8, torch.float32),
    (O.MXINT8, 32, 384, 512, 10, torch.bfloat16),
    (O.MXFP8, 32, 384, 512, 10, torch.bfloat16),
    (O.MXFP8, 32, 130, 256, 6, torch.float32),
])
def test_solver_8bit_parity(fmt, G, m, n, T, wdt):
    W, _ = synth.student_t_weight(m, n, 70, outlier_cols=3, outlier_scale=20.0,
                                  bf16=(wdt == torch.bfloat16))
    r, c, sT, tr = gpu_solve(W, fmt, G, T, wdt)
    res = O.solve(W, fmt, G, T)
    assert np.array_equal(r, res["r"]) and np.array_equal(c, res["c"])
    assert sT == res["s_T"] == 1.0
    np.testing.assert_allclose(tr, res["trace"], rtol=1e-4, atol=0)
    assert np.all(np.diff(tr) <= tr[:-1] * 1e-6)


@pytest.mark.parametrize("fmt,G", [(O.MXFP8, 32), (O.INT8, 128)])
def test_solver_8bit_alpha_only_is_rtn_at_t0(fmt, G):
    W, _ = synth.student_t_weight(256, 256, 71, outlier_cols=2, outlier_scale=20.0)
    r, c, sT, tr = gpu_solve_ex(W, fmt, G, 0, flags=O.ALPHA_ONLY)
    res = O.solve_ex(W, fmt, G, 0, flags=O.ALPHA_ONLY)
    assert np.all(c == 1.0) and np.array_equal(r, res["r"])


def test_solver_8bit_full_size_sampled_tiles():
    """A 14336 x 4096 MLP weight in MXFP8 (T = 15), sampled tiles."""
    W, _ = synth.weight("llama8b_mlp_mx", 0)
    T = 15
    r, c, sT, tr = gpu_solve(W, O.MXFP8, 32, T)
    nb = W.shape[1] // 32
    tiles = [0, nb // 2, nb - 1]
    res = O.solve(W, O.MXFP8, 32, T, tiles=tiles)
    cols = np.concatenate([np.arange(b * 32, (b + 1) * 32) for b in tiles])
    assert np.array_equal(r[:, tiles], res["r"][:, tiles])
    assert np.array_equal(c[cols], res["c"][cols])
