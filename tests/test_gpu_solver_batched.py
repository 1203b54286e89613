"""GPU tests of the batched solver entry (dq_solve_scales_batched): every
weight's scales are exactly those of its own dq_solve_scales call (tiles
are independent problems, Algorithm 1 per m x G tile), whichever weights
share its launch; traces agree up to the order of fp64 atomic adds."""
import numpy as np
import pytest
import torch

import oracle as O
from gpu_helpers import DEV, gpu_solve_ex, to_dev
from w4a4_post_quantization_dual_b200 import dq, synth

pytestmark = pytest.mark.gpu


def _outputs(Ws, G, T):
    rs = [torch.full((W.shape[0], W.shape[1] // G), -1.0, device=DEV) for W in Ws]
    cs = [torch.full((W.shape[1],), -1.0, device=DEV) for W in Ws]
    ss = [torch.zeros(1, device=DEV) for _ in Ws]
    ts = [torch.full((T + 1,), -1.0, dtype=torch.float64, device=DEV) for _ in Ws]
    return rs, cs, ss, ts


def _single(W, fmt, G, T, flags=0):
    r, c, s, t = _outputs([W], G, T)
    ws = torch.empty(dq.solve_workspace_size(T), dtype=torch.uint8, device=DEV)
    dq.dq_solve_scales_ex(W, fmt, T, r[0], c[0], s[0], flags=flags, mse_trace=t[0],
                          workspace=ws, group=G)
    return r[0], c[0], s[0], t[0]


def _batched(Ws, fmt, G, T, flags=0, traces=True):
    rs, cs, ss, ts = _outputs(Ws, G, T)
    ws = torch.empty(dq.solve_batched_workspace_size(len(Ws), T), dtype=torch.uint8,
                     device=DEV)
    dq.dq_solve_scales_batched(Ws, fmt, T, rs, cs, ss, ts if traces else None, ws,
                               flags=flags, group=G)
    return rs, cs, ss, ts


@pytest.mark.parametrize("fmt,G", [(O.NVFP4, 16), (O.MXFP4, 32), (O.MXINT4, 32), (O.INT4, 64),
                                   (O.INT4, 128)])
@pytest.mark.parametrize("flags", [0, O.ALPHA_ONLY, O.BETA_ONLY])
def test_batched_equals_separate_calls(fmt, G, flags):
    shapes = [(384, 512), (300, 256), (384, 1024), (300, 512), (384, 256)]
    Ws = [to_dev(synth.student_t_weight(m, n, 60 + i, outlier_cols=3, outlier_scale=20.0,
                                        bf16=True)[0], torch.bfloat16)
          for i, (m, n) in enumerate(shapes)]
    T = 6
    rs, cs, ss, ts = _batched(Ws, fmt, G, T, flags)
    for i, W in enumerate(Ws):
        r, c, s, t = _single(W, fmt, G, T, flags)
        assert torch.equal(rs[i], r) and torch.equal(cs[i], c) and torch.equal(ss[i], s)
        np.testing.assert_allclose(ts[i].cpu().numpy(), t.cpu().numpy(), rtol=1e-12, atol=0)
    # and the oracle's scales for one member of the batch
    Wh = Ws[1].float().cpu().numpy()
    res = O.solve_ex(Wh, fmt, G, T, flags=flags)
    assert np.array_equal(rs[1].cpu().numpy(), res["r"])
    assert np.array_equal(cs[1].cpu().numpy(), res["c"])


def test_batched_more_weights_than_one_launch_holds():
    """18 weights of one row count: two launches, no traces."""
    Ws = [to_dev(synth.student_t_weight(128, 64 * (1 + i % 3), 80 + i, bf16=True)[0],
                 torch.bfloat16) for i in range(18)]
    rs, cs, ss, _ = _batched(Ws, O.NVFP4, 16, 4, traces=False)
    for i in (0, 7, 16, 17):
        r, c, s, _ = _single(Ws[i], O.NVFP4, 16, 4)
        assert torch.equal(rs[i], r) and torch.equal(cs[i], c) and torch.equal(ss[i], s)


def test_batched_llama_layer_shapes():
    """The seven projections of one Llama-3.1-8B layer (q, k, v, o, gate, up,
    down), NVFP4, T = 5: three launches (m = 4096, 1024, 14336)."""
    shapes = [(4096, 4096), (1024, 4096), (1024, 4096), (4096, 4096), (14336, 4096),
              (14336, 4096), (4096, 14336)]
    g = torch.Generator(device=DEV)
    g.manual_seed(3)
    Ws = [(torch.randn(m, n, device=DEV, generator=g) * 0.02).to(torch.bfloat16)
          for m, n in shapes]
    rs, cs, ss, ts = _batched(Ws, O.NVFP4, 16, 5)
    for i, W in enumerate(Ws):
        r, c, s, t = _single(W, O.NVFP4, 16, 5)
        assert torch.equal(rs[i], r) and torch.equal(cs[i], c) and torch.equal(ss[i], s)
        np.testing.assert_allclose(ts[i].cpu().numpy(), t.cpu().numpy(), rtol=1e-12, atol=0)
