"""GPU parity of the solver's ablation modes and warm start (DualQuant,
Table 4 scale ablation; initialisation (alpha_0, beta_0) of Section 5.3
given by the caller) against the oracle, through dq_solve_scales_ex.

Tolerances as for the full solver (fp accumulation order differs): final
error within 1e-4 relative, >= 99.9 % identical codes, trace within 1e-4
relative per round.  What the mode fixes is compared exactly: c = 1 for
alpha-only, r = its initial value for beta-only, the projected warm-start
scales at T = 0, and the NVFP4 tensor scale."""
import numpy as np
import pytest
import torch

import oracle as O
from gpu_helpers import gpu_solve, gpu_solve_ex
from w4a4_post_quantization_dual_b200 import synth

pytestmark = pytest.mark.gpu

CASES = [
    (O.NVFP4, 16, 384, 512, torch.bfloat16),
    (O.MXFP4, 32, 384, 512, torch.bfloat16),
    (O.MXINT4, 32, 300, 512, torch.bfloat16),    # ragged row count
    (O.INT4, 64, 256, 512, torch.bfloat16),
    (O.INT4, 128, 520, 256, torch.float32),
]


def _weight(m, n, wdt, seed):
    W, _ = synth.student_t_weight(m, n, seed, outlier_cols=3, outlier_scale=20.0,
                                  bf16=(wdt == torch.bfloat16))
    return W


def _check(W, fmt, G, res, r, c, sT, tr, tiles=None):
    nb = W.shape[1] // G
    tiles = list(range(nb)) if tiles is None else tiles
    cols = np.concatenate([np.arange(b * G, (b + 1) * G) for b in tiles])
    Wt = np.ascontiguousarray(W[:, cols])
    r_g, r_o = r[:, tiles], res["r"][:, tiles]
    c_g, c_o = c[cols], res["c"][cols]
    e_g = O.error(Wt, fmt, G, r_g, c_g)
    e_o = O.error(Wt, fmt, G, r_o, c_o)
    assert abs(e_g - e_o) <= 1e-4 * e_o, (e_g, e_o)
    same = float(np.mean(O.codes(Wt, fmt, G, r_g, c_g) == O.codes(Wt, fmt, G, r_o, c_o)))
    assert same >= 0.999, same
    assert sT == res["s_T"]
    # the scale decisions are the exact ones (see test_gpu_solver)
    assert np.array_equal(r_g, r_o) and np.array_equal(c_g, c_o)
    if len(tiles) == nb:
        np.testing.assert_allclose(tr, res["trace"], rtol=1e-4, atol=0)


@pytest.mark.parametrize("fmt,G,m,n,wdt", CASES)
def test_alpha_only_parity(fmt, G, m, n, wdt):
    W = _weight(m, n, wdt, 50)
    T = 8
    r, c, sT, tr = gpu_solve_ex(W, fmt, G, T, flags=O.ALPHA_ONLY, wdtype=wdt)
    assert np.all(c == 1.0)
    res = O.solve_ex(W, fmt, G, T, flags=O.ALPHA_ONLY)
    _check(W, fmt, G, res, r, c, sT, tr)
    assert np.all(np.diff(tr) <= tr[:-1] * 1e-6)


@pytest.mark.parametrize("fmt,G,m,n,wdt", CASES)
def test_beta_only_parity(fmt, G, m, n, wdt):
    W = _weight(m, n, wdt, 51)
    T = 8
    r, c, sT, tr = gpu_solve_ex(W, fmt, G, T, flags=O.BETA_ONLY, wdtype=wdt)
    r_init = gpu_solve(W, fmt, G, 0, wdt, trace=False)[0]
    assert np.array_equal(r, r_init)
    res = O.solve_ex(W, fmt, G, T, flags=O.BETA_ONLY)
    _check(W, fmt, G, res, r, c, sT, tr)
    assert np.all(np.diff(tr) <= tr[:-1] * 1e-6)


@pytest.mark.parametrize("fmt,G,m,n,wdt", CASES)
def test_warm_start_projection_exact_and_parity(fmt, G, m, n, wdt):
    """Given r0 / c0 are projected exactly as the oracle projects them (same
    fp32 decisions); the solve from there matches the oracle's."""
    W = _weight(m, n, wdt, 52)
    g = np.random.default_rng(53)
    c0 = np.exp(g.uniform(-2, 2, n)).astype(np.float32)
    r0 = (np.abs(W).reshape(m, n // G, G).max(axis=2) * g.uniform(0.05, 0.5, (m, n // G)))
    r0 = np.maximum(r0, 1e-6).astype(np.float32)
    r, c, sT, tr = gpu_solve_ex(W, fmt, G, 0, r0=r0, c0=c0, wdtype=wdt)
    res0 = O.solve_ex(W, fmt, G, 0, r0=r0, c0=c0)
    assert np.array_equal(c, res0["c"]) and np.array_equal(r, res0["r"]) and sT == res0["s_T"]
    T = 6
    r, c, sT, tr = gpu_solve_ex(W, fmt, G, T, r0=r0, c0=c0, wdtype=wdt)
    _check(W, fmt, G, O.solve_ex(W, fmt, G, T, r0=r0, c0=c0), r, c, sT, tr)


@pytest.mark.parametrize("fmt,G,m,n,wdt", CASES)
@pytest.mark.parametrize("flags", [0, O.ALPHA_ONLY, O.BETA_ONLY])
def test_resume_in_place_continues_exactly(fmt, G, m, n, wdt, flags):
    """T1 rounds, then T2 rounds resumed in place (r0 = r, c0 = c, kept
    tensor scale) give the scales of T1 + T2 rounds bit for bit (every
    reduction on the device has a fixed order)."""
    W = _weight(m, n, wdt, 54)
    r9, c9, s9, tr9 = gpu_solve_ex(W, fmt, G, 9, flags=flags, wdtype=wdt)
    r4, c4, s4, _ = gpu_solve_ex(W, fmt, G, 4, flags=flags, wdtype=wdt)
    r, c, sT, tr = gpu_solve_ex(W, fmt, G, 5, flags=flags | O.KEEP_S, r0=r4, c0=c4, s_T=s4,
                                wdtype=wdt)
    assert np.array_equal(r, r9) and np.array_equal(c, c9) and sT == s9
    np.testing.assert_allclose(tr, tr9[4:], rtol=1e-9)


@pytest.mark.parametrize("flags", [O.ALPHA_ONLY, O.BETA_ONLY])
def test_ablation_full_size_sampled_tiles(flags):
    """A 4096 x 4096 attention projection (NVFP4, T = 15), sampled tiles."""
    W, _ = synth.weight("llama8b_attn_nvfp4", 0)
    G, T = 16, synth.WORKLOADS["llama8b_attn_nvfp4"]["T"]
    r, c, sT, tr = gpu_solve_ex(W, O.NVFP4, G, T, flags=flags)
    nb = W.shape[1] // G
    tiles = [0, nb // 2, nb - 1]
    res = O.solve_ex(W, O.NVFP4, G, T, flags=flags, tiles=tiles)
    _check(W, O.NVFP4, G, res, r, c, sT, tr, tiles=tiles)
    assert np.all(np.isfinite(tr)) and tr[-1] <= tr[0]
