"""Seeded synthetic inputs shaped like the DualQuant workloads.

This module holds input generation only -- none of the quantisation
arithmetic -- and is the one piece shared by the tests, the CPU oracle legs
and the GPU path.  Every tensor is drawn on the host with NumPy's PCG64 and
rounded to bfloat16 (round-to-nearest-even) where the workload is bf16, so
that both sides see identical bits.

Stand-ins: the paper evaluates Llama / Qwen checkpoints ("DualQuant",
Section 5, "Models and formats"); those weights are not available here, so
weights are Student-t(nu=4) draws (heavy-tailed like LLM weights) and
activations are N(0, 1) with a few outlier channels scaled up (the
channel-wise activation outliers of Section 2.2).
"""
import numpy as np
import torch

FMT = {"int4": 0, "mxint4": 1, "mxfp4": 2, "nvfp4": 3}
NATIVE_GROUP = {"int4": 64, "mxint4": 32, "mxfp4": 32, "nvfp4": 16}


def to_bf16_values(x: np.ndarray) -> np.ndarray:
    """Round fp32 values to bfloat16 (RNE) and return them as fp32."""
    t = torch.from_numpy(np.ascontiguousarray(x, np.float32))
    return t.to(torch.bfloat16).to(torch.float32).numpy()


def rng(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed))


def student_t_weight(m, n, seed, std=0.02, unit_variance=True, outlier_cols=0,
                     outlier_scale=1.0, bf16=True):
    """W (m x n) ~ Student-t(4) * scale.

    unit_variance=True divides by sqrt(2) (t_4 has variance 2) so the entries
    have standard deviation `std`; False multiplies the raw draw by `std`.
    Returns (W as fp32 array, indices of the outlier columns).
    """
    g = rng(seed)
    W = g.standard_t(4.0, size=(m, n)).astype(np.float32)
    W *= np.float32(std / np.sqrt(2.0) if unit_variance else std)
    idx = np.sort(g.choice(n, size=outlier_cols, replace=False)) if outlier_cols else \
        np.zeros(0, np.int64)
    if outlier_cols:
        W[:, idx] *= np.float32(outlier_scale)
    if bf16:
        W = to_bf16_values(W)
    return np.ascontiguousarray(W), idx


def activations(M, K, seed, outlier_channels=None, n_outliers=0, outlier_scale=1.0, bf16=True):
    """X (M x K) ~ N(0, 1) with `outlier_channels` (or `n_outliers` seeded
    channels) multiplied by `outlier_scale`."""
    g = rng(seed)
    X = g.standard_normal(size=(M, K)).astype(np.float32)
    if outlier_channels is None:
        outlier_channels = np.sort(g.choice(K, size=n_outliers, replace=False)) if n_outliers \
            else np.zeros(0, np.int64)
    if len(outlier_channels):
        X[:, outlier_channels] *= np.float32(outlier_scale)
    if bf16:
        X = to_bf16_values(X)
    return np.ascontiguousarray(X), np.asarray(outlier_channels)


# ----------------------------------------------------------------------------
# The five workloads.  Each returns plain descriptions; tensors are drawn on
# demand by weight()/acts() so large shapes are only generated when used.
# ----------------------------------------------------------------------------
WORKLOADS = {
    "tiny_layer_256": {
        "weights": [(256, 256)], "fmt": ["nvfp4"], "T": 20, "M": [16],
        "w_std": 0.02, "w_unit_variance": False, "w_outlier_cols": 4, "w_outlier_scale": 20.0,
        "x_outliers": 2, "x_outlier_scale": 30.0, "bf16": False, "seed": 0,
    },
    "llama8b_attn_nvfp4": {
        "weights": [(4096, 4096), (1024, 4096)], "fmt": ["nvfp4"], "T": 50,
        "M": [1, 16, 256, 4096], "w_std": 0.02, "w_unit_variance": True,
        "x_outlier_frac": 0.01, "x_outlier_scale": 50.0, "bf16": True, "seed": 0,
    },
    "llama8b_mlp_mx": {
        "weights": [(14336, 4096), (4096, 14336)], "fmt": ["mxfp4", "mxint4"], "T": 50,
        "M": [2048], "w_std": 0.02, "w_unit_variance": True,
        "x_outlier_frac": 0.005, "x_outlier_scale": 50.0, "bf16": True, "seed": 0,
    },
    "llama8b_sweep_224": {
        "weights": [(4096, 4096), (1024, 4096), (1024, 4096), (4096, 4096),
                    (14336, 4096), (14336, 4096), (4096, 14336)] * 32,
        "fmt": ["int4", "mxint4", "mxfp4", "nvfp4"], "int4_group": 128, "T": 50, "M": [],
        "w_std": 0.02, "w_unit_variance": True, "bf16": True, "seed": 0,
    },
    "qwen32b_mlp_nvfp4": {
        "weights": [(27648, 5120), (5120, 27648)], "fmt": ["nvfp4"], "T": 50,
        "M": [1, 8, 64, 8192], "w_std": 0.02, "w_unit_variance": True,
        "x_outlier_frac": 0.01, "x_outlier_scale": 100.0, "bf16": True, "seed": 0,
    },
}


def weight(workload: str, index: int, shape=None):
    """Weight `index` of a workload (per-weight seed = base seed + index)."""
    w = WORKLOADS[workload]
    m, n = shape if shape is not None else w["weights"][index]
    return student_t_weight(m, n, w["seed"] + index, std=w["w_std"],
                            unit_variance=w["w_unit_variance"],
                            outlier_cols=w.get("w_outlier_cols", 0),
                            outlier_scale=w.get("w_outlier_scale", 1.0), bf16=w["bf16"])


def acts(workload: str, M: int, K: int, index: int = 0, outlier_channels=None):
    """Activations for a workload.  The tiny workload places its outlier
    channels on the first outlier columns of its weight (the paper's premise
    that weight and activation outliers share channels, Section 4.2); the
    other workloads draw theirs with the activation seed."""
    w = WORKLOADS[workload]
    n_out = w.get("x_outliers")
    if n_out is None:
        n_out = int(round(w.get("x_outlier_frac", 0.0) * K))
    if (outlier_channels is None and w.get("w_outlier_cols", 0) >= (n_out or 0) > 0
            and K == w["weights"][index][1]):
        outlier_channels = weight(workload, index)[1][:n_out]
    return activations(M, K, 1000 + w["seed"] + index, outlier_channels=outlier_channels,
                       n_outliers=n_out, outlier_scale=w.get("x_outlier_scale", 1.0),
                       bf16=w["bf16"])
