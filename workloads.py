"""Seeded synthetic inputs and the layer shapes they are drawn for.

This module holds no ConvRot arithmetic: it only draws random numbers, rounds
them to bf16 storage, and builds the two kinds of rotation block that are passed
to the layer as an input (a normalized Sylvester-Hadamard matrix and a random
orthogonal matrix from the QR factorisation of a Gaussian matrix).  Both the CPU
oracle and the CUDA path receive exactly the arrays produced here.

The pages measure real diffusion-transformer checkpoints (Z-Image, FLUX.1,
Wan 2.2); none is available, so the value distributions below stand in for
them:

* activations x ~ N(0, 1) with a few outlier input channels scaled by 30
  (the outlier structure that, per the Invoke "int8 Compute" page, "Layers that
  keep unpacking", makes un-rotated per-token quantization lose the most);
* weights W ~ N(0, 0.02) with 1 % of the input columns scaled by 10;
* bias ~ N(0, 0.01).
"""

from __future__ import annotations

import dataclasses

import numpy as np
import torch

GROUP_SIZES = (4, 16, 64, 256)


@dataclasses.dataclass(frozen=True)
class Linear:
    """One ConvRot linear: y[M, N] = x[M, K] @ W[N, K]^T + b[N]."""

    name: str
    M: int
    K: int
    N: int
    G: int = 256
    n_outliers: int = 4


# The layer shapes of the synthetic workloads.  Token counts follow the models'
# latent sizes: Z-Image / FLUX.1 at 1024^2 -> 4096 image + 512 text tokens;
# Wan 2.2 at 832x480x17 frames -> latent 104x60x5 with 2x2 patches = 7800.
WORKLOADS: dict[str, list[Linear]] = {
    "single_1024": [Linear("linear", 64, 1024, 1024)],
    "zimage_dit_block": [
        Linear("qkv", 4608, 3840, 11520),
        Linear("ffn_up", 4608, 3840, 10240),
        Linear("ffn_down", 4608, 10240, 3840),
    ],
    "flux1_dev_blocks": [
        Linear("double_qkv", 4608, 3072, 9216, n_outliers=8),
        Linear("double_mlp_up", 4608, 3072, 12288, n_outliers=8),
        Linear("double_mlp_down", 4608, 12288, 3072, n_outliers=8),
        Linear("single_in_proj", 4608, 3072, 21504, n_outliers=8),
        Linear("single_out_proj", 4608, 15360, 3072, n_outliers=8),
    ],
    "wan22_a14b_video_dit": [
        Linear("qkv", 7800, 5120, 15360),
        Linear("ffn_up", 7800, 5120, 13824),
        Linear("ffn_down", 7800, 13824, 5120),
    ],
    "group_size_sweep": [
        Linear(f"k4096_m{m}_g{g}", m, 4096, 4096, G=g)
        for g in GROUP_SIZES
        for m in (1, 16, 128, 1024, 8192)
    ],
}

# Standalone weight decode of the group-size sweep: a [12288, 3072] int8 weight.
DEROTATE_SWEEP_SHAPE = (12288, 3072)

# Seed bases; the workload index is added so that every workload draws its own.
SEED_X, SEED_X_OUTLIERS, SEED_W, SEED_W_OUTLIERS, SEED_BIAS, SEED_QR = (
    1000, 2000, 3000, 4000, 5000, 6000)


def to_bf16(a: np.ndarray, dtype: torch.dtype = torch.bfloat16) -> torch.Tensor:
    """fp32 numpy array -> bf16 (or `dtype`, e.g. fp16) CPU tensor (round to nearest even)."""
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(dtype)


def make_activation(M: int, K: int, seed: int, n_outliers: int = 4,
                    outlier_seed: int | None = None, scale: float = 30.0,
                    dtype: torch.dtype = torch.bfloat16) -> torch.Tensor:
    """x ~ N(0,1) [M, K] with `n_outliers` input channels multiplied by `scale`."""
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((M, K), dtype=np.float32)
    if n_outliers:
        orng = np.random.default_rng(seed + 1 if outlier_seed is None else outlier_seed)
        cols = orng.choice(K, size=min(n_outliers, K), replace=False)
        x[:, cols] *= scale
    return to_bf16(x, dtype)


def make_weight(N: int, K: int, seed: int, outlier_frac: float = 0.01,
                outlier_seed: int | None = None, std: float = 0.02,
                scale: float = 10.0, dtype: torch.dtype = torch.bfloat16) -> torch.Tensor:
    """W ~ N(0, std) [N, K] with a fraction of its input columns multiplied by `scale`."""
    rng = np.random.default_rng(seed)
    w = rng.standard_normal((N, K), dtype=np.float32) * np.float32(std)
    n_cols = int(round(outlier_frac * K))
    if n_cols:
        orng = np.random.default_rng(seed + 1 if outlier_seed is None else outlier_seed)
        cols = orng.choice(K, size=n_cols, replace=False)
        w[:, cols] *= np.float32(scale)
    return to_bf16(w, dtype)


def make_bias(N: int, seed: int, std: float = 0.01, dtype: torch.dtype = torch.bfloat16) -> torch.Tensor:
    rng = np.random.default_rng(seed)
    return to_bf16(rng.standard_normal(N, dtype=np.float32) * np.float32(std), dtype)


def sylvester_rotation(G: int) -> np.ndarray:
    """Normalized Sylvester-Hadamard matrix H_G / sqrt(G), float32 [G, G].

    H_1 = [1], H_2n = [[H_n, H_n], [H_n, -H_n]].  For G a power of 4 every entry
    is +-2^(-log2(G)/2), exact in float32.
    """
    if G < 1 or G & (G - 1):
        raise ValueError("G must be a power of two")
    h = np.ones((1, 1), dtype=np.float64)
    while h.shape[0] < G:
        h = np.block([[h, h], [h, -h]])
    return (h / np.sqrt(G)).astype(np.float32)


def qr_rotation(G: int, seed: int = SEED_QR) -> np.ndarray:
    """Random orthogonal float32 [G, G]: Q of the QR of a Gaussian matrix, columns
    sign-fixed so that diag(R_qr) > 0 (the Haar-distributed choice)."""
    rng = np.random.default_rng(seed)
    q, r = np.linalg.qr(rng.standard_normal((G, G)))
    q = q * np.sign(np.diag(r))[None, :]
    return q.astype(np.float32)


@dataclasses.dataclass
class LayerInputs:
    x: torch.Tensor        # bf16 or fp16 [M, K]
    W: torch.Tensor        # bf16 or fp16 [N, K]
    bias: torch.Tensor     # bf16 or fp16 [N]
    R: np.ndarray          # float32 [G, G]


def make_layer_inputs(lin: Linear, index: int = 0, rotation: str = "sylvester",
                      M: int | None = None, dtype: torch.dtype = torch.bfloat16) -> LayerInputs:
    """All inputs of one linear, drawn from the seeds of workload `index`, as
    bf16 (or `dtype`, e.g. fp16) tensors."""
    m = lin.M if M is None else M
    x = make_activation(m, lin.K, SEED_X + index, lin.n_outliers, SEED_X_OUTLIERS + index,
                        dtype=dtype)
    W = make_weight(lin.N, lin.K, SEED_W + index, outlier_seed=SEED_W_OUTLIERS + index,
                    dtype=dtype)
    b = make_bias(lin.N, SEED_BIAS + index, dtype=dtype)
    if rotation == "sylvester":
        R = sylvester_rotation(lin.G)
    elif rotation == "qr":
        R = qr_rotation(lin.G)
    else:
        raise ValueError(rotation)
    return LayerInputs(x, W, b, R)
