"""Seeded synthetic inputs for the quantized linear layer.

The pages measure on trained video diffusion transformers and benchmark
suites that are not available here; these generators stand in for them with
the shapes and value distributions of the layers those pages quantize
(CogVideoX-2B/5B- and Wan-14B-shaped linears, outlier channels in
activations or weights).  Values are drawn in fp32 from numpy's PCG64
(``default_rng``) and rounded to bf16 by torch's round-to-nearest-even
conversion, so the CUDA path and the CPU oracle receive identical bf16 bytes.

This module holds no arithmetic of the quantization method and imports
nothing else from this package.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np
import torch

# Token counts of the video workloads: CogVideoX 13x30x45 latent patches plus
# 226 text tokens; Wan 21x30x52 latent patches.
M_COGVIDEOX = 13 * 30 * 45 + 226      # 17776
M_WAN = 21 * 30 * 52                  # 32760


def _rng(seed: int, *stream: int) -> np.random.Generator:
    return np.random.default_rng([seed, *stream])


def to_bf16(x32: np.ndarray) -> torch.Tensor:
    """fp32 numpy array -> bf16 torch tensor (CPU), RN-even."""
    return torch.from_numpy(np.ascontiguousarray(x32, dtype=np.float32)).to(torch.bfloat16)


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """The uint16 bit patterns of a bf16 tensor (shared memory, no copy)."""
    assert t.dtype == torch.bfloat16
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def normal(shape, std: float, seed: int, *stream: int) -> np.ndarray:
    return _rng(seed, *stream).standard_normal(size=shape, dtype=np.float32) * np.float32(std)


def activations_with_outlier_channels(m: int, k: int, frac: float, scale: float,
                                      seed: int, stream: int) -> torch.Tensor:
    """X ~ N(0,1) [m, k] with floor(frac*k) channels (drawn without
    replacement from the same stream) multiplied by ``scale``."""
    rng = _rng(seed, stream)
    x = rng.standard_normal(size=(m, k), dtype=np.float32)
    n_out = int(np.floor(frac * k))
    cols = rng.choice(k, size=n_out, replace=False)
    x[:, cols] *= np.float32(scale)
    return to_bf16(x)


def activations_fixed_outliers(m: int, k: int, n_out: int, scale: float,
                               seed: int, stream: int) -> torch.Tensor:
    rng = _rng(seed, stream)
    x = rng.standard_normal(size=(m, k), dtype=np.float32)
    cols = rng.choice(k, size=n_out, replace=False)
    x[:, cols] *= np.float32(scale)
    return to_bf16(x)


def activations_student_t_channels(m: int, k: int, frac: float, dof: float,
                                   seed: int, stream: int) -> torch.Tensor:
    """X ~ N(0,1) with floor(frac*k) channels drawn from Student-t(dof)."""
    rng = _rng(seed, stream)
    x = rng.standard_normal(size=(m, k), dtype=np.float32)
    n_out = int(np.floor(frac * k))
    cols = rng.choice(k, size=n_out, replace=False)
    x[:, cols] = rng.standard_t(dof, size=(m, n_out)).astype(np.float32)
    return to_bf16(x)


def weights(n: int, k: int, std: float, seed: int, stream: int,
            outlier_frac: float = 0.0, outlier_scale: float = 1.0) -> torch.Tensor:
    """W ~ N(0, std) [n, k] (nn.Linear layout); optionally floor(frac*k)
    input channels (columns) multiplied by ``outlier_scale``."""
    rng = _rng(seed, stream)
    w = rng.standard_normal(size=(n, k), dtype=np.float32) * np.float32(std)
    if outlier_frac > 0:
        n_out = int(np.floor(outlier_frac * k))
        cols = rng.choice(k, size=n_out, replace=False)
        w[:, cols] *= np.float32(outlier_scale)
    return to_bf16(w)


@dataclass
class Linear:
    name: str
    n: int
    k: int


# --- workload definitions ---------------------------------------------------

def single_linear(seed: int = 0):
    """Small case: X [256,1920] with 8 channels x50, W [1920,1920] N(0,0.02)."""
    x = activations_fixed_outliers(256, 1920, 8, 50.0, seed, 1)
    w = weights(1920, 1920, 0.02, seed, 2)
    return x, w


COGVIDEOX_2B = [Linear("qkv", 5760, 1920), Linear("out", 1920, 1920),
                Linear("ffn_up", 7680, 1920), Linear("ffn_down", 1920, 7680)]
COGVIDEOX_5B = [Linear("qkv", 9216, 3072), Linear("ffn_up", 12288, 3072),
                Linear("ffn_down", 3072, 12288)]
WAN_14B = [Linear("qkv", 15360, 5120), Linear("ffn_up", 13824, 5120),
           Linear("ffn_down", 5120, 13824)]


def cogvideox2b_linear(lin: Linear, m: int = M_COGVIDEOX, seed: int = 1):
    """Activations N(0,1) with 1% channels x30; weights N(0,0.02)."""
    idx = [l.name for l in COGVIDEOX_2B].index(lin.name)
    x = activations_with_outlier_channels(m, lin.k, 0.01, 30.0, seed, 10 + idx)
    w = weights(lin.n, lin.k, 0.02, seed, 20 + idx)
    return x, w


def dmpq_block_pair(block: int, m: int = M_COGVIDEOX, k: int = 1920, seed: int = 2):
    """Routing sweep block: input N(0,1); output = input + N(0, sigma_b) with
    sigma_b = 10^U(-3, 0) (log-uniform in [1e-3, 1])."""
    rng = _rng(seed, 100 + block)
    sigma = float(10.0 ** rng.uniform(-3.0, 0.0))
    x = rng.standard_normal(size=(m, k), dtype=np.float32)
    y = x + rng.standard_normal(size=(m, k), dtype=np.float32) * np.float32(sigma)
    return to_bf16(x), to_bf16(y), sigma


def dmpq_ffn_up_weights(seed: int = 2):
    return weights(7680, 1920, 0.02, seed, 200)


def cogvideox5b_qarvd_linear(lin: Linear, m: int = M_COGVIDEOX, seed: int = 3):
    """Weights N(0,0.02) with 2% input channels x20; activations N(0,1)."""
    idx = [l.name for l in COGVIDEOX_5B].index(lin.name)
    w = weights(lin.n, lin.k, 0.02, seed, 30 + idx, outlier_frac=0.02, outlier_scale=20.0)
    x = to_bf16(normal((m, lin.k), 1.0, seed, 40 + idx))
    return x, w


def wan14b_linear(lin: Linear, m: int = M_WAN, seed: int = 4):
    """Activations N(0,1) with 0.5% Student-t(3) channels; weights N(0,0.015)."""
    idx = [l.name for l in WAN_14B].index(lin.name)
    x = activations_student_t_channels(m, lin.k, 0.005, 3.0, seed, 50 + idx)
    w = weights(lin.n, lin.k, 0.015, seed, 60 + idx)
    return x, w
