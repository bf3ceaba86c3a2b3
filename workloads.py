"""Seeded synthetic inputs and workload shapes for the BitLinear matmul.

This module is shared by the tests, the smoke check and the benchmark, and it
holds none of the method's arithmetic: it only draws random latents and
activations and names the shapes. Both the CUDA path and the CPU oracle get
their inputs from here.

Recipe (no trained weights or datasets are used):
  * latent weights W [N][K] fp32, i.i.d. N(0, 0.02^2) -- the BitLinear layers
    of the ~2B-parameter decoder are stood in for by Gaussian latents;
  * activations x [M][K], i.i.d. N(0, 1), with 1% of the K channels (a seeded
    choice, the same channels for every token) multiplied by 50 as outlier
    channels, then rounded to bf16 (the tiny case keeps fp32 and has no
    outliers);
  * RMS-normalisation gains g [K] (the normalising forms of the path) are
    drawn uniformly from [0.5, 1.5);
  * every draw uses numpy's PCG64 generator seeded per (workload, matrix).
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

W_STD = 0.02
OUTLIER_FRACTION = 0.01
OUTLIER_SCALE = 50.0

# Decoder shapes of the ~2B model: (name, K = d_in, N = d_out).
LAYER_PROJECTIONS = (
    ("q", 2560, 2560),
    ("k", 2560, 640),
    ("v", 2560, 640),
    ("o", 2560, 2560),
    ("gate", 2560, 6912),
    ("up", 2560, 6912),
    ("down", 6912, 2560),
)
NUM_LAYERS = 30


def rng(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed))


def latent_weights(N: int, K: int, seed: int, std: float = W_STD) -> np.ndarray:
    """fp32 [N][K] latent weight matrix drawn from N(0, std^2)."""
    return (rng(seed).standard_normal((N, K), dtype=np.float32)
            * np.float32(std)).astype(np.float32)


def outlier_channels(K: int, seed: int,
                     fraction: float = OUTLIER_FRACTION) -> np.ndarray:
    """Sorted indices of the outlier channels (at least one when K > 0)."""
    count = max(1, int(round(K * fraction))) if K > 0 else 0
    return np.sort(rng(seed ^ 0x5EED).choice(K, size=count, replace=False))


def activations_f32(M: int, K: int, seed: int, outliers: bool = True,
                    fraction: float = OUTLIER_FRACTION,
                    scale: float = OUTLIER_SCALE) -> np.ndarray:
    """fp32 [M][K] activations ~N(0,1); outlier channels scaled by ``scale``."""
    x = rng(seed).standard_normal((M, K), dtype=np.float32)
    if outliers and K > 0:
        x[:, outlier_channels(K, seed, fraction)] *= np.float32(scale)
    return x


def norm_gains(K: int, seed: int, low: float = 0.5, high: float = 1.5) -> np.ndarray:
    """fp32 [K] RMS-normalisation gains drawn uniformly from [low, high): a
    stand-in for learned per-channel gains, which start at one."""
    return rng(seed ^ 0x6A15).uniform(low, high, size=K).astype(np.float32)


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (ties to even) and return the uint16 bit patterns.

    This is how the synthetic bf16 inputs are made; it is the input
    generator's rounding, done with torch's own conversion."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16).copy()


def activations_bf16(M: int, K: int, seed: int, outliers: bool = True) -> np.ndarray:
    """bf16 bit patterns (uint16 [M][K]) of ``activations_f32``."""
    return to_bf16_bits(activations_f32(M, K, seed, outliers))


@dataclass(frozen=True)
class Problem:
    """One BitLinear matmul: M tokens, K = d_in, N = d_out."""
    name: str
    M: int
    K: int
    N: int
    w_seed: int
    x_seed: int
    x_dtype: str = "bf16"          # "bf16" or "fp32"
    outliers: bool = True

    def weights(self) -> np.ndarray:
        return latent_weights(self.N, self.K, self.w_seed)

    def x_f32(self) -> np.ndarray:
        return activations_f32(self.M, self.K, self.x_seed, self.outliers)

    def x_input(self) -> np.ndarray:
        """The input as handed to both sides: fp32 values, or bf16 bits."""
        x = self.x_f32()
        return x if self.x_dtype == "fp32" else to_bf16_bits(x)


@dataclass
class Workload:
    name: str
    problems: list = field(default_factory=list)


def tiny() -> Workload:
    """Latent W 256x256 ~N(0,0.02), x 4x256 fp32 ~N(0,1), seed 0."""
    return Workload("tiny_256x256_m4", [
        Problem("tiny", 4, 256, 256, w_seed=0, x_seed=0, x_dtype="fp32",
                outliers=False)])


def decode_gemv_2b(M: int = 1) -> Workload:
    """Decode at the 2B shape: up 2560->6912 and down 6912->2560."""
    return Workload(f"decode_gemv_2b_m{M}", [
        Problem("up", M, 2560, 6912, w_seed=1, x_seed=101),
        Problem("down", M, 6912, 2560, w_seed=2, x_seed=102)])


def layer_set_2b(B: int, layers: int = NUM_LAYERS) -> Workload:
    """The 7 projections of each decoder layer, independent seeds."""
    probs = []
    for layer in range(layers):
        for p, (name, K, N) in enumerate(LAYER_PROJECTIONS):
            s = 1000 + 16 * layer + p
            probs.append(Problem(f"L{layer}.{name}", B, K, N, w_seed=s,
                                 x_seed=s + 500000))
    return Workload(f"layer_set_2b_b{B}", probs)


def prefill_2b(M: int = 2048) -> Workload:
    return Workload(f"prefill_2b_m{M}", [
        Problem("up", M, 2560, 6912, w_seed=3, x_seed=103),
        Problem("down", M, 6912, 2560, w_seed=4, x_seed=104)])


def large_sweep(M: int) -> Workload:
    """~100B-class layer shapes: 8192->28672 and 28672->8192."""
    return Workload(f"large_m{M}", [
        Problem("up_large", M, 8192, 28672, w_seed=5, x_seed=105),
        Problem("down_large", M, 28672, 8192, w_seed=6, x_seed=106)])
