"""Seeded synthetic inputs for the smoothed, outlier-split W4A4 linear layer.

These generators stand in for the OpenS2V-5M activations and the Wan2.2
FFN weights, which are not available here. Shapes follow the Wan2.2-14B
FFN (5120 <-> 13824); the value statistics follow the calibration figures
of "W4A4 Quantization for Inference on Wan2.2-I2V-A14B" (block_00.ffn.0:
activation column maxima above 6, weight column maxima below 0.6, a long
|x| tail beyond 1.5).

This module holds no arithmetic of the method itself: it only draws
random numbers (numpy PCG64, seeded) and converts them to BF16 with
torch's round-to-nearest-even cast. It is shared by the oracle-side tests
and the CUDA-side tests and benchmark so that both see identical inputs.
BF16 tensors are returned as numpy uint16 bit patterns.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np
import torch

WSCALE_1x32, WSCALE_TILE32x32, WSCALE_STRIP128x1 = 0, 1, 2


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 array -> BF16 bit patterns (uint16) via torch's RNE cast."""
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def bf16_bits_to_f32(h: np.ndarray) -> np.ndarray:
    return (np.asarray(h, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def _normal(rng: np.random.Generator, shape, sigma: float) -> np.ndarray:
    return rng.standard_normal(shape, dtype=np.float32) * np.float32(sigma)


def acts_gaussian_spiked(M: int, K: int, seed: int, sigma: float = 0.3,
                         n_spiked: int = 8, spike_max: float = 6.0) -> np.ndarray:
    """N(0, sigma) activations with n_spiked channels rescaled so that their
    column max |x| equals spike_max (the tiny oracle-check layer)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    ch = np.sort(rng.choice(K, size=min(n_spiked, K), replace=False))
    x = _normal(rng, (M, K), sigma)
    for j in ch:
        m = np.abs(x[:, j]).max()
        if m > 0:
            x[:, j] *= np.float32(spike_max / m)
    return to_bf16_bits(x)


def acts_heavy_tailed(M: int, K: int, seed: int, sigma: float = 0.3, frac: float = 0.01,
                      nu: float = 2.0, col_max: float = 6.0) -> np.ndarray:
    """Wan-like FFN input: N(0, sigma) bulk; a fraction `frac` of channels
    drawn from Student-t(nu) and rescaled to column max |x| = col_max, which
    leaves a tail well beyond |x| > 1.5."""
    rng = np.random.Generator(np.random.PCG64(seed))
    n_out = max(1, int(round(frac * K)))
    ch = np.sort(rng.choice(K, size=min(n_out, K), replace=False))
    x = _normal(rng, (M, K), sigma)
    t = rng.standard_t(nu, size=(M, ch.shape[0])).astype(np.float32)
    m = np.abs(t).max(axis=0)
    m[m == 0] = 1.0
    x[:, ch] = t * (np.float32(col_max) / m)[None, :]
    return to_bf16_bits(x)


def acts_gelu_boosted(M: int, K: int, seed: int, frac: float = 0.005, col_max: float = 8.0) -> np.ndarray:
    """FFN down-projection input: GELU(tanh form) of N(0, 1) pre-activations,
    with a fraction `frac` of channels scaled so their column max is col_max."""
    rng = np.random.Generator(np.random.PCG64(seed))
    n_out = max(1, int(round(frac * K)))
    ch = np.sort(rng.choice(K, size=min(n_out, K), replace=False))
    z = torch.from_numpy(rng.standard_normal((M, K), dtype=np.float32))
    x = torch.nn.functional.gelu(z, approximate="tanh").numpy()
    for j in ch:
        m = np.abs(x[:, j]).max()
        if m > 0:
            x[:, j] *= np.float32(col_max / m)
    return to_bf16_bits(x)


def weights_gaussian(K: int, N: int, seed: int, sigma: float, clip: float = 0.59) -> np.ndarray:
    """W [K][N] ~ N(0, sigma), clipped so that |w| stays below 0.6 after BF16."""
    rng = np.random.Generator(np.random.PCG64(seed))
    w = _normal(rng, (K, N), sigma)
    np.clip(w, -clip, clip, out=w)
    return to_bf16_bits(w)


@dataclass(frozen=True)
class LayerConfig:
    """One linear layer workload: X [M][K] -> Y [M][N]."""
    name: str
    M: int
    K: int
    N: int
    alpha: float
    k: int
    wmode: int
    out_bf16: bool
    x_kind: str          # "spiked" | "heavy" | "gelu"
    x_seed: int
    w_sigma: float
    w_seed: int

    def make_x(self, M: int | None = None) -> np.ndarray:
        M = self.M if M is None else M
        if self.x_kind == "spiked":
            return acts_gaussian_spiked(M, self.K, self.x_seed)
        if self.x_kind == "heavy":
            return acts_heavy_tailed(M, self.K, self.x_seed)
        if self.x_kind == "gelu":
            return acts_gelu_boosted(M, self.K, self.x_seed)
        raise ValueError(self.x_kind)

    def make_w(self) -> np.ndarray:
        return weights_gaussian(self.K, self.N, self.w_seed, self.w_sigma)

    @property
    def flops(self) -> float:
        """Effective FLOPs of the layer: 2*M*N*K over the full input width."""
        return 2.0 * self.M * self.N * self.K


# The five workloads. Seeds: tiny layer 0/1; layer c uses 1000c / 1000c+1.
TINY = LayerConfig("tiny_256x512x1024", 256, 512, 1024, 0.5, 16, WSCALE_1x32, False,
                   "spiked", 0, 0.05, 1)
UP = LayerConfig("wan_ffn_up_4096x5120x13824", 4096, 5120, 13824, 0.6, 128, WSCALE_STRIP128x1, False,
                 "heavy", 2000, 0.02, 2001)
DOWN = LayerConfig("wan_ffn_down_32760x13824x5120", 32760, 13824, 5120, 0.5, 256, WSCALE_TILE32x32, False,
                   "gelu", 3000, 0.01, 3001)
LONG = LayerConfig("wan_ffn_up_long_75600x5120x13824", 75600, 5120, 13824, 0.7, 64, WSCALE_1x32, True,
                   "heavy", 4000, 0.02, 4001)

CONFIGS = {c.name: c for c in (TINY, UP, DOWN, LONG)}


@dataclass(frozen=True)
class FFNConfig:
    """Four FFN blocks: up 5120->13824, GELU(tanh), down 13824->5120."""
    name: str = "wan_ffn_block_x4_32760x5120x13824"
    layers: int = 4
    M: int = 32760
    d_model: int = 5120
    d_ff: int = 13824
    calib_tokens: int = 2048
    k_up: int = 128
    k_down: int = 128
    alpha_up: float = 0.6
    alpha_down: float = 0.5
    wmode_up: int = WSCALE_STRIP128x1
    wmode_down: int = WSCALE_TILE32x32

    def seeds(self, layer: int):
        b = 5000 + 10 * layer
        return dict(x=b, w_up=b + 1, w_down=b + 2, calib=b + 3)

    def make_x(self, layer: int, M: int | None = None) -> np.ndarray:
        return acts_heavy_tailed(self.M if M is None else M, self.d_model, self.seeds(layer)["x"])

    def make_calib(self, layer: int) -> np.ndarray:
        return acts_heavy_tailed(self.calib_tokens, self.d_model, self.seeds(layer)["calib"])

    def make_w_up(self, layer: int) -> np.ndarray:
        return weights_gaussian(self.d_model, self.d_ff, self.seeds(layer)["w_up"], 0.02)

    def make_w_down(self, layer: int) -> np.ndarray:
        return weights_gaussian(self.d_ff, self.d_model, self.seeds(layer)["w_down"], 0.01)

    @property
    def flops(self) -> float:
        return self.layers * 2.0 * 2.0 * self.M * self.d_model * self.d_ff


FFN = FFNConfig()


def sample_rows(M: int, n: int, seed: int = 7, tile: int = 128) -> np.ndarray:
    """A sorted, stratified sample of n row indices of [0, M) that always
    includes the first row, the last row, and the first and last rows of
    the final (possibly ragged) 128-row tile."""
    rng = np.random.Generator(np.random.PCG64(seed))
    must = {0, M - 1, (M - 1) // tile * tile, min(M - 1, (M - 1) // tile * tile + 1)}
    if n >= M:
        return np.arange(M, dtype=np.int64)
    strata = np.linspace(0, M, num=max(1, n - len(must)) + 1).astype(np.int64)
    picks = [int(rng.integers(lo, max(lo + 1, hi))) for lo, hi in zip(strata[:-1], strata[1:])]
    return np.array(sorted(set(picks) | must), dtype=np.int64)
