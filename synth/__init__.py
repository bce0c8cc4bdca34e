"""Seeded synthetic inputs shared by the CUDA path's tests/bench and the oracle.

This module holds none of the method's arithmetic: it only draws random
tensors (numpy PCG64 streams with fixed seeds) in the shapes and value
distributions of the Llama-shaped linear-layer workloads, with a few fixed
activation channels scaled up to act as outliers.  Both sides receive the same
arrays.

Recipe (every stream is seeded):
  * X  ~ N(0, 1), drawn in fp32, rounded to fp16 (seed 0);
  * outlier channels = the first K_out entries of a permutation of [0, K)
    (seed 2), sorted ascending; nested for increasing K_out;
  * each outlier channel is multiplied by a fixed factor drawn uniformly from
    [20, 60] (seed 3), or by one fixed factor (x40 in the tiny case, x50 in the
    70B case) when a workload names one;
  * W  ~ N(0, 0.02), drawn in fp32, rounded to fp16 (seed 1).
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

SEED_X, SEED_W, SEED_PERM, SEED_SCALE = 0, 1, 2, 3
THRESHOLD = 6.0
TINY_CHANNELS = (3, 77, 130, 201)


def activations(M: int, K: int, channels=(), factors=None, seed: int = SEED_X) -> np.ndarray:
    """fp16 [M, K] ~ N(0,1); columns in `channels` multiplied by `factors`."""
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((M, K), dtype=np.float32)
    channels = np.asarray(channels, dtype=np.int64)
    if channels.size:
        f = np.broadcast_to(np.asarray(factors, dtype=np.float32), channels.shape)
        x[:, channels] *= f
    return x.astype(np.float16)


def weights(N: int, K: int, seed: int = SEED_W, std: float = 0.02) -> np.ndarray:
    """fp16 [N, K] ~ N(0, std)."""
    rng = np.random.default_rng(seed)
    w = rng.standard_normal((N, K), dtype=np.float32) * np.float32(std)
    return w.astype(np.float16)


def gains(K: int, seed: int = 11, std: float = 0.1) -> np.ndarray:
    """fp16 [K] ~ N(1, std): the gain of an RMS normalisation before the layer."""
    rng = np.random.default_rng(seed)
    return (1.0 + rng.standard_normal(K, dtype=np.float32) * np.float32(std)).astype(np.float16)


def outlier_channels(K: int, count: int, seed: int = SEED_PERM) -> np.ndarray:
    """Sorted int32 channel list: first `count` of a seeded permutation of [0, K)."""
    perm = np.random.default_rng(seed).permutation(K)
    return np.sort(perm[:count]).astype(np.int32)


def channel_factors(count: int, seed: int = SEED_SCALE, lo: float = 20.0, hi: float = 60.0):
    """Per-channel outlier factors ~ U[lo, hi] (fp32)."""
    return np.random.default_rng(seed).uniform(lo, hi, size=count).astype(np.float32)


@dataclass(frozen=True)
class Case:
    """One linear-layer problem: Y[M,N] = layer(X[M,K], W[N,K])."""
    name: str
    M: int
    K: int
    N: int
    k_out: int            # size of the prepacked outlier channel set
    scaled: bool = True   # whether the outlier channels of X are scaled up
    factor: float | None = None  # one fixed factor instead of U[20,60]
    mode: str = "w8"      # "w8" (W8A8) or "w4" (W4A8, group 128)
    threshold: float = THRESHOLD
    tags: tuple = field(default_factory=tuple)

    @property
    def ops_int8(self) -> int:
        return 2 * self.M * self.N * self.K

    def channels(self) -> np.ndarray:
        if self.name.startswith("tiny"):
            return np.asarray(TINY_CHANNELS[: self.k_out], dtype=np.int32)
        return outlier_channels(self.K, self.k_out)

    def make(self):
        """Return (X fp16 [M,K], W fp16 [N,K], idx int32 [k_out])."""
        idx = self.channels()
        if self.scaled and self.k_out:
            f = self.factor if self.factor is not None else channel_factors(self.k_out)
            X = activations(self.M, self.K, idx, f)
        else:
            X = activations(self.M, self.K)
        W = weights(self.N, self.K)
        return X, W, idx


def tiny() -> list[Case]:
    """Tiny W8A8 + fp16-outlier layer: M=16, K=N=256, channels {3,77,130,201} x40."""
    return [Case("tiny", 16, 256, 256, 4, factor=40.0)]


def decode(mode: str = "w8") -> list[Case]:
    """Llama-7B decode shapes: M in {1,8,16,64} x (K,N) in {(4096,4096),(4096,11008),(11008,4096)},
    64 fixed outlier channels scaled x U[20,60]."""
    out = []
    for K, N in ((4096, 4096), (4096, 11008), (11008, 4096)):
        for M in (1, 8, 16, 64):
            out.append(Case(f"decode-{mode}-M{M}-K{K}-N{N}", M, K, N, 64, mode=mode))
    return out


def prefill(mode: str = "w8", k_outs=(0, 32, 128, 256)) -> list[Case]:
    """Llama-7B prefill shapes: M in {512,2048,8192}, K=4096, N in {4096,11008},
    outlier count sweep (nested fixed channel sets)."""
    out = []
    for M in (512, 2048, 8192):
        for N in (4096, 11008):
            for ko in k_outs:
                out.append(Case(f"prefill-{mode}-M{M}-N{N}-ko{ko}", M, 4096, N, ko, mode=mode))
    return out


def llama70b(mode: str = "w8") -> list[Case]:
    """Llama-70B shapes at batch 512: (K,N) in {(8192,8192),(8192,28672),(28672,8192)};
    128 outlier channels, unscaled (amax-below-threshold fast path) or scaled x50."""
    out = []
    for K, N in ((8192, 8192), (8192, 28672), (28672, 8192)):
        out.append(Case(f"70b-{mode}-K{K}-N{N}-fast", 512, K, N, 128, scaled=False, mode=mode))
        out.append(Case(f"70b-{mode}-K{K}-N{N}-x50", 512, K, N, 128, factor=50.0, mode=mode))
    return out
