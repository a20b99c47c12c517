"""Seeded synthetic inputs shared by the tests, the smoke check and the bench.

This module holds no arithmetic of the quantized-projection method: it only
draws numbers.  Both sides (the CPU oracle's tests and the CUDA path) take
their inputs from here, so a seed names the same tensor everywhere.

Generator: SplitMix64 (Steele, Lea & Flood, "Fast splittable pseudorandom
number generators", OOPSLA 2014) -- output i (1-based) of a stream seeded
with s is mix(s + i * 0x9E3779B97F4A7C15) -- feeding the basic Box-Muller
transform in double:
    u1 = ((a >> 11) + 1) * 2^-53  in (0, 1],   u2 = (b >> 11) * 2^-53,
    z0 = sqrt(-2 ln u1) cos(2 pi u2),  z1 = sqrt(-2 ln u1) sin(2 pi u2),
emitted as z0, z1 of pair 0, then pair 1, ...; values are scaled by sigma in
double and rounded once to fp32.  Torch's RNG is not used: its streams are
not stable across versions.

Workload recipe (the pages measure on real GGUF projections; these stand in
for them with the same shapes): weights sigma = 0.02, activations sigma = 1.
"""
from __future__ import annotations

import numpy as np

_GAMMA = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)

WEIGHT_SIGMA = 0.02
ACT_SIGMA = 1.0


def splitmix64(seed: int, n: int, offset: int = 0) -> np.ndarray:
    """Outputs offset+1 .. offset+n of the SplitMix64 stream seeded with `seed`."""
    with np.errstate(over="ignore"):
        i = np.arange(offset + 1, offset + n + 1, dtype=np.uint64)
        z = np.uint64(seed & 0xFFFFFFFFFFFFFFFF) + i * _GAMMA
        z = (z ^ (z >> np.uint64(30))) * _M1
        z = (z ^ (z >> np.uint64(27))) * _M2
        return z ^ (z >> np.uint64(31))


def normal(seed: int, n: int, sigma: float = 1.0) -> np.ndarray:
    """n draws of sigma * N(0, 1) as fp32 (Box-Muller over SplitMix64)."""
    pairs = (n + 1) // 2
    r = splitmix64(seed, 2 * pairs).reshape(pairs, 2)
    u1 = ((r[:, 0] >> np.uint64(11)).astype(np.float64) + 1.0) * 2.0 ** -53
    u2 = (r[:, 1] >> np.uint64(11)).astype(np.float64) * 2.0 ** -53
    rad = np.sqrt(-2.0 * np.log(u1))
    z = np.empty((pairs, 2), np.float64)
    z[:, 0] = rad * np.cos(2.0 * np.pi * u2)
    z[:, 1] = rad * np.sin(2.0 * np.pi * u2)
    return (sigma * z.reshape(-1)[:n]).astype(np.float32)


def weights(seed: int, N: int, K: int) -> np.ndarray:
    """fp32 weight matrix [N, K] drawn i.i.d. N(0, 0.02^2)."""
    return normal(seed, N * K, WEIGHT_SIGMA).reshape(N, K)


def activations(seed: int, M: int, K: int) -> np.ndarray:
    """fp32 activations [M, K] drawn i.i.d. N(0, 1)."""
    return normal(seed, M * K, ACT_SIGMA).reshape(M, K)


# Seeds of the five workloads (weights seed 0 for the 1024 x 1024 GEMV is
# fixed by the workload statement; the others are this project's choice).
SEEDS = {
    "gemv_q8_0_1024": {"w": 0, "x": 100},
    "paired_q8_0_2x8192x4096": {"w0": 1, "w1": 2, "x_base": 1000},
    "gemv_q4_k_4096": {"w": 3, "x": 101},
    "grouped_q8_0_8x1024x4096": {"w_base": 40, "x_base": 140},
    "prefill": {"w_q4_k": 5, "w_q8_0": 6, "x_base": 200},
}
