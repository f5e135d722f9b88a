"""Seeded synthetic inputs shared by the tests, the smoke check and the benchmark.

This module holds no arithmetic of the attention method: it only draws
spatially smooth pixel-token tensors and rounds them to bf16, so that the CUDA
path and the CPU oracle can be fed the very same numbers.

Recipe (stands in for the FFHQ / ImageNet pixel tokens the method is trained
on; the datasets themselves are not used):
  * every (batch, head, channel) of Q, K and V is an independent H x W field
    of N(0, 1) noise,
  * blurred by a separable Gaussian of width ``sigma`` pixels, truncated at
    4 sigma, reflecting at the border,
  * standardised to zero mean and unit variance,
  * plus ``noise`` * N(0, 1) white noise,
  * laid out in raster order as [batch, heads, H*W, d];
  * the upstream gradient dO is plain N(0, 1) drawn from its own seed.
"""
from __future__ import annotations

import numpy as np
from scipy.ndimage import gaussian_filter1d


def round_to_bf16(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bf16 (ties to even); returns float32."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000
    return u.astype(np.uint32).view(np.float32)


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """The upper 16 bits of float32 values that are already bf16-exact."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    return (x.view(np.uint32) >> 16).astype(np.uint16)


def smooth_fields(rng: np.random.Generator, count: int, H: int, W: int, sigma: float,
                  noise: float = 0.1) -> np.ndarray:
    """``count`` independent smooth H x W fields as float32 [count, H, W]."""
    out = np.empty((count, H, W), dtype=np.float32)
    chunk = max(1, (1 << 24) // (H * W))
    for s in range(0, count, chunk):
        e = min(count, s + chunk)
        f = rng.standard_normal((e - s, H, W), dtype=np.float32)
        if sigma > 0:
            f = gaussian_filter1d(f, sigma, axis=1, mode="reflect", truncate=4.0)
            f = gaussian_filter1d(f, sigma, axis=2, mode="reflect", truncate=4.0)
        mu = f.mean(axis=(1, 2), keepdims=True)
        sd = f.std(axis=(1, 2), keepdims=True)
        f = (f - mu) / np.maximum(sd, 1e-12)
        f = f + noise * rng.standard_normal((e - s, H, W), dtype=np.float32)
        out[s:e] = f
    return out


def pixel_tokens(seed: int, batch: int, heads: int, H: int, W: int, d: int, sigma: float,
                 noise: float = 0.1, bf16: bool = True) -> np.ndarray:
    """One [batch, heads, H*W, d] raster-order token tensor of smooth fields."""
    rng = np.random.default_rng(seed)
    f = smooth_fields(rng, batch * heads * d, H, W, sigma, noise)
    t = f.reshape(batch, heads, d, H * W).transpose(0, 1, 3, 2)
    t = np.ascontiguousarray(t)
    return round_to_bf16(t) if bf16 else t


def qkv(seed: int, batch: int, heads: int, H: int, W: int, d: int, sigma: float,
        noise: float = 0.1, bf16: bool = True):
    """Q, K, V in raster order, each from its own stream of ``seed``."""
    ss = np.random.SeedSequence(seed)
    seeds = [int(s.generate_state(1)[0]) for s in ss.spawn(3)]
    return tuple(pixel_tokens(s, batch, heads, H, W, d, sigma, noise, bf16) for s in seeds)


def upstream_grad(seed: int, batch: int, heads: int, N: int, d: int, bf16: bool = True) -> np.ndarray:
    """dO ~ N(0, 1), [batch, heads, N, d]."""
    rng = np.random.default_rng(seed)
    g = rng.standard_normal((batch, heads, N, d), dtype=np.float32)
    return round_to_bf16(g) if bf16 else g


# The five workloads the method is measured on, as (name, settings).
CONFIGS = {
    "tiny32": dict(batch=1, heads=1, H=32, W=32, d=64, B=16, L=2, K=4, dtype="fp32", sigma=4.0,
                   backward=True),
    "px128_fwd": dict(batch=8, heads=6, H=128, W=128, d=64, B=16, L=3, K=8, dtype="bf16", sigma=4.0,
                      backward=False),
    "px128": dict(batch=8, heads=6, H=128, W=128, d=64, B=16, L=3, K=8, dtype="bf16", sigma=4.0,
                  backward=True),
    "px256": dict(batch=2, heads=6, H=256, W=256, d=64, B=16, L=4, K=8, dtype="bf16", sigma=4.0,
                  backward=True),
    "px512": dict(batch=1, heads=16, H=512, W=512, d=64, B=16, L=4, K=8, dtype="bf16", sigma=8.0,
                  backward=True),
}
