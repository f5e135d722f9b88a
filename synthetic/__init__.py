"""Seeded synthetic inputs shared by the tests, the smoke check and the benchmark.

This module holds no arithmetic of the attention method: it only draws
spatially smooth pixel-token tensors and rounds them to bf16, so that the CUDA
path and the CPU oracle can be fed the very same numbers.

Recipe (stands in for the FFHQ / ImageNet pixel tokens the method is trained
on; the datasets themselves are not used):
  * every (batch, head, channel) of Q, K and V is an independent H x W field
    of N(0, 1) noise,
  * blurred by a Gaussian of width ``sigma`` pixels (periodic boundary,
    applied as its exact transfer function in the Fourier domain),
  * standardised to zero mean and unit variance,
  * plus ``noise`` * N(0, 1) white noise,
  * laid out in raster order as [batch, heads, H*W, d];
  * the upstream gradient dO is plain N(0, 1) drawn from its own seed.
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import scipy.fft


def round_to_bf16(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bf16 (ties to even); returns float32."""
    x = np.array(x, dtype=np.float32, copy=True, order="C")
    u = x.view(np.uint32)              # finite values: no uint32 overflow below
    lsb = (u >> 16) & 1
    u += np.uint32(0x7FFF)
    u += lsb
    u &= np.uint32(0xFFFF0000)
    return x


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """The upper 16 bits of float32 values that are already bf16-exact."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    return (x.view(np.uint32) >> 16).astype(np.uint16)


def _gaussian_transfer(H: int, W: int, sigma: float) -> np.ndarray:
    fy = np.fft.fftfreq(H)[:, None]
    fx = np.fft.rfftfreq(W)[None, :]
    return np.exp(-2.0 * np.pi ** 2 * sigma ** 2 * (fy ** 2 + fx ** 2)).astype(np.float32)


def smooth_fields(seed: int, count: int, H: int, W: int, sigma: float, noise: float = 0.1) -> np.ndarray:
    """``count`` independent smooth H x W fields as float32 [count, H, W].

    Fields are drawn in chunks, each from its own child stream of ``seed``
    (numpy SeedSequence.spawn), so the result does not depend on the number
    of threads that draw them."""
    out = np.empty((count, H, W), dtype=np.float32)
    chunk = max(1, (1 << 21) // (H * W))
    starts = list(range(0, count, chunk))
    children = np.random.SeedSequence(seed).spawn(len(starts))
    tf = _gaussian_transfer(H, W, sigma) if sigma > 0 else None

    def one(i):
        s = starts[i]
        e = min(count, s + chunk)
        rng = np.random.default_rng(children[i])
        f = rng.standard_normal((e - s, H, W), dtype=np.float32)
        if tf is not None:
            f = scipy.fft.irfft2(scipy.fft.rfft2(f) * tf, s=(H, W)).astype(np.float32)
        mu = f.mean(axis=(1, 2), keepdims=True)
        sd = f.std(axis=(1, 2), keepdims=True)
        f = (f - mu) / np.maximum(sd, 1e-12)
        f += noise * rng.standard_normal((e - s, H, W), dtype=np.float32)
        out[s:e] = f

    with ThreadPoolExecutor(max_workers=os.cpu_count() or 1) as ex:
        list(ex.map(one, range(len(starts))))
    return out


def pixel_tokens(seed: int, batch: int, heads: int, H: int, W: int, d: int, sigma: float,
                 noise: float = 0.1, bf16: bool = True) -> np.ndarray:
    """One [batch, heads, H*W, d] raster-order token tensor of smooth fields."""
    f = smooth_fields(seed, batch * heads * d, H, W, sigma, noise)
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
    rows = batch * heads * N
    g = np.empty((rows, d), dtype=np.float32)
    chunk = max(1, (1 << 21) // d)
    starts = list(range(0, rows, chunk))
    children = np.random.SeedSequence(seed).spawn(len(starts))

    def one(i):
        s = starts[i]
        e = min(rows, s + chunk)
        g[s:e] = np.random.default_rng(children[i]).standard_normal((e - s, d), dtype=np.float32)

    with ThreadPoolExecutor(max_workers=os.cpu_count() or 1) as ex:
        list(ex.map(one, range(len(starts))))
    g = g.reshape(batch, heads, N, d)
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
