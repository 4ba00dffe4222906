"""Seeded synthetic Q/K/V for the HLA workloads.

This module only draws numbers: it holds no step of the attention method (no permutation,
no RoPE, no mask).  Tests, the oracle checks, ``smoke()`` and ``bench.py`` all take their
inputs from here, so the CUDA path and the oracle see the same bytes.

Recipe (per tensor, raster layout [B, N_raster, heads, D], segment order text | HR | LR):
  * i.i.d. N(0, 1) float32 from ``numpy.random.default_rng``; the token axis is cut into
    fixed chunks, each with its own child seed, so the values do not depend on threading;
  * the bf16 workloads add a smooth 2D sinusoid of amplitude 0.5 per channel
    c in [0, heads*D):  0.5 * sin(2 pi (u_c y / H + v_c x / W) + phi_c) with
    u_c, v_c in {1..4} and phi_c ~ U[0, 2 pi); HR tokens use (y, x) = (i, j), LR tokens
    (m, n) use (y, x) = (rho m, rho n), text tokens get no sinusoid;
  * bf16 workloads are rounded to bfloat16 (round to nearest even); the tiny workload
    stays float32.
Seeds: Q/K/V = 1000*cfg + {1, 2, 3}; sinusoid parameters = 1000*cfg + 7.

Warm-start latents (``make_warm``): the low-resolution latent [B, C, h, w] is i.i.d. N(0, 1)
plus a smooth per-channel 2D sinusoid of amplitude 1 (a stand-in for generated image
structure); the noise X_T [B, C, H, W] is i.i.d. N(0, 1); both float32.  Seeds
1000*cfg + 11 (latent), + 12 (noise), + 13 (sinusoid).
"""
from __future__ import annotations

import concurrent.futures as cf
import os
from dataclasses import dataclass, field

import numpy as np

_CHUNK_TOKENS = 4096


@dataclass(frozen=True)
class Workload:
    name: str
    cfg: int            # seed family
    H: int
    W: int
    l: int
    b: int
    rho: int
    T: int
    heads: int
    D: int
    batch: int
    dtype: str          # "bf16" or "f32" (stored input dtype)
    axes: tuple = field(default=(16, 56, 56))
    sinusoid: bool = True

    @property
    def h(self) -> int:
        return -(-self.H // self.rho) if self.rho > 0 else 0

    @property
    def w(self) -> int:
        return -(-self.W // self.rho) if self.rho > 0 else 0

    @property
    def n_raster(self) -> int:
        return self.T + self.H * self.W + self.h * self.w


WORKLOADS = {
    "tiny": Workload("tiny", 0, 32, 32, 8, 2, 4, 16, 1, 64, 1, "f32", (16, 24, 24), False),
    "1k": Workload("1k", 1, 64, 64, 16, 4, 4, 512, 24, 128, 1, "bf16"),
    "4k": Workload("4k", 2, 256, 256, 16, 4, 4, 512, 24, 128, 1, "bf16"),
    "8k": Workload("8k", 3, 512, 512, 16, 4, 4, 512, 24, 128, 1, "bf16"),
    "ragged": Workload("ragged", 4, 256, 135, 16, 16, 4, 256, 24, 128, 2, "bf16"),
    # the largest layer considered: a 16K image (1024 x 1024 HR tokens, 256 x 256 LR)
    "16k": Workload("16k", 5, 1024, 1024, 16, 4, 4, 512, 24, 128, 1, "bf16"),
}


def _normal_chunk(seed: int, chunk: int, shape) -> np.ndarray:
    rng = np.random.default_rng([seed, chunk])
    return rng.standard_normal(shape, dtype=np.float32)


def _sinusoid_params(wl: Workload):
    rng = np.random.default_rng(1000 * wl.cfg + 7)
    C = wl.heads * wl.D
    u = rng.integers(1, 5, size=C).astype(np.float64)
    v = rng.integers(1, 5, size=C).astype(np.float64)
    phi = rng.uniform(0.0, 2.0 * np.pi, size=C)
    return u, v, phi


def _token_yx(wl: Workload, t0: int, t1: int):
    """(y, x, has_sinusoid) for raster tokens [t0, t1)."""
    t = np.arange(t0, t1)
    y = np.zeros(len(t))
    x = np.zeros(len(t))
    has = np.zeros(len(t), bool)
    hr = (t >= wl.T) & (t < wl.T + wl.H * wl.W)
    r = t[hr] - wl.T
    y[hr], x[hr] = r // wl.W, r % wl.W
    has[hr] = True
    lr = t >= wl.T + wl.H * wl.W
    if lr.any():
        r = t[lr] - wl.T - wl.H * wl.W
        y[lr], x[lr] = wl.rho * (r // wl.w), wl.rho * (r % wl.w)
        has[lr] = True
    return y, x, has


def _make_chunk(wl: Workload, seed: int, ci: int, params) -> np.ndarray:
    t0 = ci * _CHUNK_TOKENS
    t1 = min(wl.n_raster, t0 + _CHUNK_TOKENS)
    x = _normal_chunk(seed, ci, (wl.batch, t1 - t0, wl.heads * wl.D))
    if wl.sinusoid:
        u, v, phi = params
        yy, xx, has = _token_yx(wl, t0, t1)
        if has.any():
            arg = 2.0 * np.pi * (np.outer(yy[has] / wl.H, u) + np.outer(xx[has] / wl.W, v)) + phi
            x[:, has, :] += (0.5 * np.sin(arg)).astype(np.float32)[None]
    return x


def make_tensor(wl: Workload, which: str, threads: int | None = None):
    """One of 'q', 'k', 'v' as a CPU torch tensor [B, N_raster, heads, D] (bf16 or fp32)."""
    import torch

    seed = 1000 * wl.cfg + {"q": 1, "k": 2, "v": 3}[which]
    params = _sinusoid_params(wl) if wl.sinusoid else None
    n_chunks = -(-wl.n_raster // _CHUNK_TOKENS)
    out_dtype = torch.bfloat16 if wl.dtype == "bf16" else torch.float32
    out = torch.empty((wl.batch, wl.n_raster, wl.heads, wl.D), dtype=out_dtype)
    flat = out.view(wl.batch, wl.n_raster, wl.heads * wl.D)

    def work(ci):
        t0 = ci * _CHUNK_TOKENS
        xc = torch.from_numpy(_make_chunk(wl, seed, ci, params))
        flat[:, t0:t0 + xc.shape[1], :] = xc.to(out_dtype)

    threads = threads or min(16, os.cpu_count() or 1)
    with cf.ThreadPoolExecutor(threads) as ex:
        list(ex.map(work, range(n_chunks)))
    return out


def make_qkv(wl: Workload, threads: int | None = None):
    return tuple(make_tensor(wl, w, threads) for w in ("q", "k", "v"))


@dataclass(frozen=True)
class WarmWorkload:
    name: str
    cfg: int
    batch: int
    C: int              # latent channels
    h: int
    w: int
    H: int
    W: int
    alpha: float        # t / T of the starting timestep
    sharpen: float      # unsharp-mask amount


WARM_WORKLOADS = {
    "warm_tiny": WarmWorkload("warm_tiny", 20, 1, 4, 16, 16, 64, 64, 0.7, 1.0),
    "warm_ragged": WarmWorkload("warm_ragged", 21, 2, 3, 13, 11, 50, 47, 0.3, 0.5),
    # 4K / 8K images: 16-channel latents at 1/8 of the pixel grid, guide at rho = 4
    "warm_4k": WarmWorkload("warm_4k", 22, 1, 16, 128, 128, 512, 512, 0.7, 1.0),
    "warm_8k": WarmWorkload("warm_8k", 23, 1, 16, 256, 256, 1024, 1024, 0.7, 1.0),
}


def make_warm(wl: WarmWorkload):
    """(x_lr [B, C, h, w], noise [B, C, H, W]) as CPU float32 torch tensors."""
    import torch

    rng = np.random.default_rng(1000 * wl.cfg + 11)
    x = rng.standard_normal((wl.batch, wl.C, wl.h, wl.w), dtype=np.float32)
    prm = np.random.default_rng(1000 * wl.cfg + 13)
    u = prm.integers(1, 4, size=wl.C)
    v = prm.integers(1, 4, size=wl.C)
    phi = prm.uniform(0.0, 2.0 * np.pi, size=wl.C)
    yy = np.arange(wl.h)[:, None] / wl.h
    xx = np.arange(wl.w)[None, :] / wl.w
    for c in range(wl.C):
        x[:, c] += np.sin(2.0 * np.pi * (u[c] * yy + v[c] * xx) + phi[c]).astype(np.float32)
    noise = np.random.default_rng(1000 * wl.cfg + 12).standard_normal(
        (wl.batch, wl.C, wl.H, wl.W), dtype=np.float32)
    return torch.from_numpy(x), torch.from_numpy(noise)
