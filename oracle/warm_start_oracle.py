"""Oracle for UltraGen's warm-start initialisation. TEST INFRASTRUCTURE ONLY.

A plain fp64 NumPy restatement of the guidance-weighted warm start. Only ``tests/``,
``__graft_entry__.smoke()`` and ``bench.py`` may import or run this module. It shares no code
with the CUDA library and imports nothing from the product package.

Sources (page title, then the section on the page):
  [UG-note]  "UltraGen: Efficient Ultra-High-Resolution Image Generation with Hierarchical
             Local Attention", papernotes.org note, 关键设计 4 (guidance-weighted warm-start
             sampling) and its blend equation.
  [UG-gist]  same title, gist.science English summary, "2. Methodology" D (Inference
             Acceleration, Warm-Start Initialization).

The method: the generated low-resolution latent X_lr is upsampled to the high-resolution
latent grid by interpolation and sharpened, giving the reference X_ref. The starting latent
is the blend X_hr = alpha * X_T + (1 - alpha) * X_ref of Gaussian noise X_T and that
reference, where alpha = t / T is the noise level of the intermediate timestep.

Readings taken where the pages leave a step open:
  W1  "Interpolate" is bilinear upsampling from the LR grid (h, w) to the HR grid (H, W)
      with half-pixel centres: along each axis the source coordinate of output index i is
      (i + 0.5) * (h / H) - 0.5, clamped below at 0; the two taps are floor of it and the
      next index (clamped to h - 1), weighted by the fractional part.
  W2  "Sharpen" is an unsharp mask: X_ref = U + s * (U - B(U)), where U is the upsampled
      latent, B the 3x3 binomial blur (1 2 1)^T (1 2 1) / 16 per channel with replicated
      edges, and s >= 0 the amount (s = 0: no sharpening).
  W3  The noise X_T is standard normal per element. The caller passes it in, or it is drawn
      from the counter-based generator Philox4x32-10 (Salmon, Moraes, Dror and Shaw,
      "Parallel random numbers: as easy as 1, 2, 3", SC 2011) followed by the Box-Muller
      transform, both restated here from their published definitions:
        element e of the flat [B, C, H, W] array uses block g = e // 4 and lane e % 4;
        counter = (g mod 2^32, g >> 32, offset mod 2^32, offset >> 32),
        key = (seed mod 2^32, seed >> 32); the block's words x0..x3 give
        u(x) = (floor(x / 2^9) + 1/2) * 2^-23 (exact in fp32), and
        lanes 0, 1 = r cos(2 pi u(x1)), r sin(2 pi u(x1)) with r = sqrt(-2 ln u(x0)),
        lanes 2, 3 the same from (x2, x3).
  W4  Layout: latents are [B, C, h, w] and [B, C, H, W] (channel-planar), any H >= h,
      W >= w; the blend uses the caller's alpha.

Parity status: each function is pinned by ``tests/test_warm_start_pins.py``: bilinear
against torch's independent interpolate, the blur against scipy's convolution, Philox
against its published known-answer vectors, Box-Muller by a Kolmogorov-Smirnov test, and
the blend by its alpha = 0 / 1 special cases and constant inputs.
"""
from __future__ import annotations

import numpy as np

_MASK32 = np.uint64(0xFFFFFFFF)


# ---------------------------------------------------------------------------- W1 interpolate
def _axis_taps(n_out: int, n_in: int):
    """Per output index along one axis: (i0, i1, frac), half-pixel centres (reading W1)."""
    i = np.arange(n_out, dtype=np.float64)
    src = (i + 0.5) * (n_in / n_out) - 0.5
    src = np.maximum(src, 0.0)
    i0 = np.floor(src).astype(np.int64)
    i0 = np.minimum(i0, n_in - 1)
    i1 = np.minimum(i0 + 1, n_in - 1)
    return i0, i1, src - i0


def bilinear_upsample(x: np.ndarray, H: int, W: int) -> np.ndarray:
    """x [..., h, w] -> [..., H, W] by bilinear interpolation ([UG-note] 关键设计 4, W1)."""
    x = np.asarray(x, dtype=np.float64)
    h, w = x.shape[-2:]
    y0, y1, fy = _axis_taps(H, h)
    x0, x1, fx = _axis_taps(W, w)
    fy = fy[:, None]
    fx = fx[None, :]
    top = x[..., y0[:, None], x0[None, :]] * (1 - fx) + x[..., y0[:, None], x1[None, :]] * fx
    bot = x[..., y1[:, None], x0[None, :]] * (1 - fx) + x[..., y1[:, None], x1[None, :]] * fx
    return top * (1 - fy) + bot * fy


# ---------------------------------------------------------------------------- W2 sharpen
def blur3(u: np.ndarray) -> np.ndarray:
    """3x3 binomial blur (1 2 1)^T (1 2 1) / 16 over the last two axes, edges replicated."""
    u = np.asarray(u, dtype=np.float64)
    pad = [(0, 0)] * (u.ndim - 2) + [(1, 1), (1, 1)]
    p = np.pad(u, pad, mode="edge")
    H, W = u.shape[-2:]
    wts = (1.0, 2.0, 1.0)
    out = np.zeros_like(u)
    for dy in range(3):
        for dx in range(3):
            out += wts[dy] * wts[dx] * p[..., dy:dy + H, dx:dx + W]
    return out / 16.0


def sharpen(u: np.ndarray, amount: float) -> np.ndarray:
    """Unsharp mask U + s (U - blur(U)) (reading W2)."""
    return u + amount * (u - blur3(u))


# ---------------------------------------------------------------------------- W3 noise
_PHILOX_M0, _PHILOX_M1 = np.uint64(0xD2511F53), np.uint64(0xCD9E8D57)
_PHILOX_W0, _PHILOX_W1 = np.uint64(0x9E3779B9), np.uint64(0xBB67AE85)


def philox4x32_10(ctr, key):
    """Philox4x32 with 10 rounds: ctr is 4 uint32-valued arrays, key 2; returns 4 arrays.

    Each round multiplies counter words 0 and 2 by the two round multipliers, and forms the
    new counter from the high halves xor-ed with the other two words and the key, and the low
    halves. The key is advanced by the two Weyl constants before every round after the first.
    """
    c0, c1, c2, c3 = (np.asarray(c, dtype=np.uint64) & _MASK32 for c in ctr)
    k0, k1 = (np.asarray(k, dtype=np.uint64) & _MASK32 for k in key)
    for rnd in range(10):
        if rnd:
            k0 = (k0 + _PHILOX_W0) & _MASK32
            k1 = (k1 + _PHILOX_W1) & _MASK32
        p0 = _PHILOX_M0 * c0
        p1 = _PHILOX_M1 * c2
        c0, c1, c2, c3 = ((p1 >> np.uint64(32)) ^ c1 ^ k0, p1 & _MASK32,
                          (p0 >> np.uint64(32)) ^ c3 ^ k1, p0 & _MASK32)
    return c0, c1, c2, c3


def uniform_open(x) -> np.ndarray:
    """Word -> (0, 1): (floor(x / 2^9) + 1/2) * 2^-23 (reading W3)."""
    return ((np.asarray(x, dtype=np.uint64) >> np.uint64(9)).astype(np.float64) + 0.5) * 2.0 ** -23


def box_muller(u1, u2):
    """Two independent standard normals from two uniforms on (0, 1)."""
    r = np.sqrt(-2.0 * np.log(u1))
    return r * np.cos(2.0 * np.pi * u2), r * np.sin(2.0 * np.pi * u2)


def philox_normals(seed: int, offset: int, n: int, first: int = 0) -> np.ndarray:
    """Normals first .. first + n - 1 of the stream (seed, offset), in fp64 (reading W3)."""
    g0 = first // 4
    n_blocks = (first + n + 3) // 4 - g0
    g = np.arange(g0, g0 + n_blocks, dtype=np.uint64)
    zeros = np.zeros_like(g)
    ctr = (g & _MASK32, g >> np.uint64(32), zeros + np.uint64(offset & 0xFFFFFFFF),
           zeros + np.uint64(offset >> 32))
    key = (np.uint64(seed & 0xFFFFFFFF), np.uint64(seed >> 32))
    x0, x1, x2, x3 = philox4x32_10(ctr, key)
    z0, z1 = box_muller(uniform_open(x0), uniform_open(x1))
    z2, z3 = box_muller(uniform_open(x2), uniform_open(x3))
    z = np.stack([z0, z1, z2, z3], axis=1).reshape(-1)
    return z[first - 4 * g0:first - 4 * g0 + n]


# ---------------------------------------------------------------------------- blend
def reference_latent(x_lr: np.ndarray, H: int, W: int, amount: float) -> np.ndarray:
    """X_ref = sharpen(Interpolate(X_lr)) ([UG-note] 关键设计 4)."""
    return sharpen(bilinear_upsample(x_lr, H, W), amount)


def warm_start(x_lr: np.ndarray, H: int, W: int, alpha: float, amount: float,
               noise: np.ndarray | None = None, seed: int = 0, offset: int = 0) -> np.ndarray:
    """X_hr = alpha X_T + (1 - alpha) X_ref ([UG-note] 关键设计 4, the blend equation).

    x_lr is [B, C, h, w]; the result is [B, C, H, W] in fp64. Without `noise`, X_T is the
    Philox/Box-Muller stream (seed, offset) over the flat output (reading W3).
    """
    x_lr = np.asarray(x_lr, dtype=np.float64)
    B, C = x_lr.shape[:2]
    ref = reference_latent(x_lr, H, W, amount)
    if noise is None:
        noise = philox_normals(seed, offset, B * C * H * W).reshape(B, C, H, W)
    noise = np.asarray(noise, dtype=np.float64)
    return alpha * noise + (1.0 - alpha) * ref
