"""GPU parity of the warm-start kernel against the fp64 oracle, through the C ABI.

Tolerance (derived from the kernel's fp32 arithmetic; M = max |x_lr|, n = max(h, w)):
  * upsampling: the source coordinate (i + 1/2) * (n_in / n_out) - 1/2 carries at most
    2^-22 (n + 1) of rounding (the fp32 ratio and two operations), which moves each of the two
    bilinear weights of an axis by as much; with |x1 - x0| <= 2M over two axes and three fused
    multiply-adds this bounds |dU| by 2^-20 (n + 2) M;
  * sharpening multiplies that by at most 1 + 2s (U and a blur of U), plus eight roundings;
  * drawn noise: logf, sqrtf and sincospif are each within two ulp, so a Box-Muller normal z
    is within 2^-19 (1 + |z|) of the fp64 transform of the same words;
  * the blend adds two roundings of the result.
For ratios that are powers of two the source coordinates are exact and the error is a few
ulp; the mean error is also checked against 2^-18.
"""
import numpy as np
import pytest

from oracle import warm_start_oracle as WO

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ug(gpu_required):
    from diffusion_transformer_ultra_b200 import build
    build.build()
    import diffusion_transformer_ultra_b200 as pkg
    return pkg


def oracle_planes(x_lr, H, W, alpha, s, planes, noise=None, seed=0, offset=0):
    """Oracle output for the listed (b, c) planes, [len(planes), H, W]."""
    B, C = x_lr.shape[:2]
    out = []
    for b, c in planes:
        lr = x_lr[b:b + 1, c:c + 1].double().numpy()
        if noise is not None:
            n = noise[b:b + 1, c:c + 1].double().numpy()
        else:
            n = WO.philox_normals(seed, offset, H * W, first=(b * C + c) * H * W).reshape(1, 1, H, W)
        out.append(WO.warm_start(lr, H, W, alpha, s, noise=n)[0, 0])
    return np.stack(out), np.stack(
        [noise[b, c].double().numpy() if noise is not None else
         WO.philox_normals(seed, offset, H * W, first=(b * C + c) * H * W).reshape(H, W)
         for b, c in planes])


def check(got, ref, noise, x_lr, alpha, s, drawn, what):
    M = float(x_lr.abs().max())
    n_in = max(x_lr.shape[-2:])
    u_err = 2.0 ** -20 * (n_in + 2) * M
    ref_err = (1 + 2 * s) * u_err + 8 * 2.0 ** -24 * (1 + s) * M
    noise_err = 2.0 ** -19 * (1 + np.abs(noise)) if drawn else 0.0
    tol = (1 - alpha) * ref_err + alpha * noise_err + 2.0 ** -22 * (1 + np.abs(ref))
    d = np.abs(got - ref)
    bad = d > tol
    assert not bad.any(), f"{what}: {bad.sum()} elements out of tolerance, max {d.max():.3e}"
    assert d.mean() <= 2.0 ** -18, f"{what}: mean error {d.mean():.3e}"


def run(ug, wl, noise_mode="given", alpha=None, s=None, misalign=False, seed=12345, offset=7):
    import torch
    x_lr, noise = ug.make_warm(wl)
    alpha = wl.alpha if alpha is None else alpha
    s = wl.sharpen if s is None else s
    shape = (wl.batch, wl.C, wl.H, wl.W)
    n_el = int(np.prod(shape))
    if misalign:
        big = torch.full((n_el + 1,), float("nan"), device="cuda")
        out = big[1:].view(shape)
        nbig = torch.empty((n_el + 1,), device="cuda")
        nd = nbig[1:].view(shape)
        nd.copy_(noise)
    else:
        out = torch.full(shape, float("nan"), device="cuda")
        nd = noise.cuda()
    ug.warm_start(x_lr.cuda(), out, alpha, s, noise=nd if noise_mode == "given" else None,
                  seed=seed, offset=offset)
    torch.cuda.synchronize()
    return x_lr, noise, out.cpu(), alpha, s


@pytest.mark.parametrize("name,mode", [("warm_tiny", "given"), ("warm_ragged", "given"),
                                       ("warm_tiny", "drawn"), ("warm_ragged", "drawn")])
def test_warm_start_full_parity(ug, name, mode):
    wl = ug.WARM_WORKLOADS[name]
    x_lr, noise, out, alpha, s = run(ug, wl, mode)
    assert not np.isnan(out.numpy()).any()
    planes = [(b, c) for b in range(wl.batch) for c in range(wl.C)]
    ref, nz = oracle_planes(x_lr, wl.H, wl.W, alpha, s, planes,
                            noise=noise if mode == "given" else None, seed=12345, offset=7)
    got = np.stack([out[b, c].double().numpy() for b, c in planes])
    check(got, ref, nz, x_lr, alpha, s, mode == "drawn", f"{name} {mode}")


def test_warm_start_special_cases(ug):
    import torch
    wl = ug.WARM_WORKLOADS["warm_ragged"]
    # alpha = 1: the output is the noise, bit for bit
    x_lr, noise, out, _, _ = run(ug, wl, "given", alpha=1.0)
    assert torch.equal(out, noise)
    # alpha = 0, no sharpening: bilinear interpolation alone
    x_lr, noise, out, _, _ = run(ug, wl, "given", alpha=0.0, s=0.0)
    ref = WO.bilinear_upsample(x_lr.double().numpy(), wl.H, wl.W)
    check(out.double().numpy(), ref, noise.double().numpy(), x_lr, 0.0, 0.0, False, "interp only")


def test_warm_start_unaligned_buffers_take_the_scalar_path(ug):
    wl = ug.WARM_WORKLOADS["warm_tiny"]            # W % 4 == 0, buffers offset by 4 bytes
    x_lr, noise, out, alpha, s = run(ug, wl, "given", misalign=True)
    planes = [(0, c) for c in range(wl.C)]
    ref, nz = oracle_planes(x_lr, wl.H, wl.W, alpha, s, planes, noise=noise)
    got = np.stack([out[0, c].double().numpy() for _, c in planes])
    check(got, ref, nz, x_lr, alpha, s, False, "unaligned")


@pytest.mark.parametrize("mode", ["given", "drawn"])
def test_warm_start_full_size_sampled_planes(ug, mode):
    """The 8K latent in the benchmark's configuration, two planes checked in full."""
    wl = ug.WARM_WORKLOADS["warm_8k"]
    x_lr, noise, out, alpha, s = run(ug, wl, mode)
    planes = [(0, 0), (0, wl.C - 1)]
    ref, nz = oracle_planes(x_lr, wl.H, wl.W, alpha, s, planes,
                            noise=noise if mode == "given" else None, seed=12345, offset=7)
    got = np.stack([out[b, c].double().numpy() for b, c in planes])
    check(got, ref, nz, x_lr, alpha, s, mode == "drawn", f"8k {mode}")
    assert not np.isnan(out.numpy()).any()


def test_warm_start_drawn_noise_is_deterministic_and_seeded(ug):
    import torch
    wl = ug.WARM_WORKLOADS["warm_tiny"]
    _, _, a, _, _ = run(ug, wl, "drawn", alpha=1.0, seed=5, offset=0)
    _, _, b, _, _ = run(ug, wl, "drawn", alpha=1.0, seed=5, offset=0)
    _, _, c, _, _ = run(ug, wl, "drawn", alpha=1.0, seed=6, offset=0)
    assert torch.equal(a, b)
    assert not torch.equal(a, c)
    z = a.double().numpy().reshape(-1)
    assert abs(z.mean()) < 5 / np.sqrt(z.size) and abs(z.var() - 1) < 5 * np.sqrt(2 / z.size)


# integer ratios take the fused kernel (W = 4 w, H = ry h with ry <= 8); the last shape has
# H % h != 0 and takes the tiled kernel
FUSED_SHAPES = [(9, 7, 9, 28), (9, 7, 18, 28), (5, 6, 15, 24), (4, 5, 32, 20), (5, 6, 17, 24)]


@pytest.mark.parametrize("shape", FUSED_SHAPES)
@pytest.mark.parametrize("mode", ["given", "drawn"])
def test_warm_start_integer_ratio_paths(ug, shape, mode):
    import dataclasses
    h, w, H, W = shape
    wl = dataclasses.replace(ug.WARM_WORKLOADS["warm_tiny"], name="warm_ratio", cfg=24, batch=2,
                             C=3, h=h, w=w, H=H, W=W, alpha=0.4, sharpen=0.8)
    x_lr, noise, out, alpha, s = run(ug, wl, mode)
    assert not np.isnan(out.numpy()).any()
    planes = [(b, c) for b in range(wl.batch) for c in range(wl.C)]
    ref, nz = oracle_planes(x_lr, H, W, alpha, s, planes,
                            noise=noise if mode == "given" else None, seed=12345, offset=7)
    got = np.stack([out[b, c].double().numpy() for b, c in planes])
    check(got, ref, nz, x_lr, alpha, s, mode == "drawn", f"{shape} {mode}")
