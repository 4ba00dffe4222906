"""Pins of the warm-start oracle against things other than itself.

* bilinear upsampling: torch's interpolate (an independent implementation of the same
  half-pixel rule) and the closed form on linear ramps;
* the 3x3 binomial blur: scipy's convolution with replicated edges, constants, ramps;
* Philox4x32-10: the known-answer vectors published with the Random123 library;
* Box-Muller: a Kolmogorov-Smirnov test against the standard normal CDF, moments and
  lane independence;
* the blend: alpha = 1 gives the noise, alpha = 0 the reference, constants stay constant.
"""
import numpy as np
import pytest

from oracle import warm_start_oracle as WO


@pytest.mark.parametrize("shape,H,W", [((2, 3, 7, 5), 28, 20), ((1, 2, 16, 16), 64, 64),
                                       ((1, 1, 13, 11), 50, 47), ((1, 1, 9, 6), 9, 6),
                                       ((1, 1, 1, 4), 3, 16)])
def test_bilinear_matches_torch_interpolate(shape, H, W):
    import torch
    rng = np.random.default_rng(1)
    x = rng.standard_normal(shape)
    ref = torch.nn.functional.interpolate(torch.from_numpy(x), size=(H, W), mode="bilinear",
                                          align_corners=False).numpy()
    np.testing.assert_allclose(WO.bilinear_upsample(x, H, W), ref, rtol=0, atol=1e-12)


def test_bilinear_reproduces_linear_ramps_in_the_interior():
    h, w, rho = 12, 10, 4
    H, W = h * rho, w * rho
    a, b, c = 0.37, -1.25, 0.5
    ii, jj = np.meshgrid(np.arange(h), np.arange(w), indexing="ij")
    x = (a * ii + b * jj + c)[None, None]
    up = WO.bilinear_upsample(x, H, W)[0, 0]
    sy = (np.arange(H) + 0.5) / rho - 0.5
    sx = (np.arange(W) + 0.5) / rho - 0.5
    exact = a * sy[:, None] + b * sx[None, :] + c
    inner = (slice(rho, H - rho), slice(rho, W - rho))   # no clamped tap
    np.testing.assert_allclose(up[inner], exact[inner], atol=1e-12)
    # at the clamped border the value is the edge value
    np.testing.assert_allclose(up[0, 0], x[0, 0, 0, 0])


def test_blur_matches_scipy_convolve_nearest():
    from scipy import ndimage
    rng = np.random.default_rng(2)
    u = rng.standard_normal((2, 3, 17, 23))
    k = np.outer([1.0, 2.0, 1.0], [1.0, 2.0, 1.0]) / 16.0
    ref = np.stack([[ndimage.convolve(u[b, c], k, mode="nearest") for c in range(3)]
                    for b in range(2)])
    np.testing.assert_allclose(WO.blur3(u), ref, atol=1e-13)


def test_blur_and_sharpen_invariants():
    u = np.full((1, 1, 8, 9), 3.25)
    np.testing.assert_allclose(WO.blur3(u), u)
    np.testing.assert_allclose(WO.sharpen(u, 1.5), u)
    ramp = np.add.outer(np.arange(10.0) * 0.5, np.arange(11.0) * -0.25)[None, None]
    np.testing.assert_allclose(WO.blur3(ramp)[..., 1:-1, 1:-1], ramp[..., 1:-1, 1:-1], atol=1e-13)
    rng = np.random.default_rng(3)
    v = rng.standard_normal((1, 2, 6, 7))
    np.testing.assert_array_equal(WO.sharpen(v, 0.0), v)
    # an isolated spike: blur spreads it over 3x3 with weights 4/16 (centre), 2/16, 1/16
    z = np.zeros((1, 1, 5, 5))
    z[0, 0, 2, 2] = 16.0
    np.testing.assert_allclose(WO.blur3(z)[0, 0, 1:4, 1:4], [[1, 2, 1], [2, 4, 2], [1, 2, 1]])
    np.testing.assert_allclose(WO.sharpen(z, 1.0)[0, 0, 2, 2], 16.0 + (16.0 - 4.0))


# Known-answer values published with the Random123 library for Philox4x32 with 10 rounds.
PHILOX_KAT = [
    ((0x00000000, 0x00000000, 0x00000000, 0x00000000), (0x00000000, 0x00000000),
     (0x6627e8d5, 0xe169c58d, 0xbc57ac4c, 0x9b00dbd8)),
    ((0xffffffff, 0xffffffff, 0xffffffff, 0xffffffff), (0xffffffff, 0xffffffff),
     (0x408f276d, 0x41c83b0e, 0xa20bc7c6, 0x6d5451fd)),
    ((0x243f6a88, 0x85a308d3, 0x13198a2e, 0x03707344), (0xa4093822, 0x299f31d0),
     (0xd16cfe09, 0x94fdcceb, 0x5001e420, 0x24126ea1)),
]


@pytest.mark.parametrize("ctr,key,out", PHILOX_KAT)
def test_philox_known_answers(ctr, key, out):
    got = WO.philox4x32_10([np.uint64(c) for c in ctr], [np.uint64(k) for k in key])
    assert tuple(int(x) for x in got) == out


def test_uniform_open_is_exact_in_fp32_and_inside_the_interval():
    x = np.array([0, 1, 511, 512, 2**31, 2**32 - 1], dtype=np.uint64)
    u = WO.uniform_open(x)
    assert np.all(u > 0) and np.all(u < 1)
    np.testing.assert_array_equal(u.astype(np.float32).astype(np.float64), u)
    assert u[0] == 2.0 ** -24 and u[-1] == 1 - 2.0 ** -24


def test_philox_normals_are_standard_normal():
    from scipy import stats
    z = WO.philox_normals(seed=1234, offset=0, n=1 << 18)
    assert abs(z.mean()) < 5 / np.sqrt(z.size)
    assert abs(z.var() - 1) < 5 * np.sqrt(2 / z.size)
    assert stats.kstest(z, "norm").pvalue > 1e-3
    lanes = z.reshape(-1, 4)
    for a, b in ((0, 1), (0, 2), (1, 3), (2, 3)):
        assert abs(np.corrcoef(lanes[:, a], lanes[:, b])[0, 1]) < 5 / np.sqrt(lanes.shape[0])
    # the stream depends on seed and offset, and a prefix does not depend on the length
    assert not np.allclose(WO.philox_normals(1234, 1, 64), z[:64])
    assert not np.allclose(WO.philox_normals(1235, 0, 64), z[:64])
    np.testing.assert_array_equal(WO.philox_normals(1234, 0, 7), z[:7])
    np.testing.assert_array_equal(WO.philox_normals(1234, 0, 9, first=1001), z[1001:1010])


def test_blend_special_cases():
    rng = np.random.default_rng(4)
    x_lr = rng.standard_normal((1, 2, 8, 8))
    noise = rng.standard_normal((1, 2, 32, 32))
    np.testing.assert_array_equal(WO.warm_start(x_lr, 32, 32, 1.0, 0.7, noise=noise), noise)
    np.testing.assert_allclose(WO.warm_start(x_lr, 32, 32, 0.0, 0.7, noise=noise),
                               WO.reference_latent(x_lr, 32, 32, 0.7))
    const = np.full((1, 1, 4, 4), -0.75)
    out = WO.warm_start(const, 16, 16, 0.3, 1.0, noise=np.zeros((1, 1, 16, 16)))
    np.testing.assert_allclose(out, 0.7 * -0.75)
    gen = WO.warm_start(x_lr, 32, 32, 1.0, 0.0, seed=9, offset=3)
    np.testing.assert_array_equal(gen.reshape(-1), WO.philox_normals(9, 3, gen.size))
