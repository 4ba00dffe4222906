"""Pins of the oracle's 8-bit Q K^T reading (scaled e4m3 Q and K after RoPE).

* the e4m3 rounding: every finite code decoded from its bit fields is a fixed point; rounding
  matches a brute-force nearest search over that decoded table (ties to the even code) and
  torch's float8_e4m3fn conversion (an independent implementation); values past 448 clamp;
* the stored codes: decoding e4m3_codes by the bit-field rule gives the rounded value back;
* the scaled quantizer: scaling the input by 2^a and the exponent by a scales the stored value
  by 2^a exactly;
* the attention: a pure-Python brute force with its own quantizer on tiny grids; inputs already
  on the e4m3 grid with RoPE off give exactly the unquantized result; Q = 0 gives exactly the
  unquantized result (V is not quantized); moving a power of two from K to Q leaves the output
  unchanged; the logits stay inside the bound that half an e4m3 spacing per factor gives.
"""
import math

import numpy as np
import pytest
import torch

from oracle import hla_oracle as O
from test_oracle_pins import TINY_GEOMS, bf_forward


def decode_e4m3(code: int) -> float:
    """Value of an e4m3 byte from its bit fields (sign 7, exponent 6..3 bias 7, mantissa
    2..0); exponent field 0 is subnormal (mantissa * 2^-9); S.1111.111 is NaN."""
    s = -1.0 if code & 0x80 else 1.0
    e = (code >> 3) & 0xF
    m = code & 0x7
    if e == 0xF and m == 0x7:
        return math.nan
    if e == 0:
        return s * m * 2.0 ** -9
    return s * (1.0 + m / 8.0) * 2.0 ** (e - 7)


TABLE = sorted({decode_e4m3(c) for c in range(256) if not math.isnan(decode_e4m3(c))})
CODE_OF = {}
for _c in range(256):
    _v = decode_e4m3(_c)
    if not math.isnan(_v) and not (_v == 0 and _c == 0x80):
        CODE_OF[_v] = _c


def bf_round_e4m3(x: float) -> float:
    """Nearest entry of the decoded table; a tie goes to the entry whose code is even."""
    if x >= TABLE[-1]:
        return TABLE[-1]
    if x <= TABLE[0]:
        return TABLE[0]
    best = min(TABLE, key=lambda t: abs(t - x))
    d = abs(best - x)
    ties = [t for t in TABLE if abs(t - x) == d]
    if len(ties) > 1:
        best = [t for t in ties if CODE_OF[t] % 2 == 0][0]
    return best


def test_table_shape():
    assert len(TABLE) == 253                      # 254 finite codes, +0 and -0 equal
    assert TABLE[-1] == 448.0 and TABLE[0] == -448.0
    assert min(t for t in TABLE if t > 0) == 2.0 ** -9


def test_every_finite_value_is_a_fixed_point():
    t = np.array(TABLE)
    np.testing.assert_array_equal(O.round_e4m3(t), t)


def test_rounding_matches_brute_force_nearest_search():
    rng = np.random.default_rng(11)
    pos = np.array([t for t in TABLE if t >= 0])
    mids = (pos[1:] + pos[:-1]) / 2                # exact ties
    x = np.concatenate([
        rng.uniform(-460, 460, 400), rng.uniform(-0.05, 0.05, 400),
        rng.standard_normal(400) * 4, mids, -mids,
        mids + 2.0 ** -30 * mids, mids - 2.0 ** -30 * mids, [449.0, 463.9, 464.0, 1e6, -1e6],
    ])
    expect = np.array([bf_round_e4m3(v) for v in x])
    np.testing.assert_array_equal(O.round_e4m3(x), expect)


def test_rounding_matches_torch_float8_e4m3fn():
    rng = np.random.default_rng(12)
    x = np.concatenate([rng.uniform(-447, 447, 20000), rng.standard_normal(20000) * 3,
                        rng.uniform(-2.0 ** -5, 2.0 ** -5, 20000)]).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    np.testing.assert_array_equal(O.round_e4m3(x.astype(np.float64)), ref)


def test_codes_decode_to_the_rounded_value():
    rng = np.random.default_rng(13)
    x = np.concatenate([rng.standard_normal(5000) * 10, rng.uniform(-0.02, 0.02, 5000),
                        [0.0, 448.0, -448.0, 1e9, 2.0 ** -9, -(2.0 ** -9)]])
    for e in (0, 3, -2):
        codes = O.e4m3_codes(x, e)
        dec = np.array([decode_e4m3(int(c)) for c in codes]) * 2.0 ** e
        np.testing.assert_array_equal(dec, O.quantize_e4m3(x, e))
        assert not ((codes & 0x7F) == 0x7F).any()  # never NaN


def test_scaled_quantizer_commutes_with_powers_of_two():
    rng = np.random.default_rng(14)
    x = rng.standard_normal(2000) * 3
    for a in (-5, -1, 2, 7):
        np.testing.assert_array_equal(O.quantize_e4m3(x * 2.0 ** a, a), O.quantize_e4m3(x, 0) * 2.0 ** a)
    # the exponent picks the range: large values fit only with a larger scale
    big = np.array([3000.0, -5000.0])
    np.testing.assert_array_equal(O.quantize_e4m3(big, 0), [448.0, -448.0])
    np.testing.assert_array_equal(O.quantize_e4m3(big, 4), [3072.0, -5120.0])


@pytest.mark.parametrize("geom", TINY_GEOMS[:3])
@pytest.mark.parametrize("q_exp,k_exp", [(0, 0), (-2, 1)])
def test_forward_matches_brute_force(geom, q_exp, k_exp):
    H, W, l, b, rho, T, axes = geom
    g = O.Geometry(H, W, l, b, rho, T)
    D = sum(axes)
    rng = np.random.default_rng(17)
    q, k, v = (rng.standard_normal((1, g.N_raster, 2, D)) * 2 for _ in range(3))
    expect = bf_forward(q, k, v, H, W, l, b, rho, T, axes,
                        quant_q=lambda x: bf_round_e4m3(x * 2.0 ** -q_exp) * 2.0 ** q_exp,
                        quant_k=lambda x: bf_round_e4m3(x * 2.0 ** -k_exp) * 2.0 ** k_exp)
    o_perm, _ = O.forward(q, k, v, g, axes, qk_format="e4m3", q_exp=q_exp, k_exp=k_exp)
    np.testing.assert_allclose(O.unpermute(o_perm, g), expect, rtol=0, atol=1e-12)


GEO = (12, 10, 4, 2, 2, 7)


def test_grid_inputs_without_rope_are_exact():
    g = O.Geometry(*GEO)
    rng = np.random.default_rng(18)
    tab = np.array([t for t in TABLE if abs(t) <= 8])
    q, k = (rng.choice(tab, (1, g.N_raster, 2, 64)) for _ in range(2))
    v = rng.standard_normal((1, g.N_raster, 2, 64))
    axes = (64, 0, 0)                              # every pair on axis 0: position 0, no rotation
    o8, _ = O.forward(q, k, v, g, axes, qk_format="e4m3")
    o, _ = O.forward(q, k, v, g, axes)
    np.testing.assert_array_equal(o8, o)


def test_zero_queries_leave_v_exact():
    g = O.Geometry(*GEO)
    rng = np.random.default_rng(19)
    q = np.zeros((1, g.N_raster, 2, 64))
    k, v = (rng.standard_normal((1, g.N_raster, 2, 64)) for _ in range(2))
    o8, _ = O.forward(q, k, v, g, (16, 24, 24), qk_format="e4m3")
    o, _ = O.forward(q, k, v, g, (16, 24, 24))
    np.testing.assert_allclose(o8, o, rtol=0, atol=1e-14)


def test_moving_a_power_of_two_between_q_and_k_changes_nothing():
    g = O.Geometry(*GEO)
    rng = np.random.default_rng(20)
    q, k, v = (rng.standard_normal((1, g.N_raster, 2, 64)) for _ in range(3))
    a = 3
    o0, _ = O.forward(q, k, v, g, (16, 24, 24), qk_format="e4m3")
    o1, _ = O.forward(q * 2.0 ** a, k * 2.0 ** -a, v, g, (16, 24, 24), qk_format="e4m3",
                      q_exp=a, k_exp=-a)
    np.testing.assert_array_equal(o1, o0)


def test_logits_stay_inside_the_half_spacing_bound():
    g = O.Geometry(*GEO)
    rng = np.random.default_rng(21)
    q, k = (rng.standard_normal((1, g.N_raster, 1, 64)) * 2 for _ in range(2))
    pos = O.positions(g)
    qr, kr = O.rope(q, pos, (16, 24, 24)), O.rope(k, pos, (16, 24, 24))
    q8, k8 = O.quantize_e4m3(qr, 0), O.quantize_e4m3(kr, 0)
    # per element: |x8 - x| <= 2^-4 |x| for normal values, <= 2^-10 below 2^-6
    for x, x8 in ((qr, q8), (kr, k8)):
        assert np.all(np.abs(x8 - x) <= np.maximum(2.0 ** -4 * np.abs(x), 2.0 ** -10) * (1 + 1e-15))
    Q, K, Q8, K8 = (a[0, :, 0, :] for a in (qr, kr, q8, k8))
    dq = np.maximum(2.0 ** -4 * np.abs(Q), 2.0 ** -10)
    dk = np.maximum(2.0 ** -4 * np.abs(K), 2.0 ** -10)
    bound = np.abs(Q) @ dk.T + dq @ np.abs(K).T + dq @ dk.T
    err = np.abs(Q8 @ K8.T - Q @ K.T)
    assert np.all(err <= bound * (1 + 1e-12))
    assert err.max() > 0.05 * bound.max()         # the quantizer really acts
