"""The FMA-pipe 2^x used for a share of the softmax exponentials: its coefficients are the
generator's output, and its fp32 evaluation (simulated here bit for bit: the 1.5*2^23 shifter,
the Horner polynomial with fused multiply-adds, the integer exponent add) stays within
1e-4 relative error of 2^x over the range the kernel feeds it."""
import importlib.util
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "diffusion_transformer_ultra_b200", "csrc")


def header_coeffs():
    txt = open(os.path.join(CSRC, "exp2_poly.h")).read()
    return [np.float32(float(v)) for v in re.findall(r"UG_EXP2_C\d ([-+0-9.e]+)f", txt)]


def fma32(a, b, c):
    # a fused multiply-add rounds once: evaluate in fp64 (exact for fp32 operands' product
    # up to 48 bits, plus c) and round to fp32
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def ex2_fma_sim(x):
    c0, c1, c2, c3 = header_coeffs()
    x = np.maximum(x.astype(np.float32), np.float32(-125.0))
    magic = np.float32(12582912.0)
    t = (x + magic).astype(np.float32)
    f = (x - (t - magic).astype(np.float32)).astype(np.float32)
    p = fma32(f, np.full_like(f, c3), np.full_like(f, c2))
    p = fma32(f, p, np.full_like(f, c1))
    p = fma32(f, p, np.full_like(f, c0))
    bits = p.view(np.int32) + (t.view(np.int32) << np.int32(23))
    return bits.view(np.float32)


def test_header_matches_generator():
    spec = importlib.util.spec_from_file_location("gen", os.path.join(CSRC, "gen_exp2_poly.py"))
    gen = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(gen)
    np.testing.assert_array_equal(np.array(header_coeffs(), np.float32), gen.fit())


def test_relative_error_over_kernel_range():
    x = np.concatenate([np.linspace(-124.9, 8.5, 2_000_001, dtype=np.float32),
                        np.arange(-124, 9, dtype=np.float32),
                        np.arange(-124, 9, dtype=np.float32) + np.float32(0.5)])
    got = ex2_fma_sim(x).astype(np.float64)
    rel = np.abs(got / np.exp2(x.astype(np.float64)) - 1)
    assert rel.max() < 1e-4


def test_masked_and_underflow_inputs_are_negligible():
    got = ex2_fma_sim(np.array([-np.inf, -1e30, -200.0, -125.0], np.float32))
    assert np.all(np.isfinite(got)) and np.all(got > 0) and np.all(got <= 2.0 ** -124)
