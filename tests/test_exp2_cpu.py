"""The kernels' FMA-pipe exp2 on the CPU: the constants in csrc/sm100.cuh are the
ones the committed Remez generator produces, and an f32 emulation of the device
function (Cody-Waite reduction with the 1.5 * 2^23 rounding constant, Horner by
fused multiply-adds, 2^n added to the exponent field) stays within the bound the
GPU test applies, over the range the softmax uses."""
import importlib.util
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "causal_flash_attention_attn_b200", "csrc")


def _generator():
    spec = importlib.util.spec_from_file_location("gen_exp2_poly", os.path.join(CSRC, "gen_exp2_poly.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def device_coefficients():
    """c0..c4 as written in exp2_poly (Horner from the highest degree down)."""
    text = open(os.path.join(CSRC, "sm100.cuh")).read()
    body = text[text.index("float exp2_poly(float y)"):]
    body = body[:body.index("\n}\n")]
    lits = [float(x) for x in re.findall(r"([0-9]\.[0-9]+e[-+][0-9]+)f", body)]
    assert len(lits) == 5, lits
    c4, c3, c2, c1, c0 = lits
    return np.array([c0, c1, c2, c3, c4], dtype=np.float32)


def f32(x):
    return np.asarray(x, dtype=np.float32)


def fma32(a, b, c):
    # a*b is exact in f64 for f32 a, b; one rounding of the sum to f32 (a double
    # rounding through f64 can differ from a true FMA in the last f32 bit, far
    # below the bound tested)
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def exp2_poly_emulated(y, c):
    y = np.maximum(f32(y), f32(-125.0))
    t = (y + f32(12582912.0)).astype(np.float32)
    n = (t - f32(12582912.0)).astype(np.float32)
    f = (y - n).astype(np.float32)
    p = fma32(f, np.full_like(f, c[4]), np.full_like(f, c[3]))
    p = fma32(p, f, np.full_like(f, c[2]))
    p = fma32(p, f, np.full_like(f, c[1]))
    p = fma32(p, f, np.full_like(f, c[0]))
    bits = (p.view(np.int32).astype(np.int64) + (t.view(np.int32).astype(np.int64) << 23)) & 0xFFFFFFFF
    return bits.astype(np.uint32).view(np.float32)


def test_constants_are_the_generators():
    gen = _generator()
    c = gen.remez_rel(4)
    err, c32 = gen.f32_horner_err(c)
    assert err < 2.8e-6
    np.testing.assert_array_equal(c32, device_coefficients())


def test_reduction_splits_y_into_integer_and_half_unit_fraction():
    y = f32(np.linspace(-125.0, 8.0, 200001))
    t = (y + f32(12582912.0)).astype(np.float32)
    n = (t - f32(12582912.0)).astype(np.float32)
    f = (y - n).astype(np.float32)
    assert np.all(n == np.round(n)) and np.all(np.abs(f) <= 0.5)
    np.testing.assert_array_equal(n.astype(np.float64) + f.astype(np.float64), y.astype(np.float64))


@pytest.mark.parametrize("lo,hi", [(-125.0, 8.0), (-12.0, 8.0), (-0.5, 0.5)])
def test_emulated_device_exp2_within_the_bound(lo, hi):
    c = device_coefficients()
    y = f32(np.concatenate([np.linspace(lo, hi, 1_000_001), [0.0, -0.5, 0.5, -1.0, 1.0]]))
    got = exp2_poly_emulated(y, c).astype(np.float64)
    exact = np.exp2(y.astype(np.float64))
    rel = np.abs(got - exact) / exact
    assert rel.max() < 4e-6, rel.max()


def test_below_range_clamps_to_two_to_the_minus_125():
    c = device_coefficients()
    got = exp2_poly_emulated(f32([-126.0, -200.0, -1e30]), c).astype(np.float64)
    np.testing.assert_allclose(got, 2.0 ** -125, rtol=4e-6)
