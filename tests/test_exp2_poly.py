"""The FMA-pipe 2^x of the compress kernels (exp2_fma.cuh), checked on the CPU.

The header's coefficients are evaluated the way the kernel does (fp32 range reduction through
x + 1.5 * 2^23, fp32 Horner steps with one rounding each, exponent added to the bit pattern) and
compared with exact 2^x; the fit that produced them is checked for the minimax property (an
error curve that equioscillates); special values are checked by hand.
"""
import importlib.util
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "cross_model_attention_map_b200", "csrc")


def header_coefficients():
    text = open(os.path.join(CSRC, "exp2_fma.cuh")).read()
    c = {int(k): float(v) for k, v in re.findall(r"kExp2C(\d) = ([-+0-9.e]+)f;", text)}
    assert sorted(c) == list(range(6))
    return np.array([c[k] for k in range(6)], dtype=np.float32)


def fma32(a, b, c):
    # fp32 fused multiply-add: the product of two fp32 values is exact in fp64
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def exp2_like_kernel(x, coef):
    x = np.maximum(np.asarray(x, dtype=np.float32), np.float32(-126.0))
    rnd = np.float32(12582912.0)
    t = (x + rnd).astype(np.float32)
    f = (x - (t - rnd).astype(np.float32)).astype(np.float32)
    p = np.full_like(f, coef[5])
    for k in (4, 3, 2, 1, 0):
        p = fma32(p, f, np.full_like(f, coef[k]))
    bits = p.view(np.uint32) + (t.view(np.uint32) << np.uint32(23))
    return bits.astype(np.uint32).view(np.float32)


def test_error_bound_against_exact_powers():
    coef = header_coefficients()
    rng = np.random.default_rng(7)
    x = np.concatenate([-rng.uniform(0.0, 126.0, 1_000_000),
                        -np.linspace(0.0, 2.0, 200_001)]).astype(np.float32)
    y = exp2_like_kernel(x, coef).astype(np.float64)
    rel = np.abs(y / np.exp2(x.astype(np.float64)) - 1.0)
    assert rel.max() < 3e-7, rel.max()


def test_special_values():
    coef = header_coefficients()
    y = exp2_like_kernel(np.array([0.0, -1.0, -2.0, -0.5, -126.0, -300.0], np.float32), coef)
    exact = np.array([1.0, 0.5, 0.25, 2.0 ** -0.5, 2.0 ** -126, 2.0 ** -126])
    assert np.allclose(y, exact, rtol=3e-7, atol=0.0)
    # integer arguments differ from exact powers of two only by the polynomial's value at f = 0
    xi = -np.arange(0, 127, dtype=np.float32)
    yi = exp2_like_kernel(xi, coef).astype(np.float64)
    assert np.all(np.abs(yi / np.exp2(xi.astype(np.float64)) - 1.0) <= 2.0 ** -23 + 1e-12)


def test_fit_is_minimax():
    spec = importlib.util.spec_from_file_location("fit_exp2_poly", os.path.join(CSRC, "fit_exp2_poly.py"))
    fit = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(fit)
    c, err = fit.remez_exp2(5)
    assert err < 1e-7
    # equioscillation: the relative error reaches +-err at deg + 2 = 7 alternating points
    f = np.linspace(-0.5, 0.5, 400001)
    e = np.polyval(c[::-1], f) / np.exp2(f) - 1.0
    peaks = [0] + [i for i in range(1, len(f) - 1)
                   if abs(e[i]) >= abs(e[i - 1]) and abs(e[i]) >= abs(e[i + 1])] + [len(f) - 1]
    big = [i for i in peaks if abs(e[i]) > 0.99 * err]
    signs = np.sign(e[big])
    runs = 1 + int(np.sum(signs[1:] != signs[:-1]))
    assert runs >= 7
    # the header holds these coefficients, rounded to fp32
    assert np.array_equal(header_coefficients(), c.astype(np.float32))


@pytest.mark.parametrize("planted", ["c1", "round"])
def test_a_planted_mistake_is_caught(planted):
    coef = header_coefficients().copy()
    x = -np.linspace(0.0, 20.0, 100_001).astype(np.float32)
    if planted == "c1":
        coef[1] *= np.float32(1.0 + 1e-5)
        y = exp2_like_kernel(x, coef)
    else:
        # reduction by truncation instead of rounding: f leaves [-1/2, 1/2]
        t = np.floor(x).astype(np.float32)
        f = (x - t).astype(np.float32)
        p = np.polyval(coef[::-1].astype(np.float64), f.astype(np.float64))
        y = (p * np.exp2(t.astype(np.float64))).astype(np.float32)
    rel = np.abs(y.astype(np.float64) / np.exp2(x.astype(np.float64)) - 1.0)
    assert rel.max() > 3e-7
