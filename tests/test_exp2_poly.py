"""The attention kernel's FMA-pipe 2^x (CPU, no GPU).

Part of every page's exponentials is computed without the MUFU unit: x = j + f
with j = round(x) (Cody-Waite additive reduction through the 1.5*2^23
shifter), p(f) ~ 2^f by a degree-3 minimax polynomial, and 2^j applied by
adding j to the exponent field of p(f).  These tests tie the kernel's
constants to the Remez fit that produced them and bound the float32 scheme's
relative error against exp2 over the kernel's input range; an input below
-125 (a masked key's -inf among them) must give exactly 0.
"""
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "windowed_memory_attention_b200", "csrc")
KERNEL = os.path.join(CSRC, "attend_sm100.cu")
BOUND = 7.5e-5          # the fit's minimax relative error on [-1/2, 1/2]


def kernel_constants():
    src = open(KERNEL).read()
    vals = {}
    for m in re.finditer(r"constexpr float kExpC(\d) = (0x[0-9a-fA-Fp.+-]+)f;", src):
        vals[int(m.group(1))] = float.fromhex(m.group(2))
    assert sorted(vals) == [0, 1, 2, 3], vals
    return np.array([vals[i] for i in range(4)], dtype=np.float32)


def fit():
    import importlib.util
    spec = importlib.util.spec_from_file_location("exp2_poly_fit", os.path.join(CSRC, "exp2_poly_fit.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod.remez()


def f32(x):
    return np.asarray(x, dtype=np.float64).astype(np.float32)


def fma32(a, b, c):
    # one rounding of a*b + c to float32 (the product of two float32 is exact in float64)
    return f32(a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64))


def exp2_scheme(x, c):
    """The kernel's float32 steps, element by element."""
    x = f32(x)
    zero = x < np.float32(-125.0)
    xc = np.maximum(x, np.float32(-125.0))
    shifter = np.float32(12582912.0)                 # 1.5 * 2^23
    t = f32(xc.astype(np.float64) + shifter)          # j = rne(x) in the low mantissa bits
    j = f32(t.astype(np.float64) - shifter)
    f = fma32(j, np.float32(-1.0) * np.ones_like(j), xc)
    p = fma32(np.full_like(f, c[3]), f, np.full_like(f, c[2]))
    p = fma32(p, f, np.full_like(f, c[1]))
    p = fma32(p, f, np.full_like(f, c[0]))
    bits = (p.view(np.uint32).astype(np.uint64) + (t.view(np.uint32).astype(np.uint64) << np.uint64(23)))
    y = (bits & np.uint64(0xFFFFFFFF)).astype(np.uint32).view(np.float32)
    return np.where(zero, np.float32(0.0), y)


def test_kernel_constants_are_the_remez_fit():
    c, err = fit()
    assert err <= BOUND
    np.testing.assert_array_equal(kernel_constants(), np.float32(c))


def test_fit_is_minimax_on_the_reduced_interval():
    # equioscillation: the relative error reaches +-E at 5 alternating points
    c, err = fit()
    g = np.linspace(-0.5, 0.5, 100001)
    e = (np.polyval(c[::-1], g) - 2.0 ** g) / 2.0 ** g
    assert abs(np.abs(e).max() - err) < 1e-7
    ext = [e[0]] + [e[i] for i in range(1, len(e) - 1) if abs(e[i]) >= abs(e[i - 1]) and abs(e[i]) >= abs(e[i + 1]) and abs(e[i]) > 0.99 * err] + [e[-1]]
    signs = np.sign([v for v in ext if abs(v) > 0.99 * err])
    assert len(signs) >= 5 and np.all(signs[1:] != signs[:-1])


@pytest.mark.parametrize("lo,hi", [(-125.0, -100.0), (-100.0, -1.0), (-1.0, 1.0), (1.0, 64.0)])
def test_relative_error_over_the_input_range(lo, hi):
    c = kernel_constants()
    rng = np.random.default_rng(7)
    x = np.concatenate([np.linspace(lo, hi, 200001), rng.uniform(lo, hi, 200000),
                        np.arange(np.ceil(lo), np.floor(hi) + 1) + 0.5,      # reduction boundaries
                        np.arange(np.ceil(lo), np.floor(hi) + 1)])
    x = f32(x)
    y = exp2_scheme(x, c).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(y - ref) / ref
    # the fit's bound plus a few float32 roundings of the Horner steps
    assert rel.max() <= BOUND + 4 * 2.0 ** -23, rel.max()


def test_masked_and_underflowing_inputs_give_exact_zero():
    c = kernel_constants()
    x = f32([-np.inf, -1e30, -126.0, -125.0001, -200.0])
    assert np.all(exp2_scheme(x, c) == 0.0)
    # -125 itself is the smallest input still represented
    assert exp2_scheme(f32([-125.0]), c)[0] > 0.0


def test_kernel_selects_zero_below_the_clamp():
    # the kernel source keeps the clamp's zero select next to the polynomial
    src = open(KERNEL).read()
    body = src[src.index("void exp2_poly2"):]
    body = body[:body.index("\n}\n")]
    assert "-125.f" in body and "? 0.f" in body
