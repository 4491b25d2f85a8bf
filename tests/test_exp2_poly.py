"""The forward kernel's FMA-pipe exp2 (Cody-Waite reduction + degree-3 minimax
polynomial): the constants compiled into the kernel are the ones the Remez
generator produces, and the kernel's float32 arithmetic, emulated here, stays
within its relative-error bound against the exact 2^x."""
import os
import re

import numpy as np

from exact_io_aware_online_b200 import exp2_poly as E

KERNEL = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                      "exact_io_aware_online_b200", "csrc", "sm100_ptx.cuh")


def _kernel_coefficients():
    body = open(KERNEL).read()
    body = body[body.index("exp2_poly2(float x0"):]
    body = body[: body.index("\n}\n")]
    vals = [float(v) for v in re.findall(r"f2\((-?[0-9.]+)f, \1f\)", body)]
    return vals[-4:]  # order of appearance in Horner form: c3, c2, c1, c0


def test_kernel_uses_the_remez_coefficients():
    coef, err = E.remez()
    got = _kernel_coefficients()
    assert len(got) == 4
    c3, c2, c1, c0 = got[0], got[1], got[2], got[3]
    np.testing.assert_allclose([c0, c1, c2, c3], [np.float32(c) for c in coef], rtol=0, atol=5e-8)
    assert err < 8e-5


def test_minimax_error_equioscillates():
    coef, err = E.remez()
    x = np.linspace(E.LO, E.HI, 100001)
    r = np.polyval(coef[::-1], x) / np.exp2(x) - 1.0
    assert abs(np.abs(r).max() - err) < 1e-9
    # a degree-3 minimax fit touches its error bound at degree + 2 = 5 points with alternating sign
    peaks = [i for i in range(1, len(x) - 1) if abs(r[i]) >= abs(r[i - 1]) and abs(r[i]) >= abs(r[i + 1])]
    peaks = [0] + peaks + [len(x) - 1]
    big = [p for p in peaks if abs(r[p]) > 0.99 * err]
    assert len(big) >= 5
    signs = np.sign(r[big])
    assert all(signs[i] != signs[i + 1] for i in range(len(signs) - 1))


def test_float32_emulation_against_exact_exp2():
    coef, _ = E.remez()
    rng = np.random.default_rng(0)
    xs = np.concatenate([np.linspace(-120, 8, 400001), rng.uniform(-30, 8, 400000)]).astype(np.float32)
    y = E.emulate_f32(xs, coef)
    rel = np.abs(y.astype(np.float64) / np.exp2(xs.astype(np.float64)) - 1.0)
    assert rel.max() < 1.5e-4
    # integers are exact powers of two up to the polynomial's value at 0
    ints = np.arange(-120, 9, dtype=np.float32)
    np.testing.assert_allclose(E.emulate_f32(ints, coef), np.exp2(ints) * np.float32(coef[0]), rtol=1e-6)
