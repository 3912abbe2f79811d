"""The prefill kernel's FMA-pipe exponential, emulated step by step in float32.

The attention kernel computes a fixed share of each row's probabilities
p = 2^x with a cubic instead of the MUFU ex2 unit (exp2_poly_x2 in
attn_prefill.cu).  This test reads the constants out of that source and
replays the same float32 operations: the rounding trick for n = round(x), the
reduced argument f = x - n, the cubic, and the exponent-field add.  It checks
the relative error over the range the kernel feeds it (x in [-125, 8]; the lazy
rescale lets x exceed 0 by up to 8), that nothing overflows into the sign bit
or turns into inf/NaN for any input (masked keys give x = -inf), and that the
result is tiny below the clamp.
"""
import pathlib
import re

import numpy as np

SRC = pathlib.Path(__file__).resolve().parents[1] / "doge_dynamic_mask_b200" / "csrc" / "attn_prefill.cu"
f32 = np.float32


def _constants():
    text = SRC.read_text()
    body = text[text.index("void exp2_poly_x2("):]
    body = body[:body.index("\n}\n")]
    clamp = float(re.search(r"fmaxf\(x0, (-?[0-9.]+)f\)", body).group(1))
    magic = float(re.search(r"f32x2\(([0-9.]+)f, \1f\);\s*// 1.5", body).group(1))
    coeffs = [float(c) for c in re.findall(r"f32x2\((0\.[0-9]+)f, \1f\)", body)]
    # Horner order in the source: c3, c2, c1, c0
    assert len(coeffs) == 4, coeffs
    return clamp, magic, [f32(c) for c in coeffs[::-1]]


def _poly(x):
    clamp, magic, (c0, c1, c2, c3) = _constants()
    x = np.maximum(x.astype(f32), f32(clamp))
    t = (x + f32(magic)).astype(f32)
    f = (x - (t - f32(magic)).astype(f32)).astype(f32)
    q = (f * c3 + c2).astype(f32)
    q = (q * f + c1).astype(f32)
    q = (q * f + c0).astype(f32)
    bits = (q.view(np.uint32).astype(np.uint64) + ((t.view(np.uint32).astype(np.uint64) << 23) & 0xFFFFFFFF))
    return (bits & 0xFFFFFFFF).astype(np.uint32).view(f32)


def test_constants_are_the_fitted_ones():
    clamp, magic, c = _constants()
    assert clamp == -126.0 and magic == 1.5 * 2 ** 23
    # the cubic is a fit of 2^f on [-1/2, 1/2]: close to the Taylor terms of 2^f
    assert abs(c[0] - 1) < 1e-3 and abs(c[1] - np.log(2)) < 1e-3
    assert abs(c[2] - np.log(2) ** 2 / 2) < 5e-3 and abs(c[3] - np.log(2) ** 3 / 6) < 5e-3


def test_relative_error_over_the_kernel_range():
    x = np.linspace(-125.0, 8.0, 1_000_001).astype(f32)
    p = _poly(x)
    rel = np.abs(p.astype(np.float64) / np.exp2(x.astype(np.float64)) - 1.0)
    # far below the bf16 rounding (2^-9 relative) that P goes through next
    assert rel.max() < 1e-4, rel.max()


def test_integers_and_half_integers():
    x = np.array([0.0, -1.0, -2.0, 1.0, 8.0, -0.5, 0.5, -7.5, -100.0], dtype=f32)
    p = _poly(x)
    np.testing.assert_allclose(p, np.exp2(x.astype(np.float64)), rtol=1e-4)


def test_no_sign_or_inf_for_any_input():
    x = np.concatenate([np.array([-np.inf, -1e30, -1e10, -130.0, -126.5, -126.0, -125.99], dtype=f32),
                        np.linspace(-200, -120, 10001).astype(f32)])
    p = _poly(x)
    assert np.isfinite(p).all() and (p >= 0).all()
    below = x <= -126.0
    assert p[below].max() <= np.exp2(-125.0)   # effectively zero next to the row maximum's weight 1


def test_cubic_is_the_minimax_fit_of_the_relative_error():
    """The cubic is the best uniform (minimax) fit of 2^f's relative error on
    [-1/2, 1/2]: by the Chebyshev alternation theorem a cubic is that fit
    exactly when its error reaches its maximum magnitude at five points with
    alternating signs (the two ends and three interior extrema)."""
    _, _, (c0, c1, c2, c3) = _constants()
    f = np.linspace(-0.5, 0.5, 400001)
    rel = (float(c0) + f * (float(c1) + f * (float(c2) + f * float(c3)))) / np.exp2(f) - 1.0
    inner = np.nonzero(np.diff(np.sign(np.diff(rel))))[0] + 1
    pts = np.concatenate([[0], inner, [len(f) - 1]])
    assert len(pts) == 5
    vals = rel[pts]
    assert (np.sign(vals[1:]) != np.sign(vals[:-1])).all()             # alternating signs
    assert np.abs(vals).min() >= 0.999 * np.abs(rel).max()              # equal magnitude
    assert np.abs(rel).max() < 7.5e-5
