"""The FMA-pipe 2^y of the masked prefill attention, checked against exp2.

The kernel (csrc/attention_tc.cu, exp2_pair_fma) evaluates some exponentials
without the ex2 unit: round y to an integer r with the 1.5 * 2^23 shifter,
evaluate a cubic for 2^(y - r), and add r to the exponent field.  This test
reads the shifter and the cubic's coefficients from the kernel source and
replays the same float32 steps on the CPU: the result must be within the
cubic's relative error bound of the true 2^y over the range the kernel feeds
it ([-126, 8]), and the clamp must send y = -inf (masked keys) below 2^-125.
"""

import os
import re

import numpy as np

SRC = os.path.join(os.path.dirname(__file__), "..", "fine_grained_top_b200", "csrc", "attention_tc.cu")


def _constants():
    text = open(SRC).read()
    vals = {}
    for name in ("kExpShift", "kExp2C0", "kExp2C1", "kExp2C2", "kExp2C3"):
        m = re.search(name + r"\s*=\s*([-+0-9.eE]+)f", text)
        assert m, name
        vals[name] = np.float32(float(m.group(1)))
    return vals


def _exp2_fma(y):
    c = _constants()
    f32 = np.float32
    y = np.maximum(y.astype(f32), f32(-126.0))
    t = (y + c["kExpShift"]).astype(f32)
    r = (t - c["kExpShift"]).astype(f32)
    fr = (y - r).astype(f32)
    p = (c["kExp2C3"] * fr + c["kExp2C2"]).astype(f32)
    p = (p * fr + c["kExp2C1"]).astype(f32)
    p = (p * fr + c["kExp2C0"]).astype(f32)
    bits = (p.view(np.uint32) + (t.view(np.uint32) << np.uint32(23))).astype(np.uint32)
    return bits.view(f32)


def test_shifter_bits_vanish():
    # the shifter's bit pattern shifted left by 23 is 0 mod 2^32, so t_bits << 23 == r << 23
    shift = _constants()["kExpShift"]
    assert (int(np.array([shift], np.float32).view(np.uint32)[0]) << 23) % (1 << 32) == 0


def test_relative_error_over_kernel_range():
    y = np.concatenate([np.linspace(-125.0, 8.0, 400001), np.arange(-125, 9) + 0.5,
                        np.arange(-125, 9).astype(np.float64)]).astype(np.float32)
    got = _exp2_fma(y).astype(np.float64)
    want = np.exp2(y.astype(np.float64))
    rel = np.abs(got / want - 1.0)
    assert rel.max() < 1e-4, rel.max()


def test_masked_keys_end_below_2_pow_minus_125():
    got = _exp2_fma(np.array([-np.inf, -1e30, -200.0, -126.0], np.float32)).astype(np.float64)
    assert np.all(got >= 0.0) and np.all(got < 2.0 ** -125)


def _remez_relative(deg, a, b, f, iters=40):
    """Minimax polynomial of degree `deg` in relative error on [a, b], by the
    Remez exchange: solve for equioscillation on deg + 2 reference points,
    move the references to the extrema of the error, repeat."""
    n = deg + 2
    x = (a + b) / 2 + (b - a) / 2 * np.cos(np.pi * np.arange(n)[::-1] / (n - 1))
    grid = np.linspace(a, b, 200001)
    for _ in range(iters):
        A = np.zeros((n, n))
        A[:, :deg + 1] = x[:, None] ** np.arange(deg + 1)
        A[:, deg + 1] = (-1.0) ** np.arange(n) * f(x)
        coef = np.linalg.solve(A, f(x))[:deg + 1]
        err = np.polyval(coef[::-1], grid) / f(grid) - 1.0
        segs = np.split(np.arange(len(grid)), np.where(np.diff(np.sign(err)) != 0)[0] + 1)
        ext = [s[np.argmax(np.abs(err[s]))] for s in segs]
        if len(ext) != n:
            break
        x = grid[ext]
    return coef, np.abs(err).max()


def test_cubic_is_the_remez_minimax_fit():
    # the kernel's coefficients are the minimax cubic for 2^f on [-1/2, 1/2]
    # in relative error, to float32 precision
    coef, emax = _remez_relative(3, -0.5, 0.5, np.exp2)
    c = _constants()
    got = np.array([c["kExp2C0"], c["kExp2C1"], c["kExp2C2"], c["kExp2C3"]], np.float64)
    assert np.allclose(got, coef, rtol=2e-7, atol=0), (got, coef)
    assert 7.4e-5 < emax < 7.6e-5
