"""Error bound and provenance of the FMA-pipe exp2 the attention kernel can use for part of the
softmax exponentials (off by default).

The constants are this repository's own fitted cubic, parsed from csrc/attn_fwd.cu; the fit is
reproduced below (float64 weighted least squares with Lawson's reweighting toward the minimax
relative error on [-1/2, 1/2], constant term pinned to 1). The device algorithm (Cody-Waite reduction
x = n + f with n = round(x), |f| <= 1/2; cubic for 2^f in Horner form; n added to the exponent
field; inputs below -127 clamped) is replayed in float32 with numpy, then compared with the exact
2^x. The kernel rounds P to bf16 (relative 2^-9), so a relative error below 1.5e-4 is far
inside the attention tolerance."""
import os
import re

import numpy as np

SRC = os.path.join(os.path.dirname(os.path.dirname(__file__)),
                   "video_diffusion_transformer_vdit_b200", "csrc", "attn_fwd.cu")


def _coeffs():
    text = open(SRC).read()
    got = {k: float(v) for k, v in re.findall(r"kExp2(C\d) = ([0-9.eE+-]+)f", text)}
    return [np.float32(got[f"C{i}"]) for i in range(4)]


def _exp2_fma(x):
    c0, c1, c2, c3 = _coeffs()
    x = np.maximum(x.astype(np.float32), np.float32(-127.0))
    big = np.float32(12582912.0)
    t = (x + big).astype(np.float32)
    r = (t - big).astype(np.float32)
    f = (x - r).astype(np.float32)
    q = (c3 * f + c2).astype(np.float32)
    q = (q * f + c1).astype(np.float32)
    q = (q * f + c0).astype(np.float32)
    n = t.view(np.int32) - np.int32(0x4B400000)
    return (q.view(np.int32) + (n << 23)).view(np.float32)


def _lawson_fit(iters=400):
    """Cubic 1 + c1 f + c2 f^2 + c3 f^3 minimising the maximum relative error to 2^f on
    [-1/2, 1/2]: Lawson's algorithm (C. L. Lawson, 1961) iterates weighted least squares,
    multiplying each sample's weight by its current absolute error, which converges to the
    minimax (equioscillating) solution."""
    f = np.linspace(-0.5, 0.5, 4001)
    e = np.exp2(f)
    a = np.stack([f / e, f ** 2 / e, f ** 3 / e], axis=1)  # relative error = a c - (1 - 1/e)
    b = 1.0 - 1.0 / e
    wt = np.full(f.size, 1.0 / f.size)
    c = None
    for _ in range(iters):
        sw = np.sqrt(wt)
        c = np.linalg.lstsq(a * sw[:, None], b * sw, rcond=None)[0]
        r = np.abs(a @ c - b)
        wt = wt * r
        wt /= wt.sum()
    return c, float(np.abs(a @ c - b).max())


def test_constants_are_the_minimax_fit():
    c, best = _lawson_fit()
    c0, c1, c2, c3 = (float(x) for x in _coeffs())
    assert c0 == 1.0
    # the kernel's constants are the fit rounded to float32
    assert np.allclose([c1, c2, c3], c, rtol=1e-5, atol=0)
    f = np.linspace(-0.5, 0.5, 4001)
    mine = np.abs((1 + c1 * f + c2 * f ** 2 + c3 * f ** 3) / np.exp2(f) - 1).max()
    assert best < 1.02e-4 and mine <= 1.001 * best


def test_relative_error_over_the_softmax_range():
    x = np.linspace(-120.0, 8.0, 2_000_001).astype(np.float32)
    got = _exp2_fma(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(got / ref - 1.0)
    assert rel.max() < 1.5e-4


def test_reduction_is_exact_at_integers_and_half_points():
    x = np.arange(-100, 9).astype(np.float32)
    c0 = _coeffs()[0]
    # at integer x, f = 0 and the result is c0 * 2^n exactly
    assert np.array_equal(_exp2_fma(x), (c0 * np.exp2(x.astype(np.float64))).astype(np.float32))
    h = (np.arange(-50, 8) + 0.5).astype(np.float32)
    assert np.all(np.abs(_exp2_fma(h) / np.exp2(h.astype(np.float64)) - 1) < 1.5e-4)


def test_masked_scores_give_exact_zero():
    x = np.array([-np.inf, -1e30, -200.0, -127.0], np.float32)
    out = _exp2_fma(x)
    assert np.all(out == 0.0) and not np.any(np.signbit(out))
    # just above the clamp the result stays a tiny non-negative number, never NaN
    y = _exp2_fma(np.array([-126.9, -126.5, -126.0], np.float32))
    assert np.all(np.isfinite(y)) and np.all(y >= 0) and np.all(y < 2e-38)
