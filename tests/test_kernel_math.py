"""Host checks of the arithmetic the kernels hard-code.

The score pass computes a quarter of its exponentials on the FMA pipe
(`exp2_quartic2` in score_kernel.cu, packed f32x2 steps): 2^x = 2^n 2^f
with n = round(x) and a
quartic for 2^f on [-1/2, 1/2]. This test reads the quartic's coefficients
from the kernel source and evaluates the same steps in fp32 (each Horner
step rounded once, as a fused multiply-add rounds) against the exact 2^x:
the relative error stays within the bound the kernel's comment states. It
also re-derives the coefficients: they are the minimax fit of the relative
error (Remez exchange, degree 4 on [-1/2, 1/2], in fp64), rounded to fp32.

The attention's softmax takes a quarter of its exponentials from a cubic
(`exp2_cubic2` in attn_fwd.cu, packed f32x2 steps); the same checks pin
it against the degree-3 fit and its stated 7.5e-5 bound.
"""
import os
import re

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "..", "rolling_kv_cache_b200", "csrc", "score_kernel.cu")
ATTN_SRC = os.path.join(HERE, "..", "rolling_kv_cache_b200", "csrc", "attn_fwd.cu")


def _packed_coefficients(src, func):
    """Coefficients of a packed Horner polynomial `func` (highest degree
    first), as the source spells them: every make_float2(a, a) from the
    first `q =` step up to the return."""
    text = open(src).read()
    body = text[text.index(func):]
    body = body[body.index("float2 q ="):body.index("return")]
    vals = re.findall(r"make_float2\(([0-9.eE+-]+)f, ([0-9.eE+-]+)f\)", body)
    assert all(a == b for a, b in vals)          # both lanes carry the same constant
    return [np.float32(float(a)) for a, _ in vals]


def _coefficients():
    return _packed_coefficients(SRC, "float2 exp2_quartic2(float2 x)")


def _packed_exp2(x, coeffs):
    """The packed exponential's steps in fp32, one lane at a time (a packed
    f32x2 instruction rounds each lane as its scalar form does): clamp at
    -126, t = x + 1.5 * 2^23, n = t - 1.5 * 2^23, f = fma(n, -1, x),
    Horner in f, then t's low bits shifted into the exponent field."""
    x = np.maximum(np.asarray(x, dtype=np.float32), np.float32(-126.0))
    magic = np.float32(12582912.0)
    t = (x + magic).astype(np.float32)
    n = (t - magic).astype(np.float32)
    f = (n.astype(np.float64) * -1.0 + x.astype(np.float64)).astype(np.float32)   # one rounding
    q = np.full_like(f, coeffs[0])
    for ck in coeffs[1:]:
        q = (q.astype(np.float64) * f.astype(np.float64) + np.float64(ck)).astype(np.float32)
    bits = (q.view(np.uint32).astype(np.int64) + (t.view(np.uint32).astype(np.int64) << 23)) & 0xFFFFFFFF
    return bits.astype(np.uint32).view(np.float32)


def _exp2_fma(x):
    """The score pass's steps, vectorised, in fp32."""
    return _packed_exp2(x, _coefficients())


def test_exp2_fma_coefficients_present():
    assert len(_coefficients()) == 5


def test_exp2_fma_relative_error():
    # the range the score pass produces: s c - lse2 <= ~0, down to the clamp
    x = np.concatenate([np.linspace(-125.0, 1.0, 400001, dtype=np.float32),
                        np.linspace(-1.0, 1.0, 200001, dtype=np.float32)])
    got = _exp2_fma(x).astype(np.float64)
    want = np.exp2(x.astype(np.float64))
    rel = np.abs(got - want) / want
    assert rel.max() <= 3e-6, rel.max()


def test_exp2_fma_integers_and_clamp():
    # integer x: f = 0, so the result is the constant term scaled by 2^x
    x = np.arange(-125, 2, dtype=np.float32)
    got = _exp2_fma(x).astype(np.float64)
    assert np.all(np.abs(got / np.exp2(x.astype(np.float64)) - 1.0) <= 1e-6)
    # -inf and anything below the clamp give 2^-126 at most: negligible next to
    # the probabilities the pass sums
    tiny = _exp2_fma(np.array([-np.inf, -1000.0, -127.5], dtype=np.float32)).astype(np.float64)
    assert np.all((tiny >= 0.0) & (tiny <= 2.0 ** -125))


def _remez_relative(deg=4, lo=-0.5, hi=0.5, iters=40):
    """Minimax polynomial of degree `deg` for 2^f on [lo, hi] in relative
    error, by the Remez exchange algorithm: start from the Chebyshev
    extrema, solve p(x_i) / 2^x_i - 1 = (-1)^i E on deg + 2 reference
    points, move the points to the extrema of the new error, repeat until
    the reference stops moving. Returns (coefficients lowest first, |E|)."""
    n = deg + 2
    x = (lo + hi) / 2 - (hi - lo) / 2 * np.cos(np.pi * np.arange(n) / (n - 1))
    grid = np.linspace(lo, hi, 200001)
    for _ in range(iters):
        A = np.zeros((n, n))
        for i in range(n):
            A[i, :deg + 1] = x[i] ** np.arange(deg + 1) / np.exp2(x[i])
            A[i, deg + 1] = -(-1.0) ** i
        sol = np.linalg.solve(A, np.ones(n))
        c, E = sol[:deg + 1], sol[deg + 1]
        e = np.polyval(c[::-1], grid) / np.exp2(grid) - 1.0
        cuts = np.concatenate([[0], np.nonzero(np.diff(np.sign(e)))[0] + 1, [len(grid)]])
        ext = np.array([a + np.argmax(np.abs(e[a:b])) for a, b in zip(cuts[:-1], cuts[1:])])
        if len(ext) != n:
            break
        x_new = grid[ext]
        if np.allclose(x_new, x, atol=1e-9):
            break
        x = x_new
    return c, abs(E)


def test_exp2_fma_coefficients_are_the_minimax_fit():
    c, E = _remez_relative()
    assert 2.5e-6 < E < 2.7e-6              # the equioscillating relative error of the degree-4 fit
    src = np.array(_coefficients()[::-1], dtype=np.float32)   # lowest degree first
    fit = c.astype(np.float32)
    # each coefficient is the fp64 minimax coefficient rounded to fp32 (within one fp32 ulp)
    ulp = np.spacing(np.abs(fit))
    assert np.all(np.abs(src.astype(np.float64) - fit.astype(np.float64)) <= ulp), (src, fit)


def _cubic_coefficients():
    return _packed_coefficients(ATTN_SRC, "float2 exp2_cubic2(float2 x)")


def _exp2_cubic2(x):
    return _packed_exp2(x, _cubic_coefficients())


def test_attention_cubic_relative_error():
    assert len(_cubic_coefficients()) == 4
    # the softmax's arguments: s c - m c, at most the rescale threshold (8) above 0
    x = np.concatenate([np.linspace(-125.0, 8.0, 400001, dtype=np.float32),
                        np.linspace(-1.0, 1.0, 200001, dtype=np.float32)])
    got = _exp2_cubic2(x).astype(np.float64)
    want = np.exp2(x.astype(np.float64))
    rel = np.abs(got - want) / want
    assert rel.max() <= 7.5e-5 * 1.02, rel.max()
    tiny = _exp2_cubic2(np.array([-np.inf, -1000.0, -126.7], dtype=np.float32)).astype(np.float64)
    assert np.all((tiny >= 0.0) & (tiny <= 2.0 ** -125))


def test_attention_cubic_is_the_minimax_fit():
    c, E = _remez_relative(deg=3)
    assert 7.4e-5 < E < 7.6e-5
    src = np.array(_cubic_coefficients()[::-1], dtype=np.float32)   # lowest degree first
    fit = c.astype(np.float32)
    ulp = np.spacing(np.abs(fit))
    assert np.all(np.abs(src.astype(np.float64) - fit.astype(np.float64)) <= ulp), (src, fit)
