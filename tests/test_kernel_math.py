"""Host checks of the arithmetic the kernels hard-code.

The score pass computes one exponential in eight on the FMA pipe
(`exp2_fma` in score_kernel.cu): 2^x = 2^n 2^f with n = round(x) and a
quartic for 2^f on [-1/2, 1/2]. This test reads the quartic's coefficients
from the kernel source and evaluates the same steps in fp32 (each Horner
step rounded once, as a fused multiply-add rounds) against the exact 2^x:
the relative error stays within the bound the kernel's comment states. It
also re-derives the coefficients: they are the minimax fit of the relative
error (Remez exchange, degree 4 on [-1/2, 1/2], in fp64), rounded to fp32.
"""
import os
import re

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "..", "rolling_kv_cache_b200", "csrc", "score_kernel.cu")


def _coefficients():
    text = open(SRC).read()
    body = text[text.index("float exp2_fma(float x)"):]
    body = body[:body.index("\n}\n")]
    lead = re.search(r"float p = ([0-9.eE+-]+)f;", body).group(1)
    rest = re.findall(r"p = fmaf\(p, f, ([0-9.eE+-]+)f\);", body)
    return [np.float32(float(c)) for c in [lead] + rest]   # highest degree first


def _exp2_fma(x):
    """The kernel's steps, vectorised, in fp32."""
    x = np.maximum(np.asarray(x, dtype=np.float32), np.float32(-126.0))
    magic = np.float32(12582912.0)
    t = (x + magic).astype(np.float32)
    f = (x - (t - magic).astype(np.float32)).astype(np.float32)
    c = _coefficients()
    p = np.full_like(f, c[0])
    for ck in c[1:]:
        p = (p.astype(np.float64) * f.astype(np.float64) + np.float64(ck)).astype(np.float32)
    n = (t.view(np.int32).astype(np.int64) - 0x4B400000).astype(np.int64)
    bits = (p.view(np.uint32).astype(np.int64) + (n << 23)) & 0xFFFFFFFF
    return bits.astype(np.uint32).view(np.float32)


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
