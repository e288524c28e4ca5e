"""Host checks of the arithmetic the kernels hard-code.

The score pass computes one exponential in eight on the FMA pipe
(`exp2_fma` in score_kernel.cu): 2^x = 2^n 2^f with n = round(x) and a
quartic for 2^f on [-1/2, 1/2]. This test reads the quartic's coefficients
from the kernel source and evaluates the same steps in fp32 (each Horner
step rounded once, as a fused multiply-add rounds) against the exact 2^x:
the relative error stays within the bound the kernel's comment states.
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
