"""The FMA-pipe 2^x used for one softmax exponential pair in four: its
constants come from the committed fit, and the float32 evaluation (range
reduction + cubic + exponent add) stays within 1e-4 relative error of exp2."""
import os
import re
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "gqa_attention_rope_b200", "csrc")
sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))
import fit_exp2_poly as F  # noqa: E402


def kernel_coefficients():
    src = open(os.path.join(CSRC, "ptx.cuh")).read()
    body = src[src.index("float ex2_poly(float x)"):]
    body = body[:body.index("return __int_as_float")]
    vals = [float(v) for v in re.findall(r"([0-9]\.[0-9]+)f", body)]
    # fmaf(f, c3, c2); fmaf(p, f, c1); fmaf(p, f, c0)
    c3, c2, c1, c0 = vals[0], vals[1], vals[2], vals[3]
    return np.array([c0, c1, c2, c3])


def emulate(x: np.ndarray, c: np.ndarray) -> np.ndarray:
    x = np.maximum(x.astype(np.float32), np.float32(-126.0))
    magic = np.float32(12582912.0)
    t = (x + magic).astype(np.float32)
    f = (x - (t - magic).astype(np.float32)).astype(np.float32)
    c = c.astype(np.float32)
    p = (f * c[3] + c[2]).astype(np.float32)
    p = (p * f + c[1]).astype(np.float32)
    p = (p * f + c[0]).astype(np.float32)
    n = t.view(np.int32) - magic.view(np.int32)
    return (p.view(np.int32) + (n << 23)).view(np.float32)


def test_kernel_constants_are_the_fit():
    fitted = F.fit()
    assert np.allclose(kernel_coefficients(), fitted, rtol=2e-7, atol=0)


def test_fit_error_bound():
    assert F.max_rel_error(F.fit()) < 8e-5


def test_float32_evaluation_error():
    c = kernel_coefficients()
    x = np.linspace(-60.0, 8.0, 1_000_001)
    got = emulate(x, c).astype(np.float64)
    ref = np.exp2(x.astype(np.float32).astype(np.float64))
    assert np.max(np.abs(got / ref - 1.0)) < 1e-4
    # exact-looking points and the clamp
    assert abs(emulate(np.array([0.0]), c)[0] - 1.0) < 1e-4
    assert emulate(np.array([-np.inf]), c)[0] < 2.0 ** -125
    assert emulate(np.array([-1000.0]), c)[0] >= 0.0
