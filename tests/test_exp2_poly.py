"""The software exp2 of the attention softmax (exp2_poly in attention_tc.cu).

It replaces ex2.approx for one score pair in eight so the MUFU and FMA pipes
share the work. Its result is rounded to bf16 (relative step 2^-8) right
after, so the bar is 1/16 of a bf16 half-step: 2^-9 / 16 = 1.2e-4 relative
error. (CUDA's exp2f is within 2 ulp, 2.4e-7; ex2.approx.ftz within about
2^-22.) These tests re-run the Remez fit, and evaluate the kernel's exact fp32
steps -- clamp to -126, range reduction by adding 1.5 * 2^23, Horner with fused
multiply-adds, exponent add -- over the whole argument range the kernel sees.
"""
import os
import re
import subprocess
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "vision_language_model_b200", "csrc")


def _coeffs():
    text = open(os.path.join(CSRC, "exp2_poly.cuh")).read()
    return [np.float32(float(v)) for v in re.findall(r"kExp2C\d = ([-+0-9.e]+)f;", text)]


def _fma32(a, b, c):
    # float64 holds a*b of two float32 exactly; one rounding to float32 = fused multiply-add
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def _exp2_poly_f32(x):
    c0, c1, c2, c3 = _coeffs()
    x = np.maximum(x.astype(np.float32), np.float32(-126.0))
    magic = np.float32(12582912.0)
    j = (x + magic).astype(np.float32)
    f = (x - (j - magic).astype(np.float32)).astype(np.float32)
    p = _fma32(_fma32(_fma32(np.full_like(f, c3), f, np.full_like(f, c2)), f, np.full_like(f, c1)), f,
               np.full_like(f, c0))
    bits = p.view(np.int32).astype(np.int64) + (j.view(np.int32).astype(np.int64) << 23)
    return (bits & 0xFFFFFFFF).astype(np.uint32).view(np.float32)


def test_header_matches_a_fresh_remez_fit():
    r = subprocess.run([sys.executable, os.path.join(CSRC, "fit_exp2_poly.py"), "--check"], capture_output=True,
                       text=True)
    assert r.returncode == 0, r.stdout + r.stderr
    assert len(_coeffs()) == 4


def test_relative_error_over_the_softmax_range():
    x = np.concatenate([np.linspace(-126.0, 8.0, 2_000_001, dtype=np.float32),
                        np.float32(np.arange(-126, 9)),                  # exact integers
                        np.float32(np.arange(-126, 8)) + np.float32(0.5)])  # rounding ties
    got = _exp2_poly_f32(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    normal = x >= -125.0  # results at least 2^-125: normal fp32 numbers
    rel = np.abs(got - ref)[normal] / ref[normal]
    assert rel.max() <= 2.0 ** -9 / 16, rel.max()
    # below that the result is within 2^-125 of the truth: nothing next to the
    # row's largest term, which is at least 1
    assert np.abs(got - ref)[~normal].max() <= 2.0 ** -125


def test_special_values():
    got = _exp2_poly_f32(np.array([0.0, 1.0, -1.0, 8.0, -300.0], dtype=np.float32)).astype(np.float64)
    np.testing.assert_allclose(got[:4], [1.0, 2.0, 0.5, 256.0], rtol=1e-4)
    assert 0.0 < got[4] < 1e-37  # clamped: never wraps to a large value
