"""The FMA-pipe exp2 the 8-bit kernel uses for 3/8 of its softmax
exponentials (the rest run on ex2.approx).

Checks that the coefficients in the kernel source are the ones the committed
fitting script produces (Remez exchange on the relative error of 2^f over
[-1/2, 1/2]) and that the kernel's steps, replayed in float32, stay within the
fit's error bound against exact 2^x over the range the kernels use it on.
"""
import os
import re
import subprocess
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "exact_attention_134_b200", "csrc")


def _kernel_coeffs():
    text = open(os.path.join(CSRC, "sm100_ptx.cuh")).read()
    body = text[text.index("float2 exp2_poly2"):]
    return [int(h, 16) for h in re.findall(r"__uint_as_float\((0x[0-9a-f]{8})u\)", body)[:4]]


def test_coefficients_match_the_fit():
    out = subprocess.run([sys.executable, os.path.join(CSRC, "exp2_poly_fit.py")],
                         capture_output=True, text=True, check=True).stdout
    fitted = [int(h, 16) for h in re.findall(r"'(0x[0-9a-f]+)'", out)]
    assert fitted == _kernel_coeffs()


def _replay(x):
    """The kernel's steps in float32 (FMA replaced by multiply-add in float64,
    rounded once to float32)."""
    f32 = np.float32
    c = [np.uint32(h).view(np.float32) for h in _kernel_coeffs()]
    x = np.maximum(x.astype(f32), f32(-125.0))
    t = (x + f32(12582912.0)).astype(f32)
    j = (t - f32(12582912.0)).astype(f32)
    f = (x - j).astype(f32)
    fma = lambda a, b, d: (a.astype(np.float64) * b + d).astype(f32)  # noqa: E731
    p = fma(f, c[3], c[2])
    p = fma(p, f, c[1])
    p = fma(p, f, c[0])
    bits = p.view(np.uint32) + (t.view(np.uint32) << np.uint32(23))
    return bits.view(np.float32)


def test_replay_error_bound():
    x = np.concatenate([np.linspace(-125, 8, 2_000_001), np.arange(-125, 9) + 0.5,
                        np.arange(-125, 9).astype(np.float64)]).astype(np.float32)
    y = _replay(x).astype(np.float64)
    rel = np.abs(y / np.exp2(x.astype(np.float64)) - 1.0)
    assert rel.max() < 8e-5


def test_clamp_below_minus_125():
    y = _replay(np.array([-200.0, -1e30, -126.0, -125.0], dtype=np.float32)).astype(np.float64)
    assert np.all(np.abs(y / 2.0 ** -125 - 1) < 8e-5)
