"""The softmax kernel evaluates a quarter of its exp2 terms with a polynomial
on the FMA pipe (exp2_poly2 in csrc/sm100_ptx.cuh). Replays that arithmetic
in float32 with numpy (shifter rounding, Horner, exponent-bit add) using the
constants parsed from the header, and checks it against numpy's exp2 over the
whole range the kernel feeds it (x <= 8, clamped at -126)."""
import os
import re

import numpy as np

HDR = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "video_diffusion_hybrid_block_b200", "csrc", "sm100_ptx.cuh")


def coeffs():
    text = open(HDR).read()
    c = {int(m.group(1)): np.float32(float(m.group(2)))
         for m in re.finditer(r"kExp2C(\d) = ([0-9.eE+-]+)f;", text)}
    return [c[i] for i in range(4)]


def exp2_poly_f32(x):
    c0, c1, c2, c3 = coeffs()
    x = np.maximum(np.asarray(x, np.float32), np.float32(-126.0))
    sh = np.float32(12582912.0)
    t = (x + sh).astype(np.float32)
    j = (t - sh).astype(np.float32)
    f = (x - j).astype(np.float32)
    q = (c3 * f + c2).astype(np.float32)
    q = (q * f + c1).astype(np.float32)
    q = (q * f + c0).astype(np.float32)
    bits = (q.view(np.uint32).astype(np.uint64) + (t.view(np.uint32).astype(np.uint64) << 23)) & 0xFFFFFFFF
    return bits.astype(np.uint32).view(np.float32)


def test_poly_matches_exp2_relative():
    x = np.concatenate([np.linspace(-125.9, 8.0, 400001, dtype=np.float32),
                        np.arange(-125, 9, dtype=np.float32)])
    got = exp2_poly_f32(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    assert np.max(np.abs(got / ref - 1)) < 1.5e-4


def test_poly_clamps_far_negative_and_masked():
    got = exp2_poly_f32(np.array([-1e30, -np.inf, -300.0], np.float32))
    assert np.all(np.isfinite(got)) and np.all(got >= 0) and np.all(got < 1e-37)
