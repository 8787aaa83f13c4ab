"""The FMA-pipe exp2 of the attention kernel (degree 3) and of the mask
score kernel (degree 5): the committed coefficients come from their
generator (Remez exchange), and each kernel's float32 step sequence (clamp,
round by adding 1.5*2^23, polynomial, exponent add) stays within 1e-4
(degree 3) and 3e-7 (degree 5) relative of exp2 over the range the kernels
use."""
import os
import re
import subprocess
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "video_transformers_b200", "csrc")


def coeffs():
    src = open(os.path.join(CSRC, "exp2_poly.h")).read()
    return [np.float32(float(v)) for v in re.findall(r"kExp2Poly\d = ([0-9eE.+-]+)f;", src)]


def test_header_is_generated():
    out = subprocess.run([sys.executable, "gen_exp2_poly.py"], cwd=CSRC, capture_output=True, text=True).stdout
    assert out == open(os.path.join(CSRC, "exp2_poly.h")).read()


def fma_pipe_exp2(x):
    c0, c1, c2, c3 = coeffs()
    x = np.maximum(x.astype(np.float32), np.float32(-126.0))
    t = (x + np.float32(12582912.0)).astype(np.float32)
    n = (t - np.float32(12582912.0)).astype(np.float32)
    f = (x - n).astype(np.float32)
    p = (c3 * f + c2).astype(np.float32)
    p = (p * f + c1).astype(np.float32)
    p = (p * f + c0).astype(np.float32)
    bits = (p.view(np.uint32) + (t.view(np.uint32) << np.uint32(23))).astype(np.uint32)
    return bits.view(np.float32)


def test_relative_error_bound():
    x = np.concatenate([np.linspace(-125.0, 20.0, 1_000_001), np.random.default_rng(0).uniform(-30, 11, 200_000)])
    got = fma_pipe_exp2(x).astype(np.float64)
    want = np.exp2(x.astype(np.float32).astype(np.float64))
    assert np.abs(got / want - 1).max() < 1e-4


def test_clamp_gives_tiny_not_zero():
    v = fma_pipe_exp2(np.array([-1000.0, -126.0]))
    assert np.all(v >= 0) and np.all(v < 2.0 ** -125)


def coeffs5():
    src = open(os.path.join(CSRC, "exp2_poly.h")).read()
    return [np.float32(float(v)) for v in re.findall(r"kExp2Poly5_\d = ([0-9eE.+-]+)f;", src)]


def fma_pipe_exp2_d5(x):
    c = coeffs5()
    assert len(c) == 6
    x = np.maximum(x.astype(np.float32), np.float32(-126.0))
    t = (x + np.float32(12582912.0)).astype(np.float32)
    n = (t - np.float32(12582912.0)).astype(np.float32)
    f = (x - n).astype(np.float32)
    p = (c[5] * f + c[4]).astype(np.float32)
    for cj in (c[3], c[2], c[1], c[0]):
        p = (p * f + cj).astype(np.float32)
    bits = (p.view(np.uint32) + (t.view(np.uint32) << np.uint32(23))).astype(np.uint32)
    return bits.view(np.float32)


def test_degree5_relative_error_bound():
    """The score kernel's block log-sum-exp feeds the level thresholds,
    which need the masses to about 1e-6: its FMA-pipe exp2 must stay near
    the special-function unit's own accuracy."""
    x = np.concatenate([np.linspace(-125.0, 0.0, 1_000_001), np.random.default_rng(1).uniform(-40, 0, 200_000)])
    got = fma_pipe_exp2_d5(x).astype(np.float64)
    want = np.exp2(x.astype(np.float32).astype(np.float64))
    assert np.abs(got / want - 1).max() < 3e-7
