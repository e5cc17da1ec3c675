"""The FMA-pipe exp2 used by the softmax for a share of the score columns.

The device code (exp2_poly2 in sm100_ptx.cuh) is replayed step by step in
float32 arithmetic and compared with the exact 2^x: the relative error must
stay below 1e-4 on the whole input range the kernel feeds it (finite scores
relative to the running max, clamped at -125), far under the bf16 rounding
(2^-9) that P goes through next.  The constants are read from the header, and
must equal the Remez fit of exp2_poly_fit.py."""
import os
import re
import subprocess
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HDR = os.path.join(ROOT, "attention_forward_tmem_b200", "csrc", "sm100_ptx.cuh")
FIT = os.path.join(ROOT, "attention_forward_tmem_b200", "csrc", "exp2_poly_fit.py")


def _coeffs():
    src = open(HDR).read()
    m = re.search(r"c0 = ([0-9.e+-]+)f, c1 = ([0-9.e+-]+)f, c2 = ([0-9.e+-]+)f, c3 = ([0-9.e+-]+)f", src)
    assert m, "coefficients not found in sm100_ptx.cuh"
    return [np.float32(v) for v in m.groups()]


def _fma32(a, b, c):
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def device_exp2(x):
    c0, c1, c2, c3 = _coeffs()
    x = np.maximum(x.astype(np.float32), np.float32(-125.0))
    shift = np.float32(12582912.0)
    t = (x + shift).astype(np.float32)
    r = (t - shift).astype(np.float32)
    f = (x - r).astype(np.float32)
    p = _fma32(f, np.full_like(f, c3), np.full_like(f, c2))
    p = _fma32(p, f, np.full_like(f, c1))
    p = _fma32(p, f, np.full_like(f, c0))
    bits = p.view(np.int32).astype(np.int64) + (t.view(np.int32).astype(np.int64) << 23)
    return (bits & 0xFFFFFFFF).astype(np.uint32).view(np.float32)


def test_relative_error_bound():
    x = np.concatenate([np.linspace(-125, 9, 2_000_001, dtype=np.float32),
                        np.float32([-0.5, 0.5, 0.0, 1e-8, -1e-8, 7.99, -124.6])])
    got = device_exp2(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(got - ref) / ref
    assert rel.max() < 1e-4, rel.max()
    assert np.all(np.isfinite(got)) and np.all(got > 0)


def test_clamp_below_range():
    """Very negative inputs give 2^-125-ish, never a wrapped exponent."""
    got = device_exp2(np.float32([-130.0, -1e6, -125.0]))
    assert np.all(got > 0) and np.all(got < 1e-37)


def test_constants_match_fit():
    out = subprocess.run([sys.executable, FIT], capture_output=True, text=True, check=True).stdout
    fit = [np.float32(float(m)) for m in re.findall(r"\(([0-9.]+e[+-][0-9]+)\)", out)]
    assert len(fit) == 4
    assert fit == _coeffs()
    assert float(re.search(r"error on \[-1/2, 1/2\]: ([0-9.e+-]+)", out).group(1)) < 1e-4
