"""Error bound of the FMA-pipe exp2 used for a share of the softmax exponentials in
the tcgen05 kernels (csrc/softmax_math.cuh, exp2_fma): the float32 steps are emulated
in NumPy and compared with exp2 in float64.  The bound (1e-4 relative) is well below
the bf16 rounding (2^-8 relative step) that every P value gets right after."""
import os
import re
import subprocess
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
KERNEL = os.path.join(ROOT, "video_dit_dynamic_gilbert_b200", "csrc", "softmax_math.cuh")
GEN = os.path.join(ROOT, "video_dit_dynamic_gilbert_b200", "csrc", "gen_exp2_poly.py")


def _kernel_coeffs():
    src = open(KERNEL).read()
    body = src[src.index("float exp2_fma("):]
    body = body[:body.index("}")]
    return [float(v) for v in re.findall(r"([0-9.]+e[-+][0-9]+)f", body)]


def _fma32(a, b, c):
    return np.float32(np.float64(a) * np.float64(b) + np.float64(c))


def _exp2_fma(x):
    x = np.maximum(np.float32(x), np.float32(-125.0))
    j = np.float32(x + np.float32(12582912.0))
    f = np.float32(x - np.float32(j - np.float32(12582912.0)))
    c3, c2, c1, c0 = [np.float32(v) for v in _kernel_coeffs()]
    p = _fma32(_fma32(_fma32(c3, f, c2), f, c1), f, c0)
    bits = (p.view(np.int32).astype(np.int64) + (j.view(np.int32).astype(np.int64) << 23)) & 0xFFFFFFFF
    return bits.astype(np.uint32).view(np.float32)


def test_coefficients_match_generator():
    out = subprocess.run([sys.executable, GEN], capture_output=True, text=True, check=True).stdout
    gen = [float(v) for v in re.findall(r"= ([0-9.e+-]+)f", out)]
    assert len(gen) == 4
    assert [np.float32(v) for v in gen[::-1]] == [np.float32(v) for v in _kernel_coeffs()]


def test_relative_error_bound():
    g = np.random.default_rng(0)
    x = np.concatenate([np.linspace(-125, 8, 400001), g.uniform(-30, 8, 200000)]).astype(np.float32)
    got = _exp2_fma(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(got - ref) / ref
    assert rel.max() < 1e-4, rel.max()
    assert np.isfinite(got).all()


def test_underflow_clamps_to_tiny_positive():
    got = _exp2_fma(np.array([-200.0, -1e30, -np.inf], dtype=np.float32))
    assert (got > 0).all() and (got < 1e-37).all()
