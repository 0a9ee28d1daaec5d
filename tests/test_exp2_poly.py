"""The kernel's FMA-pipe exp2 (csrc/exp2_fma.cuh) against fp64 exp2, on CPU.

The device routine reduces x to 2^round(x) * 2^f with f in [-1/2, 1/2] by the
1.5*2^23 rounding trick, evaluates a cubic for 2^f with fused multiply-adds,
and adds round(x) to the exponent field.  This test replays those steps in
fp32 (fused multiply-add emulated exactly: a fp32 product is exact in fp64)
with the coefficients parsed from the header, and checks the relative error
bound the kernel relies on, the clamp, and that the fitting script reproduces
the coefficients.
"""
import os
import re
import subprocess
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "causal_gqa_attention_03_b200", "csrc", "exp2_fma.cuh")
FIT = os.path.join(ROOT, "causal_gqa_attention_03_b200", "csrc", "fit_exp2_poly.py")


def coefficients():
    text = open(HEADER).read()
    vals = {}
    for name in ("c0", "c1", "c2", "c3", "kRound", "kMin"):
        m = re.search(rf"static constexpr float {name} = ([-0-9.eE+]+)f;", text)
        assert m, name
        vals[name] = np.float32(float(m.group(1)))
    return vals


def fma32(a, b, c):
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def exp2_device_model(x):
    k = coefficients()
    x = np.maximum(x.astype(np.float32), k["kMin"])
    t = (x + k["kRound"]).astype(np.float32)
    j = (t - k["kRound"]).astype(np.float32)
    f = fma32(j, np.float32(-1.0) * np.ones_like(j), x)
    p = fma32(np.full_like(f, k["c3"]), f, np.full_like(f, k["c2"]))
    p = fma32(p, f, np.full_like(f, k["c1"]))
    p = fma32(p, f, np.full_like(f, k["c0"]))
    bits = (p.view(np.uint32).astype(np.uint64) + (t.view(np.uint32).astype(np.uint64) << 23))
    return (bits & 0xFFFFFFFF).astype(np.uint32).view(np.float32)


def test_relative_error_bound_over_the_softmax_range():
    # x - m lies in [-inf, 8] under the lazy-rescale threshold of 2^8
    x = np.linspace(-125.0, 8.0, 4_000_001, dtype=np.float64).astype(np.float32)
    got = exp2_device_model(x).astype(np.float64)
    want = np.exp2(x.astype(np.float64))
    rel = np.abs(got / want - 1.0)
    assert rel.max() < 1.0e-4, rel.max()


def test_integers_and_half_integers():
    x = np.arange(-120, 9, 0.5, dtype=np.float32)
    got = exp2_device_model(x).astype(np.float64)
    assert np.all(np.abs(got / np.exp2(x.astype(np.float64)) - 1.0) < 1.0e-4)


def test_clamp_below_range_stays_tiny_and_positive():
    x = np.array([-126.0, -200.0, -1e6, -np.inf], dtype=np.float32)
    got = exp2_device_model(x)
    assert np.all(np.isfinite(got)) and np.all(got >= 0) and np.all(got < 2.0 ** -125)


def test_fit_script_reproduces_the_header_coefficients():
    out = subprocess.run([sys.executable, FIT], capture_output=True, text=True, check=True).stdout
    k = coefficients()
    for name in ("c0", "c1", "c2", "c3"):
        m = re.search(rf"{name} = ([-0-9.eE+]+)f", out)
        assert m and np.float32(float(m.group(1))) == k[name], (name, out)
