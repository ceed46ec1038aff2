"""The kernel's FMA-pipe 2^x, simulated bit for bit in fp32 on the CPU.

Checks the constants in sm100_ptx.cuh against the fitting script, the
relative error against the exact 2^x over the range the softmax produces
(x <= 8 with the rescale threshold, down to masked -inf), and that masked
entries give exactly +0.
"""
import os
import re
import subprocess
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "exact_tiled_attention_45_b200", "csrc")


def _constants():
    text = open(os.path.join(CSRC, "sm100_ptx.cuh")).read()
    vals = {}
    for name in ("EXP2_C1", "EXP2_C2", "EXP2_C3", "ROUND_MAGIC"):
        m = re.search(rf"constexpr float {name} = ([0-9.eE+-]+)f;", text)
        vals[name] = np.float32(float(m.group(1)))
    return vals


def _kernel_exp2(x):
    c = _constants()
    f32 = np.float32
    x = np.maximum(x.astype(f32), f32(-127.0))
    y = (x + c["ROUND_MAGIC"]).astype(f32)
    jf = (y + (-c["ROUND_MAGIC"])).astype(f32)
    f = (jf * f32(-1.0) + x).astype(f32)
    p = (c["EXP2_C3"] * f + c["EXP2_C2"]).astype(f32)
    p = (p * f + c["EXP2_C1"]).astype(f32)
    p = (p * f + f32(1.0)).astype(f32)
    bits = (p.view(np.uint32) + (y.view(np.uint32) << np.uint32(23))).astype(np.uint32)
    return bits.view(np.float32)


def test_constants_match_the_fit():
    out = subprocess.run([sys.executable, os.path.join(CSRC, "fit_exp2_poly.py"), "3"], capture_output=True,
                         text=True, check=True).stdout
    fitted = [np.float32(float(v)) for v in re.findall(r"c\d = ([0-9.eE+-]+)", out)]
    c = _constants()
    assert fitted[0] == np.float32(1.0)
    assert [c["EXP2_C1"], c["EXP2_C2"], c["EXP2_C3"]] == fitted[1:]


def test_relative_error_over_the_softmax_range():
    x = np.concatenate([np.linspace(-126.0, 8.5, 2_000_001), np.arange(-126, 9).astype(np.float64)])
    x32 = x.astype(np.float32)
    got = _kernel_exp2(x32).astype(np.float64)
    exact = np.exp2(x32.astype(np.float64))
    rel = np.abs(got / exact - 1.0)
    assert rel.max() < 1.1e-4, rel.max()
    assert np.all(got > 0)


def test_masked_and_tiny_inputs():
    x = np.array([-np.inf, -1e30, -1000.0, -127.0, -200.0], dtype=np.float32)
    assert np.all(_kernel_exp2(x) == 0.0)
    x = np.linspace(-127.0, -125.0, 10001).astype(np.float32)
    got = _kernel_exp2(x)
    assert np.all(got >= 0) and np.all(np.isfinite(got))
    assert np.all(got <= np.exp2(x.astype(np.float64)) * (1 + 1.1e-4) + 1e-45)


def test_exact_at_integers():
    x = np.arange(-120, 9).astype(np.float32)
    assert np.array_equal(_kernel_exp2(x), np.exp2(x.astype(np.float64)).astype(np.float32))
