"""The prefill kernel's FMA-pipe exponential, replayed bit for bit on the CPU.

The kernel computes a share of its exponentials as 2^x = 2^n * 2^f with n = rint(x), a
cubic for 2^f on [-1/2, 1/2] and n added to the exponent field. This test reads the cubic's
coefficients from the kernel source, replays the same fp32 operations in NumPy and bounds
the error against exp2 (relative 1e-4, far below bf16's 2^-9 rounding of P)."""
import os
import re

import numpy as np

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "differential_attention_v2_b200", "csrc", "prefill_sm100.cu")


def _coeffs():
    src = open(SRC).read()
    vals = {}
    for name in ("kExpC0", "kExpC1", "kExpC2", "kExpC3", "kExpShift"):
        m = re.search(name + r"\s*=\s*([0-9.eE+-]+)f", src)
        assert m, name
        vals[name] = np.float32(float(m.group(1)))
    return vals


def _kernel_exp2(x):
    c = _coeffs()
    x = np.maximum(x.astype(np.float32), np.float32(-126.0))
    t = (x + c["kExpShift"]).astype(np.float32)
    n = (t - c["kExpShift"]).astype(np.float32)
    f = (x - n).astype(np.float32)
    q = (c["kExpC3"] * f + c["kExpC2"]).astype(np.float32)
    q = (q * f + c["kExpC1"]).astype(np.float32)
    q = (q * f + c["kExpC0"]).astype(np.float32)
    bits = (q.view(np.uint32).astype(np.uint64) + (t.view(np.uint32).astype(np.uint64) << 23)) & 0xFFFFFFFF
    return bits.astype(np.uint32).view(np.float32)


def test_cubic_relative_error_on_reduced_range():
    c = _coeffs()
    f = np.linspace(-0.5, 0.5, 100001).astype(np.float32)
    q = (c["kExpC3"] * f + c["kExpC2"]).astype(np.float32)
    q = (q * f + c["kExpC1"]).astype(np.float32)
    q = (q * f + c["kExpC0"]).astype(np.float32)
    rel = np.abs(q.astype(np.float64) - np.exp2(f.astype(np.float64))) / np.exp2(f.astype(np.float64))
    assert rel.max() < 1e-4


def test_full_exp2_matches_within_bound():
    x = np.concatenate([np.linspace(-125.0, 8.0, 400001), np.random.default_rng(0).uniform(-30, 8, 100000)])
    y = _kernel_exp2(x.astype(np.float32)).astype(np.float64)
    ref = np.exp2(x.astype(np.float32).astype(np.float64))
    assert np.all(np.isfinite(y)) and np.all(y > 0)
    ok = ref > 1e-36  # below that the result is a denormal-range stand-in for ~0
    assert np.max(np.abs(y[ok] - ref[ok]) / ref[ok]) < 1e-4


def test_tiny_and_masked_range_stays_tiny():
    y = _kernel_exp2(np.array([-126.0, -200.0, -1e30, -np.inf], dtype=np.float32))
    assert np.all(np.isfinite(y)) and np.all(y >= 0) and np.all(y < 2e-38)


def test_integer_arguments_are_exact_powers_up_to_the_cubic():
    x = np.arange(-100, 9, dtype=np.float32)
    y = _kernel_exp2(x).astype(np.float64)
    np.testing.assert_allclose(y, np.exp2(x.astype(np.float64)) * float(_coeffs()["kExpC0"]), rtol=1e-7)
