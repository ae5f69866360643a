"""The kernel's polynomial 2^x (used for part of the softmax exponentials),
emulated step by step in float32 on the host, against numpy's exp2: relative
error below 2^-13 over the range the kernel feeds it, far under the 2^-9 of the
bf16 P it produces.  Constants are read from the kernel source."""
import os
import re

import numpy as np

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "exact_io_aware_72_b200", "csrc", "attn_fwd_kernel.cuh")


def constants():
    text = open(SRC).read()
    get = lambda name: np.float32(float(re.search(rf"{name}\s*=\s*([-0-9.eE]+)f", text).group(1)))
    return [get(f"kExp2Poly{i}") for i in range(4)], get("kRoundMagic")


def poly_exp2(x):
    (q0, q1, q2, q3), magic = constants()
    x = np.maximum(x.astype(np.float32), np.float32(-125.0))
    t = (x + magic).astype(np.float32)
    n = (t - magic).astype(np.float32)
    f = (x - n).astype(np.float32)
    r = (f * q3 + q2).astype(np.float32)
    r = (f * r + q1).astype(np.float32)
    r = (f * r + q0).astype(np.float32)
    bits = r.view(np.uint32) + (t.view(np.uint32) << np.uint32(23))
    return bits.view(np.float32)


def test_relative_error_bound():
    x = np.linspace(-120.0, 8.5, 2_000_001, dtype=np.float64)
    got = poly_exp2(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float32).astype(np.float64))
    rel = np.abs(got / ref - 1.0)
    assert rel.max() < 2.0 ** -13, rel.max()


def test_masked_and_tiny_inputs_stay_tiny_and_positive():
    x = np.array([-np.inf, -1e30, -500.0, -125.0, -124.5], dtype=np.float32)
    got = poly_exp2(x)
    assert np.all(got > 0) and np.all(got < 2.0 ** -123)


def test_integers_and_halves():
    x = np.arange(-60, 9, 0.5)
    got = poly_exp2(x).astype(np.float64)
    assert np.max(np.abs(got / np.exp2(x) - 1)) < 2.0 ** -13
