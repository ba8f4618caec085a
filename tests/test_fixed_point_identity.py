"""The integer identity the decode-sized W4A16 GEMM relies on, checked on the CPU.

That GEMM multiplies INT4 weights by 16-bit fixed-point activations on the int8 tensor cores:
the weight q in [-8, 7] enters as the byte q + 8 (unsigned), the activation X in
[-kFixMax, kFixMax] as two signed bytes hi = (X + 128) >> 8 and lo = X - 256 hi, and one
32-K group gives the integer sums D_hi = sum (q+8) hi and D_lo = sum (q+8) lo.  The group's
exact dot product is then recovered in fp32 without an integer-to-float conversion:
t = 256 D_hi + D_lo + (kFixBias - 8 sum X), read as fp32 bits, minus 1.5 * 2^23.  This holds
exactly while |sum q X| < 2^22, which kFixMax = 16383 guarantees for a 32-K group.

The constants are read from the library's internal header; the arithmetic here is written
from the statement above (numpy, exact integers), not taken from the kernel.
"""
import os
import re

import numpy as np

HDR = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "quantized_mixture_experts_softmax_b200", "csrc", "internal.h")


def _const(name):
    m = re.search(rf"{name}\s*=\s*(0x[0-9A-Fa-f]+|[0-9.]+f?)\s*;", open(HDR).read())
    assert m, name
    v = m.group(1)
    return int(v, 16) if v.startswith("0x") else (float(v.rstrip("f")) if "." in v else int(v))


FIX_MAX, FIX_BIAS, FIX_BIAS_F = _const("kFixMax"), _const("kFixBias"), _const("kFixBiasF")
G = 32  # K per group (one int8 MMA)


def _group_result(q, X):
    """What the GEMM computes for one 32-K group, step by step, in exact integer / fp32 terms."""
    q = np.asarray(q, np.int64)
    X = np.asarray(X, np.int64)
    u = q + 8                                     # weight byte, unsigned
    hi = (X + 128) >> 8                           # arithmetic shift
    lo = X - 256 * hi
    assert np.all((hi >= -128) & (hi <= 127)) and np.all((lo >= -128) & (lo <= 127))
    d_hi, d_lo = int((u * hi).sum()), int((u * lo).sum())   # the two s32 MMA results
    bias = FIX_BIAS - 8 * int(X.sum())           # the meta word of the group
    t = np.int64(256 * d_hi + d_lo + bias)
    assert -(1 << 31) <= t < (1 << 31)
    as_f32 = np.array([t], np.int32).view(np.float32)[0]
    return float(np.float32(as_f32) - np.float32(FIX_BIAS_F))


def test_constants_are_consistent():
    assert np.array([FIX_BIAS], np.int32).view(np.float32)[0] == np.float32(1.5 * 2 ** 23) == FIX_BIAS_F
    # the largest |sum q X| of a group stays below 2^22, the range where fp32 steps by 1 around 1.5*2^23
    assert G * 8 * FIX_MAX < 2 ** 22
    assert G * 8 * (FIX_MAX + 1) >= 2 ** 22  # and kFixMax is the largest value with that property


def test_identity_at_the_extremes():
    for qv in (-8, 7):
        for xv in (-FIX_MAX, FIX_MAX, 0, 1, -1, 127, 128, -128, -129, 255, 256):
            q = np.full(G, qv)
            X = np.full(G, xv)
            assert _group_result(q, X) == float(qv * xv * G), (qv, xv)
    # mixed signs reaching the largest magnitude
    q = np.array([-8] * G)
    X = np.array([FIX_MAX] * G)
    assert _group_result(q, X) == -8.0 * FIX_MAX * G


def test_identity_on_random_groups():
    rng = np.random.default_rng(0)
    for _ in range(20000):
        q = rng.integers(-8, 8, G)
        X = rng.integers(-FIX_MAX, FIX_MAX + 1, G)
        assert _group_result(q, X) == float((q * X).sum())


def test_identity_fails_beyond_the_range():
    """A planted violation: one step past 2^22 is no longer represented exactly (pins the bound)."""
    big = 2 ** 22 + 1
    t = np.int64(FIX_BIAS + big)
    assert float(np.array([t], np.int32).view(np.float32)[0] - np.float32(FIX_BIAS_F)) != big


def test_activation_quantization_bound():
    """X = rint(x / s) with s = max(amax, 1e-30) / kFixMax: |X| <= kFixMax and the error of
    X s against x is at most s / 2 (in the precision it is taken: fp32 on the device)."""
    rng = np.random.default_rng(1)
    x = (rng.standard_normal(128) * 3).astype(np.float32)
    s = np.float32(max(np.abs(x).max(), np.float32(1e-30)) / np.float32(FIX_MAX))
    X = np.rint(x / s).astype(np.int64)
    assert np.abs(X).max() <= FIX_MAX
    assert np.all(np.abs(X * np.float64(s) - x.astype(np.float64)) <= 0.5 * np.float64(s) * (1 + 1e-6))
