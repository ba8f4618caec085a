"""Pins for the oracle's number-format decoders/encoders and its SiLU.

Every expected value comes from tests/golden/formats.txt (hand-fixed, with the passage that
fixes each format), from a closed form, or from an independent library routine (torch's
float8_e4m3fn conversion), never from the oracle itself.
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle

GOLD = os.path.join(os.path.dirname(__file__), "golden", "formats.txt")


def _rows(kind):
    out = []
    for line in open(GOLD):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        parts = line.split()
        if parts[0] == kind:
            out.append(parts[1:])
    assert out, kind
    return out


def test_int4_hand_packed_words():
    for word, *vals in _rows("int4"):
        w = int(word, 16)
        assert [oracle.int4(w, j) for j in range(8)] == [int(v) for v in vals], word


def test_bf16_pins():
    for bits, val in _rows("bf16"):
        assert oracle.bf16(int(bits, 16)) == float(val)


def test_f16_pins_and_torch():
    for bits, val in _rows("f16"):
        assert oracle.f16(int(bits, 16)) == float(val)
    # every finite fp16 pattern against torch's decoder (library routine)
    pats = np.arange(0, 1 << 16, dtype=np.uint16)
    ref = torch.from_numpy(pats.view(np.int16).copy()).view(torch.float16).double().numpy()
    for b in list(range(0, 1 << 16, 97)) + [0x7BFF, 0xFBFF, 0x0001, 0x8001, 0x03FF]:
        if (b >> 10) & 31 == 31:
            continue
        assert oracle.f16(b) == ref[b], hex(b)


def test_e4m3_decode_pins_and_all_codes_vs_torch():
    for bits, val in _rows("e4m3"):
        assert oracle.e4m3(int(bits, 16)) == float(val)
    codes = torch.arange(256, dtype=torch.int16).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    for c in range(256):
        got = oracle.e4m3(c)
        if np.isnan(ref[c]):
            assert math.isnan(got), hex(c)
        else:
            assert got == ref[c], hex(c)


def test_e4m3_encode_pins():
    for val, bits in _rows("enc"):
        assert oracle.e4m3_encode(float(val)) == int(bits, 16), val


def test_e4m3_encode_vs_torch_in_range():
    rng = np.random.default_rng(0)
    xs = np.concatenate([
        rng.normal(0, 1, 4000), rng.normal(0, 100, 2000), rng.uniform(-448, 448, 2000),
        rng.uniform(-0.02, 0.02, 2000),
        # all exact midpoints between neighbouring finite codes (ties)
        0.5 * (np.array([oracle.e4m3(c) for c in range(0, 0x7E)]) +
               np.array([oracle.e4m3(c) for c in range(1, 0x7F)])),
    ]).astype(np.float32)
    xs = xs[np.abs(xs) <= 448]
    ref = torch.from_numpy(xs).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([oracle.e4m3_encode(float(v)) for v in xs], np.uint8)
    # torch keeps the sign of zero results; so does the oracle
    assert np.array_equal(got, ref)


def test_silu_closed_forms():
    # sigmoid(x) = (1 + tanh(x/2)) / 2, so SiLU(x) = x (1 + tanh(x/2)) / 2
    # (the tanh form cancels for very negative x, hence the looser bound there)
    for g in [-20.0, -3.0, -1.0, -0.25, 0.0, 0.5, 1.0, 2.0, 7.5]:
        rel = 1e-6 if g < -10 else 1e-14
        assert oracle.silu(g) == pytest.approx(g * (1 + math.tanh(g / 2)) / 2, rel=rel, abs=1e-300)
    assert oracle.silu(math.log(3.0)) == pytest.approx(0.75 * math.log(3.0), rel=1e-15)
    assert oracle.silu(-1000.0) == 0.0
    assert oracle.silu(1000.0) == 1000.0
