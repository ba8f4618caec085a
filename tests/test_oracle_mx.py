"""Pins for the oracle's W4A8 functions: MXFP4 weights x FP8 activations in 32-groups.

Source: the Humming issue "[Performance] W4A8 MoE GEMM significantly slower than W4A16 on
H200", opening report (weights MXFP4, activations FP8 with group size 32 along K).  Expected
values come from tests/golden/formats.txt (hand-worked), from closed forms written here
independently of the oracle's search loops, from torch's float8_e4m3fn / float8_e8m0fnu
conversions, and from a dense every-expert-then-mask formulation in torch float64.
"""
import math

import numpy as np
import torch

import oracle
import synth
from test_oracle_formats import _rows


# ------------------------------------------------------------------ element and scale formats
def test_e2m1_all_codes_hand_table():
    rows = _rows("e2m1")
    assert len(rows) == 16
    for code, val in rows:
        v = oracle.e2m1(int(code, 16))
        assert v == float(val) and math.copysign(1.0, v) == math.copysign(1.0, float(val)), code


def test_e8m0_all_codes_vs_torch():
    ref = torch.arange(256, dtype=torch.int16).to(torch.uint8).view(torch.float8_e8m0fnu).double().numpy()
    for c in range(255):
        assert oracle.e8m0(c) == ref[c] == 2.0 ** (c - 127), c
    assert math.isnan(oracle.e8m0(255)) and math.isnan(ref[255])


def _x_closed_form(amax: float) -> int:
    """Smallest X with amax <= 448 * 2^X, from frexp (amax = m * 2^e, m in [0.5, 1))."""
    if amax == 0.0:
        return -127
    m, e = math.frexp(amax)
    X = (e - 1) - 8 if 2.0 * m <= 1.75 else (e - 1) - 7
    return max(-127, min(127, X))


def _torch_codes(v: np.ndarray, X: int) -> np.ndarray:
    scaled = torch.from_numpy(v.astype(np.float64) * 2.0 ** (-X)).to(torch.float32)  # exact
    return scaled.to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def test_mx_quant_scale_pins():
    for amax, code in _rows("mxq"):
        a = np.float32(float(amax))
        v = np.zeros(32, np.float32)
        v[5] = a
        v[17] = -a / 2
        q, sc = oracle.mx_quant32(v)
        assert sc == int(code), amax
        assert sc == _x_closed_form(float(a)) + 127, amax


def test_mx_quant_random_groups_vs_closed_form_and_torch():
    rng = np.random.default_rng(0)
    for trial in range(400):
        mag = 10.0 ** rng.uniform(-35, 35)
        v = (rng.standard_normal(32) * mag).astype(np.float32)
        if trial % 7 == 0:
            v[rng.integers(0, 32, 5)] = 0.0
        if trial % 11 == 0:  # bf16-representable inputs, as the layer's x rows are
            v = (v.view(np.uint32) & 0xFFFF0000).view(np.float32)
        q, sc = oracle.mx_quant32(v)
        X = _x_closed_form(float(np.max(np.abs(v))))
        assert sc == X + 127
        assert np.array_equal(q, _torch_codes(v, X)), trial
        # nothing clipped: every code's value times the scale is within one E4M3 step of v
        assert np.all(np.abs(torch.from_numpy(q).view(torch.float8_e4m3fn).double().numpy()) <= 448.0)


def test_mx_quant_rounding_ties_to_even():
    # amax 1.75 -> X = -8, scaled values 256 * v: 272 (tie 256/288 -> 256), 304 (tie 288/320 ->
    # 320), 1.0625 * 256 = 272 again with a minus sign
    v = np.zeros(32, np.float32)
    v[0], v[1], v[2], v[3] = 1.75, 272 / 256, 304 / 256, -272 / 256
    q, sc = oracle.mx_quant32(v)
    assert sc == 119
    dec = torch.from_numpy(q).view(torch.float8_e4m3fn).double().numpy() * 2.0 ** -8
    assert list(dec[:4]) == [1.75, 1.0, 1.25, -1.0]
    assert np.array_equal(q, _torch_codes(v, -8))


# ------------------------------------------------------------------ layer
E2M1 = np.array([float(v) for _, v in _rows("e2m1")])


def _dequant(q: np.ndarray, sf: np.ndarray) -> np.ndarray:
    """[E, R, K/2] codes + [E, K/128, R, 4] scale codes -> float64 [E, R, K] (independent of
    the oracle: hand E2M1 table, torch's E8M0 decoder)."""
    E, R, K2 = q.shape
    codes = np.stack([q & 15, q >> 4], axis=-1).reshape(E, R, 2 * K2)
    s = torch.from_numpy(np.ascontiguousarray(sf)).view(torch.float8_e8m0fnu).double().numpy()
    s = s.transpose(0, 2, 1, 3).reshape(E, R, 2 * K2 // 32)
    return E2M1[codes] * np.repeat(s, 32, axis=2)


def _mx_torch(v: np.ndarray) -> np.ndarray:
    """Rows of fp32 values -> dequantized MX-FP8 values (32-groups along the last axis)."""
    n, K = v.shape
    g = v.reshape(n, K // 32, 32).astype(np.float32)
    amax = np.abs(g).max(axis=2).astype(np.float64)
    X = np.vectorize(_x_closed_form)(amax).astype(np.float64)
    scaled = torch.from_numpy(g.astype(np.float64) * np.exp2(-X)[:, :, None]).to(torch.float32)
    dec = scaled.to(torch.float8_e4m3fn).double().numpy()
    return (dec * np.exp2(X)[:, :, None]).reshape(n, K)


def _bf16_to_f64(x16: np.ndarray) -> np.ndarray:
    return (x16.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def test_w4a8_one_hot_layer():
    """One expert, one slot; a single input element, one gate / up / down weight each, placed in
    odd K positions (high nibbles) and with their own scale codes."""
    H = I = 128
    c0, j0, c1 = 5, 37, 70
    x = np.zeros((1, H), np.uint16)
    x[0, c0] = 0x3F80  # 1.0 -> group amax 1.0, X = -8, code e4m3(256) exact
    w13 = np.zeros((1, 2 * I, H // 2), np.uint8)
    w13_sf = np.full((1, H // 128, 2 * I, 4), 127, np.uint8)
    w2 = np.zeros((1, H, I // 2), np.uint8)
    w2_sf = np.full((1, I // 128, H, 4), 127, np.uint8)
    w13[0, j0, c0 // 2] = 0x4 << 4  # gate weight 2.0 (odd K index: high nibble)
    w13_sf[0, c0 // 128, j0, (c0 // 32) % 4] = 128  # x 2 -> 4.0
    w13[0, I + j0, c0 // 2] = 0x3 << 4  # up weight 1.5
    w2[0, c1, j0 // 2] = 0xA << 4  # down weight -1.0 (j0 odd)
    w2_sf[0, j0 // 128, c1, (j0 // 32) % 4] = 126  # x 1/2 -> -0.5
    ids = np.zeros((1, 1), np.int32)
    w = np.ones((1, 1), np.float32)
    out, hq = oracle.w4a8_tokens(x, ids, w, w13, w13_sf, w2, w2_sf, want_hq=True)
    g, u = 4.0, 1.5
    h = np.float32(g / (1.0 + math.exp(-g)) * u)
    hv = np.zeros((1, I), np.float32)
    hv[0, j0] = h
    hd = _mx_torch(hv)[0, j0]
    assert hq[0, 0, j0] == np.float32(hd) and np.count_nonzero(hq) == 1
    exp = np.zeros(H)
    exp[c1] = -0.5 * hd
    assert np.array_equal(out[0], exp)


def _layer_inputs(seed, T, H, I, E, k):
    x = synth.x_bf16(seed, T, H)
    ids, w, _ = oracle.route(synth.logits(seed, T, E), k)
    W = synth.mxfp4_weights(seed, H, I, range(E))
    return x, ids, w, W


def test_w4a8_dense_then_mask(seed=0):
    T, H, I, E, k = 6, 256, 256, 4, 2
    x, ids, w, W = _layer_inputs(seed, T, H, I, E, k)
    ref = oracle.w4a8_tokens(x, ids, w, W["w13"], W["w13_sf"], W["w2"], W["w2_sf"])
    W13 = _dequant(W["w13"], W["w13_sf"])
    W2 = _dequant(W["w2"], W["w2_sf"])
    xq = _mx_torch(_bf16_to_f64(x).astype(np.float32))
    out = np.zeros((T, H))
    for e in range(E):  # every expert on every token, then the routing mask
        G = xq @ W13[e].T
        h = (G[:, :I] / (1.0 + np.exp(-G[:, :I])) * G[:, I:]).astype(np.float32)
        Y = _mx_torch(h) @ W2[e].T
        for t in range(T):
            for s in range(k):
                if ids[t, s] == e:
                    out[t] += float(w[t, s]) * Y[t]
    scale = np.sqrt(np.mean(out ** 2))
    assert scale > 1e-3
    np.testing.assert_allclose(ref, out, rtol=1e-9, atol=1e-12 * scale)


def test_w4a8_weights_slice_by_expert():
    """The generator's per-expert slices reproduce the full tensors (the oracle regenerates
    single experts for full-size checks)."""
    full = synth.mxfp4_weights(3, 256, 128, range(5))
    part = synth.mxfp4_weights(3, 256, 128, [4, 1])
    for key in full:
        assert np.array_equal(part[key][0], full[key][4]) and np.array_equal(part[key][1], full[key][1])
    assert set(np.unique(full["w13_sf"])) <= set(synth.MX_SCALE_CODES)


def test_generator_expert_ids_as_numpy_int32():
    """Expert ids that come from numpy (np.unique of routing ids) give the same slices as
    Python ints, for experts whose flat offset exceeds 2^31."""
    for gen, H, I in ((synth.mxfp4_weights, 7168, 2048), (synth.w4a16_weights, 7168, 2048)):
        a = gen(0, H, I, np.array([383], np.int32))
        b = gen(0, H, I, [383])
        assert all(np.array_equal(a[k], b[k]) for k in a)


def test_w4a8_token_permutation_and_subsets():
    """Each token is computed on its own: permuting the tokens (rows of x, ids and weights)
    permutes the output rows bit for bit, and a token subset reproduces those rows exactly."""
    T, H, I, E, k = 7, 256, 128, 5, 2
    x, ids, w, W = _layer_inputs(4, T, H, I, E, k)
    full = oracle.w4a8_tokens(x, ids, w, W["w13"], W["w13_sf"], W["w2"], W["w2_sf"])
    perm = np.random.default_rng(1).permutation(T)
    permuted = oracle.w4a8_tokens(x[perm], ids[perm], w[perm], W["w13"], W["w13_sf"], W["w2"], W["w2_sf"])
    assert np.array_equal(permuted, full[perm])
    sub = np.array([5, 0, 3], np.int32)
    part = oracle.w4a8_tokens(x, ids, w, W["w13"], W["w13_sf"], W["w2"], W["w2_sf"], tokens=sub)
    assert np.array_equal(part, full[sub])
