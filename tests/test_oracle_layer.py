"""Pins for the oracle's W4A16 and block-FP8 layer arithmetic.

* One-hot probes on hand-packed weights read single dequantized weights back exactly, which
  pins the INT4 layout (nibble order, K-contiguous rows, scale per 32 K) and the e4m3
  block-scale indexing.
* Crafted single-weight layers pin the gate/up order, the SiLU and the down projection
  against closed forms.
* A dense "every expert for every token, then mask" formulation built from float64 torch
  matmuls on dequantized weights checks the routed per-token oracle on the tiny workload.
* Token-permutation invariance is checked bit-exactly.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import synth

BF16_ONE, BF16_HALF, F16_ONE = 0x3F80, 0x3F00, 0x3C00


def _dequant_w4(q, s):
    """[E,N,K/8] int32 + [E,N,K/32] bf16 -> float64 [E,N,K] (vectorised; layout pinned by
    test_gemm_one_hot_reads_hand_packed_weights)."""
    q = q.view(np.uint32)
    E, N, K8 = q.shape
    nib = np.stack([(q >> (4 * j)) & 0xF for j in range(8)], axis=-1).astype(np.int64)
    nib = np.where(nib >= 8, nib - 16, nib).reshape(E, N, K8 * 8)
    sc = torch.from_numpy(s.view(np.int16).copy()).view(torch.bfloat16).double().numpy()
    return nib * np.repeat(sc, 32, axis=2)


def test_gemm_one_hot_reads_hand_packed_weights():
    # N=3 output columns, K=32 (one scale group); hand-packed rows
    words = np.array([[0x76543210, 0xFEDCBA98, 0x0F1E2D3C, 0x00000008],
                      [0x11111111, 0x22222222, 0x88888888, 0x7FFFFFFF],
                      [0, 0, 0, 0x80000000]], np.uint32).view(np.int32)[None]
    scales = np.array([[0x3C00], [0x3F80], [0x3F00]], np.uint16)[None]  # 2^-7, 1, 0.5
    expect_q = [
        [0, 1, 2, 3, 4, 5, 6, 7, -8, -7, -6, -5, -4, -3, -2, -1, -4, 3, -3, 2, -2, 1, -1, 0, -8, 0, 0, 0, 0, 0, 0,
         0],
        [1] * 8 + [2] * 8 + [-8] * 8 + [-1] * 7 + [7],
        [0] * 31 + [-8],
    ]
    expect = np.array(expect_q, np.float64) * np.array([[2.0 ** -7], [1.0], [0.5]])
    for c in range(32):
        a = np.zeros((1, 32), np.uint16)
        a[0, c] = BF16_ONE
        out = oracle.w4a16_gemm(a, True, words, scales, np.array([0, 1], np.int32))
        assert out[0].tolist() == expect[:, c].tolist(), c
        a[0, c] = F16_ONE
        out = oracle.w4a16_gemm(a, False, words, scales, np.array([0, 1], np.int32))
        assert out[0].tolist() == expect[:, c].tolist(), c


def test_gemm_rows_follow_expert_offsets():
    a, w_q, w_s = synth.gemm_operands(3, 6, 64, 16)
    wq2 = np.concatenate([w_q, w_q[:, ::-1]], 0).copy()
    ws2 = np.concatenate([w_s, w_s[:, ::-1]], 0).copy()
    off = np.array([0, 2, 5], np.int32)  # rows 0-1 expert 0, rows 2-4 expert 1, row 5 none
    out = oracle.w4a16_gemm(a, True, wq2, ws2, off)
    W = _dequant_w4(wq2, ws2)
    A = torch.from_numpy(a.view(np.int16).copy()).view(torch.bfloat16).double().numpy()
    np.testing.assert_allclose(out[:2], A[:2] @ W[0].T, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(out[2:5], A[2:5] @ W[1].T, rtol=1e-12, atol=1e-12)
    assert np.all(out[5] == 0)


def _crafted_layer(H=32, I=32):
    """E=1 layer whose only nonzero weights are gate[0][0]=4*0.5, up[0][0]=1*0.5, down[0][0]=2*1."""
    w13_q = np.zeros((1, 2 * I, H // 8), np.uint32)
    w13_s = np.full((1, 2 * I, H // 32), BF16_HALF, np.uint16)
    w2_q = np.zeros((1, H, I // 8), np.uint32)
    w2_s = np.full((1, H, I // 32), BF16_ONE, np.uint16)
    w13_q[0, 0, 0] = 0x4       # gate row 0, K index 0: q=4, s=0.5 -> 2.0
    w13_q[0, I, 0] = 0x1       # up row 0 (= w13 row I), K index 0: q=1, s=0.5 -> 0.5
    w2_q[0, 0, 0] = 0x2        # down row 0, K index 0: q=2, s=1 -> 2.0
    return w13_q.view(np.int32), w13_s, w2_q.view(np.int32), w2_s


def test_gate_up_silu_down_closed_form():
    H = I = 32
    w13_q, w13_s, w2_q, w2_s = _crafted_layer(H, I)
    x = np.zeros((1, H), np.uint16)
    x[0, 0] = BF16_ONE
    out, h, g = oracle.w4a16_tokens(x, np.array([[0]], np.int32), np.array([[1.0]], np.float32), w13_q, w13_s,
                                    w2_q, w2_s, want_h=True, want_g=True)
    assert g[0, 0, 0] == 2.0 and g[0, 0, I] == 0.5 and np.count_nonzero(g) == 2
    silu2 = 1.0 + math.tanh(1.0)  # SiLU(2) = 2*sigmoid(2) = 1 + tanh(1)
    assert h[0, 0, 0] == pytest.approx(0.5 * silu2, rel=1e-15)
    assert np.count_nonzero(h) == 1
    assert out[0, 0] == pytest.approx(2.0 * 0.5 * silu2, rel=1e-15)  # down weight 2
    assert np.count_nonzero(out) == 1
    # a routing weight scales the whole output
    out2 = oracle.w4a16_tokens(x, np.array([[0]], np.int32), np.array([[0.25]], np.float32), w13_q, w13_s, w2_q,
                               w2_s)
    assert out2[0, 0] == pytest.approx(0.25 * 2.0 * 0.5 * silu2, rel=1e-15)


def _tiny_inputs(seed, T=16, H=256, I=128, E=8, k=2, zipf=0.0):
    x = synth.x_bf16(seed, T, H)
    lg = synth.logits(seed, T, E, zipf_s=zipf)
    ids, w32, _ = oracle.route(lg, k)
    W = synth.w4a16_weights(seed, H, I, range(E))
    return x, lg, ids, w32, W


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_dense_every_expert_then_mask_matches_routed(seed):
    T, H, I, E, k = 16, 256, 128, 8, 2
    x, lg, ids, w32, W = _tiny_inputs(seed, T, H, I, E, k)
    out = oracle.w4a16_tokens(x, ids, w32, W["w13_q"], W["w13_s"], W["w2_q"], W["w2_s"])
    X = torch.from_numpy(x.view(np.int16).copy()).view(torch.bfloat16).double()
    W13 = torch.from_numpy(_dequant_w4(W["w13_q"], W["w13_s"]))
    W2 = torch.from_numpy(_dequant_w4(W["w2_q"], W["w2_s"]))
    mask = torch.zeros(T, E, dtype=torch.float64)
    for t in range(T):
        for s in range(k):
            mask[t, ids[t, s]] = float(w32[t, s])
    dense = torch.zeros(T, H, dtype=torch.float64)
    for e in range(E):
        G = X @ W13[e].T                       # [T, 2I]
        Hh = torch.nn.functional.silu(G[:, :I]) * G[:, I:]
        dense += mask[:, e:e + 1] * (Hh @ W2[e].T)
    ref = dense.numpy()
    rms = np.sqrt(np.mean(ref ** 2))
    assert np.max(np.abs(out - ref)) <= 1e-12 * rms


def test_e1_k1_is_a_dense_ffn():
    T, H, I = 8, 256, 256
    x = synth.x_bf16(9, T, H)
    W = synth.w4a16_weights(9, H, I, [0])
    ids = np.zeros((T, 1), np.int32)
    w = np.ones((T, 1), np.float32)
    out = oracle.w4a16_tokens(x, ids, w, W["w13_q"], W["w13_s"], W["w2_q"], W["w2_s"])
    X = torch.from_numpy(x.view(np.int16).copy()).view(torch.bfloat16).double()
    W13 = torch.from_numpy(_dequant_w4(W["w13_q"], W["w13_s"]))[0]
    W2 = torch.from_numpy(_dequant_w4(W["w2_q"], W["w2_s"]))[0]
    G = torch.matmul(X, W13.T)
    ref = torch.matmul(torch.nn.functional.silu(G[:, :I]) * G[:, I:], W2.T).numpy()
    np.testing.assert_allclose(out, ref, rtol=1e-11, atol=1e-11 * np.abs(ref).max())


def test_token_permutation_invariance_bit_exact():
    T, H, I, E, k = 16, 256, 128, 8, 2
    x, lg, ids, w32, W = _tiny_inputs(4, T, H, I, E, k)
    perm = np.random.default_rng(1).permutation(T)
    out = oracle.w4a16_tokens(x, ids, w32, W["w13_q"], W["w13_s"], W["w2_q"], W["w2_s"])
    ids_p, w_p, _ = oracle.route(lg[perm], k)
    out_p = oracle.w4a16_tokens(x[perm], ids_p, w_p, W["w13_q"], W["w13_s"], W["w2_q"], W["w2_s"])
    assert np.array_equal(out[perm], out_p)


def test_token_subset_equals_full():
    T, H, I, E, k = 16, 256, 128, 8, 2
    x, lg, ids, w32, W = _tiny_inputs(5, T, H, I, E, k)
    full = oracle.w4a16_tokens(x, ids, w32, W["w13_q"], W["w13_s"], W["w2_q"], W["w2_s"])
    sub = oracle.w4a16_tokens(x, ids, w32, W["w13_q"], W["w13_s"], W["w2_q"], W["w2_s"], tokens=[3, 11, 0],
                              threads=2)
    assert np.array_equal(sub, full[[3, 11, 0]])


# ------------------------------------------------------------------------------- block-FP8

def _e4m3_values(codes):
    return torch.from_numpy(np.ascontiguousarray(codes)).view(torch.float8_e4m3fn).double().numpy()


def test_fp8_requant_pins():
    h = np.zeros(128, np.float32)
    h[:4] = [448.0, 1.0, -2.0, 0.5]
    q, s = oracle.fp8_requant(h)
    assert s == 1.0
    assert q[:4].tolist() == [0x7E, 0x38, 0xC0, 0x30] and not q[4:].any()
    q2, s2 = oracle.fp8_requant(2 * h)
    assert s2 == 2.0 and np.array_equal(q2, q)
    q0, s0 = oracle.fp8_requant(np.zeros(128, np.float32))
    assert s0 == np.float32(np.float32(1e-10) / np.float32(448.0)) and not q0.any()
    # against torch's float8 conversion (RNE) of the fp32 quotient
    hr = synth.logits(3, 1, 128)[0] * 7
    q3, s3 = oracle.fp8_requant(hr)
    assert s3 == np.float32(np.abs(hr).max() / np.float32(448.0))
    ref = torch.from_numpy(hr / np.float32(s3)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(q3, ref)


def test_fp8_one_hot_layer():
    H = I = 128
    x = np.zeros((1, H), np.uint8)
    x[0, 0] = 0x38                          # 1.0
    xs = np.array([[2.0]], np.float32)      # -> x[0] = 2
    w13 = np.zeros((1, 2 * I, H), np.uint8)
    w13_s = np.array([[[0.25], [0.5]]], np.float32)  # gate block (0,0), up block (1,0)
    w13[0, 0, 0] = 0x40                     # gate[0][0] = 2 * 0.25 -> g0 = 2*0.5 = 1
    w13[0, I, 0] = 0x38                     # up[0][0] = 1 * 0.5 -> u0 = 2*0.5 = 1
    w2 = np.zeros((1, H, I), np.uint8)
    w2[0, 0, 0] = 0x38
    w2_s = np.array([[[1.0]]], np.float32)
    out, hq = oracle.fp8_tokens(x, xs, np.array([[0]], np.int32), np.array([[1.0]], np.float32), w13, w13_s, w2,
                                w2_s, want_hq=True)
    sig1 = (1 + math.tanh(0.5)) / 2         # h0 = SiLU(1) * 1 = sigmoid(1)
    assert hq[0, 0, 0] == pytest.approx(sig1, rel=2e-7)
    assert out[0, 0] == pytest.approx(sig1, rel=2e-7)
    assert np.count_nonzero(out) == 1


@pytest.mark.parametrize("seed", [0, 1])
def test_fp8_dense_then_mask(seed):
    T, H, I, E, k = 8, 256, 256, 4, 2
    xq, xs = synth.x_e4m3(seed, T, H)
    lg = synth.logits(seed, T, E)
    ids, w32, _ = oracle.route(lg, k)
    W = synth.fp8_weights(seed, H, I, range(E))
    out, hq = oracle.fp8_tokens(xq, xs, ids, w32, W["w13"], W["w13_s"], W["w2"], W["w2_s"], want_hq=True)
    X = _e4m3_values(xq) * np.repeat(xs.astype(np.float64), 128, axis=1)
    W13 = _e4m3_values(W["w13"]) * np.repeat(np.repeat(W["w13_s"].astype(np.float64), 128, 1), 128, 2)
    W2 = _e4m3_values(W["w2"]) * np.repeat(np.repeat(W["w2_s"].astype(np.float64), 128, 1), 128, 2)
    ref = np.zeros((T, H))
    for t in range(T):
        for s in range(k):
            e = ids[t, s]
            g = torch.from_numpy(W13[e] @ X[t])
            h = (torch.nn.functional.silu(g[:I]) * g[I:]).float().numpy()   # fp32 intermediate
            hd = np.empty(I)
            for gi in range(I // 128):
                blk = h[gi * 128:(gi + 1) * 128]
                sc = np.float32(max(np.abs(blk).max(), np.float32(1e-10)) / np.float32(448.0))
                codes = torch.from_numpy(blk / sc).to(torch.float8_e4m3fn)
                hd[gi * 128:(gi + 1) * 128] = codes.double().numpy() * float(sc)
            np.testing.assert_allclose(hq[t, s], hd.astype(np.float32), rtol=0, atol=0)
            ref[t] += float(w32[t, s]) * (W2[e] @ hd)
    rms = np.sqrt(np.mean(ref ** 2))
    assert np.max(np.abs(out - ref)) <= 1e-12 * rms
