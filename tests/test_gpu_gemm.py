"""Grouped W4A16 GEMM entry (moe_w4a16_gemm) vs the oracle.

* One-hot probe: identity activations read every dequantized weight back exactly, which pins
  the GPU side's INT4 layout (nibble order, K-contiguous words, per-32 scales) independently.
* The single-expert GEMM sweep of the workload, [M,7168]x[7168,512] and [M,256]x[256,7168],
  M in {1, 64, 512, 4096, 32768} (rows sampled for the oracle when M is large).
* Ragged multi-expert offsets with empty experts and uncovered rows.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from helpers import check_tol, dev

pytestmark = pytest.mark.gpu
moe = pytest.importorskip("quantized_mixture_experts_softmax_b200")


def test_one_hot_probe_reads_weights_exactly():
    K, N = 256, 128
    idx = np.arange(N)[:, None] * (K // 8) + np.arange(K // 8)[None, :]
    words = ((idx.astype(np.uint64) * 0x9E3779B1 + 0x7F4A7C15) & 0xFFFFFFFF).astype(np.uint32)
    w_q = words.view(np.int32)[None].copy()
    # scale of row n, group g: 2^-((n + g) % 8), exact in bf16 and fp16
    w_s = ((127 - ((np.arange(N)[:, None] + np.arange(K // 32)[None, :]) % 8)) << 7).astype(np.uint16)[None]
    expect = np.empty((N, K))
    for n in range(N):
        for c in range(K):
            expect[n, c] = oracle.int4(int(words[n, c // 8]), c % 8) * 2.0 ** (-((n + c // 32) % 8))
    for a_is_bf16, one in [(True, 0x3F80), (False, 0x3C00)]:
        a = np.zeros((K, K), np.uint16)
        a[np.arange(K), np.arange(K)] = one
        out = moe.moe_w4a16_gemm(dev(a, torch.bfloat16 if a_is_bf16 else torch.float16), dev(w_q),
                                 dev(w_s, torch.bfloat16), dev(np.array([0, K], np.int32)), out_fp32=True)
        got = out.double().cpu().numpy()  # got[m][n] = W[n][m]
        assert np.array_equal(got, expect.T)


SWEEP = [(M, K, N) for (K, N) in [(7168, 512), (256, 7168)] for M in (1, 64, 512, 4096, 32768)]


@pytest.mark.parametrize("M,K,N", SWEEP)
def test_single_expert_sweep(M, K, N):
    a, w_q, w_s = synth.gemm_operands(1, M, K, N)
    out32 = moe.moe_w4a16_gemm(dev(a, torch.bfloat16), dev(w_q), dev(w_s, torch.bfloat16),
                               dev(np.array([0, M], np.int32)), out_fp32=True)
    out16 = moe.moe_w4a16_gemm(dev(a, torch.bfloat16), dev(w_q), dev(w_s, torch.bfloat16),
                               dev(np.array([0, M], np.int32)), out_fp32=False)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status() == 0
    rows = np.arange(M) if M <= 64 else np.unique(np.r_[0, M - 1, np.random.default_rng(M).choice(M, 40)])
    ref = oracle.w4a16_gemm(a[rows], True, w_q, w_s, np.array([0, len(rows)], np.int32))
    check_tol(out32.double().cpu().numpy()[rows], ref, what=f"gemm {M}x{K}x{N} fp32")
    check_tol(out16.float().cpu().numpy()[rows], ref, bf16_out=True, what=f"gemm {M}x{K}x{N} bf16")
    assert torch.equal(out32.to(torch.bfloat16).view(torch.int16), out16.view(torch.int16))


@pytest.mark.parametrize("offsets", [[0, 10, 10, 150, 290, 300], [5, 5, 77, 78, 200, 290], [0, 300, 300, 300, 300, 300]])
def test_ragged_experts(offsets):
    M, K, N, E = 300, 384, 256, 5
    a = synth.x_bf16(4, M, K)
    W = synth.w4a16_weights(4, K, N // 2, range(E))  # w13-shaped: [E, N, K/8]
    w_q, w_s = W["w13_q"], W["w13_s"]
    off = np.array(offsets, np.int32)
    sentinel = torch.full((M, N), 12345.0, dtype=torch.float32, device="cuda")
    out = moe.moe_w4a16_gemm(dev(a, torch.bfloat16), dev(w_q), dev(w_s, torch.bfloat16), dev(off), out=sentinel,
                             out_fp32=True)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status() == 0
    got = out.double().cpu().numpy()
    ref = oracle.w4a16_gemm(a, True, w_q, w_s, off)
    covered = np.zeros(M, bool)
    covered[off[0]:off[-1]] = True
    check_tol(got[covered], ref[covered], what="ragged")
    assert np.all(got[~covered] == 12345.0)


@pytest.mark.parametrize("K", [384, 1024])
@pytest.mark.parametrize("offsets", [[4, 4, 20, 21, 50, 56], [0, 60, 60, 60, 60, 60]])
def test_ragged_experts_decode_sized_split_k(K, offsets):
    """M <= 64 runs the int8 path; with few work items its K range is split (fp32 partial sums
    reduced in split order), here into 2 (K=384, a half 256-K stage last) or 4 (K=1024) parts.
    Rows outside every expert range keep their previous contents (12288, exact in bf16)."""
    M, N, E = 60, 256, 5
    a = synth.x_bf16(5, M, K)
    W = synth.w4a16_weights(5, K, N // 2, range(E))
    w_q, w_s = W["w13_q"], W["w13_s"]
    off = np.array(offsets, np.int32)
    ref = oracle.w4a16_gemm(a, True, w_q, w_s, off)
    covered = np.zeros(M, bool)
    covered[off[0]:off[-1]] = True
    outs = {}
    for fp32 in (True, False):
        init = torch.full((M, N), 12288.0, device="cuda", dtype=torch.float32 if fp32 else torch.bfloat16)
        outs[fp32] = moe.moe_w4a16_gemm(dev(a, torch.bfloat16), dev(w_q), dev(w_s, torch.bfloat16), dev(off),
                                        out=init, out_fp32=fp32)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status() == 0
    g32 = outs[True].double().cpu().numpy()
    g16 = outs[False].float().cpu().numpy()
    check_tol(g32[covered], ref[covered], what=f"split-K K={K} fp32")
    check_tol(g16[covered], ref[covered], bf16_out=True, what=f"split-K K={K} bf16")
    assert np.all(g32[~covered] == 12288.0) and np.all(g16[~covered] == 12288.0)
    assert torch.equal(outs[True].to(torch.bfloat16)[covered.tolist()].view(torch.int16),
                       outs[False][covered.tolist()].view(torch.int16))
