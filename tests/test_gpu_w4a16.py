"""Routed W4A16 layer through the C ABI vs the CPU oracle.

Gate (from the layer's stated tolerance): the fp32-output mode meets max|err| <=
1e-2*RMS(ref) + 1e-3; the bf16 output meets the same plus half a bf16 ulp of each reference
element (its own representation error) and equals the round-to-nearest-even of the fp32
output bit for bit (the two modes share every kernel but the last store).  Routing ids are
compared bit-exactly first, so both sides combine the same experts.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from helpers import W4Layer, W4Weights, check_tol, dev

pytestmark = pytest.mark.gpu
moe = pytest.importorskip("quantized_mixture_experts_softmax_b200")


def run_and_check(L: W4Layer, tokens=None, what=""):
    ids, w = moe.moe_route(L.d_lg, L.k)
    ids_ref, w_ref, _ = oracle.route(L.lg, L.k)
    assert np.array_equal(ids.cpu().numpy(), ids_ref), f"{what}: routing ids differ"
    out32 = L.forward(moe, ids, w, out_fp32=True)
    out16 = L.forward(moe, ids, w, out_fp32=False)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status() == 0
    ref = L.oracle(oracle, ids_ref, w_ref, tokens=tokens)
    g32 = out32.double().cpu().numpy()
    g16 = out16.float().cpu().numpy()
    if tokens is not None:
        g32, g16 = g32[tokens], g16[tokens]
    e32 = check_tol(g32, ref, what=what + " fp32")
    check_tol(g16, ref, bf16_out=True, what=what + " bf16")
    assert torch.equal(out32.to(torch.bfloat16).view(torch.int16), out16.view(torch.int16)), \
        f"{what}: bf16 output != RNE(fp32 output)"
    return e32


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_tiny_layer(seed):
    run_and_check(W4Layer(seed, 16, 256, 128, 8, 2), what=f"tiny seed {seed}")


def test_single_token():
    run_and_check(W4Layer(3, 1, 256, 128, 8, 2), what="T=1")


def _onehot_logits(assign, E, k, seed):
    """Logits whose top-1 expert for token t is assign[t] (the rest random below it)."""
    T = len(assign)
    lg = synth.logits(seed, T, E) * 0.1
    lg[np.arange(T), assign] += 50.0
    return lg


def test_expert_counts_at_tile_boundaries_thin():
    # T <= 64 uses thin token tiles (at most 64 rows): counts 15/16/17/1/15 and empty experts
    assign = np.repeat(np.arange(5), [15, 16, 17, 1, 15])
    E = 8
    lg = _onehot_logits(assign, E, 1, 7)
    run_and_check(W4Layer(7, len(assign), 256, 128, E, 1, logits=lg), what="thin boundaries")


def test_expert_counts_at_tile_boundaries_wide():
    # T > 64 uses token tiles of up to 256 rows: counts 129, 64, 65, 257, 0 and 1
    counts = [129, 64, 65, 257, 0, 1]
    assign = np.repeat(np.arange(len(counts)), counts)
    E = 8
    lg = _onehot_logits(assign, E, 1, 8)
    run_and_check(W4Layer(8, len(assign), 256, 128, E, 1, logits=lg), what="wide boundaries")


def test_expert_counts_straddling_the_kernel_choice():
    """T > 64: each expert runs on the int8 GEMM when it has few rows and on the fp16 GEMM when
    it has many, chosen per expert from its count in the same call; counts on both sides of
    every plausible switch point (8, 16, 32, 48, 64 rows) and of the tile heights."""
    counts = [1, 7, 8, 9, 15, 16, 17, 31, 32, 33, 47, 48, 49, 63, 64, 65, 100, 129, 0, 2]
    assign = np.repeat(np.arange(len(counts)), counts)
    E = 24
    lg = _onehot_logits(assign, E, 1, 14)
    run_and_check(W4Layer(14, len(assign), 256, 256, E, 1, logits=lg), what="mixed kernels")


def test_expert_counts_at_the_fp16_tile_height():
    """Experts on the fp16 GEMM take token tiles of at most 192 rows: counts around one, two
    and three tiles."""
    counts = [191, 192, 193, 384, 385, 577, 17]
    assign = np.repeat(np.arange(len(counts)), counts)
    E = 8
    lg = _onehot_logits(assign, E, 1, 15)
    run_and_check(W4Layer(15, len(assign), 256, 128, E, 1, logits=lg), what="192-row tiles")


def test_all_tokens_one_expert_top2():
    T, E = 300, 8
    lg = synth.logits(9, T, E)
    lg[:, 3] += 100.0
    run_and_check(W4Layer(9, T, 256, 128, E, 2, logits=lg), what="one hot expert")


def test_minimal_hidden_and_intermediate():
    run_and_check(W4Layer(10, 20, 128, 128, 4, 2), what="H=I=128")


def test_partial_last_k_block():
    # K = 384 = 256 + 128: the last weight stage is half out of bounds (zero-filled)
    run_and_check(W4Layer(11, 24, 384, 384, 4, 2), what="H=I=384")


def test_single_expert_dense_ffn():
    run_and_check(W4Layer(12, 40, 256, 256, 1, 1), what="E=1 k=1")


def test_k_equals_e():
    run_and_check(W4Layer(13, 9, 256, 128, 4, 4), what="k=E")


@pytest.mark.parametrize("T,k,E", [(64, 64, 64), (64, 65, 65), (64, 8, 512), (8, 2, 600)])
def test_decode_prologue_paths(T, k, E):
    """T <= 64: batches of at most 4096 (token, slot) pairs and 512 experts take the alignment,
    tile schedule and planes in one launch, larger ones the separate kernels; both sides of
    each limit."""
    run_and_check(W4Layer(14, T, 128, 128, E, k), what=f"T={T} k={k} E={E}")


# ---------------------------------------------------------------------- full-size model
@pytest.fixture(scope="module")
def big_weights():
    return W4Weights(0, 7168, 2048, 384)


@pytest.mark.slow
def test_decode_full_size(big_weights):
    L = W4Layer(0, 64, 7168, 2048, 384, 8, weights=big_weights)
    e = run_and_check(L, what="decode T=64")
    print(f"decode max|err|/rms = {e:.3e}")


@pytest.mark.slow
def test_prefill_sampled_tokens(big_weights):
    L = W4Layer(0, 8192, 7168, 2048, 384, 8, zipf=1.1, weights=big_weights)
    ids_ref, _, _ = oracle.route(L.lg, 8)
    counts = np.bincount(ids_ref.ravel(), minlength=384)
    hot = int(np.argmax(counts))
    active = np.nonzero(counts)[0]
    cold = active[np.argsort(counts[active])[:6]]
    rng = np.random.default_rng(0)
    toks = set(rng.choice(8192, 12, replace=False).tolist())
    toks |= set(np.nonzero((ids_ref == hot).any(1))[0][:6].tolist())
    for e in cold:
        toks |= set(np.nonzero((ids_ref == e).any(1))[0][:2].tolist())
    toks |= {0, 8191}
    tokens = np.array(sorted(toks), np.int32)
    e = run_and_check(L, tokens=tokens, what="prefill T=8192 (sampled)")
    print(f"prefill sampled {len(tokens)} tokens: max|err|/rms = {e:.3e}")
