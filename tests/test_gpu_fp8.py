"""Routed block-FP8 layer (e4m3 activations with 1x128 scales, e4m3 weights with 128x128
scales, requantized intermediate) through the C ABI vs the CPU oracle.

Gate from the layer's stated tolerance for this variant: max|err| <= 3e-2*RMS(ref) + 1e-3 on
the fp32-mode output, the same plus half a bf16 ulp on the bf16 output, and the bf16 output
equals the round-to-nearest-even of the fp32-mode output bit for bit.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from helpers import check_tol, dev

pytestmark = pytest.mark.gpu
moe = pytest.importorskip("quantized_mixture_experts_softmax_b200")


class F8Layer:
    def __init__(self, seed, T, H, I, E, k, logits=None, weights=None):
        self.T, self.H, self.I, self.E, self.k = T, H, I, E, k
        self.W = weights if weights is not None else synth.fp8_weights(seed, H, I, range(E))
        self.xq, self.xs = synth.x_e4m3(seed, T, H)
        self.lg = synth.logits(seed, T, E) if logits is None else np.ascontiguousarray(logits, np.float32)
        self.d = {k_: dev(v) for k_, v in self.W.items()}
        self.d_x, self.d_xs, self.d_lg = dev(self.xq), dev(self.xs), dev(self.lg)

    def forward(self, ids, w, out_fp32):
        return moe.moe_blockfp8_forward(self.d_x, self.d_xs, ids, w, self.d["w13"], self.d["w13_s"], self.d["w2"],
                                        self.d["w2_s"], out_fp32=out_fp32)


def run_and_check(L, tokens=None, what=""):
    ids, w = moe.moe_route(L.d_lg, L.k)
    ids_ref, w_ref, _ = oracle.route(L.lg, L.k)
    assert np.array_equal(ids.cpu().numpy(), ids_ref)
    out32 = L.forward(ids, w, True)
    out16 = L.forward(ids, w, False)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status() == 0
    ref = oracle.fp8_tokens(L.xq, L.xs, ids_ref, w_ref, L.W["w13"], L.W["w13_s"], L.W["w2"], L.W["w2_s"],
                            tokens=tokens)
    g32, g16 = out32.double().cpu().numpy(), out16.float().cpu().numpy()
    if tokens is not None:
        g32, g16 = g32[tokens], g16[tokens]
    e = check_tol(g32, ref, rel=3e-2, what=what + " fp32")
    check_tol(g16, ref, rel=3e-2, bf16_out=True, what=what + " bf16")
    assert torch.equal(out32.to(torch.bfloat16).view(torch.int16), out16.view(torch.int16))
    return e


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_tiny_fp8_layer(seed):
    run_and_check(F8Layer(seed, 16, 256, 256, 8, 2), what=f"fp8 tiny seed {seed}")


def test_fp8_single_token_and_k_equals_e():
    run_and_check(F8Layer(3, 1, 256, 128, 4, 2), what="T=1")
    run_and_check(F8Layer(4, 6, 128, 256, 4, 4), what="k=E")


def test_fp8_expert_spanning_many_token_tiles():
    T, E = 100, 8
    lg = synth.logits(5, T, E)
    lg[:, 0] += 100.0  # every token's first expert is expert 0: 100 rows = 4 token tiles
    run_and_check(F8Layer(5, T, 256, 256, E, 2, logits=lg), what="one hot expert")


@pytest.fixture(scope="module")
def fp8_model():
    return synth.fp8_weights(0, 7168, 2048, range(256))


@pytest.mark.slow
@pytest.mark.parametrize("T", [1, 16, 64, 512, 4096])
def test_fp8_config_sizes(fp8_model, T):
    L = F8Layer(0, T, 7168, 2048, 256, 8, weights=fp8_model)
    tokens = None
    if T > 64:
        rng = np.random.default_rng(T)
        tokens = np.unique(np.r_[0, T - 1, rng.choice(T, 24, replace=False)]).astype(np.int32)
    e = run_and_check(L, tokens=tokens, what=f"fp8 T={T}")
    print(f"fp8 T={T}: max|err|/rms = {e:.3e}")
