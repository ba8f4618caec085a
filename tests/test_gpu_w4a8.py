"""Routed W4A8 layer (MXFP4 weights, FP8 activations with E8M0 scales per 32 K) through the C
ABI vs the CPU oracle.

Gate: the block-FP8 variant's stated tolerance, the same class of activation quantization -
max|err| <= 3e-2*RMS(ref) + 1e-3 on the fp32-mode output, the same plus half a bf16 ulp on the
bf16 output, and the bf16 output equals the round-to-nearest-even of the fp32-mode output bit
for bit.  The quantized intermediate h is compared code by code with the oracle's: both sides
take the rounding decision on fp32 h, which the tensor cores and the fp64 oracle compute with
different rounding, so a code may move by one E4M3 step where h sits on a rounding boundary.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from helpers import check_tol, dev

pytestmark = pytest.mark.gpu
moe = pytest.importorskip("quantized_mixture_experts_softmax_b200")


class MXLayer:
    def __init__(self, seed, T, H, I, E, k, logits=None, weights=None, x=None):
        self.T, self.H, self.I, self.E, self.k = T, H, I, E, k
        self.W = weights if weights is not None else synth.mxfp4_weights(seed, H, I, range(E))
        self.x = synth.x_bf16(seed, T, H) if x is None else np.ascontiguousarray(x, np.uint16)
        self.lg = synth.logits(seed, T, E) if logits is None else np.ascontiguousarray(logits, np.float32)
        self.d = {k_: dev(v) for k_, v in self.W.items()}
        self.d_x, self.d_lg = dev(self.x, torch.bfloat16), dev(self.lg)
        self.ws = None

    def forward(self, ids, w, out_fp32):
        if self.ws is None:
            n = moe.moe_w4a8_workspace_size(self.T, self.H, self.I, self.E, self.k)
            self.ws = torch.empty(n, dtype=torch.uint8, device="cuda")
        return moe.moe_w4a8_forward(self.d_x, ids, w, self.d["w13"], self.d["w13_sf"], self.d["w2"],
                                    self.d["w2_sf"], out_fp32=out_fp32, workspace=self.ws)


def h_dequant(L):
    """The layer's quantized h, [T*k, I] in pair order, from the last forward's workspace."""
    v = moe.moe_w4a8_intermediate(L.ws, L.T, L.H, L.I, L.E, L.k)
    inv = v["inv_pos"].long()
    codes = v["h"][inv].cpu().contiguous().view(torch.float8_e4m3fn).double()
    sf = v["h_sf"][:, inv, :].permute(1, 0, 2).reshape(inv.numel(), L.I // 32).cpu().double()
    return (codes * torch.exp2(sf - 127).repeat_interleave(32, dim=1)).numpy()


def compare_h(got, ref, what):
    """Equal codes except, rarely, one E4M3 step apart (h on a rounding boundary)."""
    diff = got != ref
    frac = diff.mean()
    assert frac <= 2e-3, f"{what}: {diff.sum()} of {diff.size} h values differ"
    if diff.any():
        a, b = np.abs(got[diff]), np.abs(ref[diff])
        assert np.all(np.abs(got[diff] - ref[diff]) <= 0.13 * np.maximum(a, b) + 1e-30), f"{what}: h off by more than a step"
    return int(diff.sum())


def run_and_check(L, tokens=None, what="", check_h=True):
    ids, w = moe.moe_route(L.d_lg, L.k)
    ids_ref, w_ref, _ = oracle.route(L.lg, L.k)
    assert np.array_equal(ids.cpu().numpy(), ids_ref)
    out32 = L.forward(ids, w, True)
    torch.cuda.synchronize()
    h_gpu = h_dequant(L) if check_h else None
    out16 = L.forward(ids, w, False)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status() == 0
    ref, hq = oracle.w4a8_tokens(L.x, ids_ref, w_ref, L.W["w13"], L.W["w13_sf"], L.W["w2"], L.W["w2_sf"],
                                 tokens=tokens, want_hq=True)
    g32, g16 = out32.double().cpu().numpy(), out16.float().cpu().numpy()
    if check_h:
        rows = np.arange(L.T) if tokens is None else np.asarray(tokens)
        pairs = (rows[:, None] * L.k + np.arange(L.k)[None, :]).reshape(-1)
        compare_h(h_gpu[pairs], hq.reshape(-1, L.I).astype(np.float64), what)
    if tokens is not None:
        g32, g16 = g32[tokens], g16[tokens]
    e = check_tol(g32, ref, rel=3e-2, what=what + " fp32")
    check_tol(g16, ref, rel=3e-2, bf16_out=True, what=what + " bf16")
    assert torch.equal(out32.to(torch.bfloat16).view(torch.int16), out16.view(torch.int16))
    return e


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_tiny_w4a8_layer(seed):
    run_and_check(MXLayer(seed, 16, 256, 256, 8, 2), what=f"w4a8 tiny seed {seed}")


def test_w4a8_single_token_minimal_dims_and_k_equals_e():
    run_and_check(MXLayer(3, 1, 128, 128, 4, 2), what="T=1 H=I=128")
    run_and_check(MXLayer(4, 6, 256, 128, 4, 4), what="k=E")
    run_and_check(MXLayer(5, 9, 384, 384, 1, 1), what="E=1 K=384")


def _onehot_logits(assign, E, seed):
    lg = synth.logits(seed, len(assign), E) * 0.1
    lg[np.arange(len(assign)), assign] += 50.0
    return lg


@pytest.mark.parametrize("counts", [[15, 16, 17, 1, 31, 32, 33, 0, 64, 65], [100, 3, 0, 129],
                                    [111, 112, 113, 224, 225, 1, 97, 0]])
def test_w4a8_expert_counts_at_tile_boundaries(counts):
    """Token tiles of at most 32 rows (T <= 512) or 112 (T > 512), MMAs of 16-row multiples:
    counts around each."""
    assign = np.repeat(np.arange(len(counts)), counts)
    E = len(counts) + 2
    run_and_check(MXLayer(6, len(assign), 256, 128, E, 1, logits=_onehot_logits(assign, E, 6)),
                  what=f"counts {counts}")


def test_w4a8_wide_row_tiles():
    """T > 512: token tiles of up to 112 rows, experts spanning several."""
    T, E = 600, 4
    run_and_check(MXLayer(7, T, 128, 128, E, 2), what="T=600")


def test_w4a8_outlier_groups_and_wide_range():
    """Activation groups holding one 100x / 1000x outlier next to ordinary values, and rows
    spanning many decades: the group scales follow each group's own max."""
    T, H = 12, 256
    x = synth.x_bf16(8, T, H).view(np.uint16).copy()
    xf = (x.astype(np.uint32) << 16).view(np.float32)
    xf[0, 3] *= 100.0
    xf[1, 40] *= 1000.0
    xf[2, :] *= np.float32(2.0) ** np.arange(-24, 24, 48 / H, dtype=np.float32)[:H].round()
    xf[3, 64:96] = 0.0  # an all-zero group
    x = (xf.view(np.uint32) >> 16).astype(np.uint16)  # exact: the scaled values stay bf16
    run_and_check(MXLayer(8, T, H, 128, 4, 2, x=x), what="outliers")


def test_w4a8_nonfinite_input_is_flagged():
    L = MXLayer(9, 4, 128, 128, 4, 2)
    x = L.x.copy()
    x[1, 7] = 0x7F80  # +inf
    L.d_x = dev(x, torch.bfloat16)
    ids, w = moe.moe_route(L.d_lg, L.k)
    L.forward(ids, w, True)
    assert moe.moe_get_device_status() == moe.MOE_ERR_DEVICE_CHECK
    assert moe.moe_get_device_status() == 0


# ---------------------------------------------------------------------- full-size model
@pytest.fixture(scope="module")
def mx_model():
    return synth.mxfp4_weights(0, 7168, 2048, range(384))


@pytest.mark.slow
def test_w4a8_decode_full_size(mx_model):
    L = MXLayer(0, 64, 7168, 2048, 384, 8, weights=mx_model)
    e = run_and_check(L, what="w4a8 decode T=64")
    print(f"w4a8 decode max|err|/rms = {e:.3e}")


@pytest.mark.slow
def test_w4a8_prefill_sampled_tokens(mx_model):
    T = 8192
    lg = synth.logits(0, T, 384, zipf_s=1.1)
    L = MXLayer(0, T, 7168, 2048, 384, 8, weights=mx_model, logits=lg)
    ids_ref, _, _ = oracle.route(L.lg, 8)
    counts = np.bincount(ids_ref.ravel(), minlength=384)
    hot = int(np.argmax(counts))
    rng = np.random.default_rng(0)
    toks = set(rng.choice(T, 12, replace=False).tolist()) | {0, T - 1}
    toks |= set(np.nonzero((ids_ref == hot).any(1))[0][:6].tolist())
    tokens = np.array(sorted(toks), np.int32)
    e = run_and_check(L, tokens=tokens, what="w4a8 prefill T=8192 (sampled)")
    print(f"w4a8 prefill sampled {len(tokens)} tokens: max|err|/rms = {e:.3e}")
