"""Inputs chosen to break the layer's numerical readings, through the C ABI vs the CPU oracle.

The decode-sized W4A16 path rounds activations to 16-bit fixed point per (row, 128-K block)
and the prefill-sized path casts them to fp16; both are exact or nearly so on N(0,1) data.
These tests use what real activations have and N(0,1) has not:
  * blocks with a 100x and a 1000x outlier next to ordinary values, in fixed channels and at
    random positions, on both paths;
  * an intermediate h spanning many decades (gate/up weight scales spread over 2.5 decades);
  * bf16 values beyond the fp16 range, and an h beyond it: the int8 path takes them like any
    other value, the fp16 path scales such rows by exact powers of two (and flags an h beyond
    even that, |h| >= 2^32);
  * the block-FP8 path's requantized intermediate: its e4m3 codes and 1x128 scales against the
    oracle's, not only the layer output.
Gates as in the other layer tests: max|err| <= 1e-2*RMS(ref) + 1e-3 (3e-2 for block-FP8).
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from helpers import W4Layer, W4Weights, check_tol, dev

pytestmark = pytest.mark.gpu
moe = pytest.importorskip("quantized_mixture_experts_softmax_b200")


def f32_to_bf16_bits(a):
    """Round-to-nearest-even float32 -> bf16 bit patterns (test input construction only)."""
    b = np.ascontiguousarray(a, np.float32).view(np.uint32).astype(np.uint64)
    return ((b + ((b >> 16) & 1) + 0x7FFF) >> 16).astype(np.uint16)


def bf16_bits_to_f32(u):
    return (np.asarray(u).astype(np.uint32) << 16).view(np.float32)


def with_outliers(x_bits, seed, fixed_channels):
    """Each 128-K block of each row gets one element x100 and one x1000 (fixed channels of the
    block, or random positions per row)."""
    x = bf16_bits_to_f32(x_bits).astype(np.float32).copy()
    T, H = x.shape
    rng = np.random.default_rng(seed)
    for b in range(H // 128):
        if fixed_channels:
            c100, c1000 = b * 128 + 5, b * 128 + 77
            x[:, c100] *= 100.0
            x[:, c1000] *= 1000.0
        else:
            pos = rng.integers(0, 128, size=(T, 2))
            pos[:, 1] = np.where(pos[:, 1] == pos[:, 0], (pos[:, 0] + 1) % 128, pos[:, 1])
            rows = np.arange(T)
            x[rows, b * 128 + pos[:, 0]] *= 100.0
            x[rows, b * 128 + pos[:, 1]] *= 1000.0
    return f32_to_bf16_bits(x)


def set_x(L, bits):
    L.x = np.ascontiguousarray(bits, np.uint16)
    L.d_x = dev(L.x, torch.bfloat16)


def run_and_check(L, what, tokens=None, rel=1e-2, own_rows=()):
    """The layer gate on all tokens; tokens listed in own_rows (rows scaled up on purpose, whose
    size would otherwise set RMS(ref) for everyone) are checked one by one against their own
    RMS and left out of the common check.  Tokens are independent, so this is the same gate."""
    ids, w = moe.moe_route(L.d_lg, L.k)
    ids_ref, w_ref, _ = oracle.route(L.lg, L.k)
    assert np.array_equal(ids.cpu().numpy(), ids_ref), f"{what}: routing ids differ"
    out32 = L.forward(moe, ids, w, out_fp32=True)
    out16 = L.forward(moe, ids, w, out_fp32=False)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status() == 0, what
    ref = L.oracle(oracle, ids_ref, w_ref, tokens=tokens)
    g32, g16 = out32.double().cpu().numpy(), out16.float().cpu().numpy()
    if tokens is not None:
        g32, g16 = g32[tokens], g16[tokens]
    rest = np.setdiff1d(np.arange(len(ref)), np.asarray(own_rows, int))
    groups = [rest] + [[r] for r in own_rows]
    e = 0.0
    for rows in groups:
        e = max(e, check_tol(g32[rows], ref[rows], rel=rel, what=f"{what} fp32 rows {rows[0]}.."))
        check_tol(g16[rows], ref[rows], rel=rel, bf16_out=True, what=f"{what} bf16 rows {rows[0]}..")
    print(f"{what}: max|err|/rms = {e:.3e}")
    return e


# T <= 64: int8 path for every expert; T = 200 with an even spread over 8 experts (top-2, about
# 50 rows each) and T = 300 with one hot expert reach the fp16 path for some or all experts.
@pytest.mark.parametrize("T,hot", [(16, False), (64, False), (200, False), (300, True)])
@pytest.mark.parametrize("fixed", [True, False], ids=["fixed-channels", "random-positions"])
def test_outlier_blocks(T, hot, fixed):
    L = W4Layer(31, T, 1024, 256, 8, 2)
    if hot:
        L.lg[:, 3] += 100.0
        L.d_lg = dev(L.lg)
    set_x(L, with_outliers(L.x, 31 + T, fixed))
    run_and_check(L, f"outliers T={T} {'hot expert ' if hot else ''}{'fixed' if fixed else 'random'}")


@pytest.fixture(scope="module")
def spread_weights():
    """Gate/up weight scales spread over 2.5 decades per output row, so that g, and h = SiLU(g)
    * up, span many decades inside every 128-row group of h."""
    w = W4Weights(41, 1024, 256, 8)
    rng = np.random.default_rng(41)
    s = bf16_bits_to_f32(w.W["w13_s"]).astype(np.float64)
    mult = 10.0 ** (-2.5 * rng.random(size=(8, 512, 1)))
    w.W["w13_s"] = f32_to_bf16_bits((s * 2.5 * mult).astype(np.float32))
    w.d_w13_s = dev(w.W["w13_s"], torch.bfloat16)
    return w


@pytest.mark.parametrize("T", [32, 200])
def test_intermediate_spanning_many_decades(spread_weights, T):
    L = W4Layer(42, T, 1024, 256, 8, 2, weights=spread_weights)
    ids_ref, w_ref, _ = oracle.route(L.lg, 2)
    _, h = oracle.w4a16_tokens(L.x, ids_ref, w_ref, L.W["w13_q"], L.W["w13_s"], L.W["w2_q"], L.W["w2_s"],
                               want_h=True)
    a = np.abs(h[np.abs(h) > 0])
    span = np.log10(a.max() / np.percentile(a, 1))
    assert span > 6.0, f"h spans only {span:.1f} decades"
    run_and_check(L, f"h over {span:.1f} decades T={T}")


def test_int8_path_takes_values_beyond_fp16():
    """T <= 64: activations of any finite magnitude are exact to 16 bits of their block."""
    L = W4Layer(51, 16, 256, 128, 8, 2)
    x = bf16_bits_to_f32(L.x).copy()
    x[3, 10] = 1.0e6
    x[9, 200] = -3.0e7
    x[12, :128] *= 5.0e4
    set_x(L, f32_to_bf16_bits(x))
    run_and_check(L, "int8 path, |x| up to 3e7", own_rows=(3, 9, 12))


def _hot_layer(seed, T=200):
    """Every token's only expert is expert 0 (T rows: the fp16 GEMM)."""
    lg = synth.logits(seed, T, 8) * 0.1
    lg[:, 0] += 50.0
    return W4Layer(seed, T, 256, 128, 8, 1, logits=lg)


def test_fp16_path_takes_inputs_beyond_fp16():
    """Rows with values beyond the largest fp16 (65504) are scaled by an exact power of two to
    fit and the accumulators scaled back; h then exceeds fp16 as well and is rescaled per row."""
    L = _hot_layer(52)
    x = bf16_bits_to_f32(L.x).copy()
    x[5, 17] = 70000.0  # bf16 70144
    x[9, :] *= 3.0e3    # every value of the row scaled; |h| ~ 1e7
    x[77, 100] = -2.0e5
    set_x(L, f32_to_bf16_bits(x))
    run_and_check(L, "fp16 path, |x| up to 2e5", own_rows=(5, 9, 77))


def test_fp16_path_takes_an_intermediate_beyond_fp16():
    """Large gate/up weight scales: h = SiLU(gate) * up reaches 1e5 .. 1e7 for every token."""
    L = _hot_layer(53)
    L.W["w13_s"] = np.full_like(L.W["w13_s"], f32_to_bf16_bits(np.float32(8.0)))
    L.w.d_w13_s = dev(L.W["w13_s"], torch.bfloat16)
    ids_ref, w_ref, _ = oracle.route(L.lg, 1)
    _, h = oracle.w4a16_tokens(L.x, ids_ref, w_ref, L.W["w13_q"], L.W["w13_s"], L.W["w2_q"], L.W["w2_s"],
                               want_h=True)
    assert np.abs(h).max() > 1e6
    run_and_check(L, f"fp16 path, |h| up to {np.abs(h).max():.1e}")


def test_fp16_path_flags_an_intermediate_beyond_its_prescaled_range():
    """|h| >= 65520 * 2^16 (about 4.3e9) is beyond even the prescaled store: flagged."""
    L = _hot_layer(55)
    L.W["w13_s"] = np.full_like(L.W["w13_s"], f32_to_bf16_bits(np.float32(8.0)))
    L.w.d_w13_s = dev(L.W["w13_s"], torch.bfloat16)
    x = bf16_bits_to_f32(L.x).copy()
    x[3, :] *= 1.0e4  # |g| ~ 1e7, h ~ 1e14
    set_x(L, f32_to_bf16_bits(x))
    ids, w = moe.moe_route(L.d_lg, 1)
    moe.moe_get_device_status()
    L.forward(moe, ids, w, out_fp32=True)
    assert moe.moe_get_device_status() == moe.MOE_ERR_DEVICE_CHECK


def test_grouped_gemm_takes_inputs_beyond_fp16():
    M, K, N = 300, 256, 128  # M > 64: the fp16 path
    a, w_q, w_s = synth.gemm_operands(54, M, K, N)
    a = a.copy()
    a[100, 3] = f32_to_bf16_bits(np.array([-1.0e5], np.float32))[0]
    a[200, :] = f32_to_bf16_bits(bf16_bits_to_f32(a[200, :]) * np.float32(1.0e9))
    off = np.array([0, M], np.int32)
    moe.moe_get_device_status()
    out = moe.moe_w4a16_gemm(dev(a, torch.bfloat16), dev(w_q), dev(w_s, torch.bfloat16), dev(off), out_fp32=True)
    assert moe.moe_get_device_status() == 0
    ref = oracle.w4a16_gemm(a, True, w_q, w_s, off)
    got = out.double().cpu().numpy()
    # rows are independent: check each scale of row against itself
    for rows in (np.r_[0:100, 101:200, 201:M], [100], [200]):
        check_tol(got[rows], ref[rows], what=f"grouped GEMM rows {rows[0]}..")


# ---------------------------------------------------------------------- block-FP8 intermediate
E4M3 = np.array([oracle.e4m3(b) for b in range(256)])
MAGS = np.unique(np.abs(E4M3[np.isfinite(E4M3)]))  # the 127 non-negative e4m3 magnitudes, ascending


def _mag_index(v):
    """Index in MAGS of the magnitude nearest to |v|."""
    a = np.abs(v)
    i = np.clip(np.searchsorted(MAGS, a), 1, len(MAGS) - 1)
    return np.where(a - MAGS[i - 1] <= MAGS[i] - a, i - 1, i)


@pytest.mark.parametrize("T,E", [(24, 8), (600, 8)])  # 32-row token tiles; 64-row tiles (T > 512)
def test_fp8_requantized_h_codes_and_scales(T, E):
    """The kernel's e4m3 codes of h and their 1x128 scales equal the oracle's: scales to the
    accumulation-order difference of fp32 vs fp64 (1e-4 relative), codes exactly except for a
    few at most one code apart (values within that difference of a rounding boundary)."""
    H, I, k = 256, 512, 2
    W = synth.fp8_weights(61, H, I, range(E))
    xq, xs = synth.x_e4m3(61, T, H)
    lg = synth.logits(61, T, E)
    d = {n: dev(v) for n, v in W.items()}
    ids, w = moe.moe_route(dev(lg), k)
    ids_ref, w_ref, _ = oracle.route(lg, k)
    assert np.array_equal(ids.cpu().numpy(), ids_ref)
    ws = torch.empty(moe.moe_blockfp8_workspace_size(T, H, I, E, k), dtype=torch.uint8, device="cuda")
    moe.moe_blockfp8_forward(dev(xq), dev(xs), ids, w, d["w13"], d["w13_s"], d["w2"], d["w2_s"], out_fp32=True,
                             workspace=ws)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status() == 0
    mid = moe.moe_blockfp8_intermediate(ws, T, H, I, E, k)
    inv = mid["inv_pos"].cpu().numpy()
    codes = mid["h"].cpu().numpy()
    scales = mid["h_scale_t"].cpu().numpy()
    _, hq = oracle.fp8_tokens(xq, xs, ids_ref, w_ref, W["w13"], W["w13_s"], W["w2"], W["w2_s"], want_hq=True)
    G = I // 128
    ref = hq.astype(np.float64).reshape(T * k, G, 128)
    s_ref = np.maximum(np.abs(ref).max(2), 1e-10) / 448.0  # [T*k, G]
    s_gpu = scales[:, inv].T                               # [T*k, G]
    np.testing.assert_allclose(s_gpu, s_ref, rtol=1e-4)
    v_ref = ref / s_ref[:, :, None]
    v_gpu = E4M3[codes[inv]].reshape(T * k, G, 128)
    assert np.all(np.isfinite(v_gpu))
    i_ref, i_gpu = _mag_index(v_ref), _mag_index(v_gpu)
    assert np.all(np.abs(i_ref - i_gpu) <= 1), "a code more than one step from the oracle's"
    both = (i_ref > 0) & (i_gpu > 0)
    assert np.all(np.sign(v_ref[both]) == np.sign(v_gpu[both])), "a code of the wrong sign"
    n_diff = int((i_ref != i_gpu).sum())
    print(f"fp8 h T={T}: {n_diff} of {i_ref.size} codes one step apart; max scale rel diff "
          f"{np.max(np.abs(s_gpu / s_ref - 1)):.2e}")
    assert n_diff <= max(2, 1e-3 * i_ref.size)
