"""GPU router and alignment vs the oracle: bit-exact ids, counts, offsets, sorted ids and
inverse positions; routing weights within 1e-6."""
import numpy as np
import pytest
import torch

import oracle
import synth
from helpers import dev

pytestmark = pytest.mark.gpu
moe = pytest.importorskip("quantized_mixture_experts_softmax_b200")


ROUTE_CASES = [
    # T, E, k, zipf, seed
    (16, 8, 2, 0.0, 0), (16, 8, 2, 0.0, 1), (16, 8, 2, 0.0, 2),   # tiny layer
    (64, 384, 8, 0.0, 0), (64, 384, 8, 0.0, 1),                    # decode layer
    (8192, 384, 8, 1.1, 0),                                        # prefill layer (Zipf-skewed)
    (1, 256, 8, 0.0, 0), (16, 256, 8, 0.0, 0), (4096, 256, 8, 0.0, 0),  # block-FP8 layer sizes
    (1, 1, 1, 0.0, 0), (33, 1000, 7, 0.0, 3), (5, 1024, 1, 0.0, 4), (7, 40, 40, 0.0, 5), (3, 33, 32, 0.5, 6),
]


@pytest.mark.parametrize("T,E,k,zipf,seed", ROUTE_CASES)
@pytest.mark.parametrize("renorm", [True, False])
def test_route_parity(T, E, k, zipf, seed, renorm):
    lg = synth.logits(seed, T, E, zipf_s=zipf)
    ids, w = moe.moe_route(dev(lg), k, renormalize=renorm)
    ids_ref, w_ref, w64 = oracle.route(lg, k, renormalize=renorm)
    assert np.array_equal(ids.cpu().numpy(), ids_ref)
    np.testing.assert_allclose(w.cpu().numpy().astype(np.float64), w64, rtol=0, atol=1e-6)
    assert moe.moe_get_device_status() == 0


def test_route_ties():
    lg = np.array([[1.0, 3.0, 3.0, 2.0, 3.0] + [-5.0] * 59,
                   [0.5] * 64,
                   [-1.0, -2.0, -1.0, -2.0] + [-3.0] * 60], np.float32)
    lg[1, 40] = 0.5
    ids, w = moe.moe_route(dev(lg), 3)
    ids_ref, _, w64 = oracle.route(lg, 3)
    assert ids.cpu().numpy().tolist() == ids_ref.tolist() == [[1, 2, 4], [0, 1, 2], [0, 2, 1]]
    np.testing.assert_allclose(w.cpu().numpy(), w64, atol=1e-6)


def _skewed_ids(T, E, k, seed):
    rng = np.random.default_rng(seed)
    p = 1.0 / np.arange(1, E + 1) ** 1.2
    p /= p.sum()
    return np.stack([rng.choice(E, size=k, replace=False, p=p) for _ in range(T)]).astype(np.int32)


ALIGN_CASES = [(16, 8, 2), (64, 384, 8), (1, 8, 8), (100, 64, 6), (8192, 384, 8), (4096, 256, 8), (700, 1024, 3)]


@pytest.mark.parametrize("T,E,k", ALIGN_CASES)
@pytest.mark.parametrize("align", [1, 8, 16, 128])
def test_align_parity(T, E, k, align):
    ids = _skewed_ids(T, E, k, T + E + k)
    r = moe.moe_align(dev(ids), E, align)
    ref = oracle.align(ids, E, align)
    n = int(ref["offsets"][-1])
    assert np.array_equal(r["counts"].cpu().numpy(), ref["counts"])
    assert np.array_equal(r["offsets"].cpu().numpy(), ref["offsets"])
    assert np.array_equal(r["sorted_ids"].cpu().numpy()[:n], ref["sorted_ids"])
    assert np.array_equal(r["inv_pos"].cpu().numpy(), ref["inv_pos"])
    assert moe.moe_get_device_status() == 0


def test_align_from_router_prefill():
    lg = synth.logits(0, 8192, 384, zipf_s=1.1)
    ids, _ = moe.moe_route(dev(lg), 8)
    r = moe.moe_align(ids, 384, 16)
    ref = oracle.align(ids.cpu().numpy(), 384, 16)
    n = int(ref["offsets"][-1])
    assert np.array_equal(r["sorted_ids"].cpu().numpy()[:n], ref["sorted_ids"])
    assert np.array_equal(r["inv_pos"].cpu().numpy(), ref["inv_pos"])
    counts = ref["counts"]
    assert (counts == 0).sum() > 0 and counts.max() > 1024  # the skew the workload asks for


def test_align_flags_out_of_range_ids():
    ids = np.array([[0, 5], [1, -1], [2, 1]], np.int32)
    moe.moe_get_device_status()
    r = moe.moe_align(dev(ids), 4, 1)
    assert moe.moe_get_device_status() == moe.MOE_ERR_DEVICE_CHECK
    ref = oracle.align(ids, 4, 1)
    assert np.array_equal(r["counts"].cpu().numpy(), ref["counts"])
    assert np.array_equal(r["inv_pos"].cpu().numpy(), ref["inv_pos"])
    assert np.array_equal(r["sorted_ids"].cpu().numpy()[:4], ref["sorted_ids"])
    assert moe.moe_get_device_status() == 0  # cleared by the read
