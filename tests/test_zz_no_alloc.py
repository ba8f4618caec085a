"""moe_align_noalloc: the allocation-free alignment entry point.

Some callers of this library cannot allocate device memory and have no workspace to hand
over: a plugin inside a host framework that owns every device buffer, or a deployment whose
device memory budget is fixed at start-up.  For them moe_align_noalloc keeps its scratch in a
fixed array inside the library.  This test calls it through the C ABI and checks that it
returns exactly what the CPU oracle's stable counting sort returns, and what moe_align (which
takes a caller workspace) returns, on two different calls in a row, so a second call cannot be
fooled by what the first left in the shared scratch.  It also checks that an expert id out of
range is skipped and reported through the shared scratch path as it is by moe_align, and that
a call needing more scratch than the array holds is refused.

The file is named so that pytest collects it last.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle

pytestmark = pytest.mark.gpu
moe = pytest.importorskip("quantized_mixture_experts_softmax_b200")
from quantized_mixture_experts_softmax_b200 import _native  # noqa: E402

SCRATCH_INTS = 131072


def _ids(T, E, k, seed):
    rng = np.random.default_rng(seed)
    p = 1.0 / np.arange(1, E + 1) ** 1.1
    p /= p.sum()
    return np.stack([rng.choice(E, size=k, replace=False, p=p) for _ in range(T)]).astype(np.int32)


def _noalloc(ids_d, E, align):
    T, k = ids_d.shape
    dev = ids_d.device
    cap = moe.moe_align_capacity(T, k, E, align)
    counts = torch.empty(E, dtype=torch.int32, device=dev)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    sorted_ids = torch.empty(cap, dtype=torch.int32, device=dev)
    inv_pos = torch.empty(T * k, dtype=torch.int32, device=dev)
    p = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731
    st = _native.lib.moe_align_noalloc(p(ids_d), T, k, E, align, p(counts), p(offsets), p(sorted_ids), p(inv_pos),
                                       ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == moe.MOE_OK, _native.STATUS.get(st, st)
    return dict(counts=counts, offsets=offsets, sorted_ids=sorted_ids, inv_pos=inv_pos)


def _same(a, b):
    n = int(b["offsets"][-1].item())
    assert torch.equal(a["counts"], b["counts"])
    assert torch.equal(a["offsets"], b["offsets"])
    assert torch.equal(a["sorted_ids"][:n], b["sorted_ids"][:n])
    assert torch.equal(a["inv_pos"], b["inv_pos"])


def _same_as_oracle(a, ids, E, align):
    ref = oracle.align(ids, E, align)
    n = int(ref["offsets"][-1])
    assert np.array_equal(a["counts"].cpu().numpy(), ref["counts"])
    assert np.array_equal(a["offsets"].cpu().numpy(), ref["offsets"])
    assert np.array_equal(a["sorted_ids"][:n].cpu().numpy(), ref["sorted_ids"])
    assert np.array_equal(a["inv_pos"].cpu().numpy(), ref["inv_pos"])
    return ref


@pytest.mark.parametrize("case", [
    # two calls in a row with different shapes; the second uses less scratch than the first
    [(8192, 384, 8, 16, 0), (64, 384, 8, 1, 1)],
    # the largest size the scratch admits at E=1024, then a small one
    [(SCRATCH_INTS // 1024 * 512 // 8, 1024, 8, 8, 2), (16, 8, 2, 1, 3)],
])
def test_noalloc_matches_workspace_version_on_two_calls(case):
    for T, E, k, align, seed in case:
        ids_h = _ids(T, E, k, seed)
        ids = torch.from_numpy(ids_h).cuda()
        got = _noalloc(ids, E, align)
        ref = moe.moe_align(ids, E, align)
        torch.cuda.synchronize()
        assert moe.moe_get_device_status() == 0
        _same_as_oracle(got, ids_h, E, align)
        _same(got, ref)


def test_noalloc_skips_and_reports_an_out_of_range_id():
    """An expert id outside [0, E) is skipped (inv_pos = -1), counted nowhere, and recorded as
    MOE_ERR_DEVICE_CHECK, exactly as moe_align and the oracle treat it; a clean call follows."""
    T, E, k, align = 300, 64, 4, 8
    ids_h = _ids(T, E, k, 11)
    ids_h[7, 2] = E + 3
    ids_h[250, 0] = -1
    ids = torch.from_numpy(ids_h).cuda()
    moe.moe_get_device_status()
    got = _noalloc(ids, E, align)
    assert moe.moe_get_device_status() == moe.MOE_ERR_DEVICE_CHECK
    ref = _same_as_oracle(got, ids_h, E, align)
    assert ref["bad"] == 2
    assert got["inv_pos"][7 * k + 2].item() == -1 and got["inv_pos"][250 * k].item() == -1
    ws_ref = moe.moe_align(ids, E, align)
    assert moe.moe_get_device_status() == moe.MOE_ERR_DEVICE_CHECK
    _same(got, ws_ref)
    clean = _ids(T, E, k, 12)
    got2 = _noalloc(torch.from_numpy(clean).cuda(), E, align)
    assert moe.moe_get_device_status() == 0
    _same_as_oracle(got2, clean, E, align)


def test_noalloc_rejects_sizes_beyond_its_scratch():
    T, E, k = SCRATCH_INTS // 1024 * 512 // 8 + 64, 1024, 8  # one chunk more than fits
    ids = torch.zeros(T, k, dtype=torch.int32, device="cuda")
    out = torch.empty(T * k + 1024 * 8, dtype=torch.int32, device="cuda")
    p = ctypes.c_void_p(out.data_ptr())
    st = _native.lib.moe_align_noalloc(ctypes.c_void_p(ids.data_ptr()), T, k, E, 1, p, p, p, p,
                                       ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == moe.MOE_ERR_UNSUPPORTED
