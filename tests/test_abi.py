"""The C-ABI library: loads without a GPU, exports every symbol include/moe.h declares, and
rejects bad arguments synchronously (these paths touch no device memory)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def native():
    import __graft_entry__
    __graft_entry__.build()
    from quantized_mixture_experts_softmax_b200 import _native
    return _native


def declared_symbols():
    text = open(os.path.join(ROOT, "include", "moe.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z0-9_]+)\s*\(", text)))


def test_header_and_exports_agree(native):
    decl = declared_symbols()
    assert len(decl) >= 15
    assert sorted(native.EXPORTS) == decl
    lib = ctypes.CDLL(native.LIB_PATH)
    for name in decl:
        assert hasattr(lib, name), name


def test_status_strings(native):
    for code, name in native.STATUS.items():
        assert native.lib.moe_status_string(code).decode() == name


def test_workspace_queries(native):
    L = native.lib
    assert L.moe_align_capacity(64, 8, 384, 16) == 64 * 8 + 384 * 15
    assert L.moe_align_workspace_size(64, 8, 384) >= 384 * 4
    ws = L.moe_w4a16_workspace_size(64, 7168, 2048, 384, 8)
    # x_perm fp16 + h fp16 + y fp32 rows for T*k pairs dominate
    assert ws >= 512 * (7168 * 2 + 2048 * 2 + 7168 * 4)
    assert L.moe_w4a16_workspace_size(64, 7000, 2048, 384, 8) == 0  # H not a multiple of 128
    assert L.moe_w4a16_gemm_workspace_size(1, 7168, 512, 1) > 0
    # few work items: the K range is split (28 splits of one 256-K stage for 4 items), and the
    # workspace holds their fp32 partial sums
    assert L.moe_w4a16_gemm_workspace_size(1, 7168, 512, 1) >= 28 * 1 * 512 * 4
    assert L.moe_w4a16_gemm_workspace_size(512, 7168, 512, 1) >= 18 * 512 * 512 * 4
    # enough items (32768 rows): no partial sums beyond the fp16 copy of the activations
    assert L.moe_w4a16_gemm_workspace_size(32768, 7168, 512, 1) < 32768 * 7168 * 2 + 2 * 32768 * 512 * 4
    assert L.moe_w4a16_gemm_workspace_size(1, 7000, 512, 1) == 0


def test_argument_errors_return_codes(native):
    L = native.lib
    F = native.W4A16Args
    fake = 1 << 20  # never dereferenced: the checks fail first
    a = F(fake, fake, fake, fake, fake, fake, fake, 64, 7000, 2048, 384, 8, fake, 0)
    assert L.moe_w4a16_forward(ctypes.byref(a), ctypes.c_void_p(fake), 1 << 40, None) == native.MOE_ERR_UNSUPPORTED
    a = F(fake + 2, fake, fake, fake, fake, fake, fake, 64, 7168, 2048, 384, 8, fake, 0)
    assert L.moe_w4a16_forward(ctypes.byref(a), ctypes.c_void_p(fake), 1 << 40, None) == native.MOE_ERR_INVALID_ARG
    a = F(fake, fake, fake, fake, fake, fake, fake, 64, 7168, 2048, 384, 8, fake, 0)
    assert L.moe_w4a16_forward(ctypes.byref(a), ctypes.c_void_p(fake), 1024, None) == native.MOE_ERR_WORKSPACE
    assert L.moe_w4a16_forward(None, None, 0, None) == native.MOE_ERR_INVALID_ARG
    assert L.moe_route(ctypes.c_void_p(fake), 4, 8, 9, 1, ctypes.c_void_p(fake), ctypes.c_void_p(fake),
                       None) == native.MOE_ERR_UNSUPPORTED  # k > E
    assert L.moe_align(ctypes.c_void_p(fake), 4, 2, 8, 0, *([ctypes.c_void_p(fake)] * 5), 1 << 20,
                       None) == native.MOE_ERR_UNSUPPORTED  # align 0
    assert L.moe_debug_wait_timeout(0, None) == native.MOE_ERR_INVALID_ARG
