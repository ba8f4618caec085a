"""The C-ABI library: loads without a GPU, exports every symbol include/moe.h declares, and
rejects bad arguments synchronously.  Every call here with fake pointers fails an argument,
shape or workspace check before anything is enqueued, so no kernel ever sees those pointers,
with or without a GPU present."""
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


def test_binding_structs_match_the_header(native, tmp_path):
    """The Python argument structs have the header's field offsets and sizes (a C program built
    against include/moe.h prints them)."""
    import shutil
    import subprocess

    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    fields = {"moe_w4a16_args": [f for f, _ in native.W4A16Args._fields_],
              "moe_blockfp8_args": [f for f, _ in native.BlockFP8Args._fields_],
              "moe_w4a8_args": [f for f, _ in native.W4A8Args._fields_]}
    lines = ["#include <stdio.h>", "#include <stddef.h>", '#include "moe.h"', "int main(void) {"]
    for st, names in fields.items():
        lines.append(f'  printf("{st} size %zu\\n", sizeof({st}));')
        for n in names:
            lines.append(f'  printf("{st} {n} %zu\\n", offsetof({st}, {n}));')
    lines += ["  return 0;", "}"]
    src = tmp_path / "layout.c"
    src.write_text("\n".join(lines) + "\n")
    exe = tmp_path / "layout"
    cuda_inc = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "include")
    subprocess.check_call([gcc, "-I", os.path.join(ROOT, "include"), "-I", cuda_inc, "-o", str(exe), str(src)])
    got = {}
    for line in subprocess.check_output([str(exe)]).decode().splitlines():
        st, n, v = line.split()
        got[(st, n)] = int(v)
    for st, cls in (("moe_w4a16_args", native.W4A16Args), ("moe_blockfp8_args", native.BlockFP8Args),
                    ("moe_w4a8_args", native.W4A8Args)):
        assert got[(st, "size")] == ctypes.sizeof(cls), st
        for n in fields[st]:
            assert got[(st, n)] == getattr(cls, n).offset, (st, n)


def _w4(native, **kw):
    fake = 1 << 20
    d = dict(x=fake, topk_ids=fake, topk_w=fake, w13_q=fake, w13_s=fake, w2_q=fake, w2_s=fake,
             T=64, H=7168, I=2048, E=384, k=8, out=fake, out_fp32=0)
    d.update(kw)
    return native.W4A16Args(*[d[f] for f, _ in native.W4A16Args._fields_])


def _f8(native, **kw):
    fake = 1 << 20
    d = dict(x=fake, xs=fake, topk_ids=fake, topk_w=fake, w13=fake, w13_s=fake, w2=fake, w2_s=fake,
             T=64, H=7168, I=2048, E=256, k=8, out=fake, out_fp32=0)
    d.update(kw)
    return native.BlockFP8Args(*[d[f] for f, _ in native.BlockFP8Args._fields_])


def _mx(native, **kw):
    fake = 1 << 20
    d = dict(x=fake, topk_ids=fake, topk_w=fake, w13=fake, w13_sf=fake, w2=fake, w2_sf=fake,
             T=64, H=7168, I=2048, E=384, k=8, out=fake, out_fp32=0)
    d.update(kw)
    return native.W4A8Args(*[d[f] for f, _ in native.W4A8Args._fields_])


# shapes outside the documented limits: T >= 1, 1 <= k <= E <= 1024, H and I multiples of 128
BAD_SHAPES = [dict(T=0), dict(k=0), dict(E=0), dict(E=1025, k=8), dict(k=9, E=8), dict(H=7100), dict(I=2000),
              dict(H=0), dict(I=64)]
# pointers the calls need aligned (16 bytes for tensors read as vectors, 4 for scalars)
BAD_PTRS_W4 = ["x", "w13_q", "w13_s", "w2_q", "w2_s", "out"]
BAD_PTRS_F8 = ["x", "w13", "w2", "out"]


@pytest.mark.parametrize("kw", BAD_SHAPES, ids=lambda d: ",".join(f"{a}={b}" for a, b in d.items()))
def test_forward_shape_limits(native, kw):
    L = native.lib
    fake = ctypes.c_void_p(1 << 20)
    a = _w4(native, **kw)
    assert L.moe_w4a16_forward(ctypes.byref(a), fake, 1 << 40, None) == native.MOE_ERR_UNSUPPORTED
    assert L.moe_w4a16_workspace_size(a.T, a.H, a.I, a.E, a.k) == 0
    f = _f8(native, **kw)
    assert L.moe_blockfp8_forward(ctypes.byref(f), fake, 1 << 40, None) == native.MOE_ERR_UNSUPPORTED
    assert L.moe_blockfp8_workspace_size(f.T, f.H, f.I, f.E, f.k) == 0
    m = _mx(native, **kw)
    assert L.moe_w4a8_forward(ctypes.byref(m), fake, 1 << 40, None) == native.MOE_ERR_UNSUPPORTED
    assert L.moe_w4a8_workspace_size(m.T, m.H, m.I, m.E, m.k) == 0


@pytest.mark.parametrize("field", BAD_PTRS_W4)
def test_w4a16_forward_rejects_misaligned_or_null(native, field):
    L = native.lib
    fake = ctypes.c_void_p(1 << 20)
    for bad in (0, (1 << 20) + 8):
        a = _w4(native, **{field: bad})
        assert L.moe_w4a16_forward(ctypes.byref(a), fake, 1 << 40, None) == native.MOE_ERR_INVALID_ARG, (field, bad)
    a = _w4(native, topk_ids=(1 << 20) + 2)
    assert L.moe_w4a16_forward(ctypes.byref(a), fake, 1 << 40, None) == native.MOE_ERR_INVALID_ARG
    a = _w4(native)
    assert L.moe_w4a16_forward(ctypes.byref(a), ctypes.c_void_p((1 << 20) + 16), 1 << 40, None) == \
        native.MOE_ERR_INVALID_ARG  # workspace base must be 256-byte aligned


@pytest.mark.parametrize("field", BAD_PTRS_F8)
def test_blockfp8_forward_rejects_misaligned_or_null(native, field):
    L = native.lib
    fake = ctypes.c_void_p(1 << 20)
    for bad in (0, (1 << 20) + 8):
        f = _f8(native, **{field: bad})
        assert L.moe_blockfp8_forward(ctypes.byref(f), fake, 1 << 40, None) == native.MOE_ERR_INVALID_ARG, (field, bad)
    f = _f8(native, xs=(1 << 20) + 2)
    assert L.moe_blockfp8_forward(ctypes.byref(f), fake, 1 << 40, None) == native.MOE_ERR_INVALID_ARG


@pytest.mark.parametrize("field,bad", [("x", 8), ("w13", 16), ("w13_sf", 8), ("w2", 16), ("w2_sf", 8), ("out", 8),
                                       ("topk_ids", 2), ("topk_w", 2), ("x", None), ("w13", None)])
def test_w4a8_forward_rejects_misaligned_or_null(native, field, bad):
    """The packed weights need 32-byte alignment (the TMA's 4-bit unpacking mode), the rest 16
    (vector reads) or 4 (scalars)."""
    L = native.lib
    fake = ctypes.c_void_p(1 << 20)
    m = _mx(native, **{field: 0 if bad is None else (1 << 20) + bad})
    assert L.moe_w4a8_forward(ctypes.byref(m), fake, 1 << 40, None) == native.MOE_ERR_INVALID_ARG
    m = _mx(native)
    need = L.moe_w4a8_workspace_size(m.T, m.H, m.I, m.E, m.k)
    assert need > 0
    assert L.moe_w4a8_forward(ctypes.byref(m), fake, need - 1, None) == native.MOE_ERR_WORKSPACE
    assert L.moe_w4a8_forward(ctypes.byref(m), ctypes.c_void_p((1 << 20) + 16), 1 << 40, None) == \
        native.MOE_ERR_INVALID_ARG


def test_forward_workspace_one_byte_short(native):
    L = native.lib
    fake = ctypes.c_void_p(1 << 20)
    a = _w4(native)
    need = L.moe_w4a16_workspace_size(a.T, a.H, a.I, a.E, a.k)
    assert L.moe_w4a16_forward(ctypes.byref(a), fake, need - 1, None) == native.MOE_ERR_WORKSPACE
    f = _f8(native)
    need = L.moe_blockfp8_workspace_size(f.T, f.H, f.I, f.E, f.k)
    assert need > 0
    assert L.moe_blockfp8_forward(ctypes.byref(f), fake, need - 1, None) == native.MOE_ERR_WORKSPACE


@pytest.mark.parametrize("M,K,N,E", [(0, 7168, 512, 1), (1, 7100, 512, 1), (1, 7168, 500, 1), (1, 64, 512, 1),
                                     (1, 7168, 512, 0), (1, 7168, 512, 1025)])
def test_gemm_shape_limits(native, M, K, N, E):
    L = native.lib
    fake = ctypes.c_void_p(1 << 20)
    assert L.moe_w4a16_gemm_workspace_size(M, K, N, E) == 0
    assert L.moe_w4a16_gemm(fake, 1, fake, fake, fake, M, K, N, E, fake, 0, fake, 1 << 40, None) == \
        native.MOE_ERR_UNSUPPORTED


def test_gemm_alignment_and_workspace(native):
    L = native.lib
    ok, bad = ctypes.c_void_p(1 << 20), ctypes.c_void_p((1 << 20) + 8)
    M, K, N, E = 64, 7168, 512, 2
    need = L.moe_w4a16_gemm_workspace_size(M, K, N, E)
    args = [ok, 1, ok, ok, ok, M, K, N, E, ok, 0, ok, need, None]
    for i in (0, 2, 3, 9):  # a, w_q, w_s, out
        a = list(args)
        a[i] = bad
        assert L.moe_w4a16_gemm(*a) == native.MOE_ERR_INVALID_ARG, i
    a = list(args)
    a[12] = need - 1
    assert L.moe_w4a16_gemm(*a) == native.MOE_ERR_WORKSPACE


def test_route_and_align_limits(native):
    L = native.lib
    p = ctypes.c_void_p(1 << 20)
    for T, E, k in ((0, 8, 2), (4, 8, 0), (4, 1025, 8), (4, 0, 0)):
        assert L.moe_route(p, T, E, k, 1, p, p, None) == native.MOE_ERR_UNSUPPORTED, (T, E, k)
    assert L.moe_route(ctypes.c_void_p((1 << 20) + 2), 4, 8, 2, 1, p, p, None) == native.MOE_ERR_INVALID_ARG
    ws = L.moe_align_workspace_size(4, 2, 8)
    assert L.moe_align(p, 0, 2, 8, 16, p, p, p, p, p, ws, None) == native.MOE_ERR_UNSUPPORTED
    assert L.moe_align(p, 4, 2, 1025, 16, p, p, p, p, p, 1 << 30, None) == native.MOE_ERR_UNSUPPORTED
    assert L.moe_align(ctypes.c_void_p((1 << 20) + 2), 4, 2, 8, 16, p, p, p, p, p, ws, None) == \
        native.MOE_ERR_INVALID_ARG
    assert L.moe_align(p, 4, 2, 8, 16, p, p, p, p, p, ws - 1, None) == native.MOE_ERR_WORKSPACE


def test_align_noalloc_limits(native):
    """The allocation-free alignment call has a fixed 131072-int scratch array: one histogram
    of E experts per 512-pair chunk, so ceil(T*k/512) * E may not exceed it."""
    L = native.lib
    p = ctypes.c_void_p(1 << 20)
    # one pair past the limit (128 chunks x 1024 experts = 131072 fit): refused before any launch.
    # A call at the limit passes every check and would launch kernels on these fake pointers on
    # a machine with a GPU, so it is exercised only with real buffers in the GPU test
    # (test_zz_no_alloc.py).
    T, k, E = 65536, 1, 1024
    assert L.moe_align_noalloc(p, T + 1, k, E, 16, p, p, p, p, None) == native.MOE_ERR_UNSUPPORTED
    assert L.moe_align_noalloc(p, 0, 2, 8, 16, p, p, p, p, None) == native.MOE_ERR_UNSUPPORTED
    assert L.moe_align_noalloc(p, 4, 2, 8, 0, p, p, p, p, None) == native.MOE_ERR_UNSUPPORTED
    assert L.moe_align_noalloc(ctypes.c_void_p((1 << 20) + 2), 4, 2, 8, 16, p, p, p, p, None) == \
        native.MOE_ERR_INVALID_ARG
