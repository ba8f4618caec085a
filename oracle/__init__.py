"""CPU oracle for the routed W4A16 / block-FP8 / W4A8 MoE layer (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may
import this package.  The product path never does: it has no CPU fallback.  The oracle
(``oracle.c``, plain C compiled with gcc into ``liboracle.so``) shares no code with the CUDA
library; the only thing both sides share is the seeded input generator in ``synth/``.

Every function below is a thin ctypes marshaller around the C definition of the same name;
the arithmetic and its citations are in ``oracle.c``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SO = os.path.join(_HERE, "liboracle.so")
_SRC = os.path.join(_HERE, "oracle.c")


def build(force: bool = False) -> str:
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-o", _SO, _SRC, "-lm", "-lpthread"])
    return _SO


_lib = None


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_SO)
        i32, vp, f32 = ctypes.c_int, ctypes.c_void_p, ctypes.c_float
        L.oracle_bf16.restype = ctypes.c_double
        L.oracle_bf16.argtypes = [ctypes.c_uint16]
        L.oracle_f16.restype = ctypes.c_double
        L.oracle_f16.argtypes = [ctypes.c_uint16]
        L.oracle_int4.restype = i32
        L.oracle_int4.argtypes = [ctypes.c_uint32, i32]
        L.oracle_e4m3.restype = ctypes.c_double
        L.oracle_e4m3.argtypes = [ctypes.c_uint8]
        L.oracle_e4m3_encode.restype = ctypes.c_uint8
        L.oracle_e4m3_encode.argtypes = [f32]
        L.oracle_silu.restype = ctypes.c_double
        L.oracle_silu.argtypes = [ctypes.c_double]
        L.oracle_fp8_requant.restype = f32
        L.oracle_fp8_requant.argtypes = [vp, vp]
        L.oracle_route.argtypes = [vp, i32, i32, i32, i32, vp, vp, vp]
        L.oracle_align.restype = i32
        L.oracle_align.argtypes = [vp, i32, i32, i32, i32, vp, vp, vp, vp]
        L.oracle_w4a16_tokens.argtypes = [vp, vp, vp, i32, i32, i32, i32, i32, vp, vp, vp, vp, vp, i32, vp, vp,
                                          vp, i32]
        L.oracle_w4a16_gemm.argtypes = [vp, i32, vp, vp, vp, i32, i32, i32, i32, vp]
        L.oracle_fp8_tokens.argtypes = [vp, vp, vp, vp, i32, i32, i32, i32, i32, vp, vp, vp, vp, vp, i32, vp, vp,
                                        i32]
        L.oracle_e2m1.restype = ctypes.c_double
        L.oracle_e2m1.argtypes = [ctypes.c_uint8]
        L.oracle_e8m0.restype = ctypes.c_double
        L.oracle_e8m0.argtypes = [ctypes.c_uint8]
        L.oracle_mx_quant32.restype = ctypes.c_uint8
        L.oracle_mx_quant32.argtypes = [vp, vp]
        L.oracle_w4a8_tokens.argtypes = [vp, vp, vp, i32, i32, i32, i32, i32, vp, vp, vp, vp, vp, i32, vp, vp, i32]
        _lib = L
    return _lib


def nthreads() -> int:
    return max(1, os.cpu_count() or 1)


def _c(a, dtype):
    a = np.ascontiguousarray(a, dtype=dtype)
    return a, a.ctypes.data


# scalar decoders (exposed for the pins)
def bf16(h: int) -> float:
    return lib().oracle_bf16(h)


def f16(h: int) -> float:
    return lib().oracle_f16(h)


def int4(word: int, j: int) -> int:
    return lib().oracle_int4(word & 0xFFFFFFFF, j)


def e4m3(b: int) -> float:
    return lib().oracle_e4m3(b)


def e4m3_encode(x: float) -> int:
    return lib().oracle_e4m3_encode(x)


def silu(g: float) -> float:
    return lib().oracle_silu(g)


def fp8_requant(h):
    """1x128 group -> (e4m3 codes uint8 [128], fp32 scale)."""
    h_c, hp = _c(h, np.float32)
    assert h_c.shape == (128,)
    q = np.empty(128, np.uint8)
    s = lib().oracle_fp8_requant(hp, q.ctypes.data)
    return q, s


def route(logits: np.ndarray, k: int, renormalize: bool = True):
    """-> (ids int32 [T,k], w fp32 [T,k], w fp64 [T,k])."""
    lg, lp = _c(logits, np.float32)
    T, E = lg.shape
    ids = np.empty((T, k), np.int32)
    w32 = np.empty((T, k), np.float32)
    w64 = np.empty((T, k), np.float64)
    lib().oracle_route(lp, T, E, k, int(renormalize), ids.ctypes.data, w32.ctypes.data, w64.ctypes.data)
    return ids, w32, w64


def align(ids: np.ndarray, E: int, align: int):
    """-> dict(counts, offsets, sorted_ids [offsets[E]], inv_pos, bad)."""
    ids_c, ip = _c(ids, np.int32)
    T, k = ids_c.shape
    cap = T * k + E * (align - 1)
    counts = np.empty(E, np.int32)
    offsets = np.empty(E + 1, np.int32)
    sorted_ids = np.empty(max(cap, 1), np.int32)
    inv_pos = np.empty(T * k, np.int32)
    bad = lib().oracle_align(ip, T, k, E, align, counts.ctypes.data, offsets.ctypes.data, sorted_ids.ctypes.data,
                             inv_pos.ctypes.data)
    return dict(counts=counts, offsets=offsets, sorted_ids=sorted_ids[: offsets[E]].copy(), inv_pos=inv_pos,
                bad=bad)


def w4a16_tokens(x, ids, w, w13_q, w13_s, w2_q, w2_s, tokens=None, want_h=False, want_g=False, threads=None):
    """Routed W4A16 layer output in fp64 for `tokens` (default: all) -> out [n,H] (+ h, g)."""
    x_c, xp = _c(x, np.uint16)
    ids_c, idp = _c(ids, np.int32)
    w_c, wp = _c(w, np.float32)
    q13, q13p = _c(w13_q, np.int32)
    s13, s13p = _c(w13_s, np.uint16)
    q2, q2p = _c(w2_q, np.int32)
    s2, s2p = _c(w2_s, np.uint16)
    T, H = x_c.shape
    k = ids_c.shape[1]
    E, twoI = q13.shape[0], q13.shape[1]
    I = twoI // 2
    assert q13.shape == (E, 2 * I, H // 8) and s13.shape == (E, 2 * I, H // 32)
    assert q2.shape == (E, H, I // 8) and s2.shape == (E, H, I // 32)
    tok = np.arange(T, dtype=np.int32) if tokens is None else np.ascontiguousarray(tokens, np.int32)
    n = len(tok)
    out = np.empty((n, H), np.float64)
    h = np.empty((n, k, I), np.float64) if want_h else None
    g = np.empty((n, k, 2 * I), np.float64) if want_g else None
    lib().oracle_w4a16_tokens(xp, idp, wp, T, H, I, E, k, q13p, s13p, q2p, s2p, tok.ctypes.data, n,
                              out.ctypes.data, h.ctypes.data if want_h else None,
                              g.ctypes.data if want_g else None, threads or nthreads())
    res = [out]
    if want_h:
        res.append(h)
    if want_g:
        res.append(g)
    return res[0] if len(res) == 1 else tuple(res)


def w4a16_gemm(a, a_is_bf16, w_q, w_s, expert_offsets):
    a_c, ap = _c(a, np.uint16)
    q, qp = _c(w_q, np.int32)
    s, sp = _c(w_s, np.uint16)
    off, offp = _c(expert_offsets, np.int32)
    M, K = a_c.shape
    E, N = q.shape[0], q.shape[1]
    out = np.empty((M, N), np.float64)
    lib().oracle_w4a16_gemm(ap, int(a_is_bf16), qp, sp, offp, M, K, N, E, out.ctypes.data)
    return out


def fp8_tokens(x, xs, ids, w, w13, w13_s, w2, w2_s, tokens=None, want_hq=False, threads=None):
    x_c, xp = _c(x, np.uint8)
    xs_c, xsp = _c(xs, np.float32)
    ids_c, idp = _c(ids, np.int32)
    w_c, wp = _c(w, np.float32)
    a13, a13p = _c(w13, np.uint8)
    b13, b13p = _c(w13_s, np.float32)
    a2, a2p = _c(w2, np.uint8)
    b2, b2p = _c(w2_s, np.float32)
    T, H = x_c.shape
    k = ids_c.shape[1]
    E, twoI = a13.shape[0], a13.shape[1]
    I = twoI // 2
    tok = np.arange(T, dtype=np.int32) if tokens is None else np.ascontiguousarray(tokens, np.int32)
    n = len(tok)
    out = np.empty((n, H), np.float64)
    hq = np.empty((n, k, I), np.float32) if want_hq else None
    lib().oracle_fp8_tokens(xp, xsp, idp, wp, T, H, I, E, k, a13p, b13p, a2p, b2p, tok.ctypes.data, n,
                            out.ctypes.data, hq.ctypes.data if want_hq else None, threads or nthreads())
    return (out, hq) if want_hq else out


def e2m1(c: int) -> float:
    return lib().oracle_e2m1(c)


def e8m0(c: int) -> float:
    return lib().oracle_e8m0(c)


def mx_quant32(v):
    """32 fp32 values -> (e4m3 codes uint8 [32], E8M0 scale code)."""
    v_c, vp = _c(v, np.float32)
    assert v_c.shape == (32,)
    q = np.empty(32, np.uint8)
    sc = lib().oracle_mx_quant32(vp, q.ctypes.data)
    return q, sc


def w4a8_tokens(x, ids, w, w13, w13_sf, w2, w2_sf, tokens=None, want_hq=False, threads=None):
    """Routed W4A8 (MXFP4 weights, MX-FP8 activations) layer output in fp64 for `tokens`."""
    x_c, xp = _c(x, np.uint16)
    ids_c, idp = _c(ids, np.int32)
    w_c, wp = _c(w, np.float32)
    a13, a13p = _c(w13, np.uint8)
    b13, b13p = _c(w13_sf, np.uint8)
    a2, a2p = _c(w2, np.uint8)
    b2, b2p = _c(w2_sf, np.uint8)
    T, H = x_c.shape
    k = ids_c.shape[1]
    E, twoI = a13.shape[0], a13.shape[1]
    I = twoI // 2
    assert a13.shape == (E, 2 * I, H // 2) and b13.shape == (E, H // 128, 2 * I, 4)
    assert a2.shape == (E, H, I // 2) and b2.shape == (E, I // 128, H, 4)
    tok = np.arange(T, dtype=np.int32) if tokens is None else np.ascontiguousarray(tokens, np.int32)
    n = len(tok)
    out = np.empty((n, H), np.float64)
    hq = np.empty((n, k, I), np.float32) if want_hq else None
    lib().oracle_w4a8_tokens(xp, idp, wp, T, H, I, E, k, a13p, b13p, a2p, b2p, tok.ctypes.data, n,
                             out.ctypes.data, hq.ctypes.data if want_hq else None, threads or nthreads())
    return (out, hq) if want_hq else out
