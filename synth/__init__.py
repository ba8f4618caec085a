"""Seeded synthetic inputs shared by the CPU oracle and the CUDA path.

The generator lives in ``synth.c`` (compiled to ``libsynth.so`` next to it).  It holds no
arithmetic of the MoE layer: it only maps (seed, tensor id, flat index) to values with the
workloads' distributions.  Because it is counter-based, one expert's weights or one token's
row can be regenerated on their own, which is how the oracle gets the slices it needs for
full-size parity checks.

Distributions (the workload recipe):
  * x: bf16(N(0,1)), [T, H].
  * router logits: fp32 N(0,1), [T, E]; optionally plus b_e = -s*ln(r_e) with r a seeded
    permutation of ranks 1..E (Zipf(s)-shaped routing skew).
  * W4A16 weights: int32 words of eight uniform signed INT4 nibbles in [-8, 7]
    (nibble j = bits 4j..4j+3 = K index 8*word+j), w13 [E, 2I, H/8], w2 [E, H, I/8];
    bf16 scales bf16(U[0.005, 0.02]) per 32 K elements per output column,
    w13_s [E, 2I, H/32], w2_s [E, H, I/32].
  * W4A8: MXFP4 weights, codes uniform random bytes (two uniform E2M1 codes each, even K
    index in the low nibble), w13 [E, 2I, H/2], w2 [E, H, I/2]; E8M0 scale codes uniform in
    {120, 121, 122} (2^-7 .. 2^-5, so that the weights' spread matches the W4A16 ones) per 32 K
    elements, laid out [E, H/128, 2I, 4] and [E, I/128, H, 4]; activations bf16 x as above.
  * block-FP8: weights e4m3(N(0,1)) saturated at +-448, w13 [E, 2I, H], w2 [E, H, I];
    fp32 block scales U[0.001, 0.01] per 128x128 block, [E, 2I/128, H/128] and
    [E, H/128, I/128]; activations e4m3 with one fp32 scale per 1x128 group, produced from
    bf16(N(0,1)) by s = max(amax, 1e-10)/448, q = e4m3(z/s).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SO = os.path.join(_HERE, "libsynth.so")
_SRC = os.path.join(_HERE, "synth.c")

# Tensor ids: each logical tensor draws from its own stream.
TID = dict(x=1, logits=2, w13_q=3, w13_s=4, w2_q=5, w2_s=6, zipf_perm=7,
           x8=11, w13_8=13, w13_8s=14, w2_8=15, w2_8s=16,
           a=21, wq=23, ws=24, w13_mx=31, w13_mxs=32, w2_mx=33, w2_mxs=34)

W4_SCALE_RANGE = (0.005, 0.02)
FP8_SCALE_RANGE = (0.001, 0.01)


def build(force: bool = False) -> str:
    """Compile libsynth.so (plain C, gcc)."""
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-o", _SO, _SRC, "-lm", "-lpthread"])
    return _SO


_lib = None


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_SO)
        u64, i32, dbl, vp = ctypes.c_uint64, ctypes.c_int, ctypes.c_double, ctypes.c_void_p
        L.synth_key.restype = u64
        L.synth_key.argtypes = [u64, u64]
        L.synth_draw.restype = u64
        L.synth_draw.argtypes = [u64, u64, u64]
        L.synth_u32.argtypes = [u64, u64, u64, u64, vp, i32]
        L.synth_uniform_bf16.argtypes = [u64, u64, u64, u64, dbl, dbl, vp, i32]
        L.synth_uniform_f32.argtypes = [u64, u64, u64, u64, dbl, dbl, vp, i32]
        L.synth_normal_bf16.argtypes = [u64, u64, u64, u64, vp, i32]
        L.synth_normal_f32.argtypes = [u64, u64, u64, u64, vp, i32]
        L.synth_normal_e4m3.argtypes = [u64, u64, u64, u64, vp, i32]
        L.synth_zipf_bias.argtypes = [u64, u64, i32, dbl, vp]
        L.synth_logits.argtypes = [u64, u64, u64, u64, u64, i32, dbl, vp, i32]
        L.synth_act_e4m3.argtypes = [u64, u64, u64, u64, i32, vp, vp, i32]
        _lib = L
    return _lib


def nthreads() -> int:
    return max(1, os.cpu_count() or 1)


def _ptr(a) -> int:
    """Address of a numpy array or a torch (CPU) tensor."""
    if isinstance(a, np.ndarray):
        assert a.flags["C_CONTIGUOUS"]
        return a.ctypes.data
    assert a.is_contiguous() and a.device.type == "cpu"
    return a.data_ptr()


# ----------------------------------------------------------------- raw fills (any buffer)
def fill_u32(seed, tid, start, out):
    lib().synth_u32(seed, tid, start, out.size if isinstance(out, np.ndarray) else out.numel(),
                    _ptr(out), nthreads())


def fill_uniform_bf16(seed, tid, start, out, lo, hi):
    n = out.size if isinstance(out, np.ndarray) else out.numel()
    lib().synth_uniform_bf16(seed, tid, start, n, lo, hi, _ptr(out), nthreads())


def fill_uniform_f32(seed, tid, start, out, lo, hi):
    n = out.size if isinstance(out, np.ndarray) else out.numel()
    lib().synth_uniform_f32(seed, tid, start, n, lo, hi, _ptr(out), nthreads())


def fill_normal_bf16(seed, tid, start, out):
    n = out.size if isinstance(out, np.ndarray) else out.numel()
    lib().synth_normal_bf16(seed, tid, start, n, _ptr(out), nthreads())


def fill_normal_e4m3(seed, tid, start, out):
    n = out.size if isinstance(out, np.ndarray) else out.numel()
    lib().synth_normal_e4m3(seed, tid, start, n, _ptr(out), nthreads())


# ----------------------------------------------------------------- workload tensors (numpy)
def x_bf16(seed: int, T: int, H: int, t0: int = 0) -> np.ndarray:
    """bf16 bit patterns (uint16) of x rows [t0, t0+T) of a [*, H] activation tensor."""
    out = np.empty((T, H), np.uint16)
    fill_normal_bf16(seed, TID["x"], t0 * H, out)
    return out


def logits(seed: int, T: int, E: int, zipf_s: float = 0.0, t0: int = 0) -> np.ndarray:
    out = np.empty((T, E), np.float32)
    lib().synth_logits(seed, TID["logits"], TID["zipf_perm"], t0, T, E, float(zipf_s), out.ctypes.data,
                       nthreads())
    return out


def zipf_bias(seed: int, E: int, s: float) -> np.ndarray:
    out = np.empty(E, np.float64)
    lib().synth_zipf_bias(seed, TID["zipf_perm"], E, float(s), out.ctypes.data)
    return out


def w4a16_weights(seed: int, H: int, I: int, experts) -> dict:
    """INT4/bf16 weights for the listed global expert ids (in that order).

    Expert e of the full tensors occupies flat elements [e*per, (e+1)*per), so a subset
    reproduces exactly the corresponding slices of the full [E, ...] tensors."""
    experts = list(experts)
    n = len(experts)
    w13_q = np.empty((n, 2 * I, H // 8), np.int32)
    w13_s = np.empty((n, 2 * I, H // 32), np.uint16)
    w2_q = np.empty((n, H, I // 8), np.int32)
    w2_s = np.empty((n, H, I // 32), np.uint16)
    lo, hi = W4_SCALE_RANGE
    for i, e in enumerate(experts):
        e = int(e)  # a numpy int32 id would overflow the flat offset
        fill_u32(seed, TID["w13_q"], e * w13_q[0].size, w13_q[i])
        fill_uniform_bf16(seed, TID["w13_s"], e * w13_s[0].size, w13_s[i], lo, hi)
        fill_u32(seed, TID["w2_q"], e * w2_q[0].size, w2_q[i])
        fill_uniform_bf16(seed, TID["w2_s"], e * w2_s[0].size, w2_s[i], lo, hi)
    return dict(w13_q=w13_q, w13_s=w13_s, w2_q=w2_q, w2_s=w2_s)


def fp8_weights(seed: int, H: int, I: int, experts) -> dict:
    experts = list(experts)
    n = len(experts)
    w13 = np.empty((n, 2 * I, H), np.uint8)
    w13_s = np.empty((n, 2 * I // 128, H // 128), np.float32)
    w2 = np.empty((n, H, I), np.uint8)
    w2_s = np.empty((n, H // 128, I // 128), np.float32)
    lo, hi = FP8_SCALE_RANGE
    for i, e in enumerate(experts):
        e = int(e)  # a numpy int32 id would overflow the flat offset
        fill_normal_e4m3(seed, TID["w13_8"], e * w13[0].size, w13[i])
        fill_uniform_f32(seed, TID["w13_8s"], e * w13_s[0].size, w13_s[i], lo, hi)
        fill_normal_e4m3(seed, TID["w2_8"], e * w2[0].size, w2[i])
        fill_uniform_f32(seed, TID["w2_8s"], e * w2_s[0].size, w2_s[i], lo, hi)
    return dict(w13=w13, w13_s=w13_s, w2=w2, w2_s=w2_s)


MX_SCALE_CODES = (120, 121, 122)


def _mx_scales(seed, tid, start, out):
    u = np.empty(out.size, np.uint32)
    fill_u32(seed, tid, start, u)
    out.reshape(-1)[:] = (MX_SCALE_CODES[0] + u % len(MX_SCALE_CODES)).astype(np.uint8)


def mxfp4_weights(seed: int, H: int, I: int, experts) -> dict:
    """MXFP4 weights for the listed global expert ids (in that order), slices of the full
    [E, ...] tensors like w4a16_weights."""
    experts = list(experts)
    n = len(experts)
    w13 = np.empty((n, 2 * I, H // 2), np.uint8)
    w13_sf = np.empty((n, H // 128, 2 * I, 4), np.uint8)
    w2 = np.empty((n, H, I // 2), np.uint8)
    w2_sf = np.empty((n, I // 128, H, 4), np.uint8)
    for i, e in enumerate(experts):
        e = int(e)  # a numpy int32 id would overflow the flat offset
        fill_u32(seed, TID["w13_mx"], e * w13[0].size // 4, w13[i].view(np.uint32))
        _mx_scales(seed, TID["w13_mxs"], e * w13_sf[0].size, w13_sf[i])
        fill_u32(seed, TID["w2_mx"], e * w2[0].size // 4, w2[i].view(np.uint32))
        _mx_scales(seed, TID["w2_mxs"], e * w2_sf[0].size, w2_sf[i])
    return dict(w13=w13, w13_sf=w13_sf, w2=w2, w2_sf=w2_sf)


def x_e4m3(seed: int, T: int, H: int, t0: int = 0):
    q = np.empty((T, H), np.uint8)
    s = np.empty((T, H // 128), np.float32)
    lib().synth_act_e4m3(seed, TID["x8"], t0, T, H, q.ctypes.data, s.ctypes.data, nthreads())
    return q, s


def gemm_operands(seed: int, M: int, K: int, N: int):
    """Single-expert W4A16 GEMM operands: a bf16 [M,K], w_q int32 [1,N,K/8], w_s bf16 [1,N,K/32]."""
    a = np.empty((M, K), np.uint16)
    fill_normal_bf16(seed, TID["a"], 0, a)
    w_q = np.empty((1, N, K // 8), np.int32)
    fill_u32(seed, TID["wq"], 0, w_q)
    w_s = np.empty((1, N, K // 32), np.uint16)
    fill_uniform_bf16(seed, TID["ws"], 0, w_s, *W4_SCALE_RANGE)
    return a, w_q, w_s

