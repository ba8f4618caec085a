"""Routed, weight-quantized Mixture-of-Experts layer for B200 (sm_100a).

A thin Python binding over the C ABI in ``include/moe.h`` (``libmoe.so``, built in-tree by
``build.py``).  Each function below has the name of the C entry point it calls and only
marshals arguments: it takes CUDA torch tensors, allocates outputs and workspaces with torch
when they are not given, passes raw device pointers and the current CUDA stream, and raises
:class:`MoeError` on any non-OK status.  Every step of the layer runs in the library's
kernels; there is no CPU or PyTorch fallback.
"""
from __future__ import annotations

import ctypes

import torch

from ._native import (MOE_ERR_CUDA, MOE_ERR_DEVICE_CHECK, MOE_ERR_INVALID_ARG, MOE_ERR_TIMEOUT,  # noqa: F401
                      MOE_ERR_UNSUPPORTED, MOE_ERR_WORKSPACE, MOE_OK, BlockFP8Args, MoeError, W4A8Args, W4A16Args, check,
                      lib)

__all__ = ["moe_route", "moe_blockfp8_intermediate", "moe_align", "moe_align_capacity", "moe_w4a16_forward", "moe_w4a16_workspace_size",
           "moe_blockfp8_forward", "moe_blockfp8_workspace_size", "moe_w4a8_forward", "moe_w4a8_workspace_size",
           "moe_w4a8_intermediate", "moe_w4a16_gemm", "moe_w4a16_gemm_workspace_size",
           "moe_get_device_status", "moe_debug_wait_timeout", "moe_timing_enable", "moe_timing_read", "MoeError",
           "lib"]


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _cuda(*ts):
    for t in ts:
        if t is not None and (not t.is_cuda or not t.is_contiguous()):
            raise ValueError("expected contiguous CUDA tensors")


def _workspace(nbytes: int, workspace, device):
    if workspace is not None:
        return workspace
    return torch.empty(max(int(nbytes), 1), dtype=torch.uint8, device=device)


def moe_route(logits: torch.Tensor, k: int, renormalize: bool = True, topk_ids=None, topk_w=None, stream=None):
    """logits fp32 [T,E] -> (topk_ids int32 [T,k], topk_w fp32 [T,k])."""
    _cuda(logits)
    T, E = logits.shape
    ids = topk_ids if topk_ids is not None else torch.empty(T, k, dtype=torch.int32, device=logits.device)
    w = topk_w if topk_w is not None else torch.empty(T, k, dtype=torch.float32, device=logits.device)
    check(lib.moe_route(_p(logits), T, E, k, int(renormalize), _p(ids), _p(w), _stream(stream)), "moe_route")
    return ids, w


def moe_align_capacity(T: int, k: int, E: int, align: int) -> int:
    return lib.moe_align_capacity(T, k, E, align)


def moe_align(topk_ids: torch.Tensor, E: int, align: int, workspace=None, stream=None) -> dict:
    """topk_ids int32 [T,k] -> dict(counts [E], offsets [E+1], sorted_ids [capacity], inv_pos [T*k])."""
    _cuda(topk_ids)
    T, k = topk_ids.shape
    dev = topk_ids.device
    cap = lib.moe_align_capacity(T, k, E, align)
    counts = torch.empty(E, dtype=torch.int32, device=dev)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    sorted_ids = torch.empty(max(cap, 1), dtype=torch.int32, device=dev)
    inv_pos = torch.empty(T * k, dtype=torch.int32, device=dev)
    nbytes = lib.moe_align_workspace_size(T, k, E)
    ws = _workspace(nbytes, workspace, dev)
    check(lib.moe_align(_p(topk_ids), T, k, E, align, _p(counts), _p(offsets), _p(sorted_ids), _p(inv_pos), _p(ws),
                        ws.numel() * ws.element_size(), _stream(stream)), "moe_align")
    return dict(counts=counts, offsets=offsets, sorted_ids=sorted_ids, inv_pos=inv_pos)


def moe_w4a16_workspace_size(T: int, H: int, I: int, E: int, k: int) -> int:
    return lib.moe_w4a16_workspace_size(T, H, I, E, k)


def moe_w4a16_forward(x, topk_ids, topk_w, w13_q, w13_s, w2_q, w2_s, out=None, out_fp32: bool = False,
                      workspace=None, stream=None) -> torch.Tensor:
    """Routed W4A16 layer.  x bf16 [T,H]; topk_ids int32 [T,k]; topk_w fp32 [T,k];
    w13_q int32 [E,2I,H/8]; w13_s bf16 [E,2I,H/32]; w2_q int32 [E,H,I/8]; w2_s bf16 [E,H,I/32]
    -> out bf16 [T,H] (fp32 if out_fp32)."""
    _cuda(x, topk_ids, topk_w, w13_q, w13_s, w2_q, w2_s, out)
    T, H = x.shape
    k = topk_ids.shape[1]
    E, twoI = w13_q.shape[0], w13_q.shape[1]
    I = twoI // 2
    if out is None:
        out = torch.empty(T, H, dtype=torch.float32 if out_fp32 else torch.bfloat16, device=x.device)
    nbytes = lib.moe_w4a16_workspace_size(T, H, I, E, k)
    ws = _workspace(nbytes, workspace, x.device)
    args = W4A16Args(x.data_ptr(), topk_ids.data_ptr(), topk_w.data_ptr(), w13_q.data_ptr(), w13_s.data_ptr(),
                     w2_q.data_ptr(), w2_s.data_ptr(), T, H, I, E, k, out.data_ptr(), int(out_fp32))
    check(lib.moe_w4a16_forward(ctypes.byref(args), _p(ws), ws.numel() * ws.element_size(), _stream(stream)),
          "moe_w4a16_forward")
    return out


def moe_blockfp8_workspace_size(T: int, H: int, I: int, E: int, k: int) -> int:
    return lib.moe_blockfp8_workspace_size(T, H, I, E, k)


def moe_blockfp8_forward(x, xs, topk_ids, topk_w, w13, w13_s, w2, w2_s, out=None, out_fp32: bool = False,
                         workspace=None, stream=None) -> torch.Tensor:
    """Routed block-FP8 layer.  x e4m3 (uint8) [T,H] + xs fp32 [T,H/128]; w13 e4m3 [E,2I,H] +
    fp32 [E,2I/128,H/128]; w2 e4m3 [E,H,I] + fp32 [E,H/128,I/128] -> out bf16/fp32 [T,H]."""
    _cuda(x, xs, topk_ids, topk_w, w13, w13_s, w2, w2_s, out)
    T, H = x.shape
    k = topk_ids.shape[1]
    E, twoI = w13.shape[0], w13.shape[1]
    I = twoI // 2
    if out is None:
        out = torch.empty(T, H, dtype=torch.float32 if out_fp32 else torch.bfloat16, device=x.device)
    nbytes = lib.moe_blockfp8_workspace_size(T, H, I, E, k)
    ws = _workspace(nbytes, workspace, x.device)
    args = BlockFP8Args(x.data_ptr(), xs.data_ptr(), topk_ids.data_ptr(), topk_w.data_ptr(), w13.data_ptr(),
                        w13_s.data_ptr(), w2.data_ptr(), w2_s.data_ptr(), T, H, I, E, k, out.data_ptr(),
                        int(out_fp32))
    check(lib.moe_blockfp8_forward(ctypes.byref(args), _p(ws), ws.numel() * ws.element_size(), _stream(stream)),
          "moe_blockfp8_forward")
    return out


def moe_blockfp8_intermediate(workspace: torch.Tensor, T: int, H: int, I: int, E: int, k: int) -> dict:
    """Views into the workspace of a finished moe_blockfp8_forward(T, H, I, E, k) call:
    inv_pos int32 [T*k], h e4m3 codes uint8 [T*k, I], h_scale_t fp32 [I/128, T*k]."""
    _cuda(workspace)
    ptrs = [ctypes.c_void_p() for _ in range(3)]
    check(lib.moe_blockfp8_intermediate(_p(workspace), T, H, I, E, k, *[ctypes.byref(q) for q in ptrs]),
          "moe_blockfp8_intermediate")
    raw = workspace.view(torch.uint8).reshape(-1)
    base = raw.data_ptr()

    def view(ptr, n, dtype):
        off = ptr.value - base
        return raw[off: off + n * torch.empty((), dtype=dtype).element_size()].view(dtype)

    P = T * k
    return dict(inv_pos=view(ptrs[0], P, torch.int32), h=view(ptrs[1], P * I, torch.uint8).view(P, I),
                h_scale_t=view(ptrs[2], (I // 128) * P, torch.float32).view(I // 128, P))


def moe_w4a8_workspace_size(T: int, H: int, I: int, E: int, k: int) -> int:
    return lib.moe_w4a8_workspace_size(T, H, I, E, k)


def moe_w4a8_forward(x, topk_ids, topk_w, w13, w13_sf, w2, w2_sf, out=None, out_fp32: bool = False,
                     workspace=None, stream=None) -> torch.Tensor:
    """Routed W4A8 layer (MXFP4 weights, FP8 activations with E8M0 scales per 32 K).  x bf16
    [T,H]; w13 uint8 [E,2I,H/2] (two E2M1 codes per byte) + E8M0 uint8 [E,H/128,2I,4]; w2 uint8
    [E,H,I/2] + [E,I/128,H,4] -> out bf16/fp32 [T,H]."""
    _cuda(x, topk_ids, topk_w, w13, w13_sf, w2, w2_sf, out)
    T, H = x.shape
    k = topk_ids.shape[1]
    E, twoI = w13.shape[0], w13.shape[1]
    I = twoI // 2
    if out is None:
        out = torch.empty(T, H, dtype=torch.float32 if out_fp32 else torch.bfloat16, device=x.device)
    nbytes = lib.moe_w4a8_workspace_size(T, H, I, E, k)
    ws = _workspace(nbytes, workspace, x.device)
    args = W4A8Args(x.data_ptr(), topk_ids.data_ptr(), topk_w.data_ptr(), w13.data_ptr(), w13_sf.data_ptr(),
                    w2.data_ptr(), w2_sf.data_ptr(), T, H, I, E, k, out.data_ptr(), int(out_fp32))
    check(lib.moe_w4a8_forward(ctypes.byref(args), _p(ws), ws.numel() * ws.element_size(), _stream(stream)),
          "moe_w4a8_forward")
    return out


def moe_w4a8_intermediate(workspace: torch.Tensor, T: int, H: int, I: int, E: int, k: int) -> dict:
    """Views into the workspace of a finished moe_w4a8_forward(T, H, I, E, k) call:
    inv_pos int32 [T*k], h e4m3 codes uint8 [T*k, I], h_sf E8M0 codes uint8 [I/128, T*k, 4]."""
    _cuda(workspace)
    ptrs = [ctypes.c_void_p() for _ in range(3)]
    check(lib.moe_w4a8_intermediate(_p(workspace), T, H, I, E, k, *[ctypes.byref(q) for q in ptrs]),
          "moe_w4a8_intermediate")
    raw = workspace.view(torch.uint8).reshape(-1)
    base = raw.data_ptr()
    P = T * k
    inv = raw[ptrs[0].value - base: ptrs[0].value - base + 4 * P].view(torch.int32)
    h = raw[ptrs[1].value - base: ptrs[1].value - base + P * I].view(P, I)
    h_sf = raw[ptrs[2].value - base: ptrs[2].value - base + (I // 128) * P * 4].view(I // 128, P, 4)
    return dict(inv_pos=inv, h=h, h_sf=h_sf)


def moe_w4a16_gemm_workspace_size(M: int, K: int, N: int, E: int) -> int:
    return lib.moe_w4a16_gemm_workspace_size(M, K, N, E)


def moe_w4a16_gemm(a, w_q, w_s, expert_offsets, out=None, out_fp32: bool = False, workspace=None,
                   stream=None) -> torch.Tensor:
    """Grouped W4A16 GEMM (no activation): a bf16/fp16 [M,K]; w_q int32 [E,N,K/8];
    w_s bf16 [E,N,K/32]; expert_offsets int32 [E+1] -> out bf16/fp32 [M,N]."""
    _cuda(a, w_q, w_s, expert_offsets, out)
    M, K = a.shape
    E, N = w_q.shape[0], w_q.shape[1]
    if a.dtype not in (torch.bfloat16, torch.float16):
        raise ValueError("a must be bf16 or fp16")
    want = torch.float32 if out_fp32 else torch.bfloat16
    if out is None:
        out = torch.empty(M, N, dtype=want, device=a.device)
    elif out.dtype != want or tuple(out.shape) != (M, N):
        raise ValueError(f"out must be {want} [{M}, {N}] (out_fp32={out_fp32})")
    nbytes = lib.moe_w4a16_gemm_workspace_size(M, K, N, E)
    ws = _workspace(nbytes, workspace, a.device)
    check(lib.moe_w4a16_gemm(_p(a), int(a.dtype == torch.bfloat16), _p(w_q), _p(w_s), _p(expert_offsets), M, K, N,
                             E, _p(out), int(out_fp32), _p(ws), ws.numel() * ws.element_size(), _stream(stream)),
          "moe_w4a16_gemm")
    return out


def moe_get_device_status(stream=None) -> int:
    """Synchronises the stream; returns (and clears) the device status word."""
    return lib.moe_get_device_status(_stream(stream))


def moe_debug_wait_timeout(limit_ns: int, stream=None) -> None:
    check(lib.moe_debug_wait_timeout(int(limit_ns), _stream(stream)), "moe_debug_wait_timeout")


def moe_timing_enable(enable: bool) -> None:
    lib.moe_timing_enable(int(enable))


def moe_timing_read() -> dict:
    """{kernel name: (summed ms, launches)} since the last read (synchronises the device)."""
    n = 64
    names = (ctypes.c_char_p * n)()
    ms = (ctypes.c_double * n)()
    cnt = (ctypes.c_int * n)()
    m = lib.moe_timing_read(names, ms, cnt, n)
    return {names[i].decode(): (ms[i], cnt[i]) for i in range(min(m, n))}
