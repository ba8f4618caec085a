"""Shared helpers for the GPU parity tests (inputs from synth/, references from oracle/)."""
from __future__ import annotations

import numpy as np
import torch

import synth


def dev(a: np.ndarray, dtype=None, device="cuda") -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(a)).to(device)
    return t.view(dtype) if dtype is not None else t


def rms(a) -> float:
    return float(np.sqrt(np.mean(np.square(a, dtype=np.float64))))


def half_ulp_bf16(ref: np.ndarray) -> np.ndarray:
    a = np.abs(ref)
    e = np.floor(np.log2(np.where(a > 0, a, 1e-300)))
    return np.where(a > 0, np.exp2(e - 8), 0.0)


def check_tol(got, ref, rel=1e-2, abs_=1e-3, bf16_out=False, what=""):
    """The layer's value gate: max|err| <= rel*RMS(ref) + abs (+ half a bf16 ulp of the
    reference element when the output is bf16, its representation error)."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    tol = rel * rms(ref) + abs_
    err = np.abs(got - ref)
    lim = tol + (half_ulp_bf16(ref) if bf16_out else 0.0)
    bad = err > lim
    assert not bad.any(), (f"{what}: {int(bad.sum())} elements over tolerance; max|err| {err.max():.4e}, "
                           f"tol {tol:.4e}, rms {rms(ref):.4e}, worst at {np.unravel_index(np.argmax(err - lim), err.shape)}")
    return float(err.max() / max(rms(ref), 1e-30))


class W4Weights:
    """Host (for the oracle) and device (for the library) copies of one W4A16 expert set."""

    def __init__(self, seed, H, I, E):
        self.seed, self.H, self.I, self.E = seed, H, I, E
        self.W = synth.w4a16_weights(seed, H, I, range(E))
        self.d_w13_q = dev(self.W["w13_q"])
        self.d_w13_s = dev(self.W["w13_s"], torch.bfloat16)
        self.d_w2_q = dev(self.W["w2_q"])
        self.d_w2_s = dev(self.W["w2_s"], torch.bfloat16)


class W4Layer:
    """One routed W4A16 layer invocation: tokens x, router logits, and the expert weights."""

    def __init__(self, seed, T, H, I, E, k, zipf=0.0, logits=None, weights=None):
        self.seed, self.T, self.H, self.I, self.E, self.k = seed, T, H, I, E, k
        self.w = weights if weights is not None else W4Weights(seed, H, I, E)
        assert (self.w.H, self.w.I, self.w.E) == (H, I, E)
        self.W = self.w.W
        self.x = synth.x_bf16(seed, T, H)
        self.lg = synth.logits(seed, T, E, zipf_s=zipf) if logits is None else np.ascontiguousarray(logits, np.float32)
        self.d_x = dev(self.x, torch.bfloat16)
        self.d_lg = dev(self.lg)

    def forward(self, moe, ids, w, out_fp32):
        return moe.moe_w4a16_forward(self.d_x, ids, w, self.w.d_w13_q, self.w.d_w13_s, self.w.d_w2_q,
                                     self.w.d_w2_s, out_fp32=out_fp32)

    def oracle(self, oracle, ids, w, tokens=None):
        return oracle.w4a16_tokens(self.x, ids, w, self.W["w13_q"], self.W["w13_s"], self.W["w2_q"],
                                   self.W["w2_s"], tokens=tokens)
