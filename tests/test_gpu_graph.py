"""The layer calls that take a workspace enqueue only kernels on the caller's stream (no host
reads of device data, no allocation), so moe_route + the layer forward can be captured in a
CUDA graph.  A captured step replayed on new inputs written into the captured buffers must
give exactly the eager result (the same kernels run in both).
"""
import numpy as np
import pytest
import torch

import synth
from helpers import W4Weights, dev

pytestmark = pytest.mark.gpu
moe = pytest.importorskip("quantized_mixture_experts_softmax_b200")


def capture(step):
    g = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step()
    torch.cuda.current_stream().wait_stream(side)
    with torch.cuda.graph(g):
        step()
    return g


@pytest.mark.parametrize("T", [16, 200])  # the int8 decode-sized path and the fp16 path
def test_w4a16_step_replays_exactly(T):
    H, I, E, k = 256, 256, 8, 2
    wts = W4Weights(11, H, I, E)
    x = dev(synth.x_bf16(11, T, H), torch.bfloat16)
    lg = dev(synth.logits(11, T, E))
    ids = torch.empty(T, k, dtype=torch.int32, device="cuda")
    tw = torch.empty(T, k, dtype=torch.float32, device="cuda")
    out = torch.empty(T, H, dtype=torch.float32, device="cuda")
    ws = torch.empty(moe.moe_w4a16_workspace_size(T, H, I, E, k), dtype=torch.uint8, device="cuda")

    def step():
        moe.moe_route(lg, k, topk_ids=ids, topk_w=tw)
        moe.moe_w4a16_forward(x, ids, tw, wts.d_w13_q, wts.d_w13_s, wts.d_w2_q, wts.d_w2_s, out=out, out_fp32=True,
                              workspace=ws)

    g = capture(step)
    for seed in (12, 13):  # new inputs into the captured buffers
        x.copy_(dev(synth.x_bf16(seed, T, H), torch.bfloat16))
        lg.copy_(dev(synth.logits(seed, T, E)))
        g.replay()
        torch.cuda.synchronize()
        got = out.clone()
        step()
        torch.cuda.synchronize()
        assert moe.moe_get_device_status() == 0
        assert torch.equal(got, out), f"T={T} seed {seed}: graph replay differs from the eager step"
    del g


def test_blockfp8_step_replays_exactly():
    T, H, I, E, k = 24, 256, 256, 8, 2
    W = synth.fp8_weights(21, H, I, range(E))
    d = {n: dev(v) for n, v in W.items()}
    xq, xs = synth.x_e4m3(21, T, H)
    x, xsd = dev(xq), dev(xs)
    lg = dev(synth.logits(21, T, E))
    ids = torch.empty(T, k, dtype=torch.int32, device="cuda")
    tw = torch.empty(T, k, dtype=torch.float32, device="cuda")
    out = torch.empty(T, H, dtype=torch.float32, device="cuda")
    ws = torch.empty(moe.moe_blockfp8_workspace_size(T, H, I, E, k), dtype=torch.uint8, device="cuda")

    def step():
        moe.moe_route(lg, k, topk_ids=ids, topk_w=tw)
        moe.moe_blockfp8_forward(x, xsd, ids, tw, d["w13"], d["w13_s"], d["w2"], d["w2_s"], out=out, out_fp32=True,
                                 workspace=ws)

    g = capture(step)
    xq2, xs2 = synth.x_e4m3(22, T, H)
    x.copy_(dev(xq2))
    xsd.copy_(dev(xs2))
    g.replay()
    torch.cuda.synchronize()
    got = out.clone()
    step()
    torch.cuda.synchronize()
    assert moe.moe_get_device_status() == 0
    assert torch.equal(got, out), "graph replay differs from the eager step"
    assert np.isfinite(got.cpu().numpy()).all()
    del g
