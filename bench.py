"""Benchmark of the routed W4A16 MoE layer (router + align + permute + gate/up GEMM with SiLU*up
+ down GEMM + weighted combine) on B200, through the library's C ABI.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One JSON line on stdout (rank 0).  Workloads (seeded synthetic inputs):
  decode            T=64 tokens, hidden 7168, intermediate 2048, 384 experts, top-8, N(0,1) logits
  prefill           T=8192 tokens, same model, logits skewed by a Zipf(1.1) per-expert bias
  fp8_t{1,16,64,512,4096}   the block-FP8 layer, 256 experts, top-8
  w4a8_t64, w4a8_t8192      the W4A8 layer (MXFP4 weights, FP8 activations in 32-groups) on the
                            decode / prefill shapes and routing of the W4A16 model
  w4a8_t{1,16,512,4096}     the same layer at other token counts (N(0,1) routing)
  gemm_m{M}_k{K}_n{N}       the single-expert grouped GEMM sweep (no activation)
The layer models' experts (9.5 GB of INT4 weights + bf16 scales for W4A16) stay resident in HBM;
each step streams the active experts' weights (about 7 GB for decode), far more than the
126 MB L2, so no L2 flush is needed between layer steps (the GEMM sweep reads a 512 MB buffer
between steps instead).

--impl reference times the CPU oracle (the only other implementation of this layer; the source
pages ship no code) on a bounded sample of the same workload on the host cores.
Multi-GPU (torchrun, N>1): the layer does not shard; every rank runs an independent replica and
the line reports the max-over-ranks time.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

METRIC = "routed-MoE layer µs, TFLOPS and HBM GB/s (% roofline) at decode T=64 and prefill T=8192"
MODEL = dict(H=7168, I=2048, E=384, k=8)
WORKLOADS = {
    "decode": dict(kind="w4a16", T=64, zipf=0.0, steps=400, warmup=20),
    "prefill": dict(kind="w4a16", T=8192, zipf=1.1, steps=40, warmup=5),
}
for _t in (1, 16, 64, 512, 4096):  # block-FP8 layer, 256 experts
    WORKLOADS[f"fp8_t{_t}"] = dict(kind="fp8", T=_t, zipf=0.0, steps=200 if _t <= 512 else 60, warmup=10)
FP8_MODEL = dict(H=7168, I=2048, E=256, k=8)
# W4A8 layer: the W4A16 model's shapes and routing (384 experts, top-8), MXFP4 weights
WORKLOADS["w4a8_t64"] = dict(kind="w4a8", T=64, zipf=0.0, steps=400, warmup=20)
WORKLOADS["w4a8_t8192"] = dict(kind="w4a8", T=8192, zipf=1.1, steps=40, warmup=5)
for _t in (1, 16, 512, 4096):  # the token-count sweep of the same layer (N(0,1) routing)
    WORKLOADS[f"w4a8_t{_t}"] = dict(kind="w4a8", T=_t, zipf=0.0, steps=200 if _t <= 512 else 60, warmup=10)
# block-FP8 benchmark model: expert e holds the generated weights of expert e mod FP8_DISTINCT (each
# expert in its own memory); generating 11.3 GB of normal e4m3 values on the host takes minutes
FP8_DISTINCT = 16
FP8_DATA = (f"synthetic (seeded counter-based generator; expert e holds the generated weights of expert e mod "
            f"{FP8_DISTINCT}, each expert in its own memory)")
# the single-expert grouped-GEMM sweep: [M,7168]x[7168,512] and [M,256]x[256,7168]
for (_k, _n) in ((7168, 512), (256, 7168)):
    for _m in (1, 64, 512, 4096, 32768):
        WORKLOADS[f"gemm_m{_m}_k{_k}_n{_n}"] = dict(kind="gemm", M=_m, K=_k, N=_n, steps=50, warmup=5)
GEMM_METRIC = "grouped W4A16 GEMM µs (one expert, no activation) and % roofline"
W13_BYTES_PER_EXPERT = 2 * 2048 * 7168 // 2 + 2 * 2048 * (7168 // 32) * 2   # INT4 words + bf16 scales
W2_BYTES_PER_EXPERT = 7168 * 2048 // 2 + 7168 * (2048 // 32) * 2
W13_MX_BYTES_PER_EXPERT = 2 * 2048 * 7168 // 2 + 2 * 2048 * (7168 // 32)  # E2M1 codes + E8M0 scales
W2_MX_BYTES_PER_EXPERT = 7168 * 2048 // 2 + 7168 * (2048 // 32)


# Datasheet figures of a B200 (HGX): HBM3e 8 TB/s; dense tensor 2.25 PFLOP/s bf16/fp16, 4.5 fp8.
# Every fraction is reported against the measured peak (`frac`) and against these (`frac_spec`).
SPEC = dict(hbm=8000.0, bf16=2250.0, fp8=4500.0, src="vendor datasheet (HGX B200)")


def with_spec(roof: dict, spec_peak: float) -> dict:
    """`roof` plus the same achieved figure as a fraction of the datasheet peak."""
    roof = dict(roof)
    roof["spec_peak"] = spec_peak
    roof["frac_spec"] = round(roof["achieved"] / spec_peak, 4)
    roof["spec_source"] = SPEC["src"]
    return roof


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return dict(hbm=d["hbm_gbs"], bf16=d["bf16_tflops"], bf16_sus=d["bf16_tflops_sustained"], src="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sus=1400.0, src="fallback")


# source file of each grouped GEMM: a measured traffic figure stands only while it is unchanged
KERNEL_SOURCES = {"w4i8": "gemm_w4i8.cu", "w4a16": "gemm_w4a16.cu", "fp8": "gemm_fp8.cu", "mx": "gemm_mx.cu"}


def source_sha256(family: str) -> str:
    import hashlib
    path = os.path.join(ROOT, "quantized_mixture_experts_softmax_b200", "csrc", KERNEL_SOURCES[family])
    return hashlib.sha256(open(path, "rb").read()).hexdigest()


def load_traffic(workload: str, kernel: str, family: str):
    """DRAM bytes per launch of `kernel` on `workload` from an ncu summary under profiles/ (a line
    `traffic: workload=W kernel=K family=F bytes_per_launch=N source_sha256=H`), or None when there
    is none or the kernel's source changed since the counters were taken."""
    import glob
    import re
    sha = source_sha256(family)
    for path in sorted(glob.glob(os.path.join(ROOT, "profiles", "*.md"))):
        for line in open(path):
            m = re.match(r"\s*traffic: workload=(\S+) kernel=(\S+) family=(\S+) bytes_per_launch=(\d+) "
                         r"source_sha256=([0-9a-f]+)", line)
            if m and m.group(1) == workload and m.group(2) == kernel and m.group(3) == family and m.group(5) == sha:
                return int(m.group(4))
    return None


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples while the timed region runs."""

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = os.path.join("/tmp", f"moe_clocks_{os.getpid()}.csv")

    def __enter__(self):
        q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={q}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.2)
            self.proc.terminate()
            self.proc.wait(timeout=10)

    def summary(self):
        if not os.path.exists(self.path):
            return None
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        os.unlink(self.path)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


def dist_init():
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def max_over_ranks(v: float, world: int) -> float:
    """The slowest rank's time (every rank gets it); NCCL reduces a device tensor, gloo a host one."""
    if world == 1:
        return v
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def make_model(seed: int):
    """All 384 experts generated on the host by the seeded generator, copied to HBM."""
    import torch
    import synth
    H, I, E = MODEL["H"], MODEL["I"], MODEL["E"]
    lo, hi = synth.W4_SCALE_RANGE
    dev = torch.device("cuda")
    out = {}
    specs = [("w13_q", (E, 2 * I, H // 8), torch.int32, "u32"), ("w13_s", (E, 2 * I, H // 32), torch.bfloat16, "s"),
             ("w2_q", (E, H, I // 8), torch.int32, "u32"), ("w2_s", (E, H, I // 32), torch.bfloat16, "s")]
    for name, shape, dt, kind in specs:
        d = torch.empty(shape, dtype=dt, device=dev)
        per = int(np.prod(shape[1:]))
        chunk = 32  # experts per host chunk
        stage = torch.empty((chunk, *shape[1:]), dtype=torch.int32 if kind == "u32" else torch.int16,
                            pin_memory=True)
        for e0 in range(0, E, chunk):
            n = min(chunk, E - e0)
            buf = stage[:n]
            if kind == "u32":
                synth.fill_u32(seed, synth.TID[name], e0 * per, buf)
            else:
                synth.fill_uniform_bf16(seed, synth.TID[name], e0 * per, buf, lo, hi)
            d[e0:e0 + n].view(buf.dtype).copy_(buf, non_blocking=False)
        out[name] = d
    return out


def make_model_fp8(seed: int, distinct: int = 0):
    """All 256 block-FP8 experts, generated on the host by the seeded generator and copied to
    HBM.  With distinct > 0 only the first `distinct` experts are generated and expert e holds
    the weights of expert e mod distinct (every expert still has its own memory, so a step reads
    the same bytes from HBM; used by the default benchmark run, where generating 11.3 GB of
    normal e4m3 values on the host would take minutes)."""
    import torch
    import synth
    H, I, E = FP8_MODEL["H"], FP8_MODEL["I"], FP8_MODEL["E"]
    lo, hi = synth.FP8_SCALE_RANGE
    out = {}
    specs = [("w13", (E, 2 * I, H), torch.uint8, "w13_8"), ("w13_s", (E, 2 * I // 128, H // 128), torch.float32, "w13_8s"),
             ("w2", (E, H, I), torch.uint8, "w2_8"), ("w2_s", (E, H // 128, I // 128), torch.float32, "w2_8s")]
    gen = E if distinct <= 0 else min(distinct, E)
    for name, shape, dt, tid in specs:
        d = torch.empty(shape, dtype=dt, device="cuda")
        per = int(np.prod(shape[1:]))
        chunk = 16
        stage = torch.empty((chunk, *shape[1:]), dtype=dt, pin_memory=True)
        for e0 in range(0, gen, chunk):
            n = min(chunk, gen - e0)
            buf = stage[:n]
            if dt == torch.uint8:
                synth.fill_normal_e4m3(seed, synth.TID[tid], e0 * per, buf)
            else:
                synth.fill_uniform_f32(seed, synth.TID[tid], e0 * per, buf, lo, hi)
            d[e0:e0 + n].copy_(buf)
        for e0 in range(gen, E, gen):
            n = min(gen, E - e0)
            d[e0:e0 + n].copy_(d[:n])
        out[name] = d
    return out


def make_model_mx(seed: int):
    """All 384 MXFP4 experts (E2M1 codes and E8M0 scale codes), generated on the host by the
    seeded generator and copied to HBM."""
    import torch
    import synth
    H, I, E = MODEL["H"], MODEL["I"], MODEL["E"]
    out = {}
    chunk = 32
    for name, shape, tid in (("w13", (E, 2 * I, H // 2), "w13_mx"), ("w13_sf", (E, H // 128, 2 * I, 4), "w13_mxs"),
                             ("w2", (E, H, I // 2), "w2_mx"), ("w2_sf", (E, I // 128, H, 4), "w2_mxs")):
        d = torch.empty(shape, dtype=torch.uint8, device="cuda")
        per = int(np.prod(shape[1:]))
        for e0 in range(0, E, chunk):
            n = min(chunk, E - e0)
            buf = np.empty((n, *shape[1:]), np.uint8)
            if name.endswith("_sf"):
                synth._mx_scales(seed, synth.TID[tid], e0 * per, buf)
            else:
                synth.fill_u32(seed, synth.TID[tid], e0 * per // 4, buf.view(np.uint32))
            d[e0:e0 + n].copy_(torch.from_numpy(buf))
        out[name] = d
    return out


def make_inputs(seed: int, T: int, zipf: float, kind: str = "w4a16"):
    import synth
    if kind == "fp8":
        xq, xs = synth.x_e4m3(seed, T, FP8_MODEL["H"])
        return (xq, xs), synth.logits(seed, T, FP8_MODEL["E"], zipf_s=zipf)
    x = synth.x_bf16(seed, T, MODEL["H"])
    lg = synth.logits(seed, T, MODEL["E"], zipf_s=zipf)
    return x, lg


def layer_config(workload: str, kind: str, T: int, H: int, I: int, E: int, k: int, active: int, world: int) -> dict:
    """The `config` object of a layer workload's JSON line (the same for both arms)."""
    label = {"fp8": "block-FP8", "w4a8": "W4A8 (MXFP4 x FP8)"}.get(kind, "W4A16")
    return {"workload": f"{workload} {label} MoE layer T={T} H={H} I={I} E={E} "
                        f"top-{k}",
            "T": T, "H": H, "I": I, "E": E, "k": k, "active_experts": active,
            "parallelism": "replicas" if world > 1 else "single GPU",
            "l2": "no flush: the active experts' weights streamed per step exceed the 126 MB L2"}


def gemm_config(M: int, K: int, N: int) -> dict:
    """The `config` object of a single-GEMM sweep line (the same for both arms)."""
    return {"workload": f"single-expert W4A16 GEMM [{M},{K}]x[{K},{N}]", "M": M, "K": K, "N": N,
            "l2": "512 MB buffer read between steps; time = the library's kernels only"}


def run_gemm(args, world, rank):
    """The single-expert W4A16 GEMM sweep through moe_w4a16_gemm.  Small operands fit in L2, so
    a 512 MB buffer is read between steps (a read leaves no dirty lines to write back during the
    next step).  The step time is the call's device time: CUDA events just before and after the
    call, the flush excluded, averaged over the steps.  A second pass with the library's per-launch
    events (which keep consecutive kernels from overlapping) gives the per-kernel breakdown."""
    import torch
    import quantized_mixture_experts_softmax_b200 as moe
    import synth

    wl = WORKLOADS[args.workload]
    M, K, N = wl["M"], wl["K"], wl["N"]
    steps = args.steps if args.steps is not None else wl["steps"]
    warmup = max(3, args.warmup if args.warmup is not None else wl["warmup"])
    a, w_q, w_s = synth.gemm_operands(0, M, K, N)
    d_a = torch.from_numpy(a).cuda().view(torch.bfloat16)
    d_q = torch.from_numpy(w_q).cuda()
    d_s = torch.from_numpy(w_s).cuda().view(torch.bfloat16)
    off = torch.tensor([0, M], dtype=torch.int32, device="cuda")
    out = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(max(moe.moe_w4a16_gemm_workspace_size(M, K, N, 1), 1), dtype=torch.uint8, device="cuda")
    flush = torch.ones(128 << 20, dtype=torch.float32, device="cuda")  # 512 MB

    def step():
        moe.moe_w4a16_gemm(d_a, d_q, d_s, off, out=out, workspace=ws)

    for _ in range(warmup):
        flush.sum()
        step()
    torch.cuda.synchronize()
    assert moe.moe_get_device_status() == 0
    stream = torch.cuda.current_stream()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    with ClockSampler(torch.cuda.current_device()) as clk:
        barrier(world)
        for i in range(steps):
            flush.sum()
            ev[i][0].record(stream)
            step()
            ev[i][1].record(stream)
        torch.cuda.synchronize()
        barrier(world)
    ms_step = max_over_ranks(sum(a.elapsed_time(b) for a, b in ev) / steps, world)
    # per-kernel breakdown (events around every launch)
    moe.moe_timing_enable(True)
    moe.moe_timing_read()
    for _ in range(steps):
        flush.sum()
        step()
    moe.moe_timing_enable(False)
    kern = moe.moe_timing_read()
    assert moe.moe_get_device_status() == 0
    launches = sum(n for (_, n) in kern.values())
    peaks = load_peaks()
    bytes_ = K * N // 2 + (K // 32) * N * 2 + M * K * 2 + M * N * 2
    flops = 2.0 * M * N * K
    s_ = ms_step / 1e3
    hbm_bound = flops / bytes_ < peaks["bf16"] * 1e3 / peaks["hbm"]
    if hbm_bound:
        ach = bytes_ / s_ / 1e9
        roof = with_spec(dict(kernel="all", bound="hbm", achieved=round(ach, 1), peak=peaks["hbm"], unit="GB/s",
                              frac=round(ach / peaks["hbm"], 4), traffic=None,
                              peak_source=peaks["src"] + " (copy, burst)", algorithmic_bytes_per_launch=int(bytes_)),
                         SPEC["hbm"])
    else:
        ach = flops / s_ / 1e12
        roof = with_spec(dict(kernel="all", bound="tensor", achieved=round(ach, 1), peak=peaks["bf16"],
                              unit="TFLOP/s", frac=round(ach / peaks["bf16"], 4), traffic=None,
                              peak_source=peaks["src"] + " bf16 GEMM, burst", algorithmic_flops_per_launch=flops),
                         SPEC["bf16"])
    return {
        "metric": GEMM_METRIC, "value": round(ms_step * 1e3, 2), "unit": "µs/GEMM", "n_gpus": world,
        "steps": steps, "warmup": warmup, "ms_per_step": round(ms_step, 4), "higher_is_better": False,
        "scaling": "weak", "vs_baseline": None,
        "dtype": "w4a16 as int8 MMA + fp32 promotion" if M <= 64 else "w4a16 (fp16 MMA, fp32 acc)",
        "data": "synthetic (seeded counter-based generator)",
        "config": gemm_config(M, K, N),
        "kernels_ms_per_step": {k_: round(v[0] / steps, 4) for k_, v in kern.items()},
        "gpu_launches": launches, "roofline": roof, "clocks": clk.summary(),
    }


def _phase_roofline(kern, suffix, alg_bytes, alg_flops, t_peak, t_peak_src, peaks, traffic, t_spec):
    """Roofline of one GEMM phase (gate/up or down): the kernels whose names end with `suffix`
    (one launch each per step: the int8-MMA kernel for experts with few rows, the fp16 one for
    the rest), algorithmic bytes / flops of the phase over their summed time per step."""
    ms = sum(v[0] for n, v in kern.items() if n.endswith(suffix))
    launches = sum(v[1] for n, v in kern.items() if n.endswith(suffix))
    names = sorted(n for n in kern if n.endswith(suffix))
    if not names or ms <= 0:
        return None
    steps = max(v[1] for n, v in kern.items() if n.endswith(suffix))
    per_s = ms / steps / 1e3
    hbm_bound = (alg_flops / alg_bytes) < (t_peak * 1e3 / peaks["hbm"])
    common = dict(kernel=" + ".join(names), launches_per_step=launches // steps, launch_ms=round(per_s * 1e3, 4),
                  traffic=traffic, algorithmic_bytes_per_launch=int(alg_bytes), algorithmic_flops_per_launch=alg_flops)
    if hbm_bound:
        ach = alg_bytes / per_s / 1e9
        return with_spec(dict(bound="hbm", achieved=round(ach, 1), peak=peaks["hbm"], unit="GB/s",
                              frac=round(ach / peaks["hbm"], 4), peak_source=peaks["src"] + " (copy, burst)",
                              **common), SPEC["hbm"])
    ach = alg_flops / per_s / 1e12
    return with_spec(dict(bound="tensor", achieved=round(ach, 1), peak=t_peak, unit="TFLOP/s",
                          frac=round(ach / t_peak, 4), peak_source=t_peak_src, **common), t_spec)


def measure_layer(args, workload, W, world):
    """One layer workload on resident weights W: device-timed steps (route + layer, inputs in
    HBM), CUDA-graph replays, the end-to-end variant with host buffers, per-kernel times and the
    roofline of each GEMM phase.  Returns (result dict, host inputs for the CPU baseline)."""
    import torch
    import quantized_mixture_experts_softmax_b200 as moe

    wl = WORKLOADS[workload]
    kind = wl["kind"]
    M = FP8_MODEL if kind == "fp8" else MODEL
    T, H, I, E, k = wl["T"], M["H"], M["I"], M["E"], M["k"]
    steps = args.steps if args.steps is not None else wl["steps"]
    warmup = args.warmup if args.warmup is not None else wl["warmup"]
    warmup = max(3, warmup)
    seed = 0
    x_h, lg_h = make_inputs(seed, T, wl["zipf"], kind)
    lg = torch.from_numpy(lg_h).cuda()
    ids = torch.empty(T, k, dtype=torch.int32, device="cuda")
    tw = torch.empty(T, k, dtype=torch.float32, device="cuda")
    out = torch.empty(T, H, dtype=torch.bfloat16, device="cuda")
    if kind == "fp8":
        x = torch.from_numpy(x_h[0]).cuda()
        xs = torch.from_numpy(x_h[1]).cuda()
        ws = torch.empty(moe.moe_blockfp8_workspace_size(T, H, I, E, k), dtype=torch.uint8, device="cuda")

        def forward(xx, xxs):
            moe.moe_blockfp8_forward(xx, xxs, ids, tw, W["w13"], W["w13_s"], W["w2"], W["w2_s"], out=out,
                                     workspace=ws)
    elif kind == "w4a8":
        x = torch.from_numpy(x_h).cuda().view(torch.bfloat16)
        xs = None
        ws = torch.empty(moe.moe_w4a8_workspace_size(T, H, I, E, k), dtype=torch.uint8, device="cuda")

        def forward(xx, xxs):
            moe.moe_w4a8_forward(xx, ids, tw, W["w13"], W["w13_sf"], W["w2"], W["w2_sf"], out=out, workspace=ws)
    else:
        x = torch.from_numpy(x_h).cuda().view(torch.bfloat16)
        xs = None
        ws = torch.empty(moe.moe_w4a16_workspace_size(T, H, I, E, k), dtype=torch.uint8, device="cuda")

        def forward(xx, xxs):
            moe.moe_w4a16_forward(xx, ids, tw, W["w13_q"], W["w13_s"], W["w2_q"], W["w2_s"], out=out, workspace=ws)

    def step():
        moe.moe_route(lg, k, topk_ids=ids, topk_w=tw)
        forward(x, xs)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    assert moe.moe_get_device_status() == 0
    counts = np.bincount(ids.cpu().numpy().ravel(), minlength=E)
    active = int((counts > 0).sum())

    # ---- device-timed region (inputs resident in HBM)
    stream = torch.cuda.current_stream()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(torch.cuda.current_device()) as clk:
        moe.moe_timing_enable(True)
        moe.moe_timing_read()
        barrier(world)
        torch.cuda.synchronize()
        ev0.record(stream)
        for _ in range(steps):
            step()
        ev1.record(stream)
        torch.cuda.synchronize()
        barrier(world)
        moe.moe_timing_enable(False)
    kern = moe.moe_timing_read()
    ms_total = max_over_ranks(ev0.elapsed_time(ev1), world)
    assert moe.moe_get_device_status() == 0
    ms_step = ms_total / steps
    clocks = clk.summary()

    # ---- the same step replayed from one CUDA graph (host launch overhead removed)
    graph = None
    try:
        g = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            step()
        torch.cuda.current_stream().wait_stream(side)
        with torch.cuda.graph(g):
            step()
        for _ in range(3):
            g.replay()
        torch.cuda.synchronize()
        barrier(world)
        # an event between replays gives each replay's duration as well as the total
        reps = max(steps, 100)
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(reps + 1)]
        evs[0].record(stream)
        for i in range(reps):
            g.replay()
            evs[i + 1].record(stream)
        torch.cuda.synchronize()
        barrier(world)
        assert moe.moe_get_device_status() == 0
        per_us = np.array([evs[i].elapsed_time(evs[i + 1]) for i in range(reps)]) * 1e3
        stats = {name: round(max_over_ranks(float(v), world) / world, 2)
                 for name, v in (("median", np.median(per_us)), ("min", per_us.min()),
                                 ("p90", np.percentile(per_us, 90)))}
        graph = {"value": round(max_over_ranks(evs[0].elapsed_time(evs[-1]), world) / reps * 1e3 / world, 2),
                 "unit": "µs/layer", "replays": reps, **stats,
                 "note": "the timed step (route + layer) replayed from one CUDA graph; value = mean, "
                         "median/min/p90 over the replays (max over ranks)"}
        del g
    except Exception as exc:  # capture refused: report why instead of a number
        graph = {"value": None, "unit": "µs/layer", "note": f"capture failed: {type(exc).__name__}: {exc}"[:200]}

    # ---- end to end through the C ABI with host buffers (pinned), copies inside the region
    lg_pin = torch.from_numpy(lg_h).pin_memory()
    out_pin = torch.empty(T, H, dtype=torch.bfloat16).pin_memory()
    lg_d = torch.empty(T, E, dtype=torch.float32, device="cuda")
    if kind == "fp8":
        x_pin = torch.from_numpy(x_h[0]).pin_memory()
        xs_pin = torch.from_numpy(x_h[1]).pin_memory()
        x_d = torch.empty_like(x)
        xs_d = torch.empty_like(xs)
        h2d = T * H + T * (H // 128) * 4 + T * E * 4
    else:
        x_pin = torch.from_numpy(x_h).pin_memory()
        xs_pin = None
        x_d = torch.empty(T, H, dtype=torch.int16, device="cuda")
        xs_d = None
        h2d = T * H * 2 + T * E * 4
    d2h = T * H * 2

    def e2e_step():
        x_d.copy_(x_pin.view(x_d.dtype), non_blocking=True)
        if xs_d is not None:
            xs_d.copy_(xs_pin, non_blocking=True)
        lg_d.copy_(lg_pin, non_blocking=True)
        moe.moe_route(lg_d, k, topk_ids=ids, topk_w=tw)
        forward(x_d if kind == "fp8" else x_d.view(torch.bfloat16), xs_d)
        out_pin.copy_(out, non_blocking=True)

    for _ in range(3):
        e2e_step()
    e2e_steps = max(5, steps // 4)
    barrier(world)
    torch.cuda.synchronize()
    ev0.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    ev1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    ms_e2e = max_over_ranks(ev0.elapsed_time(ev1), world) / e2e_steps

    # ---- rooflines.  Algorithmic work: only what the method must move or compute - the active
    # experts' weights, the layer input x (gate/up) and the layer output (down); the
    # expert-sorted activation copies and y round trips are overhead, not credit.
    peaks = load_peaks()
    P = T * k
    flops = 6.0 * P * H * I
    if kind == "fp8":
        w13_b = 2 * I * H + (2 * I // 128) * (H // 128) * 4
        w2_b = H * I + (H // 128) * (I // 128) * 4
        x_in = T * H + T * (H // 128) * 4
    elif kind == "w4a8":
        w13_b, w2_b = W13_MX_BYTES_PER_EXPERT, W2_MX_BYTES_PER_EXPERT
        x_in = T * H * 2
    else:
        w13_b, w2_b = W13_BYTES_PER_EXPERT, W2_BYTES_PER_EXPERT
        x_in = T * H * 2
    out_b = T * H * 2
    layer_bytes = active * (w13_b + w2_b) + x_in + out_b + T * E * 4
    # tensor peak for the contraction's own operand type: fp16 and int8 run at the measured bf16
    # rate, e4m3 (and the e2m1 x e4m3 block-scaled kind) at twice it (the nominal dense fp8 : bf16
    # ratio)
    f8 = kind in ("fp8", "w4a8")
    t_peak = peaks["bf16"] * (2.0 if f8 else 1.0)
    t_peak_src = peaks["src"] + (" bf16 GEMM x 2 (nominal fp8:bf16)" if f8 else " bf16 GEMM, burst")
    family = {"fp8": "fp8", "w4a8": "mx"}.get(kind, "w4i8" if T <= 64 else "w4a16")
    no_traffic = bool(args.tokens or args.experts)
    phases = {}
    for suffix, alg_b, alg_f in (("gate_up", active * w13_b + x_in, 2.0 * P * H * 2 * I),
                                 ("down", active * w2_b + out_b, 2.0 * P * I * H)):
        names = [n for n in kern if n.endswith(suffix)]
        traffic = None
        if len(names) == 1 and not no_traffic:
            traffic = load_traffic(workload, names[0], family)
        phases[suffix] = _phase_roofline(kern, suffix, alg_b, alg_f, t_peak, t_peak_src, peaks, traffic,
                                         SPEC["fp8" if f8 else "bf16"])
    dom = max((v for v in phases.values() if v), key=lambda r: r["launch_ms"], default=None)
    launches = sum(n for (_, n) in kern.values())
    res = {
        "metric": METRIC, "value": round(ms_step * 1e3 / world, 2), "unit": "µs/layer",
        "n_gpus": world, "steps": steps, "warmup": warmup, "ms_per_step": round(ms_step, 4),
        "higher_is_better": False, "scaling": "weak", "vs_baseline": None,
        "dtype": {"fp8": "e4m3 (fp32 acc)",
                  "mx": "w4a8: MXFP4 weights x e4m3 activations, E8M0 scales per 32 K applied by the "
                        "block-scaled MMA (fp32 acc)",
                  "w4a16": "w4a16: fp16 MMA (fp32 acc) for experts with many rows, int8 MMA on 16-bit "
                           "fixed-point activations + fp32 promotion for the rest",
                  "w4i8": "w4a16 as int8 MMA (u8 weights x 16-bit fixed-point activations, s32) + fp32 promotion"}[family],
        "data": FP8_DATA if kind == "fp8" else "synthetic (seeded counter-based generator; random-init quantized weights)",
        "config": layer_config(workload, kind, T, H, I, E, k, active, world),
        "layer": {"us": round(ms_step * 1e3, 2), "tflops": round(flops / (ms_step * 1e-3) / 1e12, 2),
                  "hbm_gbs": round(layer_bytes / (ms_step * 1e-3) / 1e9, 1),
                  "hbm_frac": round(layer_bytes / (ms_step * 1e-3) / 1e9 / peaks["hbm"], 4),
                  "tensor_frac": round(flops / (ms_step * 1e-3) / 1e12 / t_peak, 4),
                  "hbm_frac_spec": round(layer_bytes / (ms_step * 1e-3) / 1e9 / SPEC["hbm"], 4),
                  "tensor_frac_spec": round(flops / (ms_step * 1e-3) / 1e12 / SPEC["fp8" if f8 else "bf16"],
                                            4),
                  "algorithmic_bytes": int(layer_bytes), "flops": flops},
        "kernels_ms_per_step": {n: round(v[0] / steps, 4) for n, v in sorted(kern.items(), key=lambda kv: -kv[1][0])},
        "e2e": {"value": round(ms_e2e * 1e3, 2), "unit": "µs/layer", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h},
        "gpu_launches": launches,
        "graph": graph,
        "roofline": dom,
        "phases": phases,
        "clocks": clocks,
    }
    return res, (x_h, lg_h, T, kind)


def run_ours(args, world, rank):
    wl = WORKLOADS[args.workload]
    W = {"fp8": lambda: make_model_fp8(0, distinct=FP8_DISTINCT), "w4a8": lambda: make_model_mx(0)}.get(
        wl["kind"], lambda: make_model(0))()
    return measure_layer(args, args.workload, W, world)


# the objects the default run adds to the decode line, measured in the same process
DEFAULT_EXTRAS = ("prefill", "fp8_t64", "fp8_t4096", "w4a8_t64", "w4a8_t8192")
# keys of a workload's result that stay on the top-level line only
LINE_ONLY = ("metric", "n_gpus", "higher_is_better", "scaling", "vs_baseline", "data")


def run_default(args, world, rank):
    """The default benchmark: the decode T=64 line (its `value` is the headline), with the
    prefill T=8192 workload on the same resident 384-expert model, the block-FP8 layer at T=64
    and T=4096, and the W4A8 layer at T=64 and T=8192 as nested objects, each measured like the
    line itself, with its own CPU-oracle baseline on rank 0."""
    import torch
    W = make_model(0)
    res, inp = measure_layer(args, "decode", W, world)
    results = [(res, inp)]
    sub, inp_p = measure_layer(args, "prefill", W, world)
    res["prefill"] = {k_: v for k_, v in sub.items() if k_ not in LINE_ONLY}
    results.append((res["prefill"], inp_p))
    del W
    torch.cuda.empty_cache()
    if not args.no_fp8:
        W8 = make_model_fp8(0, distinct=FP8_DISTINCT)
        for wl in ("fp8_t64", "fp8_t4096"):
            sub, inp_f = measure_layer(args, wl, W8, world)
            res[wl] = {k_: v for k_, v in sub.items() if k_ not in LINE_ONLY}
            results.append((res[wl], inp_f))
        del W8
        torch.cuda.empty_cache()
    if not args.no_w4a8:
        WM = make_model_mx(0)
        for wl in ("w4a8_t64", "w4a8_t8192"):
            sub, inp_m = measure_layer(args, wl, WM, world)
            res[wl] = {k_: v for k_, v in sub.items() if k_ not in LINE_ONLY}
            results.append((res[wl], inp_m))
        del WM
        torch.cuda.empty_cache()
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        for obj, (x_h, lg_h, T, kind) in results:
            us, sample, cores, _ = oracle_sample_time(x_h, lg_h, T, kind, budget_s=8.0)
            obj["cpu_baseline"] = {"value": round(us, 1), "unit": "µs/layer", "cores": cores, "kind": "oracle",
                                   "sample": sample}
    return res


def oracle_sample_time(x_h, lg_h, T, kind="w4a16", budget_s=15.0):
    """CPU oracle on a bounded token sample of the same workload -> (us per layer, sample, cores)."""
    import oracle
    import synth
    M = FP8_MODEL if kind == "fp8" else MODEL
    k = M["k"]
    ids, w, _ = oracle.route(lg_h, k)
    cores = oracle.nthreads()

    W8 = synth.fp8_weights(0, M["H"], M["I"], range(FP8_DISTINCT)) if kind == "fp8" else None

    def run(n):
        tok = np.arange(n, dtype=np.int32)
        used = np.unique(ids[tok])
        remap = {int(e): i for i, e in enumerate(used)}
        ids_l = np.vectorize(lambda e: remap.get(int(e), 0))(ids[tok]).astype(np.int32)
        if kind == "fp8":  # the benchmark's model: expert e has the weights of expert e mod FP8_DISTINCT
            Wt = W8
            ids_l = (ids[tok] % FP8_DISTINCT).astype(np.int32)
            t0 = time.time()
            oracle.fp8_tokens(x_h[0][tok], x_h[1][tok], ids_l, w[tok], Wt["w13"], Wt["w13_s"], Wt["w2"], Wt["w2_s"])
        elif kind == "w4a8":
            Wt = synth.mxfp4_weights(0, M["H"], M["I"], used)
            t0 = time.time()
            oracle.w4a8_tokens(x_h[tok], ids_l, w[tok], Wt["w13"], Wt["w13_sf"], Wt["w2"], Wt["w2_sf"])
        else:
            Wt = synth.w4a16_weights(0, M["H"], M["I"], used)
            t0 = time.time()
            oracle.w4a16_tokens(x_h[tok], ids_l, w[tok], Wt["w13_q"], Wt["w13_s"], Wt["w2_q"], Wt["w2_s"])
        return time.time() - t0

    n_probe = max(1, min(T, cores))
    probe = run(n_probe)
    per_tok = probe / n_probe  # wall time per token with all cores busy
    n = int(min(T, max(n_probe, budget_s / max(per_tok, 1e-9))))
    el = run(n) if n > n_probe else probe
    us_layer = el / n * T * 1e6
    return us_layer, f"{n} of {T} tokens (all {k} experts each), extrapolated linearly to {T}", cores, 0.0


def gemm_oracle_time(M, K, N, budget_s=8.0):
    """CPU oracle of the single-expert GEMM on a bounded row sample -> (us per GEMM, sample, cores)."""
    import oracle
    import synth
    a, w_q, w_s = synth.gemm_operands(0, M, K, N)
    cores = oracle.nthreads()

    def run(n):
        t0 = time.time()
        oracle.w4a16_gemm(a[:n], True, w_q, w_s, np.array([0, n], np.int32))
        return time.time() - t0

    n_probe = max(1, min(M, cores))
    per_row = run(n_probe) / n_probe
    n = int(min(M, max(n_probe, budget_s / max(per_row, 1e-9))))
    el = run(n)
    return el / n * M * 1e6, f"{n} of {M} rows, extrapolated linearly to {M}", cores


def run_reference(args, world, rank):
    wl = WORKLOADS[args.workload]
    if wl["kind"] == "gemm":
        M, K, N = wl["M"], wl["K"], wl["N"]
        steps = args.steps if args.steps is not None else 3
        warmup = args.warmup if args.warmup is not None else 1
        vals, sample, cores = [], None, None
        for i in range(warmup + steps):
            us, sample, cores = gemm_oracle_time(M, K, N)
            if i >= warmup:
                vals.append(us)
        v = statistics.median(vals)
        return {
            "metric": GEMM_METRIC, "value": round(v, 1), "unit": "µs/GEMM", "n_gpus": world, "steps": steps,
            "warmup": warmup, "ms_per_step": round(v / 1e3, 3), "higher_is_better": False, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64 (oracle)", "data": "synthetic",
            "config": gemm_config(M, K, N), "impl": "reference",
            "cpu_baseline": {"value": round(v, 1), "unit": "µs/GEMM", "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": round(v, 1), "unit": "µs/GEMM", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        }
    import oracle
    M = FP8_MODEL if wl["kind"] == "fp8" else MODEL
    T = wl["T"]
    steps = args.steps if args.steps is not None else 3
    warmup = args.warmup if args.warmup is not None else 1
    x_h, lg_h = make_inputs(0, T, wl["zipf"], wl["kind"])
    active = int(np.unique(oracle.route(lg_h, M["k"])[0]).size)  # the routing both arms compute
    vals = []
    sample = cores = None
    for i in range(warmup + steps):
        us, sample, cores, _ = oracle_sample_time(x_h, lg_h, T, wl["kind"], budget_s=8.0)
        if i >= warmup:
            vals.append(us)
    v = statistics.median(vals)
    return {
        "metric": METRIC, "value": round(v, 1), "unit": "µs/layer", "n_gpus": world, "steps": steps,
        "warmup": warmup, "ms_per_step": round(v / 1e3, 3), "higher_is_better": False, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64 (oracle)", "data": "synthetic",
        "config": layer_config(args.workload, wl["kind"], T, M["H"], M["I"], M["E"], M["k"], active, world),
        "impl": "reference",
        "cpu_baseline": {"value": round(v, 1), "unit": "µs/layer", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(v, 1), "unit": "µs/layer", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None)
    ap.add_argument("--warmup", type=int, default=None)
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default=None,
                    help="one workload's line (default: decode, with prefill and block-FP8 objects)")
    ap.add_argument("--no-fp8", action="store_true", help="default run: leave out the block-FP8 objects")
    ap.add_argument("--no-w4a8", action="store_true", help="default run: leave out the W4A8 objects")
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--experts", type=int, default=None,
                    help="override the expert count (small profiling cases only; not a bench line)")
    ap.add_argument("--tokens", type=int, default=None,
                    help="override the workload's token count (small profiling cases only; not a bench line)")
    args = ap.parse_args()
    if args.experts:
        MODEL["E"] = args.experts
        FP8_MODEL["E"] = args.experts
    if args.tokens:
        WORKLOADS[args.workload or "decode"] = dict(WORKLOADS[args.workload or "decode"], T=args.tokens)

    if args.impl == "reference":
        args.workload = args.workload or "decode"
        rank = int(os.environ.get("RANK", "0"))
        if rank != 0:
            return
        print(json.dumps(run_reference(args, int(os.environ.get("WORLD_SIZE", "1")), rank)), flush=True)
        return

    world, rank, _ = dist_init()
    if args.workload is None:
        res = run_default(args, world, rank)
        if rank == 0:
            print(json.dumps(res), flush=True)
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return
    if WORKLOADS[args.workload]["kind"] == "gemm":
        res = run_gemm(args, world, rank)
        if rank == 0:
            print(json.dumps(res), flush=True)
        return
    res, (x_h, lg_h, T, kind) = run_ours(args, world, rank)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        us, sample, cores, _ = oracle_sample_time(x_h, lg_h, T, kind)
        res["cpu_baseline"] = {"value": round(us, 1), "unit": "µs/layer", "cores": cores, "kind": "oracle",
                               "sample": sample}
    if rank == 0:
        print(json.dumps(res), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
