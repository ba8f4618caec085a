"""Host-side logic of the benchmark that decides what its JSON line reports: the clock record
(throttle reasons that reject a run), the measured-traffic lookup (used only while the kernel
source is unchanged) and the per-expert weight bytes behind the roofline's algorithmic bytes.
No GPU."""
import hashlib
import os

import numpy as np

import bench
import synth


def test_clock_summary_median_max_and_reasons(tmp_path):
    clk = bench.ClockSampler(0)
    clk.path = str(tmp_path / "clocks.csv")
    # index, clocks.sm, clocks.max.sm, power, active mask, hw_slowdown, hw_thermal, sw_thermal, sw_power_cap
    rows = [
        "0, 1965, 1965, 640.1, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
        "0, 1860, 1965, 998.7, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
        "0, 1905, 1965, 990.2, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
        "0, [N/A], 1965, 0, 0x0, Not Active, Not Active, Not Active, Not Active",  # unreadable sample
        "short line",
    ]
    open(clk.path, "w").write("\n".join(rows) + "\n")
    s = clk.summary()
    assert s == {"sm_mhz": 1905.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"], "samples": 3}
    assert not os.path.exists(clk.path)  # the sample file is removed once read


def test_clock_summary_reports_slowdowns(tmp_path):
    clk = bench.ClockSampler(0)
    clk.path = str(tmp_path / "clocks.csv")
    open(clk.path, "w").write(
        "0, 1200, 1965, 700.0, 0x8, Active, Not Active, Active, Not Active\n")
    s = clk.summary()
    assert s["reasons"] == ["hw_slowdown", "sw_thermal_slowdown"]


def test_traffic_lookup_needs_the_current_kernel_source(tmp_path, monkeypatch):
    csrc = tmp_path / "quantized_mixture_experts_softmax_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "gemm_w4i8.cu").write_text("// kernel v2\n")
    (csrc / "gemm_w4a16.cu").write_text("// another kernel\n")
    sha_now = hashlib.sha256(b"// kernel v2\n").hexdigest()
    sha_old = hashlib.sha256(b"// kernel v1\n").hexdigest()
    prof = tmp_path / "profiles"
    prof.mkdir()
    (prof / "w4i8_decode.md").write_text(
        "# summary\n"
        f"traffic: workload=decode kernel=w4a16_gemm_down family=w4i8 bytes_per_launch=111 source_sha256={sha_old}\n"
        f"traffic: workload=decode kernel=w4a16_gemm_gate_up family=w4i8 bytes_per_launch=222 "
        f"source_sha256={sha_now}\n"
        f"traffic: workload=prefill kernel=w4a16_gemm_gate_up family=w4i8 bytes_per_launch=333 "
        f"source_sha256={sha_now}\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.load_traffic("decode", "w4a16_gemm_gate_up", "w4i8") == 222
    assert bench.load_traffic("prefill", "w4a16_gemm_gate_up", "w4i8") == 333
    assert bench.load_traffic("decode", "w4a16_gemm_down", "w4i8") is None  # counters of an older source
    assert bench.load_traffic("decode", "w4a16_gemm_gate_up", "w4a16") is None  # another kernel family


def test_weight_bytes_per_expert_match_the_stored_layout():
    H, I = bench.MODEL["H"], bench.MODEL["I"]
    W = synth.w4a16_weights(0, H, I, [0])
    assert W["w13_q"].nbytes + W["w13_s"].nbytes == bench.W13_BYTES_PER_EXPERT
    assert W["w2_q"].nbytes + W["w2_s"].nbytes == bench.W2_BYTES_PER_EXPERT
    # INT4: 8 weights per int32 word, one 2-byte scale per 32 weights
    assert bench.W13_BYTES_PER_EXPERT == 2 * I * H // 2 + 2 * I * H // 32 * 2
    assert W["w13_q"].dtype == np.int32 and W["w13_q"].shape == (1, 2 * I, H // 8)


def test_w4a8_weight_bytes_per_expert_match_the_stored_layout():
    H, I = bench.MODEL["H"], bench.MODEL["I"]
    W = synth.mxfp4_weights(0, H, I, [0])
    assert W["w13"].nbytes + W["w13_sf"].nbytes == bench.W13_MX_BYTES_PER_EXPERT
    assert W["w2"].nbytes + W["w2_sf"].nbytes == bench.W2_MX_BYTES_PER_EXPERT
    # MXFP4: two E2M1 codes per byte, one 1-byte E8M0 scale per 32 weights
    assert bench.W13_MX_BYTES_PER_EXPERT == 2 * I * H // 2 + 2 * I * H // 32
    assert W["w13"].shape == (1, 2 * I, H // 2) and W["w13_sf"].shape == (1, H // 128, 2 * I, 4)


def test_workloads_cover_the_layer_configurations():
    w = bench.WORKLOADS
    assert w["decode"]["T"] == 64 and w["prefill"]["T"] == 8192
    assert bench.MODEL == dict(H=7168, I=2048, E=384, k=8)
    assert bench.FP8_MODEL == dict(H=7168, I=2048, E=256, k=8)
    assert sorted(v["T"] for n, v in w.items() if n.startswith("fp8_")) == [1, 16, 64, 512, 4096]
    # W4A8 on the decode and prefill configurations (same model and routing) plus the T sweep
    assert w["w4a8_t64"] == dict(w["decode"], kind="w4a8") and w["w4a8_t8192"] == dict(w["prefill"], kind="w4a8")
    assert {"w4a8_t64", "w4a8_t8192"} <= set(bench.DEFAULT_EXTRAS)
    for v in w.values():
        assert v["warmup"] >= 3  # the timing rule's minimum


def _args(workload, steps=1, warmup=0):
    import argparse
    return argparse.Namespace(workload=workload, steps=steps, warmup=warmup, gpus=1, impl="reference",
                              no_cpu_baseline=False, experts=None, tokens=None)


def _check_reference_line(line, metric, unit):
    assert line["impl"] == "reference"
    assert line["metric"] == metric and line["unit"] == unit and line["higher_is_better"] is False
    assert line["value"] > 0 and line["steps"] == 1
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == line["value"] and cb["unit"] == unit and cb["cores"] >= 1
    assert "of" in cb["sample"]
    assert line["e2e"] == {"value": line["value"], "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_reference_arm_layer_line(monkeypatch):
    """The oracle arm prints the contract's line with the config our arm prints for the same
    workload (checked on a reduced model so that it runs in a moment)."""
    import oracle
    for key, v in dict(H=256, I=128, E=8, k=2).items():
        monkeypatch.setitem(bench.MODEL, key, v)
    monkeypatch.setitem(bench.WORKLOADS, "decode", dict(bench.WORKLOADS["decode"], T=16))
    line = bench.run_reference(_args("decode"), 1, 0)
    _check_reference_line(line, bench.METRIC, "µs/layer")
    _, lg = bench.make_inputs(0, 16, 0.0)
    active = int(np.unique(oracle.route(lg, 2)[0]).size)
    assert line["config"] == bench.layer_config("decode", "w4a16", 16, 256, 128, 8, 2, active, 1)
    assert line["cpu_baseline"]["sample"].startswith("16 of 16 tokens")


def test_reference_arm_gemm_line():
    line = bench.run_reference(_args("gemm_m1_k7168_n512"), 1, 0)
    _check_reference_line(line, bench.GEMM_METRIC, "µs/GEMM")
    assert line["config"] == bench.gemm_config(1, 7168, 512)


def test_fractions_against_measured_and_datasheet_peaks():
    """Every roofline object carries the achieved figure over the measured peak and over the
    datasheet peak, each named."""
    import bench
    r = bench.with_spec(dict(bound="hbm", achieved=6000.0, peak=6534.8, unit="GB/s", frac=round(6000 / 6534.8, 4)),
                        bench.SPEC["hbm"])
    assert r["frac"] == round(6000 / 6534.8, 4)
    assert r["frac_spec"] == 0.75 and r["spec_peak"] == 8000.0 and "datasheet" in r["spec_source"]
    assert bench.SPEC["bf16"] == 2250.0 and bench.SPEC["fp8"] == 2 * bench.SPEC["bf16"]
