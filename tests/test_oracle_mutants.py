"""The oracle's pins catch plausible mistakes.

Each case below plants one mistake in a copy of oracle/oracle.c (a dropped sign, a reversed
index, a swapped operand, a wrong constant, a broken tie rule), builds that copy with gcc,
points the oracle package at it and runs the pin tests of tests/test_oracle_*.py.  At least
one pin must fail for every mistake.  Every planted index stays inside its array, so a mutant
can give wrong numbers but cannot touch memory it does not own.  CPU only.
"""
import ctypes
import os
import subprocess

import pytest

import oracle
import test_oracle_formats as F
import test_oracle_layer as LY
import test_oracle_mx as MX
import test_oracle_route_align as RA

SRC = os.path.join(os.path.dirname(oracle.__file__), "oracle.c")

# (name, text in oracle.c, replacement, which occurrence of the text)
MUTANTS = [
    # number formats
    ("int4_unsigned", "return n >= 8 ? n - 16 : n;", "return n;", 0),
    ("int4_offset_binary", "return n >= 8 ? n - 16 : n;", "return n - 8;", 0),
    ("int4_nibble_order", "(word >> (4 * j))", "(word >> (4 * (7 - j)))", 0),
    ("bf16_shift", "uint32_t u = (uint32_t)h << 16;", "uint32_t u = (uint32_t)h << 15;", 0),
    ("f16_bias", "ldexp(1.0 + f / 1024.0, e - 15)", "ldexp(1.0 + f / 1024.0, e - 14)", 0),
    ("e4m3_bias", "v = ldexp(1.0 + m / 8.0, e - 7);", "v = ldexp(1.0 + m / 8.0, e - 8);", 0),
    ("e4m3_subnormal", "ldexp((double)m / 8.0, -6)", "ldexp((double)m / 8.0, -7)", 0),
    ("e4m3_ties_to_odd", "(c & 1) == 0 && (best & 1) == 1", "(c & 1) == 1 && (best & 1) == 0", 0),
    ("silu_sign", "return g / (1.0 + exp(-g));", "return g / (1.0 + exp(g));", 0),
    # routing
    ("route_ties_higher_index", "l[e] > l[best]) best = e;", "l[e] >= l[best]) best = e;", 0),
    ("route_smallest_logits", "l[e] > l[best]) best = e;", "l[e] < l[best]) best = e;", 0),
    ("route_renormalise_flag_inverted", "if (renormalize) w /= S;", "if (!renormalize) w /= S;", 0),
    # alignment
    ("align_unstable", "for (int p = 0; p < P; ++p) /* ascending p: stable */",
     "for (int p = P - 1; p >= 0; --p)", 0),
    ("align_sentinel", "sorted_ids[offsets[e] + r] = P;", "sorted_ids[offsets[e] + r] = -1;", 0),
    ("align_no_padding", "(counts[e] + align - 1) / align * align", "counts[e]", 0),
    # W4A16 layer and GEMM
    ("w4_scale_group_shifted", "s[(size_t)n * (K / 32) + kk / 32]", "s[(size_t)n * (K / 32) + (kk / 32 + 1) % (K / 32)]", 0),
    ("w4_nibble_shifted", "oracle_int4(word, kk % 8)", "oracle_int4(word, (kk + 1) % 8)", 0),
    ("w4_gate_up_swapped", "h[j] = oracle_silu(g[j]) * g[I + j];", "h[j] = oracle_silu(g[I + j]) * g[j];", 0),
    ("w4_up_dropped", "h[j] = oracle_silu(g[j]) * g[I + j];", "h[j] = oracle_silu(g[j]);", 0),
    ("w4_gate_up_k_reversed", "acc += xr[c] * w4(q13, s13, H, n, c);", "acc += xr[c] * w4(q13, s13, H, n, H - 1 - c);", 0),
    ("w4_down_k_reversed", "acc += h[j] * w4(q2, s2, I, c, j);", "acc += h[j] * w4(q2, s2, I, c, I - 1 - j);", 0),
    ("w4_combine_weight_dropped", "o[c] += ws * acc;", "o[c] += acc;", 0),
    ("w4_combine_slot_reversed", "double ws = (double)J->w[(size_t)t * k + s];",
     "double ws = (double)J->w[(size_t)t * k + (k - 1 - s)];", 0),
    ("gemm_bf16_f16_swapped", "ar[c] = a_is_bf16 ? oracle_bf16(b) : oracle_f16(b);",
     "ar[c] = a_is_bf16 ? oracle_f16(b) : oracle_bf16(b);", 0),
    # block-FP8 layer
    ("fp8_requant_max_240", "/ 448.0f;", "/ 240.0f;", 0),
    ("fp8_requant_floor", "(amax > 1e-10f ? amax : 1e-10f)", "(amax > 1e-10f ? amax : 1.0f)", 0),
    ("fp8_no_requant", "hd[gi * 128 + j] = oracle_e4m3(qc[j]) * (double)sc;", "hd[gi * 128 + j] = hf[gi * 128 + j];", 0),
    ("fp8_x_scale_shifted", "J->xs[(size_t)t * GH + c / 128]", "J->xs[(size_t)t * GH + (c / 128 + 1) % GH]", 0),
    ("fp8_w13_scale_transposed", "s13[(size_t)(n / 128) * GH + c / 128]",
     "s13[(size_t)(c / 128 % (2 * I / 128)) * GH + (n / 128) % GH]", 0),
    ("fp8_w2_scale_transposed", "s2[(size_t)(c / 128) * GI + j / 128]",
     "s2[(size_t)(j / 128 % (H / 128)) * GI + (c / 128) % GI]", 0),
    ("fp8_gate_up_swapped", "hf[j] = (float)(oracle_silu(g[j]) * g[I + j]);",
     "hf[j] = (float)(oracle_silu(g[I + j]) * g[j]);", 0),
    ("fp8_combine_weight_dropped", "o[c] += ws * acc;", "o[c] += acc;", 1),
    # W4A8 (MXFP4 x MX-FP8) layer
    ("e2m1_bias", "ldexp(1.0 + 0.5 * m, e - 1)", "ldexp(1.0 + 0.5 * m, e - 2)", 0),
    ("e2m1_subnormal", "e == 0 ? 0.5 * m", "e == 0 ? 1.0 * m", 0),
    ("e8m0_bias", "ldexp(1.0, (int)c - 127)", "ldexp(1.0, (int)c - 128)", 0),
    ("mx_range_224", "amax > ldexp(448.0, X)", "amax > ldexp(224.0, X)", 0),
    ("mx_scale_one_too_large", "amax > ldexp(448.0, X)", "amax >= ldexp(448.0, X)", 0),
    ("mx_zero_group_code", "int X = -127;", "int X = -126;", 0),
    ("mx_nibble_order", "(c & 1) ? (byte >> 4) : (byte & 15)", "(c & 1) ? (byte & 15) : (byte >> 4)", 0),
    ("mx_scale_rows_and_blocks_swapped", "sf[((size_t)(c / 128) * R + n) * 4 + (c / 32) % 4]",
     "sf[((size_t)(n % (K / 128)) * R + (c / 128) % R) * 4 + (c / 32) % 4]", 0),
    ("mx_scale_group_shifted", "* 4 + (c / 32) % 4]", "* 4 + (c / 32 + 1) % 4]", 0),
    ("mx_x_not_quantized", "xr[g0 + j] = oracle_e4m3(qc[j]) * sc;", "xr[g0 + j] = v[j];", 0),
    ("mx_h_not_requantized", "hd[g0 + j] = oracle_e4m3(qc[j]) * sc;", "hd[g0 + j] = hf[g0 + j];", 0),
    ("mx_gate_up_swapped", "hf[j] = (float)(oracle_silu(g[j]) * g[I + j]);",
     "hf[j] = (float)(oracle_silu(g[I + j]) * g[j]);", 1),
    ("mx_combine_weight_dropped", "o[c] += ws * acc;", "o[c] += acc;", 2),
]

# the pin tests, called as plain functions
PINS = [
    F.test_int4_hand_packed_words, F.test_bf16_pins, F.test_f16_pins_and_torch,
    F.test_e4m3_decode_pins_and_all_codes_vs_torch, F.test_e4m3_encode_pins, F.test_silu_closed_forms,
    lambda: RA.test_route_topk_matches_bruteforce_and_invariants(16, 8, 2, 0),
    RA.test_route_ties_lower_index_wins, RA.test_route_renormalised_weights_closed_form,
    RA.test_route_without_renormalisation_is_softmax_probability,
    lambda: RA.test_align_matches_bruteforce(100, 64, 6, 4, 16), RA.test_align_flags_out_of_range_ids,
    LY.test_gemm_one_hot_reads_hand_packed_weights, LY.test_gemm_rows_follow_expert_offsets,
    LY.test_gate_up_silu_down_closed_form, lambda: LY.test_dense_every_expert_then_mask_matches_routed(0),
    LY.test_e1_k1_is_a_dense_ffn, LY.test_fp8_requant_pins, LY.test_fp8_one_hot_layer,
    lambda: LY.test_fp8_dense_then_mask(0),
    MX.test_e2m1_all_codes_hand_table, MX.test_e8m0_all_codes_vs_torch, MX.test_mx_quant_scale_pins,
    MX.test_mx_quant_random_groups_vs_closed_form_and_torch, MX.test_mx_quant_rounding_ties_to_even,
    MX.test_w4a8_one_hot_layer, lambda: MX.test_w4a8_dense_then_mask(0),
]


def _plant(text, old, new, which):
    at = -1
    for _ in range(which + 1):
        at = text.find(old, at + 1)
        assert at >= 0, f"mutation site not found: {old!r} (occurrence {which})"
    return text[:at] + new + text[at + len(old):]


def test_mutation_sites_are_where_expected():
    text = open(SRC).read()
    for name, old, _, which in MUTANTS:
        assert text.count(old) >= which + 1, name


@pytest.mark.parametrize("name,old,new,which", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_planted_mistake(name, old, new, which, tmp_path, monkeypatch):
    src = tmp_path / "oracle_mutant.c"
    so = tmp_path / "liboracle_mutant.so"
    src.write_text(_plant(open(SRC).read(), old, new, which))
    subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-o", str(so), str(src), "-lm", "-lpthread"])
    monkeypatch.setattr(oracle, "_SRC", str(src))
    monkeypatch.setattr(oracle, "_SO", str(so))
    monkeypatch.setattr(oracle, "_lib", None)
    assert isinstance(oracle.lib(), ctypes.CDLL) and oracle.lib()._name == str(so)
    caught = []
    for pin in PINS:
        try:
            pin()
        except AssertionError:
            caught.append(getattr(pin, "__name__", "pin"))
            break
    assert caught, f"no pin failed with the planted mistake {name}"


def test_pins_pass_on_the_unmodified_oracle():
    for pin in PINS:
        pin()
