"""The E8M0 exponent the CUDA kernels compute for an FP8 group (mx_exponent in csrc/common.cuh,
used by the W4A8 activation quantization and the h epilogue), checked on the CPU against its
definition - the smallest X in [-127, 127] with amax <= 448 * 2^X - over every finite float bit
pattern at a stride of 4099, plus, for each exponent field, the fractions around the 0.75
switch point (0x5FFFFF, 0x600000, 0x600001), zero and the extremes.  The function is compiled
by nvcc as host code from the library's own header; nothing runs on a GPU."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "quantized_mixture_experts_softmax_b200", "csrc")

PROGRAM = r"""
#include <cmath>
#include <cstdio>
#include <cstring>
#include "common.cuh"

static long n_checked = 0, n_bad = 0;
static void check(uint32_t u) {
  float f;
  std::memcpy(&f, &u, 4);
  int ref = -127;  // the definition, by search
  while (ref < 127 && (double)f > std::ldexp(448.0, ref)) ++ref;
  const int got = moe::mx_exponent(u);
  ++n_checked;
  if (got != ref) {
    if (n_bad < 5) std::printf("mismatch bits %08x: %d, definition %d\n", u, got, ref);
    ++n_bad;
  }
}

int main() {
  for (uint64_t u = 0; u < 0x7F800000u; u += 4099) check((uint32_t)u);
  const uint32_t fr[] = {0u, 1u, 0x5FFFFFu, 0x600000u, 0x600001u, 0x7FFFFFu};
  for (uint32_t e = 0; e < 255; ++e)
    for (uint32_t m : fr) check((e << 23) | m);
  std::printf("%ld %ld\n", n_checked, n_bad);
  return n_bad != 0;
}
"""


def test_mx_exponent_matches_its_definition(tmp_path):
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(nvcc):
        pytest.skip("no nvcc")
    src = tmp_path / "mx_exponent_check.cu"
    exe = tmp_path / "mx_exponent_check"
    src.write_text(PROGRAM)
    subprocess.check_call([nvcc, "-std=c++17", "-O2", "-gencode", "arch=compute_100a,code=sm_100a", "-I", CSRC,
                           "-I", os.path.join(ROOT, "include"), "-o", str(exe), str(src)])
    out = subprocess.run([str(exe)], capture_output=True, text=True)
    assert out.returncode == 0, out.stdout + out.stderr
    n, bad = map(int, out.stdout.split()[-2:])
    assert n > 500000 and bad == 0
