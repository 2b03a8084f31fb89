"""The kernels' division by a launch-constant divisor (divisor_magic / udiv in
csrc/common.cuh: multiply by a rounded-up reciprocal, then shift) against
integer division, on the host: nvcc compiles a host-only program that
includes the same header; no GPU is touched.

Covered: every divisor 1..3000 with every numerator below 3000 and the
numerators next to many multiples of the divisor; powers of two and their
neighbours; random divisors up to 2^31 - 1 with numerators at quotient
boundaries and at 2^31 - 1."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "sparse_long_sequence_dilated_b200", "csrc")

PROGRAM = r"""
#include <cstdio>
#include <cstdint>
#include "common.cuh"
using dil::divisor_magic;
using dil::udiv;
static uint64_t state = 88172645463325252ull;
static uint64_t next() { state ^= state << 13; state ^= state >> 7; state ^= state << 17; return state; }
static long long bad = 0, checks = 0;
static void one(uint32_t d, uint32_t mul, int sh, uint32_t n) {
  ++checks;
  if (udiv(n, mul, sh) != n / d) { if (bad < 5) printf("d=%u n=%u got %u\n", d, n, udiv(n, mul, sh)); ++bad; }
}
static void test(uint32_t d, int nsamples) {
  uint32_t mul; int sh;
  divisor_magic(d, mul, sh);
  for (uint32_t n = 0; n < 3000; ++n) one(d, mul, sh, n);
  const uint32_t qmax = 0x7fffffffu / d;
  for (int k = 0; k < nsamples; ++k) {
    const uint64_t q = next() % ((uint64_t)qmax + 1);
    for (int e = -1; e <= 1; ++e) {
      const long long n = (long long)q * d + e;
      if (n >= 0 && n <= 0x7fffffffLL) one(d, mul, sh, (uint32_t)n);
    }
  }
  one(d, mul, sh, 0x7fffffffu);
  one(d, mul, sh, 0x7ffffffeu);
}
int main() {
  for (uint32_t d = 1; d <= 3000; ++d) test(d, 200);
  for (int l = 1; l < 31; ++l) { test(1u << l, 2000); test((1u << l) + 1, 2000); test((1u << l) - 1, 2000); }
  test(0x7fffffffu, 2000);
  for (int k = 0; k < 3000; ++k) test(1 + (uint32_t)(next() % 0x7ffffffeu), 200);
  printf("checks %lld bad %lld\n", checks, bad);
  return bad != 0;
}
"""


def _nvcc():
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    return None


@pytest.mark.skipif(_nvcc() is None, reason="nvcc not found")
def test_udiv_matches_integer_division(tmp_path):
    src = tmp_path / "udiv_check.cu"
    src.write_text(PROGRAM)
    exe = tmp_path / "udiv_check"
    build = subprocess.run([_nvcc(), "-O2", "-std=c++17", "-Wno-deprecated-gpu-targets", "-I", CSRC, "-I", os.path.join(ROOT, "include"),
                            "-o", str(exe), str(src)], capture_output=True, text=True)
    assert build.returncode == 0, build.stderr[-2000:]
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=300)
    assert run.returncode == 0, run.stdout + run.stderr
    assert " bad 0" in run.stdout
