"""The kernels divide token offsets by the page size with multiply-and-shift constants the
host computes (`gqa::divisor_magic` in csrc/internal.cuh): floor(x / d) ==
umulhi(x, magic) >> shift for 0 <= x < 2^31.  This compiles the host function with the
system C++ compiler and checks it against integer division for every page size the
library accepts (multiples of 16 up to 256) and a few other divisors, on the boundary
dividends (multiples of d and their neighbours, the top of the range) and random ones."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "gqa_decode_attention_04_b200", "csrc")
INCLUDE = os.path.join(ROOT, "include")
CUDA_INCLUDE = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "include")

PROGRAM = r"""
#include <cstdio>
#include <cstdint>
#include <random>
#include "internal.cuh"

static int check(uint32_t d, uint32_t x, uint32_t m, int s) {
  const uint32_t hi = static_cast<uint32_t>((static_cast<uint64_t>(x) * m) >> 32);
  return (hi >> s) == x / d ? 0 : 1;
}

int main() {
  std::mt19937 rng(12345);
  int bad = 0;
  long n = 0;
  for (uint32_t d = 2; d <= 4096; ++d) {
    uint32_t m;
    int s;
    gqa::divisor_magic(d, &m, &s);
    const uint32_t top = 0x7fffffffu;
    for (uint32_t k = 0; k < 64; ++k)
      for (int e = -1; e <= 1; ++e) {
        const int64_t x = static_cast<int64_t>(k) * d + e;
        if (x >= 0 && x <= top) { bad += check(d, static_cast<uint32_t>(x), m, s); ++n; }
      }
    for (uint32_t j = 0; j < 3; ++j) { bad += check(d, top - j, m, s); ++n; }
    const uint32_t qtop = top / d;
    for (int e = -1; e <= 1; ++e) {
      const int64_t x = static_cast<int64_t>(qtop) * d + e;
      if (x >= 0 && x <= top) { bad += check(d, static_cast<uint32_t>(x), m, s); ++n; }
    }
    for (int r = 0; r < 2000; ++r) { bad += check(d, rng() & top, m, s); ++n; }
    if (bad) { std::printf("mismatch for d=%u\n", d); return 1; }
  }
  std::printf("ok %ld\n", n);
  return 0;
}
"""


@pytest.mark.skipif(shutil.which("g++") is None, reason="no C++ compiler")
def test_page_size_division_constants_are_exact(tmp_path):
    src = tmp_path / "magic.cpp"
    exe = tmp_path / "magic"
    src.write_text(PROGRAM)
    subprocess.run(["g++", "-std=c++17", "-O2", "-I", CSRC, "-I", INCLUDE, "-I", CUDA_INCLUDE, str(src), "-o", str(exe)],
                   check=True, capture_output=True, text=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0 and r.stdout.startswith("ok"), r.stdout + r.stderr
