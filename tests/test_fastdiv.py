"""Host-side check of the multiply-high division the prefill kernel uses to
decode its work units (csrc/fastdiv.h): the same header compiled for the CPU
must give n / d exactly for every divisor up to 4096 against a spread of
numerators, for divisors near powers of two, and for random pairs below 2^31."""
import os
import subprocess

import pytest

CSRC = os.path.join(os.path.dirname(__file__), "..", "scaled_dot_product_fa2_b200", "csrc")

CHECK = r"""
#include <cstdio>
#include <cstdint>
#include "fastdiv.h"
using sdpa::FastDiv;
static uint64_t state = 0x9E3779B97F4A7C15ull;
static uint32_t next31() {  // xorshift64*, top 31 bits
  state ^= state >> 12; state ^= state << 25; state ^= state >> 27;
  return static_cast<uint32_t>((state * 0x2545F4914F6CDD1Dull) >> 33);
}
static long bad = 0, checked = 0;
static void check(uint32_t n, uint32_t d, FastDiv f) {
  ++checked;
  if (sdpa::fastdiv(n, f) != n / d) { if (bad < 5) std::printf("n=%u d=%u got %u\n", n, d, sdpa::fastdiv(n, f)); ++bad; }
}
int main() {
  const uint32_t top = 0x7FFFFFFFu;
  for (uint32_t d = 1; d <= 4096; ++d) {
    const FastDiv f = sdpa::make_fastdiv(d);
    const uint32_t ns[] = {0u, 1u, d - 1, d, d + 1, 2 * d - 1, 2 * d, 1000 * d + 7, top, top - 1, top / d * d, top / d * d - 1};
    for (uint32_t n : ns) if (n <= top) check(n, d, f);
    for (int i = 0; i < 64; ++i) check(next31(), d, f);
  }
  for (int k = 1; k < 31; ++k)
    for (int e = -2; e <= 2; ++e) {
      const int64_t d64 = (int64_t{1} << k) + e;
      if (d64 < 1 || d64 > top) continue;
      const uint32_t d = static_cast<uint32_t>(d64);
      const FastDiv f = sdpa::make_fastdiv(d);
      for (int i = 0; i < 2000; ++i) check(next31(), d, f);
      check(top, d, f); check(d, d, f); check(d - 1, d, f);
    }
  for (int i = 0; i < 200000; ++i) {
    const uint32_t d = next31() % top + 1;
    check(next31(), d, sdpa::make_fastdiv(d));
  }
  std::printf("checked %ld bad %ld\n", checked, bad);
  return bad == 0 ? 0 : 1;
}
"""


def test_fastdiv_matches_integer_division(tmp_path):
    src = tmp_path / "fastdiv_check.cpp"
    src.write_text(CHECK)
    exe = tmp_path / "fastdiv_check"
    try:
        subprocess.run(["g++", "-O2", "-std=c++17", "-I", CSRC, str(src), "-o", str(exe)], check=True,
                       capture_output=True, text=True)
    except FileNotFoundError:
        pytest.skip("no g++")
    out = subprocess.run([str(exe)], capture_output=True, text=True)
    assert out.returncode == 0, out.stdout + out.stderr
    assert "bad 0" in out.stdout
