"""The launch-invariant divisors of the split kernels, checked on the CPU.

The kernels turn unit indices into (batch, split, kv head) and lengths into
block counts with a multiply-high by a magic number that the host computes
per launch (make_invdiv in dkv_kernels.cuh).  This test compiles that host
function with nvcc into a small CPU program, applies the kernels' quotient
formula with the 32x32 -> high-32 multiply written out in 64-bit integers,
and compares it with integer division for every divisor the library can
see (kv heads up to 4096, splits, block sizes up to 1024) and numerators
up to 2^31 - 1.
"""
import shutil
import subprocess
from pathlib import Path

import pytest

ROOT = Path(__file__).resolve().parents[1]
CSRC = ROOT / "decode_attention_host_b200" / "csrc"

PROGRAM = r"""
#include <cstdio>
#include <cstdint>
#include "dkv_kernels.cuh"

static int quotient(const dkv::InvDiv& v, uint32_t n) {
  const uint32_t hi = static_cast<uint32_t>((static_cast<uint64_t>(n) * v.m) >> 32);
  return static_cast<int>((hi + n) >> v.s);
}

int main() {
  long bad = 0, tests = 0;
  uint64_t x = 88172645463325252ull;  // xorshift64 numerators
  for (int d = 1; d <= 70000; d += (d <= 4096 ? 1 : 61)) {
    const dkv::InvDiv v = dkv::make_invdiv(d);
    for (uint32_t n = 0; n < 3000; ++n) { ++tests; bad += quotient(v, n) != static_cast<int>(n / d); }
    for (int k = 0; k < 3000; ++k) {
      x ^= x << 13; x ^= x >> 7; x ^= x << 17;
      const uint32_t n = static_cast<uint32_t>(x) & 0x7fffffffu;
      ++tests; bad += quotient(v, n) != static_cast<int>(n / d);
    }
    const uint32_t edges[] = {0x7fffffffu, 0x7ffffffeu, static_cast<uint32_t>(d) * 65535u & 0x7fffffffu};
    for (uint32_t n : edges) { ++tests; bad += quotient(v, n) != static_cast<int>(n / d); }
  }
  std::printf("%ld %ld\n", tests, bad);
  return bad != 0;
}
"""


@pytest.mark.skipif(shutil.which("nvcc") is None and not Path("/usr/local/cuda/bin/nvcc").exists(),
                    reason="nvcc not found")
def test_invariant_divisor_matches_integer_division(tmp_path):
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    src = tmp_path / "invdiv.cu"
    src.write_text(PROGRAM)
    exe = tmp_path / "invdiv"
    # the header holds sm_100a device code (packed fp32 intrinsics): compile for that target
    subprocess.run([nvcc, "-O2", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a", f"-I{CSRC}", "-o",
                    str(exe), str(src)], check=True,
                   capture_output=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True)
    tests, bad = map(int, out.stdout.split())
    assert tests > 10_000_000
    assert bad == 0 and out.returncode == 0
