"""The split-K plan and the fixed-scratch bound of the allocation-free entry point, on the CPU.

Both live in the host-only header dkv_plan.h.  A small C++ program compiled with
g++ sweeps the arguments the library can pass and checks, for every plan:
1 <= nsplit <= max(1, warps / (batch * kv heads)), nsplit within the cap when
one is given, nsplit * bps covering the blocks with no empty last split, and
bps at least the minimum split size; for the refined plan (several units per
warp), no fewer splits than one unit per warp, at most `factor` units per
warp, and units of at least the minimum tokens whenever it refines.  For the scratch bound it checks that the
returned number of slots fits the fixed array and one more does not.
"""
import shutil
import subprocess
from pathlib import Path

import pytest

ROOT = Path(__file__).resolve().parents[1]
CSRC = ROOT / "decode_attention_host_b200" / "csrc"

PROGRAM = r"""
#include <cstdio>
#include <initializer_list>
#include "dkv_plan.h"

int main() {
  long plans = 0, bad = 0, fits = 0;
  const int bss[] = {16, 32, 64, 256, 1024};
  const long warpss[] = {64, 1120, 1184, 4096};
  const long caps[] = {0, 1, 3, 40};
  for (int nblk = 1; nblk <= 70000; nblk += (nblk < 300 ? 1 : 997)) {
    for (long per : {1L, 3L, 8L, 64L, 512L, 4096L}) {
      for (int bs : bss) {
        for (long warps : warpss) {
          for (long cap : caps) {
            const dkv::SplitPlan p = dkv::plan_split(nblk, per, bs, warps, cap);
            long target = warps / per;
            if (target < 1) target = 1;
            if (cap > 0 && target > cap) target = cap;
            ++plans;
            bad += p.nsplit < 1;
            bad += p.nsplit > target;
            bad += static_cast<long>(p.nsplit) * p.bps < nblk;
            bad += static_cast<long>(p.nsplit - 1) * p.bps >= nblk;
            bad += p.bps < dkv::min_blocks_per_split(bs);
          }
        }
      }
    }
  }
  // the refined plan: never fewer splits than one unit per warp; when it
  // refines, units of at least min_tokens and at most factor units per warp
  long refined = 0;
  for (int nblk = 1; nblk <= 70000; nblk += (nblk < 300 ? 7 : 1997)) {
    for (long per : {8L, 32L, 512L}) {
      for (int bs : {16, 32, 64}) {
        for (long warps : {1184L, 4096L}) {
          for (int factor : {1, 2, 4}) {
            for (int min_tokens : {64, 1024}) {
              const dkv::SplitPlan base = dkv::plan_split(nblk, per, bs, warps, 0);
              const dkv::SplitPlan r = dkv::plan_split_refined(nblk, per, bs, warps, factor, min_tokens);
              long target = factor * warps / per;
              if (target < 1) target = 1;
              ++plans;
              bad += r.nsplit < base.nsplit;
              bad += static_cast<long>(r.nsplit) * r.bps < nblk;
              bad += static_cast<long>(r.nsplit - 1) * r.bps >= nblk;
              bad += r.bps < dkv::min_blocks_per_split(bs);
              bad += r.nsplit > target;
              if (r.nsplit != base.nsplit) {
                ++refined;
                bad += factor == 1;
                bad += static_cast<long>(r.bps) * bs < min_tokens;
              } else {
                bad += r.bps != base.bps;
              }
            }
          }
        }
      }
    }
  }
  bad += refined == 0;
  const size_t scratch = 16u << 20;
  for (size_t batch : {1ul, 2ul, 5ul, 8ul, 64ul, 300ul, 4000ul, 5000ul}) {
    for (size_t nblk : {0ul, 1ul, 2048ul, 16384ul, 100000ul}) {
      for (long hq : {4L, 32L, 64L}) {
        for (int D : {64, 128}) {
          const long s = dkv::noalloc_max_slots(scratch, batch, nblk, hq, D);
          const size_t rows = batch * hq;
          if (s > 0) {
            ++fits;
            bad += dkv::noalloc_scratch_bytes(batch, nblk, rows * s, D) > scratch;
          }
          bad += dkv::noalloc_scratch_bytes(batch, nblk, rows * (s + 1), D) <= scratch;
          bad += s < 0;
        }
      }
    }
  }
  std::printf("%ld %ld %ld\n", plans, fits, bad);
  return 0;
}
"""


@pytest.mark.skipif(shutil.which("g++") is None, reason="g++ not found")
def test_split_plan_and_scratch_bound(tmp_path):
    src = tmp_path / "plan.cpp"
    src.write_text(PROGRAM)
    exe = tmp_path / "plan"
    subprocess.run(["g++", "-O2", "-std=c++17", f"-I{CSRC}", "-o", str(exe), str(src)], check=True,
                   capture_output=True)
    plans, fits, bad = map(int, subprocess.run([str(exe)], capture_output=True, text=True,
                                               check=True).stdout.split())
    assert plans > 100_000 and fits > 50
    assert bad == 0
