// dkv_plan.h -- host-side split-K planning shared by the decode entry points
// (plain C++, no CUDA).
//
// A launch over one pool cuts the blocks each sequence holds in that pool
// into `nsplit` splits; a unit is (sequence, split, kv head) and a warp
// processes one unit at a time.  The plan makes the number of units of a
// launch at most the number of warps it can keep resident, so no warp has to
// wait for a second unit while others idle.
#pragma once

#include <cmath>
#include <cstddef>
#include <cstdint>

namespace dkv {

constexpr int kMinSplitTokens = 64;  // a split holds at least this many tokens

struct SplitPlan {
  int nsplit;  // splits per sequence
  int bps;     // blocks per split (an upper bound of the per-sequence value when splits follow a pool list)
};

// nblk: blocks a sequence may hold (the table capacity); per: batch * kv heads;
// warps: resident warps of the launch; max_nsplit: cap on nsplit (0: none).
// Guarantees 1 <= nsplit <= max(1, warps / per), nsplit <= max_nsplit when
// capped, nsplit * bps >= nblk > (nsplit - 1) * bps and bps >= the minimum
// split size in blocks.
inline SplitPlan plan_split(int nblk, long per, int block_size, long warps, long max_nsplit) {
  SplitPlan r{1, 1};
  int min_bps = (kMinSplitTokens + block_size - 1) / block_size;
  if (min_bps < 1) min_bps = 1;
  r.bps = min_bps;
  if (nblk <= 0 || per <= 0) return r;
  long target = warps / per;
  if (target < 1) target = 1;
  if (max_nsplit > 0 && target > max_nsplit) target = max_nsplit;
  long b = (nblk + target - 1) / target;
  if (b < min_bps) b = min_bps;
  r.bps = static_cast<int>(b);
  r.nsplit = static_cast<int>((nblk + b - 1) / b);
  return r;
}

// Finer splits for long units.  Units are handed out dynamically, so a batch
// of ragged lengths finishes when its longest unit does, and a plan sized by
// the table capacity makes the units of the longest sequences as long as a
// warp's whole share.  This plans for `factor` units per resident warp (a
// whole number per warp, so that no second round of units runs on part of
// the warps), stepping the factor down until each unit keeps at least
// `min_tokens` tokens, so that a unit's setup (query load, RoPE seeds,
// partial write) stays small against its tiles.  Never gives fewer splits
// than the plan for one unit per warp.
inline SplitPlan plan_split_refined(int nblk, long per, int block_size, long warps, int factor, int min_tokens) {
  const SplitPlan base = plan_split(nblk, per, block_size, warps, 0);
  for (int k = factor; k > 1; --k) {
    const SplitPlan r = plan_split(nblk, per, block_size, warps * k, 0);
    if (static_cast<long>(r.bps) * block_size >= min_tokens && r.nsplit > base.nsplit) return r;
  }
  return base;
}

// The minimum split size in blocks: the blocks-per-split floor of every plan.
inline int min_blocks_per_split(int block_size) {
  const int m = (kMinSplitTokens + block_size - 1) / block_size;
  return m < 1 ? 1 : m;
}

// theta_i(p) = p * base^(-2i/D): the D/2 per-pair frequencies in fp64 (0 when
// base == 0, no rotation).  Every entry point that rotates uses these values.
inline void rope_frequencies(double base, int D, double* freq) {
  for (int i = 0; i < D / 2; ++i) freq[i] = base > 0.0 ? std::pow(base, -2.0 * i / static_cast<double>(D)) : 0.0;
}

// ---- scratch layout of the allocation-free entry point -----------------------
// [0, 256): status word and the two launches' work counters; [256, 1024): the
// RoPE frequencies; then the per-sequence pool counts, the pool lists, the
// partial lse rows and the partial output rows, each 256-byte aligned.
constexpr size_t kNoallocHeader = 1024;

inline size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// Bytes of scratch for `batch` sequences of `nblk` table blocks and `rows`
// partial rows of head_dim D.
inline size_t noalloc_scratch_bytes(size_t batch, size_t nblk, size_t rows, int D) {
  return kNoallocHeader + align256(batch * 8) + align256(batch * nblk * 8) + align256(rows * 4) + rows * D * 4;
}

// The largest number of slots per (sequence, query head) -- host splits plus
// device splits -- whose partials fit in `scratch` bytes (0 when even one
// does not fit).  Exact: s slots fit and s + 1 do not.
inline long noalloc_max_slots(size_t scratch, size_t batch, size_t nblk, long hq, int D) {
  if (batch == 0 || hq <= 0) return 0;
  const size_t fixed = kNoallocHeader + align256(batch * 8) + align256(batch * nblk * 8);
  if (fixed >= scratch) return 0;
  const size_t per_slot = batch * static_cast<size_t>(hq) * (4 * static_cast<size_t>(D) + 4);
  // an upper bound that ignores the alignment padding of the lse rows (< 256
  // bytes, less than one slot's bytes), then at most one step down
  long s = static_cast<long>((scratch - fixed) / per_slot);
  if (s > 0 && noalloc_scratch_bytes(batch, nblk, batch * static_cast<size_t>(hq) * s, D) > scratch) --s;
  return s;
}

}  // namespace dkv
