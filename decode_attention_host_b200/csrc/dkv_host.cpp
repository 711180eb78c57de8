// dkv_host.cpp -- host-side KV placement for libdkv: the block partitioner
// (which logical blocks live in pinned host memory and which in HBM, and
// their physical ids) and the packer that writes logical K/V into the pools.
//
// SplitKernel README, Key Features: attention over a KV cache partitioned
// between host and device, with placement / offloading-ratio utilities.
// DirectKV README, Artifact Evaluation (Figure 11b): the newest blocks stay
// on the GPU while the bulk of a long context lives in host memory; this is
// the prefix-host placement below.
#include <cmath>
#include <cstdint>
#include <cstring>
#include <string>
#include <vector>

#include "dkv.h"
#include "dkv_error.h"

using dkv::set_error;

namespace {

// splitmix64 (Steele, Lea and Flood, "Fast splittable pseudorandom number
// generators", OOPSLA 2014): a 64-bit counter advanced by the golden-ratio
// increment, then a mixing function.
struct SplitMix64 {
  uint64_t x;
  explicit SplitMix64(uint64_t seed) : x(seed) {}
  uint64_t next() {
    uint64_t z = (x += 0x9e3779b97f4a7c15ull);
    z = (z ^ (z >> 30)) * 0xbf58476d1ce4e5b9ull;
    z = (z ^ (z >> 27)) * 0x94d049bb133111ebull;
    return z ^ (z >> 31);
  }
  // uniform integer in [0, n) by the multiply-high reduction
  uint32_t below(uint32_t n) { return static_cast<uint32_t>((static_cast<unsigned __int128>(next()) * n) >> 64); }
};

void shuffle(std::vector<int32_t>& v, SplitMix64& rng) {
  for (size_t i = v.size(); i > 1; --i) {
    const uint32_t j = rng.below(static_cast<uint32_t>(i));
    std::swap(v[i - 1], v[j]);
  }
}

}  // namespace

extern "C" {

int dkv_plan_blocks(const dkv_plan_params* params, const int32_t* seq_lens, int32_t batch, int32_t* block_table,
                    int32_t block_table_stride, dkv_plan_result* result) {
  if (!params || !result || batch < 0 || (batch > 0 && (!seq_lens || !block_table)))
    return set_error(DKV_ERR_INVALID_ARG, "dkv_plan_blocks: null argument or negative batch");
  const dkv_plan_params& p = *params;
  if (p.block_size < 1) return set_error(DKV_ERR_INVALID_ARG, "dkv_plan_blocks: block_size must be >= 1");
  if (!(p.host_fraction >= 0.0 && p.host_fraction <= 1.0))
    return set_error(DKV_ERR_INVALID_ARG, "dkv_plan_blocks: host_fraction must be in [0, 1]");
  if (p.placement != DKV_PLACE_PREFIX_HOST && p.placement != DKV_PLACE_RANDOM)
    return set_error(DKV_ERR_INVALID_ARG, "dkv_plan_blocks: unknown placement");
  if (block_table_stride < 1) return set_error(DKV_ERR_INVALID_ARG, "dkv_plan_blocks: stride must be >= 1");

  // 1. host (1) / device (0) flag for every logical block
  std::vector<std::vector<uint8_t>> on_host(batch);
  int64_t n_host = 0, n_dev = 0, tok_host = 0, tok_dev = 0;
  for (int b = 0; b < batch; ++b) {
    const int64_t L = seq_lens[b];
    if (L < 0) return set_error(DKV_ERR_INVALID_ARG, "dkv_plan_blocks: negative sequence length");
    const int64_t nblk = (L + p.block_size - 1) / p.block_size;
    if (nblk > block_table_stride)
      return set_error(DKV_ERR_INVALID_ARG, "dkv_plan_blocks: a sequence needs more blocks than the table stride");
    const int64_t nh = std::llround(p.host_fraction * static_cast<double>(nblk));
    std::vector<uint8_t>& f = on_host[b];
    f.assign(static_cast<size_t>(nblk), 0);
    if (p.placement == DKV_PLACE_PREFIX_HOST) {
      for (int64_t j = 0; j < nh; ++j) f[j] = 1;
    } else {
      // nh distinct blocks, uniformly at random: partial Fisher-Yates over 0..nblk-1
      SplitMix64 rng(p.seed ^ (0x5bd1e995ull * static_cast<uint64_t>(b + 1)));
      std::vector<int32_t> idx(static_cast<size_t>(nblk));
      for (int64_t j = 0; j < nblk; ++j) idx[j] = static_cast<int32_t>(j);
      for (int64_t i = 0; i < nh; ++i) {
        const uint32_t r = static_cast<uint32_t>(i) + rng.below(static_cast<uint32_t>(nblk - i));
        std::swap(idx[i], idx[r]);
        f[idx[i]] = 1;
      }
    }
    for (int64_t j = 0; j < nblk; ++j) {
      const int64_t ntok = (j + 1) * p.block_size <= L ? p.block_size : L - j * p.block_size;
      if (f[j]) {
        ++n_host;
        tok_host += ntok;
      } else {
        ++n_dev;
        tok_dev += ntok;
      }
    }
  }
  if (n_host + n_dev > INT32_MAX) return set_error(DKV_ERR_INVALID_ARG, "dkv_plan_blocks: more than 2^31-1 blocks");

  // 2. physical ids: host pool first, then device pool, optionally permuted within each pool
  std::vector<int32_t> host_ids(static_cast<size_t>(n_host)), dev_ids(static_cast<size_t>(n_dev));
  for (int64_t i = 0; i < n_host; ++i) host_ids[i] = static_cast<int32_t>(i);
  for (int64_t i = 0; i < n_dev; ++i) dev_ids[i] = static_cast<int32_t>(n_host + i);
  if (p.shuffle_ids) {
    SplitMix64 rng(p.seed ^ 0x2545f4914f6cdd1dull);
    shuffle(host_ids, rng);
    shuffle(dev_ids, rng);
  }
  size_t hi = 0, di = 0;
  for (int b = 0; b < batch; ++b) {
    int32_t* row = block_table + static_cast<size_t>(b) * block_table_stride;
    const std::vector<uint8_t>& f = on_host[b];
    for (size_t j = 0; j < f.size(); ++j) row[j] = f[j] ? host_ids[hi++] : dev_ids[di++];
    for (size_t j = f.size(); j < static_cast<size_t>(block_table_stride); ++j) row[j] = -1;
  }
  result->host_split = static_cast<int32_t>(n_host);
  result->num_dev_blocks = static_cast<int32_t>(n_dev);
  result->host_tokens = tok_host;
  result->dev_tokens = tok_dev;
  return DKV_OK;
}

int dkv_plan_offload(double kv_bytes, double host_gbs, double hbm_gbs, double hbm_budget_bytes, double hbm_alone_gbs,
                     dkv_offload_plan* plan) {
  if (!plan || !(kv_bytes > 0.0) || !(host_gbs > 0.0) || !(hbm_gbs > 0.0) || std::isnan(hbm_budget_bytes) ||
      !std::isfinite(kv_bytes) || !std::isfinite(host_gbs) || !std::isfinite(hbm_gbs) ||
      !std::isfinite(hbm_alone_gbs))
    return set_error(DKV_ERR_INVALID_ARG, "dkv_plan_offload: sizes and bandwidths must be positive and finite");
  // best split with both kernels running: the two sides finish together
  const double f_conc = host_gbs / (host_gbs + hbm_gbs);
  const double t_conc = kv_bytes / ((host_gbs + hbm_gbs) * 1e9);
  // everything in HBM, the HBM kernel alone, when that is no slower
  const bool alone_wins = hbm_alone_gbs > 0.0 && kv_bytes / (hbm_alone_gbs * 1e9) <= t_conc;
  double f_cap = 0.0;
  if (hbm_budget_bytes >= 0.0) f_cap = 1.0 - hbm_budget_bytes / kv_bytes;
  double f, t;
  if (alone_wins && f_cap <= 0.0) {
    f = 0.0;
    t = kv_bytes / (hbm_alone_gbs * 1e9);
  } else {
    f = f_conc > f_cap ? f_conc : f_cap;
    if (f > 1.0) f = 1.0;
    const double t_host = f * kv_bytes / (host_gbs * 1e9);
    const double t_dev = (1.0 - f) * kv_bytes / (hbm_gbs * 1e9);
    t = t_host > t_dev ? t_host : t_dev;
  }
  plan->host_fraction = f;
  plan->step_seconds = t;
  plan->hbm_bytes_freed = f * kv_bytes;
  plan->time_optimal_fraction = alone_wins ? 0.0 : f_conc;
  return DKV_OK;
}

int dkv_pack_kv(const uint16_t* k_logical, const uint16_t* v_logical, int64_t lmax, const int32_t* seq_lens,
                int32_t batch, int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                const int32_t* block_table, int32_t block_table_stride, int32_t host_split, int32_t num_dev_blocks,
                uint16_t* k_host, uint16_t* v_host, uint16_t* k_dev_stage, uint16_t* v_dev_stage) {
  if (batch < 0 || num_kv_heads < 1 || head_dim < 1 || block_size < 1 || block_table_stride < 1 || lmax < 0 ||
      host_split < 0 || num_dev_blocks < 0)
    return set_error(DKV_ERR_INVALID_ARG, "dkv_pack_kv: size out of range");
  if (batch > 0 && (!k_logical || !v_logical || !seq_lens || !block_table))
    return set_error(DKV_ERR_INVALID_ARG, "dkv_pack_kv: null input");
  if ((host_split > 0 && (!k_host || !v_host)) || (num_dev_blocks > 0 && (!k_dev_stage || !v_dev_stage)))
    return set_error(DKV_ERR_INVALID_ARG, "dkv_pack_kv: null pool");
  const size_t row = static_cast<size_t>(head_dim);
  const size_t tile = static_cast<size_t>(block_size) * row;           // one (block, head) tile
  const size_t blk = static_cast<size_t>(num_kv_heads) * tile;         // one block, all heads
  for (int b = 0; b < batch; ++b) {
    const int64_t L = seq_lens[b];
    if (L < 0 || L > lmax) return set_error(DKV_ERR_INVALID_ARG, "dkv_pack_kv: sequence length outside [0, lmax]");
    const int64_t nblk = (L + block_size - 1) / block_size;
    if (nblk > block_table_stride) return set_error(DKV_ERR_INVALID_ARG, "dkv_pack_kv: table too narrow");
    for (int64_t j = 0; j < nblk; ++j) {
      const int32_t id = block_table[static_cast<size_t>(b) * block_table_stride + j];
      uint16_t *kd, *vd;
      if (id >= 0 && id < host_split) {
        kd = k_host + static_cast<size_t>(id) * blk;
        vd = v_host + static_cast<size_t>(id) * blk;
      } else if (id >= host_split && id - host_split < num_dev_blocks) {
        kd = k_dev_stage + static_cast<size_t>(id - host_split) * blk;
        vd = v_dev_stage + static_cast<size_t>(id - host_split) * blk;
      } else {
        return set_error(DKV_ERR_INVALID_ARG, "dkv_pack_kv: block id outside both pools");
      }
      const int64_t t0 = j * block_size;
      const int64_t ntok = L - t0 < block_size ? L - t0 : block_size;
      for (int h = 0; h < num_kv_heads; ++h) {
        const size_t src = ((static_cast<size_t>(b) * num_kv_heads + h) * static_cast<size_t>(lmax) + t0) * row;
        std::memcpy(kd + h * tile, k_logical + src, static_cast<size_t>(ntok) * row * sizeof(uint16_t));
        std::memcpy(vd + h * tile, v_logical + src, static_cast<size_t>(ntok) * row * sizeof(uint16_t));
        if (ntok < block_size) {
          const size_t rest = static_cast<size_t>(block_size - ntok) * row * sizeof(uint16_t);
          std::memset(kd + h * tile + ntok * row, 0, rest);
          std::memset(vd + h * tile + ntok * row, 0, rest);
        }
      }
    }
  }
  return DKV_OK;
}

}  // extern "C"
