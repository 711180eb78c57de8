// dkv_api.cu -- C ABI of libdkv: handle lifetime, argument validation, the
// split-K launch plan and the fork/join of the host-stream and HBM kernels.
#include <cuda_runtime.h>

#include <climits>
#include <cmath>
#include <cstring>
#include <new>
#include <string>
#include <vector>

#include "dkv.h"
#include "dkv_error.h"
#include "dkv_append.cuh"
#include "dkv_kernels.cuh"
#include "dkv_multi.cuh"

namespace {

thread_local std::string g_err;

int fail(int code, const std::string& msg) {
  g_err = msg;
  return code;
}

}  // namespace

int dkv::set_error(int code, const std::string& msg) { return fail(code, msg); }

namespace {

int cuda_fail(cudaError_t e, const char* what) {
  g_err = std::string(what) + ": " + cudaGetErrorString(e);
  return DKV_ERR_CUDA;
}

#define DKV_CUDA(call)                                  \
  do {                                                  \
    cudaError_t e_ = (call);                            \
    if (e_ != cudaSuccess) return cuda_fail(e_, #call); \
  } while (0)

// Restores the caller's current device on scope exit.
struct DeviceGuard {
  int prev = -1;
  bool ok = false;
  explicit DeviceGuard(int dev) {
    if (cudaGetDevice(&prev) == cudaSuccess) ok = cudaSetDevice(dev) == cudaSuccess;
  }
  ~DeviceGuard() {
    if (prev >= 0) cudaSetDevice(prev);
  }
};

constexpr int kHostStages = 4;   // ring depth of the zero-copy host kernel (1 CTA per SM, few SMs)
#ifndef DKV_DEV_STAGES
#define DKV_DEV_STAGES 3
#endif
constexpr int kDevStages = DKV_DEV_STAGES;  // ring depth of the HBM kernel (build-time knob)
constexpr int kDefaultHostCtas = 16;
constexpr int kMinSplitTokens = 64;

size_t split_smem(int D, int nst) { return static_cast<size_t>(dkv::kWarps) * nst * 2 * dkv::kTileTokens * D * 2; }

using SplitFn = void (*)(dim3, size_t, cudaStream_t, const dkv::SplitParams&);
using SplitKernelPtr = const void*;

template <int D, int G, bool BF16, int NST, bool ROPE>
void launch_split(dim3 grid, size_t smem, cudaStream_t s, const dkv::SplitParams& p) {
  dkv::split_kernel<D, G, BF16, NST, ROPE><<<grid, dkv::kThreads, smem, s>>>(p);
}
template <int D, int G, bool BF16, int NST, bool ROPE>
const void* split_ptr() {
  return reinterpret_cast<const void*>(&dkv::split_kernel<D, G, BF16, NST, ROPE>);
}

struct SplitEntry {
  SplitFn fn;
  SplitKernelPtr ptr;
};

template <int NST, bool ROPE>
SplitEntry pick_split_rope(int D, int G, bool bf16) {
#define DKV_CASE(DD, GG)                                                                                   \
  if (D == DD && G == GG) {                                                                                \
    if (bf16) return {&launch_split<DD, GG, true, NST, ROPE>, split_ptr<DD, GG, true, NST, ROPE>()};      \
    return {&launch_split<DD, GG, false, NST, ROPE>, split_ptr<DD, GG, false, NST, ROPE>()};              \
  }
  DKV_CASE(64, 1)
  DKV_CASE(64, 2)
  DKV_CASE(64, 4)
  DKV_CASE(128, 1)
  DKV_CASE(128, 2)
  DKV_CASE(128, 4)
#undef DKV_CASE
  return {nullptr, nullptr};
}

template <int NST>
SplitEntry pick_split(int D, int G, bool bf16, bool rope) {
  return rope ? pick_split_rope<NST, true>(D, G, bf16) : pick_split_rope<NST, false>(D, G, bf16);
}

template <int D, bool BF16, bool ROPE>
void launch_multi(dim3 grid, size_t smem, cudaStream_t s, const dkv::SplitParams& p) {
  dkv::multi_kernel<D, BF16, ROPE><<<grid, dkv::kThreads, smem, s>>>(p);
}

SplitEntry pick_multi(int D, bool bf16, bool rope) {
#define DKV_MCASE(DD, BB, RR) \
  if (D == DD && bf16 == BB && rope == RR) \
    return {&launch_multi<DD, BB, RR>, reinterpret_cast<const void*>(&dkv::multi_kernel<DD, BB, RR>)};
  DKV_MCASE(64, false, false) DKV_MCASE(64, false, true) DKV_MCASE(64, true, false) DKV_MCASE(64, true, true)
  DKV_MCASE(128, false, false) DKV_MCASE(128, false, true) DKV_MCASE(128, true, false) DKV_MCASE(128, true, true)
#undef DKV_MCASE
  return {nullptr, nullptr};
}

// shared memory of the multi-token kernel: per warp a 2-stage (K, V) ring and one rotated-K lo tile
size_t multi_smem(int D) { return static_cast<size_t>(dkv::kWarps) * 5 * dkv::kTileTokens * D * 2; }

using MergeFn = void (*)(dim3, size_t, cudaStream_t, const dkv::MergeParams&);
template <int D, int NG>
void launch_merge(dim3 grid, size_t smem, cudaStream_t s, const dkv::MergeParams& p) {
  dkv::merge_kernel<D, NG><<<grid, NG * D, smem, s>>>(p);
}

}  // namespace

struct dkv_handle {
  dkv_config cfg{};
  int G = 0;
  int sm_count = 0;
  int units_target = 0;
  size_t part_rows = 0;
  float qscale = 0.f;
  int host_ctas = 0;
  float* part_o = nullptr;
  float* part_lse = nullptr;
  int32_t* status = nullptr;
  double* inv_freq = nullptr;
  cudaStream_t aux = nullptr;
  cudaEvent_t ev_fork = nullptr;
  cudaEvent_t ev_join = nullptr;
  SplitEntry host_kernel{}, dev_kernel{}, multi_kernel{};
  MergeFn merge = nullptr;
  const void* ok_host[2] = {nullptr, nullptr};
  const void* ok_dev[4] = {nullptr, nullptr, nullptr, nullptr};
  int last_launches = 0;
  // per-kernel event pairs while profiling: [kernel][call] -> (start, stop)
  int prof_capacity = 0;
  int prof_used[3] = {0, 0, 0};
  std::vector<cudaEvent_t> prof_events[3];
};

namespace {

void prof_release(dkv_handle* h) {
  for (auto& v : h->prof_events) {
    for (cudaEvent_t e : v)
      if (e) cudaEventDestroy(e);
    v.clear();
  }
  h->prof_capacity = 0;
  h->prof_used[0] = h->prof_used[1] = h->prof_used[2] = 0;
}

// Records the start (stop == false) or stop event of kernel k of the current call.
int prof_mark(dkv_handle* h, int k, cudaStream_t s, bool stop) {
  if (h->prof_used[k] >= h->prof_capacity) return DKV_OK;
  cudaEvent_t e = h->prof_events[k][2 * h->prof_used[k] + (stop ? 1 : 0)];
  DKV_CUDA(cudaEventRecord(e, s));
  if (stop) ++h->prof_used[k];
  return DKV_OK;
}

void release(dkv_handle* h) {
  if (!h) return;
  DeviceGuard g(h->cfg.device);
  if (h->aux) cudaStreamSynchronize(h->aux);
  prof_release(h);
  cudaFree(h->part_o);
  cudaFree(h->part_lse);
  cudaFree(h->status);
  cudaFree(h->inv_freq);
  if (h->ev_fork) cudaEventDestroy(h->ev_fork);
  if (h->ev_join) cudaEventDestroy(h->ev_join);
  if (h->aux) cudaStreamDestroy(h->aux);
  delete h;
}

void plan_splits(const dkv_handle* h, int batch, int stride, int* nsplit, int* bps, int num_queries = 1) {
  const int nblk = stride < h->cfg.max_blocks_per_seq ? stride : h->cfg.max_blocks_per_seq;
  if (nblk <= 0 || batch <= 0) {
    *nsplit = 1;
    *bps = 1;
    return;
  }
  // one unit (b, split, kv head) per warp of a full wave, whatever the number
  // of query tokens: a unit carries all Tq * G query rows of its kv head
  (void)num_queries;
  const long per = static_cast<long>(batch) * h->cfg.num_kv_heads;
  const int target = static_cast<int>((h->units_target + per - 1) / per) > 0
                         ? static_cast<int>((h->units_target + per - 1) / per)
                         : 1;
  int min_bps = (kMinSplitTokens + h->cfg.block_size - 1) / h->cfg.block_size;
  if (min_bps < 1) min_bps = 1;
  int b = (nblk + target - 1) / target;
  if (b < min_bps) b = min_bps;
  *bps = b;
  *nsplit = (nblk + b - 1) / b;
}

int check_host_pool(dkv_handle* h, const void* p, int which) {
  if (h->ok_host[which] == p) return DKV_OK;
  cudaPointerAttributes a{};
  cudaError_t e = cudaPointerGetAttributes(&a, p);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(DKV_ERR_INVALID_ARG, "host pool pointer is not known to CUDA (use dkv_host_pool_alloc)");
  }
  if (a.type != cudaMemoryTypeHost || a.devicePointer == nullptr || a.devicePointer != p)
    return fail(DKV_ERR_INVALID_ARG, "host pool must be mapped pinned host memory passed by its device alias");
  h->ok_host[which] = p;
  return DKV_OK;
}

int check_dev_pool(dkv_handle* h, const void* p, int which) {
  if (h->ok_dev[which] == p) return DKV_OK;
  cudaPointerAttributes a{};
  cudaError_t e = cudaPointerGetAttributes(&a, p);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(DKV_ERR_INVALID_ARG, "device pool pointer is not known to CUDA");
  }
  if (!((a.type == cudaMemoryTypeDevice || a.type == cudaMemoryTypeManaged) && a.device == h->cfg.device))
    return fail(DKV_ERR_INVALID_ARG, "device pool must be device memory of the handle's GPU");
  h->ok_dev[which] = p;
  return DKV_OK;
}

}  // namespace

extern "C" {

const char* dkv_last_error_string(void) { return g_err.c_str(); }

int dkv_create(const dkv_config* cfg, dkv_handle** out) {
  if (!cfg || !out) return fail(DKV_ERR_INVALID_ARG, "dkv_create: null argument");
  *out = nullptr;
  const dkv_config& c = *cfg;
  if (c.num_q_heads < 1 || c.num_kv_heads < 1 || c.num_q_heads % c.num_kv_heads != 0)
    return fail(DKV_ERR_INVALID_ARG, "num_q_heads must be a positive multiple of num_kv_heads");
  if (c.block_size < 16 || c.block_size > 1024 || c.block_size % 16 != 0)
    return fail(DKV_ERR_INVALID_ARG, "block_size must be a multiple of 16 in [16, 1024]");
  if (c.kv_dtype != DKV_KV_F16 && c.kv_dtype != DKV_KV_BF16) return fail(DKV_ERR_INVALID_ARG, "kv_dtype");
  if (!(c.rope_base >= 0.0) || !std::isfinite(c.rope_base) || (c.rope_base > 0.0 && c.rope_base <= 1.0))
    return fail(DKV_ERR_INVALID_ARG, "rope_base must be 0 (off) or > 1");
  if (!(c.scale >= 0.0) || !std::isfinite(c.scale)) return fail(DKV_ERR_INVALID_ARG, "scale must be >= 0");
  if (c.max_batch < 1 || c.max_blocks_per_seq < 1) return fail(DKV_ERR_INVALID_ARG, "max_batch / max_blocks_per_seq");
  if (static_cast<long long>(c.max_blocks_per_seq) * c.block_size > (1LL << 30))
    return fail(DKV_ERR_INVALID_ARG, "max_blocks_per_seq * block_size exceeds 2^30 tokens");
  if (c.host_ctas < 0) return fail(DKV_ERR_INVALID_ARG, "host_ctas must be >= 0");
  if (c.num_kv_heads > 4096) return fail(DKV_ERR_INVALID_ARG, "num_kv_heads must be <= 4096");
  const int G = c.num_q_heads / c.num_kv_heads;
  if (c.head_dim != 64 && c.head_dim != 128) return fail(DKV_ERR_UNSUPPORTED, "head_dim must be 64 or 128");
  if (G != 1 && G != 2 && G != 4) return fail(DKV_ERR_UNSUPPORTED, "query group size must be 1, 2 or 4");
  int ndev = 0;
  DKV_CUDA(cudaGetDeviceCount(&ndev));
  if (c.device < 0 || c.device >= ndev) return fail(DKV_ERR_INVALID_ARG, "device ordinal out of range");

  DeviceGuard guard(c.device);
  if (!guard.ok) return fail(DKV_ERR_CUDA, "cudaSetDevice failed");
  dkv_handle* h = new (std::nothrow) dkv_handle();
  if (!h) return fail(DKV_ERR_NO_MEMORY, "handle allocation");
  h->cfg = c;
  h->G = G;
  const bool bf16 = c.kv_dtype == DKV_KV_BF16;
  const double scale = c.scale > 0.0 ? c.scale : 1.0 / std::sqrt(static_cast<double>(c.head_dim));
  h->qscale = static_cast<float>(scale * 1.4426950408889634);  // * log2(e)
  h->host_ctas = c.host_ctas > 0 ? c.host_ctas : kDefaultHostCtas;
  const bool rope = c.rope_base > 0.0;
  h->host_kernel = pick_split<kHostStages>(c.head_dim, G, bf16, rope);
  h->dev_kernel = pick_split<kDevStages>(c.head_dim, G, bf16, rope);
  h->multi_kernel = pick_multi(c.head_dim, bf16, c.rope_base > 0.0);
  h->merge = c.head_dim == 64 ? &launch_merge<64, 16> : &launch_merge<128, 8>;

  auto bail = [&](int code) {
    release(h);
    return code;
  };
  cudaError_t e = cudaDeviceGetAttribute(&h->sm_count, cudaDevAttrMultiProcessorCount, c.device);
  if (e != cudaSuccess) return bail(cuda_fail(e, "cudaDeviceGetAttribute"));
  h->units_target = h->sm_count * 8;  // one unit per warp of a full wave (2 CTAs x 4 warps per SM)
  // partial rows: batch * Tq * Hq * 2 * nsplit with nsplit <= units_target / (batch * Hkv) + 1 and
  // Tq * G <= 16 rows per unit (multi-token queries), batch * Tq <= max_batch
  h->part_rows = 2ull * (static_cast<size_t>(dkv::kMultiMaxRows) * h->units_target +
                         static_cast<size_t>(G) * c.max_batch * c.num_kv_heads);
  e = cudaFuncSetAttribute(h->host_kernel.ptr, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(split_smem(c.head_dim, kHostStages)));
  if (e != cudaSuccess) return bail(cuda_fail(e, "cudaFuncSetAttribute(host kernel)"));
  e = cudaFuncSetAttribute(h->dev_kernel.ptr, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(split_smem(c.head_dim, kDevStages)));
  if (e != cudaSuccess) return bail(cuda_fail(e, "cudaFuncSetAttribute(HBM kernel)"));
  e = cudaFuncSetAttribute(h->multi_kernel.ptr, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(multi_smem(c.head_dim)));
  if (e != cudaSuccess) return bail(cuda_fail(e, "cudaFuncSetAttribute(multi-token kernel)"));
  if (cudaMalloc(&h->part_o, h->part_rows * c.head_dim * sizeof(float)) != cudaSuccess ||
      cudaMalloc(&h->part_lse, h->part_rows * sizeof(float)) != cudaSuccess ||
      cudaMalloc(&h->status, sizeof(int32_t)) != cudaSuccess ||
      cudaMalloc(&h->inv_freq, sizeof(double) * (c.head_dim / 2)) != cudaSuccess) {
    cudaGetLastError();
    return bail(fail(DKV_ERR_NO_MEMORY, "workspace allocation failed"));
  }
  // theta_i(p) = p * base^(-2i/D): the per-pair frequencies, in fp64
  double freq[64];
  for (int i = 0; i < c.head_dim / 2; ++i)
    freq[i] = c.rope_base > 0.0 ? std::pow(c.rope_base, -2.0 * i / static_cast<double>(c.head_dim)) : 0.0;
  e = cudaMemcpy(h->inv_freq, freq, sizeof(double) * (c.head_dim / 2), cudaMemcpyHostToDevice);
  if (e != cudaSuccess) return bail(cuda_fail(e, "cudaMemcpy(inv_freq)"));
  e = cudaMemset(h->status, 0, sizeof(int32_t));
  if (e != cudaSuccess) return bail(cuda_fail(e, "cudaMemset(status)"));
  int lo = 0, hi = 0;
  e = cudaDeviceGetStreamPriorityRange(&lo, &hi);
  if (e != cudaSuccess) return bail(cuda_fail(e, "cudaDeviceGetStreamPriorityRange"));
  e = cudaStreamCreateWithPriority(&h->aux, cudaStreamNonBlocking, hi);
  if (e != cudaSuccess) return bail(cuda_fail(e, "cudaStreamCreateWithPriority"));
  e = cudaEventCreateWithFlags(&h->ev_fork, cudaEventDisableTiming);
  if (e != cudaSuccess) return bail(cuda_fail(e, "cudaEventCreate"));
  e = cudaEventCreateWithFlags(&h->ev_join, cudaEventDisableTiming);
  if (e != cudaSuccess) return bail(cuda_fail(e, "cudaEventCreate"));
  *out = h;
  return DKV_OK;
}

int dkv_destroy(dkv_handle* h) {
  release(h);
  return DKV_OK;
}

int dkv_query_plan(const dkv_handle* h, int32_t batch, int32_t block_table_stride, int32_t* num_splits,
                   int32_t* blocks_per_split) {
  if (!h || !num_splits || !blocks_per_split) return fail(DKV_ERR_INVALID_ARG, "dkv_query_plan: null argument");
  if (batch < 0 || batch > h->cfg.max_batch || block_table_stride < 1)
    return fail(DKV_ERR_INVALID_ARG, "dkv_query_plan: batch or stride out of range");
  int ns, b;
  plan_splits(h, batch, block_table_stride, &ns, &b);
  *num_splits = ns;
  *blocks_per_split = b;
  return DKV_OK;
}

int dkv_last_launch_count(const dkv_handle* h, int32_t* count) {
  if (!h || !count) return fail(DKV_ERR_INVALID_ARG, "dkv_last_launch_count: null argument");
  *count = h->last_launches;
  return DKV_OK;
}

}  // extern "C"

namespace {

// One decode step.  k_stage == nullptr: zero-copy (host kernel on the aux
// stream reads the mapped host pools).  Otherwise the staged-prefetch
// comparator: the host pools are first copied into k_stage / v_stage.
int decode_impl(dkv_handle* h, const float* q, const void* k_host, const void* v_host, const void* k_dev,
                const void* v_dev, const int32_t* block_table, const int32_t* seq_lens, int32_t host_split, float* out,
                dkv_stream_t stream, int32_t batch, int32_t block_table_stride, int32_t num_dev_blocks, void* k_stage,
                void* v_stage, int32_t num_queries = 0) {
  const bool staged = k_stage != nullptr || v_stage != nullptr;
  const bool multi = num_queries > 0;  // the multi-token kernel (num_queries >= 1 query tokens per sequence)
  const int nq = multi ? num_queries : 1;
  if (multi && (h == nullptr || num_queries * (h->cfg.num_q_heads / h->cfg.num_kv_heads) > dkv::kMultiMaxRows ||
                static_cast<long long>(batch) * num_queries > h->cfg.max_batch))
    return fail(DKV_ERR_INVALID_ARG, "num_queries * group size must be <= 16 and batch * num_queries <= max_batch");
  if (!h) return fail(DKV_ERR_INVALID_ARG, "dkv_attn_decode: null handle");
  if (batch < 0 || batch > h->cfg.max_batch) return fail(DKV_ERR_INVALID_ARG, "batch outside [0, max_batch]");
  if (batch == 0) {
    h->last_launches = 0;
    return DKV_OK;
  }
  if (!q || !out || !block_table || !seq_lens) return fail(DKV_ERR_INVALID_ARG, "null q / out / table / seq_lens");
  if (block_table_stride < 1) return fail(DKV_ERR_INVALID_ARG, "block_table_stride must be >= 1");
  if (host_split < 0 || num_dev_blocks < 0 || static_cast<long long>(host_split) + num_dev_blocks > INT_MAX)
    return fail(DKV_ERR_INVALID_ARG, "host_split / num_dev_blocks out of range");
  if (host_split > 0 && (!k_host || !v_host)) return fail(DKV_ERR_INVALID_ARG, "host pool pointers are null");
  if (num_dev_blocks > 0 && (!k_dev || !v_dev)) return fail(DKV_ERR_INVALID_ARG, "device pool pointers are null");
  if (reinterpret_cast<uintptr_t>(q) % 8 != 0)
    return fail(DKV_ERR_INVALID_ARG, "q must be 8-byte aligned");
  if ((host_split > 0 && (reinterpret_cast<uintptr_t>(k_host) | reinterpret_cast<uintptr_t>(v_host)) % 16 != 0) ||
      (num_dev_blocks > 0 && (reinterpret_cast<uintptr_t>(k_dev) | reinterpret_cast<uintptr_t>(v_dev)) % 16 != 0))
    return fail(DKV_ERR_INVALID_ARG, "K/V pools must be 16-byte aligned");

  DeviceGuard guard(h->cfg.device);
  if (!guard.ok) return fail(DKV_ERR_CUDA, "cudaSetDevice failed");
  int rc;
  if (host_split > 0) {
    if ((rc = check_host_pool(h, k_host, 0)) != DKV_OK) return rc;
    if ((rc = check_host_pool(h, v_host, 1)) != DKV_OK) return rc;
  }
  if (num_dev_blocks > 0) {
    if ((rc = check_dev_pool(h, k_dev, 0)) != DKV_OK) return rc;
    if ((rc = check_dev_pool(h, v_dev, 1)) != DKV_OK) return rc;
  }
  if (staged && host_split > 0) {
    if (!k_stage || !v_stage) return fail(DKV_ERR_INVALID_ARG, "staging pools must both be given");
    if ((reinterpret_cast<uintptr_t>(k_stage) | reinterpret_cast<uintptr_t>(v_stage)) % 16 != 0)
      return fail(DKV_ERR_INVALID_ARG, "staging pools must be 16-byte aligned");
    if ((rc = check_dev_pool(h, k_stage, 2)) != DKV_OK) return rc;
    if ((rc = check_dev_pool(h, v_stage, 3)) != DKV_OK) return rc;
  }

  const dkv_config& c = h->cfg;
  int nsplit, bps;
  plan_splits(h, batch, block_table_stride, &nsplit, &bps, nq);
  const int nslots = 2 * nsplit;
  if (static_cast<size_t>(batch) * nq * c.num_q_heads * nslots > h->part_rows)
    return fail(DKV_ERR_INVALID_ARG, "internal: split plan exceeds the workspace");
  const int n_units = batch * nsplit * c.num_kv_heads;
  const int nblk_cap = block_table_stride < c.max_blocks_per_seq ? block_table_stride : c.max_blocks_per_seq;

  dkv::SplitParams sp{};
  sp.q = q;
  sp.table = block_table;
  sp.seq_lens = seq_lens;
  sp.inv_freq = h->inv_freq;
  sp.part_o = h->part_o;
  sp.part_lse = h->part_lse;
  sp.status = h->status;
  sp.hq = c.num_q_heads;
  sp.hkv = c.num_kv_heads;
  sp.block_size = c.block_size;
  sp.stride = block_table_stride;
  sp.nsplit = nsplit;
  sp.bps = bps;
  sp.nslots = nslots;
  sp.id_total = host_split + num_dev_blocks;
  sp.max_len = nblk_cap * c.block_size;
  sp.n_units = n_units;
  sp.rope = c.rope_base > 0.0 ? 1 : 0;
  sp.qscale = h->qscale;
  sp.extra_tokens = nq - 1;
  sp.num_queries = nq;
  dkv::set_divisors(sp);
  const SplitEntry& host_k = multi ? h->multi_kernel : h->host_kernel;
  const SplitEntry& dev_k = multi ? h->multi_kernel : h->dev_kernel;
  const size_t host_smem = multi ? multi_smem(c.head_dim) : split_smem(c.head_dim, kHostStages);
  const size_t dev_smem = multi ? multi_smem(c.head_dim) : split_smem(c.head_dim, kDevStages);

  const int unit_ctas = (n_units + dkv::kWarps - 1) / dkv::kWarps;
  int launches = 0;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (host_split > 0 && staged) {
    // copy engine: pinned host pools -> HBM staging pools, then the HBM kernel reads them
    const size_t bytes = static_cast<size_t>(host_split) * c.num_kv_heads * c.block_size * c.head_dim * 2;
    if ((rc = prof_mark(h, 0, s, false)) != DKV_OK) return rc;
    DKV_CUDA(cudaMemcpyAsync(k_stage, k_host, bytes, cudaMemcpyHostToDevice, s));
    DKV_CUDA(cudaMemcpyAsync(v_stage, v_host, bytes, cudaMemcpyHostToDevice, s));
    dkv::SplitParams hp = sp;
    hp.k_pool = static_cast<const uint16_t*>(k_stage);
    hp.v_pool = static_cast<const uint16_t*>(v_stage);
    hp.id_lo = 0;
    hp.id_hi = host_split;
    hp.slot_base = 0;
    const int dev_ctas = unit_ctas < 2 * h->sm_count ? unit_ctas : 2 * h->sm_count;
    dev_k.fn(dim3(dev_ctas), dev_smem, s, hp);
    DKV_CUDA(cudaGetLastError());
    if ((rc = prof_mark(h, 0, s, true)) != DKV_OK) return rc;
    ++launches;
  } else if (host_split > 0) {
    DKV_CUDA(cudaEventRecord(h->ev_fork, s));
    DKV_CUDA(cudaStreamWaitEvent(h->aux, h->ev_fork, 0));
    dkv::SplitParams hp = sp;
    hp.k_pool = static_cast<const uint16_t*>(k_host);
    hp.v_pool = static_cast<const uint16_t*>(v_host);
    hp.id_lo = 0;
    hp.id_hi = host_split;
    hp.slot_base = 0;
    const int grid = unit_ctas < h->host_ctas ? unit_ctas : h->host_ctas;
    if ((rc = prof_mark(h, 0, h->aux, false)) != DKV_OK) return rc;
    host_k.fn(dim3(grid), host_smem, h->aux, hp);
    DKV_CUDA(cudaGetLastError());
    if ((rc = prof_mark(h, 0, h->aux, true)) != DKV_OK) return rc;
    DKV_CUDA(cudaEventRecord(h->ev_join, h->aux));
    ++launches;
  }
  if (num_dev_blocks > 0) {
    dkv::SplitParams dp = sp;
    dp.k_pool = static_cast<const uint16_t*>(k_dev);
    dp.v_pool = static_cast<const uint16_t*>(v_dev);
    dp.id_lo = host_split;
    dp.id_hi = host_split + num_dev_blocks;
    dp.slot_base = nsplit;
    if ((rc = prof_mark(h, 1, s, false)) != DKV_OK) return rc;
    const int dev_ctas = unit_ctas < 2 * h->sm_count ? unit_ctas : 2 * h->sm_count;  // one resident wave
    dev_k.fn(dim3(dev_ctas), dev_smem, s, dp);
    DKV_CUDA(cudaGetLastError());
    if ((rc = prof_mark(h, 1, s, true)) != DKV_OK) return rc;
    ++launches;
  }
  if (host_split > 0 && !staged) DKV_CUDA(cudaStreamWaitEvent(s, h->ev_join, 0));
  dkv::MergeParams mp{};
  mp.part_o = h->part_o;
  mp.part_lse = h->part_lse;
  mp.out = out;
  mp.nslots = nslots;
  mp.nsplit = nsplit;
  mp.has_host = host_split > 0;
  mp.has_dev = num_dev_blocks > 0;
  if ((rc = prof_mark(h, 2, s, false)) != DKV_OK) return rc;
  h->merge(dim3(batch * nq * c.num_q_heads), nslots * sizeof(float), s, mp);
  DKV_CUDA(cudaGetLastError());
  if ((rc = prof_mark(h, 2, s, true)) != DKV_OK) return rc;
  ++launches;
  h->last_launches = launches;
  return DKV_OK;
}

}  // namespace

extern "C" {

int dkv_attn_decode(dkv_handle* h, const float* q, const void* k_host, const void* v_host, const void* k_dev,
                    const void* v_dev, const int32_t* block_table, const int32_t* seq_lens, int32_t host_split,
                    float* out, dkv_stream_t stream, int32_t batch, int32_t block_table_stride,
                    int32_t num_dev_blocks) {
  return decode_impl(h, q, k_host, v_host, k_dev, v_dev, block_table, seq_lens, host_split, out, stream, batch,
                     block_table_stride, num_dev_blocks, nullptr, nullptr);
}

int dkv_append_kv(dkv_handle* h, const float* x, const void* w_k, const void* w_v, int32_t hidden,
                  const int32_t* block_table, const int32_t* seq_lens, int32_t host_split, void* k_host,
                  void* v_host, void* k_dev, void* v_dev, dkv_stream_t stream, int32_t batch,
                  int32_t block_table_stride, int32_t num_dev_blocks) {
  if (!h) return fail(DKV_ERR_INVALID_ARG, "dkv_append_kv: null handle");
  const dkv_config& c = h->cfg;
  if (batch < 0 || batch > c.max_batch) return fail(DKV_ERR_INVALID_ARG, "batch outside [0, max_batch]");
  if (batch == 0) return DKV_OK;
  if (!x || !w_k || !w_v || !block_table || !seq_lens) return fail(DKV_ERR_INVALID_ARG, "dkv_append_kv: null pointer");
  if (hidden <= 0 || hidden % 8 != 0) return fail(DKV_ERR_INVALID_ARG, "hidden must be a positive multiple of 8");
  if (block_table_stride < 1 || host_split < 0 || num_dev_blocks < 0 ||
      static_cast<long long>(host_split) + num_dev_blocks > INT_MAX)
    return fail(DKV_ERR_INVALID_ARG, "table stride / host_split / num_dev_blocks out of range");
  if ((host_split > 0 && (!k_host || !v_host)) || (num_dev_blocks > 0 && (!k_dev || !v_dev)))
    return fail(DKV_ERR_INVALID_ARG, "pool pointers are null");
  auto mis16 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) != 0; };
  if (mis16(x) || mis16(w_k) || mis16(w_v) || (host_split > 0 && (mis16(k_host) || mis16(v_host))) ||
      (num_dev_blocks > 0 && (mis16(k_dev) || mis16(v_dev))))
    return fail(DKV_ERR_INVALID_ARG, "x, weights and pools must be 16-byte aligned");
  DeviceGuard guard(c.device);
  if (!guard.ok) return fail(DKV_ERR_CUDA, "cudaSetDevice failed");
  int rc;
  if (host_split > 0) {
    if ((rc = check_host_pool(h, k_host, 0)) != DKV_OK) return rc;
    if ((rc = check_host_pool(h, v_host, 1)) != DKV_OK) return rc;
  }
  if (num_dev_blocks > 0) {
    if ((rc = check_dev_pool(h, k_dev, 0)) != DKV_OK) return rc;
    if ((rc = check_dev_pool(h, v_dev, 1)) != DKV_OK) return rc;
  }
  dkv::AppendParams ap{};
  ap.x = x;
  ap.w_k = static_cast<const uint16_t*>(w_k);
  ap.w_v = static_cast<const uint16_t*>(w_v);
  ap.table = block_table;
  ap.seq_lens = seq_lens;
  ap.k_host = static_cast<uint16_t*>(k_host);
  ap.v_host = static_cast<uint16_t*>(v_host);
  ap.k_dev = static_cast<uint16_t*>(k_dev);
  ap.v_dev = static_cast<uint16_t*>(v_dev);
  ap.status = h->status;
  ap.batch = batch;
  ap.hidden = hidden;
  ap.hkv = c.num_kv_heads;
  ap.head_dim = c.head_dim;
  ap.block_size = c.block_size;
  ap.stride = block_table_stride;
  ap.host_split = host_split;
  ap.num_dev_blocks = num_dev_blocks;
  ap.max_len = (block_table_stride < c.max_blocks_per_seq ? block_table_stride : c.max_blocks_per_seq) * c.block_size;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const dim3 grid(2 * c.num_kv_heads * c.head_dim / dkv::kAppendRows);
  if (c.kv_dtype == DKV_KV_BF16)
    dkv::append_kernel<true><<<grid, dkv::kAppendRows * 32, 0, s>>>(ap);
  else
    dkv::append_kernel<false><<<grid, dkv::kAppendRows * 32, 0, s>>>(ap);
  DKV_CUDA(cudaGetLastError());
  return DKV_OK;
}

int dkv_attn_decode_multi(dkv_handle* h, int32_t num_queries, const float* q, const void* k_host, const void* v_host,
                          const void* k_dev, const void* v_dev, const int32_t* block_table, const int32_t* seq_lens,
                          int32_t host_split, float* out, dkv_stream_t stream, int32_t batch,
                          int32_t block_table_stride, int32_t num_dev_blocks) {
  if (!h || num_queries < 1) return fail(DKV_ERR_INVALID_ARG, "dkv_attn_decode_multi: null handle or num_queries < 1");
  return decode_impl(h, q, k_host, v_host, k_dev, v_dev, block_table, seq_lens, host_split, out, stream, batch,
                     block_table_stride, num_dev_blocks, nullptr, nullptr, num_queries);
}

int dkv_attn_decode_staged(dkv_handle* h, const float* q, const void* k_host, const void* v_host, const void* k_dev,
                           const void* v_dev, const int32_t* block_table, const int32_t* seq_lens,
                           int32_t host_split, float* out, dkv_stream_t stream, int32_t batch,
                           int32_t block_table_stride, int32_t num_dev_blocks, void* k_stage, void* v_stage) {
  if (host_split > 0 && (!k_stage || !v_stage))
    return fail(DKV_ERR_INVALID_ARG, "dkv_attn_decode_staged: staging pools are null");
  return decode_impl(h, q, k_host, v_host, k_dev, v_dev, block_table, seq_lens, host_split, out, stream, batch,
                     block_table_stride, num_dev_blocks, host_split > 0 ? k_stage : nullptr,
                     host_split > 0 ? v_stage : nullptr);
}

int dkv_profile_begin(dkv_handle* h, int32_t max_calls) {
  if (!h || max_calls < 1 || max_calls > (1 << 20)) return fail(DKV_ERR_INVALID_ARG, "dkv_profile_begin: bad argument");
  DeviceGuard guard(h->cfg.device);
  prof_release(h);
  for (auto& v : h->prof_events) {
    v.assign(2 * static_cast<size_t>(max_calls), nullptr);
    for (cudaEvent_t& e : v) {
      cudaError_t err = cudaEventCreate(&e);
      if (err != cudaSuccess) {
        e = nullptr;
        prof_release(h);
        return cuda_fail(err, "cudaEventCreate");
      }
    }
  }
  h->prof_capacity = max_calls;
  return DKV_OK;
}

int dkv_profile_end(dkv_handle* h, float* ms, int32_t* counts) {
  if (!h || !ms || !counts) return fail(DKV_ERR_INVALID_ARG, "dkv_profile_end: null argument");
  DeviceGuard guard(h->cfg.device);
  cudaError_t err = cudaDeviceSynchronize();
  if (err != cudaSuccess) {
    prof_release(h);
    return cuda_fail(err, "cudaDeviceSynchronize");
  }
  for (int k = 0; k < 3; ++k) {
    double total = 0.0;
    for (int i = 0; i < h->prof_used[k]; ++i) {
      float t = 0.f;
      err = cudaEventElapsedTime(&t, h->prof_events[k][2 * i], h->prof_events[k][2 * i + 1]);
      if (err != cudaSuccess) {
        prof_release(h);
        return cuda_fail(err, "cudaEventElapsedTime");
      }
      total += t;
    }
    ms[k] = static_cast<float>(total);
    counts[k] = h->prof_used[k];
  }
  prof_release(h);
  return DKV_OK;
}

int dkv_get_status(dkv_handle* h, int32_t* status) {
  if (!h || !status) return fail(DKV_ERR_INVALID_ARG, "dkv_get_status: null argument");
  DeviceGuard guard(h->cfg.device);
  DKV_CUDA(cudaDeviceSynchronize());
  int32_t v = 0;
  DKV_CUDA(cudaMemcpy(&v, h->status, sizeof(v), cudaMemcpyDeviceToHost));
  DKV_CUDA(cudaMemset(h->status, 0, sizeof(int32_t)));
  *status = v;
  return DKV_OK;
}

int dkv_host_pool_alloc(size_t bytes, void** ptr) {
  if (!ptr || bytes == 0) return fail(DKV_ERR_INVALID_ARG, "dkv_host_pool_alloc: null pointer or zero size");
  *ptr = nullptr;
  cudaError_t e = cudaHostAlloc(ptr, bytes, cudaHostAllocMapped | cudaHostAllocPortable);
  if (e != cudaSuccess) {
    cudaGetLastError();
    *ptr = nullptr;
    return fail(e == cudaErrorMemoryAllocation ? DKV_ERR_NO_MEMORY : DKV_ERR_CUDA,
                std::string("cudaHostAlloc: ") + cudaGetErrorString(e));
  }
  return DKV_OK;
}

int dkv_host_pool_free(void* ptr) {
  if (!ptr) return DKV_OK;
  DKV_CUDA(cudaFreeHost(ptr));
  return DKV_OK;
}

}  // extern "C"
