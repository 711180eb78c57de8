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
#include "dkv_plan.h"
#include "dkv_tma.h"

namespace {

thread_local std::string g_err;
thread_local int g_fail_alloc = 0;   // test hook: the n-th device allocation of the next dkv_create fails
thread_local int g_stall_copy = 0;   // test hook: the next HBM launch leaves one tile copy unissued

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

#ifndef DKV_HOST_STAGES
#define DKV_HOST_STAGES 3
#endif
constexpr int kHostStages = DKV_HOST_STAGES;  // ring depth of the zero-copy host kernel (build-time knob)
#ifndef DKV_DEV_STAGES
#define DKV_DEV_STAGES 3
#endif
constexpr int kDevStages = DKV_DEV_STAGES;  // ring depth of the HBM kernel (build-time knob)
// How the HBM kernel moves its tiles (build-time knob): 0 always 16-byte
// cp.async; 1 (default) tensor copies when it runs beside the zero-copy host
// kernel and cp.async when it has the GPU to itself; 2 always tensor copies.
// Beside the host stream the cp.async loads of the HBM kernel slow to less
// than half speed while the tensor copies keep theirs; alone, cp.async is a
// few percent faster.
#ifndef DKV_DEV_TMA
#define DKV_DEV_TMA 1
#endif
constexpr int kDevTmaMode = DKV_DEV_TMA;
// How the zero-copy host kernel reads the mapped host pools (build-time
// knob): 0 (default) 16-byte cp.async; 1 tensor copies through tensor maps
// over the host pools.  Both reach the same share of the PCIe copy-engine
// rate (about 0.92); the link, not the SM's load path, sets it.
#ifndef DKV_HOST_TMA
#define DKV_HOST_TMA 0
#endif
constexpr bool kHostTma = DKV_HOST_TMA != 0;
// Units per resident warp of the HBM kernel (single- or multi-token) when all
// blocks sit in HBM and the batch holds 2 or more sequences (build-time
// knobs): up to DKV_DEV_REFINE (1 to 8; the partial-row workspace covers 8)
// while each unit keeps at least DKV_DEV_UNIT_TOKENS tokens.  With ragged
// lengths the plan, sized by the table capacity, otherwise gives the longest
// sequences units as long as a warp's whole share (an all-HBM batch of 16
// sequences of 1k-16k tokens ran 1.9x faster with 2 units per warp, with 4
// query tokens 1.95x); uniform batches are unchanged within 1%.  One sequence
// cannot be ragged and keeps one unit per warp.
#ifndef DKV_DEV_REFINE
#define DKV_DEV_REFINE 2
#endif
#ifndef DKV_DEV_UNIT_TOKENS
#define DKV_DEV_UNIT_TOKENS 1024
#endif
constexpr int kDevRefine = DKV_DEV_REFINE;
constexpr int kDevUnitTokens = DKV_DEV_UNIT_TOKENS;
static_assert(kDevRefine >= 1 && kDevRefine <= 8, "DKV_DEV_REFINE must be 1..8");
// CTAs of the zero-copy host kernel when the configuration leaves it to the
// library: every count from 4 to 24 keeps the PCIe link at 0.91-0.925 of the
// copy engine's rate, but the HBM kernel beside it loses speed as the count
// grows (its L2 shares the host kernel's long-latency sysmem reads: 4970,
// 4800, 4490, 3780 GB/s with 4, 8, 16, 24 host CTAs).  A call whose host part
// carries the step takes 16 (0.924 against 0.917 with 8 on a 90%-host step);
// one whose host part is small against its HBM part takes 8 (for a 1M-token
// sequence, 4 GiB of KV, the planned placement under a 99% HBM budget then
// ran 1.00 ms, with 1.1% of the blocks on the host, against 1.31 ms with 16
// host CTAs, with 1.5%).
constexpr int kDefaultHostCtas = 16;
constexpr int kLightHostCtas = 8;
// The host part carries the step when its blocks are at least this share of
// the HBM part's: B_pcie / B_hbm is about 1/100, so from 1/50 on the host
// stream takes at least twice as long as the HBM kernel.
constexpr int kHostCarriesDenominator = 50;
constexpr int kListThreads = 1024;  // threads of the pool-lists kernel

// cudaMalloc, or a simulated out-of-memory failure when the test hook
// (dkv_debug_fail_alloc) has armed this allocation.
cudaError_t dev_alloc(void** p, size_t bytes, int* counter) {
  if (g_fail_alloc > 0 && ++*counter == g_fail_alloc) {
    g_fail_alloc = 0;
    *p = nullptr;
    return cudaErrorMemoryAllocation;
  }
  return cudaMalloc(p, bytes);
}

size_t split_smem(int D, int nst) { return dkv::split_smem_bytes(D, nst); }

using SplitFn = void (*)(dim3, size_t, cudaStream_t, const dkv::SplitParams&, const dkv::TileMaps&);
using SplitKernelPtr = const void*;

template <int D, int G, bool BF16, int NST, bool ROPE, bool TMA>
void launch_split(dim3 grid, size_t smem, cudaStream_t s, const dkv::SplitParams& p, const dkv::TileMaps& m) {
  dkv::split_kernel<D, G, BF16, NST, ROPE, TMA><<<grid, dkv::kThreads, smem, s>>>(p, m);
}
template <int D, int G, bool BF16, int NST, bool ROPE, bool TMA>
const void* split_ptr() {
  return reinterpret_cast<const void*>(&dkv::split_kernel<D, G, BF16, NST, ROPE, TMA>);
}

struct SplitEntry {
  SplitFn fn;
  SplitKernelPtr ptr;
};

// TMA: the HBM launch (tiles by tensor copies); otherwise the zero-copy host
// launch (16-byte cp.async from mapped host memory).
template <int NST, bool ROPE, bool TMA>
SplitEntry pick_split_rope(int D, int G, bool bf16) {
#define DKV_CASE(DD, GG)                                                                                     \
  if (D == DD && G == GG) {                                                                                  \
    if (bf16) return {&launch_split<DD, GG, true, NST, ROPE, TMA>, split_ptr<DD, GG, true, NST, ROPE, TMA>()}; \
    return {&launch_split<DD, GG, false, NST, ROPE, TMA>, split_ptr<DD, GG, false, NST, ROPE, TMA>()};         \
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

template <int NST, bool TMA>
SplitEntry pick_split(int D, int G, bool bf16, bool rope) {
  return rope ? pick_split_rope<NST, true, TMA>(D, G, bf16) : pick_split_rope<NST, false, TMA>(D, G, bf16);
}

template <int D, bool BF16, bool ROPE>
void launch_multi(dim3 grid, size_t smem, cudaStream_t s, const dkv::SplitParams& p, const dkv::TileMaps&) {
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
size_t multi_smem(int D) { return dkv::multi_smem_bytes(D); }

// The append kernel for `nb` sequences per pass (1, 2, 4, 8 or 16).
template <bool BF16, int NB>
cudaError_t launch_append_nb(dim3 grid, cudaStream_t s, const dkv::AppendParams& ap) {
  const size_t smem = dkv::append_smem_bytes(NB);
  // once per process and instance (the attribute holds for every device): the
  // kernel's static and dynamic shared memory together may pass 48 KB
  static const cudaError_t set = cudaFuncSetAttribute(dkv::append_kernel<BF16, NB>,
                                                      cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                      static_cast<int>(smem));
  if (set != cudaSuccess) return set;
  dkv::append_kernel<BF16, NB><<<grid, dkv::kAppendWarps * 32, smem, s>>>(ap);
  return cudaGetLastError();
}
template <bool BF16>
cudaError_t launch_append_t(int nb, dim3 grid, cudaStream_t s, const dkv::AppendParams& ap) {
  switch (nb) {
    case 1: return launch_append_nb<BF16, 1>(grid, s, ap);
    case 2: return launch_append_nb<BF16, 2>(grid, s, ap);
    case 4: return launch_append_nb<BF16, 4>(grid, s, ap);
    case 8: return launch_append_nb<BF16, 8>(grid, s, ap);
    default: return launch_append_nb<BF16, dkv::kAppendBatch>(grid, s, ap);
  }
}
cudaError_t launch_append(bool bf16, int nb, dim3 grid, cudaStream_t s, const dkv::AppendParams& ap) {
  return bf16 ? launch_append_t<true>(nb, grid, s, ap) : launch_append_t<false>(nb, grid, s, ap);
}

// The merge, optionally as a programmatic dependent launch of the split kernel
// just before it on the stream: its grid is set up while that kernel drains
// and its first instruction waits for that kernel's results.
using MergeFn = cudaError_t (*)(int, cudaStream_t, const dkv::MergeParams&, bool);
template <int D>
cudaError_t launch_merge(int rows, cudaStream_t s, const dkv::MergeParams& p, bool dependent) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(rows);
  cfg.blockDim = dim3(32 * dkv::merge_warps(p.nslots, D));
  cfg.dynamicSmemBytes = 0;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = dependent ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, dkv::merge_kernel<D>, p);
}

}  // namespace

struct dkv_handle {
  dkv_config cfg{};
  int G = 0;
  int sm_count = 0;
  int beside_host = 0;        // HBM-kernel CTAs that fit on an SM beside a host-kernel CTA (0 or 1)
  int units_target = 0;       // warps of the widest split launch (one resident wave: 2 CTAs per SM)
  size_t part_rows = 0;
  float qscale = 0.f;
  int host_ctas = 0;           // the configuration's count; 0: chosen per call
  float* part_o = nullptr;
  float* part_lse = nullptr;
  int32_t* status = nullptr;
  int32_t* work = nullptr;    // [4]: work counters of the host-side and the device-side split launch
  int2* lists = nullptr;      // [max_batch][max_blocks_per_seq]: per-pool block lists of a mixed call
  int2* counts = nullptr;     // [max_batch]
  double* inv_freq = nullptr;
  cudaStream_t aux = nullptr;
  cudaEvent_t ev_fork = nullptr;
  cudaEvent_t ev_join = nullptr;
  SplitEntry host_kernel{}, dev_kernel{}, dev_tma_kernel{}, multi_kernel{};  // dev: cp.async; dev_tma: tensor copies
  // tensor maps of the last device pool and staging pool the HBM kernel read
  struct PoolMaps {
    const void* k = nullptr;
    const void* v = nullptr;
    long long rows = -1;
    dkv::TileMaps maps{};
  } dev_maps, stage_maps, host_maps;
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
  cudaFree(h->work);
  cudaFree(h->lists);
  cudaFree(h->counts);
  cudaFree(h->inv_freq);
  if (h->ev_fork) cudaEventDestroy(h->ev_fork);
  if (h->ev_join) cudaEventDestroy(h->ev_join);
  if (h->aux) cudaStreamDestroy(h->aux);
  delete h;
}

// Warps a split launch can keep resident: 2 CTAs of kWarps warps per SM, less
// the SMs' share the zero-copy host kernel's host_ctas CTAs hold while it runs
// beside it (host_ctas = 0: it does not).
long launch_warps(const dkv_handle* h, int host_ctas) {
  const long ctas = 2L * h->sm_count - static_cast<long>(host_ctas) * (2 - h->beside_host);
  return dkv::kWarps * (ctas > 1 ? ctas : 1);
}

// Whether the host part of a call with these pool sizes carries its step.
bool host_carries(long long host_blocks, long long dev_blocks) {
  return host_blocks * kHostCarriesDenominator >= dev_blocks;
}

// CTAs of the zero-copy host kernel for a call with these pool sizes.
int call_host_ctas(const dkv_handle* h, long long host_blocks, long long dev_blocks) {
  if (h->host_ctas > 0) return h->host_ctas;
  return host_carries(host_blocks, dev_blocks) ? kDefaultHostCtas : kLightHostCtas;
}

// Split plan of the HBM kernel of a call whose blocks all sit in HBM (the
// only split launch of the call).
dkv::SplitPlan alone_plan(const dkv_handle* h, int nblk, int batch) {
  const long per = static_cast<long>(batch) * h->cfg.num_kv_heads;
  return dkv::plan_split_refined(nblk, per, h->cfg.block_size, launch_warps(h, 0),
                                 batch < 2 ? 1 : kDevRefine, kDevUnitTokens);
}

// Whether one CTA of kernel b fits on an SM that holds one CTA of kernel a,
// by registers and shared memory.
int fits_beside(const void* a, size_t smem_a, const void* b, size_t smem_b, int device) {
  cudaFuncAttributes fa{}, fb{};
  int regs_sm = 0, smem_sm = 0, reserved = 0;
  if (cudaFuncGetAttributes(&fa, a) != cudaSuccess || cudaFuncGetAttributes(&fb, b) != cudaSuccess ||
      cudaDeviceGetAttribute(&regs_sm, cudaDevAttrMaxRegistersPerMultiprocessor, device) != cudaSuccess ||
      cudaDeviceGetAttribute(&smem_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, device) != cudaSuccess ||
      cudaDeviceGetAttribute(&reserved, cudaDevAttrReservedSharedMemoryPerBlock, device) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  const long regs = static_cast<long>(fa.numRegs + fb.numRegs) * dkv::kThreads;
  const size_t smem = smem_a + smem_b + fa.sharedSizeBytes + fb.sharedSizeBytes + 2 * static_cast<size_t>(reserved);
  return regs <= regs_sm && smem <= static_cast<size_t>(smem_sm) ? 1 : 0;
}

// The tensor maps of a device-resident pool pair of `blocks` blocks (cached per handle).
int pool_maps(dkv_handle* h, dkv_handle::PoolMaps& cache, const void* k, const void* v, long long blocks,
              const dkv::TileMaps** out) {
  const long long rows = blocks * h->cfg.num_kv_heads * h->cfg.block_size;
  if (rows >= (1LL << 31)) return fail(DKV_ERR_INVALID_ARG, "a pool holds 2^31 or more token rows");
  if (cache.k != k || cache.v != v || cache.rows != rows) {
    cache.rows = -1;
    if (!dkv::encode_pool_map(&cache.maps.k, k, rows, h->cfg.head_dim, true) ||
        !dkv::encode_pool_map(&cache.maps.v, v, rows, h->cfg.head_dim, false))
      return fail(DKV_ERR_CUDA, "cuTensorMapEncodeTiled rejected the pool's tensor map");
    cache.k = k;
    cache.v = v;
    cache.rows = rows;
  }
  *out = &cache.maps;
  return DKV_OK;
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
  h->host_ctas = c.host_ctas;
  const bool rope = c.rope_base > 0.0;
  h->host_kernel = pick_split<kHostStages, kHostTma>(c.head_dim, G, bf16, rope);
  h->dev_kernel = pick_split<kDevStages, false>(c.head_dim, G, bf16, rope);
  h->dev_tma_kernel = pick_split<kDevStages, true>(c.head_dim, G, bf16, rope);
  h->multi_kernel = pick_multi(c.head_dim, bf16, c.rope_base > 0.0);
  h->merge = c.head_dim == 64 ? &launch_merge<64> : &launch_merge<128>;

  auto bail = [&](int code) {
    release(h);
    return code;
  };
  cudaError_t e = cudaDeviceGetAttribute(&h->sm_count, cudaDevAttrMultiProcessorCount, c.device);
  if (e != cudaSuccess) return bail(cuda_fail(e, "cudaDeviceGetAttribute"));
  h->beside_host = fits_beside(h->host_kernel.ptr, split_smem(c.head_dim, kHostStages),
                               (kDevTmaMode == 0 ? h->dev_kernel : h->dev_tma_kernel).ptr,
                               split_smem(c.head_dim, kDevStages), c.device);
  h->units_target = static_cast<int>(launch_warps(h, 0));
  // partial rows: batch * Tq * Hq * (host splits + device splits), each launch's
  // splits <= max(1, units_target / (batch * Hkv)); Tq * G <= 16 rows per unit
  // (multi-token queries) and batch * Tq <= max_batch
  h->part_rows = 2ull * (static_cast<size_t>(dkv::kMultiMaxRows) * h->units_target +
                         static_cast<size_t>(G) * c.max_batch * c.num_kv_heads);
  const size_t list_entries = static_cast<size_t>(c.max_batch) * c.max_blocks_per_seq;
  e = cudaFuncSetAttribute(h->host_kernel.ptr, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(split_smem(c.head_dim, kHostStages)));
  if (e != cudaSuccess) return bail(cuda_fail(e, "cudaFuncSetAttribute(host kernel)"));
  for (const SplitEntry* k : {&h->dev_kernel, &h->dev_tma_kernel}) {
    e = cudaFuncSetAttribute(k->ptr, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(split_smem(c.head_dim, kDevStages)));
    if (e != cudaSuccess) return bail(cuda_fail(e, "cudaFuncSetAttribute(HBM kernel)"));
  }
  e = cudaFuncSetAttribute(h->multi_kernel.ptr, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(multi_smem(c.head_dim)));
  if (e != cudaSuccess) return bail(cuda_fail(e, "cudaFuncSetAttribute(multi-token kernel)"));
  // every kernel of a step prefers the largest shared-memory carveout, so an SM
  // need not change its L1/shared split between the step's kernels
  {
    const void* all[] = {h->host_kernel.ptr, h->dev_kernel.ptr, h->dev_tma_kernel.ptr, h->multi_kernel.ptr,
                         reinterpret_cast<const void*>(&dkv::lists_kernel<kListThreads>),
                         reinterpret_cast<const void*>(c.head_dim == 64 ? &dkv::merge_kernel<64>
                                                                         : &dkv::merge_kernel<128>)};
    for (const void* f : all) {
      e = cudaFuncSetAttribute(f, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
      if (e != cudaSuccess) return bail(cuda_fail(e, "cudaFuncSetAttribute(carveout)"));
    }
  }
  int nalloc = 0;
  const bool armed = g_fail_alloc > 0;
  if (dev_alloc(reinterpret_cast<void**>(&h->part_o), h->part_rows * c.head_dim * sizeof(float), &nalloc) ||
      dev_alloc(reinterpret_cast<void**>(&h->part_lse), h->part_rows * sizeof(float), &nalloc) ||
      dev_alloc(reinterpret_cast<void**>(&h->status), sizeof(int32_t), &nalloc) ||
      dev_alloc(reinterpret_cast<void**>(&h->work), 4 * sizeof(int32_t), &nalloc) ||
      dev_alloc(reinterpret_cast<void**>(&h->lists), list_entries * sizeof(int2), &nalloc) ||
      dev_alloc(reinterpret_cast<void**>(&h->counts), c.max_batch * sizeof(int2), &nalloc) ||
      dev_alloc(reinterpret_cast<void**>(&h->inv_freq), sizeof(double) * (c.head_dim / 2), &nalloc)) {
    cudaGetLastError();
    return bail(fail(DKV_ERR_NO_MEMORY, "workspace allocation failed"));
  }
  if (armed) g_fail_alloc = 0;   // the hook covers one dkv_create only
  double freq[64];
  dkv::rope_frequencies(c.rope_base, c.head_dim, freq);
  e = cudaMemcpy(h->inv_freq, freq, sizeof(double) * (c.head_dim / 2), cudaMemcpyHostToDevice);
  if (e != cudaSuccess) return bail(cuda_fail(e, "cudaMemcpy(inv_freq)"));
  e = cudaMemset(h->status, 0, sizeof(int32_t));
  if (e != cudaSuccess) return bail(cuda_fail(e, "cudaMemset(status)"));
  e = cudaMemset(h->work, 0, 4 * sizeof(int32_t));
  if (e != cudaSuccess) return bail(cuda_fail(e, "cudaMemset(work counters)"));
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
  const int nblk = block_table_stride < h->cfg.max_blocks_per_seq ? block_table_stride : h->cfg.max_blocks_per_seq;
  const dkv::SplitPlan pl = alone_plan(h, nblk, batch);
  *num_splits = pl.nsplit;
  *blocks_per_split = pl.bps;
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
  // Launches: the host-side one (zero-copy host kernel on the auxiliary stream,
  // or for the staged comparator the HBM kernel over the staging pools) and the
  // device-side one (HBM kernel over the device pool).  With no pool at all the
  // device-side launch still runs, so that table entries are checked.
  const bool run_host = host_split > 0;
  const bool run_dev = num_dev_blocks > 0 || !run_host;
  const bool concurrent = run_host && !staged;   // host kernel beside the HBM kernel
  const bool use_lists = run_host && run_dev;    // each launch walks the list of its own pool's blocks
  const int nblk_cap = block_table_stride < c.max_blocks_per_seq ? block_table_stride : c.max_blocks_per_seq;
  const long per = static_cast<long>(batch) * c.num_kv_heads;
  const int host_ctas = concurrent ? call_host_ctas(h, host_split, num_dev_blocks) : 0;
  const long host_warps = staged ? launch_warps(h, 0) : static_cast<long>(dkv::kWarps) * host_ctas;
  const dkv::SplitPlan ph = dkv::plan_split(nblk_cap, per, c.block_size, host_warps, 0);
  // Beside the host stream the HBM launch plans one unit per warp while the
  // host part carries the step (finer units there speed up a kernel that does
  // not set the step and slow the host stream beside it: 1.8-5% on 10-25%
  // host placements) and two while the HBM part does (16 ragged sequences
  // with 1% of their blocks on the host: 790 -> 663 us).
  const dkv::SplitPlan pd =
      !run_host ? alone_plan(h, nblk_cap, batch)
                : dkv::plan_split_refined(nblk_cap, per, c.block_size, launch_warps(h, host_ctas),
                                          staged || batch < 2 || host_carries(host_split, num_dev_blocks)
                                              ? 1 : kDevRefine,
                                          kDevUnitTokens);
  const int nsplit_h = run_host ? ph.nsplit : 0;
  const int nsplit_d = run_dev ? pd.nsplit : 0;
  const int nslots = nsplit_h + nsplit_d;
  if (static_cast<size_t>(batch) * nq * c.num_q_heads * nslots > h->part_rows)
    return fail(DKV_ERR_INVALID_ARG, "internal: split plan exceeds the workspace");
  const int min_bps = dkv::min_blocks_per_split(c.block_size);

  dkv::SplitParams sp{};
  sp.lists = use_lists ? h->lists : nullptr;
  sp.counts = h->counts;
  sp.list_stride = nblk_cap;
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
  sp.nslots = nslots;
  sp.id_total = host_split + num_dev_blocks;
  sp.max_len = nblk_cap * c.block_size;
  sp.rope = c.rope_base > 0.0 ? 1 : 0;
  sp.qscale = h->qscale;
  sp.extra_tokens = nq - 1;
  sp.num_queries = nq;
  auto launch_params = [&](int nsplit, int bps, int slot_base, bool dev_list, int32_t* work) {
    dkv::SplitParams lp = sp;
    lp.nsplit = nsplit;
    lp.bps = use_lists ? min_bps : bps;
    lp.slot_base = slot_base;
    lp.list_dev = dev_list ? 1 : 0;
    lp.work = work;
    lp.n_units = batch * nsplit * c.num_kv_heads;
    dkv::set_divisors(lp);
    return lp;
  };
  const bool dev_tma = !multi && (kDevTmaMode == 2 || (kDevTmaMode == 1 && concurrent));
  const SplitEntry& host_k = multi ? h->multi_kernel : h->host_kernel;
  const SplitEntry& dev_k = multi ? h->multi_kernel : (dev_tma ? h->dev_tma_kernel : h->dev_kernel);
  const SplitEntry& stage_k = multi ? h->multi_kernel : (kDevTmaMode == 2 ? h->dev_tma_kernel : h->dev_kernel);
  const size_t host_smem = multi ? multi_smem(c.head_dim) : split_smem(c.head_dim, kHostStages);
  const size_t dev_smem = multi ? multi_smem(c.head_dim) : split_smem(c.head_dim, kDevStages);
  auto ctas_for = [&](const dkv::SplitParams& lp, int cap) {
    const int u = (lp.n_units + dkv::kWarps - 1) / dkv::kWarps;
    return u < cap ? u : cap;
  };

  int launches = 0;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  static const dkv::TileMaps no_maps{};   // for launches that copy with cp.async
  if (use_lists) {
    dkv::ListParams lp{};
    lp.table = block_table;
    lp.seq_lens = seq_lens;
    lp.lists = h->lists;
    lp.counts = h->counts;
    lp.stride = block_table_stride;
    lp.list_stride = nblk_cap;
    lp.block_size = c.block_size;
    lp.host_split = host_split;
    lp.id_total = host_split + num_dev_blocks;
    lp.max_len = sp.max_len;
    lp.extra_tokens = nq - 1;
    lp.invalid_to_dev = 1;
    dkv::lists_kernel<kListThreads><<<batch, kListThreads, 0, s>>>(lp);
    DKV_CUDA(cudaGetLastError());
    ++launches;
  }
  bool merge_follows_split = false;   // the merge directly follows a split kernel on `s`
  if (run_host && staged) {
    // copy engine: pinned host pools -> HBM staging pools, then the HBM kernel reads them
    const size_t bytes = static_cast<size_t>(host_split) * c.num_kv_heads * c.block_size * c.head_dim * 2;
    if ((rc = prof_mark(h, 0, s, false)) != DKV_OK) return rc;
    DKV_CUDA(cudaMemcpyAsync(k_stage, k_host, bytes, cudaMemcpyHostToDevice, s));
    DKV_CUDA(cudaMemcpyAsync(v_stage, v_host, bytes, cudaMemcpyHostToDevice, s));
    dkv::SplitParams hp = launch_params(nsplit_h, ph.bps, 0, false, h->work);
    hp.k_pool = static_cast<const uint16_t*>(k_stage);
    hp.v_pool = static_cast<const uint16_t*>(v_stage);
    hp.id_lo = 0;
    hp.id_hi = host_split;
    const dkv::TileMaps* maps = &no_maps;
    if (!multi && kDevTmaMode == 2 && (rc = pool_maps(h, h->stage_maps, k_stage, v_stage, host_split, &maps)) != DKV_OK)
      return rc;
    stage_k.fn(dim3(ctas_for(hp, 2 * h->sm_count)), dev_smem, s, hp, *maps);
    DKV_CUDA(cudaGetLastError());
    if ((rc = prof_mark(h, 0, s, true)) != DKV_OK) return rc;
    ++launches;
  } else if (run_host) {
    DKV_CUDA(cudaEventRecord(h->ev_fork, s));
    DKV_CUDA(cudaStreamWaitEvent(h->aux, h->ev_fork, 0));
    dkv::SplitParams hp = launch_params(nsplit_h, ph.bps, 0, false, h->work);
    hp.k_pool = static_cast<const uint16_t*>(k_host);
    hp.v_pool = static_cast<const uint16_t*>(v_host);
    hp.id_lo = 0;
    hp.id_hi = host_split;
    const dkv::TileMaps* hmaps = &no_maps;
    if (kHostTma && !multi && (rc = pool_maps(h, h->host_maps, k_host, v_host, host_split, &hmaps)) != DKV_OK)
      return rc;
    if ((rc = prof_mark(h, 0, h->aux, false)) != DKV_OK) return rc;
    host_k.fn(dim3(ctas_for(hp, host_ctas)), host_smem, h->aux, hp, *hmaps);
    DKV_CUDA(cudaGetLastError());
    if ((rc = prof_mark(h, 0, h->aux, true)) != DKV_OK) return rc;
    DKV_CUDA(cudaEventRecord(h->ev_join, h->aux));
    ++launches;
  }
  if (run_dev) {
    dkv::SplitParams dp = launch_params(nsplit_d, pd.bps, nsplit_h, true, h->work + 2);
    dp.k_pool = static_cast<const uint16_t*>(k_dev);
    dp.v_pool = static_cast<const uint16_t*>(v_dev);
    dp.id_lo = host_split;
    dp.id_hi = host_split + num_dev_blocks;
    if (dev_tma && g_stall_copy) {
      dp.stall_first_copy = 1;
      g_stall_copy = 0;
    }
    const dkv::TileMaps* maps = &no_maps;
    if (dev_tma && num_dev_blocks > 0 &&
        (rc = pool_maps(h, h->dev_maps, k_dev, v_dev, num_dev_blocks, &maps)) != DKV_OK)
      return rc;
    if ((rc = prof_mark(h, 1, s, false)) != DKV_OK) return rc;
    // at most one resident wave of CTAs; units are handed out dynamically, so
    // CTAs that find no SM free until others finish simply find no work left
    dev_k.fn(dim3(ctas_for(dp, 2 * h->sm_count)), dev_smem, s, dp, *maps);
    DKV_CUDA(cudaGetLastError());
    if ((rc = prof_mark(h, 1, s, true)) != DKV_OK) return rc;
    ++launches;
    merge_follows_split = !concurrent && h->prof_capacity == 0;
  }
  if (concurrent) DKV_CUDA(cudaStreamWaitEvent(s, h->ev_join, 0));
  dkv::MergeParams mp{};
  mp.part_o = h->part_o;
  mp.part_lse = h->part_lse;
  mp.out = out;
  mp.nslots = nslots;
  mp.nsplit = nsplit_h;
  mp.has_host = run_host;
  mp.has_dev = run_dev;
  if ((rc = prof_mark(h, 2, s, false)) != DKV_OK) return rc;
  DKV_CUDA(h->merge(batch * nq * c.num_q_heads, s, mp, merge_follows_split));
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
  // sequences per pass: the smallest of 1, 2, 4, 8, 16 that covers the batch (16 for larger batches)
  const int nb = batch > 8 ? dkv::kAppendBatch : batch > 4 ? 8 : batch > 2 ? 4 : batch;
  const dim3 grid(2 * c.num_kv_heads * c.head_dim / dkv::append_cta_rows(nb));
  DKV_CUDA(launch_append(c.kv_dtype == DKV_KV_BF16, nb, grid, s, ap));
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

int dkv_profile_timeline(dkv_handle* h, int32_t call, float* t_ms) {
  if (!h || !t_ms || call < 0) return fail(DKV_ERR_INVALID_ARG, "dkv_profile_timeline: bad argument");
  DeviceGuard guard(h->cfg.device);
  DKV_CUDA(cudaDeviceSynchronize());
  // the kernels of call `call`: kernel k took part if its call-th event pair was recorded
  const cudaEvent_t none = nullptr;
  cudaEvent_t ev[3][2] = {{none, none}, {none, none}, {none, none}};
  for (int k = 0; k < 3; ++k)
    if (call < h->prof_used[k]) {
      ev[k][0] = h->prof_events[k][2 * call];
      ev[k][1] = h->prof_events[k][2 * call + 1];
    }
  // reference: the earliest start among the kernels that ran
  int ref = -1;
  for (int k = 0; k < 3 && ref < 0; ++k)
    if (ev[k][0]) ref = k;
  if (ref < 0) return fail(DKV_ERR_INVALID_ARG, "dkv_profile_timeline: no kernel of that call was recorded");
  for (int k = 0; k < 3; ++k) {
    if (!ev[k][0]) continue;
    float d = 0.f;
    DKV_CUDA(cudaEventElapsedTime(&d, ev[ref][0], ev[k][0]));
    if (d < 0.f) ref = k;
  }
  for (int k = 0; k < 3; ++k) {
    for (int e = 0; e < 2; ++e) {
      if (!ev[k][0]) {
        t_ms[2 * k + e] = -1.f;
        continue;
      }
      float d = 0.f;
      DKV_CUDA(cudaEventElapsedTime(&d, ev[ref][0], ev[k][e]));
      t_ms[2 * k + e] = d;
    }
  }
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

int dkv_debug_fail_alloc(int32_t nth) {
  if (nth < 0) return fail(DKV_ERR_INVALID_ARG, "dkv_debug_fail_alloc: nth must be >= 0");
  g_fail_alloc = nth;
  return DKV_OK;
}

int dkv_debug_stall_copy(int32_t enable) {
  g_stall_copy = enable ? 1 : 0;
  return DKV_OK;
}

int dkv_debug_rope(int32_t kv_dtype, int32_t head_dim, double rope_base, const void* k, const int32_t* tile_pos,
                   int32_t num_tiles, float* k_out, const float* q, const int32_t* q_pos, int32_t num_q,
                   float* q_out, dkv_stream_t stream) {
  if (kv_dtype != DKV_KV_F16 && kv_dtype != DKV_KV_BF16) return fail(DKV_ERR_INVALID_ARG, "dkv_debug_rope: kv_dtype");
  if (head_dim != 64 && head_dim != 128) return fail(DKV_ERR_UNSUPPORTED, "dkv_debug_rope: head_dim must be 64 or 128");
  if (!(rope_base > 1.0) || !std::isfinite(rope_base)) return fail(DKV_ERR_INVALID_ARG, "dkv_debug_rope: rope_base must be > 1");
  if (num_tiles < 0 || num_q < 0 || (num_tiles > 0 && (!k || !tile_pos || !k_out)) ||
      (num_q > 0 && (!q || !q_pos || !q_out)))
    return fail(DKV_ERR_INVALID_ARG, "dkv_debug_rope: null pointer or negative count");
  if ((reinterpret_cast<uintptr_t>(k) & 15u) || (reinterpret_cast<uintptr_t>(k_out) & 7u) ||
      (reinterpret_cast<uintptr_t>(q) & 7u) || (reinterpret_cast<uintptr_t>(q_out) & 7u))
    return fail(DKV_ERR_INVALID_ARG, "dkv_debug_rope: k must be 16-byte and k_out, q, q_out 8-byte aligned");
  if (num_tiles == 0 && num_q == 0) return DKV_OK;
  dkv::RopeFreqs fr{};
  dkv::rope_frequencies(rope_base, head_dim, fr.w);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const uint16_t* k16 = static_cast<const uint16_t*>(k);
  const bool bf16 = kv_dtype == DKV_KV_BF16;
  if (head_dim == 64 && bf16)
    dkv::rope_debug_kernel<64, true><<<1, 32, 0, s>>>(fr, k16, tile_pos, num_tiles, k_out, q, q_pos, num_q, q_out);
  else if (head_dim == 64)
    dkv::rope_debug_kernel<64, false><<<1, 32, 0, s>>>(fr, k16, tile_pos, num_tiles, k_out, q, q_pos, num_q, q_out);
  else if (bf16)
    dkv::rope_debug_kernel<128, true><<<1, 32, 0, s>>>(fr, k16, tile_pos, num_tiles, k_out, q, q_pos, num_q, q_out);
  else
    dkv::rope_debug_kernel<128, false><<<1, 32, 0, s>>>(fr, k16, tile_pos, num_tiles, k_out, q, q_pos, num_q, q_out);
  DKV_CUDA(cudaGetLastError());
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
