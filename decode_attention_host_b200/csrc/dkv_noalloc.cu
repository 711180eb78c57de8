// dkv_noalloc.cu -- decode attention for callers that cannot allocate.
//
// dkv_attn_decode needs a handle, and dkv_create allocates the handle's
// workspace (split partials, a status word, an auxiliary stream, events).
// Some callers cannot do that.  One case is a serving engine that reserves
// all GPU memory for its own allocator at start-up, so a later cudaMalloc
// from a library fails or breaks the engine's accounting.  Another is a
// latency-critical decode loop, where cudaMalloc and cudaFree may
// synchronise the device.  A third is a plugin behind a plain C interface
// that receives raw pointers on every call and has nowhere to keep a handle.
// dkv_attn_decode_noalloc serves these callers.  It launches the same split
// and merge kernels, but its scratch memory is the fixed array below, which
// is compiled into this library.  Every GPU that loads the library holds the
// array until the process exits.
//
// The array is shared by every call on a device and keeps what the last call
// left in it.  Calls that overlap on the GPU (on different streams, or from
// different threads) therefore race on it: the caller must order them.  The
// status word is cleared at the start of each call; every partial slot the
// merge reads is written by the same call before it is read.
#include <cuda_runtime.h>

#include <mutex>
#include <string>

#include "dkv.h"
#include "dkv_error.h"
#include "dkv_kernels.cuh"
#include "dkv_plan.h"
#include "dkv_tma.h"

namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[DKV_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
#ifndef DKV_HOST_STAGES
#define DKV_HOST_STAGES 3
#endif
constexpr int kHostStages = DKV_HOST_STAGES;
#ifndef DKV_DEV_STAGES
#define DKV_DEV_STAGES 3
#endif
constexpr int kDevStages = DKV_DEV_STAGES;
// HBM-kernel copy path, as in dkv_api.cu: here the split kernels run one
// after the other, never beside each other, so tensor copies are used only
// when the knob asks for them always (2).
#ifndef DKV_DEV_TMA
#define DKV_DEV_TMA 1
#endif
constexpr bool kDevTma = DKV_DEV_TMA == 2;
constexpr int kHostCtas = 16;
constexpr int kListThreads = 1024;
constexpr size_t kStatusOffset = 0;     // int32 status word
constexpr size_t kWorkOffset = 16;      // int32 [4]: work counters of the host-side and device-side launches
constexpr size_t kFreqOffset = 256;     // up to 64 fp64 RoPE frequencies
static_assert(kFreqOffset + 64 * sizeof(double) <= dkv::kNoallocHeader, "header layout");

// Per-device set-up: the device address of the scratch array and the SM
// count.  Done once per device, on the first call.
struct DeviceSetup {
  std::mutex mu;
  bool done = false;
  unsigned char* scratch = nullptr;
  int sm_count = 0;
};
DeviceSetup g_setup[kMaxDevices];

size_t split_smem(int D, int nst) { return dkv::split_smem_bytes(D, nst); }

using SplitLaunch = void (*)(dim3, size_t, cudaStream_t, const dkv::SplitParams&, const dkv::TileMaps&);
struct SplitVariant {
  SplitLaunch launch;
  const void* fn;
};

template <int D, int G, bool BF16, int NST, bool ROPE, bool TMA>
void launch_split(dim3 grid, size_t smem, cudaStream_t s, const dkv::SplitParams& p, const dkv::TileMaps& m) {
  dkv::split_kernel<D, G, BF16, NST, ROPE, TMA><<<grid, dkv::kThreads, smem, s>>>(p, m);
}

// TMA: the HBM launch; otherwise the zero-copy host launch.
template <int NST, bool ROPE, bool TMA>
SplitVariant pick_rope(int D, int G, bool bf16) {
#define DKV_NA_CASE(DD, GG)                                                                                     \
  if (D == DD && G == GG)                                                                                       \
    return bf16 ? SplitVariant{&launch_split<DD, GG, true, NST, ROPE, TMA>,                                     \
                               reinterpret_cast<const void*>(&dkv::split_kernel<DD, GG, true, NST, ROPE, TMA>)} \
                : SplitVariant{&launch_split<DD, GG, false, NST, ROPE, TMA>,                                    \
                               reinterpret_cast<const void*>(&dkv::split_kernel<DD, GG, false, NST, ROPE, TMA>)};
  DKV_NA_CASE(64, 1)
  DKV_NA_CASE(64, 2)
  DKV_NA_CASE(64, 4)
  DKV_NA_CASE(128, 1)
  DKV_NA_CASE(128, 2)
  DKV_NA_CASE(128, 4)
#undef DKV_NA_CASE
  return {nullptr, nullptr};
}

template <int NST, bool TMA>
SplitVariant pick(int D, int G, bool bf16, bool rope) {
  return rope ? pick_rope<NST, true, TMA>(D, G, bf16) : pick_rope<NST, false, TMA>(D, G, bf16);
}

// Start of every call: the RoPE frequencies (computed on the host, exactly as
// dkv_create computes them, and passed by value), a cleared status word and
// cleared work counters.
__global__ void noalloc_init_kernel(const __grid_constant__ dkv::RopeFreqs fr, unsigned char* base, int D) {
  const int i = threadIdx.x;
  double* freq = reinterpret_cast<double*>(base + kFreqOffset);
  if (i < D / 2) freq[i] = fr.w[i];
  if (i == 0) *reinterpret_cast<int32_t*>(base + kStatusOffset) = 0;
  if (i < 4) reinterpret_cast<int32_t*>(base + kWorkOffset)[i] = 0;
}

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

int cuda_error(cudaError_t e, const char* what) {
  return dkv::set_error(DKV_ERR_CUDA, std::string(what) + ": " + cudaGetErrorString(e));
}

int setup_device(int dev, const SplitVariant& host_k, const SplitVariant& dev_k, int D, DeviceSetup** out) {
  DeviceSetup& st = g_setup[dev];
  std::lock_guard<std::mutex> lock(st.mu);
  if (!st.done) {
    void* ptr = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
    if (e != cudaSuccess) return cuda_error(e, "cudaGetSymbolAddress(no-alloc scratch)");
    e = cudaDeviceGetAttribute(&st.sm_count, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return cuda_error(e, "cudaDeviceGetAttribute");
    st.scratch = static_cast<unsigned char*>(ptr);
    st.done = true;
  }
  // per kernel variant: the dynamic shared-memory opt-in (idempotent)
  cudaError_t e = cudaFuncSetAttribute(host_k.fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(split_smem(D, kHostStages)));
  if (e != cudaSuccess) return cuda_error(e, "cudaFuncSetAttribute");
  e = cudaFuncSetAttribute(dev_k.fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(split_smem(D, kDevStages)));
  if (e != cudaSuccess) return cuda_error(e, "cudaFuncSetAttribute");
  *out = &st;
  return DKV_OK;
}

// Memory of `dev` that its kernels can use as a device pool (as dkv_attn_decode accepts it).
bool device_pool_ok(const void* p, int dev) {
  cudaPointerAttributes a{};
  if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  return (a.type == cudaMemoryTypeDevice || a.type == cudaMemoryTypeManaged) && a.device == dev;
}

bool host_pool_ok(const void* p) {
  cudaPointerAttributes a{};
  if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  return a.type == cudaMemoryTypeHost && a.devicePointer == p;
}

}  // namespace

extern "C" DKV_API int dkv_attn_decode_noalloc(const dkv_config* cfg, const float* q, const void* k_host,
                                               const void* v_host, const void* k_dev, const void* v_dev,
                                               const int32_t* block_table, const int32_t* seq_lens,
                                               int32_t host_split, float* out, int32_t* status_out,
                                               dkv_stream_t stream, int32_t batch, int32_t block_table_stride,
                                               int32_t num_dev_blocks) {
  using dkv::set_error;
  if (!cfg) return set_error(DKV_ERR_INVALID_ARG, "dkv_attn_decode_noalloc: null config");
  const dkv_config& c = *cfg;
  if (c.num_q_heads < 1 || c.num_kv_heads < 1 || c.num_kv_heads > 4096 || c.num_q_heads % c.num_kv_heads != 0 ||
      c.block_size < 16 || c.block_size > 1024 || c.block_size % 16 != 0 ||
      (c.kv_dtype != DKV_KV_F16 && c.kv_dtype != DKV_KV_BF16) || !(c.rope_base >= 0.0) || !(c.rope_base < 1e300) ||
      (c.rope_base > 0.0 && c.rope_base <= 1.0) || !(c.scale >= 0.0) || !(c.scale < 1e300) ||
      c.max_blocks_per_seq < 1 || static_cast<long long>(c.max_blocks_per_seq) * c.block_size > (1LL << 30) ||
      c.host_ctas < 0 || c.device < 0 || c.device >= kMaxDevices)
    return set_error(DKV_ERR_INVALID_ARG, "dkv_attn_decode_noalloc: config field out of range");
  const int G = c.num_q_heads / c.num_kv_heads;
  if ((c.head_dim != 64 && c.head_dim != 128) || (G != 1 && G != 2 && G != 4))
    return set_error(DKV_ERR_UNSUPPORTED, "dkv_attn_decode_noalloc: head_dim must be 64/128 and G 1/2/4");
  if (batch < 0) return set_error(DKV_ERR_INVALID_ARG, "dkv_attn_decode_noalloc: negative batch");
  if (batch == 0) return DKV_OK;
  if (!q || !out || !block_table || !seq_lens || block_table_stride < 1 || host_split < 0 || num_dev_blocks < 0 ||
      static_cast<long long>(host_split) + num_dev_blocks > 0x7fffffffLL || (host_split > 0 && (!k_host || !v_host)) ||
      (num_dev_blocks > 0 && (!k_dev || !v_dev)))
    return set_error(DKV_ERR_INVALID_ARG, "dkv_attn_decode_noalloc: null pointer or size out of range");
  if (reinterpret_cast<uintptr_t>(q) % 8 != 0 ||
      (host_split > 0 && (reinterpret_cast<uintptr_t>(k_host) | reinterpret_cast<uintptr_t>(v_host)) % 16 != 0) ||
      (num_dev_blocks > 0 && (reinterpret_cast<uintptr_t>(k_dev) | reinterpret_cast<uintptr_t>(v_dev)) % 16 != 0))
    return set_error(DKV_ERR_INVALID_ARG, "dkv_attn_decode_noalloc: q must be 8-byte and pools 16-byte aligned");
  const int D = c.head_dim;
  const bool run_host = host_split > 0;
  const bool run_dev = num_dev_blocks > 0 || !run_host;
  const bool use_lists = run_host && run_dev;
  const int nblk = block_table_stride < c.max_blocks_per_seq ? block_table_stride : c.max_blocks_per_seq;
  // the split partials (and, with both pools, the per-pool block lists) must fit in the fixed array
  const long max_slots = dkv::noalloc_max_slots(DKV_NOALLOC_SCRATCH_BYTES, batch, use_lists ? nblk : 0,
                                                c.num_q_heads, D);
  const long launches_split = (run_host ? 1 : 0) + (run_dev ? 1 : 0);
  if (max_slots < launches_split)
    return set_error(DKV_ERR_INVALID_ARG,
                     "dkv_attn_decode_noalloc: batch * num_q_heads (and, with both pools, batch * table blocks) "
                     "is too large for the fixed scratch of DKV_NOALLOC_SCRATCH_BYTES bytes");

  int prev = -1;
  cudaError_t e = cudaGetDevice(&prev);
  if (e != cudaSuccess) return cuda_error(e, "cudaGetDevice");
  if (prev != c.device && (e = cudaSetDevice(c.device)) != cudaSuccess) return cuda_error(e, "cudaSetDevice");
  struct Restore {
    int prev, dev;
    ~Restore() {
      if (prev != dev) cudaSetDevice(prev);
    }
  } restore{prev, c.device};

  const bool bf16 = c.kv_dtype == DKV_KV_BF16;
  const SplitVariant host_k = pick<kHostStages, false>(D, G, bf16, c.rope_base > 0.0);
  const SplitVariant dev_k = pick<kDevStages, kDevTma>(D, G, bf16, c.rope_base > 0.0);
  DeviceSetup* st = nullptr;
  int rc = setup_device(c.device, host_k, dev_k, D, &st);
  if (rc != DKV_OK) return rc;
  if (run_host && (!host_pool_ok(k_host) || !host_pool_ok(v_host)))
    return set_error(DKV_ERR_INVALID_ARG, "dkv_attn_decode_noalloc: host pools must be mapped pinned memory");
  if (num_dev_blocks > 0 && (!device_pool_ok(k_dev, c.device) || !device_pool_ok(v_dev, c.device)))
    return set_error(DKV_ERR_INVALID_ARG, "dkv_attn_decode_noalloc: device pools must be memory of cfg->device");
  // tensor maps of the device pool for the HBM kernel's tile copies (host-side encoding, no allocation)
  dkv::TileMaps maps{};
  if (kDevTma && num_dev_blocks > 0) {
    const long long rows = static_cast<long long>(num_dev_blocks) * c.num_kv_heads * c.block_size;
    if (rows >= (1LL << 31))
      return set_error(DKV_ERR_INVALID_ARG, "dkv_attn_decode_noalloc: a pool holds 2^31 or more token rows");
    if (!dkv::encode_pool_map(&maps.k, k_dev, rows, c.head_dim, true) ||
        !dkv::encode_pool_map(&maps.v, v_dev, rows, c.head_dim, false))
      return set_error(DKV_ERR_CUDA, "dkv_attn_decode_noalloc: cuTensorMapEncodeTiled rejected the pool's tensor map");
  }

  // split plan: as dkv_attn_decode plans it (the launches run one after the
  // other here, so the HBM launch has every SM), each side capped to its share
  // of the slots that fit in the scratch
  const int host_ctas = c.host_ctas > 0 ? c.host_ctas : kHostCtas;
  const long per = static_cast<long>(batch) * c.num_kv_heads;
  const long cap = max_slots / launches_split;
  const dkv::SplitPlan ph = dkv::plan_split(nblk, per, c.block_size, static_cast<long>(dkv::kWarps) * host_ctas, cap);
  const dkv::SplitPlan pd =
      dkv::plan_split(nblk, per, c.block_size, static_cast<long>(dkv::kWarps) * 2 * st->sm_count, cap);
  const int nsplit_h = run_host ? ph.nsplit : 0;
  const int nsplit_d = run_dev ? pd.nsplit : 0;
  const int nslots = nsplit_h + nsplit_d;
  const size_t rows = static_cast<size_t>(batch) * c.num_q_heads * nslots;
  const size_t list_bytes = use_lists ? static_cast<size_t>(batch) * nblk * 8 : 0;
  if (dkv::noalloc_scratch_bytes(batch, use_lists ? nblk : 0, rows, D) > DKV_NOALLOC_SCRATCH_BYTES)
    return set_error(DKV_ERR_INVALID_ARG, "dkv_attn_decode_noalloc: internal: plan exceeds the scratch");

  unsigned char* base = st->scratch;
  int32_t* status = reinterpret_cast<int32_t*>(base + kStatusOffset);
  int32_t* work = reinterpret_cast<int32_t*>(base + kWorkOffset);
  double* freq = reinterpret_cast<double*>(base + kFreqOffset);
  unsigned char* cur = base + dkv::kNoallocHeader;
  int2* counts = reinterpret_cast<int2*>(cur);
  cur += dkv::align256(static_cast<size_t>(batch) * 8);
  int2* lists = reinterpret_cast<int2*>(cur);
  cur += dkv::align256(list_bytes);
  float* part_lse = reinterpret_cast<float*>(cur);
  cur += dkv::align256(rows * 4);
  float* part_o = reinterpret_cast<float*>(cur);

  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  dkv::RopeFreqs fr{};
  dkv::rope_frequencies(c.rope_base, D, fr.w);
  noalloc_init_kernel<<<1, 64, 0, s>>>(fr, base, D);
  if ((e = cudaGetLastError()) != cudaSuccess) return cuda_error(e, "init kernel launch");

  const double scale = c.scale > 0.0 ? c.scale : 1.0 / sqrt(static_cast<double>(D));
  dkv::SplitParams sp{};
  sp.lists = use_lists ? lists : nullptr;
  sp.counts = counts;
  sp.list_stride = nblk;
  sp.q = q;
  sp.table = block_table;
  sp.seq_lens = seq_lens;
  sp.inv_freq = freq;
  sp.part_o = part_o;
  sp.part_lse = part_lse;
  sp.status = status;
  sp.hq = c.num_q_heads;
  sp.hkv = c.num_kv_heads;
  sp.block_size = c.block_size;
  sp.stride = block_table_stride;
  sp.nslots = nslots;
  sp.id_total = host_split + num_dev_blocks;
  sp.max_len = nblk * c.block_size;
  sp.rope = c.rope_base > 0.0 ? 1 : 0;
  sp.qscale = static_cast<float>(scale * 1.4426950408889634);
  sp.extra_tokens = 0;
  sp.num_queries = 1;
  const int min_bps = dkv::min_blocks_per_split(c.block_size);
  auto launch_params = [&](int nsplit, int bps, int slot_base, bool dev_list, int32_t* w) {
    dkv::SplitParams lp = sp;
    lp.nsplit = nsplit;
    lp.bps = use_lists ? min_bps : bps;
    lp.slot_base = slot_base;
    lp.list_dev = dev_list ? 1 : 0;
    lp.work = w;
    lp.n_units = batch * nsplit * c.num_kv_heads;
    dkv::set_divisors(lp);
    return lp;
  };
  auto ctas_for = [&](const dkv::SplitParams& lp, int limit) {
    const int u = (lp.n_units + dkv::kWarps - 1) / dkv::kWarps;
    return u < limit ? u : limit;
  };

  if (use_lists) {
    dkv::ListParams lp{};
    lp.table = block_table;
    lp.seq_lens = seq_lens;
    lp.lists = lists;
    lp.counts = counts;
    lp.stride = block_table_stride;
    lp.list_stride = nblk;
    lp.block_size = c.block_size;
    lp.host_split = host_split;
    lp.id_total = host_split + num_dev_blocks;
    lp.max_len = sp.max_len;
    lp.extra_tokens = 0;
    lp.invalid_to_dev = 1;
    dkv::lists_kernel<kListThreads><<<batch, kListThreads, 0, s>>>(lp);
    if ((e = cudaGetLastError()) != cudaSuccess) return cuda_error(e, "pool-lists kernel launch");
  }
  if (run_host) {
    dkv::SplitParams hp = launch_params(nsplit_h, ph.bps, 0, false, work);
    hp.k_pool = static_cast<const uint16_t*>(k_host);
    hp.v_pool = static_cast<const uint16_t*>(v_host);
    hp.id_lo = 0;
    hp.id_hi = host_split;
    host_k.launch(dim3(ctas_for(hp, host_ctas)), split_smem(D, kHostStages), s, hp, dkv::TileMaps{});
    if ((e = cudaGetLastError()) != cudaSuccess) return cuda_error(e, "host kernel launch");
  }
  if (run_dev) {
    dkv::SplitParams dp = launch_params(nsplit_d, pd.bps, nsplit_h, true, work + 2);
    dp.k_pool = static_cast<const uint16_t*>(k_dev);
    dp.v_pool = static_cast<const uint16_t*>(v_dev);
    dp.id_lo = host_split;
    dp.id_hi = host_split + num_dev_blocks;
    dev_k.launch(dim3(ctas_for(dp, 2 * st->sm_count)), split_smem(D, kDevStages), s, dp, maps);
    if ((e = cudaGetLastError()) != cudaSuccess) return cuda_error(e, "HBM kernel launch");
  }
  dkv::MergeParams mp{};
  mp.part_o = part_o;
  mp.part_lse = part_lse;
  mp.out = out;
  mp.nslots = nslots;
  mp.nsplit = nsplit_h;
  mp.has_host = run_host;
  mp.has_dev = run_dev;
  const int merge_rows = batch * c.num_q_heads;
  e = D == 64 ? launch_merge<64>(merge_rows, s, mp, run_dev) : launch_merge<128>(merge_rows, s, mp, run_dev);
  if (e != cudaSuccess) return cuda_error(e, "merge kernel launch");
  if (status_out &&
      (e = cudaMemcpyAsync(status_out, status, sizeof(int32_t), cudaMemcpyDeviceToDevice, s)) != cudaSuccess)
    return cuda_error(e, "cudaMemcpyAsync(status)");
  return DKV_OK;
}
