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

namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[DKV_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
constexpr int kHostStages = 4;
#ifndef DKV_DEV_STAGES
#define DKV_DEV_STAGES 3
#endif
constexpr int kDevStages = DKV_DEV_STAGES;
constexpr int kHostCtas = 16;
constexpr int kMinSplitTokens = 64;
constexpr size_t kStatusOffset = 0;     // int32 status word
constexpr size_t kFreqOffset = 256;     // up to 64 fp64 RoPE frequencies
constexpr size_t kPartOffset = 1024;    // split partials (lse rows, then output rows)

// Per-device set-up: the device address of the scratch array and the
// kernels' shared-memory limits.  Done once per device, on the first call.
struct DeviceSetup {
  std::mutex mu;
  bool done = false;
  unsigned char* scratch = nullptr;
  int sm_count = 0;
};
DeviceSetup g_setup[kMaxDevices];

size_t split_smem(int D, int nst) { return static_cast<size_t>(dkv::kWarps) * nst * 2 * dkv::kTileTokens * D * 2; }

using SplitLaunch = void (*)(dim3, size_t, cudaStream_t, const dkv::SplitParams&);
struct SplitVariant {
  SplitLaunch launch;
  const void* fn;
};

template <int D, int G, bool BF16, int NST, bool ROPE>
void launch_split(dim3 grid, size_t smem, cudaStream_t s, const dkv::SplitParams& p) {
  dkv::split_kernel<D, G, BF16, NST, ROPE><<<grid, dkv::kThreads, smem, s>>>(p);
}

template <int NST, bool ROPE>
SplitVariant pick_rope(int D, int G, bool bf16) {
#define DKV_NA_CASE(DD, GG)                                                                                \
  if (D == DD && G == GG)                                                                                  \
    return bf16 ? SplitVariant{&launch_split<DD, GG, true, NST, ROPE>,                                     \
                               reinterpret_cast<const void*>(&dkv::split_kernel<DD, GG, true, NST, ROPE>)} \
                : SplitVariant{&launch_split<DD, GG, false, NST, ROPE>,                                    \
                               reinterpret_cast<const void*>(&dkv::split_kernel<DD, GG, false, NST, ROPE>)};
  DKV_NA_CASE(64, 1)
  DKV_NA_CASE(64, 2)
  DKV_NA_CASE(64, 4)
  DKV_NA_CASE(128, 1)
  DKV_NA_CASE(128, 2)
  DKV_NA_CASE(128, 4)
#undef DKV_NA_CASE
  return {nullptr, nullptr};
}

template <int NST>
SplitVariant pick(int D, int G, bool bf16, bool rope) {
  return rope ? pick_rope<NST, true>(D, G, bf16) : pick_rope<NST, false>(D, G, bf16);
}

// theta_i(p) = p * base^(-2i/D), written into the scratch array each call.
__global__ void noalloc_freq_kernel(double* freq, double base, int D) {
  const int i = threadIdx.x;
  if (i < D / 2) freq[i] = base > 0.0 ? pow(base, -2.0 * i / static_cast<double>(D)) : 0.0;
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

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// Bytes of scratch the partials of (rows, D) need, including the header.
size_t scratch_bytes(size_t rows, int D) { return kPartOffset + align256(rows * 4) + rows * D * 4; }

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
  if (c.num_q_heads < 1 || c.num_kv_heads < 1 || c.num_kv_heads > 4096 || c.num_q_heads % c.num_kv_heads != 0 || c.block_size < 16 ||
      c.block_size > 1024 || c.block_size % 16 != 0 || (c.kv_dtype != DKV_KV_F16 && c.kv_dtype != DKV_KV_BF16) ||
      !(c.rope_base >= 0.0) || !(c.rope_base < 1e300) || (c.rope_base > 0.0 && c.rope_base <= 1.0) ||
      !(c.scale >= 0.0) || !(c.scale < 1e300) || c.max_blocks_per_seq < 1 ||
      static_cast<long long>(c.max_blocks_per_seq) * c.block_size > (1LL << 30) || c.device < 0 ||
      c.device >= kMaxDevices)
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
  // even one split per side must fit in the fixed scratch array
  const size_t min_rows = static_cast<size_t>(batch) * c.num_q_heads * 2;
  if (scratch_bytes(min_rows, D) > DKV_NOALLOC_SCRATCH_BYTES)
    return set_error(DKV_ERR_INVALID_ARG,
                     "dkv_attn_decode_noalloc: batch * num_q_heads is too large for the fixed scratch of "
                     "DKV_NOALLOC_SCRATCH_BYTES bytes");

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
  const SplitVariant host_k = pick<kHostStages>(D, G, bf16, c.rope_base > 0.0);
  const SplitVariant dev_k = pick<kDevStages>(D, G, bf16, c.rope_base > 0.0);
  DeviceSetup* st = nullptr;
  int rc = setup_device(c.device, host_k, dev_k, D, &st);
  if (rc != DKV_OK) return rc;

  if (host_split > 0) {
    cudaPointerAttributes a{};
    if (cudaPointerGetAttributes(&a, k_host) != cudaSuccess || a.type != cudaMemoryTypeHost ||
        a.devicePointer != k_host || cudaPointerGetAttributes(&a, v_host) != cudaSuccess ||
        a.type != cudaMemoryTypeHost || a.devicePointer != v_host) {
      cudaGetLastError();
      return set_error(DKV_ERR_INVALID_ARG, "dkv_attn_decode_noalloc: host pools must be mapped pinned memory");
    }
  }
  if (num_dev_blocks > 0) {
    cudaPointerAttributes a{};
    if (cudaPointerGetAttributes(&a, k_dev) != cudaSuccess || a.type != cudaMemoryTypeDevice ||
        a.device != c.device || cudaPointerGetAttributes(&a, v_dev) != cudaSuccess ||
        a.type != cudaMemoryTypeDevice || a.device != c.device) {
      cudaGetLastError();
      return set_error(DKV_ERR_INVALID_ARG, "dkv_attn_decode_noalloc: device pools must be memory of cfg->device");
    }
  }

  // split plan: as in dkv_attn_decode, then narrowed until the partials fit the scratch
  const int nblk = block_table_stride < c.max_blocks_per_seq ? block_table_stride : c.max_blocks_per_seq;
  const long per = static_cast<long>(batch) * c.num_kv_heads;
  const long units_target = static_cast<long>(st->sm_count) * 8;
  int target = static_cast<int>((units_target + per - 1) / per);
  if (target < 1) target = 1;
  int bps = (nblk + target - 1) / target;
  const int min_bps = (kMinSplitTokens + c.block_size - 1) / c.block_size;
  if (bps < min_bps) bps = min_bps;
  int nsplit = (nblk + bps - 1) / bps;
  const size_t rows_per_split = static_cast<size_t>(batch) * c.num_q_heads * 2;
  while (nsplit > 1 && scratch_bytes(rows_per_split * nsplit, D) > DKV_NOALLOC_SCRATCH_BYTES) {
    ++bps;
    nsplit = (nblk + bps - 1) / bps;
  }
  const int nslots = 2 * nsplit;
  const size_t rows = static_cast<size_t>(batch) * c.num_q_heads * nslots;

  unsigned char* base = st->scratch;
  int32_t* status = reinterpret_cast<int32_t*>(base + kStatusOffset);
  double* freq = reinterpret_cast<double*>(base + kFreqOffset);
  float* part_lse = reinterpret_cast<float*>(base + kPartOffset);
  float* part_o = reinterpret_cast<float*>(base + kPartOffset + align256(rows * 4));

  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if ((e = cudaMemsetAsync(status, 0, sizeof(int32_t), s)) != cudaSuccess) return cuda_error(e, "cudaMemsetAsync");
  noalloc_freq_kernel<<<1, 64, 0, s>>>(freq, c.rope_base, D);
  if ((e = cudaGetLastError()) != cudaSuccess) return cuda_error(e, "freq kernel launch");

  const double scale = c.scale > 0.0 ? c.scale : 1.0 / sqrt(static_cast<double>(D));
  dkv::SplitParams sp{};
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
  sp.nsplit = nsplit;
  sp.bps = bps;
  sp.nslots = nslots;
  sp.id_total = host_split + num_dev_blocks;
  sp.max_len = nblk * c.block_size;
  sp.n_units = batch * nsplit * c.num_kv_heads;
  sp.rope = c.rope_base > 0.0 ? 1 : 0;
  sp.qscale = static_cast<float>(scale * 1.4426950408889634);
  sp.extra_tokens = 0;
  sp.num_queries = 1;
  dkv::set_divisors(sp);
  const int unit_ctas = (sp.n_units + dkv::kWarps - 1) / dkv::kWarps;

  if (host_split > 0) {
    dkv::SplitParams hp = sp;
    hp.k_pool = static_cast<const uint16_t*>(k_host);
    hp.v_pool = static_cast<const uint16_t*>(v_host);
    hp.id_lo = 0;
    hp.id_hi = host_split;
    hp.slot_base = 0;
    const int host_ctas = c.host_ctas > 0 ? c.host_ctas : kHostCtas;
    host_k.launch(dim3(unit_ctas < host_ctas ? unit_ctas : host_ctas), split_smem(D, kHostStages), s, hp);
    if ((e = cudaGetLastError()) != cudaSuccess) return cuda_error(e, "host kernel launch");
  }
  if (num_dev_blocks > 0) {
    dkv::SplitParams dp = sp;
    dp.k_pool = static_cast<const uint16_t*>(k_dev);
    dp.v_pool = static_cast<const uint16_t*>(v_dev);
    dp.id_lo = host_split;
    dp.id_hi = host_split + num_dev_blocks;
    dp.slot_base = nsplit;
    const int dev_ctas = unit_ctas < 2 * st->sm_count ? unit_ctas : 2 * st->sm_count;  // one resident wave
    dev_k.launch(dim3(dev_ctas), split_smem(D, kDevStages), s, dp);
    if ((e = cudaGetLastError()) != cudaSuccess) return cuda_error(e, "HBM kernel launch");
  }
  dkv::MergeParams mp{};
  mp.part_o = part_o;
  mp.part_lse = part_lse;
  mp.out = out;
  mp.nslots = nslots;
  mp.nsplit = nsplit;
  mp.has_host = host_split > 0;
  mp.has_dev = num_dev_blocks > 0;
  if (D == 64)
    dkv::merge_kernel<64, 16><<<batch * c.num_q_heads, 16 * 64, nslots * sizeof(float), s>>>(mp);
  else
    dkv::merge_kernel<128, 8><<<batch * c.num_q_heads, 8 * 128, nslots * sizeof(float), s>>>(mp);
  if ((e = cudaGetLastError()) != cudaSuccess) return cuda_error(e, "merge kernel launch");
  if (status_out &&
      (e = cudaMemcpyAsync(status_out, status, sizeof(int32_t), cudaMemcpyDeviceToDevice, s)) != cudaSuccess)
    return cuda_error(e, "cudaMemcpyAsync(status)");
  return DKV_OK;
}
