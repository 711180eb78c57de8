// dkv_append.cuh -- write side of the cache: the K/V projection of the new
// token of every sequence and its store into the paged pools (DirectKV README,
// opening summary: the fused kernel includes the K/V projection; Step 6 checks
// K and V of new tokens).
//
// y[b][r] = sum_h W[r][h] x[b][h] for the 2*Hkv*D output rows r (K rows, then
// V rows), accumulated in fp32, rounded to the 16-bit storage type (nearest,
// ties to even) and stored un-rotated at row seq_lens[b] % S of the block that
// holds position seq_lens[b], in the host or the device pool.
//
// The product is bound by the weight bytes (batch is small), so it runs on the
// CUDA cores: one warp per output row reads the weight row once with 16-byte
// loads and applies it to every sequence; a CTA covers 8 consecutive rows
// (8 dims of one head), so each sequence's 8 results leave as one 16-byte
// store -- over PCIe when the block is host-resident.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace dkv {

constexpr int kAppendRows = 8;                 // output rows per CTA (one warp each)
constexpr int kAppendBatch = 8;                // sequences per pass over a weight row

struct AppendParams {
  const float* x;           // [B][H]
  const uint16_t* w_k;      // [Hkv*D][H]
  const uint16_t* w_v;      // [Hkv*D][H]
  const int32_t* table;     // [B][stride]
  const int32_t* seq_lens;  // [B]
  uint16_t* k_host;
  uint16_t* v_host;
  uint16_t* k_dev;
  uint16_t* v_dev;
  int32_t* status;
  int32_t batch, hidden, hkv, head_dim, block_size, stride, host_split, num_dev_blocks, max_len;
};

template <bool BF16>
__device__ __forceinline__ uint16_t round16(float v) {
  if constexpr (BF16) {
    const __nv_bfloat16 h = __float2bfloat16_rn(v);
    return *reinterpret_cast<const uint16_t*>(&h);
  } else {
    const __half h = __float2half_rn(v);
    return *reinterpret_cast<const uint16_t*>(&h);
  }
}

template <bool BF16>
__device__ __forceinline__ void widen8(const uint4& u, float (&w)[8]) {
  const uint32_t a[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    if constexpr (BF16) {
      w[2 * i] = __uint_as_float(a[i] << 16);
      w[2 * i + 1] = __uint_as_float(a[i] & 0xffff0000u);
    } else {
      const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&a[i]));
      w[2 * i] = f.x;
      w[2 * i + 1] = f.y;
    }
  }
}

// grid.x = 2*Hkv*D / 8 ; block = 8 warps
template <bool BF16>
__global__ void __launch_bounds__(kAppendRows * 32) append_kernel(const AppendParams p) {
  __shared__ __align__(16) uint16_t s_out[kAppendBatch][kAppendRows];
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int rows_kv = p.hkv * p.head_dim;
  const int row0 = blockIdx.x * kAppendRows;        // first output row of this CTA
  const bool is_v = row0 >= rows_kv;
  const int r_local = row0 - (is_v ? rows_kv : 0);  // row inside W_k or W_v
  const int h = r_local / p.head_dim;
  const int d0 = r_local % p.head_dim;              // multiple of 8
  const uint16_t* wrow = (is_v ? p.w_v : p.w_k) + static_cast<size_t>(r_local + warp) * p.hidden;

  for (int b0 = 0; b0 < p.batch; b0 += kAppendBatch) {
    const int nb = min(kAppendBatch, p.batch - b0);
    float acc[kAppendBatch];
#pragma unroll
    for (int i = 0; i < kAppendBatch; ++i) acc[i] = 0.f;
    for (int c = lane * 8; c < p.hidden; c += 32 * 8) {
      float w[8];
      widen8<BF16>(*reinterpret_cast<const uint4*>(wrow + c), w);
#pragma unroll
      for (int i = 0; i < kAppendBatch; ++i) {
        if (i < nb) {
          const float* xr = p.x + static_cast<size_t>(b0 + i) * p.hidden + c;
          const float4 x0 = __ldg(reinterpret_cast<const float4*>(xr));
          const float4 x1 = __ldg(reinterpret_cast<const float4*>(xr + 4));
          float a = acc[i];
          a = fmaf(w[0], x0.x, a);
          a = fmaf(w[1], x0.y, a);
          a = fmaf(w[2], x0.z, a);
          a = fmaf(w[3], x0.w, a);
          a = fmaf(w[4], x1.x, a);
          a = fmaf(w[5], x1.y, a);
          a = fmaf(w[6], x1.z, a);
          a = fmaf(w[7], x1.w, a);
          acc[i] = a;
        }
      }
    }
#pragma unroll
    for (int i = 0; i < kAppendBatch; ++i) {
      float a = acc[i];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
      if (lane == 0 && i < nb) s_out[i][warp] = round16<BF16>(a);
    }
    __syncthreads();
    if (threadIdx.x < nb) {
      const int b = b0 + threadIdx.x;
      const int L = p.seq_lens[b];  // position of the new token
      uint16_t* dst = nullptr;
      if (L < 0 || L >= p.max_len) {
        atomicOr(p.status, 2);
      } else {
        const int id = p.table[static_cast<size_t>(b) * p.stride + L / p.block_size];
        size_t blk;
        uint16_t* pool = nullptr;
        if (id >= 0 && id < p.host_split) {
          blk = static_cast<size_t>(id);
          pool = is_v ? p.v_host : p.k_host;
        } else if (id >= p.host_split && id - p.host_split < p.num_dev_blocks) {
          blk = static_cast<size_t>(id - p.host_split);
          pool = is_v ? p.v_dev : p.k_dev;
        } else {
          atomicOr(p.status, 1);
        }
        if (pool)
          dst = pool + ((blk * p.hkv + h) * p.block_size + (L % p.block_size)) * p.head_dim + d0;
      }
      if (dst) *reinterpret_cast<uint4*>(dst) = *reinterpret_cast<const uint4*>(&s_out[threadIdx.x][0]);
    }
    __syncthreads();
  }
}

}  // namespace dkv
