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
// CUDA cores.  A CTA owns 8 consecutive output rows (16 with 16 sequences per
// pass), dims of one head, so each sequence's results leave as 16-byte stores
// -- over PCIe when the block is host-resident.  Its 8 warps split the hidden
// dimension: in each warp, 4 lanes share a row and read a 64-byte run of it
// (16 bytes each), 8 rows side by side; every weight byte is read once for up
// to 16 sequences, whose hidden states the CTA stages in shared memory.  Lane
// partials are combined by shuffles, the warps' through shared memory.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace dkv {

constexpr int kAppendRows = 8;                 // row slots of a CTA (lane / 4); a lane covers 1 or 2 rows
constexpr int kAppendWarps = 8;                // warps per CTA, each over part of the hidden dimension
constexpr int kAppendBatch = 16;               // sequences per pass over the weights

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

// Columns a CTA's lanes cover in one step (8 warps x 4 lanes x 8 columns).
constexpr int kAppendStep = kAppendWarps * 4 * 8;

// Steps per stage of x in shared memory for NB sequences per pass: the more
// sequences, the more work per weight byte hides the loads' latency, so the
// fewer weight loads need to be in flight per lane (one stage's worth).
__host__ __device__ constexpr int append_group(int nb) { return nb <= 2 ? 16 : (nb <= 4 ? 8 : 4); }

// Rows per lane: with 16 sequences per pass a lane takes two rows (16 per
// CTA), so x is staged once for twice the weight bytes.
__host__ __device__ constexpr int append_rows_per_lane(int nb) { return nb >= 16 ? 2 : 1; }

// Output rows per CTA (8 or 16 dims of one head; head_dim is 64 or 128).
__host__ __device__ constexpr int append_cta_rows(int nb) { return kAppendRows * append_rows_per_lane(nb); }

// Dynamic shared memory of append_kernel<*, NB>: x of NB sequences over one
// stage of columns.
__host__ __device__ constexpr size_t append_smem_bytes(int nb) {
  return static_cast<size_t>(nb) * kAppendStep * append_group(nb) * sizeof(float);
}

// grid.x = 2*Hkv*D / append_cta_rows(NB); block = kAppendWarps warps.  NB:
// sequences per pass over the weights (1, 2, 4, 8 or 16, the smallest that
// covers the batch up to 16), so that a small batch issues no work for absent
// sequences.  The hidden dimension is walked in stages of kGroup steps: each
// lane first issues its weight loads of the stage, then the CTA stages x of
// those columns in shared memory (every lane of a row reads it there, not
// from L2), so the two latencies overlap.
template <bool BF16, int NB>
__global__ void __launch_bounds__(kAppendWarps * 32, 2) append_kernel(const AppendParams p) {
  static_assert(NB >= 1 && NB <= kAppendBatch, "1..16 sequences per pass");
  constexpr int RL = append_rows_per_lane(NB);     // rows per lane: r and r + 8
  constexpr int kRows = kAppendRows * RL;          // output rows of this CTA
  constexpr int kGroup = append_group(NB);         // steps per stage
  constexpr int kCols = kAppendStep * kGroup;      // columns per stage
  extern __shared__ __align__(16) float s_x[];     // [NB][kCols]
  __shared__ float s_part[kAppendWarps][NB][kRows];
  __shared__ __align__(16) uint16_t s_out[NB][kRows];
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int r = lane >> 2;                          // first row of this lane among the CTA's
  const int q = lane & 3;                           // its 16-byte column in the row's 64-byte run
  const int rows_kv = p.hkv * p.head_dim;
  const int row0 = blockIdx.x * kRows;              // first output row of this CTA
  const bool is_v = row0 >= rows_kv;
  const int r_local = row0 - (is_v ? rows_kv : 0);  // row inside W_k or W_v
  const int h = r_local / p.head_dim;
  const int d0 = r_local % p.head_dim;              // multiple of kRows
  const uint16_t* wbase = (is_v ? p.w_v : p.w_k) + static_cast<size_t>(r_local + r) * p.hidden;
  const int col = (warp * 4 + q) * 8;               // this lane's 8 columns inside a step
  auto load_w = [&](int j, int c) {                 // row r + 8j, columns c .. c+7
    return c < p.hidden ? *reinterpret_cast<const uint4*>(wbase + static_cast<size_t>(8 * j) * p.hidden + c)
                        : make_uint4(0u, 0u, 0u, 0u);
  };

  for (int b0 = 0; b0 < p.batch; b0 += NB) {
    const int nb = min(NB, p.batch - b0);
    // destination (dims d0 ..) of sequence b0 + threadIdx.x (threads < nb),
    // looked up while the projection runs: its position, the table entry, the pool
    uint16_t* dst = nullptr;
    if (threadIdx.x < nb) {
      const int b = b0 + threadIdx.x;
      const int L = p.seq_lens[b];  // position of the new token
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
        if (pool) dst = pool + ((blk * p.hkv + h) * p.block_size + (L % p.block_size)) * p.head_dim + d0;
      }
    }
    float acc[RL][NB];
#pragma unroll
    for (int j = 0; j < RL; ++j)
#pragma unroll
      for (int i = 0; i < NB; ++i) acc[j][i] = 0.f;
    for (int g0 = 0; g0 < p.hidden; g0 += kCols) {
      // this lane's weights of the stage, in flight while x is staged
      uint4 raw[RL][kGroup];
#pragma unroll
      for (int u = 0; u < kGroup; ++u)
#pragma unroll
        for (int j = 0; j < RL; ++j) raw[j][u] = load_w(j, g0 + col + u * kAppendStep);
      // x of this stage (zeros for absent sequences and past the hidden size)
      for (int e = threadIdx.x * 4; e < NB * kCols; e += kAppendWarps * 32 * 4) {
        const int i = e / kCols, cc = e % kCols;
        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
        if (i < nb && g0 + cc < p.hidden)
          v = __ldg(reinterpret_cast<const float4*>(p.x + static_cast<size_t>(b0 + i) * p.hidden + g0 + cc));
        *reinterpret_cast<float4*>(s_x + e) = v;
      }
      __syncthreads();
#pragma unroll
      for (int u = 0; u < kGroup; ++u) {
        float w[RL][8];
#pragma unroll
        for (int j = 0; j < RL; ++j) widen8<BF16>(raw[j][u], w[j]);   // zeros past the hidden size
        const int cs = col + u * kAppendStep;   // column inside the stage
#pragma unroll
        for (int i = 0; i < NB; ++i) {
          const float4 x0 = *reinterpret_cast<const float4*>(s_x + i * kCols + cs);
          const float4 x1 = *reinterpret_cast<const float4*>(s_x + i * kCols + cs + 4);
#pragma unroll
          for (int j = 0; j < RL; ++j) {
            float a = acc[j][i];
            a = fmaf(w[j][0], x0.x, a);
            a = fmaf(w[j][1], x0.y, a);
            a = fmaf(w[j][2], x0.z, a);
            a = fmaf(w[j][3], x0.w, a);
            a = fmaf(w[j][4], x1.x, a);
            a = fmaf(w[j][5], x1.y, a);
            a = fmaf(w[j][6], x1.z, a);
            a = fmaf(w[j][7], x1.w, a);
            acc[j][i] = a;
          }
        }
      }
      __syncthreads();   // before the next stage overwrites s_x
    }
    // the 4 lanes of a row, then the warps
#pragma unroll
    for (int j = 0; j < RL; ++j) {
#pragma unroll
      for (int i = 0; i < NB; ++i) {
        float a = acc[j][i];
        a += __shfl_xor_sync(0xffffffffu, a, 1);
        a += __shfl_xor_sync(0xffffffffu, a, 2);
        if (q == 0) s_part[warp][i][r + 8 * j] = a;
      }
    }
    __syncthreads();
    for (int t = threadIdx.x; t < NB * kRows; t += kAppendWarps * 32) {
      const int i = t / kRows, rr = t % kRows;
      if (i < nb) {
        float a = 0.f;
#pragma unroll
        for (int w = 0; w < kAppendWarps; ++w) a += s_part[w][i][rr];
        s_out[i][rr] = round16<BF16>(a);
      }
    }
    __syncthreads();
    if (dst) {
#pragma unroll
      for (int j = 0; j < RL; ++j)
        *reinterpret_cast<uint4*>(dst + 8 * j) = *reinterpret_cast<const uint4*>(&s_out[threadIdx.x][8 * j]);
    }
    __syncthreads();
  }
}

}  // namespace dkv
