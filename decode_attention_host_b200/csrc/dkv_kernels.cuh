// dkv_kernels.cuh -- sm_100a kernels of libdkv.
//
// 1. split_kernel: split-K decode attention over the KV blocks of ONE
//    residency (host-mapped pinned memory, or HBM).  Launched twice per step:
//    a small persistent grid that streams host-resident blocks zero-copy over
//    PCIe straight into shared memory (DirectKV README, opening summary and
//    Attribution: KV tokens loaded from CPU-pinned buffers into the attention
//    kernel with no GPU staging buffer; SplitKernel README, Overview: stream
//    offloaded data directly into shared memory instead of prefetching into
//    HBM), and a wide grid over the HBM-resident blocks.
// 2. merge_kernel: log-sum-exp combine of all split partials into the output
//    (the host/device partition of the KV cache in the SplitKernel README,
//    Key Features, leaves one partial per side and split).
//
// Work decomposition.  The logical blocks of sequence b are cut into
// `nsplit` splits of `bps` consecutive blocks.  A unit is (b, split c, kv
// head h); one warp owns a unit at a time and handles the G = Hq/Hkv query
// heads of that kv head.  A warp walks its units (u = warp id, then + total
// warps), keeps a private ring of NST shared-memory stages filled with
// 16-token K/V tiles by 16-byte cp.async copies (rows past the sequence end
// are zero-filled, no bytes read), and prefetches across unit boundaries so
// the copy stream never drains.  Blocks whose id belongs to the other pool
// are skipped; ids outside both pools poison the unit (NaN) and set a status
// bit -- there is no trap.
//
// Lane layout inside a warp.  8 lanes share one token: lane li (0..7) of
// token group tg (0..3) owns the NeoX pairs i in [li*PPL, li*PPL+PPL),
// i.e. dims i and i + D/2 (PPL = D/16).  The 16 tokens of a tile are split
// tg, tg+4, tg+8, tg+12 over the four token groups.  Scores are reduced over
// the 8 lanes of a token group with three xor-shuffles; each token group
// keeps its own online-softmax state (running max, sum, un-normalised
// output) over its tokens, and the four states are merged once per unit.
//
// RoPE.  theta_i(p) = p * base^(-2i/D).  The angle at the first token of a
// tile is formed in fp64 and reduced modulo 2*pi before the fp32 sin/cos, so
// positions up to 2^24 keep full accuracy; the three later tokens of the same
// lane follow by multiplying with exp(i*4*theta_i(1)) (exact-to-fp32 step,
// error growth < 1e-6 over a tile).  Scores carry scale*log2(e) so the
// softmax works with exp2.
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace dkv {

constexpr int kTileTokens = 16;
constexpr int kWarps = 4;
constexpr int kThreads = kWarps * 32;
constexpr uint32_t kFull = 0xffffffffu;
constexpr int kFlagPoison = 1 << 8;

struct SplitParams {
  const float* q;           // [B][Hq][D]
  const uint16_t* k_pool;   // [nblocks][Hkv][S][D] of this residency
  const uint16_t* v_pool;
  const int32_t* table;     // [B][stride]
  const int32_t* seq_lens;  // [B]
  const double* inv_freq;   // [D/2]
  float* part_o;            // [B][Hq][nslots][D]
  float* part_lse;          // [B][Hq][nslots], log2 domain
  int32_t* status;
  int32_t hq, hkv, block_size, stride, nsplit, bps, nslots, slot_base;
  int32_t id_lo, id_hi;     // ids in [id_lo, id_hi) live in this pool at (id - id_lo)
  int32_t id_total;         // ids in [0, id_total) are valid in some pool
  int32_t max_len;          // largest valid seq_len
  int32_t n_units;          // B * nsplit * Hkv
  int32_t rope;             // 0: no rotation
  float qscale;             // softmax scale * log2(e)
};

struct MergeParams {
  const float* part_o;
  const float* part_lse;
  float* out;               // [B][Hq][D]
  int32_t nslots, nsplit, has_host, has_dev;
};

// One tile of the copy stream.  unit < 0 marks the end of the stream.
struct TileDesc {
  int32_t unit;
  int32_t pidx;  // block index inside this pool
  int32_t p0;    // logical position of the tile's first token
  int32_t meta;  // valid tokens (0..16) | kFlagPoison | kv head << 16
};

// ----------------------------------------------------------------------------- small helpers

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// 16-byte async copy global -> shared; src_bytes == 0 writes zeros and reads nothing.
__device__ __forceinline__ void cp_async16(void* dst, const void* src, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(smem_u32(dst)), "l"(src), "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

// cos/sin of pos * w with the angle reduced modulo 2*pi in fp64 first.
__device__ __forceinline__ void rope_cs(int pos, double w, float& c, float& s) {
  const double th = static_cast<double>(pos) * w;
  const double n = rint(th * 0.15915494309189535);        // 1 / (2*pi)
  const double r = fma(-n, 6.283185307179586, th);        // |r| <= pi (+ rounding)
  __sincosf(static_cast<float>(r), &s, &c);
}

// Two consecutive 16-bit elements (one 32-bit word) widened to an fp32 pair.
template <bool BF16>
__device__ __forceinline__ float2 widen2(uint32_t w) {
  if constexpr (BF16) {
    return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
  } else {
    __half2 h = *reinterpret_cast<__half2*>(&w);
    return __half22float2(h);
  }
}

// NP2 = PPL/2 fp32 pairs from PPL consecutive 16-bit elements in shared memory.
template <int NP2, bool BF16>
__device__ __forceinline__ void load_pairs(const char* src, float2 (&x)[NP2]) {
  if constexpr (NP2 == 4) {
    const uint4 u = *reinterpret_cast<const uint4*>(src);
    x[0] = widen2<BF16>(u.x);
    x[1] = widen2<BF16>(u.y);
    x[2] = widen2<BF16>(u.z);
    x[3] = widen2<BF16>(u.w);
  } else {
    static_assert(NP2 == 2, "head_dim 64 or 128");
    const uint2 u = *reinterpret_cast<const uint2*>(src);
    x[0] = widen2<BF16>(u.x);
    x[1] = widen2<BF16>(u.y);
  }
}

__device__ __forceinline__ float2 f2(float a) { return make_float2(a, a); }

// ----------------------------------------------------------------------------- tile stream

// Enumerates, for one warp, the tiles of this residency over its units.  All
// lanes run it in lockstep with identical results; block-table reads are
// uniform (one broadcast load per block).
struct TileStream {
  int unit, unit_stride;
  int b, h, L, j, j_end, sub, pidx;
  bool started, emitted, bad_len;

  __device__ void begin_unit(const SplitParams& p) {
    h = unit % p.hkv;
    const int bc = unit / p.hkv;
    const int c = bc % p.nsplit;
    b = bc / p.nsplit;
    L = p.seq_lens[b];
    bad_len = (L < 0 || L > p.max_len);
    const int nblk = bad_len ? 0 : (L + p.block_size - 1) / p.block_size;
    j = c * p.bps;
    j_end = min(j + p.bps, nblk);
    sub = 0;
    emitted = false;
    started = true;
  }
  __device__ void next_unit() {
    unit += unit_stride;
    started = false;
  }

  __device__ TileDesc next(const SplitParams& p, int lane) {
    while (unit < p.n_units) {
      if (!started) begin_unit(p);
      if (bad_len) {
        if (lane == 0) atomicOr(p.status, 2);
        TileDesc d{unit, 0, 0, kFlagPoison | (h << 16)};
        next_unit();
        return d;
      }
      while (j < j_end) {
        if (sub == 0) {
          const int id = p.table[static_cast<size_t>(b) * p.stride + j];
          if (id >= p.id_lo && id < p.id_hi) {
            pidx = id - p.id_lo;
          } else if (id >= 0 && id < p.id_total) {
            ++j;  // lives in the other pool
            continue;
          } else {
            if (lane == 0) atomicOr(p.status, 1);
            ++j;
            emitted = true;
            return TileDesc{unit, 0, 0, kFlagPoison | (h << 16)};
          }
        }
        const int p0 = j * p.block_size + sub * kTileTokens;
        const int nvalid = min(kTileTokens, L - p0);
        TileDesc d{unit, pidx, p0, nvalid | (h << 16)};
        emitted = true;
        ++sub;
        if (sub * kTileTokens >= p.block_size || p0 + kTileTokens >= L) {
          sub = 0;
          ++j;
        }
        return d;
      }
      const bool was_emitted = emitted;
      const int u = unit;
      next_unit();
      if (!was_emitted) return TileDesc{u, 0, 0, h << 16};  // empty unit: still reported once
    }
    return TileDesc{-1, 0, 0, 0};
  }
};

// ----------------------------------------------------------------------------- split kernel

template <int D, int G, bool BF16, int NST>
__global__ void __launch_bounds__(kThreads) split_kernel(const SplitParams p) {
  constexpr int PPL = D / 16;                  // NeoX pairs per lane
  constexpr int NP2 = PPL / 2;                 // fp32 pairs per half-row per lane
  constexpr int ROW = D * 2;                   // bytes of one token row
  constexpr int TILE = kTileTokens * ROW;      // bytes of one K (or V) tile
  constexpr int CPR = ROW / 16;                // 16-byte chunks per row
  extern __shared__ __align__(128) char smem[];
  __shared__ TileDesc meta[kWarps][NST];
  __shared__ double s_freq[D / 2];             // base^(-2i/D)
  __shared__ float2 s_step[D / 2];             // exp(i * 4 * theta_i(1)): the 4-token step

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int tg = lane >> 3;
  const int li = lane & 7;
  char* ring = smem + static_cast<size_t>(warp) * NST * 2 * TILE;

  for (int i = threadIdx.x; i < D / 2; i += kThreads) {
    const double w = p.rope ? p.inv_freq[i] : 0.0;
    float c, sn;
    rope_cs(4, w, c, sn);
    s_freq[i] = w;
    s_step[i] = make_float2(c, sn);
  }
  __syncthreads();

  TileStream ts;
  ts.unit = blockIdx.x * kWarps + warp;
  ts.unit_stride = gridDim.x * kWarps;
  ts.started = false;

  auto issue = [&](const TileDesc& d, int slot) {
    const int nvalid = d.meta & 0xff;
    if (d.unit < 0 || (d.meta & kFlagPoison) || nvalid == 0) return;
    const int h = d.meta >> 16;
    const size_t row0 = (static_cast<size_t>(d.pidx) * p.hkv + h) * p.block_size + (d.p0 % p.block_size);
    const char* gk = reinterpret_cast<const char*>(p.k_pool + row0 * D);
    const char* gv = reinterpret_cast<const char*>(p.v_pool + row0 * D);
    char* sk = ring + static_cast<size_t>(slot) * 2 * TILE;
    char* sv = sk + TILE;
#pragma unroll
    for (int e = lane; e < kTileTokens * CPR; e += 32) {
      const int nb = (e / CPR) < nvalid ? 16 : 0;
      cp_async16(sk + e * 16, nb ? gk + e * 16 : gk, nb);
      cp_async16(sv + e * 16, nb ? gv + e * 16 : gv, nb);
    }
  };

  // per-unit state: rotated, pre-scaled queries and un-normalised outputs of
  // this lane's dims, as fp32 pairs (first half X, second half Y)
  float2 QX[G][NP2], QY[G][NP2];
  float2 AX[G][NP2], AY[G][NP2];
  float mrun[G], lrun[G];
  bool poisoned = false;
  int cur = -1;

  // cos/sin of pos * theta for this lane's pairs, as fp32 pairs
  auto seeds = [&](int pos, float2 (&C)[NP2], float2 (&S)[NP2]) {
#pragma unroll
    for (int j = 0; j < NP2; ++j) {
      float c0, s0, c1, s1;
      rope_cs(pos, s_freq[li * PPL + 2 * j], c0, s0);
      rope_cs(pos, s_freq[li * PPL + 2 * j + 1], c1, s1);
      C[j] = make_float2(c0, c1);
      S[j] = make_float2(s0, s1);
    }
  };

  auto init_unit = [&](int unit, int h) {
    const int b = (unit / p.hkv) / p.nsplit;
    const int L = p.seq_lens[b];
    float2 C[NP2], S[NP2];
    if (p.rope) {
      seeds(L, C, S);
    } else {
#pragma unroll
      for (int j = 0; j < NP2; ++j) {
        C[j] = f2(1.f);
        S[j] = f2(0.f);
      }
    }
    const float2 qs = f2(p.qscale);
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const float* qg = p.q + (static_cast<size_t>(b) * p.hq + h * G + g) * D;
#pragma unroll
      for (int j = 0; j < NP2; ++j) {
        const float2 x = *reinterpret_cast<const float2*>(qg + li * PPL + 2 * j);
        const float2 y = *reinterpret_cast<const float2*>(qg + D / 2 + li * PPL + 2 * j);
        // x' = x c - y s ; y' = y c + x s, then the softmax scale (with log2 e)
        const float2 xr = __ffma2_rn(make_float2(-y.x, -y.y), S[j], __fmul2_rn(x, C[j]));
        const float2 yr = __ffma2_rn(x, S[j], __fmul2_rn(y, C[j]));
        QX[g][j] = __fmul2_rn(xr, qs);
        QY[g][j] = __fmul2_rn(yr, qs);
        AX[g][j] = f2(0.f);
        AY[g][j] = f2(0.f);
      }
      mrun[g] = -1e30f;
      lrun[g] = 0.f;
    }
    poisoned = false;
  };

  auto finalize = [&](int unit, int h) {
    const int bc = unit / p.hkv;
    const int c = bc % p.nsplit;
    const int b = bc / p.nsplit;
#pragma unroll
    for (int g = 0; g < G; ++g) {
      float M = fmaxf(mrun[g], __shfl_xor_sync(kFull, mrun[g], 8));
      M = fmaxf(M, __shfl_xor_sync(kFull, M, 16));
      const float f = exp2f(mrun[g] - M);
      float l = lrun[g] * f;
      l += __shfl_xor_sync(kFull, l, 8);
      l += __shfl_xor_sync(kFull, l, 16);
      const float2 ff = f2(f);
#pragma unroll
      for (int j = 0; j < NP2; ++j) {
        float2 a = __fmul2_rn(AX[g][j], ff);
        a.x += __shfl_xor_sync(kFull, a.x, 8);
        a.y += __shfl_xor_sync(kFull, a.y, 8);
        a.x += __shfl_xor_sync(kFull, a.x, 16);
        a.y += __shfl_xor_sync(kFull, a.y, 16);
        AX[g][j] = a;
        float2 y = __fmul2_rn(AY[g][j], ff);
        y.x += __shfl_xor_sync(kFull, y.x, 8);
        y.y += __shfl_xor_sync(kFull, y.y, 8);
        y.x += __shfl_xor_sync(kFull, y.x, 16);
        y.y += __shfl_xor_sync(kFull, y.y, 16);
        AY[g][j] = y;
      }
      if (tg == 0) {
        const size_t row = (static_cast<size_t>(b) * p.hq + h * G + g) * p.nslots + p.slot_base + c;
        float* o = p.part_o + row * D;
        const float qnan = __int_as_float(0x7fc00000);
        const float2 inv = f2(poisoned ? qnan : (l > 0.f ? 1.f / l : 0.f));
        float lse = l > 0.f ? M + __log2f(l) : -INFINITY;
        if (poisoned) lse = qnan;
#pragma unroll
        for (int j = 0; j < NP2; j += 2) {
          const float2 x0 = __fmul2_rn(AX[g][j], inv), x1 = __fmul2_rn(AX[g][j + 1], inv);
          const float2 y0 = __fmul2_rn(AY[g][j], inv), y1 = __fmul2_rn(AY[g][j + 1], inv);
          *reinterpret_cast<float4*>(o + li * PPL + 2 * j) = make_float4(x0.x, x0.y, x1.x, x1.y);
          *reinterpret_cast<float4*>(o + D / 2 + li * PPL + 2 * j) = make_float4(y0.x, y0.y, y1.x, y1.y);
        }
        if (li == 0) p.part_lse[row] = lse;
      }
    }
  };

  auto compute = [&](int slot, const TileDesc& d) {
    const char* sk = ring + static_cast<size_t>(slot) * 2 * TILE;
    const char* sv = sk + TILE;
    const int nvalid = d.meta & 0xff;
    float2 C[NP2], S[NP2], E[NP2], F[NP2];
    if (p.rope) {
      seeds(d.p0 + tg, C, S);
#pragma unroll
      for (int j = 0; j < NP2; ++j) {
        const float2 a = s_step[li * PPL + 2 * j], b = s_step[li * PPL + 2 * j + 1];
        E[j] = make_float2(a.x, b.x);
        F[j] = make_float2(a.y, b.y);
      }
    }
    float sc[4][G];
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      const char* row = sk + (tg + 4 * m) * ROW;
      float2 X[NP2], Y[NP2];
      load_pairs<NP2, BF16>(row + li * PPL * 2, X);
      load_pairs<NP2, BF16>(row + D + li * PPL * 2, Y);
      if (p.rope) {
#pragma unroll
        for (int j = 0; j < NP2; ++j) {
          const float2 x = X[j], y = Y[j];
          X[j] = __ffma2_rn(make_float2(-y.x, -y.y), S[j], __fmul2_rn(x, C[j]));
          Y[j] = __ffma2_rn(x, S[j], __fmul2_rn(y, C[j]));
          if (m < 3) {  // advance 4 positions: (C + iS)(E + iF)
            const float2 cn = __ffma2_rn(make_float2(-S[j].x, -S[j].y), F[j], __fmul2_rn(C[j], E[j]));
            S[j] = __ffma2_rn(C[j], F[j], __fmul2_rn(S[j], E[j]));
            C[j] = cn;
          }
        }
      }
#pragma unroll
      for (int g = 0; g < G; ++g) {
        float2 a = __fmul2_rn(QX[g][0], X[0]);
        a = __ffma2_rn(QY[g][0], Y[0], a);
#pragma unroll
        for (int j = 1; j < NP2; ++j) {
          a = __ffma2_rn(QX[g][j], X[j], a);
          a = __ffma2_rn(QY[g][j], Y[j], a);
        }
        sc[m][g] = a.x + a.y;
      }
    }
#pragma unroll
    for (int m = 0; m < 4; ++m)
#pragma unroll
      for (int g = 0; g < G; ++g) {
        float a = sc[m][g];
        a += __shfl_xor_sync(kFull, a, 1);
        a += __shfl_xor_sync(kFull, a, 2);
        a += __shfl_xor_sync(kFull, a, 4);
        sc[m][g] = (tg + 4 * m) < nvalid ? a : -INFINITY;
      }
    float pr[4][G];
#pragma unroll
    for (int g = 0; g < G; ++g) {
      float mx = fmaxf(fmaxf(sc[0][g], sc[1][g]), fmaxf(sc[2][g], sc[3][g]));
      mx = fmaxf(mx, mrun[g]);
      const float alpha = exp2f(mrun[g] - mx);
      float sum = 0.f;
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        pr[m][g] = exp2f(sc[m][g] - mx);
        sum += pr[m][g];
      }
      lrun[g] = lrun[g] * alpha + sum;
      mrun[g] = mx;
      if (alpha != 1.f) {
        const float2 al = f2(alpha);
#pragma unroll
        for (int j = 0; j < NP2; ++j) {
          AX[g][j] = __fmul2_rn(AX[g][j], al);
          AY[g][j] = __fmul2_rn(AY[g][j], al);
        }
      }
    }
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      const char* row = sv + (tg + 4 * m) * ROW;
      float2 X[NP2], Y[NP2];
      load_pairs<NP2, BF16>(row + li * PPL * 2, X);
      load_pairs<NP2, BF16>(row + D + li * PPL * 2, Y);
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const float2 pp = f2(pr[m][g]);
#pragma unroll
        for (int j = 0; j < NP2; ++j) {
          AX[g][j] = __ffma2_rn(pp, X[j], AX[g][j]);
          AY[g][j] = __ffma2_rn(pp, Y[j], AY[g][j]);
        }
      }
    }
  };

  // prologue: NST-1 tiles in flight
#pragma unroll 1
  for (int s = 0; s < NST - 1; ++s) {
    const TileDesc d = ts.next(p, lane);
    if (lane == 0) meta[warp][s] = d;
    issue(d, s);
    cp_async_commit();
  }
  int cur_h = 0;
#pragma unroll 1
  for (int k = 0;; ++k) {
    {
      const int slot = (k + NST - 1) % NST;
      const TileDesc d = ts.next(p, lane);
      if (lane == 0) meta[warp][slot] = d;
      issue(d, slot);
      cp_async_commit();
    }
    cp_async_wait<NST - 1>();
    __syncwarp();
    const int slot = k % NST;
    const TileDesc d = meta[warp][slot];
    if (d.unit < 0) break;
    if (d.unit != cur) {
      if (cur >= 0) finalize(cur, cur_h);
      cur = d.unit;
      cur_h = d.meta >> 16;
      init_unit(cur, cur_h);
    }
    if (d.meta & kFlagPoison) poisoned = true;
    else if ((d.meta & 0xff) > 0) compute(slot, d);
    __syncwarp();
  }
  if (cur >= 0) finalize(cur, cur_h);
  cp_async_wait<0>();
}

// ----------------------------------------------------------------------------- merge kernel

// One CTA per (b, hq); blockDim = NG * D threads: NG slot groups x D dims.
template <int D, int NG>
__global__ void __launch_bounds__(NG * D) merge_kernel(const MergeParams p) {
  extern __shared__ float wts[];  // [nslots]
  __shared__ float red_m[NG * D / 32], red_z[NG * D / 32];
  __shared__ int red_nan[NG * D / 32];
  __shared__ float part[NG][D];
  const int row = blockIdx.x;
  const int tid = threadIdx.x;
  const float* lse = p.part_lse + static_cast<size_t>(row) * p.nslots;
  const float* o = p.part_o + static_cast<size_t>(row) * p.nslots * D;
  auto valid = [&](int i) { return i < p.nsplit ? p.has_host != 0 : p.has_dev != 0; };

  float mx = -INFINITY;
  int nan = 0;
  for (int i = tid; i < p.nslots; i += NG * D) {
    if (!valid(i)) continue;
    const float v = lse[i];
    nan |= isnan(v) ? 1 : 0;
    mx = fmaxf(mx, v);
  }
  for (int off = 16; off > 0; off >>= 1) {
    mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, off));
    nan |= __shfl_xor_sync(kFull, nan, off);
  }
  if ((tid & 31) == 0) { red_m[tid >> 5] = mx; red_nan[tid >> 5] = nan; }
  __syncthreads();
  mx = -INFINITY;
  nan = 0;
#pragma unroll
  for (int i = 0; i < NG * D / 32; ++i) { mx = fmaxf(mx, red_m[i]); nan |= red_nan[i]; }

  float* dst = p.out + static_cast<size_t>(row) * D;
  if (nan || mx == -INFINITY) {
    if (tid < D) dst[tid] = nan ? __int_as_float(0x7fc00000) : 0.f;
    return;
  }
  float z = 0.f;
  for (int i = tid; i < p.nslots; i += NG * D) {
    const float wi = valid(i) ? exp2f(lse[i] - mx) : 0.f;
    wts[i] = wi;
    z += wi;
  }
  for (int off = 16; off > 0; off >>= 1) z += __shfl_xor_sync(kFull, z, off);
  if ((tid & 31) == 0) red_z[tid >> 5] = z;
  __syncthreads();
  z = 0.f;
#pragma unroll
  for (int i = 0; i < NG * D / 32; ++i) z += red_z[i];

  const int d = tid % D;
  const int grp = tid / D;
  float acc = 0.f;
#pragma unroll 4
  for (int i = grp; i < p.nslots; i += NG) {
    const float wi = wts[i];
    if (wi != 0.f) acc = fmaf(wi, o[static_cast<size_t>(i) * D + d], acc);
  }
  part[grp][d] = acc;
  __syncthreads();
  if (tid < D) {
    float t = 0.f;
#pragma unroll
    for (int g = 0; g < NG; ++g) t += part[g][tid];
    dst[tid] = t / z;
  }
}

}  // namespace dkv
