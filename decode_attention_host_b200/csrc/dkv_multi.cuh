// dkv_multi.cuh -- multi-token queries over the split cache (speculative
// verification, chunked prefill): Tq query tokens per sequence, query i at
// position L + i attending to the cached tokens t < L + i (the cache already
// holds the tokens L .. L + Tq - 2).  Tq = 1 is single-token decode.
//
// Per unit (sequence b, split c, kv head h) the Tq * G query rows (<= 16) share
// every K/V tile, so both contractions run on the tensor cores (mma.sync
// m16n8k16, rows r = i * G + g):
//   - a rotation pass applies NeoX RoPE to each 16-token K tile in shared
//     memory (the same lane layout and chained angle recurrence as the decode
//     kernel) and rewrites it as a 16-bit "hi" tile in place plus a "lo"
//     remainder tile, so rotated K keeps ~2^-16 relative precision;
//   - S = Q K^T with Q = q_hi + q_lo and K = k_hi + k_lo: three mmas per k-step
//     (q_hi k_hi + q_hi k_lo + q_lo k_hi);
//   - the C layout of S is the A layout of the PV product, so the causal mask
//     and the online softmax run in registers per row, and P = p_hi + p_lo
//     multiplies V (ldmatrix.trans) in two mmas per 8 output columns.
// Both K and V tiles are stored XOR-swizzled (16-byte chunk ^ row mod 8) so
// that every ldmatrix phase hits 8 distinct bank groups.
#pragma once

#include "dkv_kernels.cuh"

namespace dkv {

constexpr int kMultiMaxRows = 16;
#ifndef DKV_MULTI_STAGES
#define DKV_MULTI_STAGES 2
#endif
constexpr int kMultiStages = DKV_MULTI_STAGES;  // ring depth of the multi-token kernel (build-time knob)

// Dynamic shared memory of multi_kernel<D, *, *>: per warp the K and V tiles
// of every ring stage plus the lo tile of the rotated K.
__host__ __device__ constexpr size_t multi_smem_bytes(int D) {
  return static_cast<size_t>(kWarps) * (2 * kMultiStages + 1) * kTileTokens * D * 2;
}

template <int D, bool BF16, bool ROPE>
__global__ void __launch_bounds__(kThreads) multi_kernel(const SplitParams p) {
  constexpr int NST = kMultiStages;            // ring depth (NST - 1 tiles in flight)
  constexpr int PPL = D / 16;                  // NeoX pairs per lane in the rotation pass
  constexpr int NP2 = PPL / 2;
  constexpr int ROW = D * 2;
  constexpr int TILE = kTileTokens * ROW;
  constexpr int CPR = ROW / 16;
  constexpr int NT = D / 8;                    // 8-wide output column tiles
  constexpr int KS = D / 16;                   // k-steps of the QK product
  extern __shared__ __align__(128) char smem[];
  __shared__ TileDesc meta[kWarps][NST];
  __shared__ double s_freq[PPL][8];
  __shared__ float2 s_e[NP2][8], s_f[NP2][8];

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int tg = lane >> 3;
  const int li = lane & 7;
  const int gT = lane >> 2;                    // fragment row (and row + 8)
  const int cT = lane & 3;                     // fragment column pair
  char* ring = smem + static_cast<size_t>(warp) * (2 * NST + 1) * TILE;
  char* klo = ring + 2 * NST * TILE;           // lo part of the rotated K tile
  const int G = p.hq / p.hkv;
  const int R = p.num_queries * G;

  for (int i = threadIdx.x; i < D / 2; i += kThreads) {
    const double w = ROPE ? p.inv_freq[i] : 0.0;
    const int l = i / PPL, r = i % PPL;
    s_freq[r][l] = w;
    float c, sn;
    rope_cs(4, w, c, sn);
    reinterpret_cast<float*>(&s_e[r >> 1][l])[r & 1] = c;
    reinterpret_cast<float*>(&s_f[r >> 1][l])[r & 1] = sn;
  }
  __syncthreads();

  TileStream ts;
  ts.grab(p, lane);

  constexpr int KCOPIES = kTileTokens * CPR / 32;
  int vofs[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int e = lane + 32 * k;
    vofs[k] = swz<ROW>(e / CPR, e % CPR);
  }
  auto issue = [&](const TileDesc& d, int slot) {
    const int nvalid = d.meta & 0xff;
    if (d.unit < 0 || (d.meta & kFlagPoison) || nvalid == 0) return;
    const int h = d.meta >> 16;
    const size_t row0 = (static_cast<size_t>(d.pidx) * p.hkv + h) * p.block_size + ((d.meta >> kSubShift) & kSubMask) * kTileTokens;
    const char* gk = reinterpret_cast<const char*>(p.k_pool + row0 * D) + lane * 16;
    const char* gv = reinterpret_cast<const char*>(p.v_pool + row0 * D) + lane * 16;
    char* sk = ring + static_cast<size_t>(slot) * 2 * TILE;
    char* sv = sk + TILE;
#pragma unroll
    for (int k = 0; k < KCOPIES; ++k) {
      const int nb = (nvalid == kTileTokens || (lane + 32 * k) / CPR < nvalid) ? 16 : 0;
      const int o = vofs[k & 3] + (k >> 2) * 2048;
      cp_async16(sk + o, nb ? gk + 512 * k : gk - lane * 16, nb);
      cp_async16(sv + o, nb ? gv + 512 * k : gv - lane * 16, nb);
    }
  };

  // per-unit state: Q fragments (hi, lo), PV accumulators, softmax state of
  // this thread's two rows r0 = gT and r1 = gT + 8
  uint32_t qah[KS][4], qal[KS][4];
  float acc[NT][4];
  float m0 = -1e30f, m1 = -1e30f, l0 = 0.f, l1 = 0.f;
  int lim0 = 0, lim1 = 0;                      // rows see positions < lim
  bool poisoned = false;
  int cur = -1, cur_h = 0;
  float2 Cc[NP2], Sc[NP2];
  int next_pos = -1, chain = 0;

  auto freq_of = [&](int i) { return s_freq[i % PPL][i / PPL]; };

  auto init_unit = [&](int unit, int h) {
    const int b = p.div_nsplit.div(p.div_hkv.div(unit));
    const int L = p.seq_lens[b];
    const int rows[2] = {gT, gT + 8};
    uint32_t hi[2][KS][2], lo[2][KS][2];
#pragma unroll
    for (int rr = 0; rr < 2; ++rr) {
      const int r = rows[rr];
      const bool live = r < R;
      const int i = live ? r / G : 0;
      const int g = live ? r % G : 0;
      const float* qr = p.q + ((static_cast<size_t>(b) * p.num_queries + i) * p.hq + h * G + g) * D;
      const int pos = L + i;
#pragma unroll
      for (int s = 0; s < KS / 2; ++s) {
#pragma unroll
        for (int half = 0; half < 2; ++half) {   // dims 16s + 8*half + 2c + {0,1}
          const int d = 16 * s + 8 * half + 2 * cT;
          float2 x = live ? *reinterpret_cast<const float2*>(qr + d) : f2(0.f);
          float2 y = live ? *reinterpret_cast<const float2*>(qr + d + D / 2) : f2(0.f);
          if constexpr (ROPE) {
            float c0, s0, c1, s1;
            rope_cs(pos, freq_of(d), c0, s0);
            rope_cs(pos, freq_of(d + 1), c1, s1);
            const float2 C = make_float2(c0, c1), S = make_float2(s0, s1);
            const float2 xc = __fmul2_rn(x, C), ys = __fmul2_rn(y, S);
            const float2 yr = __ffma2_rn(x, S, __fmul2_rn(y, C));
            x = make_float2(xc.x - ys.x, xc.y - ys.y);
            y = yr;
          }
          const float2 qs = f2(p.qscale);
          x = __fmul2_rn(x, qs);
          y = __fmul2_rn(y, qs);
          split_hi_lo<BF16>(x, hi[rr][s][half], lo[rr][s][half]);
          split_hi_lo<BF16>(y, hi[rr][s + KS / 2][half], lo[rr][s + KS / 2][half]);
        }
      }
    }
#pragma unroll
    for (int s = 0; s < KS; ++s) {
      qah[s][0] = hi[0][s][0];
      qah[s][1] = hi[1][s][0];
      qah[s][2] = hi[0][s][1];
      qah[s][3] = hi[1][s][1];
      qal[s][0] = lo[0][s][0];
      qal[s][1] = lo[1][s][0];
      qal[s][2] = lo[0][s][1];
      qal[s][3] = lo[1][s][1];
    }
    lim0 = gT < R ? L + gT / G : -1;
    lim1 = gT + 8 < R ? L + (gT + 8) / G : -1;
#pragma unroll
    for (int n = 0; n < NT; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;
    m0 = m1 = -1e30f;
    l0 = l1 = 0.f;
    poisoned = false;
  };

  auto finalize = [&](int unit, int h) {
    const int bc = p.div_hkv.div(unit);
    const int b = p.div_nsplit.div(bc);
    const int c = bc - b * p.nsplit;
    float t0 = l0, t1 = l1;
    t0 += __shfl_xor_sync(kFull, t0, 1);
    t0 += __shfl_xor_sync(kFull, t0, 2);
    t1 += __shfl_xor_sync(kFull, t1, 1);
    t1 += __shfl_xor_sync(kFull, t1, 2);
    const float qnan = __int_as_float(0x7fc00000);
#pragma unroll
    for (int rr = 0; rr < 2; ++rr) {
      const int r = gT + 8 * rr;
      if (r >= R) continue;
      const int i = r / G, g = r % G;
      const float l = rr ? t1 : t0;
      const float M = rr ? m1 : m0;
      const size_t row = ((static_cast<size_t>(b) * p.num_queries + i) * p.hq + h * G + g) * p.nslots + p.slot_base + c;
      float* o = p.part_o + row * D;
      const float inv = poisoned ? qnan : (l > 0.f ? 1.f / l : 0.f);
#pragma unroll
      for (int n = 0; n < NT; ++n)
        *reinterpret_cast<float2*>(o + 8 * n + 2 * cT) = make_float2(acc[n][2 * rr] * inv, acc[n][2 * rr + 1] * inv);
      if (cT == 0) p.part_lse[row] = poisoned ? qnan : (l > 0.f ? M + __log2f(l) : -INFINITY);
    }
  };

  auto compute = [&](int slot, const TileDesc& d) {
    char* sk = ring + static_cast<size_t>(slot) * 2 * TILE;
    const char* sv = sk + TILE;
    const int nvalid = d.meta & 0xff;
    // ---- rotation pass: K tile -> rotated hi (in place) + lo (klo), same swizzled layout
    // the rotation state stays in registers while positions continue, with
    // a fresh fp64-reduced seed at least every 16 tiles (at most 64 fp32 steps)
    float2 (&C)[NP2] = Cc;
    float2 (&S)[NP2] = Sc;
    if constexpr (ROPE) {
      if (d.p0 == next_pos && chain < 16) {
        ++chain;
      } else {
#pragma unroll
        for (int j = 0; j < NP2; ++j) {
          float c0, s0, c1, s1;
          rope_cs(d.p0 + tg, s_freq[2 * j][li], c0, s0);
          rope_cs(d.p0 + tg, s_freq[2 * j + 1][li], c1, s1);
          C[j] = make_float2(c0, c1);
          S[j] = make_float2(s0, s1);
        }
        chain = 1;
      }
    }
    constexpr int XB = PPL * 2;                // bytes of this lane's run in each half-row
    const int bx = li * XB;
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      const int t = tg + 4 * m;
      const int ox = swz<ROW>(t, bx >> 4) + (bx & 15);
      const int oy = swz<ROW>(t, (D + bx) >> 4) + ((D + bx) & 15);
      float2 X[NP2], Y[NP2];
      load_pairs<NP2, BF16>(sk + ox, X);
      load_pairs<NP2, BF16>(sk + oy, Y);
      if constexpr (ROPE) {
#pragma unroll
        for (int j = 0; j < NP2; ++j) {
          const float2 x = X[j], y = Y[j];
          const float2 ns = __fmul2_rn(S[j], make_float2(-1.f, -1.f));
          X[j] = __ffma2_rn(y, ns, __fmul2_rn(x, C[j]));
          Y[j] = __ffma2_rn(x, S[j], __fmul2_rn(y, C[j]));
          const float2 e = s_e[j][li], f = s_f[j][li];
          const float2 cn = __ffma2_rn(ns, f, __fmul2_rn(C[j], e));
          S[j] = __ffma2_rn(C[j], f, __fmul2_rn(S[j], e));
          C[j] = cn;
        }
      }
      uint32_t xh[NP2], xl[NP2], yh[NP2], yl[NP2];
#pragma unroll
      for (int j = 0; j < NP2; ++j) {
        split_hi_lo<BF16>(X[j], xh[j], xl[j]);
        split_hi_lo<BF16>(Y[j], yh[j], yl[j]);
      }
      if constexpr (NP2 == 4) {
        *reinterpret_cast<uint4*>(sk + ox) = make_uint4(xh[0], xh[1], xh[2], xh[3]);
        *reinterpret_cast<uint4*>(sk + oy) = make_uint4(yh[0], yh[1], yh[2], yh[3]);
        *reinterpret_cast<uint4*>(klo + ox) = make_uint4(xl[0], xl[1], xl[2], xl[3]);
        *reinterpret_cast<uint4*>(klo + oy) = make_uint4(yl[0], yl[1], yl[2], yl[3]);
      } else {
        *reinterpret_cast<uint2*>(sk + ox) = make_uint2(xh[0], xh[1]);
        *reinterpret_cast<uint2*>(sk + oy) = make_uint2(yh[0], yh[1]);
        *reinterpret_cast<uint2*>(klo + ox) = make_uint2(xl[0], xl[1]);
        *reinterpret_cast<uint2*>(klo + oy) = make_uint2(yl[0], yl[1]);
      }
    }
    if constexpr (ROPE) next_pos = d.p0 + kTileTokens;
    __syncwarp();
    // ---- S = Q K^T on the tensor cores: tokens 0..7 (S0) and 8..15 (S1)
    float S0[4] = {0.f, 0.f, 0.f, 0.f}, S1[4] = {0.f, 0.f, 0.f, 0.f};
    const int krow = (lane & 7) + ((lane >> 4) << 3);
    const int kcol = (lane >> 3) & 1;
#pragma unroll
    for (int s = 0; s < KS; ++s) {
      const int off = swz<ROW>(krow, 2 * s + kcol);
      uint32_t h0, h1, h2, h3, w0, w1, w2, w3;
      ldsm_x4(sk + off, h0, h1, h2, h3);
      ldsm_x4(klo + off, w0, w1, w2, w3);
      mma16816_full<BF16>(S0, qah[s], h0, h1);
      mma16816_full<BF16>(S1, qah[s], h2, h3);
      mma16816_full<BF16>(S0, qah[s], w0, w1);
      mma16816_full<BF16>(S1, qah[s], w2, w3);
      mma16816_full<BF16>(S0, qal[s], h0, h1);
      mma16816_full<BF16>(S1, qal[s], h2, h3);
    }
    // ---- causal mask and online softmax for rows r0 = gT (S*[0..1]) and r1 = gT + 8 (S*[2..3])
    float v0[4] = {S0[0], S0[1], S1[0], S1[1]};
    float v1[4] = {S0[2], S0[3], S1[2], S1[3]};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int t = 2 * cT + (k & 1) + 8 * (k >> 1);
      const int pos = d.p0 + t;
      const bool in = t < nvalid;
      v0[k] = (in && pos < lim0) ? v0[k] : -INFINITY;
      v1[k] = (in && pos < lim1) ? v1[k] : -INFINITY;
    }
    // The row's reference max (shared by its 4 lanes) is raised only when a
    // score of the tile exceeds it by more than kLazyMax (log2 units); the
    // weights 2^(s - m) then stay below 2^kLazyMax and the sum and the output
    // keep the same reference, so the result is exact up to rounding.
    float tm0 = fmaxf(fmaxf(v0[0], v0[1]), fmaxf(v0[2], v0[3]));
    float tm1 = fmaxf(fmaxf(v1[0], v1[1]), fmaxf(v1[2], v1[3]));
    if (__any_sync(kFull, tm0 > m0 + kLazyMax || tm1 > m1 + kLazyMax)) {
      tm0 = fmaxf(tm0, __shfl_xor_sync(kFull, tm0, 1));
      tm0 = fmaxf(tm0, __shfl_xor_sync(kFull, tm0, 2));
      tm1 = fmaxf(tm1, __shfl_xor_sync(kFull, tm1, 1));
      tm1 = fmaxf(tm1, __shfl_xor_sync(kFull, tm1, 2));
      const float mx0 = fmaxf(m0, tm0), mx1 = fmaxf(m1, tm1);
      const float al0 = ex2(m0 - mx0), al1 = ex2(m1 - mx1);
      l0 *= al0;
      l1 *= al1;
      m0 = mx0;
      m1 = mx1;
#pragma unroll
      for (int n = 0; n < NT; ++n) {
        acc[n][0] *= al0;
        acc[n][1] *= al0;
        acc[n][2] *= al1;
        acc[n][3] *= al1;
      }
    }
    float p0[4], p1[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      p0[k] = ex2(v0[k] - m0);
      p1[k] = ex2(v1[k] - m1);
    }
    l0 += (p0[0] + p0[1]) + (p0[2] + p0[3]);
    l1 += (p1[0] + p1[1]) + (p1[2] + p1[3]);
    // A fragments of P: {r0 tokens 2c.., r1 tokens 2c.., r0 tokens 8+2c.., r1 tokens 8+2c..}
    uint32_t ph[4], pl[4];
    split_hi_lo<BF16>(make_float2(p0[0], p0[1]), ph[0], pl[0]);
    split_hi_lo<BF16>(make_float2(p1[0], p1[1]), ph[1], pl[1]);
    split_hi_lo<BF16>(make_float2(p0[2], p0[3]), ph[2], pl[2]);
    split_hi_lo<BF16>(make_float2(p1[2], p1[3]), ph[3], pl[3]);
    // ---- O += P V on the tensor cores
    const int vrow = (lane & 7) | (lane & 8);
#pragma unroll
    for (int qd = 0; qd < D / 16; ++qd) {
      uint32_t b0, b1, b2, b3;
      ldsm_x4_t(sv + swz<ROW>(vrow, 2 * qd + (lane >> 4)), b0, b1, b2, b3);
      mma16816_full<BF16>(acc[2 * qd], ph, b0, b1);
      mma16816_full<BF16>(acc[2 * qd + 1], ph, b2, b3);
      mma16816_full<BF16>(acc[2 * qd], pl, b0, b1);
      mma16816_full<BF16>(acc[2 * qd + 1], pl, b2, b3);
    }
  };

#pragma unroll 1
  for (int s = 0; s < NST - 1; ++s) {
    const TileDesc d = ts.next(p, lane);
    if (lane == 0) meta[warp][s] = d;
    issue(d, s);
    cp_async_commit();
  }
  int fill = NST - 1, slot = 0;  // ring stage being filled, stage being consumed
#pragma unroll 1
  for (;;) {
    {
      const TileDesc d = ts.next(p, lane);
      if (lane == 0) meta[warp][fill] = d;
      issue(d, fill);
      cp_async_commit();
      fill = fill + 1 == NST ? 0 : fill + 1;
    }
    cp_async_wait<NST - 1>();
    __syncwarp();
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
    slot = slot + 1 == NST ? 0 : slot + 1;
  }
  if (cur >= 0) finalize(cur, cur_h);
  cp_async_wait<0>();
  finish_launch(p.work);
}

}  // namespace dkv
