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
// tg, tg+4, tg+8, tg+12 over the four token groups.  The partial scores of
// the 8 lanes of a token group are combined by a three-step xor
// reduce-scatter, after which each lane owns the scores of one query head;
// the online softmax keeps one running max and sum per head, and the
// softmax weights drive the PV product on the tensor cores.
//
// RoPE.  theta_i(p) = p * base^(-2i/D).  A seed angle is formed in fp64 and
// reduced modulo 2*pi before the fp32 sin/cos, so positions up to 2^24 keep
// full accuracy; the later tokens of a lane follow by multiplying with
// exp(i*4*theta_i(1)), across tiles too while positions continue, with a
// fresh seed at least every 16 tiles (at most 64 fp32 steps, error ~1e-5).
// Scores carry scale*log2(e) so the softmax works with exp2.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace dkv {

constexpr int kTileTokens = 16;
constexpr int kWarps = 4;
constexpr int kThreads = kWarps * 32;
constexpr uint32_t kFull = 0xffffffffu;
constexpr int kFlagPoison = 1 << 8;
constexpr int kSubShift = 9;                   // tile index inside its block (block_size <= 1024)
constexpr int kSubMask = 63;
constexpr float kLazyMax = 8.f;                // softmax reference max lags the true max by < 2^8
constexpr int kStatusTimeout = 4;              // a tile copy did not complete in time (DKV_STATUS_COPY_TIMEOUT)
constexpr int kStatusLayout = 8;               // shared memory not aligned for the tile copies (DKV_STATUS_INTERNAL)
constexpr unsigned long long kWaitLimitNs = 2000000000ull;  // bound of every wait on a tile copy

// Division by a divisor fixed for the launch, by multiplication (Granlund and
// Montgomery, "Division by invariant integers using multiplication", 1994):
// with s = ceil(log2 d) and m = floor(2^32 (2^s - d) / d) + 1, the quotient
// n / d equals (umulhi(n, m) + n) >> s for every 0 <= n < 2^31 (the sum then
// stays below 2^32).  Replaces the per-unit runtime divisions of the kernels.
struct InvDiv {
  uint32_t d, m, s;
  __device__ __forceinline__ int div(int n) const {
    return static_cast<int>((__umulhi(static_cast<uint32_t>(n), m) + static_cast<uint32_t>(n)) >> s);
  }
};

inline InvDiv make_invdiv(int32_t d) {
  InvDiv r{static_cast<uint32_t>(d), 0u, 0u};
  while ((1ull << r.s) < static_cast<uint64_t>(d)) ++r.s;
  r.m = static_cast<uint32_t>(((1ull << 32) * ((1ull << r.s) - static_cast<uint64_t>(d))) / static_cast<uint64_t>(d) + 1);
  return r;
}

struct SplitParams {
  int32_t* work;            // [2]: next unit to hand out, CTAs finished; zero between launches
  const int2* lists;        // [B][list_stride]: (logical block, id) of each pool, or nullptr: logical order
  const int2* counts;       // [B]: (host, device) list lengths
  int32_t list_stride;
  int32_t list_dev;         // this launch walks the device list (the back of each row), else the host list
  const float* q;           // [B][Hq][D]
  const uint16_t* k_pool;   // [nblocks][Hkv][S][D] of this residency
  const uint16_t* v_pool;
  const int32_t* table;     // [B][stride]
  const int32_t* seq_lens;  // [B]
  const double* inv_freq;   // [D/2]
  float* part_o;            // [B][Hq][nslots][D]
  float* part_lse;          // [B][Hq][nslots], log2 domain
  int32_t* status;
  int32_t hq, hkv, block_size, stride, nsplit, nslots, slot_base;
  int32_t bps;              // blocks per split; with lists the minimum, the per-sequence value follows its list
  int32_t id_lo, id_hi;     // ids in [id_lo, id_hi) live in this pool at (id - id_lo)
  int32_t id_total;         // ids in [0, id_total) are valid in some pool
  int32_t max_len;          // largest valid seq_len
  int32_t n_units;          // B * nsplit * Hkv
  int32_t rope;             // 0: no rotation
  float qscale;             // softmax scale * log2(e)
  int32_t stall_first_copy; // test hook: the first tile of unit 0 arms its barrier but issues no copy
  int32_t extra_tokens;     // tokens past seq_lens that belong to the unit (multi-token queries: Tq - 1)
  int32_t num_queries;      // query tokens per sequence (1 for decode)
  InvDiv div_hkv, div_nsplit, div_bs;  // hkv, nsplit, block_size (set_divisors)
};

// Fill the divisor fields from hkv, nsplit and block_size (all >= 1).
inline void set_divisors(SplitParams& p) {
  p.div_hkv = make_invdiv(p.hkv);
  p.div_nsplit = make_invdiv(p.nsplit);
  p.div_bs = make_invdiv(p.block_size);
}

struct MergeParams {
  const float* part_o;
  const float* part_lse;
  float* out;               // [B][Hq][D]
  int32_t nslots;           // slots per row: host splits, then device splits
  int32_t nsplit;           // host slots (the first nsplit of each row)
  int32_t has_host, has_dev;
};

// The per-pool block lists of one call with blocks in both pools.
struct ListParams {
  const int32_t* table;     // [B][stride]
  const int32_t* seq_lens;  // [B]
  int2* lists;              // [B][list_stride]
  int2* counts;             // [B]
  int32_t stride, list_stride, block_size, host_split, id_total, max_len, extra_tokens;
  int32_t invalid_to_dev;   // ids outside both pools go to the device list (else to the host list)
};

// One tile of the copy stream.  unit < 0 marks the end of the stream.
struct TileDesc {
  int32_t unit;
  int32_t pidx;  // block index inside this pool
  int32_t p0;    // logical position of the tile's first token
  int32_t meta;  // valid tokens (0..16) | kFlagPoison | tile in block << kSubShift | kv head << 16
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

// ---- shared-memory tiles and the tensor copies that can fill them
//
// A K tile (16 token rows of D 16-bit elements) is stored as it comes, row
// after row: the 8 lanes of a token group read one row's 8 chunks.  A V tile
// is stored as D/64 sub-tiles of 16 rows x 128 bytes with the 128-byte
// swizzle: inside each 1024-byte group of 8 rows, 16-byte chunk c of row r
// lands at chunk c ^ (r mod 8), so the 8 rows of one ldmatrix phase touch 8
// distinct bank groups.  tile_off gives that V layout to every producer (the
// 16-byte cp.async, the tensor copies) and to the PV loop.

// Tensor maps of the K pool (boxes of 16 plain rows) and the V pool (boxes
// of 16 rows x 64 elements, 128-byte swizzle) of one launch; unused by
// cp.async launches.
struct TileMaps {
  CUtensorMap k, v;
};

// Byte offset of 16-byte chunk `chunk` (0 .. D/8-1) of token row `row` in a tile.
__device__ __forceinline__ int tile_off(int row, int chunk) {
  return (chunk >> 3) * (kTileTokens * 128) + row * 128 + (((chunk & 7) ^ (row & 7)) << 4);
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_init_fence() { asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory"); }
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(bar), "r"(parity)
      : "memory");
  return done != 0;
}
__device__ __forceinline__ unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
// Wait for phase `parity` of the barrier, giving up after kWaitLimitNs.
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = global_ns();
  for (unsigned i = 1;; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 63u) == 0 && global_ns() - t0 > kWaitLimitNs) return false;
  }
}
// Orders this thread's earlier generic-proxy accesses to shared memory before
// its later async-proxy (tensor copy) writes to it.
__device__ __forceinline__ void fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
// One box of the tensor map at (x, y) into shared memory, completing on `bar`
// (CTA-local destination; no multicast).
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
      ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
      : "memory");
}

// cos/sin of pos * w with the angle reduced modulo 2*pi in fp64 first.
__device__ __forceinline__ void rope_cs(int pos, double w, float& c, float& s) {
  const double th = static_cast<double>(pos) * w;
  const double n = rint(th * 0.15915494309189535);        // 1 / (2*pi)
  const double r = fma(-n, 6.283185307179586, th);        // |r| <= pi (+ rounding)
  __sincosf(static_cast<float>(r), &s, &c);
}

// ----------------------------------------------------------------------------- RoPE of the split kernel
//
// Lane li of a token group owns the NeoX pairs i = li*PPL + r, r < PPL, held
// as NP2 = PPL/2 float2 values: element j of a row's "X" array holds dims
// (li*PPL + 2j, li*PPL + 2j + 1), the "Y" array the same dims + D/2.  The
// tables below are filled once per CTA; the decode kernels and dkv_debug_rope
// run the same functions on them.

constexpr int kRopeChainTiles = 16;  // tiles that may follow one fp64-reduced seed

template <int PPL>
struct RopeTables {
  double freq[PPL][8];                 // [r][li]: base^(-2i/D), i = li*PPL + r
  float2 e[PPL / 2][8], f[PPL / 2][8]; // cos / sin of the 4-position step, pairs (2j, 2j+1)
};

// Fill the tables from the D/2 frequencies (all threads of the block; the
// caller synchronises).  rope == false stores zero frequencies.
template <int D>
__device__ __forceinline__ void rope_fill_tables(RopeTables<D / 16>& t, const double* inv_freq, bool rope,
                                                 int tid, int nthreads) {
  constexpr int PPL = D / 16;
  for (int i = tid; i < D / 2; i += nthreads) {
    const double w = rope ? inv_freq[i] : 0.0;
    const int l = i / PPL, r = i % PPL;
    t.freq[r][l] = w;
    float c, sn;
    rope_cs(4, w, c, sn);
    reinterpret_cast<float*>(&t.e[r >> 1][l])[r & 1] = c;
    reinterpret_cast<float*>(&t.f[r >> 1][l])[r & 1] = sn;
  }
}

// cos / sin of position pos for the pairs of lane li.
template <int PPL>
__device__ __forceinline__ void rope_seed(const RopeTables<PPL>& t, int li, int pos, float2 (&C)[PPL / 2],
                                          float2 (&S)[PPL / 2]) {
#pragma unroll
  for (int j = 0; j < PPL / 2; ++j) {
    float c0, s0, c1, s1;
    rope_cs(pos, t.freq[2 * j][li], c0, s0);
    rope_cs(pos, t.freq[2 * j + 1][li], c1, s1);
    C[j] = make_float2(c0, c1);
    S[j] = make_float2(s0, s1);
  }
}

// Start of a K tile whose first token (of this lane's token group tg) sits at
// p0 + tg: continue the rotation state when the tile follows the previous
// one (p0 == next_pos) and fewer than kRopeChainTiles tiles have shared the
// current seed, else take a fresh fp64-reduced seed.
template <int PPL>
__device__ __forceinline__ void rope_tile_start(const RopeTables<PPL>& t, int li, int tg, int p0, int& next_pos,
                                                int& chain, float2 (&C)[PPL / 2], float2 (&S)[PPL / 2]) {
  if (p0 == next_pos && chain < kRopeChainTiles) {
    ++chain;
  } else {
    rope_seed<PPL>(t, li, p0 + tg, C, S);
    chain = 1;
  }
  next_pos = p0 + 16;
}

// Rotate one key row by the angle state (C, S): x' = x c - y s, y' = y c + x s;
// then advance the state 4 positions with the step factors (E, F).  After the
// fourth row of a tile the state is that of the tile 16 positions on.
template <int NP2>
__device__ __forceinline__ void rope_rotate_advance(float2 (&X)[NP2], float2 (&Y)[NP2], float2 (&C)[NP2],
                                                    float2 (&S)[NP2], const float2 (&E)[NP2],
                                                    const float2 (&F)[NP2]) {
#pragma unroll
  for (int j = 0; j < NP2; ++j) {
    const float2 x = X[j], y = Y[j];
    const float2 ns = __fmul2_rn(S[j], make_float2(-1.f, -1.f));
    X[j] = __ffma2_rn(y, ns, __fmul2_rn(x, C[j]));      // x c - y s
    Y[j] = __ffma2_rn(x, S[j], __fmul2_rn(y, C[j]));    // y c + x s
    // (C + iS)(E + iF)
    const float2 cn = __ffma2_rn(ns, F[j], __fmul2_rn(C[j], E[j]));
    S[j] = __ffma2_rn(C[j], F[j], __fmul2_rn(S[j], E[j]));
    C[j] = cn;
  }
}

// A query pair (x = dims i, y = dims i + D/2) rotated by (C, S) and scaled by qs.
__device__ __forceinline__ void rope_query(float2 x, float2 y, float2 C, float2 S, float2 qs, float2& X, float2& Y) {
  const float2 xr = __fmul2_rn(x, C);
  const float2 yr = __fmul2_rn(y, C);
  const float2 ys = __fmul2_rn(y, S);
  X = __fmul2_rn(make_float2(xr.x - ys.x, xr.y - ys.y), qs);   // x c - y s
  Y = __fmul2_rn(__ffma2_rn(x, S, yr), qs);                    // y c + x s
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

// 2^x in one MUFU op (flushes subnormal results to zero; 2^-inf = 0).
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Byte offset of 16-byte chunk c of row r in a tile of ROW-byte rows.  The
// chunk index is XORed with the row (mod 8), so the 8 rows read by one
// ldmatrix phase, and the 8 lanes of one token row, hit 8 distinct bank groups.
template <int ROW>
__device__ __forceinline__ int swz(int r, int c) {
  return r * ROW + ((c ^ (r & 7)) << 4);
}

// Four 8x8 b16 matrices from shared memory, transposed (mma B operand).
__device__ __forceinline__ void ldsm_x4_t(const void* p, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(smem_u32(p)));
}

// Four 8x8 b16 matrices from shared memory (mma B operand of a row-major [n][k] tile).
__device__ __forceinline__ void ldsm_x4(const void* p, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(smem_u32(p)));
}

// D(16x8,f32) += A(16x16) * B(16x8) with all four C rows live.
template <bool BF16>
__device__ __forceinline__ void mma16816_full(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  if constexpr (BF16) {
    asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
                 "{%0,%1,%2,%3};\n"
                 : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
                 : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  } else {
    asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
                 "{%0,%1,%2,%3};\n"
                 : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
                 : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  }
}

// D(16x8,f32) += A(16x16) * B(16x8), A and B both bf16 or both fp16, for A
// whose rows 8..15 are zero: only the C/D rows 0..7 (c[0], c[1]) are kept; the
// rows 8..15 take a zero input and their outputs are discarded, so they cost
// no accumulator registers and chain no dependency between calls.
template <bool BF16>
__device__ __forceinline__ void mma16816_top(float (&c)[2], const uint32_t (&a)[2], uint32_t b0, uint32_t b1) {
  float d2, d3;
  if constexpr (BF16) {
    asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
                 "{%10,%11,%12,%12};\n"
                 : "=f"(c[0]), "=f"(c[1]), "=f"(d2), "=f"(d3)
                 : "r"(a[0]), "r"(0u), "r"(a[1]), "r"(0u), "r"(b0), "r"(b1), "f"(c[0]), "f"(c[1]), "f"(0.f));
  } else {
    asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
                 "{%10,%11,%12,%12};\n"
                 : "=f"(c[0]), "=f"(c[1]), "=f"(d2), "=f"(d3)
                 : "r"(a[0]), "r"(0u), "r"(a[1]), "r"(0u), "r"(b0), "r"(b1), "f"(c[0]), "f"(c[1]), "f"(0.f));
  }
}

// p ~= hi + lo with hi, lo in the 16-bit type of V: returns packed hi pair and lo pair.
template <bool BF16>
__device__ __forceinline__ void split_hi_lo(float2 p, uint32_t& hi, uint32_t& lo) {
  if constexpr (BF16) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(p.x, p.y);
    const float2 hf = __bfloat1622float2(h);
    const __nv_bfloat162 l = __floats2bfloat162_rn(p.x - hf.x, p.y - hf.y);
    hi = *reinterpret_cast<const uint32_t*>(&h);
    lo = *reinterpret_cast<const uint32_t*>(&l);
  } else {
    const __half2 h = __floats2half2_rn(p.x, p.y);
    const float2 hf = __half22float2(h);
    const __half2 l = __floats2half2_rn(p.x - hf.x, p.y - hf.y);
    hi = *reinterpret_cast<const uint32_t*>(&h);
    lo = *reinterpret_cast<const uint32_t*>(&l);
  }
}

// ----------------------------------------------------------------------------- tile stream

// Enumerates, for one warp, the tiles of this residency over its units.  All
// lanes run it in lockstep with identical results; block-table and list reads
// are uniform (one broadcast load per block).  Units are handed out one at a
// time from the launch's work counter, so a warp that finishes early takes
// the next unit and CTAs that start late find the work already taken.
//
// Without lists, split c of sequence b covers the logical blocks
// [c*bps, (c+1)*bps) and skips those of the other pool.  With lists (a call
// whose blocks sit in both pools), split c covers entries
// [c*n', (c+1)*n') of the sequence's list of this pool's blocks, n' =
// max(bps, ceil(n/nsplit)), so every split of a launch holds blocks of its
// own pool and the work of a launch is even whatever the placement.
struct TileStream {
  int unit;
  int b, h, L, j, j_end, sub, pidx, blk;
  const int2* lbase;
  bool started, emitted, bad_len;

  __device__ void grab(const SplitParams& p, int lane) {
    int u = 0;
    if (lane == 0) u = atomicAdd(p.work, 1);
    unit = __shfl_sync(kFull, u, 0);
    started = false;
  }

  __device__ void begin_unit(const SplitParams& p) {
    const int bc = p.div_hkv.div(unit);
    h = unit - bc * p.hkv;
    b = p.div_nsplit.div(bc);
    const int c = bc - b * p.nsplit;
    L = p.seq_lens[b];
    bad_len = (L < 0 || L + p.extra_tokens > p.max_len);
    L += p.extra_tokens;
    if (p.lists) {
      const int2 cnt = p.counts[b];
      const int n = bad_len ? 0 : (p.list_dev ? cnt.y : cnt.x);
      lbase = p.lists + static_cast<size_t>(b) * p.list_stride + (p.list_dev ? p.list_stride - n : 0);
      const int per = max(p.bps, p.div_nsplit.div(n + p.nsplit - 1));
      j = c * per;
      j_end = min(j + per, n);
    } else {
      const int nblk = bad_len ? 0 : p.div_bs.div(L + p.block_size - 1);
      j = c * p.bps;
      j_end = min(j + p.bps, nblk);
    }
    sub = 0;
    emitted = false;
    started = true;
  }

  __device__ TileDesc next(const SplitParams& p, int lane) {
    while (unit < p.n_units) {
      if (!started) begin_unit(p);
      if (bad_len) {
        if (lane == 0) atomicOr(p.status, 2);
        TileDesc d{unit, 0, 0, kFlagPoison | (h << 16)};
        grab(p, lane);
        return d;
      }
      while (j < j_end) {
        if (sub == 0) {
          int id;
          if (p.lists) {
            const int2 e = lbase[j];
            blk = e.x;
            id = e.y;
          } else {
            blk = j;
            id = p.table[static_cast<size_t>(b) * p.stride + j];
          }
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
        const int p0 = blk * p.block_size + sub * kTileTokens;
        const int nvalid = min(kTileTokens, L - p0);
        TileDesc d{unit, pidx, p0, nvalid | (sub << kSubShift) | (h << 16)};
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
      grab(p, lane);
      if (!was_emitted) return TileDesc{u, 0, 0, h << 16};  // empty unit: still reported once
    }
    return TileDesc{-1, 0, 0, 0};
  }
};

// End of a split launch: lets a dependent launch (the merge) be scheduled,
// then the last CTA to finish clears the work counter for the next launch on
// the same workspace.  Every warp of every CTA has stopped taking units by
// the time the last CTA counts itself.
__device__ __forceinline__ void finish_launch(int32_t* work) {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    const unsigned done = atomicAdd(reinterpret_cast<unsigned*>(work + 1), 1u);
    if (done == gridDim.x - 1) {
      atomicExch(work, 0);
      atomicExch(work + 1, 0);
    }
  }
}

// ----------------------------------------------------------------------------- pool lists

// One CTA per sequence: the blocks j < ceil((L_b + extra)/S) of its table row,
// split by pool into (logical block, id) entries kept in logical order; host
// blocks fill the front of the row, device blocks its back.  A sequence with
// an invalid length gets empty lists (the split kernels poison its units).
// The row is read in coalesced chunks of T entries: a first pass counts the
// device entries (where the device list starts), a second places every entry
// at its rank, from warp ballots and the warps' totals in shared memory.
template <int T>
__global__ void __launch_bounds__(T) lists_kernel(const ListParams p) {
  static_assert(T % 32 == 0 && T <= 1024, "block of whole warps");
  constexpr int NW = T / 32;
  __shared__ int2 s_warp[NW];
  __shared__ int s_red[NW];
  const int b = blockIdx.x;
  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  const int L0 = p.seq_lens[b];
  const long long Le = static_cast<long long>(L0) + p.extra_tokens;
  const int n = (L0 < 0 || Le > p.max_len) ? 0 : static_cast<int>((Le + p.block_size - 1) / p.block_size);
  const int32_t* row = p.table + static_cast<size_t>(b) * p.stride;
  auto to_dev = [&](int id) {
    const bool valid = id >= 0 && id < p.id_total;
    return valid ? id >= p.host_split : p.invalid_to_dev != 0;
  };
  // pass 1: device entries of the row
  int nd = 0;
  for (int j = tid; j < n; j += T) nd += to_dev(row[j]) ? 1 : 0;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) nd += __shfl_xor_sync(kFull, nd, o);
  if (lane == 0) s_red[warp] = nd;
  __syncthreads();
  int td = 0;
#pragma unroll
  for (int w = 0; w < NW; ++w) td += s_red[w];
  // pass 2: ranks, chunk by chunk
  int2* out = p.lists + static_cast<size_t>(b) * p.list_stride;
  const unsigned lt = (1u << lane) - 1u;
  int base_h = 0, base_d = p.list_stride - td;
  for (int c0 = 0; c0 < n; c0 += T) {
    const int j = c0 + tid;
    const bool live = j < n;
    const int id = live ? row[j] : 0;
    const bool dev = live && to_dev(id);
    const bool host = live && !dev;
    const unsigned bh = __ballot_sync(kFull, host);
    const unsigned bd = __ballot_sync(kFull, dev);
    if (lane == 0) s_warp[warp] = make_int2(__popc(bh), __popc(bd));
    __syncthreads();
    int oh = 0, od = 0, ch = 0, cd = 0;
#pragma unroll
    for (int w = 0; w < NW; ++w) {
      const int2 v = s_warp[w];
      if (w < warp) {
        oh += v.x;
        od += v.y;
      }
      ch += v.x;
      cd += v.y;
    }
    if (host) out[base_h + oh + __popc(bh & lt)] = make_int2(j, id);
    if (dev) out[base_d + od + __popc(bd & lt)] = make_int2(j, id);
    base_h += ch;
    base_d += cd;
    __syncthreads();   // s_warp is rewritten by the next chunk
  }
  if (tid == 0) p.counts[b] = make_int2(base_h, td);
}

// ----------------------------------------------------------------------------- split kernel

// Shared memory of the split kernel besides the tile rings (all of it is
// dynamic, rings first, so the rings start at the 1024-byte aligned base of
// the block's shared memory).
template <int PPL, int NST>
struct SplitSmemTail {
  uint64_t bar[kWarps][NST];                 // per ring stage: completion of its tensor copies
  TileDesc meta[kWarps][NST];
  alignas(16) float s_p[kWarps][4][4][4];    // softmax weights of the tile: [head][token group][m]
  RopeTables<PPL> rope;
};

// Dynamic shared memory of split_kernel<D, *, *, NST, *, *>.
__host__ __device__ constexpr size_t split_smem_bytes(int D, int nst) {
  return static_cast<size_t>(kWarps) * nst * 2 * kTileTokens * D * 2 +
         (D == 64 ? sizeof(SplitSmemTail<4, 4>) : sizeof(SplitSmemTail<8, 4>));
}

template <int D, int G, bool BF16, int NST, bool ROPE, bool TMA>
__global__ void __launch_bounds__(kThreads) split_kernel(const SplitParams p, const __grid_constant__ TileMaps maps) {
  static_assert(G >= 1 && G <= 4, "query group of 1, 2 or 4 heads");
  static_assert(NST <= 4, "SplitSmemTail is sized for up to 4 stages");
  constexpr int PPL = D / 16;                  // NeoX pairs per lane
  constexpr int NP2 = PPL / 2;                 // fp32 pairs per half-row per lane
  constexpr int ROW = D * 2;                   // bytes of one token row
  constexpr int TILE = kTileTokens * ROW;      // bytes of one K (or V) tile
  constexpr int CPR = ROW / 16;                // 16-byte chunks per row
  constexpr int NT = D / 8;                    // 8-wide output column tiles of the PV mma
  static_assert(G <= 4, "hi rows 0..3 and lo rows 4..7 of the PV mma");
  extern __shared__ __align__(1024) char split_smem[];
  char* const smem = split_smem;
  SplitSmemTail<PPL, NST>& tail =
      *reinterpret_cast<SplitSmemTail<PPL, NST>*>(smem + static_cast<size_t>(kWarps) * NST * 2 * TILE);
  auto& meta = tail.meta;
  auto& s_rope = tail.rope;
  auto& s_p = tail.s_p;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int tg = lane >> 3;                    // token group (K side)
  const int li = lane & 7;                     // lane in token group
  const int gT = lane >> 2;                    // head row of the mma fragments
  const int cT = lane & 3;                     // column pair of the mma fragments
  char* ring = smem + static_cast<size_t>(warp) * NST * 2 * TILE;

  if constexpr (TMA) {
    // the swizzled tensor copies need 1024-byte aligned tiles; report and do
    // nothing rather than copy into a misaligned ring
    if (smem_u32(smem) & 1023u) {
      if (threadIdx.x == 0) atomicOr(p.status, kStatusLayout);
      finish_launch(p.work);
      return;
    }
    if (lane == 0) {
#pragma unroll
      for (int s = 0; s < NST; ++s) mbar_init(smem_u32(&tail.bar[warp][s]), 1);
      mbar_init_fence();
    }
  }
  rope_fill_tables<D>(s_rope, p.inv_freq, ROPE, threadIdx.x, kThreads);
  __syncthreads();

  // 4-position step factors of this lane's pairs, kept in registers
  float2 re[NP2], rf[NP2];
#pragma unroll
  for (int j = 0; j < NP2; ++j) {
    re[j] = s_rope.e[j][li];
    rf[j] = s_rope.f[j][li];
  }

  TileStream ts;
  ts.grab(p, lane);

  // Tile copies.  TMA: lane 0 arms the stage's barrier with the tile's bytes
  // and issues D/64 boxes for K and for V; a stage with nothing to copy gets a
  // plain arrival, so every stage completes exactly once per use.  cp.async:
  // copy e = lane + 32 k moves 16-byte chunk (e mod CPR) of row (e / CPR);
  // its shared-memory offset repeats every 4 copies plus 1024 bytes (8 rows).
  constexpr int KCOPIES = kTileTokens * CPR / 32;
  int dofs[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int e = lane + 32 * k;
    dofs[k] = tile_off(e / CPR, e % CPR);
  }
  // ldmatrix offsets of this lane inside a V tile: row (lane & 15), chunk
  // 2 qd + (lane >> 4); chunks c and c + 8 differ by the 2048-byte half, so
  // four values cover qd = 0..D/16-1.
  int vofs_q[4];
#pragma unroll
  for (int q4 = 0; q4 < 4; ++q4) vofs_q[q4] = tile_off((lane & 7) | (lane & 8), 2 * q4 + (lane >> 4));
  // test hook (dkv_debug_stall_copy): the first tile copy of unit 0 is left
  // unissued.  Units are handed out once each, so exactly one warp of the
  // launch meets it, whichever CTA runs first.
  bool stall_armed = TMA && p.stall_first_copy;
  uint32_t phase = 0;     // per stage: parity of its next completion (TMA)
  uint32_t inflight = 0;  // per stage: tensor copies issued and not yet waited for (TMA)
  bool broken = false;    // a copy did not complete in time: no more copies, every later tile poisoned (TMA)
  auto issue = [&](const TileDesc& d, int slot) {
    const int nvalid = d.meta & 0xff;
    const bool copy = !(d.unit < 0 || (d.meta & kFlagPoison) || nvalid == 0);
    const int h = d.meta >> 16;
    const int sub = (d.meta >> kSubShift) & kSubMask;
    char* sk = ring + static_cast<size_t>(slot) * 2 * TILE;
    char* sv = sk + TILE;
    if constexpr (TMA) {
      if (broken) return;
      if (lane == 0) {
        const uint32_t bar = smem_u32(&tail.bar[warp][slot]);
        if (copy) {
          const int row0 = (d.pidx * p.hkv + h) * p.block_size + sub * kTileTokens;
          mbar_arrive_expect_tx(bar, 2 * TILE);
          // the test hook leaves one stage armed with nothing to complete it
          if (!(stall_armed && d.unit == 0)) {
            tma_load_2d(smem_u32(sk), &maps.k, 0, row0, bar);   // K: one box of 16 plain rows
#pragma unroll
            for (int x = 0; x < D / 64; ++x)                    // V: D/64 swizzled 64-element halves
              tma_load_2d(smem_u32(sv + x * kTileTokens * 128), &maps.v, 64 * x, row0, bar);
          }
        } else {
          mbar_arrive(bar);
        }
      }
      if (copy) {
        inflight |= 1u << slot;
        if (d.unit == 0) stall_armed = false;
      }
    } else {
      if (!copy) return;
      const size_t row0 = (static_cast<size_t>(d.pidx) * p.hkv + h) * p.block_size + sub * kTileTokens;
      const char* gk = reinterpret_cast<const char*>(p.k_pool + row0 * D) + lane * 16;
      const char* gv = reinterpret_cast<const char*>(p.v_pool + row0 * D) + lane * 16;
      if (nvalid == kTileTokens) {
#pragma unroll
        for (int k = 0; k < KCOPIES; ++k) {
          cp_async16(sk + lane * 16 + 512 * k, gk + 512 * k, 16);
          cp_async16(sv + dofs[k & 3] + (k >> 2) * 1024, gv + 512 * k, 16);
        }
      } else {
#pragma unroll
        for (int k = 0; k < KCOPIES; ++k) {
          const int nb = (lane + 32 * k) / CPR < nvalid ? 16 : 0;   // rows past the end: zeros, nothing read
          cp_async16(sk + lane * 16 + 512 * k, nb ? gk + 512 * k : gk - lane * 16, nb);
          cp_async16(sv + dofs[k & 3] + (k >> 2) * 1024, nb ? gv + 512 * k : gv - lane * 16, nb);
        }
      }
    }
  };
  // Completion of stage `slot` before its tile is read.  TMA: bounded wait on
  // the stage's barrier; rows of V past the sequence end hold whatever the
  // block stores there, so they are zeroed (their weights are 0, but 0 * NaN
  // is not).  Returns false if the tile cannot be used.
  auto await_stage = [&](const TileDesc& d, int slot) {
    if constexpr (TMA) {
      if (broken) return false;
      const bool ok = mbar_wait_bounded(smem_u32(&tail.bar[warp][slot]), (phase >> slot) & 1u);
      if (!__all_sync(kFull, ok)) {
        broken = true;
        if (lane == 0) atomicOr(p.status, kStatusTimeout);
        return false;
      }
      phase ^= 1u << slot;
      inflight &= ~(1u << slot);
      const int nvalid = d.meta & 0xff;
      if (d.unit >= 0 && !(d.meta & kFlagPoison) && nvalid > 0 && nvalid < kTileTokens) {
        char* sv = ring + static_cast<size_t>(slot) * 2 * TILE + TILE;
        for (int e = lane; e < (kTileTokens - nvalid) * CPR; e += 32)
          *reinterpret_cast<uint4*>(sv + tile_off(nvalid + e / CPR, e % CPR)) = make_uint4(0u, 0u, 0u, 0u);
        fence_proxy_async();   // before a later tensor copy overwrites this stage
      }
      __syncwarp();
      return true;
    } else {
      cp_async_wait<NST - 1>();
      __syncwarp();
      return true;
    }
  };

  // per-unit state.  QX/QY: rotated, pre-scaled queries of this lane's dims.
  // acc: PV accumulators in mma C layout (rows 0..7): rows 0..G-1 hold the
  // bf16/fp16 "hi" part of the weights (lanes 0..4G-1), rows 4..4+G-1 the "lo"
  // remainder (lanes 16..16+4G-1); out = row g + row 4+g.
  float2 QX[G][NP2], QY[G][NP2];
  float acc[NT][2];
  // After the reduce-scatter of the scores, lane li of every token group owns
  // head gl of the softmax (G=4: gl = li/2; G=2: li/4; G=1: 0) and keeps that
  // head's running max and (lane-partial) running sum.
  constexpr int HL = 8 / G;                    // lanes per head inside a token group
  const int gl = li / HL;
  float mrun = -1e30f, lrun = 0.f;
  bool poisoned = false;
  int cur = -1;
  // RoPE factors carried from one tile to the next when positions continue
  float2 Cc[NP2], Sc[NP2];
  int next_pos = -1, chain = 0;

  auto init_unit = [&](int unit, int h) {
    const int b = p.div_nsplit.div(p.div_hkv.div(unit));
    const int L = p.seq_lens[b];
    float2 C[NP2], S[NP2];
    if constexpr (ROPE) {
      rope_seed<PPL>(s_rope, li, L, C, S);
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
        rope_query(x, y, C[j], S[j], qs, QX[g][j], QY[g][j]);
      }
    }
    mrun = -1e30f;
    lrun = 0.f;
#pragma unroll
    for (int n = 0; n < NT; ++n) acc[n][0] = acc[n][1] = 0.f;
    poisoned = false;
  };

  // lanes of one head: the HL lanes of a token group (xor < HL) and the 4 groups (xor 8, 16)
  auto head_sum = [&](float v) {
#pragma unroll
    for (int o = 1; o < HL; o <<= 1) v += __shfl_xor_sync(kFull, v, o);
    v += __shfl_xor_sync(kFull, v, 8);
    v += __shfl_xor_sync(kFull, v, 16);
    return v;
  };
  auto head_max = [&](float v) {
#pragma unroll
    for (int o = 1; o < HL; o <<= 1) v = fmaxf(v, __shfl_xor_sync(kFull, v, o));
    v = fmaxf(v, __shfl_xor_sync(kFull, v, 8));
    v = fmaxf(v, __shfl_xor_sync(kFull, v, 16));
    return v;
  };

  auto finalize = [&](int unit, int h) {
    const int bc = p.div_hkv.div(unit);
    const int b = p.div_nsplit.div(bc);
    const int c = bc - b * p.nsplit;
    const float ltot = head_sum(lrun);
    // hi rows (lanes 0..15) + lo rows (lanes 16..31) of the same head and columns
#pragma unroll
    for (int n = 0; n < NT; ++n) {
      acc[n][0] += __shfl_xor_sync(kFull, acc[n][0], 16);
      acc[n][1] += __shfl_xor_sync(kFull, acc[n][1], 16);
    }
    // the output lanes of head gT take its sum and max from lane gT * HL
    const float l = __shfl_sync(kFull, ltot, (gT & 3) * HL);
    const float M = __shfl_sync(kFull, mrun, (gT & 3) * HL);
    if (gT < G) {
      const size_t row = (static_cast<size_t>(b) * p.hq + h * G + gT) * p.nslots + p.slot_base + c;
      float* o = p.part_o + row * D;
      const float qnan = __int_as_float(0x7fc00000);
      const float inv = poisoned ? qnan : (l > 0.f ? 1.f / l : 0.f);
#pragma unroll
      for (int n = 0; n < NT; ++n)
        *reinterpret_cast<float2*>(o + 8 * n + 2 * cT) = make_float2(acc[n][0] * inv, acc[n][1] * inv);
      if (cT == 0) p.part_lse[row] = poisoned ? qnan : (l > 0.f ? M + __log2f(l) : -INFINITY);
    }
  };

  auto compute = [&](int slot, const TileDesc& d) {
    const char* sk = ring + static_cast<size_t>(slot) * 2 * TILE;
    const char* sv = sk + TILE;
    const int nvalid = d.meta & 0xff;
    // ---- scores: rotate K rows on the fly (CUDA cores, fp32 pairs).  The
    // rotation state (Cc, Sc) carries over when this tile continues the
    // previous one; a fresh fp64-reduced seed at least every 16 tiles.
    if constexpr (ROPE) rope_tile_start<PPL>(s_rope, li, tg, d.p0, next_pos, chain, Cc, Sc);
    float2 (&C)[NP2] = Cc;
    float2 (&S)[NP2] = Sc;
    float v[4 * G];  // partial scores, index g * 4 + m
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      float2 X[NP2], Y[NP2];
      const char* krow = sk + (tg + 4 * m) * ROW + li * PPL * 2;   // K rows are stored as they come
      load_pairs<NP2, BF16>(krow, X);
      load_pairs<NP2, BF16>(krow + D, Y);
      if constexpr (ROPE) rope_rotate_advance<NP2>(X, Y, C, S, re, rf);
#pragma unroll
      for (int g = 0; g < G; ++g) {
        float2 a = __ffma2_rn(QY[g][0], Y[0], __fmul2_rn(QX[g][0], X[0]));
#pragma unroll
        for (int j = 1; j < NP2; ++j) {
          a = __ffma2_rn(QX[g][j], X[j], a);
          a = __ffma2_rn(QY[g][j], Y[j], a);
        }
        v[g * 4 + m] = a.x + a.y;
      }
    }
    // ---- reduce-scatter over the 8 lanes of the token group: halve the value
    // set at each xor step; lane li ends with scores g*4+m = li*(4G/8) + k
    constexpr int NV = 4 * G;
    constexpr int NH = NV >= 8 ? NV / 8 : 1;  // values held per lane at the end
#pragma unroll
    for (int b = 4, n = NV; b >= 1; b >>= 1) {
      if (n > 1) {
        const bool up = (li & b) != 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          if (i < n / 2) {
            const float send = up ? v[i] : v[i + n / 2];
            const float keep = up ? v[i + n / 2] : v[i];
            v[i] = keep + __shfl_xor_sync(kFull, send, b);
          }
        }
        n >>= 1;
      } else {
        v[0] += __shfl_xor_sync(kFull, v[0], b);
      }
    }
    // this lane's tokens (G=4: m = 2(li&1)+k; G=2: m = li&3; G=1: m = li>>1)
    float sc[NH];
    int mt[NH];
#pragma unroll
    for (int k = 0; k < NH; ++k) {
      const int j = (G == 4) ? (li * 2 + k) : (G == 2 ? li : (li >> 1));
      mt[k] = j & 3;
      sc[k] = (tg + 4 * mt[k]) < nvalid ? v[k] : -INFINITY;
    }
    // ---- online softmax for head gl.  The reference max mrun (shared by the
    // head's lanes) is raised only when a score of the tile exceeds it by more
    // than kLazyMax (log2 units), so the weights 2^(s - mrun) stay below
    // 2^kLazyMax.  The running sum and the output use the same reference, so
    // the result is exact up to rounding; most tiles skip the cross-lane max,
    // the rescale factor and the accumulator rescale.
    float tm = sc[0];
#pragma unroll
    for (int k = 1; k < NH; ++k) tm = fmaxf(tm, sc[k]);
    if (__any_sync(kFull, tm > mrun + kLazyMax)) {
      tm = head_max(tm);
      const float mx = fmaxf(mrun, tm);
      const float alpha = ex2(mrun - mx);
      lrun *= alpha;
      mrun = mx;
      const float al = __shfl_sync(kFull, alpha, (gT & 3) * HL);
#pragma unroll
      for (int n = 0; n < NT; ++n) {
        acc[n][0] *= al;
        acc[n][1] *= al;
      }
    }
    float psum = 0.f;
    float pv[NH];
#pragma unroll
    for (int k = 0; k < NH; ++k) {
      pv[k] = ex2(sc[k] - mrun);
      psum += pv[k];
    }
    if constexpr (G == 4) {
      *reinterpret_cast<float2*>(&s_p[warp][gl][tg][mt[0]]) = make_float2(pv[0], pv[1]);
    } else if constexpr (G == 2) {
      s_p[warp][gl][tg][mt[0]] = pv[0];
    } else {
      if ((li & 1) == 0) s_p[warp][0][tg][mt[0]] = pv[0];
      if (li & 1) psum = 0.f;  // the odd lane holds a duplicate of its even neighbour's token
    }
    lrun += psum;
    __syncwarp();
    // ---- PV on the tensor cores.  A rows 0..7 (lane >> 2): rows 0..3 hi,
    // rows 4..7 lo, of head (lane >> 2) & 3; B = V from the swizzled tile.
    uint32_t a[2] = {0u, 0u};
    const int gA = gT & 3;
    if (gA < G) {
      // tokens 2c, 2c+1 (a[0]) and 2c+8, 2c+9 (a[1]); token t lives at [t % 4][t / 4]
      const float* sp = &s_p[warp][gA][0][0];
      const int t0 = 2 * cT;
      const float2 pa = make_float2(sp[(t0 & 3) * 4 + (t0 >> 2)], sp[((t0 + 1) & 3) * 4 + (t0 >> 2)]);
      const float2 pb = make_float2(sp[(t0 & 3) * 4 + (t0 >> 2) + 2], sp[((t0 + 1) & 3) * 4 + (t0 >> 2) + 2]);
      uint32_t ha, la, hb, lb;
      split_hi_lo<BF16>(pa, ha, la);
      split_hi_lo<BF16>(pb, hb, lb);
      a[0] = lane < 16 ? ha : la;
      a[1] = lane < 16 ? hb : lb;
    }
#pragma unroll
    for (int qd = 0; qd < D / 16; ++qd) {
      uint32_t b0, b1, b2, b3;
      ldsm_x4_t(sv + vofs_q[qd & 3] + (qd >> 2) * (kTileTokens * 128), b0, b1, b2, b3);
      mma16816_top<BF16>(acc[2 * qd], a, b0, b1);
      mma16816_top<BF16>(acc[2 * qd + 1], a, b2, b3);
    }
  };

  // prologue: NST-1 tiles in flight
#pragma unroll 1
  for (int s = 0; s < NST - 1; ++s) {
    const TileDesc d = ts.next(p, lane);
    if (lane == 0) meta[warp][s] = d;
    issue(d, s);
    if constexpr (!TMA) cp_async_commit();
  }
  int cur_h = 0;
  int fill = NST - 1, slot = 0;  // ring stage being filled, stage being consumed
#pragma unroll 1
  for (;;) {
    {
      const TileDesc d = ts.next(p, lane);
      if (lane == 0) meta[warp][fill] = d;
      issue(d, fill);
      if constexpr (!TMA) cp_async_commit();
      fill = fill + 1 == NST ? 0 : fill + 1;
    }
    __syncwarp();
    const TileDesc d = meta[warp][slot];
    const bool usable = await_stage(d, slot);
    if (d.unit < 0) break;
    if (d.unit != cur) {
      if (cur >= 0) finalize(cur, cur_h);
      cur = d.unit;
      cur_h = d.meta >> 16;
      init_unit(cur, cur_h);
    }
    if ((d.meta & kFlagPoison) || !usable) poisoned = true;
    else if ((d.meta & 0xff) > 0) compute(slot, d);
    __syncwarp();
    slot = slot + 1 == NST ? 0 : slot + 1;
  }
  if (cur >= 0) finalize(cur, cur_h);
  if constexpr (TMA) {
    // after a timed-out copy, give the copies still in flight a bounded time to
    // land before the block's shared memory is released
    if (inflight) {
#pragma unroll 1
      for (int s = 0; s < NST; ++s)
        if (inflight & (1u << s)) mbar_wait_bounded(smem_u32(&tail.bar[warp][s]), (phase >> s) & 1u);
    }
  } else {
    cp_async_wait<0>();
  }
  finish_launch(p.work);
}

// ----------------------------------------------------------------------------- RoPE check kernel

// The D/2 RoPE frequencies passed by value (head_dim <= 128).
struct RopeFreqs {
  double w[64];
};

// dkv_debug_rope: one warp runs the split kernel's RoPE steps on its own data.
// Key tiles are walked in order, as a warp walks the tiles of its units: the
// same lane layout, seeds, 4-position recurrence and chaining rule, so row r
// of tile i is rotated at position tile_pos[i] + r exactly as the decode
// kernel rotates a K row it holds in shared memory.  Queries are rotated as
// init_unit rotates them, with a scale of 1.
template <int D, bool BF16>
__global__ void __launch_bounds__(32) rope_debug_kernel(const __grid_constant__ RopeFreqs fr, const uint16_t* k,
                                                        const int32_t* tile_pos, int num_tiles, float* k_out,
                                                        const float* q, const int32_t* q_pos, int num_q,
                                                        float* q_out) {
  constexpr int PPL = D / 16;
  constexpr int NP2 = PPL / 2;
  __shared__ RopeTables<PPL> t;
  const int lane = threadIdx.x;
  const int tg = lane >> 3;
  const int li = lane & 7;
  rope_fill_tables<D>(t, fr.w, true, lane, 32);
  __syncthreads();
  float2 E[NP2], F[NP2], C[NP2], S[NP2];
#pragma unroll
  for (int j = 0; j < NP2; ++j) {
    E[j] = t.e[j][li];
    F[j] = t.f[j][li];
  }
  int next_pos = -1, chain = 0;
  for (int i = 0; i < num_tiles; ++i) {
    rope_tile_start<PPL>(t, li, tg, tile_pos[i], next_pos, chain, C, S);
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      const size_t row = static_cast<size_t>(i) * kTileTokens + tg + 4 * m;
      const char* src = reinterpret_cast<const char*>(k + row * D) + li * PPL * 2;
      float2 X[NP2], Y[NP2];
      load_pairs<NP2, BF16>(src, X);
      load_pairs<NP2, BF16>(src + D, Y);
      rope_rotate_advance<NP2>(X, Y, C, S, E, F);
      float* o = k_out + row * D + li * PPL;
#pragma unroll
      for (int j = 0; j < NP2; ++j) {
        *reinterpret_cast<float2*>(o + 2 * j) = X[j];
        *reinterpret_cast<float2*>(o + D / 2 + 2 * j) = Y[j];
      }
    }
  }
  for (int n = 0; n < num_q; ++n) {
    float2 Cq[NP2], Sq[NP2];
    rope_seed<PPL>(t, li, q_pos[n], Cq, Sq);
    const float* qn = q + static_cast<size_t>(n) * D + li * PPL;
    float* o = q_out + static_cast<size_t>(n) * D + li * PPL;
#pragma unroll
    for (int j = 0; j < NP2; ++j) {
      float2 X, Y;
      rope_query(*reinterpret_cast<const float2*>(qn + 2 * j), *reinterpret_cast<const float2*>(qn + D / 2 + 2 * j),
                 Cq[j], Sq[j], make_float2(1.f, 1.f), X, Y);
      if (tg == 0) {
        *reinterpret_cast<float2*>(o + 2 * j) = X;
        *reinterpret_cast<float2*>(o + D / 2 + 2 * j) = Y;
      }
    }
  }
}

// ----------------------------------------------------------------------------- merge kernel

// One CTA per output row (b, hq); blockDim = 32 * W threads, W = the slot
// warps (merge_warps).  Warp w takes slots w, w + W, ... and keeps its own
// online combine of them: a running max m_w, sum z_w = sum 2^(lse_i - m_w)
// and acc_w = sum 2^(lse_i - m_w) o_i for its lane's D/32 dims, so the lse
// and the partial outputs are read in one pass.  After one barrier the first
// D threads rescale the warps' results to the row's max and divide.  A NaN
// slot makes the row NaN; a row with no valid non-empty slot is zero.
constexpr int kMergeMaxWarps = 32;

// slot warps of a merge CTA: one per slot up to 32, at least D/32 for the
// final combine
__host__ __device__ constexpr int merge_warps(int nslots, int D) {
  return nslots >= kMergeMaxWarps ? kMergeMaxWarps : (nslots > D / 32 ? nslots : D / 32);
}

template <int D>
__global__ void __launch_bounds__(kMergeMaxWarps * 32) merge_kernel(const MergeParams p) {
  constexpr int V = D / 32;  // dims per lane
  static_assert(V == 2 || V == 4, "head_dim 64 or 128");
  __shared__ float s_acc[kMergeMaxWarps][D];
  __shared__ float s_m[kMergeMaxWarps], s_z[kMergeMaxWarps];
  __shared__ int s_nan[kMergeMaxWarps];
  // launched as a programmatic dependent of the split kernel: wait until that
  // grid has completed and its partials are visible (no-op otherwise)
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int row = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nw = blockDim.x >> 5;
  const float* lse = p.part_lse + static_cast<size_t>(row) * p.nslots;
  const float* o = p.part_o + static_cast<size_t>(row) * p.nslots * D + lane * V;

  float m = -INFINITY, z = 0.f;
  float acc[V];
#pragma unroll
  for (int k = 0; k < V; ++k) acc[k] = 0.f;
  int nan = 0;
#pragma unroll 2
  for (int i = warp; i < p.nslots; i += nw) {
    if (!(i < p.nsplit ? p.has_host : p.has_dev)) continue;
    const float l = lse[i];
    float x[V];
    if constexpr (V == 4) {
      const float4 t = *reinterpret_cast<const float4*>(o + static_cast<size_t>(i) * D);
      x[0] = t.x; x[1] = t.y; x[2] = t.z; x[3] = t.w;
    } else {
      const float2 t = *reinterpret_cast<const float2*>(o + static_cast<size_t>(i) * D);
      x[0] = t.x; x[1] = t.y;
    }
    if (isnan(l)) {
      nan = 1;
      continue;
    }
    if (l == -INFINITY) continue;  // empty split
    if (l > m) {
      const float r = exp2f(m - l);  // 0 while m is -inf
      z *= r;
#pragma unroll
      for (int k = 0; k < V; ++k) acc[k] *= r;
      m = l;
    }
    const float w = exp2f(l - m);
    z += w;
#pragma unroll
    for (int k = 0; k < V; ++k) acc[k] = fmaf(w, x[k], acc[k]);
  }
#pragma unroll
  for (int k = 0; k < V; ++k) s_acc[warp][lane * V + k] = acc[k];
  if (lane == 0) {
    s_m[warp] = m;
    s_z[warp] = z;
    s_nan[warp] = nan;
  }
  __syncthreads();
  if (threadIdx.x >= D) return;
  // thread d: lane w of its warp holds slot warp w's rescale factor
  const float mw = lane < nw ? s_m[lane] : -INFINITY;
  const int anynan = __any_sync(kFull, lane < nw && s_nan[lane] != 0);
  float M = mw;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(kFull, M, off));
  float* dst = p.out + static_cast<size_t>(row) * D;
  const int d = threadIdx.x;
  if (anynan || M == -INFINITY) {
    dst[d] = anynan ? __int_as_float(0x7fc00000) : 0.f;
    return;
  }
  const float sc = mw == -INFINITY ? 0.f : exp2f(mw - M);
  float Z = lane < nw ? s_z[lane] * sc : 0.f;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) Z += __shfl_xor_sync(kFull, Z, off);
  float a = 0.f;
  for (int w = 0; w < nw; ++w) a = fmaf(__shfl_sync(kFull, sc, w), s_acc[w][d], a);
  dst[d] = a / Z;
}

}  // namespace dkv
