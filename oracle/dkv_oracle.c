/*
 * dkv_oracle.c -- slow, plain, fp64 CPU oracle for single-token decode
 * attention with NeoX RoPE over a KV cache.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may include, link
 * or call this file: only the tests, the smoke check of __graft_entry__ and
 * the CPU-baseline leg of bench.py use it.  It shares no code, header, table
 * or constant with the CUDA library.
 *
 * What it computes (the plain definition, no blocking or reordering):
 *   DirectKV README, opening summary: decode attention is ordinary multi-head
 *   attention whose keys carry NeoX RoPE; the method reads the cache from
 *   host or device memory but approximates nothing, so the exact softmax
 *   attention over the logical token sequence is the result to reproduce.
 *   SplitKernel README, Key Features ("attention with host/device KV cache
 *   partitioning"): the placement of a block changes where it is read from,
 *   never the result -- so this oracle works on the LOGICAL sequence and
 *   has no notion of pages, pools or placement at all.
 *
 * Readings taken where the pages are silent (each one listed in the design
 * notes of the repository):
 *   - NeoX RoPE is the GPT-NeoX "rotate half" form over the whole head dim:
 *       theta_i = p * base^(-2i/D),  i < D/2
 *       x'_i       = x_i cos(theta_i) - x_{i+D/2} sin(theta_i)
 *       x'_{i+D/2} = x_{i+D/2} cos(theta_i) + x_i sin(theta_i)
 *     base == 0 means "no rotation".
 *   - token t of a sequence sits at position t; the query of a sequence of
 *     length L sits at position L.
 *   - query head hq reads KV head hq / G with G = Hq / Hkv (consecutive
 *     grouping).
 *   - scale == 0 means 1/sqrt(D).
 *   - L == 0 gives an all-zero output row.
 *   - K and V are stored as raw IEEE binary16 or bfloat16 bit patterns; the
 *     stored values are exact inputs and are decoded exactly here.
 *
 * Build: gcc -O2 -fopenmp -shared -fPIC dkv_oracle.c -lm
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_KV_F16 0
#define ORACLE_KV_BF16 1

/* IEEE 754 binary16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits. */
double oracle_f16_to_f64(uint16_t h) {
  int sign = (h >> 15) & 1;
  int expo = (h >> 10) & 0x1f;
  int frac = h & 0x3ff;
  double mag;
  if (expo == 0)
    mag = ldexp((double)frac, -24); /* subnormal: frac * 2^-14 * 2^-10 */
  else if (expo == 31)
    mag = frac ? NAN : INFINITY;
  else
    mag = ldexp((double)(1024 + frac), expo - 25); /* (1 + frac/2^10) 2^(e-15) */
  return sign ? -mag : mag;
}

/* bfloat16 is the upper half of an IEEE binary32 bit pattern. */
double oracle_bf16_to_f64(uint16_t b) {
  uint32_t u = ((uint32_t)b) << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

static double decode16(uint16_t x, int kv_dtype) {
  return kv_dtype == ORACLE_KV_BF16 ? oracle_bf16_to_f64(x) : oracle_f16_to_f64(x);
}

/* NeoX rotate-half RoPE of one head vector x[D] at position pos, into y[D]. */
void oracle_rope(const double* x, int D, double pos, double base, double* y) {
  int half = D / 2;
  if (base == 0.0) {
    for (int i = 0; i < D; ++i) y[i] = x[i];
    return;
  }
  for (int i = 0; i < half; ++i) {
    double theta = pos * pow(base, -2.0 * (double)i / (double)D);
    double c = cos(theta), s = sin(theta);
    double a = x[i], b = x[i + half];
    y[i] = a * c - b * s;
    y[i + half] = b * c + a * s;
  }
}

/*
 * Decode attention, logical layout.
 *   q        [B][Hq][D]         fp32
 *   k, v     [B][Hkv][Lmax][D]  raw 16-bit (kv_dtype)
 *   seq_lens [B]                0 <= L_b <= Lmax
 *   group_mask [B*Hkv] or NULL: compute only groups (b, h) with mask != 0;
 *              rows of other groups are left untouched.
 *   out      [B][Hq][D]         fp64
 * Returns 0, or -1 on bad arguments.
 */
int oracle_decode(int B, int Hq, int Hkv, int D, int64_t Lmax, const float* q, const uint16_t* k,
                  const uint16_t* v, const int32_t* seq_lens, int kv_dtype, double rope_base,
                  double scale, const uint8_t* group_mask, double* out) {
  if (B < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || D <= 0 || D % 2 != 0 || Lmax < 0) return -1;
  for (int b = 0; b < B; ++b)
    if (seq_lens[b] < 0 || seq_lens[b] > Lmax) return -1;
  const int G = Hq / Hkv;
  const double sc = scale != 0.0 ? scale : 1.0 / sqrt((double)D);
  int ngroups = B * Hkv;
  int failed = 0;

#pragma omp parallel for schedule(dynamic, 1)
  for (int gidx = 0; gidx < ngroups; ++gidx) {
    int b = gidx / Hkv, h = gidx % Hkv;
    if (group_mask && !group_mask[gidx]) continue;
    int64_t L = seq_lens[b];
    double* qhat = (double*)malloc(sizeof(double) * (size_t)G * D);
    double* xk = (double*)malloc(sizeof(double) * (size_t)D);
    double* khat = (double*)malloc(sizeof(double) * (size_t)D);
    double* s = (double*)malloc(sizeof(double) * (size_t)G * (size_t)(L > 0 ? L : 1));
    if (!qhat || !xk || !khat || !s) {
      failed = 1;
      free(qhat); free(xk); free(khat); free(s);
      continue;
    }
    /* rotate the G queries of this group at position L */
    for (int g = 0; g < G; ++g) {
      const float* qr = q + ((size_t)b * Hq + (size_t)h * G + g) * D;
      for (int d = 0; d < D; ++d) xk[d] = (double)qr[d];
      oracle_rope(xk, D, (double)L, rope_base, qhat + (size_t)g * D);
    }
    /* scores s[g][t] = scale * <RoPE(q_g, L), RoPE(k_t, t)> */
    const uint16_t* kb = k + ((size_t)b * Hkv + h) * (size_t)Lmax * D;
    for (int64_t t = 0; t < L; ++t) {
      for (int d = 0; d < D; ++d) xk[d] = decode16(kb[(size_t)t * D + d], kv_dtype);
      oracle_rope(xk, D, (double)t, rope_base, khat);
      for (int g = 0; g < G; ++g) {
        double acc = 0.0;
        for (int d = 0; d < D; ++d) acc += qhat[(size_t)g * D + d] * khat[d];
        s[(size_t)g * L + t] = sc * acc;
      }
    }
    /* exact two-pass softmax per query head, then the V-weighted sum */
    const uint16_t* vb = v + ((size_t)b * Hkv + h) * (size_t)Lmax * D;
    for (int g = 0; g < G; ++g) {
      double* o = out + ((size_t)b * Hq + (size_t)h * G + g) * D;
      for (int d = 0; d < D; ++d) o[d] = 0.0;
      if (L == 0) continue;
      double* sg = s + (size_t)g * L;
      double m = -INFINITY;
      for (int64_t t = 0; t < L; ++t) m = sg[t] > m ? sg[t] : m;
      double z = 0.0;
      for (int64_t t = 0; t < L; ++t) {
        sg[t] = exp(sg[t] - m);
        z += sg[t];
      }
      for (int64_t t = 0; t < L; ++t) {
        double w = sg[t] / z;
        for (int d = 0; d < D; ++d) o[d] += w * decode16(vb[(size_t)t * D + d], kv_dtype);
      }
    }
    free(qhat); free(xk); free(khat); free(s);
  }
  return failed ? -2 : 0;
}

/*
 * K/V projection of one new token per sequence (the write side of the cache).
 *   DirectKV README, opening summary: the fused kernel includes the K/V
 *   projection of the new token; Step 6 reports K and V errors for "all new
 *   KV".  The projection is a plain matrix-vector product per sequence:
 *     y[b][r] = sum_h w[r][h] * x[b][h]
 *   x    [B][H]  fp32
 *   w    [R][H]  raw 16-bit (kv_dtype), row r = kv head r / D, dim r % D
 *   y    [B][R]  fp64 (exact products, fp64 sums)
 */
int oracle_project(int B, int R, int H, const float* x, const uint16_t* w, int kv_dtype, double* y) {
  if (B < 0 || R < 0 || H < 0) return -1;
#pragma omp parallel for schedule(static)
  for (int r = 0; r < R; ++r) {
    for (int b = 0; b < B; ++b) {
      double acc = 0.0;
      for (int h = 0; h < H; ++h) acc += decode16(w[(size_t)r * H + h], kv_dtype) * (double)x[(size_t)b * H + h];
      y[(size_t)b * R + r] = acc;
    }
  }
  return 0;
}
