/*
 * Seeded synthetic inputs for the routed-MoE layer tests and benchmark.
 *
 * This module only DRAWS inputs: random numbers, the rounding of drawn
 * weights/hidden states to their storage formats (bf16, FP8 e4m3 with one
 * fp32 scale per 128x128 block, NVFP4 = e2m1 with one e4m3 scale per 16
 * elements and one fp32 scale per tensor), and permutations.  It holds none
 * of the layer's arithmetic (no router, gating, permutation, cache, FFN or
 * combine), so both the oracle and the CUDA path can consume its output.
 *
 * Random numbers: Philox4x32-10, the counter-based generator published by
 * Salmon, Moraes, Dror and Shaw, "Parallel Random Numbers: As Easy as 1, 2, 3"
 * (SC'11).  Key = (seed, stream tag); counter = (block index, a, b, c) where
 * (a, b, c) name a sub-stream (expert, matrix, step, row, attempt ...).
 * Normals: Box-Muller on two uniforms (u = (x + 0.5) / 2^32), in double.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#define PHILOX_M0 0xD2511F53u
#define PHILOX_M1 0xCD9E8D57u
#define PHILOX_W0 0x9E3779B9u
#define PHILOX_W1 0xBB67AE85u

void synth_philox(const uint32_t ctr_in[4], const uint32_t key_in[2], uint32_t out[4]) {
  uint32_t c0 = ctr_in[0], c1 = ctr_in[1], c2 = ctr_in[2], c3 = ctr_in[3];
  uint32_t k0 = key_in[0], k1 = key_in[1];
  for (int r = 0; r < 10; ++r) {
    if (r) { k0 += PHILOX_W0; k1 += PHILOX_W1; }
    uint64_t p0 = (uint64_t)PHILOX_M0 * c0;
    uint64_t p1 = (uint64_t)PHILOX_M1 * c2;
    uint32_t n0 = (uint32_t)(p1 >> 32) ^ c1 ^ k0;
    uint32_t n1 = (uint32_t)p1;
    uint32_t n2 = (uint32_t)(p0 >> 32) ^ c3 ^ k1;
    uint32_t n3 = (uint32_t)p0;
    c0 = n0; c1 = n1; c2 = n2; c3 = n3;
  }
  out[0] = c0; out[1] = c1; out[2] = c2; out[3] = c3;
}

static inline double u01(uint32_t x) { return ((double)x + 0.5) * (1.0 / 4294967296.0); }

/* out[j] = sigma * N(0,1), j in [0,n); element j comes from counter block j/4. */
void synth_normal(uint32_t seed, uint32_t tag, uint32_t a, uint32_t b, uint32_t c,
                  int64_t n, double sigma, float* out) {
  const double two_pi = 6.283185307179586476925286766559;
  int64_t nblk = (n + 3) / 4;
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < nblk; ++i) {
    uint32_t ctr[4] = {(uint32_t)i, a, b, c}, key[2] = {seed, tag}, r[4];
    synth_philox(ctr, key, r);
    double z[4];
    double rad0 = sqrt(-2.0 * log(u01(r[0]))), th0 = two_pi * u01(r[1]);
    double rad1 = sqrt(-2.0 * log(u01(r[2]))), th1 = two_pi * u01(r[3]);
    z[0] = rad0 * cos(th0); z[1] = rad0 * sin(th0);
    z[2] = rad1 * cos(th1); z[3] = rad1 * sin(th1);
    for (int l = 0; l < 4; ++l) {
      int64_t j = i * 4 + l;
      if (j < n) out[j] = (float)(sigma * z[l]);
    }
  }
}

/* out[j] = lo + (hi - lo) * U(0,1). */
void synth_uniform(uint32_t seed, uint32_t tag, uint32_t a, uint32_t b, uint32_t c,
                   int64_t n, double lo, double hi, float* out) {
  int64_t nblk = (n + 3) / 4;
  for (int64_t i = 0; i < nblk; ++i) {
    uint32_t ctr[4] = {(uint32_t)i, a, b, c}, key[2] = {seed, tag}, r[4];
    synth_philox(ctr, key, r);
    for (int l = 0; l < 4; ++l) {
      int64_t j = i * 4 + l;
      if (j < n) out[j] = (float)(lo + (hi - lo) * u01(r[l]));
    }
  }
}

/* Fisher-Yates shuffle of 0..n-1; step i draws counter (i, 0, 0, 0). */
void synth_permutation(uint32_t seed, uint32_t tag, int32_t n, int32_t* out) {
  for (int32_t i = 0; i < n; ++i) out[i] = i;
  for (int32_t i = n - 1; i > 0; --i) {
    uint32_t ctr[4] = {(uint32_t)i, 0, 0, 0}, key[2] = {seed, tag}, r[4];
    synth_philox(ctr, key, r);
    uint64_t x = ((uint64_t)r[0] << 32) | r[1];
    int32_t j = (int32_t)(x % (uint64_t)(i + 1));
    int32_t t = out[i]; out[i] = out[j]; out[j] = t;
  }
}

/* Round fp32 to bf16, nearest-even (inputs are finite). */
void synth_bf16_from_f32(const float* in, int64_t n, uint16_t* out) {
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i) {
    uint32_t u; memcpy(&u, &in[i], 4);
    u += 0x7FFFu + ((u >> 16) & 1u);
    out[i] = (uint16_t)(u >> 16);
  }
}

/* ---- storage-format rounding of drawn weights --------------------------- */

/* FP8 E4M3 (OCP): bias 7, 3 mantissa bits, max finite 448, no infinities.
 * Round to nearest even, saturating to +-448. */
static uint8_t gen_e4m3(float v) {
  uint8_t sign = (v < 0.0f) ? 0x80 : 0x00;
  double a = fabs((double)v);
  if (a >= 448.0) return sign | 0x7E;
  if (a == 0.0) return sign;
  int e = (int)floor(log2(a));
  if (e < -6) e = -6;
  /* make sure 2^e <= a for the normal range (log2 rounding guard) */
  if (e > -6 && ldexp(1.0, e) > a) e -= 1;
  if (ldexp(1.0, e + 1) <= a) e += 1;
  double step = ldexp(1.0, e - 3);
  double nq = rint(a / step);          /* exact division by a power of two */
  double val = nq * step;
  if (val >= 448.0) return sign | 0x7E;
  if (val < ldexp(1.0, -6)) {           /* subnormal: m * 2^-9 */
    int m = (int)(val / ldexp(1.0, -9));
    return sign | (uint8_t)m;
  }
  int ee = (int)floor(log2(val));
  if (ldexp(1.0, ee) > val) ee -= 1;
  if (ldexp(1.0, ee + 1) <= val) ee += 1;
  int m = (int)(val / ldexp(1.0, ee) * 8.0) - 8;
  return sign | (uint8_t)(((ee + 7) << 3) | m);
}

static double gen_e4m3_value(uint8_t q) {
  int s = q >> 7, e = (q >> 3) & 0xF, m = q & 7;
  double v = (e == 0) ? ldexp((double)m, -9) : ldexp(1.0 + m / 8.0, e - 7);
  return s ? -v : v;
}

/* FP4 E2M1: grid {0, .5, 1, 1.5, 2, 3, 4, 6}; nearest, ties to the even code,
 * saturating to +-6.  Returns a 4-bit code (bit 3 = sign). */
static uint8_t gen_e2m1(float v) {
  static const double grid[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};
  uint8_t sign = (v < 0.0f) ? 0x8 : 0x0;
  double a = fabs((double)v);
  int best = 0;
  double bd = a;
  for (int c = 1; c < 8; ++c) {
    double dd = fabs(a - grid[c]);
    if (dd < bd || (dd == bd && (c & 1) == 0 && (best & 1) == 1)) { bd = dd; best = c; }
  }
  if (best == 0) return 0; /* +0 */
  return sign | (uint8_t)best;
}

/* W [R][C] fp32 -> q [R][C] e4m3, s [R/128][C/128] fp32 with s = amax/448. */
void synth_quant_fp8_b128(const float* W, int32_t R, int32_t C, uint8_t* q, float* s) {
  int32_t RB = R / 128, CB = C / 128;
#pragma omp parallel for collapse(2) schedule(static)
  for (int32_t rb = 0; rb < RB; ++rb)
    for (int32_t cb = 0; cb < CB; ++cb) {
      float amax = 0.0f;
      for (int r = 0; r < 128; ++r)
        for (int c = 0; c < 128; ++c) {
          float a = fabsf(W[(int64_t)(rb * 128 + r) * C + cb * 128 + c]);
          if (a > amax) amax = a;
        }
      float sc = amax / 448.0f;
      s[rb * CB + cb] = sc;
      for (int r = 0; r < 128; ++r)
        for (int c = 0; c < 128; ++c) {
          int64_t i = (int64_t)(rb * 128 + r) * C + cb * 128 + c;
          q[i] = (sc == 0.0f) ? 0 : gen_e4m3(W[i] / sc);
        }
    }
}

/* W [R][C] fp32 -> NVFP4: s_t = amax(W)/(6*448); per 16 consecutive elements of
 * a row, s16 = e4m3(amax_blk / (6*s_t)); q = e2m1(w / (s16 * s_t)).
 * q packed two per byte along C, element 2j in the low nibble. */
void synth_quant_nvfp4(const float* W, int32_t R, int32_t C, uint8_t* qp, uint8_t* s16, float* s_t_out) {
  float amax = 0.0f;
  int64_t n = (int64_t)R * C;
  for (int64_t i = 0; i < n; ++i) { float a = fabsf(W[i]); if (a > amax) amax = a; }
  float s_t = amax / 2688.0f;
  *s_t_out = s_t;
  float denom = 6.0f * s_t;
  int32_t CB = C / 16;
#pragma omp parallel for schedule(static)
  for (int32_t r = 0; r < R; ++r) {
    for (int32_t cb = 0; cb < CB; ++cb) {
      const float* w = W + (int64_t)r * C + cb * 16;
      float ab = 0.0f;
      for (int j = 0; j < 16; ++j) { float a = fabsf(w[j]); if (a > ab) ab = a; }
      uint8_t sc = (denom == 0.0f) ? 0 : gen_e4m3(ab / denom);
      s16[(int64_t)r * CB + cb] = sc;
      float scale = (float)gen_e4m3_value(sc) * s_t;
      for (int j = 0; j < 16; j += 2) {
        uint8_t lo = (scale == 0.0f) ? 0 : gen_e2m1(w[j] / scale);
        uint8_t hi = (scale == 0.0f) ? 0 : gen_e2m1(w[j + 1] / scale);
        qp[(int64_t)r * (C / 2) + cb * 8 + j / 2] = (uint8_t)(lo | (hi << 4));
      }
    }
  }
}

/* W [R][C] fp32 -> MXFP4 (OCP Microscaling v1.0): per 32 consecutive elements
 * of a row one E8M0 scale code e (value 2^(e-127)) with e - 127 =
 * floor(log2(block amax)) - 2 clamped to [-127, 127] (an all-zero block gets
 * e = 127), and E2M1 codes of w / 2^(e-127), nearest with ties to even,
 * saturating at 6.  q packed two per byte along C, element 2j in the low
 * nibble; s [R][C/32]. */
void synth_quant_mxfp4(const float* W, int32_t R, int32_t C, uint8_t* qp, uint8_t* s32) {
  int32_t CB = C / 32;
#pragma omp parallel for schedule(static)
  for (int32_t r = 0; r < R; ++r) {
    for (int32_t cb = 0; cb < CB; ++cb) {
      const float* w = W + (int64_t)r * C + cb * 32;
      float ab = 0.0f;
      for (int j = 0; j < 32; ++j) { float a = fabsf(w[j]); if (a > ab) ab = a; }
      int e = 0;
      if (ab > 0.0f) {
        int ex;
        frexp((double)ab, &ex);             /* ab = m * 2^ex, m in [0.5, 1): floor(log2 ab) = ex - 1 */
        e = ex - 1 - 2;
        if (e < -127) e = -127;
        if (e > 127) e = 127;
      }
      s32[(int64_t)r * CB + cb] = (uint8_t)(e + 127);
      double X = ldexp(1.0, e);
      for (int j = 0; j < 32; j += 2) {
        uint8_t lo = gen_e2m1((float)(w[j] / X)), hi = gen_e2m1((float)(w[j + 1] / X));
        qp[(int64_t)r * (C / 2) + cb * 16 + j / 2] = (uint8_t)(lo | (hi << 4));
      }
    }
  }
}
