// Host-side SwiGLU expert FFN for the bandwidth-adaptive miss split.
//
// The pages' q* policy (freelamp.com FreeToken article, section 2.1
// "bandwidth-adaptive execution"; chenxutan.com FreeToken article, "choosing
// among the five MoE backends", `cpu` and `hybrid`) computes part of a step's
// missed experts on the host CPU, straight from the expert banks in host
// memory, while the rest cross PCIe to the GPU.  This file is that host
// computation: the same expert FFN as the GPU kernels (activation
// quantisation included), in fp32 on a pool of host threads, reading each
// weight row once for all of an expert's rows.  It is not a fallback: the
// library only runs it for the experts the split assigns to the host.
//
// Number formats: bf16 (upper half of an fp32), OCP FP8 E4M3 (bias 7, 3
// mantissa bits, subnormals m * 2^-9, max 448).  Weight rows of FP8 banks carry
// one fp32 scale per 128 x 128 block.
#include <atomic>
#include <cmath>
#include <condition_variable>
#include <cstdint>
#include <cstring>
#include <functional>
#include <immintrin.h>
#include <mutex>
#include <thread>
#include <vector>

#include "ftm.h"
#include "ftm_host_ffn.h"

namespace ftm {
namespace {

// ---- number formats ---------------------------------------------------------
inline float bits_f32(uint32_t u) {
  float f;
  std::memcpy(&f, &u, 4);
  return f;
}

inline uint32_t f32_bits(float f) {
  uint32_t u;
  std::memcpy(&u, &f, 4);
  return u;
}

inline float bf16_value(uint16_t v) { return bits_f32(static_cast<uint32_t>(v) << 16); }

// fp32 -> bf16, round to nearest, ties to even (NaN kept quiet).
inline uint16_t bf16_round(float f) {
  const uint32_t u = f32_bits(f);
  if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu)) return static_cast<uint16_t>((u >> 16) | 0x40u);
  return static_cast<uint16_t>((u + 0x7FFFu + ((u >> 16) & 1u)) >> 16);
}

// Nearest E4M3 value of a >= 0 (ties to the even mantissa), saturating at 448.
// Normal range: the quantum is 2^(e-3) for a in [2^e, 2^(e+1)); below 2^-6 the
// subnormal quantum 2^-9.  rint rounds half to even, and the integer it
// returns is 8 + mantissa (normal) or the mantissa (subnormal), so even
// integers are even codes.
inline float e4m3_round(float a) {
  if (!(a < 448.0f)) return 448.0f;
  if (a < 0x1p-6f) return std::rint(a * 512.0f) * 0x1p-9f;
  int e;
  std::frexp(a, &e);              // a = f * 2^e, f in [0.5, 1): a in [2^(e-1), 2^e)
  const float quantum = std::ldexp(1.0f, e - 4);
  return std::fmin(std::rint(a / quantum) * quantum, 448.0f);
}

// FP8 activation quantisation of one row, in place: groups of 128, scale
// amax / 448 (fp32), v <- e4m3(v / s) * s; an all-zero group stays zero.
void quant_fp8_row(float* v, int K) {
  for (int g = 0; g < K; g += 128) {
    float amax = 0.0f;
    for (int j = 0; j < 128; ++j) amax = std::fmax(amax, std::fabs(v[g + j]));
    const float s = amax / 448.0f;
    for (int j = 0; j < 128; ++j) {
      if (s == 0.0f) { v[g + j] = 0.0f; continue; }
      const float q = v[g + j] / s;
      const float r = e4m3_round(std::fabs(q));
      v[g + j] = (q < 0.0f ? -r : r) * s;
    }
  }
}

// E2M1 magnitudes by code (1 sign, 2 exponent bits with bias 1, 1 mantissa bit).
constexpr float kE2m1[8] = {0.0f, 0.5f, 1.0f, 1.5f, 2.0f, 3.0f, 4.0f, 6.0f};

// Nearest E2M1 magnitude of a >= 0, ties to the even code, saturating at 6.
// The midpoints between neighbours are 0.25, 0.75, 1.25, 1.75, 2.5, 3.5 and 5;
// at a midpoint the even code (0, 1, 1, 2, 2, 4, 4) wins.
inline float e2m1_round(float a) {
  if (a <= 0.25f) return 0.0f;
  if (a < 0.75f) return 0.5f;
  if (a <= 1.25f) return 1.0f;
  if (a < 1.75f) return 1.5f;
  if (a <= 2.5f) return 2.0f;
  if (a < 3.5f) return 3.0f;
  if (a <= 5.0f) return 4.0f;
  return 6.0f;
}

// NVFP4 activation quantisation of one row, in place: groups of 16 with the
// per-tensor global scale g: s16 = e4m3(amax / (6 g)), u = s16 * g,
// v <- e2m1(v / u) * u (a group with u = 0 becomes zero).
void quant_nvfp4_row(float* v, int K, float g) {
  const float six_g = 6.0f * g;
  for (int b = 0; b < K; b += 16) {
    float amax = 0.0f;
    for (int j = 0; j < 16; ++j) amax = std::fmax(amax, std::fabs(v[b + j]));
    const float u = e4m3_round(amax / six_g) * g;
    for (int j = 0; j < 16; ++j) {
      if (u == 0.0f) { v[b + j] = 0.0f; continue; }
      const float q = v[b + j] / u;
      const float r = e2m1_round(std::fabs(q));
      v[b + j] = (q < 0.0f ? -r : r) * u;
    }
  }
}

// MXFP4 activation quantisation of one row, in place (OCP MX): groups of 32
// share X = 2^e, e = floor(log2 amax) - 2 clamped to [-127, 127] (floor(log2)
// read exactly from frexp); v <- e2m1(v / X) * X.  An all-zero group stays zero.
void quant_mx_row(float* v, int K) {
  for (int b = 0; b < K; b += 32) {
    float amax = 0.0f;
    for (int j = 0; j < 32; ++j) amax = std::fmax(amax, std::fabs(v[b + j]));
    if (amax == 0.0f) continue;
    int k;
    std::frexp(amax, &k);                 // amax in [2^(k-1), 2^k)
    int e = (k - 1) - 2;
    e = e < -127 ? -127 : e > 127 ? 127 : e;
    const double X = std::ldexp(1.0, e);  // 2^-127 is below fp32's range: scale in double
    for (int j = 0; j < 32; ++j) {
      const float q = static_cast<float>(v[b + j] / X);
      const float r = e2m1_round(std::fabs(q));
      v[b + j] = static_cast<float>((q < 0.0f ? -r : r) * X);
    }
  }
}

// Per-group fp32 scales of one weight row of an NVFP4 / MXFP4 bank, read
// through the 512-byte chunk layout: chunk (row block rb, column block kb) of
// four scale groups at (rb * nkb + kb) * 512, the scale of local row r for its
// group j at byte (r % 32) * 16 + (r / 32) * 4 + j.  `r_in_block` and `rb` are
// the row's place in that layout (gate/up rows in paired order).  NVFP4:
// e4m3(code) * s_t; MXFP4: 2^(code - 127).
void fp4_row_scales(const uint8_t* chunks, int rb, int r_in_block, int K, bool mx, float s_t, float* out) {
  const int group = mx ? 32 : 16;
  const int ng = K / group, nkb = ng / 4;
  const uint8_t* base = chunks + static_cast<size_t>(rb) * nkb * 512 + (r_in_block % 32) * 16 + (r_in_block / 32) * 4;
  for (int gi = 0; gi < ng; ++gi) {
    const uint8_t c = base[static_cast<size_t>(gi / 4) * 512 + gi % 4];
    if (mx) out[gi] = static_cast<float>(std::ldexp(1.0, static_cast<int>(c) - 127));
    else {
      const uint32_t em = c & 0x7Fu;
      const float mag = (em >> 3) ? bits_f32((em << 20) + (120u << 23)) : static_cast<float>(em) * 0x1p-9f;
      out[gi] = ((c & 0x80u) ? -mag : mag) * s_t;
    }
  }
}

// ---- dot products of one weight row with n activation rows ---------------------
// Eight partial sums per row so the compiler can keep them in one vector.
__attribute__((target_clones("arch=haswell", "default")))
void dot_f32(const float* w, int K, const float* x, int ldx, int n, float* out) {
  for (int r = 0; r < n; ++r) {
    const float* xr = x + static_cast<size_t>(r) * ldx;
    float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    for (int c = 0; c < K; c += 8)
      for (int l = 0; l < 8; ++l) acc[l] += w[c + l] * xr[c + l];
    out[r] = ((acc[0] + acc[1]) + (acc[2] + acc[3])) + ((acc[4] + acc[5]) + (acc[6] + acc[7]));
  }
}

// Weight rows converted 128 columns at a time into a small buffer, then dotted
// with every activation row; FP8 blocks are scaled once per block and row.
__attribute__((target_clones("arch=haswell", "default")))
void dot_block(const float* wb, const float* x, int ldx, int n, float scale, float* out) {
  for (int r = 0; r < n; ++r) {
    const float* xr = x + static_cast<size_t>(r) * ldx;
    float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    for (int c = 0; c < 128; c += 8)
      for (int l = 0; l < 8; ++l) acc[l] += wb[c + l] * xr[c + l];
    out[r] += scale * (((acc[0] + acc[1]) + (acc[2] + acc[3])) + ((acc[4] + acc[5]) + (acc[6] + acc[7])));
  }
}

__attribute__((target_clones("arch=haswell", "default")))
void convert_bf16(const uint16_t* w, float* out) {
  for (int c = 0; c < 128; ++c) out[c] = bits_f32(static_cast<uint32_t>(w[c]) << 16);
}

// E4M3 code -> value.  Normal codes (exponent field 1..15) map onto the fp32
// bit pattern with the exponent rebased from 7 to 127 and the 3 mantissa bits
// on top of fp32's 23; exponent field 0 is m * 2^-9.  (Codes 0x7F / 0xFF, NaN,
// do not occur in weights and decode as 480.)
__attribute__((target_clones("arch=haswell", "default")))
void convert_e4m3(const uint8_t* w, float* out) {
  for (int c = 0; c < 128; ++c) {
    const uint32_t b = w[c], em = b & 0x7Fu;
    const float normal = bits_f32((em << 20) + (120u << 23));
    const float sub = static_cast<float>(em) * 0x1p-9f;
    const float v = (em >> 3) ? normal : sub;
    out[c] = bits_f32(f32_bits(v) | ((b & 0x80u) << 24));
  }
}

// ---- AVX2 + FMA path (chosen at run time) ----------------------------------------
// 8 weights per vector: E4M3 codes widened to 32 bits and rebuilt as fp32 with
// the same bit rule as convert_e4m3 (normal codes by integer shift and add,
// exponent field 0 as m * 2^-9 by a convert and multiply, then the sign);
// bf16 by a 16-bit shift.
__attribute__((target("avx2,fma"))) inline __m256 e4m3x8(const uint8_t* p) {
  const __m256i v = _mm256_cvtepu8_epi32(_mm_loadl_epi64(reinterpret_cast<const __m128i*>(p)));
  const __m256i em = _mm256_and_si256(v, _mm256_set1_epi32(0x7F));
  const __m256 normal =
      _mm256_castsi256_ps(_mm256_add_epi32(_mm256_slli_epi32(em, 20), _mm256_set1_epi32(120 << 23)));
  const __m256 sub = _mm256_mul_ps(_mm256_cvtepi32_ps(em), _mm256_set1_ps(0x1p-9f));
  const __m256 isn = _mm256_castsi256_ps(_mm256_cmpgt_epi32(em, _mm256_set1_epi32(7)));
  const __m256 val = _mm256_blendv_ps(sub, normal, isn);
  const __m256i sign = _mm256_slli_epi32(_mm256_and_si256(v, _mm256_set1_epi32(0x80)), 24);
  return _mm256_or_ps(val, _mm256_castsi256_ps(sign));
}

// 32 E4M3 codes to fp32 through their exact fp16 images (every E4M3 value is
// an fp16 value).  Normal codes (exponent field 1..15): fp16 = (code & 0x7F) << 7
// plus 8 << 10 (the exponent rebased from 7 to 15), so the fp16 high byte is
// ((code >> 1) & 0x3F) + 0x20 and the low byte (code & 1) << 7.  Exponent field
// 0 (m * 2^-9, m = code & 7) has a low byte of 0 and a high byte from an
// 8-entry table: 0, 2^-9, 2^-8, 1.5 2^-8, 2^-7, 1.25 2^-7, 1.5 2^-7, 1.75 2^-7.
// The sign bit carries over.  Bytes are interleaved into fp16 words and
// widened with F16C; out[0..3] hold elements 0-7, 8-15, 16-23, 24-31.
__attribute__((target("avx2,fma,f16c"))) inline void e4m3x32(const uint8_t* p, __m256 out[4]) {
  const __m256i b = _mm256_loadu_si256(reinterpret_cast<const __m256i*>(p));
  const __m256i sub_hi = _mm256_setr_epi8(0x00, 0x18, 0x1C, 0x1E, 0x20, 0x21, 0x22, 0x23, 0, 0, 0, 0, 0, 0, 0, 0,
                                          0x00, 0x18, 0x1C, 0x1E, 0x20, 0x21, 0x22, 0x23, 0, 0, 0, 0, 0, 0, 0, 0);
  const __m256i sign = _mm256_and_si256(b, _mm256_set1_epi8(static_cast<char>(0x80)));
  const __m256i hi_n = _mm256_add_epi8(_mm256_and_si256(_mm256_srli_epi16(b, 1), _mm256_set1_epi8(0x3F)),
                                       _mm256_set1_epi8(0x20));
  const __m256i hi_s = _mm256_shuffle_epi8(sub_hi, _mm256_and_si256(b, _mm256_set1_epi8(0x07)));
  const __m256i is_sub = _mm256_cmpeq_epi8(_mm256_and_si256(b, _mm256_set1_epi8(0x78)), _mm256_setzero_si256());
  const __m256i hi = _mm256_or_si256(_mm256_blendv_epi8(hi_n, hi_s, is_sub), sign);
  const __m256i lo = _mm256_andnot_si256(is_sub, _mm256_slli_epi16(_mm256_and_si256(b, _mm256_set1_epi8(1)), 7));
  const __m256i w0 = _mm256_unpacklo_epi8(lo, hi);   // elements 0-7 | 16-23
  const __m256i w1 = _mm256_unpackhi_epi8(lo, hi);   // elements 8-15 | 24-31
  out[0] = _mm256_cvtph_ps(_mm256_castsi256_si128(w0));
  out[1] = _mm256_cvtph_ps(_mm256_castsi256_si128(w1));
  out[2] = _mm256_cvtph_ps(_mm256_extracti128_si256(w0, 1));
  out[3] = _mm256_cvtph_ps(_mm256_extracti128_si256(w1, 1));
}

__attribute__((target("avx2,fma"))) inline __m256 bf16x8(const uint8_t* p) {
  const __m256i v = _mm256_cvtepu16_epi32(_mm_loadu_si128(reinterpret_cast<const __m128i*>(p)));
  return _mm256_castsi256_ps(_mm256_slli_epi32(v, 16));
}

__attribute__((target("avx2,fma"))) inline float hsum8(__m256 v) {
  const __m128 s = _mm_add_ps(_mm256_castps256_ps128(v), _mm256_extractf128_ps(v, 1));
  const __m128 t = _mm_add_ps(s, _mm_movehl_ps(s, s));
  return _mm_cvtss_f32(_mm_add_ss(t, _mm_shuffle_ps(t, t, 1)));
}

const bool g_f16c = __builtin_cpu_supports("avx2") && __builtin_cpu_supports("fma") &&
                    __builtin_cpu_supports("f16c");

// FP8 rows, NR (1..4) activation rows per pass: 32 weights decoded at a time,
// four independent accumulators per row, one hsum and scale per 128-block.
template <int NR>
__attribute__((target("avx2,fma,f16c"))) void dot_rows_fp8_avx2(const uint8_t* w, const float* sc, int K,
                                                                const float* x, int ldx, float* out) {
  float tot[NR] = {};
  for (int c0 = 0; c0 < K; c0 += 128) {
    __m256 a[NR][4];
    for (int r = 0; r < NR; ++r)
      for (int v = 0; v < 4; ++v) a[r][v] = _mm256_setzero_ps();
    for (int c = c0; c < c0 + 128; c += 32) {
      __m256 wv[4];
      e4m3x32(w + c, wv);
      for (int r = 0; r < NR; ++r)
        for (int v = 0; v < 4; ++v)
          a[r][v] = _mm256_fmadd_ps(wv[v], _mm256_loadu_ps(x + static_cast<size_t>(r) * ldx + c + 8 * v), a[r][v]);
    }
    for (int r = 0; r < NR; ++r)
      tot[r] += sc[c0 / 128] * hsum8(_mm256_add_ps(_mm256_add_ps(a[r][0], a[r][1]), _mm256_add_ps(a[r][2], a[r][3])));
  }
  for (int r = 0; r < NR; ++r) out[r] = tot[r];
}

// NR (1..4) activation rows per pass: each block of 128 weights is decoded
// once and multiplied into every row's accumulators in registers, two
// independent accumulators per row so consecutive FMAs do not wait on each
// other.
template <bool FP8, int NR>
__attribute__((target("avx2,fma"))) void dot_rows_avx2(const uint8_t* w, const float* sc, int K, const float* x,
                                                       int ldx, float* out) {
  constexpr int kEb = FP8 ? 1 : 2;   // bytes per weight
  float tot[NR] = {};
  for (int c0 = 0; c0 < K; c0 += 128) {
    __m256 a0[NR], a1[NR];
    for (int r = 0; r < NR; ++r) a0[r] = a1[r] = _mm256_setzero_ps();
    for (int c = c0; c < c0 + 128; c += 16) {
      const __m256 w0 = FP8 ? e4m3x8(w + c) : bf16x8(w + static_cast<size_t>(c) * kEb);
      const __m256 w1 = FP8 ? e4m3x8(w + c + 8) : bf16x8(w + static_cast<size_t>(c + 8) * kEb);
      for (int r = 0; r < NR; ++r) {
        a0[r] = _mm256_fmadd_ps(w0, _mm256_loadu_ps(x + static_cast<size_t>(r) * ldx + c), a0[r]);
        a1[r] = _mm256_fmadd_ps(w1, _mm256_loadu_ps(x + static_cast<size_t>(r) * ldx + c + 8), a1[r]);
      }
    }
    const float s = FP8 ? sc[c0 / 128] : 1.0f;
    for (int r = 0; r < NR; ++r) tot[r] += s * hsum8(_mm256_add_ps(a0[r], a1[r]));
  }
  for (int r = 0; r < NR; ++r) out[r] = tot[r];
}

template <bool FP8>
void dot_row_avx2(const uint8_t* w, const float* sc, int K, const float* x, int ldx, int n, float* out) {
  if (FP8 && g_f16c) {
    for (int r0 = 0; r0 < n; r0 += 4) {
      const float* xr = x + static_cast<size_t>(r0) * ldx;
      switch (n - r0 < 4 ? n - r0 : 4) {
        case 1: dot_rows_fp8_avx2<1>(w, sc, K, xr, ldx, out + r0); break;
        case 2: dot_rows_fp8_avx2<2>(w, sc, K, xr, ldx, out + r0); break;
        case 3: dot_rows_fp8_avx2<3>(w, sc, K, xr, ldx, out + r0); break;
        default: dot_rows_fp8_avx2<4>(w, sc, K, xr, ldx, out + r0); break;
      }
    }
    return;
  }
  for (int r0 = 0; r0 < n; r0 += 4) {
    const float* xr = x + static_cast<size_t>(r0) * ldx;
    switch (n - r0 < 4 ? n - r0 : 4) {
      case 1: dot_rows_avx2<FP8, 1>(w, sc, K, xr, ldx, out + r0); break;
      case 2: dot_rows_avx2<FP8, 2>(w, sc, K, xr, ldx, out + r0); break;
      case 3: dot_rows_avx2<FP8, 3>(w, sc, K, xr, ldx, out + r0); break;
      default: dot_rows_avx2<FP8, 4>(w, sc, K, xr, ldx, out + r0); break;
    }
  }
}

// 8 packed E2M1 codes (4 bytes, element 2j in the low nibble of byte j): lane l
// takes bits 4l..4l+3 of the little-endian word, the magnitude from the
// 8-entry table, the sign from the code's top bit.
__attribute__((target("avx2,fma"))) inline __m256 e2m1x8(const uint8_t* p) {
  uint32_t word;
  std::memcpy(&word, p, 4);
  const __m256i nib = _mm256_and_si256(
      _mm256_srlv_epi32(_mm256_set1_epi32(static_cast<int>(word)), _mm256_setr_epi32(0, 4, 8, 12, 16, 20, 24, 28)),
      _mm256_set1_epi32(0xF));
  const __m256 mag = _mm256_permutevar8x32_ps(_mm256_loadu_ps(kE2m1), _mm256_and_si256(nib, _mm256_set1_epi32(7)));
  const __m256i sign = _mm256_slli_epi32(_mm256_and_si256(nib, _mm256_set1_epi32(8)), 28);
  return _mm256_or_ps(mag, _mm256_castsi256_ps(sign));
}

// FP4 rows: each group of `group` weights (16 NVFP4, 32 MXFP4) decoded and
// multiplied by its scale once, then into every row's accumulators.
template <int NR>
__attribute__((target("avx2,fma"))) void dot_rows_fp4_avx2(const uint8_t* w, const float* sc, int K, int group,
                                                           const float* x, int ldx, float* out) {
  __m256 a0[NR], a1[NR];
  for (int r = 0; r < NR; ++r) a0[r] = a1[r] = _mm256_setzero_ps();
  for (int c = 0; c < K; c += 16) {
    const __m256 s = _mm256_set1_ps(sc[c / group]);
    const __m256 w0 = _mm256_mul_ps(e2m1x8(w + c / 2), s);
    const __m256 w1 = _mm256_mul_ps(e2m1x8(w + c / 2 + 4), s);
    for (int r = 0; r < NR; ++r) {
      a0[r] = _mm256_fmadd_ps(w0, _mm256_loadu_ps(x + static_cast<size_t>(r) * ldx + c), a0[r]);
      a1[r] = _mm256_fmadd_ps(w1, _mm256_loadu_ps(x + static_cast<size_t>(r) * ldx + c + 8), a1[r]);
    }
  }
  for (int r = 0; r < NR; ++r) out[r] = hsum8(_mm256_add_ps(a0[r], a1[r]));
}

void dot_row_fp4_avx2(const uint8_t* w, const float* sc, int K, int group, const float* x, int ldx, int n,
                      float* out) {
  for (int r0 = 0; r0 < n; r0 += 4) {
    const float* xr = x + static_cast<size_t>(r0) * ldx;
    switch (n - r0 < 4 ? n - r0 : 4) {
      case 1: dot_rows_fp4_avx2<1>(w, sc, K, group, xr, ldx, out + r0); break;
      case 2: dot_rows_fp4_avx2<2>(w, sc, K, group, xr, ldx, out + r0); break;
      case 3: dot_rows_fp4_avx2<3>(w, sc, K, group, xr, ldx, out + r0); break;
      default: dot_rows_fp4_avx2<4>(w, sc, K, group, xr, ldx, out + r0); break;
    }
  }
}

const bool g_avx2 = __builtin_cpu_supports("avx2") && __builtin_cpu_supports("fma");

// out[r] = sum_c W[row][c] * x[r][c] for one row of a weight matrix with K
// columns.  `sc` = the row's fp32 scales: FP8 one per 128-column block, NVFP4
// one per 16 columns (s_t included), MXFP4 one per 32.
void dot_row(int wdtype, const uint8_t* wrow, const float* sc, int K, const float* x, int ldx, int n, float* out) {
  if (wdtype == FTM_NVFP4 || wdtype == FTM_MXFP4) {
    const int group = wdtype == FTM_NVFP4 ? 16 : 32;
    if (g_avx2) {
      dot_row_fp4_avx2(wrow, sc, K, group, x, ldx, n, out);
      return;
    }
    for (int r = 0; r < n; ++r) {
      const float* xr = x + static_cast<size_t>(r) * ldx;
      float acc = 0.0f;
      for (int c = 0; c < K; ++c) {
        const uint8_t b = wrow[c / 2];
        const uint8_t nib = (c & 1) ? (b >> 4) : (b & 15);
        const float v = (nib & 8) ? -kE2m1[nib & 7] : kE2m1[nib & 7];
        acc += v * sc[c / group] * xr[c];
      }
      out[r] = acc;
    }
    return;
  }
  if (wdtype == FTM_F32) {
    dot_f32(reinterpret_cast<const float*>(wrow), K, x, ldx, n, out);
    return;
  }
  if (g_avx2) {
    if (wdtype == FTM_FP8_E4M3_B128) dot_row_avx2<true>(wrow, sc, K, x, ldx, n, out);
    else dot_row_avx2<false>(wrow, sc, K, x, ldx, n, out);
    return;
  }
  for (int r = 0; r < n; ++r) out[r] = 0.0f;
  alignas(32) float wb[128];
  for (int c = 0; c < K; c += 128) {
    if (wdtype == FTM_BF16) convert_bf16(reinterpret_cast<const uint16_t*>(wrow) + c, wb);
    else convert_e4m3(wrow + c, wb);
    dot_block(wb, x + c, ldx, n, wdtype == FTM_FP8_E4M3_B128 ? sc[c / 128] : 1.0f, out);
  }
}

// ---- a fork-join pool of host threads ------------------------------------------
class Pool {
 public:
  ~Pool() {
    {
      std::lock_guard<std::mutex> g(m_);
      stop_ = true;
      ++gen_;
    }
    cv_.notify_all();
    for (auto& t : th_) t.join();
  }

  // body(i) for i in [0, n), over `threads` threads (the caller is one of them).
  void run(int threads, int64_t n, const std::function<void(int64_t)>& body) {
    if (n <= 0) return;
    if (threads < 1) threads = 1;
    if (threads > n) threads = static_cast<int>(n);
    std::lock_guard<std::mutex> one(run_);
    grow(threads - 1);
    {
      std::lock_guard<std::mutex> g(m_);
      body_ = &body;
      n_ = n;
      next_.store(0);
      workers_ = threads - 1;
      pending_ = threads - 1;
      ++gen_;
    }
    cv_.notify_all();
    drain();
    std::unique_lock<std::mutex> g(m_);
    done_.wait(g, [&] { return pending_ == 0; });
    body_ = nullptr;
  }

 private:
  void grow(int want) {
    while (static_cast<int>(th_.size()) < want) {
      // a new worker starts from the generation current now (run() bumps it
      // after grow()), so it cannot miss the run it was created for
      const int id = static_cast<int>(th_.size());
      const uint64_t g0 = gen_;
      th_.emplace_back([this, id, g0] { loop(id, g0); });
    }
  }

  void drain() {
    for (;;) {
      const int64_t i = next_.fetch_add(1);
      if (i >= n_) return;
      (*body_)(i);
    }
  }

  void loop(int id, uint64_t seen) {
    for (;;) {
      std::unique_lock<std::mutex> g(m_);
      cv_.wait(g, [&] { return gen_ != seen; });
      seen = gen_;
      if (stop_) return;
      const bool mine = id < workers_;
      g.unlock();
      if (!mine) continue;
      drain();
      g.lock();
      if (--pending_ == 0) done_.notify_one();
    }
  }

  std::mutex run_, m_;
  std::condition_variable cv_, done_;
  std::vector<std::thread> th_;
  const std::function<void(int64_t)>* body_ = nullptr;
  int64_t n_ = 0;
  std::atomic<int64_t> next_{0};
  int workers_ = 0, pending_ = 0;
  uint64_t gen_ = 0;
  bool stop_ = false;
};

Pool& pool() {
  static Pool p;
  return p;
}

constexpr int kRowsPerItem = 16;   // weight rows per work item

}  // namespace

size_t host_ffn_scratch_bytes(const ftm_layer_desc* L, int64_t rows) {
  return static_cast<size_t>(rows) * (L->d + L->I) * sizeof(float);
}

int host_ffn_supported(int wdtype) {
  return wdtype >= FTM_F32 && wdtype <= FTM_MXFP4;
}

int host_threads(int threads) {
  if (threads > 0) return threads;
  const unsigned hc = std::thread::hardware_concurrency();
  return hc ? static_cast<int>(hc) : 1;
}

// Every group's rows through gate/up, SwiGLU and down.  Activations are bf16
// (fp32 for FTM_F32 layers), one row pointer per row.  Quantised layers
// quantise x and h before each contraction as the GPU kernels do: FP8 per 128
// (amax / 448), NVFP4 per 16 with the global scales act_scale = {gx, gh}
// (NULL: 1, 1), MXFP4 per 32 (E8M0).
void host_ffn_groups(const ftm_layer_desc* L, const ftm_bank_layout* bl, const HostGroup* groups, int ng,
                     const float* act_scale, float* scratch, int threads) {
  const int d = L->d, I = L->I, wd = L->wdtype;
  const bool f32 = wd == FTM_F32, fp4 = wd == FTM_NVFP4 || wd == FTM_MXFP4, mx = wd == FTM_MXFP4;
  const size_t elt = f32 ? 4 : 2;
  auto row_bytes = [&](int K) -> size_t {
    return wd == FTM_F32 ? 4u * K : wd == FTM_BF16 ? 2u * K : fp4 ? K / 2u : static_cast<size_t>(K);
  };
  const size_t wrow_gu = row_bytes(d), wrow_d = row_bytes(I);
  const float gx = act_scale ? act_scale[0] : 1.0f, gh = act_scale ? act_scale[1] : 1.0f;
  auto quant = [&](float* v, int K, float g) {
    if (wd == FTM_FP8_E4M3_B128) quant_fp8_row(v, K);
    else if (wd == FTM_NVFP4) quant_nvfp4_row(v, K, g);
    else if (wd == FTM_MXFP4) quant_mx_row(v, K);
  };
  // NVFP4 per-tensor weight scales {gate, up, down}
  auto s_t = [&](const HostGroup& G, int which) -> float {
    if (wd != FTM_NVFP4) return 1.0f;
    float v;
    std::memcpy(&v, G.bank + bl->s_t_off + 4 * which, 4);
    return v;
  };
  std::vector<int64_t> row0(ng + 1, 0);
  for (int g = 0; g < ng; ++g) row0[g + 1] = row0[g] + groups[g].n;
  const int64_t N = row0[ng];
  if (N == 0) return;
  float* xs = scratch;                                 // [N][d]
  float* hs = scratch + static_cast<size_t>(N) * d;    // [N][I]
  const int nt = host_threads(threads);
  // 1. activations to fp32 (quantised for FP8 layers)
  std::vector<std::pair<int, int>> rows(N);
  for (int g = 0; g < ng; ++g)
    for (int r = 0; r < groups[g].n; ++r) rows[row0[g] + r] = {g, r};
  pool().run(nt, N, [&](int64_t i) {
    const HostGroup& G = groups[rows[i].first];
    const uint8_t* src = G.x[rows[i].second];
    float* dst = xs + static_cast<size_t>(i) * d;
    if (f32) std::memcpy(dst, src, sizeof(float) * d);
    else
      for (int c = 0; c < d; ++c) dst[c] = bf16_value(reinterpret_cast<const uint16_t*>(src)[c]);
    quant(dst, d, gx);
  });
  // 2. gate/up + SwiGLU: items of kRowsPerItem intermediate rows of one group
  const int ib = (I + kRowsPerItem - 1) / kRowsPerItem;
  pool().run(nt, static_cast<int64_t>(ng) * ib, [&](int64_t it) {
    const int g = static_cast<int>(it / ib), i0 = static_cast<int>(it % ib) * kRowsPerItem;
    const HostGroup& G = groups[g];
    const int n = G.n;
    if (n == 0) return;
    const uint8_t* wgu = G.bank + bl->w_gu_off;
    const float* sgu = reinterpret_cast<const float*>(G.bank + bl->s_gu_off);
    const float* x = xs + static_cast<size_t>(row0[g]) * d;
    std::vector<float> gv(n), uv(n), gs(fp4 ? d / 16 : 0), us(fp4 ? d / 16 : 0);
    const float st_g = s_t(G, 0), st_u = s_t(G, 1);
    for (int i = i0; i < i0 + kRowsPerItem && i < I; ++i) {
      const int up = I + i;
      const float* sg = sgu + static_cast<size_t>(i / 128) * (d / 128);
      const float* su = sgu + static_cast<size_t>(up / 128) * (d / 128);
      if (fp4) {   // paired order: block i / 64 holds gate rows then the same up rows
        fp4_row_scales(G.bank + bl->s_gu_off, i / 64, i % 64, d, mx, st_g, gs.data());
        fp4_row_scales(G.bank + bl->s_gu_off, i / 64, 64 + i % 64, d, mx, st_u, us.data());
        sg = gs.data();
        su = us.data();
      }
      dot_row(wd, wgu + static_cast<size_t>(i) * wrow_gu, sg, d, x, d, n, gv.data());
      dot_row(wd, wgu + static_cast<size_t>(up) * wrow_gu, su, d, x, d, n, uv.data());
      for (int r = 0; r < n; ++r) {
        const float gg = gv[r];
        hs[static_cast<size_t>(row0[g] + r) * I + i] = gg / (1.0f + std::exp(-gg)) * uv[r];
      }
    }
  });
  if (wd != FTM_F32 && wd != FTM_BF16)
    pool().run(nt, N, [&](int64_t i) { quant(hs + static_cast<size_t>(i) * I, I, gh); });
  // 3. down projection, written straight to each row's output
  const int jb = (d + kRowsPerItem - 1) / kRowsPerItem;
  pool().run(nt, static_cast<int64_t>(ng) * jb, [&](int64_t it) {
    const int g = static_cast<int>(it / jb), j0 = static_cast<int>(it % jb) * kRowsPerItem;
    const HostGroup& G = groups[g];
    const int n = G.n;
    if (n == 0) return;
    const uint8_t* wdn = G.bank + bl->w_d_off;
    const float* sd = reinterpret_cast<const float*>(G.bank + bl->s_d_off);
    const float* h = hs + static_cast<size_t>(row0[g]) * I;
    std::vector<float> yv(n), ds(fp4 ? I / 16 : 0);
    const float st_d = s_t(G, 2);
    for (int j = j0; j < j0 + kRowsPerItem && j < d; ++j) {
      const float* sj = sd + static_cast<size_t>(j / 128) * (I / 128);
      if (fp4) {
        fp4_row_scales(G.bank + bl->s_d_off, j / 128, j % 128, I, mx, st_d, ds.data());
        sj = ds.data();
      }
      dot_row(wd, wdn + static_cast<size_t>(j) * wrow_d, sj, I, h, I, n, yv.data());
      for (int r = 0; r < n; ++r) {
        uint8_t* dst = G.y[r] + static_cast<size_t>(j) * elt;
        if (f32) std::memcpy(dst, &yv[r], 4);
        else {
          const uint16_t b = bf16_round(yv[r]);
          std::memcpy(dst, &b, 2);
        }
      }
    }
  });
}

}  // namespace ftm
