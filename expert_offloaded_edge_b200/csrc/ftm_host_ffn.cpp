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

__attribute__((target("avx2,fma"))) inline __m256 bf16x8(const uint8_t* p) {
  const __m256i v = _mm256_cvtepu16_epi32(_mm_loadu_si128(reinterpret_cast<const __m128i*>(p)));
  return _mm256_castsi256_ps(_mm256_slli_epi32(v, 16));
}

__attribute__((target("avx2,fma"))) inline float hsum8(__m256 v) {
  const __m128 s = _mm_add_ps(_mm256_castps256_ps128(v), _mm256_extractf128_ps(v, 1));
  const __m128 t = _mm_add_ps(s, _mm_movehl_ps(s, s));
  return _mm_cvtss_f32(_mm_add_ss(t, _mm_shuffle_ps(t, t, 1)));
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

const bool g_avx2 = __builtin_cpu_supports("avx2") && __builtin_cpu_supports("fma");

// out[r] = sum_c W[row][c] * x[r][c] for one row of a weight matrix with K
// columns.  `sc` = the row's fp32 block scales (FP8), one per 128 columns.
void dot_row(int wdtype, const uint8_t* wrow, const float* sc, int K, const float* x, int ldx, int n, float* out) {
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
  return wdtype == FTM_F32 || wdtype == FTM_BF16 || wdtype == FTM_FP8_E4M3_B128;
}

int host_threads(int threads) {
  if (threads > 0) return threads;
  const unsigned hc = std::thread::hardware_concurrency();
  return hc ? static_cast<int>(hc) : 1;
}

// Every group's rows through gate/up, SwiGLU and down.  Activations are bf16
// (fp32 for FTM_F32 layers), one row pointer per row; FP8 layers quantise x and
// h per 128-group before each contraction, as the GPU kernels do.
void host_ffn_groups(const ftm_layer_desc* L, const ftm_bank_layout* bl, const HostGroup* groups, int ng,
                     float* scratch, int threads) {
  const int d = L->d, I = L->I, wd = L->wdtype;
  const bool f32 = wd == FTM_F32;
  const size_t elt = f32 ? 4 : 2;
  const size_t wrow_gu = static_cast<size_t>(d) * (wd == FTM_F32 ? 4 : wd == FTM_BF16 ? 2 : 1);
  const size_t wrow_d = static_cast<size_t>(I) * (wd == FTM_F32 ? 4 : wd == FTM_BF16 ? 2 : 1);
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
    if (wd == FTM_FP8_E4M3_B128) quant_fp8_row(dst, d);
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
    std::vector<float> gv(n), uv(n);
    for (int i = i0; i < i0 + kRowsPerItem && i < I; ++i) {
      const int up = I + i;
      dot_row(wd, wgu + static_cast<size_t>(i) * wrow_gu, sgu + static_cast<size_t>(i / 128) * (d / 128), d, x, d, n,
              gv.data());
      dot_row(wd, wgu + static_cast<size_t>(up) * wrow_gu, sgu + static_cast<size_t>(up / 128) * (d / 128), d, x, d,
              n, uv.data());
      for (int r = 0; r < n; ++r) {
        const float gg = gv[r];
        hs[static_cast<size_t>(row0[g] + r) * I + i] = gg / (1.0f + std::exp(-gg)) * uv[r];
      }
    }
  });
  if (wd == FTM_FP8_E4M3_B128)
    pool().run(nt, N, [&](int64_t i) { quant_fp8_row(hs + static_cast<size_t>(i) * I, I); });
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
    std::vector<float> yv(n);
    for (int j = j0; j < j0 + kRowsPerItem && j < d; ++j) {
      dot_row(wd, wdn + static_cast<size_t>(j) * wrow_d, sd + static_cast<size_t>(j / 128) * (I / 128), I, h, I, n,
              yv.data());
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
