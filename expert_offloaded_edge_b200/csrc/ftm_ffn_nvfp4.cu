// NVFP4 grouped SwiGLU FFN: e2m1 weights with one e4m3 scale per 16 elements
// and one fp32 scale per tensor; activations quantised to e2m1 with one e4m3
// scale per 16 elements and a per-tensor fp32 global scale (x: gx, the SwiGLU
// output h: gh; static values supplied with the layer, 1 when absent):
// s16 = e4m3(amax / (6 g)), codes = e2m1(v / (s16 g)).  The accumulators are
// scaled by (weight tensor scale) x (activation global scale).
//
// The contraction is tcgen05.mma kind::mxf4nvf4 with hardware block scaling:
// each MMA (K = 64) takes the four scales of every A row and every B row from
// TMEM.  The scales travel global -> shared memory by bulk copy (512-byte
// chunks in the layout the MMA expects) and shared -> TMEM by tcgen05.cp
// (32x128b, replicated to the four lane quadrants), issued by the MMA thread
// right before the MMAs that use them.
//
// Scale-chunk layout (weights and activations alike): one 512-byte chunk per
// (block of rows, 64 elements of K); the scale of local row r (< 128) for the
// j-th 16-element group of the chunk is byte (r % 32) * 16 + (r / 32) * 4 + j.
// Weight chunks cover 128-row blocks; activation chunks cover BN-row blocks,
// and every expert group of activation rows is padded to a multiple of BN rows
// so each token tile is exactly one block.
#include "ftm_gemm.cuh"

namespace ftm {

constexpr int kF4StageK = 256;         // K per stage: 128 bytes of packed e2m1 = one swizzle row
constexpr uint32_t kSfChunk = 512;     // bytes of one scale chunk (128 rows x four scale groups)
// NVFP4 CTA-pair gate/up: the token scales of one K step for a 224-row block, the chunk of rows 0-127 four
// times then the chunk of rows 128-255 four times (the TMEM image of two 32x128b.warpx4 copies)
constexpr uint32_t kRepChunkBytes = 4096;

// The two block-scale formats of the e2m1 kernels.  NVFP4 (MX = false): one
// e4m3 scale per 16 elements, a chunk covers K = 64, one MMA (K = 64) reads
// all four bytes of a row's 32-bit scale column.  MXFP4 (MX = true, OCP MX):
// one E8M0 scale per 32 elements, a chunk covers K = 128, and the two MMAs of
// a chunk read bytes 0-1 and 2-3 of the column (scale-factor ids 0 and 2).
template <bool MX>
struct F4Fmt {
  static constexpr int kGroup = MX ? 32 : 16;             // elements per scale
  static constexpr int kChunkK = 4 * kGroup;              // K covered by one chunk
  static constexpr int kChunks = kF4StageK / kChunkK;     // chunks per stage (per 128-row operand tile)
  static constexpr uint32_t kSfStage = kChunks * kSfChunk;
};

// ---- conversions ---------------------------------------------------------------
__device__ __forceinline__ uint8_t f32_to_e4m3_sat(float v) {
  uint16_t r;
  asm("{\n\t.reg .b16 t;\n\tcvt.rn.satfinite.e4m3x2.f32 t, %1, %2;\n\tmov.b16 %0, t;\n\t}" : "=h"(r) : "f"(0.f), "f"(v));
  return static_cast<uint8_t>(r & 0xFF);
}

__device__ __forceinline__ float e4m3_to_f32(uint8_t q) {
  uint32_t h2;
  const uint16_t in = q;
  asm("{\n\t.reg .b16 t;\n\tmov.b16 t, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, t;\n\t}" : "=r"(h2) : "h"(in));
  return __half2float(__ushort_as_half(static_cast<unsigned short>(h2 & 0xFFFF)));
}

// byte = e2m1(hi) << 4 | e2m1(lo), round to nearest even, saturating at 6.
__device__ __forceinline__ uint8_t f32x2_to_e2m1x2(float hi, float lo) {
  uint16_t r;
  asm("{\n\t.reg .b8 t;\n\tcvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\tcvt.u16.u8 %0, t;\n\t}"
      : "=h"(r)
      : "f"(hi), "f"(lo));
  return static_cast<uint8_t>(r & 0xFF);
}

__host__ __device__ constexpr uint32_t idesc_nvf4(int M, int N) {
  // a/b format E2M1 (1) at bits 7 and 10; scale format UE4M3 (0) at bit 23; K = 64
  return (1u << 7) | (1u << 10) | (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

// MXFP4: scale format UE8M0 (bit 23); sf_id (0 or 2) = the byte of the 32-bit
// scale column this MMA starts at, for A (bits 29-30) and B (bits 4-5).
__host__ __device__ constexpr uint32_t idesc_mxf4(int M, int N, uint32_t sf_id) {
  return idesc_nvf4(M, N) | (1u << 23) | (sf_id << 29) | (sf_id << 4);
}

// The block scale of a tile's TMEM scale address for sf_id (its top two bits
// carry the byte offset, as the instruction descriptor does).
__device__ __forceinline__ uint32_t sf_addr(uint32_t taddr, uint32_t sf_id) { return taddr | (sf_id << 30); }

__device__ __forceinline__ void umma_nvf4(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                          uint32_t sfa, uint32_t sfb, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t}\n" ::"r"(
          d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
      : "memory");
}

__device__ __forceinline__ void umma_mxf4(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                          uint32_t sfa, uint32_t sfb, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block32 [%0], %1, %2, %3, [%5], [%6], p;\n\t}\n" ::"r"(
          d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
      : "memory");
}

// E8M0 code of a 32-group (OCP MX): 2^(code - 127) with code - 127 =
// floor(log2 amax) - 2, clamped to [-127, 127]; an all-zero group gets 127.
// Exponent read from the bits: a subnormal amax (< 2^-126) clamps to -127.
__device__ __forceinline__ int mx_scale_code(float amax) {
  if (amax == 0.f) return 127;
  const int be = static_cast<int>((__float_as_uint(amax) >> 23) & 0xFF);
  int e = be - 127 - 2;
  if (be == 0) e = -127;
  return e < -127 ? 0 : e + 127;
}

// 2^(127 - code): the exact power of two that divides a group by its scale
// (always a normal float for the codes mx_scale_code returns from finite input).
__device__ __forceinline__ float mx_inv_scale(int code) { return __uint_as_float(static_cast<uint32_t>(254 - code) << 23); }

// shared -> TMEM copy of one 512-byte scale chunk: 32 rows x 16 bytes,
// replicated into the four 32-lane quadrants (4 columns each).
__device__ __forceinline__ void tmem_cp_sf(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}

// Descriptor of a 512-byte chunk: no swizzle, 8-row core matrices of 16-byte
// rows stored contiguously (stride between 8-row groups 128 bytes).
__device__ __forceinline__ uint64_t smem_desc_sf(uint32_t saddr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>(16u >> 4) << 16;      // leading byte offset (one 16-byte column only)
  d |= static_cast<uint64_t>(128u >> 4) << 32;     // stride byte offset: 8 rows x 16 bytes
  d |= static_cast<uint64_t>(1u) << 46;            // version
  return d;                                         // layout type 0: no swizzle
}

__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_u32(dst)),
               "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ uint32_t sf_byte(int r, int j) { return (r % 32) * 16 + (r / 32) * 4 + j; }

// 128-row A tiles per stage: narrow gate/up token tiles take two paired blocks
// (128 intermediate indices) so a stage still streams 32 KB of weights per
// 4 KB of activations; 128-token tiles take one (the TMEM budget).
__host__ __device__ constexpr int nvfp4_a_tiles(int BN, bool gated) { return gated && BN <= 64 ? 2 : 1; }

// ---------------------------------------------------------------------------
// Padded row offsets: prow0[g] = sum_{g' < g} roundup(rows_g', BN), g = 0..G.
// ---------------------------------------------------------------------------
__global__ void pad_offsets_kernel(const int32_t* __restrict__ offsets, int E, int has_shared, int T, int BN,
                                   int32_t* __restrict__ prow0) {
  __shared__ int32_t rows[kMaxGroups];
  pdl_wait();
  pdl_trigger();

  const int G = E + (has_shared ? 1 : 0);
  for (int g = threadIdx.x; g < G; g += blockDim.x) {
    const int r = g < E ? offsets[g + 1] - offsets[g] : T;
    rows[g] = (r + BN - 1) / BN * BN;
  }
  __syncthreads();
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    const int per = (G + 31) / 32, b = lane * per, en = min(G, b + per);
    int s = 0;
    for (int g = b; g < en; ++g) s += rows[g];
    int incl = s;
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    int run = incl - s;
    for (int g = b; g < en; ++g) { prow0[g] = run; run += rows[g]; }
    if (lane == 31) prow0[G] = incl;
  }
}

// ---------------------------------------------------------------------------
// Quantisation of x, once per token: xq_tok [T][d/2] packed e2m1 and s_tok
// [T][d/G] scale bytes (G = 16 e4m3 scales for NVFP4, 32 E8M0 codes for
// MXFP4); every four consecutive scale bytes of a token are the 32-bit word a
// scale chunk keeps together for one row.  One warp per token; each lane
// quantises whole groups (NVFP4: two 16-byte loads -> 8 packed bytes + one
// scale; MXFP4: four loads -> 16 packed bytes + one code).
// ---------------------------------------------------------------------------
template <bool MX>
__global__ void __launch_bounds__(256) quant_tokens_f4_kernel(const uint16_t* __restrict__ x, int T, int d,
                                                              const float* __restrict__ act_scale,
                                                              uint8_t* __restrict__ xq_tok,
                                                              uint8_t* __restrict__ s_tok) {
  constexpr int G = F4Fmt<MX>::kGroup;
  pdl_wait();
  pdl_trigger();
  const float gx = (!MX && act_scale) ? act_scale[0] : 1.f;
  const float six_gx = 6.0f * gx;
  const int ng = d / G;
  const int lane = threadIdx.x % 32, warp = threadIdx.x / 32, nwarps = blockDim.x / 32;
  for (int t = blockIdx.x * nwarps + warp; t < T; t += gridDim.x * nwarps) {
    for (int g = lane; g < ng; g += 32) {
      float v[G];
      const uint4* p = reinterpret_cast<const uint4*>(x + static_cast<size_t>(t) * d + g * G);
#pragma unroll
      for (int u = 0; u < G / 8; ++u) {
        const uint4 w4 = p[u];
        const uint32_t w[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          v[8 * u + 2 * i] = bf16_bits_to_f32(w[i] & 0xFFFF);
          v[8 * u + 2 * i + 1] = bf16_bits_to_f32(w[i] >> 16);
        }
      }
      float amax = 0.f;
#pragma unroll
      for (int i = 0; i < G; ++i) amax = fmaxf(amax, fabsf(v[i]));
      uint8_t sq;
      if constexpr (MX) {
        const int code = mx_scale_code(amax);
        const float mul = mx_inv_scale(code);      // exact: v * 2^-e == v / 2^e
        sq = static_cast<uint8_t>(code);
        uint32_t packed[4] = {0, 0, 0, 0};
#pragma unroll
        for (int i = 0; i < 16; ++i)
          packed[i / 4] |= static_cast<uint32_t>(f32x2_to_e2m1x2(v[2 * i + 1] * mul, v[2 * i] * mul)) << (8 * (i % 4));
        *reinterpret_cast<uint4*>(xq_tok + static_cast<size_t>(t) * (d / 2) + g * 16) =
            make_uint4(packed[0], packed[1], packed[2], packed[3]);
      } else {
        sq = f32_to_e4m3_sat(amax / six_gx);
        const float sc = e4m3_to_f32(sq) * gx;
        uint32_t packed[2] = {0, 0};
        if (sc != 0.f) {
#pragma unroll
          for (int i = 0; i < 8; ++i)
            packed[i / 4] |= static_cast<uint32_t>(f32x2_to_e2m1x2(v[2 * i + 1] / sc, v[2 * i] / sc)) << (8 * (i % 4));
        }
        *reinterpret_cast<uint2*>(xq_tok + static_cast<size_t>(t) * (d / 2) + g * 8) = make_uint2(packed[0], packed[1]);
      }
      s_tok[static_cast<size_t>(t) * ng + g] = sq;
    }
  }
}

// ---------------------------------------------------------------------------
// Gather of the quantised tokens into the padded activation rows.  Packed
// codes: one warp per padded row copies its token's d/2 bytes (16-byte
// vectors).  Scale words (one per chunk of four groups: d/64 for NVFP4, d/128
// for MXFP4): one warp per 128-row chunk block and eight chunk columns, lane l
// collecting the words of rows l, l+32, l+64 and l+96 (the 16 bytes it owns in
// each 512-byte chunk), so every store is a full coalesced chunk (rows past a
// group's end are zeros).  The padded group offsets sit in shared memory.
// ---------------------------------------------------------------------------
template <bool MX>
__global__ void __launch_bounds__(256) gather_f4_kernel(const uint8_t* __restrict__ xq_tok,
                                                          const uint8_t* __restrict__ s_tok,
                                                          const int32_t* __restrict__ perm,
                                                          const int32_t* __restrict__ offsets,
                                                          const int32_t* __restrict__ prow0, int E, int has_shared,
                                                          int T, int k, int d, int BN, int replicate,
                                                          uint8_t* __restrict__ xq, uint8_t* __restrict__ sfx) {
  __shared__ int32_t s_prow0[kMaxGroups + 1];
  pdl_wait();
  pdl_trigger();
  const int G = E + (has_shared ? 1 : 0);
  for (int i = threadIdx.x; i <= G; i += blockDim.x) s_prow0[i] = prow0[i];
  __syncthreads();
  const int rows_pad = s_prow0[G];
  const int nkc = d / F4Fmt<MX>::kChunkK, nvec = d / 32;    // scale words, 16-byte vectors per packed row
  const int nsub = (BN + 127) / 128;               // 128-row scale chunks per BN-row block
  const int lane = threadIdx.x % 32, warp = threadIdx.x / 32, nwarps = blockDim.x / 32;
  // the source token of padded row pr, or -1 past its group's end
  auto token_of = [&](int pr) -> int {
    int lo = 0, hi = G;  // s_prow0[lo] <= pr < s_prow0[hi]
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (s_prow0[mid] <= pr) lo = mid; else hi = mid;
    }
    const int local = pr - s_prow0[lo];
    const int rows = lo < E ? offsets[lo + 1] - offsets[lo] : T;
    return local >= rows ? -1 : (lo < E ? perm[offsets[lo] + local] / k : local);
  };
  for (int pr = blockIdx.x * nwarps + warp; pr < rows_pad; pr += gridDim.x * nwarps) {
    int src = -1;
    if (lane == 0) src = token_of(pr);
    src = __shfl_sync(0xffffffffu, src, 0);
    const uint4* s = reinterpret_cast<const uint4*>(xq_tok + static_cast<size_t>(src < 0 ? 0 : src) * (d / 2));
    uint4* dst = reinterpret_cast<uint4*>(xq + static_cast<size_t>(pr) * (d / 2));
    for (int c0 = 0; c0 < nvec; c0 += 32 * 8) {     // up to 8 loads in flight per lane, then the stores
      uint4 v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int c = c0 + u * 32 + lane;
        v[u] = (c < nvec && src >= 0) ? s[c] : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int c = c0 + u * 32 + lane;
        if (c < nvec) dst[c] = v[u];
      }
    }
  }
  const uint32_t* sw = reinterpret_cast<const uint32_t*>(s_tok);
  const int ncb = (rows_pad / BN) * nsub;             // 128-row chunk blocks
  const int nkg = (nkc + 7) / 8;                       // groups of eight chunk columns
  for (long long it = static_cast<long long>(blockIdx.x) * nwarps + warp; it < static_cast<long long>(ncb) * nkg;
       it += static_cast<long long>(gridDim.x) * nwarps) {
    const int cb = static_cast<int>(it / nkg), kg = static_cast<int>(it % nkg);
    const int blk = cb / nsub, sub = cb % nsub;
    int src[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int i = sub * 128 + lane + 32 * q;          // row within the BN-row block
      src[q] = i < BN ? token_of(blk * BN + i) : -1;
    }
    uint4 w[8];
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      const int kb = kg * 8 + kk;
      uint32_t v[4];
#pragma unroll
      for (int q = 0; q < 4; ++q)
        v[q] = (kb < nkc && src[q] >= 0) ? sw[static_cast<size_t>(src[q]) * nkc + kb] : 0u;
      w[kk] = make_uint4(v[0], v[1], v[2], v[3]);
    }
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      const int kb = kg * 8 + kk;
      if (kb >= nkc) continue;
      if (replicate) {   // the K step's 4 KB block: [chunk of rows 0-127 x 4][chunk of rows 128-255 x 4]
        uint8_t* b = sfx + (static_cast<size_t>(blk) * nkc + kb) * kRepChunkBytes + sub * 2048 + lane * 16;
#pragma unroll
        for (int r = 0; r < 4; ++r) *reinterpret_cast<uint4*>(b + r * kSfChunk) = w[kk];
      } else {
        *reinterpret_cast<uint4*>(sfx + (static_cast<size_t>(cb) * nkc + kb) * kSfChunk + lane * 16) = w[kk];
      }
    }
  }
}

// ---------------------------------------------------------------------------
// GEMM1 epilogue: quantise one thread's 16 consecutive intermediate values
// (16-group `grp` of the 64-wide paired block mb, for one token row) and store
// the packed codes (q_dst, 8 bytes) and the scale into out_sf: chunk row
// block rb, row rr of the chunk, Nw intermediate columns.  NVFP4: e4m3 scale
// of amax / (6 gh) times gh.  MXFP4: the 32-group is this thread's 16 values
// and those of lane ^ 1 (all 32 lanes must call); the even lane stores the
// code.  Padding rows are quantised too (never read back).  REP (NVFP4 on CTA
// pairs): rb is the 224-row block and rr the row in it, and the scale goes to
// the block's replicated layout (each 128-row chunk four times per K step).
// ---------------------------------------------------------------------------
template <bool MX, bool REP = false>
__device__ __forceinline__ void quant_store_h(const float (&h)[16], float gh, float six_gh, uint8_t* q_dst,
                                              uint8_t* out_sf, size_t rb, int rr, int mb, int grp, int Nw) {
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(h[i]));
  uint32_t packed[2] = {0u, 0u};
  if constexpr (MX) {
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
    const int code = mx_scale_code(amax);
    const float mul = mx_inv_scale(code);
#pragma unroll
    for (int i = 0; i < 16; i += 2)
      packed[i / 8] |= static_cast<uint32_t>(f32x2_to_e2m1x2(h[i + 1] * mul, h[i] * mul)) << (4 * (i % 8));
    *reinterpret_cast<uint2*>(q_dst) = make_uint2(packed[0], packed[1]);
    if ((grp & 1) == 0)
      out_sf[(rb * (Nw / 128) + mb / 2) * kSfChunk + sf_byte(rr, (mb & 1) * 2 + grp / 2)] = static_cast<uint8_t>(code);
  } else {
    const uint8_t sq = f32_to_e4m3_sat(amax / six_gh);
    const float sc = e4m3_to_f32(sq) * gh;
    if (sc != 0.f) {
#pragma unroll
      for (int i = 0; i < 16; i += 2)
        packed[i / 8] |= static_cast<uint32_t>(f32x2_to_e2m1x2(h[i + 1] / sc, h[i] / sc)) << (4 * (i % 8));
    }
    *reinterpret_cast<uint2*>(q_dst) = make_uint2(packed[0], packed[1]);
    if constexpr (REP) {
      uint8_t* b = out_sf + (rb * (Nw / 64) + mb) * kRepChunkBytes + (rr / 128) * 2048 + sf_byte(rr % 128, grp);
#pragma unroll
      for (int r = 0; r < 4; ++r) b[r * kSfChunk] = sq;
    } else {
      out_sf[(rb * (Nw / 64) + mb) * kSfChunk + sf_byte(rr, grp)] = sq;
    }
  }
}

// ---------------------------------------------------------------------------
// The grouped GEMM.
//   A: packed e2m1 weights via a 3-D map {K bytes, rows, slot} (shared: 2-D)
//   weight scale chunks at bank + wsf_off; per-tensor scales at bank + st_off
//   B: packed e2m1 activations {K bytes, rows_pad}, scale chunks act_sf
//   GATED: out_q (e2m1 H [rows_pad][Nw/2]) + out_sf (chunks); else out_bf16 [rows][Nw]
//
// Every stage holds NP 128-row A tiles (nvfp4_a_tiles), so each 64-deep K step
// is NP MMAs of M = 128 x N = BN.  Gate/up GEMM: an A tile is 64 gate rows and the same 64
// up rows (two 64-row boxes), matching the paired order of the gate/up scale
// chunks, so the accumulator's lane i and lane i + 64 hold gate and up of one
// intermediate index; the epilogue pairs them across warps through shared
// memory, applies the per-tensor scales and SwiGLU, then transposes H so each
// thread quantises one token's 16 consecutive intermediate values.
// ---------------------------------------------------------------------------
constexpr int kF4Threads = 224;   // warps 0 TMA, 1 MMA, 2-5 epilogue, 6 scale copies

template <int BN, bool GATED, bool MX>
__global__ void __launch_bounds__(kF4Threads, 1)
    ffn_nvfp4_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmAsh,
                     const __grid_constant__ CUtensorMap tmB, const int32_t* __restrict__ offsets,
                     const int32_t* __restrict__ prow0, const int32_t* __restrict__ slot_of_expert, int E,
                     int has_shared, int T, int P, int K, int Nw, int up_row0, const uint8_t* __restrict__ pool,
                     const uint8_t* __restrict__ shared_bank, size_t bank_bytes, size_t wsf_off, size_t st_off,
                     int st_idx, const uint8_t* __restrict__ act_sf, uint8_t* __restrict__ out_q,
                     uint8_t* __restrict__ out_sf, uint16_t* __restrict__ out_bf16,
                     const float* __restrict__ act_scale, int stages) {
  using Fmt = F4Fmt<MX>;
  constexpr uint32_t kSfStage = Fmt::kSfStage;
  constexpr int kCh = Fmt::kChunks;                 // scale chunks per stage and operand tile
  constexpr uint32_t kBBytes = ((BN * 128 + 1023) / 1024) * 1024;
  constexpr int NP = nvfp4_a_tiles(BN, GATED);     // 128-row A tiles per stage, one accumulator each
  constexpr uint32_t kStageBytes = NP * kATileBytes + kBBytes + (NP + 1) * kSfStage;
  constexpr uint32_t kTx = NP * kATileBytes + BN * 128 + (NP + 1) * kSfStage;
  constexpr uint32_t kAccCols = NP * BN;
  constexpr uint32_t kSfCols = 4 * kCh * (NP + 1); // SFA per A tile | SFB: kCh chunks x 4 columns each
  // Ring of scale-factor column sets, one per stage in flight: the copies for
  // stage s + 1 never overwrite columns the MMAs of stage s still read.
  constexpr uint32_t kSfSets = 4;
  constexpr uint32_t kUsedCols = 2 * kAccCols + kSfSets * kSfCols;
  static_assert(kUsedCols <= 512, "TMEM budget");
  constexpr uint32_t kTmemCols = kUsedCols <= 256 ? 256 : 512;
  constexpr uint32_t kIdesc = idesc_nvf4(128, BN);
  constexpr int kRowsPerTile = (GATED ? 64 : 128) * NP;   // output rows (intermediate / hidden) per tile

  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full_bar[8], empty_bar[8], tfull_bar[2], tempty_bar[2];
  // the scale warp copies a stage's chunks into scale set g % kSfSets (g = stages so far), then commits
  // sf_ready[stage]; the MMA thread commits sf_free[set] once the MMAs reading the set are done
  __shared__ __align__(8) uint64_t sf_ready[8], sf_free[4];
  __shared__ uint32_t tmem_holder;
  __shared__ int32_t tile_start[kMaxGroups + 1], grp_rows[kMaxGroups], grp_row0[kMaxGroups];
  // gate/up epilogue: half-chunks crossing between gate and up warps, and a
  // 32-token x 64-intermediate block of H (16-groups padded to 17 floats)
  __shared__ float xbuf[GATED ? 128 * 17 : 1];
  __shared__ float tbuf[GATED ? 32 * 68 : 1];

  const uint32_t smem_base = (smem_u32(smem_raw) + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (smem_base - smem_u32(smem_raw));
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int G = E + (has_shared ? 1 : 0);
  const int MT = Nw / kRowsPerTile;
  const int KB = K / kF4StageK;
  const int Kc = K / Fmt::kChunkK;                  // scale chunks along K of one 128-row block

  if (threadIdx.x == 0) {
    for (int s = 0; s < stages; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
      mbar_init(&sf_ready[s], 1);
    }
    for (int r = 0; r < static_cast<int>(kSfSets); ++r) mbar_init(&sf_free[r], 1);
    for (int a = 0; a < 2; ++a) { mbar_init(&tfull_bar[a], 1); mbar_init(&tempty_bar[a], 4); }
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&tmem_holder, kTmemCols);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmAsh);
    tma_prefetch_desc(&tmB);
  }
  pdl_wait();      // the group offsets come from earlier kernels
  pdl_trigger();
  build_tile_table(offsets, E, has_shared, T, P, MT, BN, tile_start, grp_rows, grp_row0);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = tmem_holder;
  const uint32_t tmem_sf0 = tmem_base + 2 * kAccCols;
  const int total = tile_start[G];

  auto a_tile = [&](int s, int p) -> uint8_t* {
    return smem + static_cast<size_t>(s) * kStageBytes + p * kATileBytes;
  };
  auto b_tile = [&](int s) -> uint8_t* { return smem + static_cast<size_t>(s) * kStageBytes + NP * kATileBytes; };
  auto sf_tile = [&](int s, int which) -> uint8_t* {   // which: p < NP weights of A tile p, NP activations
    return smem + static_cast<size_t>(s) * kStageBytes + NP * kATileBytes + kBBytes + which * kSfStage;
  };

  if (warp == 0) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
        const TileInfo ti = decode_tile(t, tile_start, grp_rows, grp_row0, G, BN);
        const int slot = ti.g < E ? slot_of_expert[ti.g] : 0;
        const uint8_t* bank = ti.g < E ? pool + static_cast<size_t>(slot) * bank_bytes : shared_bank;
        const uint8_t* wsf = bank + wsf_off + static_cast<size_t>(ti.m) * NP * Kc * kSfChunk;
        const int prow = prow0[ti.g] + ti.n * BN;
        const uint8_t* asf = act_sf + static_cast<size_t>(prow / BN) * Kc * kSfChunk;
        const int r0 = ti.m * kRowsPerTile;
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait(&empty_bar[stage], phase ^ 1u)) { ok = false; break; }
          mbar_arrive_expect_tx(&full_bar[stage], kTx);
          const int kc = kb * (kF4StageK / 2);   // byte coordinate along K
#pragma unroll
          for (int p = 0; p < NP; ++p) {
            // gate/up: tile p is the paired block of 64 gate rows and the same 64 up rows
            const int rp = r0 + p * (GATED ? 64 : 128);
            if (ti.g < E) {
              tma_load_3d(a_tile(stage, p), &tmA, &full_bar[stage], kc, rp, slot);
              if (GATED)
                tma_load_3d(a_tile(stage, p) + kATileBytes / 2, &tmA, &full_bar[stage], kc, up_row0 + rp, slot);
            } else {
              tma_load_2d(a_tile(stage, p), &tmAsh, &full_bar[stage], kc, rp);
              if (GATED) tma_load_2d(a_tile(stage, p) + kATileBytes / 2, &tmAsh, &full_bar[stage], kc, up_row0 + rp);
            }
            bulk_load(sf_tile(stage, p), wsf + (static_cast<size_t>(p) * Kc + kCh * kb) * kSfChunk, kSfStage,
                      &full_bar[stage]);
          }
          tma_load_2d(b_tile(stage), &tmB, &full_bar[stage], kc, prow);
          bulk_load(sf_tile(stage, NP), asf + static_cast<size_t>(kCh * kb) * kSfChunk, kSfStage, &full_bar[stage]);
          if (++stage == stages) { stage = 0; phase ^= 1u; }
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      int it = 0;
      uint32_t sf_set = 0;
      for (int t = blockIdx.x; t < total && ok; t += gridDim.x, ++it) {
        const int ab = it & 1;
        const uint32_t aphase = (it >> 1) & 1;
        if (!mbar_wait(&tempty_bar[ab], aphase ^ 1u)) break;
        tc_fence_after();
        const uint32_t d = tmem_base + ab * kAccCols;
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait(&full_bar[stage], phase)) { ok = false; break; }
          if (!mbar_wait(&sf_ready[stage], phase)) { ok = false; break; }   // the stage's scales are in TMEM
          tc_fence_after();
          const uint32_t cur_set = sf_set;
          const uint32_t tmem_sf = tmem_sf0 + sf_set * kSfCols;
          if (++sf_set == kSfSets) sf_set = 0;
          const uint32_t sb = smem_u32(b_tile(stage));
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const int c = kk * kCh / 4;                    // the chunk of this K step
#pragma unroll
            for (int p = 0; p < NP; ++p) {
              const uint32_t sfa = tmem_sf + 4 * kCh * p + 4 * c, sfb = tmem_sf + 4 * kCh * NP + 4 * c;
              const uint64_t ad = smem_desc_sw128(smem_u32(a_tile(stage, p)) + kk * 32);
              const uint64_t bd = smem_desc_sw128(sb + kk * 32);
              const uint32_t acc = (kb | kk) != 0 ? 1u : 0u;
              if constexpr (MX) {
                const uint32_t sf_id = 2u * (kk & 1);      // bytes 0-1 or 2-3 of the chunk's columns
                umma_mxf4(d + p * BN, ad, bd, idesc_mxf4(128, BN, sf_id), sf_addr(sfa, sf_id), sf_addr(sfb, sf_id),
                          acc);
              } else {
                umma_nvf4(d + p * BN, ad, bd, kIdesc, sfa, sfb, acc);
              }
            }
          }
          umma_commit(&sf_free[cur_set]);   // the scale warp may refill this set
          umma_commit(&empty_bar[stage]);
          if (++stage == stages) { stage = 0; phase ^= 1u; }
        }
        if (ok) umma_commit(&tfull_bar[ab]);
      }
    }
    __syncwarp();
  } else if (warp == 6) {
    // scale warp: copies each stage's weight and token scale chunks into the next TMEM set, ahead of the MMAs
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      uint32_t g = 0;   // stages copied so far
      for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
        for (int kb = 0; kb < KB; ++kb, ++g) {
          if (!mbar_wait(&full_bar[stage], phase)) { ok = false; break; }
          const uint32_t set = g % kSfSets;
          // the set is free once the MMAs of the stage kSfSets earlier are done
          if (g >= kSfSets && !mbar_wait(&sf_free[set], (g / kSfSets - 1) & 1u)) { ok = false; break; }
          tc_fence_after();
          const uint32_t tmem_sf = tmem_sf0 + set * kSfCols;
#pragma unroll
          for (int c = 0; c < kCh; ++c) {
#pragma unroll
            for (int p = 0; p <= NP; ++p)
              tmem_cp_sf(tmem_sf + 4 * kCh * p + 4 * c, smem_desc_sf(smem_u32(sf_tile(stage, p)) + c * kSfChunk));
          }
          umma_commit(&sf_ready[stage]);
          if (++stage == stages) { stage = 0; phase ^= 1u; }
        }
      }
    }
    __syncwarp();
  } else {
    const int q = warp % 4;
    int it = 0;
    for (int t = blockIdx.x; t < total; t += gridDim.x, ++it) {
      const TileInfo ti = decode_tile(t, tile_start, grp_rows, grp_row0, G, BN);
      const int ab = it & 1;
      const uint32_t aphase = (it >> 1) & 1;
      if (!epilogue_all(mbar_wait(&tfull_bar[ab], aphase))) break;
      tc_fence_after();
      const int valid = min(BN, ti.rows - ti.n * BN);
      const uint8_t* bank = ti.g < E ? pool + static_cast<size_t>(slot_of_expert[ti.g]) * bank_bytes : shared_bank;
      const float* st = reinterpret_cast<const float*>(bank + st_off);   // NVFP4 only
      const uint32_t tb = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + ab * kAccCols;
      if (GATED) {
        // H = silu(s_gate * gate) * (s_up * up) in fp32 (NVFP4: weight tensor
        // scale x activation global scale; MXFP4: no tensor scale), then the
        // e2m1 codes and block scales of H (quant_store_h).
        const bool gate_warp = q < 2;
        const float gx = (!MX && act_scale) ? act_scale[0] : 1.f, gh = (!MX && act_scale) ? act_scale[1] : 1.f;
        const float six_gh = 6.0f * gh;
        const float s_row = MX ? 1.f : st[st_idx + (gate_warp ? 0 : 1)] * gx;
        const int me = q * 32 + lane, partner = (q ^ 2) * 32 + lane;
        const int il = (q % 2) * 32 + lane;               // intermediate index within the tile
        const int col_off = gate_warp ? 0 : 16;           // the 16 columns of a chunk this warp evaluates
        const int tslot = (il / 16) * 17 + il % 16;
        const int prow = prow0[ti.g] + ti.n * BN;
        const int blk = prow / BN;
        const int tok = me >> 2, grp = me & 3;            // quantisation: one (token, 16-group) per thread
        for (int p = 0; p < NP; ++p) {   // accumulator p = paired block mb of 64 intermediate indices
          const int mb = ti.m * NP + p;
          for (int c0 = 0; c0 < BN; c0 += 32) {
            float v[32];
            tmem_ld16(tb + p * BN + c0, v);
            tmem_ld16(tb + p * BN + c0 + 16, v + 16);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] *= s_row;
#pragma unroll
            for (int j = 0; j < 16; ++j) xbuf[me * 17 + j] = gate_warp ? v[16 + j] : v[j];
            epilogue_bar();
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              const float other = xbuf[partner * 17 + j];
              tbuf[(col_off + j) * 68 + tslot] = gate_warp ? silu(v[j]) * other : silu(other) * v[16 + j];
            }
            epilogue_bar();
            float h[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) h[i] = tbuf[tok * 68 + grp * 17 + i];
            const int i0 = mb * 64 + grp * 16;
            quant_store_h<MX>(h, gh, six_gh, out_q + static_cast<size_t>(prow + c0 + tok) * (Nw / 2) + i0 / 2, out_sf,
                              static_cast<size_t>(blk), c0 + tok, mb, grp, Nw);
          }
        }
      } else {
        const float s_a = MX ? 1.f : st[st_idx] * (act_scale ? act_scale[1] : 1.f);
        const int wrow = ti.m * 128 + q * 32 + lane;
        uint16_t* obase = out_bf16 + static_cast<size_t>(ti.row0 + ti.n * BN) * Nw + wrow;
        for (int c0 = 0; c0 < valid; c0 += 16) {
          float a[16];
          tmem_ld16(tb + c0, a);
          tmem_ld_wait();
#pragma unroll
          for (int jj = 0; jj < 16; ++jj) {
            if (c0 + jj < valid) {
              const __nv_bfloat16 hb = __float2bfloat16_rn(a[jj] * s_a);
              obase[static_cast<size_t>(c0 + jj) * Nw] = *reinterpret_cast<const uint16_t*>(&hb);
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty_bar[ab]);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, kTmemCols);
}

// ---------------------------------------------------------------------------
// Prefill-size NVFP4 GEMMs on CTA pairs (tcgen05 cta_group::2).
//
// A pair tile is M = 256 weight rows (128 staged by each CTA) by N <= 224
// tokens (N/2 staged by each CTA), K = 256 per stage: four block-scaled MMAs
// of K = 64, issued by the even CTA.  Every load of a stage -- weights, tokens
// and both kinds of scale chunks -- is a TMA copy with .cta_group::2 whose
// bytes count on the even CTA's full barrier.  The scale chunks are viewed as
// rows of 256 bytes (a 2 KB stage slice = 8 rows).  Each CTA's TMEM holds its
// 128 rows for all N columns (two 224-column accumulators), the weight scales
// of its own rows and the token scales of all N tokens (two 128-row chunks),
// copied smem -> TMEM by one tcgen05.cp.cta_group::2 per chunk.
// Tokens are padded per expert group to 224-row blocks; the activation scale
// chunks of a block are its two 128-row halves.  A group's last tile runs the
// MMA at N = the next multiple of 32 above its token count.
// No TMA multicast: every CTA loads its own tiles.
// ---------------------------------------------------------------------------
constexpr int kQN = 224;                        // tokens per pair tile (padded block; a multiple of the 32-row scale groups)
constexpr int kQH = kQN / 2;                    // token rows staged per CTA
constexpr uint32_t kQABytes = 128 * 128;        // 128 weight rows x 256 e2m1
constexpr uint32_t kQBBytes = kQH * 128;        // 112 token rows x 256 e2m1
constexpr int kQStages = 5;
constexpr uint32_t kQSfCol = 2 * kQN;           // TMEM: accumulators [0, 448), then the ring of scale units
constexpr int kQThreads = 224;                  // warps 0 TMA, 1 MMA, 2-5 epilogue, 6 scale copies

// Stage layout of the pair kernel per scale format: A tile | B tile | the
// stage's scale chunks of this CTA's 128 weight rows | of the token block's
// two 128-row halves.  In TMEM a chunk per operand takes 12 columns: 4 of
// weight scales + 2 x 4 of token scales.  The scales travel in units of two K
// steps, 24 columns for NVFP4 (a chunk per K step) and 12 for MXFP4 (one chunk
// read through scale-factor ids 0 and 2), cycling through a ring of kRing unit
// slots in the columns left after the accumulators, so the copies of a unit
// overlap the MMAs of the ones before.
template <bool MX, bool GATED>
struct Q2Fmt {
  // NVFP4: the token scales (x for gate/up, H for down) arrive replicated (per K step a 4 KB block holding
  // each of the two 128-row chunks four times, the TMEM layout of the 32x128b.warpx4 copies), so one
  // 128x256b copy moves a K step's token scales; four stages then fit shared memory instead of five
  static constexpr bool kRep = !MX;
  static constexpr int kStages = kRep ? 4 : kQStages;
  static constexpr uint32_t kSfa = F4Fmt<MX>::kSfStage;
  static constexpr uint32_t kSfb = kRep ? 4 * kRepChunkBytes : 2 * F4Fmt<MX>::kSfStage;
  static constexpr uint32_t kStage = kQABytes + kQBBytes + kSfa + kSfb;
  static constexpr int kUnitK = MX ? 4 : 2;               // K steps per scale unit
  static constexpr int kUnits = 4 / kUnitK;               // scale units per stage (4 K steps)
  static constexpr int kUnitChunks = MX ? kUnitK / 2 : kUnitK;
  static constexpr uint32_t kUnitCols = 12 * kUnitChunks;
  static constexpr uint32_t kRing = (512 - kQSfCol) / kUnitCols < 5 ? (512 - kQSfCol) / kUnitCols : 5;
  static_assert(kRing >= 2, "scale copies overlap MMAs");
  static_assert(kStage % 1024 == 0, "stages keep the 1024-byte alignment of the swizzled tiles");
  static_assert(kQSfCol + kRing * kUnitCols <= 512, "TMEM budget");
};

__device__ __forceinline__ int quad_tile_n(int valid) { return min(kQN, (valid + 31) & ~31); }

__device__ __forceinline__ void umma2_nvf4(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                           uint32_t sfa, uint32_t sfb, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t}\n" ::"r"(
          d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
      : "memory");
}

__device__ __forceinline__ void umma2_mxf4(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                           uint32_t sfa, uint32_t sfb, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.block32 [%0], %1, %2, %3, [%5], [%6], p;\n\t}\n" ::"r"(
          d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
      : "memory");
}

// Both CTAs of the pair: copy one 512-byte scale chunk from this offset of
// each CTA's shared memory into the same columns of its own TMEM.
__device__ __forceinline__ void tmem_cp_sf2(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::2.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}

// Both CTAs of the pair: copy 128 rows of 32 bytes (8 columns) from this
// offset of each CTA's shared memory into the same columns of its own TMEM.
__device__ __forceinline__ void tmem_cp_wide2(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::2.128x256b [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}

// Descriptor of a replicated 4 KB token-scale block: no swizzle, 128 rows of
// two 16-byte columns, the second column 2048 bytes after the first (leading
// byte offset), 8-row groups 128 bytes apart (stride byte offset).
__device__ __forceinline__ uint64_t smem_desc_rep(uint32_t saddr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>(2048u >> 4) << 16;
  d |= static_cast<uint64_t>(128u >> 4) << 32;
  d |= static_cast<uint64_t>(1u) << 46;            // version; layout type 0: no swizzle
  return d;
}

// Arrive on this CTA's barrier once the executing thread's pair operations complete.
__device__ __forceinline__ void umma2_commit_local(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

template <bool GATED, bool MX>
__global__ void __launch_bounds__(kQThreads, 1)
    ffn_nvfp4_tc2_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmAsh,
                         const __grid_constant__ CUtensorMap tmB, const __grid_constant__ CUtensorMap tmSfa,
                         const __grid_constant__ CUtensorMap tmSfaSh, const __grid_constant__ CUtensorMap tmSfb,
                         const int32_t* __restrict__ offsets, const int32_t* __restrict__ prow0,
                         const int32_t* __restrict__ slot_of_expert, int E, int has_shared, int T, int P, int K,
                         int Nw, int up_row0, const uint8_t* __restrict__ pool,
                         const uint8_t* __restrict__ shared_bank, size_t bank_bytes, size_t st_off, int st_idx,
                         uint8_t* __restrict__ out_q, uint8_t* __restrict__ out_sf, uint16_t* __restrict__ out_bf16,
                         const float* __restrict__ act_scale) {
  constexpr uint32_t kTmemCols = 512;
  constexpr int kRowsPerPair = GATED ? 128 : 256;   // output rows (intermediate / hidden) per pair tile
  using Q = Q2Fmt<MX, GATED>;
  constexpr int kCh = F4Fmt<MX>::kChunks;
  constexpr uint32_t kQStage = Q::kStage;

  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full_bar[Q::kStages], empty_bar[Q::kStages], tfull_bar[2], tempty_bar[2];
  // Scale copies and MMAs run from different threads.  Scale unit u (counted over the whole kernel) uses
  // TMEM slot u % kRing.  sf_ready[stage * kUnits + j] = unit j of the stage in that smem slot is in TMEM
  // (one barrier per stage slot and unit, so a barrier is reused only once per trip round the stages);
  // sf_free[slot] = the MMAs that read the TMEM slot are done.  The copies run up to kRing - 1 units ahead.
  __shared__ __align__(8) uint64_t sf_ready[Q::kStages * Q::kUnits], sf_free[Q::kRing];
  __shared__ uint32_t tmem_holder;
  __shared__ int32_t tile_start[kMaxGroups + 1], grp_rows[kMaxGroups], grp_row0[kMaxGroups];
  __shared__ float xbuf[GATED ? 128 * 17 : 1];
  __shared__ float tbuf[GATED ? 32 * 68 : 1];
  constexpr int kYPitch = 40;   // bf16 per staging row: 32 columns + 16 bytes, rows stay 16-byte aligned
  __shared__ __align__(16) uint16_t ybuf[GATED ? 8 : 4 * 32 * kYPitch];

  const uint32_t smem_base = (smem_u32(smem_raw) + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (smem_base - smem_u32(smem_raw));
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const uint32_t rank = cluster_rank();
  const bool leader = rank == 0;
  const int npairs = gridDim.x / 2;
  const int pair = blockIdx.x / 2;
  const int G = E + (has_shared ? 1 : 0);
  const int MT = Nw / kRowsPerPair;
  const int KB = K / kF4StageK;
  const int Kc = K / F4Fmt<MX>::kChunkK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < Q::kStages; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    for (int r = 0; r < Q::kStages * Q::kUnits; ++r) mbar_init(&sf_ready[r], 1);
    for (int r = 0; r < Q::kRing; ++r) mbar_init(&sf_free[r], 1);
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull_bar[a], 1);
      mbar_init(&tempty_bar[a], 8);
    }
    fence_mbar_init();
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&tmem_holder)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmAsh);
    tma_prefetch_desc(&tmB);
    tma_prefetch_desc(&tmSfa);
    tma_prefetch_desc(&tmSfaSh);
    tma_prefetch_desc(&tmSfb);
  }
  pdl_wait();
  pdl_trigger();
  build_tile_table(offsets, E, has_shared, T, P, MT, kQN, tile_start, grp_rows, grp_row0);
  tc_fence_before();
  cluster_sync_all();     // barriers initialised and TMEM allocated in both CTAs
  tc_fence_after();
  const uint32_t tmem_base = tmem_holder;
  const int total = tile_start[G];

  auto a_tile = [&](int s) -> uint8_t* { return smem + static_cast<size_t>(s) * kQStage; };
  auto b_tile = [&](int s) -> uint8_t* { return a_tile(s) + kQABytes; };
  auto sfa_tile = [&](int s) -> uint8_t* { return a_tile(s) + kQABytes + kQBBytes; };
  auto sfb_tile = [&](int s) -> uint8_t* { return a_tile(s) + kQABytes + kQBBytes + Q::kSfa; };

  if (warp == 0) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int t = pair; t < total && ok; t += npairs) {
        const TileInfo ti = decode_tile(t, tile_start, grp_rows, grp_row0, G, kQN);
        const int ntile = quad_tile_n(min(kQN, ti.rows - ti.n * kQN));
        const bool routed = ti.g < E;
        const int slot = routed ? slot_of_expert[ti.g] : 0;
        const int prow = prow0[ti.g] + ti.n * kQN;
        const int blk = prow / kQN;
        const int brow = prow + static_cast<int>(rank) * (ntile / 2);
        const int wb = ti.m * 2 + static_cast<int>(rank);   // this CTA's 128-row weight block (paired for gate/up)
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait_cl(&empty_bar[stage], phase ^ 1u)) { ok = false; break; }
          if (leader) mbar_arrive_expect_tx(&full_bar[stage], 2 * kQStage);
          const uint32_t lbar = mapa_rank(smem_u32(&full_bar[stage]), 0);   // the even CTA's barrier
          const int kc = kb * (kF4StageK / 2);                              // byte coordinate along K
          const int sfa_row = (wb * Kc + kCh * kb) * 2;                      // 256-byte rows of the chunks
          if (GATED) {
            if (routed) {
              tma2_load_3d(a_tile(stage), &tmA, lbar, kc, wb * 64, slot);
              tma2_load_3d(a_tile(stage) + kQABytes / 2, &tmA, lbar, kc, up_row0 + wb * 64, slot);
            } else {
              tma2_load_2d(a_tile(stage), &tmAsh, lbar, kc, wb * 64);
              tma2_load_2d(a_tile(stage) + kQABytes / 2, &tmAsh, lbar, kc, up_row0 + wb * 64);
            }
          } else {
            if (routed) tma2_load_3d(a_tile(stage), &tmA, lbar, kc, wb * 128, slot);
            else tma2_load_2d(a_tile(stage), &tmAsh, lbar, kc, wb * 128);
          }
          if (routed) tma2_load_3d(sfa_tile(stage), &tmSfa, lbar, 0, sfa_row, slot);
          else tma2_load_2d(sfa_tile(stage), &tmSfaSh, lbar, 0, sfa_row);
          tma2_load_2d(b_tile(stage), &tmB, lbar, kc, brow);
          if (Q::kRep) {   // the stage's four replicated K steps: 16 KB = 64 rows of 256 bytes
            tma2_load_2d(sfb_tile(stage), &tmSfb, lbar, 0, (blk * Kc + kCh * kb) * (kRepChunkBytes / 256));
          } else {
#pragma unroll
            for (int h = 0; h < 2; ++h)
              tma2_load_2d(sfb_tile(stage) + h * Q::kSfa, &tmSfb, lbar, 0, ((blk * 2 + h) * Kc + kCh * kb) * 2);
          }
          if (++stage == Q::kStages) { stage = 0; phase ^= 1u; }
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (leader && lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      int it = 0;
      uint32_t u = 0;   // scale units consumed so far (unsigned: the ring index is a mask or a shift)
      for (int t = pair; t < total && ok; t += npairs, ++it) {
        const TileInfo ti = decode_tile(t, tile_start, grp_rows, grp_row0, G, kQN);
        const int ntile = quad_tile_n(min(kQN, ti.rows - ti.n * kQN));
        const uint32_t idesc = MX ? idesc_mxf4(256, ntile, 0) : idesc_nvf4(256, ntile);
        const int ab = it & 1;
        const uint32_t aphase = (it >> 1) & 1;
        if (!mbar_wait_cl(&tempty_bar[ab], aphase ^ 1u)) break;
        tc_fence_after();
        const uint32_t d = tmem_base + ab * kQN;
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait_cl(&full_bar[stage], phase)) { ok = false; break; }
          const uint32_t sa = smem_u32(a_tile(stage)), sb = smem_u32(b_tile(stage));
#pragma unroll
          for (int j = 0; j < Q::kUnits; ++j, ++u) {
            const uint32_t slot = u % Q::kRing;
            if (!mbar_wait_cl(&sf_ready[stage * Q::kUnits + j], phase)) { ok = false; break; }
            tc_fence_after();
            const uint32_t sf = tmem_base + kQSfCol + Q::kUnitCols * slot;
#pragma unroll
            for (int jj = 0; jj < Q::kUnitK; ++jj) {          // the unit's K steps
              const int kk = Q::kUnitK * j + jj;
              const uint64_t ad = smem_desc_sw128(sa + kk * 32), bd = smem_desc_sw128(sb + kk * 32);
              const uint32_t acc = (kb | kk) != 0 ? 1u : 0u;
              const uint32_t c = MX ? jj / 2 : jj;                 // the K step's chunk within the unit
              const uint32_t sfa = sf + 4 * c, sfb = sf + 4 * Q::kUnitChunks + 8 * c;
              if constexpr (MX) {                                   // bytes 0-1 or 2-3 of the chunk's columns
                const uint32_t sf_id = 2u * (jj & 1);
                umma2_mxf4(d, ad, bd, idesc | (sf_id << 29) | (sf_id << 4), sf_addr(sfa, sf_id),
                           sf_addr(sfb, sf_id), acc);
              } else {
                umma2_nvf4(d, ad, bd, idesc, sfa, sfb, acc);
              }
            }
            umma2_commit_local(&sf_free[slot]);
          }
          if (!ok) break;
          umma2_commit_both(&empty_bar[stage]);
          if (++stage == Q::kStages) { stage = 0; phase ^= 1u; }
        }
        if (ok) umma2_commit_both(&tfull_bar[ab]);
      }
    }
    __syncwarp();
  } else if (warp == 6) {
    // the even CTA copies each stage's scales into TMEM (both CTAs) ahead of the MMA thread
    if (leader && lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      uint32_t u = 0;   // scale units copied so far
      for (int t = pair; t < total && ok; t += npairs) {
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait_cl(&full_bar[stage], phase)) { ok = false; break; }
          const uint32_t ssa = smem_u32(sfa_tile(stage)), ssb = smem_u32(sfb_tile(stage));
#pragma unroll
          for (int j = 0; j < Q::kUnits; ++j, ++u) {
            // the slot is free once the MMAs of the unit kRing earlier are done
            const uint32_t slot = u % Q::kRing;
            if (u >= Q::kRing && !mbar_wait_cl(&sf_free[slot], (u / Q::kRing - 1) & 1u)) { ok = false; break; }
            tc_fence_after();
            const uint32_t sf = tmem_base + kQSfCol + Q::kUnitCols * slot;
#pragma unroll
            for (int c = 0; c < Q::kUnitChunks; ++c) {   // NVFP4 one chunk per K step, MXFP4 one per two
              const uint32_t off = (j * Q::kUnitChunks + c) * kSfChunk;
              tmem_cp_sf2(sf + 4 * c, smem_desc_sf(ssa + off));                          // this CTA's weight rows
              if (Q::kRep) {                                                             // all 224 tokens at once
                tmem_cp_wide2(sf + 4 * Q::kUnitChunks + 8 * c,
                              smem_desc_rep(ssb + (j * Q::kUnitChunks + c) * kRepChunkBytes));
              } else {
                tmem_cp_sf2(sf + 4 * Q::kUnitChunks + 8 * c, smem_desc_sf(ssb + off));   // tokens 0-127
                tmem_cp_sf2(sf + 4 * Q::kUnitChunks + 8 * c + 4, smem_desc_sf(ssb + Q::kSfa + off));  // 128-223
              }
            }
            umma2_commit_local(&sf_ready[stage * Q::kUnits + j]);
          }
          if (!ok) break;
          if (++stage == Q::kStages) { stage = 0; phase ^= 1u; }
        }
      }
    }
    __syncwarp();
  } else {
    const int q = warp % 4;           // TMEM lane quadrant
    const uint32_t tempty0 = mapa_rank(smem_u32(&tempty_bar[0]), 0);
    const uint32_t tempty1 = mapa_rank(smem_u32(&tempty_bar[1]), 0);
    int it = 0;
    for (int t = pair; t < total; t += npairs, ++it) {
      const TileInfo ti = decode_tile(t, tile_start, grp_rows, grp_row0, G, kQN);
      const int valid = min(kQN, ti.rows - ti.n * kQN);
      const int ntile = quad_tile_n(valid);
      const int ab = it & 1;
      const uint32_t aphase = (it >> 1) & 1;
      if (!epilogue_all(mbar_wait_cl(&tfull_bar[ab], aphase))) break;
      tc_fence_after();
      const uint8_t* bank = ti.g < E ? pool + static_cast<size_t>(slot_of_expert[ti.g]) * bank_bytes : shared_bank;
      const float* st = reinterpret_cast<const float*>(bank + st_off);
      const uint32_t tb = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + ab * kQN;
      if (GATED) {
        // this CTA's rows: 64 gate + the same 64 up rows of paired block pb
        const int pb = ti.m * 2 + static_cast<int>(rank);
        const bool gate_warp = q < 2;
        const float gx = (!MX && act_scale) ? act_scale[0] : 1.f, gh = (!MX && act_scale) ? act_scale[1] : 1.f;
        const float six_gh = 6.0f * gh;
        const float s_row = MX ? 1.f : st[st_idx + (gate_warp ? 0 : 1)] * gx;
        const int me = q * 32 + lane, partner = (q ^ 2) * 32 + lane;
        const int il = (q % 2) * 32 + lane;
        const int col_off = gate_warp ? 0 : 16;
        const int tslot = (il / 16) * 17 + il % 16;
        const int prow = prow0[ti.g] + ti.n * kQN;
        const int blk = prow / kQN;
        const int tok = me >> 2, grp = me & 3;
        for (int c0 = 0; c0 < ntile; c0 += 32) {
          float v[32];
          tmem_ld16(tb + c0, v);
          tmem_ld16(tb + c0 + 16, v + 16);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] *= s_row;
#pragma unroll
          for (int j = 0; j < 16; ++j) xbuf[me * 17 + j] = gate_warp ? v[16 + j] : v[j];
          epilogue_bar();
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const float other = xbuf[partner * 17 + j];
            tbuf[(col_off + j) * 68 + tslot] = gate_warp ? silu(v[j]) * other : silu(other) * v[16 + j];
          }
          epilogue_bar();
          float h[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) h[i] = tbuf[tok * 68 + grp * 17 + i];
          const int tr = c0 + tok;   // token row within the 224-row block
          if constexpr (MX)
            quant_store_h<MX>(h, gh, six_gh, out_q + static_cast<size_t>(prow + tr) * (Nw / 2) + (pb * 64 + grp * 16) / 2,
                              out_sf, static_cast<size_t>(blk * 2 + tr / 128), tr % 128, pb, grp, Nw);
          else
            quant_store_h<MX, true>(h, gh, six_gh,
                                    out_q + static_cast<size_t>(prow + tr) * (Nw / 2) + (pb * 64 + grp * 16) / 2, out_sf,
                                    static_cast<size_t>(blk), tr, pb, grp, Nw);
        }
      } else {
        // lane = output column, TMEM column = token: 32 tokens at a time go through the warp's staging
        // rows so that each store is 16 bytes of one token's row
        const float s_a = MX ? 1.f : st[st_idx] * (act_scale ? act_scale[1] : 1.f);
        const int w0 = ti.m * 256 + static_cast<int>(rank) * 128 + q * 32;
        uint16_t* o = out_bf16 + static_cast<size_t>(ti.row0 + ti.n * kQN) * Nw + w0;
        uint16_t* yb = ybuf + (warp - 2) * (32 * kYPitch);
        for (int c0 = 0; c0 < valid; c0 += 32) {
          float a[32];
          tmem_ld16(tb + c0, a);
          tmem_ld16(tb + c0 + 16, a + 16);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const __nv_bfloat16 hb = __float2bfloat16_rn(a[j] * s_a);
            yb[j * kYPitch + lane] = *reinterpret_cast<const uint16_t*>(&hb);
          }
          __syncwarp();
#pragma unroll
          for (int r = 0; r < 4; ++r) {
            const int j = r * 8 + lane / 4, part = lane % 4;
            if (c0 + j < valid)
              *reinterpret_cast<uint4*>(o + static_cast<size_t>(c0 + j) * Nw + part * 8) =
                  *reinterpret_cast<const uint4*>(yb + j * kYPitch + part * 8);
          }
          __syncwarp();
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (leader) mbar_arrive(&tempty_bar[ab]);
        else mbar_arrive_remote(ab ? tempty1 : tempty0);
      }
    }
  }
  tc_fence_before();
  __syncwarp();
  cluster_sync_all();     // no CTA leaves while its pair may still signal it
  tc_fence_after();
  if (warp == 1)
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(kTmemCols) : "memory");
}

// ---------------------------------------------------------------------------
// Host
// ---------------------------------------------------------------------------
static bool make_map_f4(CUtensorMap* m, const void* base, uint64_t K, uint64_t rows, uint64_t slots,
                        uint64_t slot_pitch, uint32_t box_rows) {
  // packed e2m1: K/2 bytes per row, addressed as bytes
  return make_map_sw128(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, base, K / 2, rows, K / 2, slots, slot_pitch, box_rows);
}

// Token tile: the smallest of 32 / 64 / 128 that holds an average group, so
// decode batches pad little and prefill batches get wide MMAs.
int nvfp4_token_tile(int P, int E) {
  const int avg = (P + E - 1) / E;
  return avg <= 32 ? 32 : avg <= 96 ? 64 : 128;
}

static size_t al256(size_t b) { return (b + 255) & ~static_cast<size_t>(255); }

// Upper bound of the padded activation rows for token tile BN.
static int64_t nvfp4_rows_pad(int64_t P, int T, int G, int has_shared, int BN) {
  return P + (has_shared ? T : 0) + static_cast<int64_t>(G) * (BN - 1);
}

// Bytes of the gathered token-scale region: 128-row chunks (at most rows_pad / 32 + one partial block per
// group), or for the NVFP4 pair path one replicated 4 KB block per 224-row block and K step.
static int64_t sfx_region_bytes(int64_t rp, int G, int d) {
  const int64_t chunks = (rp / 32 + G + 1) * (d / 64) * kSfChunk;
  const int64_t replicated = (rp / kQN + 1) * (d / 64) * static_cast<int64_t>(kRepChunkBytes);
  return chunks > replicated ? chunks : replicated;
}

// Workspace: prow0 | Xq [rows_pad][d/2] | SFx chunks | Hq [rows_pad][I/2] | SFh chunks |
//            per-token Xq [T][d/2] | per-token scales [T][d/16]
size_t nvfp4_ffn_workspace_bytes(int64_t P, int T, int E, int has_shared, int d, int I) {
  const int G = E + (has_shared ? 1 : 0);
  const int64_t rp = nvfp4_rows_pad(P, T, G, has_shared, kQN);   // the largest tile bounds all
  return al256(sizeof(int32_t) * (G + 1)) + al256(rp * (d / 2)) + al256(sfx_region_bytes(rp, G, d)) +
         al256(rp * (I / 2)) + al256(sfx_region_bytes(rp, G, I)) + al256(static_cast<int64_t>(T) * (d / 2)) +
         al256(static_cast<int64_t>(T) * (d / 16));
}

template <int BN, bool GATED, bool MX>
static cudaError_t launch_nvfp4(const CUtensorMap& mA, const CUtensorMap& mAsh, const CUtensorMap& mB,
                                const FfnArgs& a, const int32_t* prow0, int K, int Nw, int up_row0, size_t wsf_off,
                                size_t st_off, int st_idx, const uint8_t* act_sf, uint8_t* out_q, uint8_t* out_sf,
                                uint16_t* out_bf16, cudaStream_t st) {
  constexpr uint32_t kBBytes = ((BN * 128 + 1023) / 1024) * 1024;
  constexpr int NP = nvfp4_a_tiles(BN, GATED);
  constexpr uint32_t kStageBytes = NP * kATileBytes + kBBytes + (NP + 1) * F4Fmt<MX>::kSfStage;
  int stages = (200 * 1024 - 1024) / static_cast<int>(kStageBytes);
  if (stages > 8) stages = 8;
  const size_t smem = 1024 + static_cast<size_t>(stages) * kStageBytes;
  auto kern = ffn_nvfp4_kernel<BN, GATED, MX>;
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (err != cudaSuccess) return err;
  const int P = a.T * a.k;
  const int G = a.E + (a.has_shared ? 1 : 0);
  const long max_tiles = static_cast<long>((P + BN - 1) / BN + G) * (Nw / ((GATED ? 64 : 128) * NP));
  const int grid = static_cast<int>(max_tiles < num_sms() ? max_tiles : num_sms());
  return launch_pdl(kern, dim3(grid), dim3(kF4Threads), smem, st, mA, mAsh, mB, a.offsets, prow0, a.slot_of_expert,
                    a.E, a.has_shared, a.T, P, K, Nw, up_row0, a.pool, a.shared_bank, a.bank_bytes, wsf_off, st_off,
                    st_idx, act_sf, out_q, out_sf, out_bf16, a.act_scale, stages);
}

// ---- CTA-pair launch (prefill-size groups) -----------------------------------
// Groups averaging >= 192 rows run on CTA pairs with 224-token tiles.
static bool nvfp4_pair_applicable(int P, int E) { return (P + E - 1) / E >= 192; }

// Scale chunks as rows of 256 bytes (a stage's chunks = box_rows rows: 8 for
// NVFP4's four chunks, 4 for MXFP4's two), no swizzle:
// dims {256, rows[, slots]}, box {256, box_rows[, 1]}.
static bool make_map_rows256(CUtensorMap* m, const void* base, uint64_t bytes, uint64_t slots, uint64_t slot_pitch,
                             uint32_t box_rows) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {256, bytes / 256, slots};
  cuuint64_t strides[2] = {256, slot_pitch};
  cuuint32_t box[3] = {256, box_rows, 1};
  cuuint32_t es[3] = {1, 1, 1};
  const cuuint32_t rank = slots > 0 ? 3 : 2;
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, rank, const_cast<void*>(base), dims, strides, box, es,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <bool GATED, bool MX>
static cudaError_t launch_nvfp4_tc2_one(const CUtensorMap* maps, const FfnArgs& a, const int32_t* prow0, int K,
                                        int Nw, int up_row0, size_t st_off, int st_idx, uint8_t* out_q,
                                        uint8_t* out_sf, uint16_t* out_bf16, cudaStream_t st) {
  const size_t smem = 1024 + static_cast<size_t>(Q2Fmt<MX, GATED>::kStages) * Q2Fmt<MX, GATED>::kStage;
  auto kern = ffn_nvfp4_tc2_kernel<GATED, MX>;
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (err != cudaSuccess) return err;
  const int P = a.T * a.k;
  const int G = a.E + (a.has_shared ? 1 : 0);
  const long tiles = static_cast<long>((P + kQN - 1) / kQN + G) * (Nw / (GATED ? 128 : 256));
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(kQThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  static int pairs_max = 0;   // co-resident pairs of this instantiation (not every SM may find a partner)
  if (!pairs_max) {
    cfg.gridDim = dim3(num_sms());
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n <= 0) {
      (void)cudaGetLastError();
      n = num_sms() / 2;
    }
    pairs_max = n < num_sms() / 2 ? n : num_sms() / 2;
  }
  const int pairs = static_cast<int>(tiles < pairs_max ? tiles : pairs_max);
  cfg.gridDim = dim3(2 * pairs);
  cfg.numAttrs = 2;
  return count_launch(cudaLaunchKernelEx(&cfg, kern, maps[0], maps[1], maps[2], maps[3], maps[4], maps[5], a.offsets, prow0,
                            a.slot_of_expert, a.E, a.has_shared, a.T, P, K, Nw, up_row0, a.pool, a.shared_bank,
                            a.bank_bytes, st_off, st_idx, out_q, out_sf, out_bf16, a.act_scale));
}

// Both GEMMs on CTA pairs; xq/sfx (gathered, padded to 224-row blocks) are ready.
template <bool MX>
static const char* launch_nvfp4_gemms_tc2(const FfnArgs& a, const int32_t* prow0, size_t s_gu_off, size_t s_d_off,
                                          size_t s_t_off, int64_t rp, uint8_t* xq, uint8_t* sfx, size_t sfx_bytes,
                                          uint8_t* hq, uint8_t* sfh, size_t sfh_bytes, cudaStream_t st,
                                          cudaError_t* cerr) {
  constexpr int G = F4Fmt<MX>::kGroup;
  constexpr uint32_t kBox = 2 * F4Fmt<MX>::kChunks;   // 256-byte rows of a stage's chunks
  const uint64_t S = static_cast<uint64_t>(a.S);
  const uint64_t s_gu_bytes = 2ull * a.I * (a.d / G), s_d_bytes = static_cast<uint64_t>(a.d) * (a.I / G);
  // maps per GEMM: A, A (shared expert), B, A scales, A scales (shared expert), B scales
  CUtensorMap m1[6], m2[6];
  bool ok = make_map_f4(&m1[0], a.pool + a.w_gu_off, a.d, 2ull * a.I, S, a.bank_bytes, 64) &&
            make_map_f4(&m1[2], xq, a.d, static_cast<uint64_t>(rp), 0, 0, kQH) &&
            make_map_rows256(&m1[3], a.pool + s_gu_off, s_gu_bytes, S, a.bank_bytes, kBox) &&
            make_map_rows256(&m1[5], sfx, sfx_bytes, 0, 0, MX ? kBox : 4 * kRepChunkBytes / 256) &&
            make_map_f4(&m2[0], a.pool + a.w_d_off, a.I, a.d, S, a.bank_bytes, 128) &&
            make_map_f4(&m2[2], hq, a.I, static_cast<uint64_t>(rp), 0, 0, kQH) &&
            make_map_rows256(&m2[3], a.pool + s_d_off, s_d_bytes, S, a.bank_bytes, kBox) &&
            make_map_rows256(&m2[5], sfh, sfh_bytes, 0, 0, MX ? kBox : 4 * kRepChunkBytes / 256);
  if (ok && a.has_shared) {
    ok = make_map_f4(&m1[1], a.shared_bank + a.w_gu_off, a.d, 2ull * a.I, 0, 0, 64) &&
         make_map_rows256(&m1[4], a.shared_bank + s_gu_off, s_gu_bytes, 0, 0, kBox) &&
         make_map_f4(&m2[1], a.shared_bank + a.w_d_off, a.I, a.d, 0, 0, 128) &&
         make_map_rows256(&m2[4], a.shared_bank + s_d_off, s_d_bytes, 0, 0, kBox);
  } else {
    m1[1] = m1[0];
    m1[4] = m1[3];
    m2[1] = m2[0];
    m2[4] = m2[3];
  }
  if (!ok) return "cuTensorMapEncodeTiled failed";
  prof_mark(FTM_K_GEMM1, st, false);
  *cerr = launch_nvfp4_tc2_one<true, MX>(m1, a, prow0, a.d, a.I, a.I, s_t_off, 0, hq, sfh, nullptr, st);
  prof_mark(FTM_K_GEMM1, st, true);
  if (*cerr != cudaSuccess) return "nvfp4 pair gemm1 launch failed";
  prof_mark(FTM_K_GEMM2, st, false);
  *cerr = launch_nvfp4_tc2_one<false, MX>(m2, a, prow0, a.I, a.d, 0, s_t_off, 2, nullptr, nullptr,
                                          reinterpret_cast<uint16_t*>(a.y), st);
  prof_mark(FTM_K_GEMM2, st, true);
  if (*cerr != cudaSuccess) return "nvfp4 pair gemm2 launch failed";
  return nullptr;
}

template <bool MX>
static const char* launch_f4(const FfnArgs& a, size_t s_gu_off, size_t s_d_off, size_t s_t_off, uint8_t* ws,
                             cudaStream_t st, cudaError_t* cerr) {
  constexpr int kCK = F4Fmt<MX>::kChunkK;
  const int P = a.T * a.k;
  const int G = a.E + (a.has_shared ? 1 : 0);
  *cerr = cudaSuccess;
  if (P + (a.has_shared ? a.T : 0) == 0) return nullptr;
  const bool pair = nvfp4_pair_applicable(P, a.E);
  const int BN = pair ? kQN : nvfp4_token_tile(P, a.E);
  const int64_t rp = nvfp4_rows_pad(P, a.T, G, a.has_shared, kQN);
  const int64_t blocks = rp / 32 + G + 1;
  int32_t* prow0 = reinterpret_cast<int32_t*>(ws);
  uint8_t* xq = ws + al256(sizeof(int32_t) * (G + 1));
  uint8_t* sfx = xq + al256(rp * (a.d / 2));
  // regions sized for NVFP4's chunks (MXFP4 uses half of each scale region)
  uint8_t* hq = sfx + al256(sfx_region_bytes(rp, G, a.d));
  uint8_t* sfh = hq + al256(rp * (a.I / 2));
  uint8_t* xq_tok = sfh + al256(sfx_region_bytes(rp, G, a.I));
  uint8_t* s_tok = xq_tok + al256(static_cast<int64_t>(a.T) * (a.d / 2));
  prof_mark(FTM_K_GATHER, st, false);
  // each token is quantised once, then its packed row is copied into every
  // padded row that uses it (k routed picks + the shared expert)
  *cerr = launch_pdl(pad_offsets_kernel, dim3(1), dim3(512), 0, st, a.offsets, a.E, a.has_shared, a.T, BN, prow0);
  if (*cerr == cudaSuccess) {
    const int grid = a.T / 8 + 1 < 148 * 8 ? a.T / 8 + 1 : 148 * 8;
    *cerr = launch_pdl(quant_tokens_f4_kernel<MX>, dim3(grid), dim3(256), 0, st,
                       reinterpret_cast<const uint16_t*>(a.x), a.T, a.d, a.act_scale, xq_tok, s_tok);
  }
  if (*cerr == cudaSuccess) {
    const int grid = static_cast<int>(rp / 8 + 1 < 148 * 8 ? rp / 8 + 1 : 148 * 8);
    *cerr = launch_pdl(gather_f4_kernel<MX>, dim3(grid), dim3(256), 0, st, xq_tok, s_tok, a.perm, a.offsets, prow0,
                       a.E, a.has_shared, a.T, a.k, a.d, BN, !MX && pair ? 1 : 0, xq, sfx);
  }
  prof_mark(FTM_K_GATHER, st, true);
  if (*cerr != cudaSuccess) return "nvfp4 gather launch failed";
  if (pair)
    return launch_nvfp4_gemms_tc2<MX>(a, prow0, s_gu_off, s_d_off, s_t_off, rp, xq, sfx,
                                      MX ? blocks * (a.d / kCK) * kSfChunk : sfx_region_bytes(rp, G, a.d), hq, sfh,
                                      MX ? blocks * (a.I / kCK) * kSfChunk : sfx_region_bytes(rp, G, a.I), st, cerr);
  CUtensorMap mA1, mAsh1, mB1, mA2, mAsh2, mB2;
  const uint64_t S = static_cast<uint64_t>(a.S);
  // gate/up boxes are 64 rows: a tile stages 64 gate rows and the same 64 up rows
  bool ok = make_map_f4(&mA1, a.pool + a.w_gu_off, a.d, 2ull * a.I, S, a.bank_bytes, 64) &&
            make_map_f4(&mA2, a.pool + a.w_d_off, a.I, a.d, S, a.bank_bytes, 128) &&
            make_map_f4(&mB1, xq, a.d, static_cast<uint64_t>(rp), 0, 0, BN) &&
            make_map_f4(&mB2, hq, a.I, static_cast<uint64_t>(rp), 0, 0, BN);
  if (ok && a.has_shared) {
    ok = make_map_f4(&mAsh1, a.shared_bank + a.w_gu_off, a.d, 2ull * a.I, 0, 0, 64) &&
         make_map_f4(&mAsh2, a.shared_bank + a.w_d_off, a.I, a.d, 0, 0, 128);
  } else {
    mAsh1 = mA1;
    mAsh2 = mA2;
  }
  if (!ok) return "cuTensorMapEncodeTiled failed";
  prof_mark(FTM_K_GEMM1, st, false);
  *cerr = BN == 32 ? launch_nvfp4<32, true, MX>(mA1, mAsh1, mB1, a, prow0, a.d, a.I, a.I, s_gu_off, s_t_off, 0, sfx, hq,
                                            sfh, nullptr, st)
          : BN == 64 ? launch_nvfp4<64, true, MX>(mA1, mAsh1, mB1, a, prow0, a.d, a.I, a.I, s_gu_off, s_t_off, 0, sfx, hq,
                                              sfh, nullptr, st)
                     : launch_nvfp4<128, true, MX>(mA1, mAsh1, mB1, a, prow0, a.d, a.I, a.I, s_gu_off, s_t_off, 0, sfx,
                                               hq, sfh, nullptr, st);
  prof_mark(FTM_K_GEMM1, st, true);
  if (*cerr != cudaSuccess) return "nvfp4 gemm1 launch failed";
  prof_mark(FTM_K_GEMM2, st, false);
  uint16_t* y = reinterpret_cast<uint16_t*>(a.y);
  *cerr = BN == 32 ? launch_nvfp4<32, false, MX>(mA2, mAsh2, mB2, a, prow0, a.I, a.d, 0, s_d_off, s_t_off, 2, sfh,
                                             nullptr, nullptr, y, st)
          : BN == 64 ? launch_nvfp4<64, false, MX>(mA2, mAsh2, mB2, a, prow0, a.I, a.d, 0, s_d_off, s_t_off, 2, sfh,
                                               nullptr, nullptr, y, st)
                     : launch_nvfp4<128, false, MX>(mA2, mAsh2, mB2, a, prow0, a.I, a.d, 0, s_d_off, s_t_off, 2, sfh,
                                                nullptr, nullptr, y, st);
  prof_mark(FTM_K_GEMM2, st, true);
  if (*cerr != cudaSuccess) return "nvfp4 gemm2 launch failed";
  return nullptr;
}

const char* launch_expert_ffn_nvfp4(const FfnArgs& a, size_t s_gu_off, size_t s_d_off, size_t s_t_off, uint8_t* ws,
                                    cudaStream_t st, cudaError_t* cerr) {
  return launch_f4<false>(a, s_gu_off, s_d_off, s_t_off, ws, st, cerr);
}

// MXFP4: the same kernels with E8M0 scales per 32 elements; no tensor scale.
const char* launch_expert_ffn_mxfp4(const FfnArgs& a, size_t s_gu_off, size_t s_d_off, uint8_t* ws, cudaStream_t st,
                                    cudaError_t* cerr) {
  return launch_f4<true>(a, s_gu_off, s_d_off, 0, ws, st, cerr);
}

}  // namespace ftm
