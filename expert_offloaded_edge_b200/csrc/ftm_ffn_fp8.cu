// FP8 (e4m3, one fp32 scale per 128x128 weight block) grouped SwiGLU FFN.
//
// Weights stay e4m3 in the slot pool; activations (the gathered hidden rows
// and the SwiGLU output) are quantised per row in 1x128 groups along K,
// s = amax/448, e4m3 round-to-nearest-even.  The contraction runs on the
// tensor cores in tcgen05 kind::f8f6f4.  Both operands change scale every 128
// elements of K, so each 128-deep K block is accumulated in its own TMEM
// buffer and the epilogue warps fold it into fp32 registers with the product
// of the two scales ("promotion"); two TMEM buffers let the MMA of block kb+1
// overlap the promotion of block kb.
//
// GEMM1 epilogue: SwiGLU, then the 1x128 quantisation of H is exactly one
// 128-row weight tile, so the group amax is a reduction across the four
// epilogue warps.  GEMM2 epilogue: bf16 Y.
#include "ftm_gemm.cuh"

namespace ftm {

constexpr uint32_t kF8StageK = 128;          // K per stage = one scale block = one 128-byte swizzle row
constexpr int kF8MaxKB = 64;                  // K <= 8192 (scales of a tile staged in shared memory)

__host__ __device__ constexpr uint32_t idesc_e4m3_f32(int M, int N) {
  // c_format F32 (bit 4); a/b format E4M3 = 0; K-major; N>>3 at 17; M>>4 at 24
  return (1u << 4) | (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

__device__ __forceinline__ void umma_f8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                        uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// e4m3 of v (round to nearest even, saturating to +-448).
__device__ __forceinline__ uint8_t f32_to_e4m3(float v) {
  uint16_t r;
  asm("{\n\t.reg .b16 t;\n\tcvt.rn.satfinite.e4m3x2.f32 t, %1, %2;\n\tmov.b16 %0, t;\n\t}" : "=h"(r) : "f"(0.f), "f"(v));
  return static_cast<uint8_t>(r & 0xFF);
}

// ---------------------------------------------------------------------------
// Gather + quantise: Xq[pos] = e4m3(x[perm[pos]/k] / s), s per 128-group.
// One warp per (row, group); lane holds 4 consecutive elements.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) gather_quant_fp8_kernel(const uint16_t* __restrict__ x,
                                                              const int32_t* __restrict__ perm, int P, int k, int T,
                                                              int has_shared, int d, uint8_t* __restrict__ xq,
                                                              float* __restrict__ sx) {
  pdl_wait();
  pdl_trigger();
  const int rows = P + (has_shared ? T : 0);
  const int groups = d / 128;
  const int lane = threadIdx.x % 32;
  const long total = static_cast<long>(rows) * groups;
  for (long w = (static_cast<long>(blockIdx.x) * blockDim.x + threadIdx.x) / 32; w < total;
       w += static_cast<long>(gridDim.x) * blockDim.x / 32) {
    const int r = static_cast<int>(w / groups), g = static_cast<int>(w % groups);
    const int q = r < P ? perm[r] : 0;
    if (q < 0) continue;     // no pair placed here (ids out of range); warp-uniform
    const int src = r < P ? q / k : r - P;
    const uint2 u = *reinterpret_cast<const uint2*>(x + static_cast<size_t>(src) * d + g * 128 + lane * 4);
    float v[4] = {bf16_bits_to_f32(u.x & 0xFFFF), bf16_bits_to_f32(u.x >> 16), bf16_bits_to_f32(u.y & 0xFFFF),
                  bf16_bits_to_f32(u.y >> 16)};
    float amax = fmaxf(fmaxf(fabsf(v[0]), fabsf(v[1])), fmaxf(fabsf(v[2]), fabsf(v[3])));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    const float s = amax / 448.0f;
    uint32_t packed = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint8_t q = s == 0.f ? 0 : f32_to_e4m3(v[i] / s);
      packed |= static_cast<uint32_t>(q) << (8 * i);
    }
    *reinterpret_cast<uint32_t*>(xq + static_cast<size_t>(r) * d + g * 128 + lane * 4) = packed;
    if (lane == 0) sx[static_cast<size_t>(r) * groups + g] = s;
  }
}

// ---------------------------------------------------------------------------
// The grouped GEMM.
//   A: weights (e4m3) through a 3-D map {K, rows, slot} (shared expert: 2-D map)
//   B: activations (e4m3) {K, rows_total}, scales sact [rows_total][K/128]
//   weight scales: bank + wscale_off, fp32 [rows/128][K/128]
//   GATED: out_q (e4m3 H [rows][Nw]) + out_s (fp32 [rows][Nw/128]); else out_bf16 [rows][Nw]
// ---------------------------------------------------------------------------
template <int BN, bool GATED>
__global__ void __launch_bounds__(kTcThreads, 1)
    ffn_fp8_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmAsh,
                   const __grid_constant__ CUtensorMap tmB, const int32_t* __restrict__ offsets,
                   const int32_t* __restrict__ slot_of_expert, int E, int has_shared, int T, int P, int K, int Nw,
                   int up_row0, const uint8_t* __restrict__ pool, const uint8_t* __restrict__ shared_bank,
                   size_t bank_bytes, size_t wscale_off, const float* __restrict__ sact, uint8_t* __restrict__ out_q,
                   float* __restrict__ out_s, uint16_t* __restrict__ out_bf16, int stages) {
  constexpr uint32_t kBBytes = ((BN * 128 + 1023) / 1024) * 1024;
  constexpr uint32_t kStageBytes = kATileBytes * (GATED ? 2 : 1) + kBBytes;
  constexpr uint32_t kTx = kATileBytes * (GATED ? 2 : 1) + BN * 128;
  constexpr uint32_t kAccCols = GATED ? 2 * BN : BN;
  constexpr uint32_t kTmemCols = 2 * kAccCols < 32 ? 32 : 2 * kAccCols;
  constexpr uint32_t kIdesc = idesc_e4m3_f32(128, BN);

  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full_bar[8], empty_bar[8], pfull_bar[2], pempty_bar[2];
  __shared__ uint32_t tmem_holder;
  __shared__ int32_t tile_start[kMaxGroups + 1], grp_rows[kMaxGroups], grp_row0[kMaxGroups];
  __shared__ float red[4][BN];
  __shared__ float s_sact[BN * kF8MaxKB], s_wsc[2][kF8MaxKB];

  const uint32_t smem_base = (smem_u32(smem_raw) + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (smem_base - smem_u32(smem_raw));
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int G = E + (has_shared ? 1 : 0);
  const int MT = Nw / 128;
  const int KB = K / kF8StageK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < stages; ++s) { mbar_init(&full_bar[s], 1); mbar_init(&empty_bar[s], 1); }
    for (int a = 0; a < 2; ++a) { mbar_init(&pfull_bar[a], 1); mbar_init(&pempty_bar[a], 4); }
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
  const int total = tile_start[G];

  auto a_tile = [&](int s, int which) -> uint8_t* {
    return smem + static_cast<size_t>(s) * kStageBytes + which * kATileBytes;
  };
  auto b_tile = [&](int s) -> uint8_t* {
    return smem + static_cast<size_t>(s) * kStageBytes + kATileBytes * (GATED ? 2 : 1);
  };

  if (warp == 0) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
        const TileInfo ti = decode_tile(t, tile_start, grp_rows, grp_row0, G, BN);
        const int slot = ti.g < E ? slot_of_expert[ti.g] : 0;
        const int brow = ti.row0 + ti.n * BN;
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait(&empty_bar[stage], phase ^ 1u)) { ok = false; break; }
          mbar_arrive_expect_tx(&full_bar[stage], kTx);
          const int kc = kb * kF8StageK;
          if (ti.g < E) {
            tma_load_3d(a_tile(stage, 0), &tmA, &full_bar[stage], kc, ti.m * 128, slot);
            if (GATED) tma_load_3d(a_tile(stage, 1), &tmA, &full_bar[stage], kc, up_row0 + ti.m * 128, slot);
          } else {
            tma_load_2d(a_tile(stage, 0), &tmAsh, &full_bar[stage], kc, ti.m * 128);
            if (GATED) tma_load_2d(a_tile(stage, 1), &tmAsh, &full_bar[stage], kc, up_row0 + ti.m * 128);
          }
          tma_load_2d(b_tile(stage), &tmB, &full_bar[stage], kc, brow);
          if (++stage == stages) { stage = 0; phase ^= 1u; }
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t kcount = 0;   // K blocks issued so far: partial buffer = kcount & 1
      bool ok = true;
      for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
        for (int kb = 0; kb < KB; ++kb, ++kcount) {
          const uint32_t pb = kcount & 1u, pph = (kcount >> 1) & 1u;
          if (!mbar_wait(&full_bar[stage], phase)) { ok = false; break; }
          if (!mbar_wait(&pempty_bar[pb], pph ^ 1u)) { ok = false; break; }
          tc_fence_after();
          const uint32_t d_g = tmem_base + pb * kAccCols;
          const uint32_t sa = smem_u32(a_tile(stage, 0));
          const uint32_t sb = smem_u32(b_tile(stage));
#pragma unroll
          for (int kk = 0; kk < static_cast<int>(kF8StageK / 32); ++kk) {
            const uint64_t bdesc = smem_desc_sw128(sb + kk * 32);
            const uint32_t acc = kk != 0 ? 1u : 0u;
            umma_f8(d_g, smem_desc_sw128(sa + kk * 32), bdesc, kIdesc, acc);
            if (GATED) umma_f8(d_g + BN, smem_desc_sw128(sa + kATileBytes + kk * 32), bdesc, kIdesc, acc);
          }
          umma_commit(&empty_bar[stage]);
          umma_commit(&pfull_bar[pb]);
          if (++stage == stages) { stage = 0; phase ^= 1u; }
        }
      }
    }
    __syncwarp();
  } else {
    const int q = warp % 4;  // TMEM lane quadrant of this warp
    const int et = threadIdx.x - 64;   // 0..127 within the epilogue group
    uint32_t kcount = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
      const TileInfo ti = decode_tile(t, tile_start, grp_rows, grp_row0, G, BN);
      const int valid = min(BN, ti.rows - ti.n * BN);
      const int rowbase = ti.row0 + ti.n * BN;
      const uint8_t* bank = ti.g < E ? pool + static_cast<size_t>(slot_of_expert[ti.g]) * bank_bytes : shared_bank;
      const float* wsc = reinterpret_cast<const float*>(bank + wscale_off);
      // the tile's scales, staged once so the per-K-block promotion reads shared memory only
      epilogue_bar();   // readers of the previous tile are done
      for (int i = et; i < BN * KB; i += 128) {
        const int c = i / KB, kb = i % KB;
        s_sact[i] = c < valid ? sact[static_cast<size_t>(rowbase + c) * KB + kb] : 0.f;
      }
      for (int i = et; i < KB; i += 128) {
        s_wsc[0][i] = wsc[static_cast<size_t>(ti.m) * KB + i];
        if (GATED) s_wsc[1][i] = wsc[static_cast<size_t>(up_row0 / 128 + ti.m) * KB + i];
      }
      epilogue_bar();
      float acc_g[BN], acc_u[GATED ? BN : 1];
#pragma unroll
      for (int c = 0; c < BN; ++c) acc_g[c] = 0.f;
#pragma unroll
      for (int c = 0; c < (GATED ? BN : 1); ++c) acc_u[c] = 0.f;
      for (int kb = 0; kb < KB; ++kb, ++kcount) {
        const uint32_t pb = kcount & 1u, pph = (kcount >> 1) & 1u;
        const float sa_g = s_wsc[0][kb];
        const float sa_u = GATED ? s_wsc[1][kb] : 0.f;
        float sb[BN];
#pragma unroll
        for (int c = 0; c < BN; ++c) sb[c] = s_sact[c * KB + kb];
        if (!epilogue_all(mbar_wait(&pfull_bar[pb], pph))) { ok = false; break; }
        tc_fence_after();
        const uint32_t tb = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + pb * kAccCols;
#pragma unroll
        for (int c0 = 0; c0 < BN; c0 += 16) {
          float pg[16];
          tmem_ld16(tb + c0, pg);
          if (GATED) {
            float pu[16];
            tmem_ld16(tb + BN + c0, pu);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              acc_g[c0 + j] = fmaf(pg[j], sa_g * sb[c0 + j], acc_g[c0 + j]);
              acc_u[c0 + j] = fmaf(pu[j], sa_u * sb[c0 + j], acc_u[c0 + j]);
            }
          } else {
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 16; ++j) acc_g[c0 + j] = fmaf(pg[j], sa_g * sb[c0 + j], acc_g[c0 + j]);
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&pempty_bar[pb]);
      }
      if (!ok) break;
      const int wrow = ti.m * 128 + q * 32 + lane;   // output column (intermediate / hidden index)
      if (GATED) {
        // SwiGLU, then e4m3 quantisation per (token, 128-group) = this tile's 128 rows
        float hv[BN];
#pragma unroll
        for (int c = 0; c < BN; ++c) {
          hv[c] = silu(acc_g[c]) * acc_u[c];
          float a = fabsf(hv[c]);
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
          if (lane == 0) red[q][c] = a;
        }
        epilogue_bar();
        const int nI = Nw / 128;
#pragma unroll
        for (int c = 0; c < BN; ++c) {
          if (c < valid) {
            const float amax = fmaxf(fmaxf(red[0][c], red[1][c]), fmaxf(red[2][c], red[3][c]));
            const float s = amax / 448.0f;
            out_q[static_cast<size_t>(rowbase + c) * Nw + wrow] = s == 0.f ? 0 : f32_to_e4m3(hv[c] / s);
            if (et == 0) out_s[static_cast<size_t>(rowbase + c) * nI + ti.m] = s;
          }
        }
        epilogue_bar();   // red[] is reused by the next tile
      } else {
#pragma unroll
        for (int c = 0; c < BN; ++c) {
          if (c < valid) {
            const __nv_bfloat16 hb = __float2bfloat16_rn(acc_g[c]);
            out_bf16[static_cast<size_t>(rowbase + c) * Nw + wrow] = *reinterpret_cast<const uint16_t*>(&hb);
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, kTmemCols);
}

// ---------------------------------------------------------------------------
// Host
// ---------------------------------------------------------------------------
static bool make_map_u8(CUtensorMap* m, const void* base, uint64_t K, uint64_t rows, uint64_t slots,
                        uint64_t slot_pitch, uint32_t box_rows) {
  return make_map_sw128(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, base, K, rows, K, slots, slot_pitch, box_rows);
}

template <int BN, bool GATED>
static cudaError_t launch_fp8(const CUtensorMap& mA, const CUtensorMap& mAsh, const CUtensorMap& mB,
                              const FfnArgs& a, int K, int Nw, int up_row0, size_t wscale_off, const float* sact,
                              uint8_t* out_q, float* out_s, uint16_t* out_bf16, cudaStream_t st) {
  constexpr uint32_t kBBytes = ((BN * 128 + 1023) / 1024) * 1024;
  constexpr uint32_t kStageBytes = kATileBytes * (GATED ? 2 : 1) + kBBytes;
  int stages = (200 * 1024 - 1024) / static_cast<int>(kStageBytes);
  if (stages > 8) stages = 8;
  const size_t smem = 1024 + static_cast<size_t>(stages) * kStageBytes;
  auto kern = ffn_fp8_kernel<BN, GATED>;
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (err != cudaSuccess) return err;
  const int P = a.T * a.k;
  const int G = a.E + (a.has_shared ? 1 : 0);
  const long max_tiles = static_cast<long>((P + BN - 1) / BN + G) * (Nw / 128);
  const int grid = static_cast<int>(max_tiles < num_sms() ? max_tiles : num_sms());
  return launch_pdl(kern, dim3(grid), dim3(kTcThreads), smem, st, mA, mAsh, mB, a.offsets, a.slot_of_expert, a.E,
                    a.has_shared, a.T, P, K, Nw, up_row0, a.pool, a.shared_bank, a.bank_bytes, wscale_off, sact, out_q,
                    out_s, out_bf16, stages);
}

template <bool GATED>
static cudaError_t launch_fp8_bn(int bn, const CUtensorMap& mA, const CUtensorMap& mAsh, const CUtensorMap& mB,
                                 const FfnArgs& a, int K, int Nw, int up_row0, size_t wscale_off, const float* sact,
                                 uint8_t* out_q, float* out_s, uint16_t* out_bf16, cudaStream_t st) {
  if (bn <= 16)
    return launch_fp8<16, GATED>(mA, mAsh, mB, a, K, Nw, up_row0, wscale_off, sact, out_q, out_s, out_bf16, st);
  return launch_fp8<32, GATED>(mA, mAsh, mB, a, K, Nw, up_row0, wscale_off, sact, out_q, out_s, out_bf16, st);
}

// Workspace: Xq [rows][d] | sx [rows][d/128] | Hq [rows][I] | sh [rows][I/128] (256-byte aligned parts).
size_t fp8_ffn_workspace_bytes(int64_t rows, int d, int I) {
  auto al = [](size_t b) { return (b + 255) & ~static_cast<size_t>(255); };
  return al(rows * d) + al(rows * (d / 128) * 4) + al(rows * I) + al(rows * (I / 128) * 4);
}

const char* launch_expert_ffn_fp8(const FfnArgs& a, size_t s_gu_off, size_t s_d_off, uint8_t* ws, cudaStream_t st,
                                  cudaError_t* cerr) {
  auto al = [](size_t b) { return (b + 255) & ~static_cast<size_t>(255); };
  const int P = a.T * a.k;
  const int rows = P + (a.has_shared ? a.T : 0);
  *cerr = cudaSuccess;
  if (rows == 0) return nullptr;
  if (a.d / 128 > kF8MaxKB || a.I / 128 > kF8MaxKB) return "FP8 FFN supports d, I <= 8192";
  uint8_t* xq = ws;
  float* sx = reinterpret_cast<float*>(xq + al(static_cast<size_t>(rows) * a.d));
  uint8_t* hq = reinterpret_cast<uint8_t*>(sx) + al(static_cast<size_t>(rows) * (a.d / 128) * 4);
  float* sh = reinterpret_cast<float*>(hq + al(static_cast<size_t>(rows) * a.I));
  {
    const long warps = static_cast<long>(rows) * (a.d / 128);
    const int grid = static_cast<int>(warps / 8 + 1 < 148 * 16 ? warps / 8 + 1 : 148 * 16);
    prof_mark(FTM_K_GATHER, st, false);
    *cerr = launch_pdl(gather_quant_fp8_kernel, dim3(grid), dim3(256), 0, st, reinterpret_cast<const uint16_t*>(a.x),
                       a.perm, P, a.k, a.T, a.has_shared, a.d, xq, sx);
    prof_mark(FTM_K_GATHER, st, true);
    if (*cerr != cudaSuccess) return "fp8 gather launch failed";
  }
  const int per = (P + a.E - 1) / a.E;
  const int bn = per <= 16 ? 16 : 32;
  CUtensorMap mA1, mAsh1, mB1, mA2, mAsh2, mB2;
  const uint64_t S = static_cast<uint64_t>(a.S);
  bool ok = make_map_u8(&mA1, a.pool + a.w_gu_off, a.d, 2ull * a.I, S, a.bank_bytes, 128) &&
            make_map_u8(&mA2, a.pool + a.w_d_off, a.I, a.d, S, a.bank_bytes, 128) &&
            make_map_u8(&mB1, xq, a.d, rows, 0, 0, bn) && make_map_u8(&mB2, hq, a.I, rows, 0, 0, bn);
  if (ok && a.has_shared) {
    ok = make_map_u8(&mAsh1, a.shared_bank + a.w_gu_off, a.d, 2ull * a.I, 0, 0, 128) &&
         make_map_u8(&mAsh2, a.shared_bank + a.w_d_off, a.I, a.d, 0, 0, 128);
  } else {
    mAsh1 = mA1;
    mAsh2 = mA2;
  }
  if (!ok) return "cuTensorMapEncodeTiled failed";
  prof_mark(FTM_K_GEMM1, st, false);
  *cerr = launch_fp8_bn<true>(bn, mA1, mAsh1, mB1, a, a.d, a.I, a.I, s_gu_off, sx, hq, sh, nullptr, st);
  prof_mark(FTM_K_GEMM1, st, true);
  if (*cerr != cudaSuccess) return "fp8 gemm1 launch failed";
  prof_mark(FTM_K_GEMM2, st, false);
  *cerr = launch_fp8_bn<false>(bn, mA2, mAsh2, mB2, a, a.I, a.d, 0, s_d_off, sh, nullptr, nullptr,
                               reinterpret_cast<uint16_t*>(a.y), st);
  prof_mark(FTM_K_GEMM2, st, true);
  if (*cerr != cudaSuccess) return "fp8 gemm2 launch failed";
  return nullptr;
}

}  // namespace ftm
