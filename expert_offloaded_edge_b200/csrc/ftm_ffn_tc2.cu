// Prefill-size bf16 grouped GEMMs on CTA pairs (tcgen05 cta_group::2).
//
// A pair of CTAs (a cluster of 2) computes one 256 x 256 tile (a group's last
// token tile may be narrower, see pair_tile_n): the MMA M side
// is 256 weight rows (128 staged by each CTA), the N side 256 tokens (128
// staged by each CTA), so each CTA moves 32 KB per 64-deep K step for 2.1 M
// multiply-adds -- a third less shared-memory fill per flop than the 128 x 256
// single-CTA tile.  The even CTA's MMA thread issues tcgen05.mma.cta_group::2;
// both CTAs' TMA loads complete on the even CTA's barrier; the MMA commit is
// multicast to both CTAs' barriers; each CTA's TMEM holds its 128 weight rows
// for all 256 tokens.
//
// Gate/up GEMM: each CTA's 128 weight rows are 64 gate rows and the matching
// 64 up rows of one 128-wide slice of the intermediate dimension, so SwiGLU
// pairs lane i with lane i + 64 of the same CTA; half of each chunk of gate
// values crosses to the up warps and half of the up values to the gate warps
// through shared memory, so all four epilogue warps share the SwiGLU work.
// Down GEMM: 256 consecutive output rows per pair.
// No TMA multicast: every CTA loads its own tiles.
#include "ftm_gemm.cuh"

namespace ftm {

constexpr int kP2BN = 256;                    // tokens per pair tile (128 per CTA)
constexpr int kP2BK = 64;                     // bf16 K per stage (128-byte rows)
constexpr uint32_t kP2ABytes = 128 * 128;     // 128 weight rows x 64 bf16 per CTA
constexpr uint32_t kP2BBytes = 128 * 128;     // 128 tokens x 64 bf16 per CTA
constexpr uint32_t kP2Stage = kP2ABytes + kP2BBytes;
constexpr int kP2Stages = 6;

// MMA width (tokens) of a pair tile holding `valid` tokens: full tiles use
// N = 256; the last, partial tile of a group shrinks N to the next multiple of
// 32, so a group's ragged tail costs MMA time in proportion to its tokens.
// Columns [0, N/2) come from the even CTA's B rows, [N/2, N) from the odd
// CTA's, so each CTA stages its token rows from tile row rank * N/2.
__device__ __forceinline__ int pair_tile_n(int valid) { return min(kP2BN, (valid + 31) & ~31); }

__device__ __forceinline__ void umma2_f16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

template <bool GATED>
__global__ void __launch_bounds__(kTcThreads, 1)
    ffn_tc2_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmAsh,
                   const __grid_constant__ CUtensorMap tmB, const int32_t* __restrict__ offsets,
                   const int32_t* __restrict__ slot_of_expert, int E, int has_shared, int T, int P, int K, int Nw,
                   int up_row0, uint16_t* __restrict__ out, int ld_out) {
  constexpr uint32_t kTmemCols = 512;              // two 256-column accumulators
  constexpr int kRowsPerPair = GATED ? 128 : 256; // weight-dim extent of a pair tile

  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full_bar[kP2Stages], empty_bar[kP2Stages], tfull_bar[2], tempty_bar[2];
  __shared__ uint32_t tmem_holder;
  __shared__ int32_t tile_start[kMaxGroups + 1], grp_rows[kMaxGroups], grp_row0[kMaxGroups];
  // half-chunks crossing between the gate and up warps, double-buffered
  __shared__ float xbuf[GATED ? 2 * 128 * 17 : 1];
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
  const int KB = K / kP2BK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kP2Stages; ++s) { mbar_init(&full_bar[s], 1); mbar_init(&empty_bar[s], 1); }
    for (int a = 0; a < 2; ++a) { mbar_init(&tfull_bar[a], 1); mbar_init(&tempty_bar[a], 8); }
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
  }
  pdl_wait();
  pdl_trigger();
  build_tile_table(offsets, E, has_shared, T, P, MT, kP2BN, tile_start, grp_rows, grp_row0);
  tc_fence_before();
  cluster_sync_all();     // barriers initialised and TMEM allocated in both CTAs
  tc_fence_after();
  const uint32_t tmem_base = tmem_holder;
  const int total = tile_start[G];

  auto a_tile = [&](int s) -> uint8_t* { return smem + static_cast<size_t>(s) * kP2Stage; };
  auto b_tile = [&](int s) -> uint8_t* { return smem + static_cast<size_t>(s) * kP2Stage + kP2ABytes; };

  if (warp == 0) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int t = pair; t < total && ok; t += npairs) {
        const TileInfo ti = decode_tile(t, tile_start, grp_rows, grp_row0, G, kP2BN);
        const int slot = ti.g < E ? slot_of_expert[ti.g] : 0;
        const int ntile = pair_tile_n(min(kP2BN, ti.rows - ti.n * kP2BN));
        const int brow = ti.row0 + ti.n * kP2BN + static_cast<int>(rank) * (ntile / 2);
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait_cl(&empty_bar[stage], phase ^ 1u)) { ok = false; break; }
          if (leader) mbar_arrive_expect_tx(&full_bar[stage], 2 * kP2Stage);
          const uint32_t lbar = mapa_rank(smem_u32(&full_bar[stage]), 0);   // the even CTA's barrier
          const int kc = kb * kP2BK;
          if (GATED) {
            // 64 gate rows then the matching 64 up rows of this CTA's half of the slice
            const int r0 = ti.m * 128 + static_cast<int>(rank) * 64;
            if (ti.g < E) {
              tma2_load_3d(a_tile(stage), &tmA, lbar, kc, r0, slot);
              tma2_load_3d(a_tile(stage) + 64 * 128, &tmA, lbar, kc, up_row0 + r0, slot);
            } else {
              tma2_load_2d(a_tile(stage), &tmAsh, lbar, kc, r0);
              tma2_load_2d(a_tile(stage) + 64 * 128, &tmAsh, lbar, kc, up_row0 + r0);
            }
          } else {
            const int r0 = ti.m * 256 + static_cast<int>(rank) * 128;
            if (ti.g < E) tma2_load_3d(a_tile(stage), &tmA, lbar, kc, r0, slot);
            else tma2_load_2d(a_tile(stage), &tmAsh, lbar, kc, r0);
          }
          tma2_load_2d(b_tile(stage), &tmB, lbar, kc, brow);
          if (++stage == kP2Stages) { stage = 0; phase ^= 1u; }
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
      for (int t = pair; t < total && ok; t += npairs, ++it) {
        const int ab = it & 1;
        const uint32_t aphase = (it >> 1) & 1;
        const TileInfo ti = decode_tile(t, tile_start, grp_rows, grp_row0, G, kP2BN);
        const uint32_t idesc = idesc_bf16_f32(256, pair_tile_n(min(kP2BN, ti.rows - ti.n * kP2BN)));
        if (!mbar_wait_cl(&tempty_bar[ab], aphase ^ 1u)) break;
        tc_fence_after();
        const uint32_t d = tmem_base + ab * kP2BN;
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait_cl(&full_bar[stage], phase)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sa = smem_u32(a_tile(stage));
          const uint32_t sb = smem_u32(b_tile(stage));
#pragma unroll
          for (int kk = 0; kk < kP2BK / 16; ++kk)
            umma2_f16(d, smem_desc_sw128(sa + kk * 32), smem_desc_sw128(sb + kk * 32), idesc, (kb | kk) != 0 ? 1u : 0u);
          umma2_commit_both(&empty_bar[stage]);
          if (++stage == kP2Stages) { stage = 0; phase ^= 1u; }
        }
        if (ok) umma2_commit_both(&tfull_bar[ab]);
      }
    }
    __syncwarp();
  } else {
    const int q = warp % 4;           // TMEM lane quadrant
    const uint32_t tempty0 = mapa_rank(smem_u32(&tempty_bar[0]), 0);
    const uint32_t tempty1 = mapa_rank(smem_u32(&tempty_bar[1]), 0);
    int it = 0;
    for (int t = pair; t < total; t += npairs, ++it) {
      const TileInfo ti = decode_tile(t, tile_start, grp_rows, grp_row0, G, kP2BN);
      const int ab = it & 1;
      const uint32_t aphase = (it >> 1) & 1;
      if (!epilogue_all(mbar_wait_cl(&tfull_bar[ab], aphase))) break;
      tc_fence_after();
      const int valid = min(kP2BN, ti.rows - ti.n * kP2BN);
      const uint32_t tb = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + ab * kP2BN;
      const size_t rowbase = static_cast<size_t>(ti.row0 + ti.n * kP2BN);
      if (GATED) {
        // Lanes 0-63 hold gate rows, lanes 64-127 the up rows of the same
        // intermediate index i = m*128 + rank*64 + (lane % 64).  Per 32-column
        // chunk, a gate warp hands its upper 16 gate columns to its up warp
        // (quadrant q + 2) and takes that warp's lower 16 up columns, so all
        // four warps evaluate SwiGLU on 16 columns each.  Two buffers: a
        // buffer is rewritten only after the barrier of the next chunk, which
        // every warp reaches after reading it.
        const int ii = ti.m * 128 + static_cast<int>(rank) * 64 + (q % 2) * 32 + lane;
        const bool gate_warp = q < 2;
        const int me = q * 32 + lane, partner = (q ^ 2) * 32 + lane;
        const int col_off = gate_warp ? 0 : 16;      // the half this warp evaluates
        uint16_t* o = out + rowbase * ld_out + ii;
        int buf = 0;
        for (int c0 = 0; c0 < valid; c0 += 32, buf ^= 1) {
          float v[32];
          tmem_ld16(tb + c0, v);
          tmem_ld16(tb + c0 + 16, v + 16);
          tmem_ld_wait();
          float* xb = xbuf + buf * (128 * 17);
#pragma unroll
          for (int j = 0; j < 16; ++j) xb[me * 17 + j] = gate_warp ? v[16 + j] : v[j];
          epilogue_bar();
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int c = c0 + col_off + j;
            if (c < valid) {
              const float other = xb[partner * 17 + j];
              const float h = gate_warp ? silu(v[j]) * other : silu(other) * v[16 + j];
              const __nv_bfloat16 hb = __float2bfloat16_rn(h);
              o[static_cast<size_t>(c) * ld_out] = *reinterpret_cast<const uint16_t*>(&hb);
            }
          }
        }
      } else {
        // lane = output column, TMEM column = token: 32 tokens at a time go through the warp's staging
        // rows so that each store is 16 bytes of one token's row
        const int w0 = ti.m * 256 + static_cast<int>(rank) * 128 + q * 32;
        uint16_t* o = out + rowbase * ld_out + w0;
        uint16_t* yb = ybuf + (warp - 2) * (32 * kYPitch);
        for (int c0 = 0; c0 < valid; c0 += 32) {
          float v[32];
          tmem_ld16(tb + c0, v);
          tmem_ld16(tb + c0 + 16, v + 16);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const __nv_bfloat16 hb = __float2bfloat16_rn(v[j]);
            yb[j * kYPitch + lane] = *reinterpret_cast<const uint16_t*>(&hb);
          }
          __syncwarp();
#pragma unroll
          for (int r = 0; r < 4; ++r) {
            const int j = r * 8 + lane / 4, part = lane % 4;
            if (c0 + j < valid)
              *reinterpret_cast<uint4*>(o + static_cast<size_t>(c0 + j) * ld_out + part * 8) =
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
  cluster_sync_all();     // no CTA leaves while its pair may still signal it
  tc_fence_after();
  if (warp == 1)
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(kTmemCols) : "memory");
}

// Host: launches both GEMMs of a prefill-size bf16 layer on CTA pairs.
bool tc2_applicable(int P, int E, int I, int d) {
  return (P + E - 1) / E >= 192 && I % 128 == 0 && d % 256 == 0;
}

template <bool GATED>
static cudaError_t launch_tc2_one(const CUtensorMap& mA, const CUtensorMap& mAsh, const CUtensorMap& mB,
                                  const FfnArgs& a, int K, int Nw, int up_row0, uint16_t* out, int ld_out,
                                  cudaStream_t st) {
  const size_t smem = 1024 + static_cast<size_t>(kP2Stages) * kP2Stage;
  auto kern = ffn_tc2_kernel<GATED>;
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (err != cudaSuccess) return err;
  const int P = a.T * a.k;
  const int G = a.E + (a.has_shared ? 1 : 0);
  const long tiles = static_cast<long>((P + kP2BN - 1) / kP2BN + G) * (Nw / (GATED ? 128 : 256));
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(kTcThreads);
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
  // one wave of pairs: as many as the GPCs can hold at once (not every SM may find a partner)
  static int pairs_max[2] = {0, 0};
  if (!pairs_max[GATED]) {
    cfg.gridDim = dim3(num_sms());
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n <= 0) {
      (void)cudaGetLastError();
      n = num_sms() / 2;
    }
    pairs_max[GATED] = n < num_sms() / 2 ? n : num_sms() / 2;
  }
  const int pairs = static_cast<int>(tiles < pairs_max[GATED] ? tiles : pairs_max[GATED]);
  cfg.gridDim = dim3(2 * pairs);
  cfg.numAttrs = 2;
  return count_launch(cudaLaunchKernelEx(&cfg, kern, mA, mAsh, mB, a.offsets, a.slot_of_expert, a.E, a.has_shared, a.T, P, K, Nw,
                            up_row0, out, ld_out));
}

static bool map_bf16(CUtensorMap* m, const void* base, uint64_t K, uint64_t rows, uint64_t row_pitch, uint64_t slots,
                     uint64_t slot_pitch, uint32_t box_rows) {
  return make_map_sw128(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, K, rows, row_pitch, slots, slot_pitch,
                        box_rows);
}

const char* launch_ffn_gemms_tc2(const FfnArgs& a, int rows, cudaStream_t st, cudaError_t* cerr) {
  CUtensorMap mA1, mAsh1, mB1, mA2, mAsh2, mB2;
  const uint64_t S = static_cast<uint64_t>(a.S);
  // gate/up weight boxes are 64 rows (a CTA takes 64 gate + 64 up rows); down-weight and token boxes 128
  bool ok = map_bf16(&mA1, a.pool + a.w_gu_off, a.d, 2ull * a.I, 2ull * a.d, S, a.bank_bytes, 64) &&
            map_bf16(&mA2, a.pool + a.w_d_off, a.I, a.d, 2ull * a.I, S, a.bank_bytes, 128) &&
            map_bf16(&mB1, a.xp, a.d, rows, 2ull * a.d, 0, 0, 128) &&
            map_bf16(&mB2, a.h, a.I, rows, 2ull * a.I, 0, 0, 128);
  if (ok && a.has_shared) {
    ok = map_bf16(&mAsh1, a.shared_bank + a.w_gu_off, a.d, 2ull * a.I, 2ull * a.d, 0, 0, 64) &&
         map_bf16(&mAsh2, a.shared_bank + a.w_d_off, a.I, a.d, 2ull * a.I, 0, 0, 128);
  } else {
    mAsh1 = mA1;
    mAsh2 = mA2;
  }
  if (!ok) return "cuTensorMapEncodeTiled failed";
  prof_mark(FTM_K_GEMM1, st, false);
  *cerr = launch_tc2_one<true>(mA1, mAsh1, mB1, a, a.d, a.I, a.I, reinterpret_cast<uint16_t*>(a.h), a.I, st);
  prof_mark(FTM_K_GEMM1, st, true);
  if (*cerr != cudaSuccess) return "pair gemm1 launch failed";
  prof_mark(FTM_K_GEMM2, st, false);
  *cerr = launch_tc2_one<false>(mA2, mAsh2, mB2, a, a.I, a.d, 0, reinterpret_cast<uint16_t*>(a.y), a.d, st);
  prof_mark(FTM_K_GEMM2, st, true);
  if (*cerr != cudaSuccess) return "pair gemm2 launch failed";
  return nullptr;
}

}  // namespace ftm
