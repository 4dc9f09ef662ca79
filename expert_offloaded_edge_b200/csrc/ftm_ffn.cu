// Grouped SwiGLU expert FFN over the slot-indexed expert pool (steps a5-a7).
//
// Rows of the permuted activation matrix X_p are grouped by expert (group e =
// rows offsets[e]..offsets[e+1]); the shared expert, when present, is one more
// group over all T tokens (rows P..P+T-1).  Expert e's weights are the bank
// slot_pool[slot_of_expert[e]]; the kernel never copies weights.
//
//   GEMM1 (+SwiGLU): H[r][i] = silu(X_p[r] . Wg[i]) * (X_p[r] . Wu[i])
//   GEMM2          : Y[r][j] = H[r] . Wd[j]
//
// bf16 layers run the tensor-core kernel below: weights on the MMA M side
// (128 weight rows per tile), tokens on the N side (BN tokens per tile), so a
// decode-sized group of a few tokens still streams full 128-row weight tiles
// (the decode step is bound by the expert weight bytes).  Persistent CTAs walk
// a (group, weight tile, token tile) list; warp 0 issues TMA loads (weights via
// a 3-D tensor map whose third coordinate is the slot), warp 1 issues tcgen05
// MMAs into a double-buffered TMEM accumulator, warps 2-5 drain TMEM, apply
// SwiGLU and store.  fp32 layers run a plain SIMT kernel; FP8 layers run the
// block-scaled kernel in ftm_ffn_fp8.cu.
#include "ftm_gemm.cuh"

namespace ftm {

__device__ int32_t g_dev_status = 0;

// ---------------------------------------------------------------------------
// Gather: X_p[pos] = x[perm[pos] / k] (pos < P); X_p[P + t] = x[t] (shared rows).
// One warp per row (grid-strided); each lane moves up to 8 of the row's
// 16-byte vectors per round, all loads of a round issued before its stores.
__global__ void __launch_bounds__(256) gather_rows_kernel(const uint8_t* __restrict__ x,
                                                          const int32_t* __restrict__ perm, int P, int k, int T,
                                                          int has_shared, int row_bytes, uint8_t* __restrict__ xp) {
  pdl_wait();
  pdl_trigger();
  const int rows = P + (has_shared ? T : 0);
  const int nv = row_bytes / 16;
  const int lane = threadIdx.x & 31;
  const int wpb = blockDim.x >> 5;
  for (int r = blockIdx.x * wpb + (threadIdx.x >> 5); r < rows; r += gridDim.x * wpb) {
    const int q = r < P ? perm[r] : 0;
    if (q < 0) continue;     // no pair placed here (ids out of range); no group reads this row
    const int src = r < P ? q / k : r - P;
    const uint4* s = reinterpret_cast<const uint4*>(x + static_cast<size_t>(src) * row_bytes);
    uint4* dd = reinterpret_cast<uint4*>(xp + static_cast<size_t>(r) * row_bytes);
    for (int c0 = 0; c0 < nv; c0 += 32 * 8) {
      uint4 v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int c = c0 + u * 32 + lane;
        if (c < nv) v[u] = s[c];
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int c = c0 + u * 32 + lane;
        if (c < nv) dd[c] = v[u];
      }
    }
  }
}

// group of row r (binary search over offsets[0..E]); r >= P -> shared group E.
__device__ __forceinline__ int group_of_row(const int32_t* offsets, int E, int P, int r) {
  if (r >= P) return E;
  int lo = 0, hi = E;  // offsets[lo] <= r < offsets[hi]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (offsets[mid] <= r) lo = mid; else hi = mid;
  }
  return lo;
}

// ---------------------------------------------------------------------------
// SIMT path (fp32 layers): one warp per output element, lanes split the dot.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) simt_gemm1_kernel(const float* __restrict__ xp, const int32_t* __restrict__ offsets,
                                                         const int32_t* __restrict__ slot_of_expert, int E, int P,
                                                         int d, int I, const uint8_t* __restrict__ pool,
                                                         const uint8_t* __restrict__ shared_bank, size_t bank_bytes,
                                                         size_t wgu_off, float* __restrict__ h) {
  pdl_wait();
  pdl_trigger();
  const int r = blockIdx.x;
  const int g = group_of_row(offsets, E, P, r);
  const float* W = reinterpret_cast<const float*>(
      (g < E ? pool + static_cast<size_t>(slot_of_expert[g]) * bank_bytes : shared_bank) + wgu_off);
  const float* x = xp + static_cast<size_t>(r) * d;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  for (int i = blockIdx.y * 8 + warp; i < I; i += gridDim.y * 8) {
    const float* wg = W + static_cast<size_t>(i) * d;
    const float* wu = W + static_cast<size_t>(I + i) * d;
    float a = 0.f, b = 0.f;
    for (int c = lane; c < d; c += 32) { a = fmaf(x[c], wg[c], a); b = fmaf(x[c], wu[c], b); }
    a = warp_sum(a);
    b = warp_sum(b);
    if (lane == 0) h[static_cast<size_t>(r) * I + i] = silu(a) * b;
  }
}

__global__ void __launch_bounds__(256) simt_gemm2_kernel(const float* __restrict__ h, const int32_t* __restrict__ offsets,
                                                         const int32_t* __restrict__ slot_of_expert, int E, int P,
                                                         int d, int I, const uint8_t* __restrict__ pool,
                                                         const uint8_t* __restrict__ shared_bank, size_t bank_bytes,
                                                         size_t wd_off, float* __restrict__ y) {
  pdl_wait();
  pdl_trigger();
  const int r = blockIdx.x;
  const int g = group_of_row(offsets, E, P, r);
  const float* W = reinterpret_cast<const float*>(
      (g < E ? pool + static_cast<size_t>(slot_of_expert[g]) * bank_bytes : shared_bank) + wd_off);
  const float* hr = h + static_cast<size_t>(r) * I;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  for (int j = blockIdx.y * 8 + warp; j < d; j += gridDim.y * 8) {
    const float* wd = W + static_cast<size_t>(j) * I;
    float a = 0.f;
    for (int c = lane; c < I; c += 32) a = fmaf(hr[c], wd[c], a);
    a = warp_sum(a);
    if (lane == 0) y[static_cast<size_t>(r) * d + j] = a;
  }
}

// ---------------------------------------------------------------------------
// Tensor-core path (bf16): persistent warp-specialised tcgen05 grouped GEMM.
// ---------------------------------------------------------------------------
constexpr int kBK = 64;               // K per stage: 64 bf16 = one 128-byte swizzle row

template <int BN, bool GATED>
__global__ void __launch_bounds__(kTcThreads, 1)
    ffn_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmAsh,
                  const __grid_constant__ CUtensorMap tmB, const int32_t* __restrict__ offsets,
                  const int32_t* __restrict__ slot_of_expert, int E, int has_shared, int T, int P, int K, int Nw,
                  int up_row0, uint16_t* __restrict__ out, int ld_out, int stages) {
  constexpr uint32_t kBBytes = ((BN * 128 + 1023) / 1024) * 1024;
  constexpr uint32_t kStageBytes = kATileBytes * (GATED ? 2 : 1) + kBBytes;
  constexpr uint32_t kTx = kATileBytes * (GATED ? 2 : 1) + BN * 128;
  constexpr uint32_t kAccCols = GATED ? 2 * BN : BN;
  constexpr uint32_t kTmemCols = 2 * kAccCols < 32 ? 32 : 2 * kAccCols;
  constexpr uint32_t kIdesc = idesc_bf16_f32(128, BN);
  constexpr int kRedStride = GATED ? 36 : 20;     // floats per thread row of a split-K partial chunk

  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full_bar[8], empty_bar[8], tfull_bar[2], tempty_bar[2], red_full, red_empty;
  __shared__ uint32_t tmem_holder;
  __shared__ int32_t tile_start[kMaxGroups + 1], grp_rows[kMaxGroups], grp_row0[kMaxGroups];

  const uint32_t smem_base = (smem_u32(smem_raw) + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (smem_base - smem_u32(smem_raw));
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int G = E + (has_shared ? 1 : 0);
  const int MT = Nw / 128;
  const int KB = K / kBK;
  // Split-K: a cluster of ks CTAs shares each tile, rank kr accumulating
  // k-blocks [kb0, kb1); the other ranks hand their partial sums to rank 0
  // through its shared memory, and rank 0 adds them in rank order (so the
  // result does not depend on timing) and runs the epilogue.
  const int ks = static_cast<int>(cluster_nranks());
  const int kr = static_cast<int>(cluster_rank());
  const int kb0 = kr * KB / ks, kb1 = (kr + 1) * KB / ks;
  const int cl = blockIdx.x / ks, ncl = gridDim.x / ks;
  float* red = reinterpret_cast<float*>(smem + static_cast<size_t>(stages) * kStageBytes);

  if (threadIdx.x == 0) {
    for (int s = 0; s < stages; ++s) { mbar_init(&full_bar[s], 1); mbar_init(&empty_bar[s], 1); }
    for (int a = 0; a < 2; ++a) { mbar_init(&tfull_bar[a], 1); mbar_init(&tempty_bar[a], 4); }
    mbar_init(&red_full, 128 * (ks - 1 > 0 ? ks - 1 : 1));
    mbar_init(&red_empty, 128);
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
  if (ks > 1) cluster_sync_all();   // every rank's barriers exist before any remote arrival
  else __syncthreads();
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
      for (int t = cl; t < total && ok; t += ncl) {
        const TileInfo ti = decode_tile(t, tile_start, grp_rows, grp_row0, G, BN);
        const int slot = ti.g < E ? slot_of_expert[ti.g] : 0;
        const int brow = ti.row0 + ti.n * BN;
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(&empty_bar[stage], phase ^ 1u)) { ok = false; break; }
          mbar_arrive_expect_tx(&full_bar[stage], kTx);
          if (ti.g < E) {
            tma_load_3d(a_tile(stage, 0), &tmA, &full_bar[stage], kb * kBK, ti.m * 128, slot);
            if (GATED) tma_load_3d(a_tile(stage, 1), &tmA, &full_bar[stage], kb * kBK, up_row0 + ti.m * 128, slot);
          } else {
            tma_load_2d(a_tile(stage, 0), &tmAsh, &full_bar[stage], kb * kBK, ti.m * 128);
            if (GATED) tma_load_2d(a_tile(stage, 1), &tmAsh, &full_bar[stage], kb * kBK, up_row0 + ti.m * 128);
          }
          tma_load_2d(b_tile(stage), &tmB, &full_bar[stage], kb * kBK, brow);
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
      for (int t = cl; t < total && ok; t += ncl, ++it) {
        const int ab = it & 1;
        const uint32_t aphase = (it >> 1) & 1;
        if (!mbar_wait(&tempty_bar[ab], aphase ^ 1u)) break;
        tc_fence_after();
        const uint32_t d_g = tmem_base + ab * kAccCols;
        const uint32_t d_u = d_g + BN;
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(&full_bar[stage], phase)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sa = smem_u32(a_tile(stage, 0));
          const uint32_t sb = smem_u32(b_tile(stage));
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk) {
            const uint64_t bdesc = smem_desc_sw128(sb + kk * 32);
            const uint32_t acc = (kb != kb0 || kk != 0) ? 1u : 0u;
            umma_f16(d_g, smem_desc_sw128(sa + kk * 32), bdesc, kIdesc, acc);
            if (GATED) umma_f16(d_u, smem_desc_sw128(sa + kATileBytes + kk * 32), bdesc, kIdesc, acc);
          }
          umma_commit(&empty_bar[stage]);
          if (++stage == stages) { stage = 0; phase ^= 1u; }
        }
        if (ok) umma_commit(&tfull_bar[ab]);
      }
    }
    __syncwarp();
  } else {
    const int q = warp % 4;  // TMEM lane quadrant this warp may access
    const int er = q * 32 + lane;  // accumulator row (TMEM lane) of this thread
    // split-K exchange: rank r > 0 writes its chunk into slot r - 1 of rank 0's buffer
    const uint32_t red_slot = kr > 0 ? mapa_rank(smem_u32(red + ((kr - 1) * 128 + er) * kRedStride), 0) : 0u;
    uint32_t chunk = 0;  // partial-sum chunks exchanged so far (parity of red_full / red_empty)
    bool ok = true;
    int it = 0;
    for (int t = cl; t < total && ok; t += ncl, ++it) {
      const TileInfo ti = decode_tile(t, tile_start, grp_rows, grp_row0, G, BN);
      const int ab = it & 1;
      const uint32_t aphase = (it >> 1) & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(&tfull_bar[ab], aphase))) break;
      tc_fence_after();
      const int valid = min(BN, ti.rows - ti.n * BN);
      const int wrow = ti.m * 128 + er;
      const uint32_t tb = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + ab * kAccCols;
      uint16_t* obase = out + static_cast<size_t>(ti.row0 + ti.n * BN) * ld_out + wrow;
      for (int c0 = 0; c0 < valid; c0 += 16, ++chunk) {
        float a[16], b[16];
        tmem_ld16(tb + c0, a);
        if (GATED) tmem_ld16(tb + BN + c0, b);
        tmem_ld_wait();
        if (ks > 1) {
          const uint32_t ph = chunk & 1u;
          if (kr > 0) {
            // hand the partial chunk to rank 0 once it has consumed the previous one
            if (!__all_sync(0xffffffffu, mbar_wait_cl(&red_empty, ph ^ 1u))) { ok = false; break; }
#pragma unroll
            for (int j = 0; j < 16; j += 4) {
              st_cluster_v4(red_slot + 4u * j, a[j], a[j + 1], a[j + 2], a[j + 3]);
              if (GATED) st_cluster_v4(red_slot + 4u * (16 + j), b[j], b[j + 1], b[j + 2], b[j + 3]);
            }
            mbar_arrive_remote(mapa_rank(smem_u32(&red_full), 0));
            continue;
          }
          if (!__all_sync(0xffffffffu, mbar_wait_cl(&red_full, ph))) { ok = false; break; }
          for (int r = 1; r < ks; ++r) {
            const float4* pr = reinterpret_cast<const float4*>(red + ((r - 1) * 128 + er) * kRedStride);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const float4 u = pr[j];
              a[4 * j] += u.x; a[4 * j + 1] += u.y; a[4 * j + 2] += u.z; a[4 * j + 3] += u.w;
              if (GATED) {
                const float4 w = pr[4 + j];
                b[4 * j] += w.x; b[4 * j + 1] += w.y; b[4 * j + 2] += w.z; b[4 * j + 3] += w.w;
              }
            }
          }
          for (int r = 1; r < ks; ++r) mbar_arrive_remote(mapa_rank(smem_u32(&red_empty), static_cast<uint32_t>(r)));
        }
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          if (c0 + j < valid) {
            const float v = GATED ? silu(a[j]) * b[j] : a[j];
            const __nv_bfloat16 hv = __float2bfloat16_rn(v);
            obase[static_cast<size_t>(c0 + j) * ld_out] = *reinterpret_cast<const uint16_t*>(&hv);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty_bar[ab]);
    }
  }
  tc_fence_before();
  __syncwarp();
  if (ks > 1) cluster_sync_all();   // no rank leaves while another may still write to or signal it
  else __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, kTmemCols);
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------
// bf16 K-major map: dims {K, rows[, slots]}, box {64, box_rows[, 1]}, 128-byte swizzle.
static bool make_map_bf16(CUtensorMap* m, const void* base, uint64_t K, uint64_t rows, uint64_t row_pitch,
                          uint64_t slots, uint64_t slot_pitch, uint32_t box_rows) {
  return make_map_sw128(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, K, rows, row_pitch, slots, slot_pitch,
                        box_rows);
}

// Upper bound on the tiles of a launch, from sizes alone: at most min(E, P)
// routed groups are non-empty and their token tiles number at most
// min(P, ceil(P / BN) + groups); the shared expert adds ceil(T / BN).
static long tile_bound(int P, int T, int E, int has_shared, int BN, int MT) {
  const long groups = E < P ? E : P;
  long routed = (P + BN - 1) / BN + groups;
  if (routed > P) routed = P;
  return (routed + (has_shared ? (T + BN - 1) / BN : 0)) * MT;
}

template <int BN, bool GATED>
static cudaError_t launch_tc(const CUtensorMap& mA, const CUtensorMap& mAsh, const CUtensorMap& mB,
                             const FfnArgs& a, int K, int Nw, int up_row0, uint16_t* out, int ld_out,
                             cudaStream_t st) {
  constexpr uint32_t kBBytes = ((BN * 128 + 1023) / 1024) * 1024;
  constexpr uint32_t kStageBytes = kATileBytes * (GATED ? 2 : 1) + kBBytes;
  constexpr int kRedStride = GATED ? 36 : 20;
  const int P = a.T * a.k;
  const long tiles = tile_bound(P, a.T, a.E, a.has_shared, BN, Nw / 128);
  const int KB = K / kBK;
  auto kern = ffn_tc_kernel<BN, GATED>;
  auto stages_for = [](int ks) {
    const int red_bytes = (ks - 1) * 128 * kRedStride * 4;
    const int s = (200 * 1024 - 1024 - red_bytes) / static_cast<int>(kStageBytes);
    return s > 8 ? 8 : s;
  };
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(kTcThreads);
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  // Split-K when the tiles cannot fill the GPU: a cluster of ks CTAs per tile,
  // the largest ks <= 4 (and <= the k-blocks) whose clusters all fit at once
  // (one wave: a second wave of clusters would double the kernel time).  When
  // one CTA per SM leaves too few clusters, a configuration with fewer stages
  // lets two CTAs share an SM (only when twice their tensor memory fits).
  constexpr uint32_t kAccCols = GATED ? 2 * BN : BN;
  constexpr uint32_t kTmemCols = 2 * kAccCols < 32 ? 32 : 2 * kAccCols;
  auto smem_of = [&](int ks, int st) {
    return 1024 + static_cast<size_t>(st) * kStageBytes + static_cast<size_t>(ks - 1) * 128 * kRedStride * 4;
  };
  auto stages_two_per_sm = [&](int ks) {       // stages that fit half an SM's shared memory
    const int budget = 113 * 1024 - 1024 - (ks - 1) * 128 * kRedStride * 4;
    const int st = budget / static_cast<int>(kStageBytes);
    return st < stages_for(ks) ? st : stages_for(ks);
  };
  static int max_clusters[5][2] = {};   // co-resident clusters of ks CTAs, per ks and config (1 or 2 CTAs per SM)
  auto clusters = [&](int c, int two) -> int {
    if (!max_clusters[c][two]) {
      const int st = two ? stages_two_per_sm(c) : stages_for(c);
      const size_t sm = smem_of(c, st);
      cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(sm));
      int n = 0;
      if (e == cudaSuccess) {
        attr[0].val.clusterDim.x = c;
        cfg.numAttrs = 1;
        cfg.dynamicSmemBytes = sm;
        cfg.gridDim = dim3(num_sms() / c * c);
        if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n <= 0) n = 0;
      }
      (void)cudaGetLastError();
      max_clusters[c][two] = n > 0 ? n : -1;
    }
    return max_clusters[c][two];
  };
  int ks = 1, stages = stages_for(1);
  if (tiles > 0 && tiles < num_sms()) {
    for (int c = 4; c >= 2 && ks == 1; --c) {
      if (c > KB) continue;
      if (2 * tiles <= num_sms() && c * tiles <= num_sms() && tiles <= clusters(c, 0)) {
        ks = c;
        stages = stages_for(c);
      } else if (2 * kTmemCols <= 512 && stages_two_per_sm(c) >= 3 && c * tiles <= 2 * num_sms() &&
                 tiles <= clusters(c, 1)) {
        ks = c;
        stages = stages_two_per_sm(c);
      }
    }
  }
  const size_t smem = smem_of(ks, stages);
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (err != cudaSuccess) return err;
  if (ks == 1) {
    const int grid = static_cast<int>(tiles < num_sms() ? tiles : num_sms());
    return launch_pdl(kern, dim3(grid), dim3(kTcThreads), smem, st, mA, mAsh, mB, a.offsets, a.slot_of_expert, a.E,
                      a.has_shared, a.T, P, K, Nw, up_row0, out, ld_out, stages);
  }
  attr[0].val.clusterDim.x = ks;
  cfg.dynamicSmemBytes = smem;
  cfg.gridDim = dim3(static_cast<unsigned>(tiles * ks));
  cfg.numAttrs = 2;
  return count_launch(cudaLaunchKernelEx(&cfg, kern, mA, mAsh, mB, a.offsets, a.slot_of_expert, a.E, a.has_shared, a.T, P, K, Nw,
                            up_row0, out, ld_out, stages));
}

template <bool GATED>
static cudaError_t launch_tc_bn(int bn, const CUtensorMap& mA, const CUtensorMap& mAsh, const CUtensorMap& mB,
                                const FfnArgs& a, int K, int Nw, int up_row0, uint16_t* out, int ld_out,
                                cudaStream_t st) {
  switch (bn) {
    case 16: return launch_tc<16, GATED>(mA, mAsh, mB, a, K, Nw, up_row0, out, ld_out, st);
    case 32: return launch_tc<32, GATED>(mA, mAsh, mB, a, K, Nw, up_row0, out, ld_out, st);
    case 64: return launch_tc<64, GATED>(mA, mAsh, mB, a, K, Nw, up_row0, out, ld_out, st);
    case 128: return launch_tc<128, GATED>(mA, mAsh, mB, a, K, Nw, up_row0, out, ld_out, st);
    default:
      // 256-token tiles only without the gate/up pair (TMEM holds 2 x 256 fp32 columns)
      if (GATED) return launch_tc<128, GATED>(mA, mAsh, mB, a, K, Nw, up_row0, out, ld_out, st);
      return launch_tc<256, false>(mA, mAsh, mB, a, K, Nw, up_row0, out, ld_out, st);
  }
}

bool tc2_applicable(int P, int E, int I, int d);
const char* launch_ffn_gemms_tc2(const FfnArgs& a, int rows, cudaStream_t st, cudaError_t* cerr);

int ffn_token_tile(int P, int E) {
  const int per = (P + E - 1) / E;
  return per <= 16 ? 16 : per <= 32 ? 32 : per <= 64 ? 64 : 128;
}

// Returns a message on failure, nullptr on success.
const char* launch_expert_ffn(const FfnArgs& a, cudaStream_t st, cudaError_t* cerr) {
  const int P = a.T * a.k;
  const int rows = P + (a.has_shared ? a.T : 0);
  *cerr = cudaSuccess;
  if (rows == 0) return nullptr;
  const int elt = a.f32 ? 4 : 2;
  {
    const int blocks = (rows + 7) / 8;   // 8 rows (warps) per block
    const int grid = blocks < 148 * 16 ? blocks : 148 * 16;
    prof_mark(FTM_K_GATHER, st, false);
    *cerr = launch_pdl(gather_rows_kernel, dim3(grid), dim3(256), 0, st, a.x, a.perm, P, a.k, a.T, a.has_shared,
                       a.d * elt, a.xp);
    prof_mark(FTM_K_GATHER, st, true);
    if (*cerr != cudaSuccess) return "gather launch failed";
  }
  if (a.f32) {
    dim3 g1(rows, (a.I + 63) / 64), g2(rows, (a.d + 63) / 64);
    prof_mark(FTM_K_GEMM1, st, false);
    *cerr = launch_pdl(simt_gemm1_kernel, g1, dim3(256), 0, st, reinterpret_cast<const float*>(a.xp), a.offsets,
                       a.slot_of_expert, a.E, P, a.d, a.I, a.pool, a.shared_bank, a.bank_bytes, a.w_gu_off,
                       reinterpret_cast<float*>(a.h));
    prof_mark(FTM_K_GEMM1, st, true);
    if (*cerr != cudaSuccess) return "simt gemm1 launch failed";
    prof_mark(FTM_K_GEMM2, st, false);
    *cerr = launch_pdl(simt_gemm2_kernel, g2, dim3(256), 0, st, reinterpret_cast<const float*>(a.h), a.offsets,
                       a.slot_of_expert, a.E, P, a.d, a.I, a.pool, a.shared_bank, a.bank_bytes, a.w_d_off,
                       reinterpret_cast<float*>(a.y));
    prof_mark(FTM_K_GEMM2, st, true);
    if (*cerr != cudaSuccess) return "simt gemm2 launch failed";
    return nullptr;
  }
  // bf16 tensor-core path: CTA pairs for prefill-size groups, single CTAs otherwise
  if (tc2_applicable(P, a.E, a.I, a.d)) return launch_ffn_gemms_tc2(a, rows, st, cerr);
  const int bn = ffn_token_tile(P, a.E);
  const int bn2 = (P + a.E - 1) / a.E >= 192 ? 256 : bn;
  CUtensorMap mA1, mAsh1, mB1, mA2, mAsh2, mB2;
  const uint64_t S = static_cast<uint64_t>(a.S);
  bool ok = make_map_bf16(&mA1, a.pool + a.w_gu_off, a.d, 2ull * a.I, 2ull * a.d, S, a.bank_bytes, 128) &&
            make_map_bf16(&mA2, a.pool + a.w_d_off, a.I, a.d, 2ull * a.I, S, a.bank_bytes, 128) &&
            make_map_bf16(&mB1, a.xp, a.d, rows, 2ull * a.d, 0, 0, bn) &&
            make_map_bf16(&mB2, a.h, a.I, rows, 2ull * a.I, 0, 0, bn2);
  if (ok && a.has_shared) {
    ok = make_map_bf16(&mAsh1, a.shared_bank + a.w_gu_off, a.d, 2ull * a.I, 2ull * a.d, 0, 0, 128) &&
         make_map_bf16(&mAsh2, a.shared_bank + a.w_d_off, a.I, a.d, 2ull * a.I, 0, 0, 128);
  } else {
    mAsh1 = mA1;
    mAsh2 = mA2;
  }
  if (!ok) return "cuTensorMapEncodeTiled failed";
  prof_mark(FTM_K_GEMM1, st, false);
  *cerr = launch_tc_bn<true>(bn, mA1, mAsh1, mB1, a, a.d, a.I, a.I, reinterpret_cast<uint16_t*>(a.h), a.I, st);
  prof_mark(FTM_K_GEMM1, st, true);
  if (*cerr != cudaSuccess) return "tensor-core gemm1 launch failed";
  prof_mark(FTM_K_GEMM2, st, false);
  *cerr = launch_tc_bn<false>(bn2, mA2, mAsh2, mB2, a, a.I, a.d, 0, reinterpret_cast<uint16_t*>(a.y), a.d, st);
  prof_mark(FTM_K_GEMM2, st, true);
  if (*cerr != cudaSuccess) return "tensor-core gemm2 launch failed";
  return nullptr;
}

}  // namespace ftm
