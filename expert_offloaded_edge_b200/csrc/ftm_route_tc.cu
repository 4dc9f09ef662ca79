// Router for large token counts on the tensor cores (steps a1, a2), bf16
// layers with E <= 256.
//
// logits = x . Wr^T with tcgen05 kind::f16: 128 tokens on the MMA M side, the
// E router rows on the N side (padded to NE, a multiple of 16; rows past E
// are read as zero), K = 64 per stage, fp32 accumulation in TMEM.  A
// persistent CTA walks 128-token tiles: warp 0 streams x and Wr tiles with
// TMA, warp 1 issues the MMAs into a double-buffered accumulator, and each of
// the four epilogue warps owns 32 tokens: thread i reads its token's E logits
// from TMEM lane i (32 columns per wait), adds the bias and selects the top k
// (one scan with register insertion for k = 2, 4, 6, 8; k passes otherwise),
// then writes the softmax over the k picks.  The picks live in registers; no
// shared-memory staging of logits, no global scratch, one launch.
#include "ftm_gemm.cuh"

namespace ftm {

constexpr int kRtBK = 64;             // K per stage (bf16, one 128-byte swizzle row)
constexpr int kRtBM = 128;            // tokens per tile (the MMA M)
constexpr int kRtMaxK = 16;
constexpr int kRtMaxNE = 256;         // experts (MMA N) at most
constexpr int kRtMaxStages = 8;
constexpr uint32_t kRtXBytes = kRtBM * 128;          // 128 tokens x 64 bf16
// a stage is the x tile and NE router rows x 64 bf16 (NE a multiple of 16, so every tile stays 1024-aligned);
// as many stages as fit 199 KB, at most 8: 6 for E = 128, 5 for E = 160, 4 for E = 256
constexpr uint32_t kRtTmemCols = 2 * kRtMaxNE;       // two accumulators of up to 256 columns

// Gates of one token from its top k (pv descending, pi ids): softmax over the
// k picks, written at row tok.
template <int NK>
__device__ __forceinline__ void write_gates(const float (&pv)[NK], const int (&pi)[NK], int k, int tok, int T,
                                            int32_t* __restrict__ topk_ids, float* __restrict__ topk_w) {
  if (tok >= T) return;
  float ex[NK];
  float sum = 0.f;
#pragma unroll
  for (int j = 0; j < NK; ++j) {
    ex[j] = j < k ? expf(pv[j] - pv[0]) : 0.f;
    sum += ex[j];
  }
#pragma unroll
  for (int j = 0; j < NK; ++j) {
    if (j < k) {
      topk_ids[static_cast<size_t>(tok) * k + j] = pi[j];
      topk_w[static_cast<size_t>(tok) * k + j] = ex[j] / sum;
    }
  }
}

// Route one token (the TMEM lane of the calling thread holds its logits in
// columns [0, NE), read 32 per wait) for a k known at compile time: one scan
// with insertion into a sorted register list.  Experts are visited in
// ascending id and an entry moves only for a strictly larger logit, so equal
// logits keep the lower id first; NaN and -inf logits never enter.
template <int K>
__device__ __forceinline__ void route_token_k(uint32_t tb, int NE, int E, const float* s_bias, int tok, int T,
                                              int32_t* __restrict__ topk_ids, float* __restrict__ topk_w) {
  float pv[K];
  int pi[K];
#pragma unroll
  for (int j = 0; j < K; ++j) { pv[j] = -INFINITY; pi[j] = 0x7FFFFFFF; }
  for (int c0 = 0; c0 < NE; c0 += 32) {
    float v[32];
    tmem_ld16(tb + c0, v);
    if (c0 + 16 < NE) tmem_ld16(tb + c0 + 16, v + 16);
    tmem_ld_wait();
#pragma unroll
    for (int jj = 0; jj < 32; ++jj) {
      const int e = c0 + jj;
      const float val = v[jj] + s_bias[e < kRtMaxNE ? e : 0];
      if (e < E && val > pv[K - 1]) {
        // position j takes the old entry j-1 if val is above it, else val if val is above the old entry j
#pragma unroll
        for (int j = K - 1; j >= 0; --j) {
          if (j > 0 && val > pv[j - 1]) {
            pv[j] = pv[j - 1];
            pi[j] = pi[j - 1];
          } else if (val > pv[j]) {
            pv[j] = val;
            pi[j] = e;
          }
        }
      }
    }
  }
  write_gates<K>(pv, pi, K, tok, T, topk_ids, topk_w);
}

// Any k <= 16: k passes, each taking the largest logit (then lowest id) below
// the previous pick.  Same order and exclusions as route_token_k.
__device__ __forceinline__ void route_token_any(uint32_t tb, int NE, int E, int k, const float* s_bias, int tok,
                                                int T, int32_t* __restrict__ topk_ids, float* __restrict__ topk_w) {
  float pv[kRtMaxK];
  int pi[kRtMaxK];
  float prev_v = INFINITY;
  int prev_e = -1;
#pragma unroll
  for (int p = 0; p < kRtMaxK; ++p) {
    float bv = -INFINITY;
    int be = 0x7FFFFFFF;
    if (p < k) {
      for (int c0 = 0; c0 < NE; c0 += 32) {
        float v[32];
        tmem_ld16(tb + c0, v);
        if (c0 + 16 < NE) tmem_ld16(tb + c0 + 16, v + 16);
        tmem_ld_wait();
#pragma unroll
        for (int jj = 0; jj < 32; ++jj) {
          const int e = c0 + jj;
          const float val = v[jj] + s_bias[e < kRtMaxNE ? e : 0];
          const bool below = val < prev_v || (val == prev_v && e > prev_e);
          if (e < E && below && val > bv) {
            bv = val;
            be = e;
          }
        }
      }
    }
    pv[p] = bv;
    pi[p] = be;
    prev_v = bv;
    prev_e = be;
  }
  write_gates<kRtMaxK>(pv, pi, k, tok, T, topk_ids, topk_w);
}

__global__ void __launch_bounds__(kTcThreads, 1)
    route_tc_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW, int T, int d,
                    const float* __restrict__ bias, int E, int NE, int k, int32_t* __restrict__ topk_ids,
                    float* __restrict__ topk_w, int stages) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full_bar[kRtMaxStages], empty_bar[kRtMaxStages], tfull_bar[2], tempty_bar[2];
  __shared__ uint32_t tmem_holder;
  __shared__ float s_bias[kRtMaxNE];

  const uint32_t smem_base = (smem_u32(smem_raw) + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (smem_base - smem_u32(smem_raw));
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int tiles = (T + kRtBM - 1) / kRtBM;
  const int KB = d / kRtBK;
  const uint32_t tx = kRtXBytes + static_cast<uint32_t>(NE) * 128;
  const uint32_t idesc = idesc_bf16_f32(kRtBM, NE);

  if (threadIdx.x == 0) {
    for (int s = 0; s < stages; ++s) { mbar_init(&full_bar[s], 1); mbar_init(&empty_bar[s], 1); }
    for (int a = 0; a < 2; ++a) { mbar_init(&tfull_bar[a], 1); mbar_init(&tempty_bar[a], 4); }
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&tmem_holder, kRtTmemCols);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmX);
    tma_prefetch_desc(&tmW);
  }
  for (int e = threadIdx.x; e < kRtMaxNE; e += blockDim.x) s_bias[e] = (bias != nullptr && e < E) ? bias[e] : 0.f;
  pdl_wait();
  pdl_trigger();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = tmem_holder;
  const size_t stage_bytes = kRtXBytes + static_cast<size_t>(NE) * 128;
  auto x_tile = [&](int s) -> uint8_t* { return smem + static_cast<size_t>(s) * stage_bytes; };
  auto w_tile = [&](int s) -> uint8_t* { return smem + static_cast<size_t>(s) * stage_bytes + kRtXBytes; };

  if (warp == 0) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x) {
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait(&empty_bar[stage], phase ^ 1u)) { ok = false; break; }
          mbar_arrive_expect_tx(&full_bar[stage], tx);
          tma_load_2d(x_tile(stage), &tmX, &full_bar[stage], kb * kRtBK, t * kRtBM);
          tma_load_2d(w_tile(stage), &tmW, &full_bar[stage], kb * kRtBK, 0);
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
      for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x, ++it) {
        const int ab = it & 1;
        const uint32_t aphase = (it >> 1) & 1;
        if (!mbar_wait(&tempty_bar[ab], aphase ^ 1u)) break;
        tc_fence_after();
        const uint32_t dacc = tmem_base + ab * kRtMaxNE;
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait(&full_bar[stage], phase)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sx = smem_u32(x_tile(stage)), sw = smem_u32(w_tile(stage));
#pragma unroll
          for (int kk = 0; kk < kRtBK / 16; ++kk)
            umma_f16(dacc, smem_desc_sw128(sx + kk * 32), smem_desc_sw128(sw + kk * 32), idesc,
                     (kb | kk) != 0 ? 1u : 0u);
          umma_commit(&empty_bar[stage]);
          if (++stage == stages) { stage = 0; phase ^= 1u; }
        }
        if (ok) umma_commit(&tfull_bar[ab]);
      }
    }
    __syncwarp();
  } else {
    const int q = warp % 4;           // TMEM lane quadrant: tokens q*32 .. q*32+31 of the tile
    int it = 0;
    for (int t = blockIdx.x; t < tiles; t += gridDim.x, ++it) {
      const int ab = it & 1;
      const uint32_t aphase = (it >> 1) & 1;
      if (!epilogue_all(mbar_wait(&tfull_bar[ab], aphase))) break;
      tc_fence_after();
      const uint32_t tb = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + ab * kRtMaxNE;
      const int tok = t * kRtBM + q * 32 + lane;
      switch (k) {
        case 8: route_token_k<8>(tb, NE, E, s_bias, tok, T, topk_ids, topk_w); break;
        case 6: route_token_k<6>(tb, NE, E, s_bias, tok, T, topk_ids, topk_w); break;
        case 4: route_token_k<4>(tb, NE, E, s_bias, tok, T, topk_ids, topk_w); break;
        case 2: route_token_k<2>(tb, NE, E, s_bias, tok, T, topk_ids, topk_w); break;
        default: route_token_any(tb, NE, E, k, s_bias, tok, T, topk_ids, topk_w); break;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty_bar[ab]);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, kRtTmemCols);
}

// true when the tensor-core router handles this call (bf16, E <= 256, enough
// tokens for 16 or more 128-token tiles; smaller batches use the cluster router)
bool route_tc_applicable(bool f32, int T, int E, int k) { return !f32 && E <= kRtMaxNE && k <= kRtMaxK && T >= 2048; }

cudaError_t launch_route_tc(const void* x, int T, int d, const void* wr, const float* bias, int E, int k,
                            int32_t* ids, float* w, cudaStream_t st) {
  const int NE = (E + 15) / 16 * 16;
  CUtensorMap mX, mW;
  if (!make_map_sw128(&mX, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, x, d, T, 2ull * d, 0, 0, kRtBM) ||
      !make_map_sw128(&mW, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, wr, d, E, 2ull * d, 0, 0, NE))
    return cudaErrorInvalidValue;
  const int tiles = (T + kRtBM - 1) / kRtBM;
  const int grid = tiles < num_sms() ? tiles : num_sms();
  const size_t stage_bytes = kRtXBytes + static_cast<size_t>(NE) * 128;
  int stages = static_cast<int>((199 * 1024) / stage_bytes);
  if (stages > kRtMaxStages) stages = kRtMaxStages;
  const size_t smem = 1024 + static_cast<size_t>(stages) * stage_bytes;
  cudaError_t e = cudaFuncSetAttribute(route_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  return launch_pdl(route_tc_kernel, dim3(grid), dim3(kTcThreads), smem, st, mX, mW, T, d, bias, E, NE, k, ids, w,
                    stages);
}

}  // namespace ftm
