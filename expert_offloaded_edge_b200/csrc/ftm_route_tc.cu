// Router for large token counts on the tensor cores (steps a1, a2), bf16
// layers with E <= 256.
//
// logits^T = Wr . x^T with tcgen05 kind::f16: the router rows are the MMA M
// side (one or two 128-row tiles, rows past E read as zero), tokens the N side
// (64 or 128 per tile), fp32 accumulation in TMEM.  A persistent CTA walks token
// tiles: warp 0 streams Wr and x tiles with TMA, warp 1 issues the MMAs into a
// double-buffered accumulator, and the four epilogue warps move the logits
// (+ bias) into shared memory as [token][expert] and then pick the top k of
// each token with a warp-wide argmax per pick (ties to the lower id) followed
// by the softmax over the picks.  No global scratch, one launch.
#include "ftm_gemm.cuh"

namespace ftm {

constexpr int kRtBK = 64;          // K per stage (bf16, one 128-byte swizzle row)
constexpr int kRtMaxK = 16;
constexpr int kRtHalf = 64;        // tokens whose logits the epilogue stages in shared memory at a time

// MA: number of 128-row router tiles (E <= 128 * MA); kRtBN: tokens per tile
// (an MMA costs about the same for any N <= 256, so large batches take 128)
template <int MA, int kRtStages, int kRtBN>
__global__ void __launch_bounds__(kTcThreads, 1)
    route_tc_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX, int T, int d,
                    const float* __restrict__ bias, int E, int k, int32_t* __restrict__ topk_ids,
                    float* __restrict__ topk_w) {
  constexpr uint32_t kWBytes = 128 * 128;                  // 128 rows x 64 bf16
  constexpr uint32_t kXBytes = kRtBN * 128;                // kRtBN rows x 64 bf16
  constexpr uint32_t kStageBytes = MA * kWBytes + kXBytes;
  constexpr uint32_t kAccCols = MA * kRtBN;
  constexpr uint32_t kTmemCols = 2 * kAccCols;              // 256 or 512
  constexpr uint32_t kIdesc = idesc_bf16_f32(128, kRtBN);
  constexpr int kLd = MA * 128 + 1;                          // logits row pitch (floats), padded

  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full_bar[kRtStages], empty_bar[kRtStages], tfull_bar[2], tempty_bar[2];
  __shared__ uint32_t tmem_holder;

  const uint32_t smem_base = (smem_u32(smem_raw) + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (smem_base - smem_u32(smem_raw));
  float* lg = reinterpret_cast<float*>(smem + kRtStages * kStageBytes);   // [kRtHalf][kLd]
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int tiles = (T + kRtBN - 1) / kRtBN;
  const int KB = d / kRtBK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kRtStages; ++s) { mbar_init(&full_bar[s], 1); mbar_init(&empty_bar[s], 1); }
    for (int a = 0; a < 2; ++a) { mbar_init(&tfull_bar[a], 1); mbar_init(&tempty_bar[a], 4); }
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&tmem_holder, kTmemCols);
    tmem_relinquish();
  }
  pdl_wait();
  pdl_trigger();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = tmem_holder;
  auto w_tile = [&](int s, int h) -> uint8_t* { return smem + static_cast<size_t>(s) * kStageBytes + h * kWBytes; };
  auto x_tile = [&](int s) -> uint8_t* { return smem + static_cast<size_t>(s) * kStageBytes + MA * kWBytes; };

  if (warp == 0) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x) {
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait(&empty_bar[stage], phase ^ 1u)) { ok = false; break; }
          mbar_arrive_expect_tx(&full_bar[stage], kStageBytes);
#pragma unroll
          for (int h = 0; h < MA; ++h) tma_load_2d(w_tile(stage, h), &tmW, &full_bar[stage], kb * kRtBK, h * 128);
          tma_load_2d(x_tile(stage), &tmX, &full_bar[stage], kb * kRtBK, t * kRtBN);
          if (++stage == kRtStages) { stage = 0; phase ^= 1u; }
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
        const uint32_t dacc = tmem_base + ab * kAccCols;
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait(&full_bar[stage], phase)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sx = smem_u32(x_tile(stage));
#pragma unroll
          for (int kk = 0; kk < kRtBK / 16; ++kk) {
            const uint64_t bdesc = smem_desc_sw128(sx + kk * 32);
#pragma unroll
            for (int h = 0; h < MA; ++h)
              umma_f16(dacc + h * kRtBN, smem_desc_sw128(smem_u32(w_tile(stage, h)) + kk * 32), bdesc, kIdesc,
                       (kb | kk) != 0 ? 1u : 0u);
          }
          umma_commit(&empty_bar[stage]);
          if (++stage == kRtStages) { stage = 0; phase ^= 1u; }
        }
        if (ok) umma_commit(&tfull_bar[ab]);
      }
    }
    __syncwarp();
  } else {
    const int q = warp % 4;
    const int ew = warp - 2;          // 0..3: this warp's share of the tile's tokens
    int it = 0;
    for (int t = blockIdx.x; t < tiles; t += gridDim.x, ++it) {
      const int ab = it & 1;
      const uint32_t aphase = (it >> 1) & 1;
      if (!epilogue_all(mbar_wait(&tfull_bar[ab], aphase))) break;
      tc_fence_after();
      for (int half = 0; half < kRtBN / kRtHalf; ++half) {
        // logits (+bias) of expert row h*128 + q*32 + lane for 64 tokens -> lg[token][expert]
#pragma unroll
        for (int h = 0; h < MA; ++h) {
          const int e = h * 128 + q * 32 + lane;
          const float b = (bias != nullptr && e < E) ? bias[e] : 0.f;
          const uint32_t tb =
              tmem_base + (static_cast<uint32_t>(q * 32) << 16) + ab * kAccCols + h * kRtBN + half * kRtHalf;
#pragma unroll
          for (int c0 = 0; c0 < kRtHalf; c0 += 16) {
            float v[16];
            tmem_ld16(tb + c0, v);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 16; ++j) lg[(c0 + j) * kLd + e] = v[j] + b;
          }
        }
        if (half == kRtBN / kRtHalf - 1) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&tempty_bar[ab]);
        }
        epilogue_bar();
        // top-k: each epilogue warp takes 16 tokens of the half
        for (int c = ew * (kRtHalf / 4); c < (ew + 1) * (kRtHalf / 4); ++c) {
          const int tok = t * kRtBN + half * kRtHalf + c;
          if (tok >= T) break;
          float v[MA * 4];
#pragma unroll
          for (int i = 0; i < MA * 4; ++i) {
            const int e = lane + 32 * i;
            v[i] = e < E ? lg[c * kLd + e] : -INFINITY;
          }
          float pv[kRtMaxK];
          int pi[kRtMaxK];
#pragma unroll
          for (int j = 0; j < kRtMaxK; ++j) {
            if (j >= k) break;
            float bv = -INFINITY;
            int bi = 0x7FFFFFFF;
#pragma unroll
            for (int i = 0; i < MA * 4; ++i) {
              const int e = lane + 32 * i;
              if (e < E && (v[i] > bv || (v[i] == bv && e < bi))) { bv = v[i]; bi = e; }
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
              const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
              const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
              if (ov > bv || (ov == bv && oi < bi)) { bv = ov; bi = oi; }
            }
            pv[j] = bv;
            pi[j] = bi;
#pragma unroll
            for (int i = 0; i < MA * 4; ++i)
              if (lane + 32 * i == bi) v[i] = -INFINITY;
          }
          // lane j < k writes pick j
          float ex = 0.f, s = 0.f;
#pragma unroll
          for (int j = 0; j < kRtMaxK; ++j) {
            if (j >= k) break;
            const float e_j = expf(pv[j] - pv[0]);
            s += e_j;
            if (lane == j) ex = e_j;
          }
          if (lane < k) {
            int id = 0;
#pragma unroll
            for (int j = 0; j < kRtMaxK; ++j)
              if (j == lane) id = pi[j];
            topk_ids[static_cast<size_t>(tok) * k + lane] = id;
            topk_w[static_cast<size_t>(tok) * k + lane] = ex / s;
          }
        }
        epilogue_bar();   // lg is rewritten by the next half or tile
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, kTmemCols);
}

// true when the tensor-core router handles this call (bf16, E <= 256, many tokens)
bool route_tc_applicable(bool f32, int T, int E, int k) { return !f32 && E <= 256 && k <= kRtMaxK && T >= 256; }

template <int MA, int kRtStages, int kRtBN>
static cudaError_t launch_route_tc_tile(const void* x, int T, int d, const void* wr, const float* bias, int E, int k,
                                       int32_t* ids, float* w, cudaStream_t st) {
  CUtensorMap mW, mX;
  if (!make_map_sw128(&mW, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, wr, d, E, 2ull * d, 0, 0, 128) ||
      !make_map_sw128(&mX, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, x, d, T, 2ull * d, 0, 0, kRtBN))
    return cudaErrorInvalidValue;
  const int tiles = (T + kRtBN - 1) / kRtBN;
  const int grid = tiles < num_sms() ? tiles : num_sms();
  constexpr uint32_t stage = MA * 128 * 128 + kRtBN * 128;
  const size_t smem = 1024 + kRtStages * stage + sizeof(float) * kRtHalf * (MA * 128 + 1);
  auto kern = route_tc_kernel<MA, kRtStages, kRtBN>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  return launch_pdl(kern, dim3(grid), dim3(kTcThreads), smem, st, mW, mX, T, d, bias, E, k, ids, w);
}

cudaError_t launch_route_tc(const void* x, int T, int d, const void* wr, const float* bias, int E, int k,
                            int32_t* ids, float* w, cudaStream_t st) {
  // 128-token tiles once 64-token tiles would take more than one round of CTAs
  const bool wide = (T + 63) / 64 > num_sms();
  if (E <= 128)
    return wide ? launch_route_tc_tile<1, 4, 128>(x, T, d, wr, bias, E, k, ids, w, st)
                : launch_route_tc_tile<1, 4, 64>(x, T, d, wr, bias, E, k, ids, w, st);
  return wide ? launch_route_tc_tile<2, 3, 128>(x, T, d, wr, bias, E, k, ids, w, st)
              : launch_route_tc_tile<2, 3, 64>(x, T, d, wr, bias, E, k, ids, w, st);
}

}  // namespace ftm
