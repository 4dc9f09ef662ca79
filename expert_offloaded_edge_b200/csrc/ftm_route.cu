// Router GEMV/GEMM + softmax + top-k + renormalisation (steps a1, a2).
//
// One thread-block cluster per tile of TT tokens.  The E experts are split
// over the cluster's CTAs; each CTA streams its slice of the router matrix
// once (16-byte loads, one warp per expert row, fp32 accumulation) against the
// token tile held in shared memory, and writes its logits straight into the
// shared memory of cluster rank 0 (distributed shared memory).  After one
// cluster barrier rank 0 runs the gating: one warp per token does k rounds of
// warp-wide argmax (ties to the lower expert id) and the softmax over the k
// picks, which equals the softmax over all E experts renormalised over the
// picks.  No global scratch, one launch.
#include <cooperative_groups.h>

#include "ftm_common.cuh"

namespace cg = cooperative_groups;

namespace ftm {

constexpr int kRouteCluster = 8;
constexpr int kRouteWarps = 16;
constexpr int kMaxE = 512;
constexpr int kMaxK = 16;

template <typename Tin>
struct RouteIO;

template <>
struct RouteIO<float> {
  static constexpr int kVec = 4;  // elements per 16-byte load
  __device__ static void load(const void* p, float* v) {
    float4 f = *reinterpret_cast<const float4*>(p);
    v[0] = f.x; v[1] = f.y; v[2] = f.z; v[3] = f.w;
  }
};

template <>
struct RouteIO<uint16_t> {
  static constexpr int kVec = 8;
  __device__ static void load(const void* p, float* v) {
    uint4 u = *reinterpret_cast<const uint4*>(p);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      v[2 * i] = __uint_as_float(w[i] << 16);
      v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
  }
};

template <typename Tin, int TT>
__global__ void __launch_bounds__(kRouteWarps * 32) route_topk_kernel(const Tin* __restrict__ x, int T, int d,
                                                                       const Tin* __restrict__ wr,
                                                                       const float* __restrict__ bias, int E, int k,
                                                                       int32_t* __restrict__ topk_ids,
                                                                       float* __restrict__ topk_w) {
  using IO = RouteIO<Tin>;
  constexpr int V = IO::kVec;
  extern __shared__ __align__(16) uint8_t smem[];
  float* logits = reinterpret_cast<float*>(smem);                  // [TT][E] (rank 0's is the real one)
  Tin* xs = reinterpret_cast<Tin*>(smem + sizeof(float) * TT * kMaxE);  // [TT][d]

  cg::cluster_group cluster = cg::this_cluster();
  const int rank = static_cast<int>(cluster.block_rank());
  const int tile = blockIdx.x / kRouteCluster;
  const int t0 = tile * TT;
  const int nt = min(TT, T - t0);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  pdl_wait();
  pdl_trigger();

  // token tile -> shared memory (rows beyond T are zero); 8 loads in flight per thread
  const int vec_per_row = d / V;
  const int nvec = TT * vec_per_row;
  for (int base = threadIdx.x; base < nvec; base += 8 * blockDim.x) {
    uint4 v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int i = base + u * blockDim.x;
      const int r = i / vec_per_row, c = i % vec_per_row;
      v[u] = make_uint4(0, 0, 0, 0);
      if (i < nvec && r < nt) v[u] = *reinterpret_cast<const uint4*>(x + static_cast<size_t>(t0 + r) * d + c * V);
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int i = base + u * blockDim.x;
      if (i < nvec) *reinterpret_cast<uint4*>(xs + static_cast<size_t>(i) * V) = v[u];
    }
  }
  __syncthreads();

  float* logits0 = cluster.map_shared_rank(logits, 0);
  const int per_rank = (E + kRouteCluster - 1) / kRouteCluster;
  const int e_begin = rank * per_rank, e_end = min(E, e_begin + per_rank);
  for (int e = e_begin + warp; e < e_end; e += kRouteWarps) {
    float acc[TT];
#pragma unroll
    for (int t = 0; t < TT; ++t) acc[t] = 0.f;
    const Tin* wrow = wr + static_cast<size_t>(e) * d;
#pragma unroll 8
    for (int c = lane * V; c < d; c += 32 * V) {
      float w[V];
      IO::load(wrow + c, w);
#pragma unroll
      for (int t = 0; t < TT; ++t) {
        float xv[V];
        IO::load(xs + static_cast<size_t>(t) * d + c, xv);
#pragma unroll
        for (int i = 0; i < V; ++i) acc[t] = fmaf(xv[i], w[i], acc[t]);
      }
    }
    const float b = bias ? bias[e] : 0.f;
#pragma unroll
    for (int t = 0; t < TT; ++t) {
      const float s = warp_sum(acc[t]);
      if (lane == 0) logits0[t * kMaxE + e] = s + b;
    }
  }
  cluster.sync();
  if (rank != 0) return;

  // gating: one warp per token
  for (int t = warp; t < nt; t += kRouteWarps) {
    float v[kMaxE / 32];
#pragma unroll
    for (int i = 0; i < kMaxE / 32; ++i) {
      const int e = lane + 32 * i;
      v[i] = (e < E) ? logits[t * kMaxE + e] : -INFINITY;
    }
    float pick_val[kMaxK];
    int pick_id[kMaxK];
    for (int j = 0; j < k; ++j) {
      float bv = -INFINITY;
      int bi = 0x7FFFFFFF;
#pragma unroll
      for (int i = 0; i < kMaxE / 32; ++i) {
        const int e = lane + 32 * i;
        if (e < E && (v[i] > bv || (v[i] == bv && e < bi))) { bv = v[i]; bi = e; }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
        const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
        if (ov > bv || (ov == bv && oi < bi)) { bv = ov; bi = oi; }
      }
      pick_val[j] = bv;
      pick_id[j] = bi;
#pragma unroll
      for (int i = 0; i < kMaxE / 32; ++i)
        if (lane + 32 * i == bi) v[i] = -INFINITY;
    }
    if (lane == 0) {
      const float m = pick_val[0];
      float s = 0.f;
      float ex[kMaxK];
      for (int j = 0; j < k; ++j) { ex[j] = expf(pick_val[j] - m); s += ex[j]; }
      const size_t base = static_cast<size_t>(t0 + t) * k;
      for (int j = 0; j < k; ++j) {
        topk_ids[base + j] = pick_id[j];
        topk_w[base + j] = ex[j] / s;
      }
    }
  }
}

template <typename Tin, int TT>
static cudaError_t launch_route_tt(const void* x, int T, int d, const void* wr, const float* bias, int E, int k,
                                   int32_t* ids, float* w, cudaStream_t st) {
  const int tiles = (T + TT - 1) / TT;
  const size_t smem = sizeof(float) * TT * kMaxE + sizeof(Tin) * static_cast<size_t>(TT) * d;
  auto kern = route_topk_kernel<Tin, TT>;
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (err != cudaSuccess) return err;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(tiles * kRouteCluster);
  cfg.blockDim = dim3(kRouteWarps * 32);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = kRouteCluster;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return count_launch(cudaLaunchKernelEx(&cfg, kern, static_cast<const Tin*>(x), T, d, static_cast<const Tin*>(wr), bias, E, k,
                            ids, w));
}

bool route_tc_applicable(bool f32, int T, int E, int k);
cudaError_t launch_route_tc(const void* x, int T, int d, const void* wr, const float* bias, int E, int k,
                            int32_t* ids, float* w, cudaStream_t st);

// Large bf16 batches go to the tensor-core router.  Otherwise the token tile
// is small enough that the batch spreads over ~16 clusters (each thread's dot
// products are the latency of the kernel) and the x tile fits next to the
// logits buffer.
cudaError_t launch_route(bool f32, const void* x, int T, int d, const void* wr, const float* bias, int E, int k,
                         int32_t* ids, float* w, cudaStream_t st) {
  if (route_tc_applicable(f32, T, E, k)) return launch_route_tc(x, T, d, wr, bias, E, k, ids, w, st);
  const size_t elt = f32 ? 4 : 2;
  const size_t budget = 160 * 1024 - sizeof(float) * 16 * kMaxE;
  if (T <= 32) {
    return f32 ? launch_route_tt<float, 1>(x, T, d, wr, bias, E, k, ids, w, st)
               : launch_route_tt<uint16_t, 1>(x, T, d, wr, bias, E, k, ids, w, st);
  }
  if (T <= 128 && 4 * d * elt <= budget) {
    return f32 ? launch_route_tt<float, 4>(x, T, d, wr, bias, E, k, ids, w, st)
               : launch_route_tt<uint16_t, 4>(x, T, d, wr, bias, E, k, ids, w, st);
  }
  if (16 * d * elt <= budget && T >= 16) {
    return f32 ? launch_route_tt<float, 16>(x, T, d, wr, bias, E, k, ids, w, st)
               : launch_route_tt<uint16_t, 16>(x, T, d, wr, bias, E, k, ids, w, st);
  }
  if (8 * d * elt <= budget && T >= 8) {
    return f32 ? launch_route_tt<float, 8>(x, T, d, wr, bias, E, k, ids, w, st)
               : launch_route_tt<uint16_t, 8>(x, T, d, wr, bias, E, k, ids, w, st);
  }
  if (4 * d * elt <= budget && T >= 4) {
    return f32 ? launch_route_tt<float, 4>(x, T, d, wr, bias, E, k, ids, w, st)
               : launch_route_tt<uint16_t, 4>(x, T, d, wr, bias, E, k, ids, w, st);
  }
  return f32 ? launch_route_tt<float, 1>(x, T, d, wr, bias, E, k, ids, w, st)
             : launch_route_tt<uint16_t, 1>(x, T, d, wr, bias, E, k, ids, w, st);
}

}  // namespace ftm
