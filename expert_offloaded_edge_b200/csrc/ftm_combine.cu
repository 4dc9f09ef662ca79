// Weighted un-permute and combine (step a8):
//   out[t] = sum_{j ascending} g[t][j] * y[inv[t*k + j]]  (+ y[P + t] for the shared expert)
// fp32 accumulation, fixed summation order (deterministic).  One block per
// token (grid-strided), 16-byte loads and stores along d.
#include "ftm_common.cuh"

namespace ftm {

template <bool F32>
__global__ void __launch_bounds__(256) combine_kernel(const void* __restrict__ y, const int32_t* __restrict__ inv,
                                                      const float* __restrict__ gw, int T, int k, int d, int P,
                                                      int has_shared, void* __restrict__ out) {
  constexpr int V = F32 ? 4 : 8;   // elements per 16-byte vector
  __shared__ int32_t s_row[17];
  __shared__ float s_g[17];
  const int nv = d / V;
  const int nterms = k + (has_shared ? 1 : 0);
  pdl_wait();
  pdl_trigger();
  for (int t = blockIdx.x; t < T; t += gridDim.x) {
    // the token's rows and weights first, so the row loads below are independent
    if (threadIdx.x < nterms) {
      const int j = threadIdx.x;
      int row = j < k ? inv[static_cast<size_t>(t) * k + j] : P + t;
      if (j < k && (row < 0 || row >= P)) {   // a pair the permutation skipped (id out of range)
        report_bad_index();
        row = -1;
      }
      s_row[j] = row;
      s_g[j] = j < k ? gw[static_cast<size_t>(t) * k + j] : 1.f;
    }
    __syncthreads();
    for (int c = threadIdx.x; c < nv; c += blockDim.x) {
      float acc[V];
#pragma unroll
      for (int i = 0; i < V; ++i) acc[i] = 0.f;
#pragma unroll 4
      for (int j = 0; j < nterms; ++j) {
        const int row = s_row[j];
        if (row < 0) continue;
        const float g = s_g[j];
        const uint4 u = *reinterpret_cast<const uint4*>(static_cast<const uint8_t*>(y) +
                                                        (static_cast<size_t>(row) * d + static_cast<size_t>(c) * V) *
                                                            (F32 ? 4 : 2));
        if constexpr (F32) {
          const float f[4] = {__uint_as_float(u.x), __uint_as_float(u.y), __uint_as_float(u.z), __uint_as_float(u.w)};
#pragma unroll
          for (int i = 0; i < 4; ++i) acc[i] = fmaf(g, f[i], acc[i]);
        } else {
          const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            acc[2 * i] = fmaf(g, __uint_as_float(w[i] << 16), acc[2 * i]);
            acc[2 * i + 1] = fmaf(g, __uint_as_float(w[i] & 0xFFFF0000u), acc[2 * i + 1]);
          }
        }
      }
      uint4 o;
      if constexpr (F32) {
        o = make_uint4(__float_as_uint(acc[0]), __float_as_uint(acc[1]), __float_as_uint(acc[2]),
                       __float_as_uint(acc[3]));
      } else {
        uint32_t w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const __nv_bfloat162 b = __floats2bfloat162_rn(acc[2 * i], acc[2 * i + 1]);
          w[i] = *reinterpret_cast<const uint32_t*>(&b);
        }
        o = make_uint4(w[0], w[1], w[2], w[3]);
      }
      *reinterpret_cast<uint4*>(static_cast<uint8_t*>(out) +
                                (static_cast<size_t>(t) * d + static_cast<size_t>(c) * V) * (F32 ? 4 : 2)) = o;
    }
    __syncthreads();   // s_row / s_g are rewritten for the next token
  }
}

cudaError_t launch_combine(bool f32, const void* y, const int32_t* inv, const float* gw, int T, int k, int d, int P,
                           int has_shared, void* out, cudaStream_t st) {
  const int grid = T < 148 * 16 ? T : 148 * 16;
  if (f32)
    return launch_pdl(combine_kernel<true>, dim3(grid), dim3(256), 0, st, y, inv, gw, T, k, d, P, has_shared, out);
  else
    return launch_pdl(combine_kernel<false>, dim3(grid), dim3(256), 0, st, y, inv, gw, T, k, d, P, has_shared, out);
  return cudaGetLastError();
}

}  // namespace ftm
