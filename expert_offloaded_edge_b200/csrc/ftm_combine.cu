// Weighted un-permute and combine (step a8):
//   out[t] = sum_{j ascending} g[t][j] * y[inv[t*k + j]]  (+ y[P + t] for the shared expert)
// fp32 accumulation, fixed summation order (deterministic).  A warp takes one
// item at a time (grid-strided): a whole token for large batches, one
// 32-vector slice of d for small ones, so even a single token spreads over
// d / 256 (bf16) warps; 16-byte loads and stores.
#include "ftm_common.cuh"

namespace ftm {

constexpr int kMaxTerms = 17;   // k <= 16 routed picks + the shared expert

// Per item: lane j < k fetches the token's j-th row index and gate (lane k:
// the shared expert's row, gate 1) into the warp's shared-memory slots, then
// each lane issues all of the token's row loads for its 16-byte vector before
// the fused multiply-adds.  The terms are added in ascending j, so the result
// does not depend on the schedule.
template <bool F32, int MAXT>
__global__ void __launch_bounds__(256, MAXT <= 9 ? 3 : 2) combine_kernel(const void* __restrict__ y, const int32_t* __restrict__ inv,
                                                      const float* __restrict__ gw, int T, int k, int d, int P,
                                                      int has_shared, int spi, void* __restrict__ out) {
  constexpr int V = F32 ? 4 : 8;   // elements per 16-byte vector
  constexpr int EB = F32 ? 4 : 2;  // bytes per element
  const int nv = d / V;
  const int nterms = k + (has_shared ? 1 : 0);
  const int lane = threadIdx.x & 31;
  const int wpb = blockDim.x >> 5;
  __shared__ int s_rows[8][MAXT];
  __shared__ float s_gs[8][MAXT];
  pdl_wait();
  pdl_trigger();
  const int nch = (nv + 31) / 32;                    // 32-vector slices of a row
  const int ipt = (nch + spi - 1) / spi;             // items per token (spi slices each)
  const long long items = static_cast<long long>(T) * ipt;
  for (long long item = static_cast<long long>(blockIdx.x) * wpb + (threadIdx.x >> 5); item < items;
       item += static_cast<long long>(gridDim.x) * wpb) {
    const int t = static_cast<int>(item / ipt);
    const int c0 = static_cast<int>(item % ipt) * spi * 32;
    int my_row = -1;
    float my_g = 0.f;
    if (lane < nterms) {
      int row = lane < k ? inv[static_cast<size_t>(t) * k + lane] : P + t;
      if (lane < k && (row < 0 || row >= P)) {   // a pair the permutation skipped (id out of range)
        report_bad_index();
        row = -1;
      }
      my_row = row;
      my_g = lane < k ? gw[static_cast<size_t>(t) * k + lane] : 1.f;
    }
    // the warp's copy of the token's rows and gates
    int* rows = s_rows[threadIdx.x >> 5];
    float* gs = s_gs[threadIdx.x >> 5];
    if (lane < MAXT) {
      rows[lane] = lane < nterms ? my_row : -1;
      gs[lane] = my_g;
    }
    __syncwarp();
    for (int c = c0 + lane; c < nv && c < c0 + spi * 32; c += 32) {
      uint4 u[MAXT];
#pragma unroll
      for (int j = 0; j < MAXT; ++j)
        if (j < nterms && rows[j] >= 0)
          u[j] = *reinterpret_cast<const uint4*>(static_cast<const uint8_t*>(y) +
                                                 (static_cast<size_t>(rows[j]) * d + static_cast<size_t>(c) * V) * EB);
      float acc[V];
#pragma unroll
      for (int i = 0; i < V; ++i) acc[i] = 0.f;
#pragma unroll
      for (int j = 0; j < MAXT; ++j) {
        if (j >= nterms || rows[j] < 0) continue;
        const float g = gs[j];
        if constexpr (F32) {
          const float f[4] = {__uint_as_float(u[j].x), __uint_as_float(u[j].y), __uint_as_float(u[j].z),
                              __uint_as_float(u[j].w)};
#pragma unroll
          for (int i = 0; i < 4; ++i) acc[i] = fmaf(g, f[i], acc[i]);
        } else {
          const uint32_t w[4] = {u[j].x, u[j].y, u[j].z, u[j].w};
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
                                (static_cast<size_t>(t) * d + static_cast<size_t>(c) * V) * EB) = o;
    }
    __syncwarp();   // the warp's rows and gates are rewritten for its next item
  }
}

cudaError_t launch_combine(bool f32, const void* y, const int32_t* inv, const float* gw, int T, int k, int d, int P,
                           int has_shared, void* out, cudaStream_t st) {
  // a warp takes a whole token when the batch alone fills the GPU (its rows and gates are read once), else one
  // 32-vector slice of d at a time so that a few tokens still spread over many warps
  const int V = f32 ? 4 : 8;
  const int nch = (d / V + 31) / 32;
  const int spi = T >= 148 * 8 ? nch : 1;
  const long long items = static_cast<long long>(T) * ((nch + spi - 1) / spi);
  const long long blocks = (items + 7) / 8;   // 8 items (warps) per block
  const int grid = static_cast<int>(blocks < 148 * 8 ? blocks : 148 * 8);
  // up to 8 routed picks + the shared expert: a 9-term register file, which lets three blocks share an SM
  const bool small = k + (has_shared ? 1 : 0) <= 9;
  if (f32)
    return small ? launch_pdl(combine_kernel<true, 9>, dim3(grid), dim3(256), 0, st, y, inv, gw, T, k, d, P, has_shared,
                              spi, out)
                 : launch_pdl(combine_kernel<true, kMaxTerms>, dim3(grid), dim3(256), 0, st, y, inv, gw, T, k, d, P,
                              has_shared, spi, out);
  return small ? launch_pdl(combine_kernel<false, 9>, dim3(grid), dim3(256), 0, st, y, inv, gw, T, k, d, P, has_shared,
                            spi, out)
               : launch_pdl(combine_kernel<false, kMaxTerms>, dim3(grid), dim3(256), 0, st, y, inv, gw, T, k, d, P,
                            has_shared, spi, out);
}

}  // namespace ftm
