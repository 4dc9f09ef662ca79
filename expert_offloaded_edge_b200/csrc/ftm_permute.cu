// Expert histogram, prefix sum and stable permutation of the (token, pick)
// pairs by expert (step a3).
//
// Stable counting sort, deterministic by construction (no order-dependent
// atomics): ranks inside a warp come from __match_any_sync + popc of the lower
// lanes, ranks across warps from per-warp per-expert counts in shared memory,
// ranks across blocks from per-chunk histograms and a column scan.  Small P
// runs as one block in one launch; large P as histogram / scan / scatter over
// chunks of kChunk pairs (larger P).
#include "ftm_common.cuh"

namespace ftm {

constexpr int kPermThreads = 1024;
constexpr int kPermWarps = kPermThreads / 32;
constexpr int kSingleMax = 4096;   // pairs one block sorts in one launch
constexpr int kChunk = 1024;       // pairs per block of the three-pass sort (one round of the block's threads)

// Warp 0 only: out[e] = sum_{e' < e} in[e'] for e in [0, E); returns the total in out[E].
__device__ void warp0_exclusive_scan(const int32_t* in, int32_t* out, int E) {
  const int lane = threadIdx.x % 32;
  const int per = (E + 31) / 32;
  const int b = lane * per, en = min(E, b + per);
  int s = 0;
  for (int e = b; e < en; ++e) s += in[e];
  int incl = s;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  int run = incl - s;
  for (int e = b; e < en; ++e) { const int c = in[e]; out[e] = run; run += c; }
  if (lane == 31) out[E] = incl;
}

// cnt[e] += number of pairs in [q0, q1) routed to e (shared memory).  An id
// outside [0, E) is not counted and is reported in the device status word.
__device__ __forceinline__ void count_ids(const int32_t* __restrict__ ids, int q0, int q1, int E, int32_t* cnt) {
  for (int q = q0 + threadIdx.x; q < q1; q += blockDim.x) {
    const int e = ids[q];
    if (e >= 0 && e < E) atomicAdd(&cnt[e], 1);
    else report_bad_index();
  }
}

// Place pairs [q_begin, q_end) in order; base[e] (shared) is the next free
// position of expert e and is advanced.  wcnt (shared, [warps][E]) must be zero.
__device__ void stable_scatter(const int32_t* __restrict__ ids, int q_begin, int q_end, int32_t* base,
                               int32_t* wcnt, int E, int32_t* __restrict__ perm, int32_t* __restrict__ inv) {
  const int nw = blockDim.x / 32, warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const unsigned lt_mask = (1u << lane) - 1u;
  for (int r0 = q_begin; r0 < q_end; r0 += blockDim.x) {
    const int q = r0 + threadIdx.x;
    const int e_in = q < q_end ? ids[q] : E;
    const bool valid = q < q_end && e_in >= 0 && e_in < E;   // an id outside [0, E) is skipped
    const int e = valid ? e_in : E;
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    const int rank_w = __popc(peers & lt_mask);
    if (valid && rank_w == 0) wcnt[warp * E + e] = __popc(peers);
    __syncthreads();
    if (q < q_end && !valid) inv[q] = -1;
    if (valid) {
      int before = 0;
      for (int w = 0; w < warp; ++w) before += wcnt[w * E + e];
      const int pos = base[e] + before + rank_w;
      perm[pos] = q;
      inv[q] = pos;
    }
    __syncthreads();
    for (int x = threadIdx.x; x < E; x += blockDim.x) {
      int s = 0;
      for (int w = 0; w < nw; ++w) { s += wcnt[w * E + x]; wcnt[w * E + x] = 0; }
      base[x] += s;
    }
    __syncthreads();
  }
}

// One block does everything (P <= kSingleMax).
__global__ void __launch_bounds__(kPermThreads) permute_single_kernel(const int32_t* __restrict__ ids, int P, int E,
                                                                      int32_t* __restrict__ counts,
                                                                      int32_t* __restrict__ offsets,
                                                                      int32_t* __restrict__ perm,
                                                                      int32_t* __restrict__ inv) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ int32_t sm[];
  int32_t* cnt = sm;                 // [E]
  int32_t* base = cnt + E;           // [E+1]
  int32_t* wcnt = base + E + 1;      // [warps][E]
  for (int i = threadIdx.x; i < E; i += blockDim.x) cnt[i] = 0;
  for (int i = threadIdx.x; i < kPermWarps * E; i += blockDim.x) wcnt[i] = 0;
  __syncthreads();
  count_ids(ids, 0, P, E, cnt);
  __syncthreads();
  if (threadIdx.x < 32) warp0_exclusive_scan(cnt, base, E);
  __syncthreads();
  for (int i = threadIdx.x; i <= E; i += blockDim.x) offsets[i] = base[i];
  for (int i = threadIdx.x; i < E; i += blockDim.x) counts[i] = cnt[i];
  __syncthreads();
  stable_scatter(ids, 0, P, base, wcnt, E, perm, inv);
  // positions past the last placed pair (only when ids held out-of-range values)
  for (int pos = base[E] + threadIdx.x; pos < P; pos += blockDim.x) perm[pos] = -1;
}

// Large P, pass 1: per-chunk histogram hist[c][e].
__global__ void __launch_bounds__(kPermThreads) permute_hist_kernel(const int32_t* __restrict__ ids, int P, int E,
                                                                    int32_t* __restrict__ hist) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ int32_t sm[];
  for (int i = threadIdx.x; i < E; i += blockDim.x) sm[i] = 0;
  __syncthreads();
  const int q0 = blockIdx.x * kChunk, q1 = min(P, q0 + kChunk);
  count_ids(ids, q0, q1, E, sm);
  __syncthreads();
  for (int i = threadIdx.x; i < E; i += blockDim.x) hist[static_cast<size_t>(blockIdx.x) * E + i] = sm[i];
}

// Large P, pass 2 (one block): counts, offsets, and hist[c][e] <- start of chunk c's run of expert e.
__global__ void __launch_bounds__(kPermThreads) permute_scan_kernel(int nchunks, int E, int P,
                                                                    int32_t* __restrict__ hist,
                                                                    int32_t* __restrict__ counts,
                                                                    int32_t* __restrict__ offsets,
                                                                    int32_t* __restrict__ perm) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ int32_t sm[];
  int32_t* tot = sm;          // [E]
  int32_t* off = sm + E;      // [E+1]
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int s = 0;
    for (int c = 0; c < nchunks; ++c) s += hist[static_cast<size_t>(c) * E + e];
    tot[e] = s;
  }
  __syncthreads();
  if (threadIdx.x < 32) warp0_exclusive_scan(tot, off, E);
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    counts[e] = tot[e];
    int run = off[e];
    for (int c = 0; c < nchunks; ++c) {
      const size_t i = static_cast<size_t>(c) * E + e;
      const int h = hist[i];
      hist[i] = run;
      run += h;
    }
  }
  for (int e = threadIdx.x; e <= E; e += blockDim.x) offsets[e] = off[e];
  // positions past the last placed pair (only when ids held out-of-range values)
  for (int pos = off[E] + threadIdx.x; pos < P; pos += blockDim.x) perm[pos] = -1;
}

// Large P, pass 3: each chunk places its pairs in order from its bases.
__global__ void __launch_bounds__(kPermThreads) permute_scatter_kernel(const int32_t* __restrict__ ids, int P, int E,
                                                                       const int32_t* __restrict__ hist,
                                                                       int32_t* __restrict__ perm,
                                                                       int32_t* __restrict__ inv) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ int32_t sm[];
  int32_t* base = sm;            // [E]
  int32_t* wcnt = sm + E;        // [warps][E]
  for (int i = threadIdx.x; i < E; i += blockDim.x) base[i] = hist[static_cast<size_t>(blockIdx.x) * E + i];
  for (int i = threadIdx.x; i < kPermWarps * E; i += blockDim.x) wcnt[i] = 0;
  __syncthreads();
  const int q0 = blockIdx.x * kChunk, q1 = min(P, q0 + kChunk);
  stable_scatter(ids, q0, q1, base, wcnt, E, perm, inv);
}

size_t permute_workspace_bytes(int E, int64_t P) {
  if (P <= kSingleMax) return 0;
  const int64_t nchunks = (P + kChunk - 1) / kChunk;
  return static_cast<size_t>(nchunks * E) * sizeof(int32_t);
}

cudaError_t launch_permute(const int32_t* ids, int P, int E, int32_t* counts, int32_t* offsets, int32_t* perm,
                           int32_t* inv, void* ws, cudaStream_t st) {
  const size_t wsm = sizeof(int32_t) * (static_cast<size_t>(kPermWarps) * E + 2 * E + 1);
  if (P <= kSingleMax) {
    cudaError_t err = cudaFuncSetAttribute(permute_single_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           static_cast<int>(wsm));
    if (err != cudaSuccess) return err;
    return launch_pdl(permute_single_kernel, dim3(1), dim3(kPermThreads), wsm, st, ids, P, E, counts, offsets, perm,
                      inv);
  }
  const int nchunks = (P + kChunk - 1) / kChunk;
  int32_t* hist = static_cast<int32_t*>(ws);
  cudaError_t err = cudaFuncSetAttribute(permute_scatter_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(wsm));
  if (err != cudaSuccess) return err;
  err = launch_pdl(permute_hist_kernel, dim3(nchunks), dim3(kPermThreads), sizeof(int32_t) * E, st, ids, P, E, hist);
  if (err != cudaSuccess) return err;
  err = launch_pdl(permute_scan_kernel, dim3(1), dim3(kPermThreads), sizeof(int32_t) * (2 * E + 1), st, nchunks, E,
                   P, hist, counts, offsets, perm);
  if (err != cudaSuccess) return err;
  return launch_pdl(permute_scatter_kernel, dim3(nchunks), dim3(kPermThreads), wsm, st, ids, P, E, hist, perm, inv);
}

}  // namespace ftm
