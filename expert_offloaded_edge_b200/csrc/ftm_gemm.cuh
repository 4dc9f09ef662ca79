// Pieces shared by the grouped expert GEMM kernels (bf16 and FP8): the
// persistent tile list over (group, weight tile, token tile), and the host-side
// TMA tensor-map encoding.
#pragma once

#include "ftm_common.cuh"

namespace ftm {

constexpr int kTcThreads = 192;       // warp 0 TMA, warp 1 MMA + TMEM owner, warps 2-5 epilogue
constexpr int kMaxGroups = 520;       // E <= 512 routed groups + the shared expert
constexpr uint32_t kATileBytes = 128 * 128;   // one 128-row x 128-byte weight tile

// z * sigmoid(z) with the fast exponential and division intrinsics (relative
// error ~1e-6, far below the bf16 rounding of the result).  For z << 0 the
// denominator overflows to +inf and the quotient is -0.
__device__ __forceinline__ float silu(float z) { return __fdividef(z, 1.f + __expf(-z)); }

// ---- thread-block cluster helpers ------------------------------------------
__device__ __forceinline__ uint32_t cluster_nranks() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(r));
  return r;
}

// Store four floats into shared memory of a CTA of this cluster (address from mapa_rank).
__device__ __forceinline__ void st_cluster_v4(uint32_t cluster_addr, float a, float b, float c, float d) {
  asm volatile("st.shared::cluster.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(cluster_addr), "f"(a), "f"(b), "f"(c),
               "f"(d)
               : "memory");
}

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

__device__ __forceinline__ uint32_t mapa_rank(uint32_t saddr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
  return r;
}

__device__ __forceinline__ void mbar_arrive_remote(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait_cl(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait with cluster-scope acquire (the barrier also receives arrivals
// and transaction bytes from the other CTA of the pair).
__device__ __forceinline__ bool mbar_wait_cl(uint64_t* bar, uint32_t parity) {
  if (mbar_try_wait_cl(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait_cl(bar, parity)) return true;
    if ((it & 255u) == 0) {
      if (*reinterpret_cast<volatile int32_t*>(&g_dev_status) != 0) return false;
      if (globaltimer() - t0 > kWaitLimitNs) {
        atomicExch(&g_dev_status, kDevErrTimeout);
        return false;
      }
    }
  }
}

// ---- CTA-pair (cta_group::2) copies and commits ----------------------------
// TMA loads into this CTA's shared memory whose completion is counted on the
// barrier at cluster address leader_bar (the even CTA's).
__device__ __forceinline__ void tma2_load_2d(void* dst, const CUtensorMap* m, uint32_t leader_bar, int32_t c0,
                                             int32_t c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, "
      "%4}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(leader_bar), "r"(c0), "r"(c1)
      : "memory");
}

__device__ __forceinline__ void tma2_load_3d(void* dst, const CUtensorMap* m, uint32_t leader_bar, int32_t c0,
                                             int32_t c1, int32_t c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, "
      "%4, %5}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(leader_bar), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

// Arrive on the barrier at this offset in both CTAs of the pair once the
// issued MMAs complete.
__device__ __forceinline__ void umma2_commit_both(uint64_t* bar) {
  const uint16_t mask = 0x3;
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
          smem_u32(bar)),
      "h"(mask)
      : "memory");
}

struct TileInfo {
  int g, m, n, rows, row0;
};

// Group g < E holds rows offsets[g]..offsets[g+1] of the permuted activations;
// group E (shared expert) holds rows P..P+T-1.  Each group has ceil(rows/BN)
// token tiles times MT weight tiles; tile_start is their exclusive prefix.
// Called by all threads of the block; ends with __syncthreads().
__device__ __forceinline__ void build_tile_table(const int32_t* offsets, int E, int has_shared, int T, int P,
                                                 int MT, int BN, int32_t* tile_start, int32_t* grp_rows,
                                                 int32_t* grp_row0) {
  const int G = E + (has_shared ? 1 : 0);
  for (int g = threadIdx.x; g < G; g += blockDim.x) {
    grp_rows[g] = g < E ? offsets[g + 1] - offsets[g] : T;
    grp_row0[g] = g < E ? offsets[g] : P;
  }
  __syncthreads();
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    const int per = (G + 31) / 32, b = lane * per, en = min(G, b + per);
    int s = 0;
    for (int g = b; g < en; ++g) s += ((grp_rows[g] + BN - 1) / BN) * MT;
    int incl = s;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    int run = incl - s;
    for (int g = b; g < en; ++g) { tile_start[g] = run; run += ((grp_rows[g] + BN - 1) / BN) * MT; }
    if (lane == 31) tile_start[G] = incl;
  }
  __syncthreads();
}

// Tile t -> (group, weight tile m, token tile n); token tiles vary fastest so
// consecutive tiles share a weight tile.
__device__ __forceinline__ TileInfo decode_tile(int t, const int32_t* tile_start, const int32_t* grp_rows,
                                                const int32_t* grp_row0, int G, int BN) {
  int lo = 0, hi = G;  // tile_start[lo] <= t < tile_start[hi]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (tile_start[mid] <= t) lo = mid; else hi = mid;
  }
  TileInfo ti;
  ti.g = lo;
  ti.rows = grp_rows[lo];
  ti.row0 = grp_row0[lo];
  const int ntok = (ti.rows + BN - 1) / BN;
  const int local = t - tile_start[lo];
  ti.m = local / ntok;
  ti.n = local % ntok;
  return ti;
}

// Named barrier over the four epilogue warps (warps 2-5).
__device__ __forceinline__ void epilogue_bar() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

// Named-barrier AND over the four epilogue warps: every epilogue warp gets the
// same answer, so they leave their loop together (no warp is left waiting at a
// later named barrier for one that gave up).
__device__ __forceinline__ bool epilogue_all(bool p) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred pi, po;\n\t"
      "setp.ne.u32 pi, %1, 0;\n\t"
      "bar.red.and.pred po, 1, 128, pi;\n\t"
      "selp.u32 %0, 1, 0, po;\n\t}\n"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(p))
      : "memory");
  return r != 0;
}

// ---- host -------------------------------------------------------------------

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// K-major map with a 128-byte inner box and 128-byte swizzle: dims {K, rows[, slots]}
// (elements), box {128 bytes of K, box_rows[, 1]}.
inline bool make_map_sw128(CUtensorMap* m, CUtensorMapDataType dt, uint32_t elt_bytes, const void* base, uint64_t K,
                           uint64_t rows, uint64_t row_pitch, uint64_t slots, uint64_t slot_pitch,
                           uint32_t box_rows) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {K, rows, slots};
  cuuint64_t strides[2] = {row_pitch, slot_pitch};
  cuuint32_t box[3] = {128u / elt_bytes, box_rows, 1};
  cuuint32_t es[3] = {1, 1, 1};
  const cuuint32_t rank = slots > 0 ? 3 : 2;
  CUresult r = enc(m, dt, rank, const_cast<void*>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

inline int num_sms() {
  static int n = 0;
  if (!n) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}

}  // namespace ftm
