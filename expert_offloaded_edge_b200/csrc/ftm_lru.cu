// LRU slot-table lookup and update (step a4), one block.
//
// The pages' `offload` backend keeps a set of LRU slots in VRAM and copies
// misses over PCIe (chenxutan.com FreeToken article, "choosing among the five
// MoE backends"); the cache is global and evicts the expert unused for the
// longest time (claypier.com "FreeToken MoE edge runtime", first section).
//
// The cache may be shared by several layers: its entries are keys, layer l's
// expert e being key l*E + e (key_base = l*E for the layer looked up).
// Step s: mark the distinct requested experts of the layer (all E of them for
// whole-layer staging, ids == nullptr); hits get last_use = s; the misses, in
// ascending key, take the slots with last_use < reserve (reserve <= s; slots
// used since `reserve` are held back for compute still in flight) in order of
// (last_use, slot index).  Because each placement sets last_use = s >=
// reserve, the i-th miss simply takes the i-th candidate of that order, so
// the whole step is a rank computation with no sequential dependence.  When
// the misses outnumber the candidates the step is refused before any write.
//
// Workspace (device int32): [0] status, [1] distinct, [2] hits, [3] misses,
// [4 .. 4+2E) miss list (key, slot) pairs, then a backup for rollback: the
// layer's slot_of_key[key_base .. key_base+E), key_of_slot[S], last_use[S]
// (int64).
#include "ftm_common.cuh"

namespace ftm {

constexpr int kLruThreads = 1024;

size_t lru_workspace_bytes(int E, int S) {
  size_t b = sizeof(int32_t) * (4 + 2 * static_cast<size_t>(E) + E + S);
  b = (b + 7) & ~static_cast<size_t>(7);
  return b + sizeof(int64_t) * S;
}

__device__ __forceinline__ int64_t* lru_backup_lu(int32_t* ws, int E, int S) {
  size_t off = sizeof(int32_t) * (4 + 2 * static_cast<size_t>(E) + E + S);
  off = (off + 7) & ~static_cast<size_t>(7);
  return reinterpret_cast<int64_t*>(reinterpret_cast<uint8_t*>(ws) + off);
}

// skip (nullable, [E]): experts flagged nonzero are not requests even when
// routed (the experts the bandwidth-adaptive split computes on the host).
__global__ void __launch_bounds__(kLruThreads) lru_step_kernel(const int32_t* __restrict__ ids, int P, int E, int S,
                                                               int64_t step, int64_t reserve, int key_base,
                                                               const int32_t* __restrict__ skip,
                                                               int32_t* __restrict__ slot_of_key,
                                                               int32_t* __restrict__ key_of_slot,
                                                               int64_t* __restrict__ last_use,
                                                               int32_t* __restrict__ ws) {
  extern __shared__ int32_t sm[];
  int32_t* want = sm;              // [E] 0/1
  int32_t* miss_rank = want + E;   // [E+1] exclusive scan of miss flags
  int32_t* cand = miss_rank + E + 1;  // [S] candidate flag
  int32_t* victim = cand + S;      // [S] candidate of each rank
  __shared__ int32_t s_distinct, s_hits, s_misses, s_free, s_bad;
  pdl_wait();
  pdl_trigger();
  int32_t* soe = slot_of_key + key_base;   // this layer's entries

  for (int e = threadIdx.x; e < E; e += blockDim.x) want[e] = ids ? 0 : 1;
  if (threadIdx.x == 0) { s_distinct = 0; s_hits = 0; s_misses = 0; s_free = 0; s_bad = 0; }
  __syncthreads();
  if (ids) {
    for (int q = threadIdx.x; q < P; q += blockDim.x) {
      const int e = ids[q];
      if (e >= 0 && e < E) {
        if (!skip || !skip[e]) want[e] = 1;
      } else {
        s_bad = 1;
      }
    }
  }
  __syncthreads();
  if (s_bad) {   // an id outside [0, E): the state is left untouched
    if (threadIdx.x == 0) {
      report_bad_index();
      ws[0] = FTM_ERR_INVALID_ARG; ws[1] = 0; ws[2] = 0; ws[3] = 0;
    }
    return;
  }
  // capacity: the misses must not outnumber the slots they may take
  for (int e = threadIdx.x; e < E; e += blockDim.x)
    if (want[e]) {
      atomicAdd(&s_distinct, 1);
      if (soe[e] < 0) atomicAdd(&s_misses, 1);
    }
  for (int j = threadIdx.x; j < S; j += blockDim.x) {
    const int k = key_of_slot[j] - key_base;
    const bool hit = k >= 0 && k < E && want[k];
    if (last_use[j] < reserve && !hit) atomicAdd(&s_free, 1);
  }
  __syncthreads();
  const int distinct = s_distinct;
  if (s_misses > s_free) {
    if (threadIdx.x == 0) { ws[0] = FTM_ERR_CAPACITY; ws[1] = distinct; ws[2] = 0; ws[3] = 0; }
    return;
  }
  // backup for rollback
  int32_t* bk_soe = ws + 4 + 2 * E;
  int32_t* bk_eos = bk_soe + E;
  int64_t* bk_lu = lru_backup_lu(ws, E, S);
  for (int e = threadIdx.x; e < E; e += blockDim.x) bk_soe[e] = soe[e];
  for (int j = threadIdx.x; j < S; j += blockDim.x) { bk_eos[j] = key_of_slot[j]; bk_lu[j] = last_use[j]; }
  __syncthreads();

  // hits
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    const int sl = soe[e];
    const bool miss = want[e] && sl < 0;
    if (want[e] && sl >= 0) { last_use[sl] = step; atomicAdd(&s_hits, 1); }
    want[e] = miss ? 1 : 0;   // from here on: miss flag
  }
  __syncthreads();
  if (threadIdx.x < 32) {
    // exclusive scan of miss flags (warp 0)
    const int lane = threadIdx.x;
    const int per = (E + 31) / 32, b = lane * per, en = min(E, b + per);
    int s = 0;
    for (int e = b; e < en; ++e) s += want[e];
    int incl = s;
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    int run = incl - s;
    for (int e = b; e < en; ++e) { miss_rank[e] = run; run += want[e]; }
    if (lane == 31) miss_rank[E] = incl;
  }
  for (int j = threadIdx.x; j < S; j += blockDim.x) cand[j] = last_use[j] < reserve ? 1 : 0;
  __syncthreads();
  // rank of each candidate slot in (last_use, index) order
  for (int j = threadIdx.x; j < S; j += blockDim.x) {
    if (!cand[j]) continue;
    const int64_t lj = last_use[j];
    int r = 0;
    for (int i = 0; i < S; ++i)
      if (cand[i]) {
        const int64_t li = last_use[i];
        r += (li < lj || (li == lj && i < j)) ? 1 : 0;
      }
    victim[r] = j;
  }
  __syncthreads();
  const int misses = miss_rank[E];
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    if (!want[e]) continue;
    const int r = miss_rank[e];
    const int sl = victim[r];
    const int old = key_of_slot[sl];
    if (old >= 0) slot_of_key[old] = -1;
    soe[e] = sl;
    key_of_slot[sl] = key_base + e;
    last_use[sl] = step;
    ws[4 + 2 * r] = key_base + e;
    ws[4 + 2 * r + 1] = sl;
  }
  if (threadIdx.x == 0) { ws[0] = FTM_OK; ws[1] = distinct; ws[2] = s_hits; ws[3] = misses; }
}

cudaError_t launch_lru_step(const int32_t* ids, int P, int E, int S, int64_t step, int64_t reserve, int key_base,
                            const int32_t* skip, int32_t* soe, int32_t* eos, int64_t* lu, int32_t* ws,
                            cudaStream_t st) {
  const size_t smem = sizeof(int32_t) * (2 * static_cast<size_t>(E) + 1 + 2 * S);
  cudaError_t err =
      cudaFuncSetAttribute(lru_step_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (err != cudaSuccess) return err;
  return launch_pdl(lru_step_kernel, dim3(1), dim3(kLruThreads), smem, st, ids, P, E, S, step, reserve, key_base,
                    skip, soe, eos, lu, ws);
}

// Group labels of a cache step whose expert FFN runs in two launches, the hit
// experts' while the misses are copied and the copied misses' after: a pair
// routed to a resident expert e keeps label e, one routed to an expert not in
// the cache (the state before this step's lookup) gets E + e.  A permutation
// over 2E groups then holds the hits at positions 0 .. P_hit - 1 and the
// misses, still grouped by expert, after them.  Ids outside [0, E) are copied
// through (the lookup refuses the step before they are used).
__global__ void miss_relabel_kernel(const int32_t* __restrict__ ids, int P, int E, const int32_t* __restrict__ soe,
                                    int32_t* __restrict__ ids2) {
  pdl_wait();
  pdl_trigger();
  for (int q = blockIdx.x * blockDim.x + threadIdx.x; q < P; q += gridDim.x * blockDim.x) {
    const int e = ids[q];
    ids2[q] = (e >= 0 && e < E && soe[e] < 0) ? E + e : e;
  }
}

cudaError_t launch_miss_relabel(const int32_t* ids, int P, int E, const int32_t* soe, int32_t* ids2,
                                cudaStream_t st) {
  const int blocks = P > 0 ? (P + 255) / 256 < 148 ? (P + 255) / 256 : 148 : 1;
  return launch_pdl(miss_relabel_kernel, dim3(blocks), dim3(256), 0, st, ids, P, E, soe, ids2);
}

// ---------------------------------------------------------------------------
// Bandwidth-adaptive miss split (the pages' q* policy: freelamp.com FreeToken
// article, section 2.1; chenxutan.com FreeToken article, "choosing among the
// five MoE backends", `hybrid`).  Of the m experts a step requests that are not
// resident, q are copied over PCIe and computed on the GPU and m - q are
// computed on the host from host memory, the two sides overlapped.  With a
// PCIe bandwidth Bp and a host FFN bandwidth Bh (expert bytes per second each
// side moves), both sides finish together when q / Bp = (m - q) / Bh, i.e.
// q = m Bp / (Bp + Bh); q is that value rounded to the nearest integer (halves
// up), computed in fp64 as floor(m * Bp / (Bp + Bh) + 0.5).  The host takes the
// m - q misses with the fewest pairs (ties: the lower expert id): its cost per
// expert grows with the rows, a copy's does not.
//   ids2[q] = 2E for a pair of a host expert, E + e for one of an expert
//   copied this step, e for a resident expert (ids outside [0, E) copied
//   through; the lookup rejects them); skip[e] = 1 for a host expert, else 0
//   (the lookup's mask); out (int32): [0] m, [1] q, [2] host experts H = m - q,
//   [3] their pairs, [4 .. 4+H) the host experts in order (fewest pairs
//   first).
// One block; the residency read is the state before the step's lookup.
__global__ void __launch_bounds__(kLruThreads) hybrid_split_kernel(const int32_t* __restrict__ ids, int P, int E,
                                                                   const int32_t* __restrict__ soe, double bp,
                                                                   double bh, int32_t* __restrict__ ids2,
                                                                   int32_t* __restrict__ skip,
                                                                   int32_t* __restrict__ out) {
  extern __shared__ int32_t sm[];
  int32_t* cnt = sm;          // [E] pairs per expert
  int32_t* host = sm + E;     // [E] 1: miss (then: host expert)
  int32_t* rank = sm + 2 * E; // [E] rank of a miss, -1 otherwise
  __shared__ int32_t s_m, s_h, s_rows;
  pdl_wait();
  pdl_trigger();
  for (int e = threadIdx.x; e < E; e += blockDim.x) cnt[e] = 0;
  if (threadIdx.x == 0) { s_m = 0; s_rows = 0; }
  __syncthreads();
  for (int q = threadIdx.x; q < P; q += blockDim.x) {
    const int e = ids[q];
    if (e >= 0 && e < E) atomicAdd(&cnt[e], 1);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    host[e] = cnt[e] > 0 && soe[e] < 0;
    if (host[e]) atomicAdd(&s_m, 1);
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const int m = s_m;
    int q = static_cast<int>(floor(static_cast<double>(m) * bp / (bp + bh) + 0.5));
    q = q < 0 ? 0 : q > m ? m : q;
    s_h = m - q;
  }
  __syncthreads();
  const int H = s_h;
  for (int e = threadIdx.x; e < E; e += blockDim.x) {   // rank among the misses by (pairs, id)
    int r = -1;
    if (host[e]) {
      r = 0;
      for (int f = 0; f < E; ++f)
        r += (host[f] && (cnt[f] < cnt[e] || (cnt[f] == cnt[e] && f < e))) ? 1 : 0;
    }
    rank[e] = r;
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    const int r = rank[e];
    host[e] = r >= 0 && r < H;
    skip[e] = host[e];
    if (host[e]) {
      out[4 + r] = e;
      atomicAdd(&s_rows, cnt[e]);
    }
  }
  __syncthreads();
  for (int q = threadIdx.x; q < P; q += blockDim.x) {
    const int e = ids[q];
    ids2[q] = (e >= 0 && e < E) ? (host[e] ? 2 * E : rank[e] >= 0 ? E + e : e) : e;
  }
  if (threadIdx.x == 0) { out[0] = s_m; out[1] = s_m - H; out[2] = H; out[3] = s_rows; }
}

cudaError_t launch_hybrid_split(const int32_t* ids, int P, int E, const int32_t* soe, double bp, double bh,
                                int32_t* ids2, int32_t* skip, int32_t* out, cudaStream_t st) {
  const size_t smem = sizeof(int32_t) * 3 * static_cast<size_t>(E);
  return launch_pdl(hybrid_split_kernel, dim3(1), dim3(kLruThreads), smem, st, ids, P, E, soe, bp, bh, ids2, skip,
                    out);
}

// Rollback of a step whose miss copies could not all be issued: the state
// before the step comes back from the backup (the layer's entries, every
// slot's key and last_use, and -- through the slots' old keys -- the entries
// of the keys the step evicted), except that the first n_dirty slots of the
// miss list (whose banks a copy may already have overwritten) are left empty
// and their previous keys unmapped.
__global__ void lru_restore_kernel(int E, int S, int key_base, int32_t* __restrict__ slot_of_key,
                                   int32_t* __restrict__ key_of_slot, int64_t* __restrict__ last_use,
                                   int32_t* __restrict__ ws, int n_dirty) {
  const int32_t* bk_soe = ws + 4 + 2 * E;
  const int32_t* bk_eos = bk_soe + E;
  const int64_t* bk_lu = lru_backup_lu(ws, E, S);
  for (int e = threadIdx.x; e < E; e += blockDim.x) slot_of_key[key_base + e] = bk_soe[e];
  __syncthreads();
  for (int j = threadIdx.x; j < S; j += blockDim.x) {
    key_of_slot[j] = bk_eos[j];
    last_use[j] = bk_lu[j];
    if (bk_eos[j] >= 0) slot_of_key[bk_eos[j]] = j;
  }
  __syncthreads();
  for (int i = threadIdx.x; i < n_dirty; i += blockDim.x) {
    const int sl = ws[4 + 2 * i + 1];
    const int old = bk_eos[sl];
    if (old >= 0) slot_of_key[old] = -1;
    key_of_slot[sl] = -1;
    last_use[sl] = -1;
  }
}

cudaError_t launch_lru_restore(int E, int S, int key_base, int32_t* soe, int32_t* eos, int64_t* lu, int32_t* ws,
                               int n_dirty, cudaStream_t st) {
  lru_restore_kernel<<<1, kLruThreads, 0, st>>>(E, S, key_base, soe, eos, lu, ws, n_dirty);
  return count_launch(cudaGetLastError());
}

// ---------------------------------------------------------------------------
// Elastic slot-pool resize (the pages: the expert cache's share of VRAM can be
// changed at run time without restarting or reloading weights; pomoai.com
// FreeToken hub, two-level expert memory; freelamp.com FreeToken article,
// section 2.3 "elastic memory management", `ftctl cache --moe <slots>`).
// The min(S_new, resident) most recently used resident experts stay (largest
// last_use first, ties to the lower old slot), compacted into slots 0.. in
// their old slot order, keeping their last_use; the rest are evicted.
//
// One block: each resident slot's rank in keep order is a count over the other
// slots (no sort); warp 0 scans the keep flags into new slot indices.  The
// move list goes to the workspace: ws[0] = kept, ws[1 + i] = old slot of new
// slot i; the bank copies then run on the device from that list.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kLruThreads) slot_resize_kernel(int E, int S_old,
                                                                  const int32_t* __restrict__ eos_old,
                                                                  const int64_t* __restrict__ lu_old, int S_new,
                                                                  int32_t* __restrict__ soe_new,
                                                                  int32_t* __restrict__ eos_new,
                                                                  int64_t* __restrict__ lu_new,
                                                                  int32_t* __restrict__ ws) {
  extern __shared__ __align__(8) uint8_t sm_raw[];
  int64_t* s_lu = reinterpret_cast<int64_t*>(sm_raw);            // [S_old]
  int32_t* s_eos = reinterpret_cast<int32_t*>(s_lu + S_old);     // [S_old]
  int32_t* s_pos = s_eos + S_old;                                 // [S_old] keep flag, then new slot (or -1)
  pdl_wait();
  pdl_trigger();
  for (int j = threadIdx.x; j < S_old; j += blockDim.x) { s_lu[j] = lu_old[j]; s_eos[j] = eos_old[j]; }
  for (int e = threadIdx.x; e < E; e += blockDim.x) soe_new[e] = -1;
  for (int j = threadIdx.x; j < S_new; j += blockDim.x) { eos_new[j] = -1; lu_new[j] = -1; }
  __syncthreads();
  for (int j = threadIdx.x; j < S_old; j += blockDim.x) {
    int keep = 0;
    if (s_eos[j] >= 0) {
      int before = 0;   // resident slots that come earlier in keep order
      for (int i = 0; i < S_old; ++i)
        before += (s_eos[i] >= 0 && (s_lu[i] > s_lu[j] || (s_lu[i] == s_lu[j] && i < j))) ? 1 : 0;
      keep = before < S_new;
    }
    s_pos[j] = keep;
  }
  __syncthreads();
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    const int per = (S_old + 31) / 32, b = lane * per, en = min(S_old, b + per);
    int cnt = 0;
    for (int j = b; j < en; ++j) cnt += s_pos[j];
    int incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    int run = incl - cnt;
    for (int j = b; j < en; ++j) {
      const int k = s_pos[j];
      s_pos[j] = k ? run : -1;
      run += k;
    }
    if (lane == 31) ws[0] = incl;
  }
  __syncthreads();
  for (int j = threadIdx.x; j < S_old; j += blockDim.x) {
    const int n = s_pos[j];
    if (n < 0) continue;
    eos_new[n] = s_eos[j];
    lu_new[n] = s_lu[j];
    soe_new[s_eos[j]] = n;
    ws[1 + n] = j;
  }
}

// Bank moves of a resize: new slot y <- old slot ws[1 + y] for y < ws[0];
// blockIdx.y = new slot, blocks along x stride over the bank in 16-byte vectors.
__global__ void bank_move_kernel(const uint8_t* __restrict__ old_pool, uint8_t* __restrict__ new_pool,
                                 size_t bank_bytes, const int32_t* __restrict__ ws) {
  pdl_wait();
  pdl_trigger();
  const int y = blockIdx.y;
  if (y >= ws[0]) return;
  const uint4* src = reinterpret_cast<const uint4*>(old_pool + static_cast<size_t>(ws[1 + y]) * bank_bytes);
  uint4* dst = reinterpret_cast<uint4*>(new_pool + static_cast<size_t>(y) * bank_bytes);
  const size_t n = bank_bytes / 16;
  for (size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<size_t>(gridDim.x) * blockDim.x)
    dst[i] = src[i];
}

cudaError_t launch_slot_resize(int E, int S_old, const int32_t* eos_old, const int64_t* lu_old, int S_new,
                               int32_t* soe_new, int32_t* eos_new, int64_t* lu_new, const void* old_pool,
                               void* new_pool, size_t bank_bytes, int32_t* ws, cudaStream_t st) {
  const size_t smem = (sizeof(int64_t) + 2 * sizeof(int32_t)) * static_cast<size_t>(S_old);
  cudaError_t err =
      cudaFuncSetAttribute(slot_resize_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (err != cudaSuccess) return err;
  err = launch_pdl(slot_resize_kernel, dim3(1), dim3(kLruThreads), smem, st, E, S_old, eos_old, lu_old, S_new,
                   soe_new, eos_new, lu_new, ws);
  if (err != cudaSuccess) return err;
  const int moves = S_old < S_new ? S_old : S_new;
  const size_t vec = bank_bytes / 16;
  const int bx = static_cast<int>((vec + 256 * 16 - 1) / (256 * 16) < 64 ? (vec + 256 * 16 - 1) / (256 * 16) : 64);
  return launch_pdl(bank_move_kernel, dim3(bx > 0 ? bx : 1, moves), dim3(256), 0, st,
                    static_cast<const uint8_t*>(old_pool), static_cast<uint8_t*>(new_pool), bank_bytes,
                    static_cast<const int32_t*>(ws));
}

}  // namespace ftm
