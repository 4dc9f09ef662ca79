// C ABI of the routed-MoE layer: argument validation, workspace carving, the
// miss-copy orchestration of the slot cache, and the whole-layer sequence.
// Every computation step runs in the kernels of the sibling .cu files.
#include <stdarg.h>
#include <atomic>
#include <cmath>
#include <vector>
#include <stdio.h>
#include <string.h>

#include <chrono>

#include "ftm_common.cuh"
#include "ftm_host_ffn.h"

namespace ftm {
cudaError_t launch_route(bool f32, const void* x, int T, int d, const void* wr, const float* bias, int E, int k,
                         int32_t* ids, float* w, cudaStream_t st);
cudaError_t launch_permute(const int32_t* ids, int P, int E, int32_t* counts, int32_t* offsets, int32_t* perm,
                           int32_t* inv, void* ws, cudaStream_t st);
size_t permute_workspace_bytes(int E, int64_t P);
size_t lru_workspace_bytes(int E, int S);
cudaError_t launch_lru_step(const int32_t* ids, int P, int E, int S, int64_t step, int64_t reserve, int key_base,
                            const int32_t* skip, int32_t* soe, int32_t* eos, int64_t* lu, int32_t* ws,
                            cudaStream_t st);
cudaError_t launch_hybrid_split(const int32_t* ids, int P, int E, const int32_t* soe, double bp, double bh,
                                int32_t* ids2, int32_t* skip, int32_t* out, cudaStream_t st);
cudaError_t launch_miss_relabel(const int32_t* ids, int P, int E, const int32_t* soe, int32_t* ids2,
                                cudaStream_t st);
cudaError_t launch_lru_restore(int E, int S, int key_base, int32_t* soe, int32_t* eos, int64_t* lu, int32_t* ws,
                               int n_dirty, cudaStream_t st);
cudaError_t launch_slot_resize(int E, int S_old, const int32_t* eos_old, const int64_t* lu_old, int S_new,
                               int32_t* soe_new, int32_t* eos_new, int64_t* lu_new, const void* old_pool,
                               void* new_pool, size_t bank_bytes, int32_t* ws, cudaStream_t st);
cudaError_t launch_wait_selftest(cudaStream_t st);
cudaError_t launch_combine(bool f32, const void* y, const int32_t* inv, const float* gw, int T, int k, int d, int P,
                           int has_shared, void* out, cudaStream_t st);
const char* launch_expert_ffn(const FfnArgs& a, cudaStream_t st, cudaError_t* cerr);
size_t fp8_ffn_workspace_bytes(int64_t rows, int d, int I);
size_t nvfp4_ffn_workspace_bytes(int64_t P, int T, int E, int has_shared, int d, int I);
const char* launch_expert_ffn_nvfp4(const FfnArgs& a, size_t s_gu_off, size_t s_d_off, size_t s_t_off, uint8_t* ws,
                                    cudaStream_t st, cudaError_t* cerr);
const char* launch_expert_ffn_fp8(const FfnArgs& a, size_t s_gu_off, size_t s_d_off, uint8_t* ws, cudaStream_t st,
                                  cudaError_t* cerr);
const char* launch_expert_ffn_mxfp4(const FfnArgs& a, size_t s_gu_off, size_t s_d_off, uint8_t* ws, cudaStream_t st,
                                    cudaError_t* cerr);
}  // namespace ftm

using namespace ftm;

namespace {

thread_local char g_err[512] = "";
thread_local cudaEvent_t g_prof[FTM_K_COUNT][2] = {};

ftm_status fail(ftm_status s, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return s;
}

ftm_status cuda_fail(cudaError_t e, const char* what) {
  return fail(FTM_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

ftm_status ok() {
  g_err[0] = 0;
  return FTM_OK;
}

inline cudaStream_t S_(void* s) { return static_cast<cudaStream_t>(s); }

constexpr size_t kAlign = 256;
inline size_t al(size_t b) { return (b + kAlign - 1) & ~(kAlign - 1); }
inline bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

ftm_status check_desc(const ftm_layer_desc* L) {
  if (!L) return fail(FTM_ERR_INVALID_ARG, "layer descriptor is NULL");
  if (L->reserved != 0) return fail(FTM_ERR_INVALID_ARG, "reserved field must be 0");
  if (L->wdtype < FTM_F32 || L->wdtype > FTM_MXFP4) return fail(FTM_ERR_INVALID_ARG, "unknown wdtype %d", L->wdtype);
  const int q = (L->wdtype == FTM_NVFP4 || L->wdtype == FTM_MXFP4) ? 256 : 128;
  if (L->d <= 0 || L->d % q) return fail(FTM_ERR_INVALID_ARG, "d=%d must be a positive multiple of %d", L->d, q);
  if (L->I <= 0 || L->I % q) return fail(FTM_ERR_INVALID_ARG, "I=%d must be a positive multiple of %d", L->I, q);
  if (L->E < 1 || L->E > 512) return fail(FTM_ERR_INVALID_ARG, "E=%d out of [1, 512]", L->E);
  if (L->k < 1 || L->k > 16 || L->k > L->E) return fail(FTM_ERR_INVALID_ARG, "k=%d out of [1, min(E,16)]", L->k);
  if (L->S < 1) return fail(FTM_ERR_INVALID_ARG, "S=%d must be >= 1", L->S);
  if (L->has_shared != 0 && L->has_shared != 1) return fail(FTM_ERR_INVALID_ARG, "has_shared must be 0 or 1");
  return FTM_OK;
}

ftm_status check_T(int32_t T) {
  if (T < 0) return fail(FTM_ERR_INVALID_ARG, "T=%d is negative", T);
  if (static_cast<int64_t>(T) * 16 > (1ll << 30)) return fail(FTM_ERR_INVALID_ARG, "T=%d too large", T);
  return FTM_OK;
}

void bank_layout(const ftm_layer_desc* L, ftm_bank_layout* b) {
  memset(b, 0, sizeof(*b));
  const uint64_t d = L->d, I = L->I;
  uint64_t wgu = 0, wd = 0, sgu = 0, sd = 0, st = 0;
  switch (L->wdtype) {
    case FTM_F32: wgu = 2 * I * d * 4; wd = d * I * 4; break;
    case FTM_BF16: wgu = 2 * I * d * 2; wd = d * I * 2; break;
    case FTM_FP8_E4M3_B128:
      wgu = 2 * I * d; wd = d * I;
      sgu = (2 * I / 128) * (d / 128) * 4; sd = (d / 128) * (I / 128) * 4;
      break;
    case FTM_NVFP4:
      wgu = 2 * I * d / 2; wd = d * I / 2;
      sgu = 2 * I * (d / 16); sd = d * (I / 16); st = 16;
      break;
    case FTM_MXFP4:
      wgu = 2 * I * d / 2; wd = d * I / 2;
      sgu = 2 * I * (d / 32); sd = d * (I / 32);
      break;
  }
  uint64_t off = 0;
  b->w_gu_off = off; b->w_gu_bytes = wgu; off = al(off + wgu);
  b->w_d_off = off; b->w_d_bytes = wd; off = al(off + wd);
  b->s_gu_off = off; b->s_gu_bytes = sgu; off = al(off + sgu);
  b->s_d_off = off; b->s_d_bytes = sd; off = al(off + sd);
  b->s_t_off = off; b->s_t_bytes = st; off = al(off + st);
  b->bank_bytes = off;
}

int64_t ffn_rows(const ftm_layer_desc* L, int32_t T) {
  return static_cast<int64_t>(T) * L->k + (L->has_shared ? T : 0);
}

size_t act_elt(const ftm_layer_desc* L) { return L->wdtype == FTM_F32 ? 4 : 2; }

size_t ffn_ws_bytes(const ftm_layer_desc* L, int32_t T) {
  const size_t rows = static_cast<size_t>(ffn_rows(L, T));
  if (L->wdtype == FTM_FP8_E4M3_B128) return fp8_ffn_workspace_bytes(static_cast<int64_t>(rows), L->d, L->I);
  if (L->wdtype == FTM_NVFP4 || L->wdtype == FTM_MXFP4)   // MXFP4 needs at most NVFP4's scratch
    return nvfp4_ffn_workspace_bytes(static_cast<int64_t>(T) * L->k, T, L->E, L->has_shared, L->d, L->I);
  return al(rows * L->d * act_elt(L)) + al(rows * L->I * act_elt(L));
}

// Whole-layer workspace carving.
struct LayerWs {
  int32_t* ids;
  float* gates;
  int32_t* counts;
  int32_t* offsets;
  int32_t* perm;
  int32_t* inv;
  void* perm_ws;
  uint8_t* ffn_ws;
  void* y;
  int32_t* lru_ws;
  // cache steps: group labels (hits e, misses E + e, host experts 2E), their
  // counts / offsets over 2E + 1 groups and the permutation's workspace
  int32_t* ids2;
  int32_t* counts2;
  int32_t* offsets2;
  void* perm_ws2;
  size_t total;
};

LayerWs carve(const ftm_layer_desc* L, int32_t T, uint8_t* base) {
  LayerWs w;
  const size_t P = static_cast<size_t>(T) * L->k;
  size_t off = 0;
  auto take = [&](size_t bytes) { uint8_t* p = base ? base + off : nullptr; off += al(bytes); return p; };
  w.ids = reinterpret_cast<int32_t*>(take(P * 4));
  w.gates = reinterpret_cast<float*>(take(P * 4));
  w.counts = reinterpret_cast<int32_t*>(take(static_cast<size_t>(L->E) * 4));
  w.offsets = reinterpret_cast<int32_t*>(take((static_cast<size_t>(L->E) + 1) * 4));
  w.perm = reinterpret_cast<int32_t*>(take(P * 4));
  w.inv = reinterpret_cast<int32_t*>(take(P * 4));
  w.perm_ws = take(permute_workspace_bytes(L->E, static_cast<int64_t>(P)));
  w.ffn_ws = take(ffn_ws_bytes(L, T));
  w.y = take(static_cast<size_t>(ffn_rows(L, T)) * L->d * act_elt(L));
  w.lru_ws = reinterpret_cast<int32_t*>(take(lru_workspace_bytes(L->E, L->S)));
  const size_t G2 = 2 * static_cast<size_t>(L->E) + 1;
  w.ids2 = reinterpret_cast<int32_t*>(take(P * 4));
  w.counts2 = reinterpret_cast<int32_t*>(take(G2 * 4));
  w.offsets2 = reinterpret_cast<int32_t*>(take((G2 + 1) * 4));
  w.perm_ws2 = take(permute_workspace_bytes(static_cast<int>(G2), static_cast<int64_t>(P)));
  w.total = off;
  return w;
}

// Workspace of the hybrid layer: the layer's own (its perm / inv hold the
// permutation over 2E + 1 groups), then the split's output and the lookup's
// skip mask.
struct HybridWs {
  LayerWs w;
  int32_t* split;
  int32_t* skip;
  size_t total;
};

HybridWs carve_hybrid(const ftm_layer_desc* L, int32_t T, uint8_t* base) {
  HybridWs h;
  h.w = carve(L, T, base);
  const size_t E = static_cast<size_t>(L->E);
  size_t off = h.w.total;
  auto take = [&](size_t bytes) { uint8_t* p = base ? base + off : nullptr; off += al(bytes); return p; };
  h.split = reinterpret_cast<int32_t*>(take((4 + E) * 4));
  h.skip = reinterpret_cast<int32_t*>(take(E * 4));
  h.total = off;
  return h;
}

// Pinned host workspace of the hybrid layer (64-byte aligned pieces).
struct HybridHost {
  int32_t* split;          // [4 + E] the split's output
  int32_t* ids;            // [P] routed ids
  int32_t* perm;           // [P] the E + 1-group permutation
  int32_t* offsets;        // [2E + 2]
  uint8_t* x;              // [T][d] activations
  uint8_t* y;              // [P][d] outputs of the host rows
  float* scratch;          // host FFN scratch
  const uint8_t** xrow;    // [P]
  uint8_t** yrow;          // [P]
  HostGroup* groups;       // [E]
  int32_t* gidx;           // [E] host group of an expert, -1
  int32_t* gpos;           // [E + 1] first row of each host group
  float* act;              // [2] NVFP4 activation global scales
  size_t total;
};

HybridHost carve_host(const ftm_layer_desc* L, int32_t T, void* base_v) {
  HybridHost h;
  uint8_t* base = static_cast<uint8_t*>(base_v);
  const size_t P = static_cast<size_t>(T) * L->k, E = static_cast<size_t>(L->E);
  const size_t row = static_cast<size_t>(L->d) * act_elt(L);
  size_t off = 0;
  auto take = [&](size_t bytes) { uint8_t* p = base ? base + off : nullptr; off += (bytes + 63) & ~size_t{63}; return p; };
  h.split = reinterpret_cast<int32_t*>(take((4 + E) * 4));
  h.ids = reinterpret_cast<int32_t*>(take(P * 4));
  h.perm = reinterpret_cast<int32_t*>(take(P * 4));
  h.offsets = reinterpret_cast<int32_t*>(take((2 * E + 2) * 4));
  h.x = take(static_cast<size_t>(T) * row);
  h.y = take(P * row);
  h.scratch = reinterpret_cast<float*>(take(host_ffn_scratch_bytes(L, static_cast<int64_t>(P))));
  h.xrow = reinterpret_cast<const uint8_t**>(take(P * sizeof(void*)));
  h.yrow = reinterpret_cast<uint8_t**>(take(P * sizeof(void*)));
  h.groups = reinterpret_cast<HostGroup*>(take(E * sizeof(HostGroup)));
  h.gidx = reinterpret_cast<int32_t*>(take(E * 4));
  h.gpos = reinterpret_cast<int32_t*>(take((E + 1) * 4));
  h.act = reinterpret_cast<float*>(take(2 * sizeof(float)));
  h.total = off;
  return h;
}

ftm_status check_ws(void* ws, size_t have, size_t need, const char* who) {
  if (need && !ws) return fail(FTM_ERR_INVALID_ARG, "%s: workspace is NULL (%zu bytes needed)", who, need);
  if (have < need) return fail(FTM_ERR_INVALID_ARG, "%s: workspace %zu bytes < %zu needed", who, have, need);
  if (ws && !aligned(ws, kAlign)) return fail(FTM_ERR_INVALID_ARG, "%s: workspace not 256-byte aligned", who);
  return FTM_OK;
}

cudaEvent_t copy_event() {
  static thread_local cudaEvent_t ev = nullptr;
  static thread_local int dev = -1;
  int cur = 0;
  cudaGetDevice(&cur);
  if (!ev || dev != cur) {
    if (ev) cudaEventDestroy(ev);
    ev = nullptr;
    if (cudaEventCreateWithFlags(&ev, cudaEventDisableTiming) != cudaSuccess) ev = nullptr;
    dev = cur;
  }
  return ev;
}

// Cache arguments shared by the lookup and the staging calls.
ftm_status check_cache(const ftm_layer_desc* L, const ftm_slot_cache* C, const char* who) {
  if (!C || !C->slot_of_expert || !C->expert_of_slot || !C->last_use || !C->slot_pool || !C->host_pool ||
      !C->host_scratch)
    return fail(FTM_ERR_INVALID_ARG, "%s: cache has a NULL member", who);
  if (L->S > 4096) return fail(FTM_ERR_UNSUPPORTED, "LRU cache supports S <= 4096 (S=%d)", L->S);
  const int n_keys = C->n_keys ? C->n_keys : L->E;
  if (n_keys < L->E || C->key_base < 0 || static_cast<int64_t>(C->key_base) + L->E > n_keys)
    return fail(FTM_ERR_INVALID_ARG, "%s: key_base=%d + E=%d outside the cache's %d keys", who, C->key_base, L->E,
                n_keys);
  cudaPointerAttributes pa;
  if (cudaPointerGetAttributes(&pa, C->host_pool) != cudaSuccess || pa.type != cudaMemoryTypeHost) {
    cudaGetLastError();
    return fail(FTM_ERR_INVALID_ARG, "%s: host_pool is not pinned host memory", who);
  }
  return FTM_OK;
}

cudaEvent_t list_event() {
  static thread_local cudaEvent_t ev = nullptr;
  static thread_local int dev = -1;
  int cur = 0;
  cudaGetDevice(&cur);
  if (!ev || dev != cur) {
    if (ev) cudaEventDestroy(ev);
    ev = nullptr;
    if (cudaEventCreateWithFlags(&ev, cudaEventDisableTiming) != cudaSuccess) ev = nullptr;
    dev = cur;
  }
  return ev;
}

// One cache step of the layer at C->key_base: the lookup/update kernel on
// `lru_stream` (ids == nullptr: all E experts of the layer), after `after`
// when given, the miss list read back (the host waits for that kernel only),
// then one bank copy per miss on `copy_stream` (also after `after`).  Victims
// are the slots with last_use < reserve.  On a copy failure the state is
// rolled back (slots a copy may have written left empty).  skip (device,
// [E], nullable): experts flagged nonzero are not requests (see
// hybrid_split_kernel).
ftm_status cache_step(const ftm_layer_desc* L, ftm_slot_cache* C, const int32_t* ids, int P, int64_t reserve,
                      int32_t* ws, cudaStream_t lru_stream, cudaStream_t copy_stream, cudaEvent_t after,
                      int* misses_out, const int32_t* skip = nullptr) {
  *misses_out = 0;
  cudaError_t e;
  // the step rewrites the entries of the keys it evicts: the compute that
  // reads them (done when `after` completes) must be over first
  if (after && (e = cudaStreamWaitEvent(lru_stream, after, 0)) != cudaSuccess) return cuda_fail(e, "lru stream wait");
  prof_mark(FTM_K_LRU, lru_stream, false);
  e = launch_lru_step(ids, P, L->E, L->S, C->step, reserve, C->key_base, skip, C->slot_of_expert,
                                  C->expert_of_slot, C->last_use, ws, lru_stream);
  prof_mark(FTM_K_LRU, lru_stream, true);
  if (e != cudaSuccess) return cuda_fail(e, "lru step launch");
  const size_t hdr = sizeof(int32_t) * (4 + 2 * static_cast<size_t>(L->E));
  if ((e = cudaMemcpyAsync(C->host_scratch, ws, hdr, cudaMemcpyDeviceToHost, lru_stream)) != cudaSuccess)
    return cuda_fail(e, "miss list copy");
  cudaEvent_t lev = list_event();
  if (!lev) return fail(FTM_ERR_CUDA, "could not create the miss-list event");
  if ((e = cudaEventRecord(lev, lru_stream)) != cudaSuccess) return cuda_fail(e, "miss list event record");
  if ((e = cudaEventSynchronize(lev)) != cudaSuccess) return cuda_fail(e, "lru step");
  const int32_t* h = C->host_scratch;
  C->last_distinct = h[1];
  C->last_hits = h[2];
  C->last_misses = h[3];
  if (h[0] == FTM_ERR_INVALID_ARG)
    return fail(FTM_ERR_INVALID_ARG, "step %lld: topk_ids holds an expert id outside [0, %d); state unchanged",
                static_cast<long long>(C->step), L->E);
  if (h[0] == FTM_ERR_CAPACITY)
    return fail(FTM_ERR_CAPACITY, "step %lld requests %d distinct experts, more than the %d slots it may fill",
                static_cast<long long>(C->step), h[1], L->S);
  ftm_bank_layout bl;
  bank_layout(L, &bl);
  const int misses = h[3];
  if (misses > 0 && after && copy_stream != lru_stream &&
      (e = cudaStreamWaitEvent(copy_stream, after, 0)) != cudaSuccess)
    return cuda_fail(e, "copy stream wait");
  bool copy_failed = false;
  const char* why = nullptr;
  int n_dirty = 0;     // miss-list slots a copy may have written
  for (int i = 0; i < misses && !copy_failed; ++i) {
    if (C->fail_before_copy > 0 && i + 1 == C->fail_before_copy) {
      copy_failed = true;
      why = "injected copy failure (fail_before_copy)";
      break;
    }
    const int key = h[4 + 2 * i], sl = h[4 + 2 * i + 1];
    e = cudaMemcpyAsync(static_cast<uint8_t*>(C->slot_pool) + static_cast<size_t>(sl) * bl.bank_bytes,
                        static_cast<const uint8_t*>(C->host_pool) + static_cast<size_t>(key) * bl.bank_bytes,
                        bl.bank_bytes, cudaMemcpyHostToDevice, copy_stream);
    n_dirty = i + 1;     // a copy that failed to issue may still have started
    if (e != cudaSuccess) { copy_failed = true; why = cudaGetErrorString(e); }
  }
  if (copy_failed) {
    C->fail_before_copy = 0;
    cudaError_t e2 = launch_lru_restore(L->E, L->S, C->key_base, C->slot_of_expert, C->expert_of_slot, C->last_use,
                                        ws, n_dirty, lru_stream);
    if (e2 == cudaSuccess) e2 = cudaStreamSynchronize(lru_stream);
    return fail(FTM_ERR_CUDA, "a miss copy failed (%s) with %d of %d copies issued; slot state rolled back, the "
                "%d slot(s) a copy may have written left empty%s", why, n_dirty, misses, n_dirty,
                e2 == cudaSuccess ? "" : " -- rollback failed too");
  }
  C->step += 1;
  *misses_out = misses;
  return FTM_OK;
}

// The expert FFN of a cache step in two launches over the permutation of 2E
// groups (w.offsets2, labels from miss_relabel_kernel or hybrid_split_kernel):
// groups 0..E-1, the hit experts (and the shared expert), at once, so their
// tiles run while the misses are copied; after the copies (an event on the
// copy stream), groups E..2E-1, the copied misses, with no shared expert.  Both
// write Y at the pairs' positions, so the combine reads it through w.inv.  The
// profile events of the FFN's kernels bracket the first launch only.
ftm_status ffn_hits_then_misses(const ftm_layer_desc* L, const ftm_layer_weights* W, const ftm_slot_cache* C,
                                const void* x, int T, const LayerWs& w, int misses, cudaStream_t cs,
                                cudaStream_t ps) {
  const int32_t* soe = C->slot_of_expert + C->key_base;
  ftm_status s = ftm_expert_ffn(L, x, T, w.offsets2, w.perm, soe, C->slot_pool, W->shared_bank, W->act_scale, w.y,
                                w.ffn_ws, ffn_ws_bytes(L, T), cs);
  if (s || misses == 0) return s;
  cudaError_t e;
  cudaEvent_t ev = copy_event();
  if (!ev) return fail(FTM_ERR_CUDA, "could not create the copy event");
  if ((e = cudaEventRecord(ev, ps)) != cudaSuccess) return cuda_fail(e, "copy event record");
  if ((e = cudaStreamWaitEvent(cs, ev, 0)) != cudaSuccess) return cuda_fail(e, "copy event wait");
  ftm_layer_desc Lm = *L;
  Lm.has_shared = 0;
  const int hooks[3] = {FTM_K_GATHER, FTM_K_GEMM1, FTM_K_GEMM2};
  cudaEvent_t saved[3][2];
  for (int i = 0; i < 3; ++i) {
    saved[i][0] = g_prof[hooks[i]][0];
    saved[i][1] = g_prof[hooks[i]][1];
    g_prof[hooks[i]][0] = g_prof[hooks[i]][1] = nullptr;
  }
  s = ftm_expert_ffn(&Lm, x, T, w.offsets2 + L->E, w.perm, soe, C->slot_pool, nullptr, W->act_scale, w.y, w.ffn_ws,
                     ffn_ws_bytes(&Lm, T), cs);
  for (int i = 0; i < 3; ++i) {
    g_prof[hooks[i]][0] = saved[i][0];
    g_prof[hooks[i]][1] = saved[i][1];
  }
  return s;
}

thread_local char g_warn[256] = "";

// Events of the multi-layer pipeline, per thread and device: [0, 1] a layer's
// experts are in their slots (by layer parity), [2, 3] a layer's compute is
// done, [4] the work enqueued before the call.
cudaEvent_t pipe_event(int i) {
  static thread_local cudaEvent_t ev[5] = {};
  static thread_local int dev = -1;
  int cur = 0;
  cudaGetDevice(&cur);
  if (dev != cur) {
    for (auto& x : ev) {
      if (x) cudaEventDestroy(x);
      x = nullptr;
    }
    dev = cur;
  }
  if (!ev[i] && cudaEventCreateWithFlags(&ev[i], cudaEventDisableTiming) != cudaSuccess) ev[i] = nullptr;
  return ev[i];
}

}  // namespace

ftm_status ftm::report_error(ftm_status s, const char* msg) { return fail(s, "%s", msg); }

namespace {
std::atomic<unsigned long long> g_launches{0};
}

cudaError_t ftm::count_launch(cudaError_t e) {
  if (e == cudaSuccess) g_launches.fetch_add(1, std::memory_order_relaxed);
  return e;
}

void ftm::prof_mark(int which, cudaStream_t st, bool stop) {
  if (which < 0 || which >= FTM_K_COUNT || !g_prof[which][stop ? 1 : 0]) return;
  // under stream capture the record must become a graph node of its own
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  cudaStreamIsCapturing(st, &cs);
  if (cs == cudaStreamCaptureStatusActive)
    cudaEventRecordWithFlags(g_prof[which][stop ? 1 : 0], st, cudaEventRecordExternal);
  else
    cudaEventRecord(g_prof[which][stop ? 1 : 0], st);
}

extern "C" {

const char* ftm_last_error(void) { return g_err; }

uint64_t ftm_kernel_launches(void) { return g_launches.load(std::memory_order_relaxed); }

ftm_status ftm_set_profile_events(int32_t which, void* start_event, void* stop_event) {
  if (which < 0 || which >= FTM_K_COUNT) return fail(FTM_ERR_INVALID_ARG, "kernel id %d out of range", which);
  if ((start_event == nullptr) != (stop_event == nullptr))
    return fail(FTM_ERR_INVALID_ARG, "start and stop events must both be set or both be NULL");
  g_prof[which][0] = static_cast<cudaEvent_t>(start_event);
  g_prof[which][1] = static_cast<cudaEvent_t>(stop_event);
  return ok();
}

ftm_status ftm_selftest_bounded_wait(int32_t* observed, void* stream) {
  if (observed == nullptr) return fail(FTM_ERR_INVALID_ARG, "ftm_selftest_bounded_wait: observed is NULL");
  cudaError_t e = ftm::launch_wait_selftest(S_(stream));
  if (e == cudaSuccess) e = cudaStreamSynchronize(S_(stream));
  if (e != cudaSuccess) return fail(FTM_ERR_CUDA, "ftm_selftest_bounded_wait: %s", cudaGetErrorString(e));
  *observed = ftm_device_status(1);
  return FTM_OK;
}

int32_t ftm_device_status(int32_t reset) {
  cudaDeviceSynchronize();
  int32_t v = 0;
  if (cudaMemcpyFromSymbol(&v, g_dev_status, sizeof(v)) != cudaSuccess) return -1;
  if (reset) {
    const int32_t z = 0;
    cudaMemcpyToSymbol(g_dev_status, &z, sizeof(z));
  }
  return v;
}

ftm_status ftm_get_bank_layout(const ftm_layer_desc* L, ftm_bank_layout* out) {
  ftm_status s = check_desc(L);
  if (s) return s;
  if (!out) return fail(FTM_ERR_INVALID_ARG, "out is NULL");
  bank_layout(L, out);
  return ok();
}

ftm_status ftm_route(const ftm_layer_desc* L, const void* x, int32_t T, const void* w_router, const float* bias,
                     int32_t* topk_ids, float* topk_w, void* stream) {
  ftm_status s = check_desc(L);
  if (s || (s = check_T(T))) return s;
  if (T == 0) return ok();
  if (!x || !w_router || !topk_ids || !topk_w) return fail(FTM_ERR_INVALID_ARG, "ftm_route: NULL pointer");
  if (!aligned(x, 16) || !aligned(w_router, 16)) return fail(FTM_ERR_INVALID_ARG, "ftm_route: x/w_router not 16-byte aligned");
  prof_mark(FTM_K_ROUTE, S_(stream), false);
  cudaError_t e = launch_route(L->wdtype == FTM_F32, x, T, L->d, w_router, bias, L->E, L->k, topk_ids, topk_w, S_(stream));
  prof_mark(FTM_K_ROUTE, S_(stream), true);
  if (e != cudaSuccess) return cuda_fail(e, "ftm_route launch");
  return ok();
}

size_t ftm_permute_workspace_bytes(const ftm_layer_desc* L, int32_t T) {
  if (check_desc(L) || T < 0) return 0;
  return permute_workspace_bytes(L->E, static_cast<int64_t>(T) * L->k);
}

ftm_status ftm_permute(const ftm_layer_desc* L, const int32_t* topk_ids, int32_t T, int32_t* counts, int32_t* offsets,
                       int32_t* perm, int32_t* inv, void* workspace, size_t ws_bytes, void* stream) {
  ftm_status s = check_desc(L);
  if (s || (s = check_T(T))) return s;
  if (!counts || !offsets) return fail(FTM_ERR_INVALID_ARG, "ftm_permute: NULL counts/offsets");
  const int64_t P = static_cast<int64_t>(T) * L->k;
  if (P > 0 && (!topk_ids || !perm || !inv)) return fail(FTM_ERR_INVALID_ARG, "ftm_permute: NULL pointer");
  if ((s = check_ws(workspace, ws_bytes, permute_workspace_bytes(L->E, P), "ftm_permute"))) return s;
  prof_mark(FTM_K_PERMUTE, S_(stream), false);
  cudaError_t e = launch_permute(topk_ids, static_cast<int>(P), L->E, counts, offsets, perm, inv, workspace, S_(stream));
  prof_mark(FTM_K_PERMUTE, S_(stream), true);
  if (e != cudaSuccess) return cuda_fail(e, "ftm_permute launch");
  return ok();
}

size_t ftm_slot_host_scratch_ints(const ftm_layer_desc* L) {
  if (check_desc(L)) return 0;
  return 4 + 2 * static_cast<size_t>(L->E);
}

size_t ftm_slot_workspace_bytes(const ftm_layer_desc* L) {
  if (check_desc(L)) return 0;
  return lru_workspace_bytes(L->E, L->S);
}

ftm_status ftm_slot_resize(const ftm_layer_desc* L, const ftm_slot_cache* C, int32_t S_new, ftm_slot_cache* C_new,
                           void* workspace, size_t ws_bytes, void* stream) {
  ftm_status s = check_desc(L);
  if (s) return s;
  if (!C || !C->slot_of_expert || !C->expert_of_slot || !C->last_use || !C->slot_pool)
    return fail(FTM_ERR_INVALID_ARG, "ftm_slot_resize: cache has a NULL member");
  if (!C_new || !C_new->slot_of_expert || !C_new->expert_of_slot || !C_new->last_use || !C_new->slot_pool)
    return fail(FTM_ERR_INVALID_ARG, "ftm_slot_resize: new cache has a NULL member");
  if (S_new < 1) return fail(FTM_ERR_INVALID_ARG, "ftm_slot_resize: S_new=%d < 1", S_new);
  if (L->S > 4096 || S_new > 4096)
    return fail(FTM_ERR_UNSUPPORTED, "LRU cache supports S <= 4096 (S=%d, S_new=%d)", L->S, S_new);
  ftm_bank_layout bl;
  if ((s = ftm_get_bank_layout(L, &bl))) return s;
  // the new pool and state must not overlap the old ones (the moves read the old pool while writing the new)
  const uintptr_t o0 = reinterpret_cast<uintptr_t>(C->slot_pool), o1 = o0 + bl.bank_bytes * L->S;
  const uintptr_t n0 = reinterpret_cast<uintptr_t>(C_new->slot_pool), n1 = n0 + bl.bank_bytes * S_new;
  if (n0 < o1 && o0 < n1) return fail(FTM_ERR_INVALID_ARG, "ftm_slot_resize: new slot pool overlaps the old one");
  if (C_new->slot_of_expert == C->slot_of_expert || C_new->expert_of_slot == C->expert_of_slot ||
      C_new->last_use == C->last_use)
    return fail(FTM_ERR_INVALID_ARG, "ftm_slot_resize: new state arrays must be distinct from the old ones");
  if ((s = check_ws(workspace, ws_bytes, lru_workspace_bytes(L->E, L->S), "ftm_slot_resize"))) return s;
  const int n_keys = C->n_keys ? C->n_keys : L->E;
  cudaError_t e = launch_slot_resize(n_keys, L->S, C->expert_of_slot, C->last_use, S_new, C_new->slot_of_expert,
                                     C_new->expert_of_slot, C_new->last_use, C->slot_pool, C_new->slot_pool,
                                     bl.bank_bytes, static_cast<int32_t*>(workspace), S_(stream));
  if (e != cudaSuccess) return cuda_fail(e, "slot resize launch");
  C_new->step = C->step;
  C_new->n_keys = C->n_keys;
  C_new->key_base = C->key_base;
  C_new->last_distinct = C_new->last_hits = C_new->last_misses = 0;
  return FTM_OK;
}

ftm_status ftm_slot_lookup_update(const ftm_layer_desc* L, ftm_slot_cache* C, const int32_t* topk_ids, int32_t T,
                                  void* workspace, size_t ws_bytes, void* compute_stream, void* copy_stream) {
  ftm_status s = check_desc(L);
  if (s || (s = check_T(T))) return s;
  const int64_t P = static_cast<int64_t>(T) * L->k;
  if (P > 0 && !topk_ids) return fail(FTM_ERR_INVALID_ARG, "ftm_slot_lookup_update: NULL topk_ids");
  if ((s = check_cache(L, C, "ftm_slot_lookup_update"))) return s;
  if ((s = check_ws(workspace, ws_bytes, lru_workspace_bytes(L->E, L->S), "ftm_slot_lookup_update"))) return s;
  cudaStream_t cs = S_(compute_stream), ps = S_(copy_stream);
  // the victims were last used by steps whose compute is ahead of the lookup
  // kernel on the compute stream, and the host waits for that kernel before
  // it issues any copy: no copy can overwrite a bank still being read
  int misses = 0;
  if ((s = cache_step(L, C, topk_ids, static_cast<int>(P), C->step, static_cast<int32_t*>(workspace), cs, ps, nullptr,
                      &misses)))
    return s;
  if (misses > 0) {
    cudaEvent_t ev = copy_event();
    cudaError_t e;
    if (!ev) return fail(FTM_ERR_CUDA, "could not create the copy event");
    if ((e = cudaEventRecord(ev, ps)) != cudaSuccess) return cuda_fail(e, "copy event record");
    if ((e = cudaStreamWaitEvent(cs, ev, 0)) != cudaSuccess) return cuda_fail(e, "copy event wait");
  }
  return ok();
}

ftm_status ftm_slot_stage_layer(const ftm_layer_desc* L, ftm_slot_cache* C, int32_t layer, int32_t hold_previous,
                                void* after_event, void* workspace, size_t ws_bytes, void* copy_stream,
                                void* ready_event) {
  ftm_status s = check_desc(L);
  if (s) return s;
  if (!C) return fail(FTM_ERR_INVALID_ARG, "ftm_slot_stage_layer: cache is NULL");
  const int n_keys = C->n_keys ? C->n_keys : L->E;
  if (layer < 0 || static_cast<int64_t>(layer + 1) * L->E > n_keys)
    return fail(FTM_ERR_INVALID_ARG, "ftm_slot_stage_layer: layer %d outside the cache's %d keys", layer, n_keys);
  const int32_t base_saved = C->key_base;
  C->key_base = layer * L->E;
  s = check_cache(L, C, "ftm_slot_stage_layer");
  if (!s) s = check_ws(workspace, ws_bytes, lru_workspace_bytes(L->E, L->S), "ftm_slot_stage_layer");
  if (s) { C->key_base = base_saved; return s; }
  cudaStream_t ps = S_(copy_stream);
  int misses = 0;
  const int64_t reserve = hold_previous ? C->step - 1 : C->step;
  s = cache_step(L, C, nullptr, 0, reserve, static_cast<int32_t*>(workspace), ps, ps,
                 static_cast<cudaEvent_t>(after_event), &misses);
  if (s) { C->key_base = base_saved; return s; }
  cudaError_t e;
  if (ready_event && (e = cudaEventRecord(static_cast<cudaEvent_t>(ready_event), ps)) != cudaSuccess)
    return cuda_fail(e, "ready event record");
  return ok();
}

size_t ftm_ffn_workspace_bytes(const ftm_layer_desc* L, int32_t T) {
  if (check_desc(L) || T < 0) return 0;
  return ffn_ws_bytes(L, T);
}

ftm_status ftm_expert_ffn(const ftm_layer_desc* L, const void* x, int32_t T, const int32_t* offsets,
                          const int32_t* perm, const int32_t* slot_of_expert, const void* slot_pool,
                          const void* shared_bank, const float* act_scale, void* y, void* workspace, size_t ws_bytes,
                          void* stream) {
  ftm_status s = check_desc(L);
  if (s || (s = check_T(T))) return s;
  if (T == 0) return ok();
  if (!x || !offsets || !perm || !slot_of_expert || !slot_pool || !y)
    return fail(FTM_ERR_INVALID_ARG, "ftm_expert_ffn: NULL pointer");
  if (L->has_shared && !shared_bank) return fail(FTM_ERR_INVALID_ARG, "ftm_expert_ffn: layer has a shared expert but shared_bank is NULL");
  if (!aligned(slot_pool, 256) || (shared_bank && !aligned(shared_bank, 256)) || !aligned(x, 16) || !aligned(y, 16))
    return fail(FTM_ERR_INVALID_ARG, "ftm_expert_ffn: misaligned pointer (pool/bank 256 B, x/y 16 B)");
  if ((s = check_ws(workspace, ws_bytes, ffn_ws_bytes(L, T), "ftm_expert_ffn"))) return s;
  ftm_bank_layout bl;
  bank_layout(L, &bl);
  FfnArgs a;
  a.d = L->d; a.E = L->E; a.k = L->k; a.I = L->I; a.has_shared = L->has_shared; a.S = L->S;
  a.f32 = L->wdtype == FTM_F32;
  a.x = static_cast<const uint8_t*>(x);
  a.T = T;
  a.offsets = offsets; a.perm = perm; a.slot_of_expert = slot_of_expert;
  a.pool = static_cast<const uint8_t*>(slot_pool);
  a.shared_bank = static_cast<const uint8_t*>(shared_bank);
  a.bank_bytes = bl.bank_bytes; a.w_gu_off = bl.w_gu_off; a.w_d_off = bl.w_d_off;
  a.y = y;
  a.act_scale = act_scale;
  const size_t rows = static_cast<size_t>(ffn_rows(L, T));
  a.xp = static_cast<uint8_t*>(workspace);
  a.h = a.xp + al(rows * L->d * act_elt(L));
  cudaError_t ce;
  const char* msg;
  if (L->wdtype == FTM_MXFP4)
    msg = launch_expert_ffn_mxfp4(a, bl.s_gu_off, bl.s_d_off, static_cast<uint8_t*>(workspace), S_(stream), &ce);
  else if (L->wdtype == FTM_FP8_E4M3_B128)
    msg = launch_expert_ffn_fp8(a, bl.s_gu_off, bl.s_d_off, static_cast<uint8_t*>(workspace), S_(stream), &ce);
  else if (L->wdtype == FTM_NVFP4)
    msg = launch_expert_ffn_nvfp4(a, bl.s_gu_off, bl.s_d_off, bl.s_t_off, static_cast<uint8_t*>(workspace),
                                  S_(stream), &ce);
  else
    msg = launch_expert_ffn(a, S_(stream), &ce);
  if (msg) return ce != cudaSuccess ? cuda_fail(ce, msg) : fail(FTM_ERR_CUDA, "%s", msg);
  return ok();
}

ftm_status ftm_combine(const ftm_layer_desc* L, const void* y, const int32_t* inv, const float* topk_w, int32_t T,
                       void* out, void* stream) {
  ftm_status s = check_desc(L);
  if (s || (s = check_T(T))) return s;
  if (T == 0) return ok();
  if (!y || !inv || !topk_w || !out) return fail(FTM_ERR_INVALID_ARG, "ftm_combine: NULL pointer");
  if (!aligned(y, 16) || !aligned(out, 16)) return fail(FTM_ERR_INVALID_ARG, "ftm_combine: y/out not 16-byte aligned");
  prof_mark(FTM_K_COMBINE, S_(stream), false);
  cudaError_t e = launch_combine(L->wdtype == FTM_F32, y, inv, topk_w, T, L->k, L->d, T * L->k, L->has_shared, out,
                                 S_(stream));
  prof_mark(FTM_K_COMBINE, S_(stream), true);
  if (e != cudaSuccess) return cuda_fail(e, "ftm_combine launch");
  return ok();
}

size_t ftm_workspace_bytes(const ftm_layer_desc* L, int32_t T_max) {
  if (check_desc(L) || T_max < 0) return 0;
  return carve(L, T_max, nullptr).total;
}

ftm_status ftm_moe_layer_forward(const ftm_layer_desc* L, const ftm_layer_weights* W, ftm_slot_cache* C,
                                 const void* x, int32_t T, void* out, void* workspace, size_t ws_bytes, void* stream,
                                 void* copy_stream) {
  ftm_status s = check_desc(L);
  if (s || (s = check_T(T))) return s;
  if (!W || !W->w_router) return fail(FTM_ERR_INVALID_ARG, "ftm_moe_layer_forward: NULL weights");
  if (T == 0) return ok();
  LayerWs w = carve(L, T, static_cast<uint8_t*>(workspace));
  if ((s = check_ws(workspace, ws_bytes, w.total, "ftm_moe_layer_forward"))) return s;
  if ((s = ftm_route(L, x, T, W->w_router, W->router_bias, w.ids, w.gates, stream))) return s;
  if (C && L->wdtype != FTM_F32) {
    // cache step with the hit experts' FFN overlapping the miss copies: the
    // pairs labelled against the residency before the lookup (misses as E + e)
    // and permuted over 2E groups, then the lookup (the host waits for it), the
    // copies, and the FFN in two launches (ffn_hits_then_misses)
    if ((s = check_cache(L, C, "ftm_moe_layer_forward"))) return s;
    cudaStream_t cs = S_(stream), ps = S_(copy_stream);
    const int P = T * L->k, E = L->E;
    cudaError_t e = launch_miss_relabel(w.ids, P, E, C->slot_of_expert + C->key_base, w.ids2, cs);
    if (e != cudaSuccess) return cuda_fail(e, "relabel launch");
    prof_mark(FTM_K_PERMUTE, cs, false);
    e = launch_permute(w.ids2, P, 2 * E, w.counts2, w.offsets2, w.perm, w.inv, w.perm_ws2, cs);
    prof_mark(FTM_K_PERMUTE, cs, true);
    if (e != cudaSuccess) return cuda_fail(e, "permute launch");
    int misses = 0;
    if ((s = cache_step(L, C, w.ids, P, C->step, w.lru_ws, cs, ps, nullptr, &misses))) return s;
    if ((s = ffn_hits_then_misses(L, W, C, x, T, w, misses, cs, ps))) return s;
    return ftm_combine(L, w.y, w.inv, w.gates, T, out, stream);
  }
  if ((s = ftm_permute(L, w.ids, T, w.counts, w.offsets, w.perm, w.inv, w.perm_ws,
                       permute_workspace_bytes(L->E, static_cast<int64_t>(T) * L->k), stream)))
    return s;
  const void* pool = W->slot_pool;
  const int32_t* soe = W->slot_of_expert;
  if (C) {   // fp32 layers: their SIMT FFN computes every row, so it runs once, after the copies
    if ((s = ftm_slot_lookup_update(L, C, w.ids, T, w.lru_ws, lru_workspace_bytes(L->E, L->S), stream, copy_stream)))
      return s;
    pool = C->slot_pool;
    soe = C->slot_of_expert + C->key_base;
  }
  if (!pool || !soe) return fail(FTM_ERR_INVALID_ARG, "ftm_moe_layer_forward: no slot pool / slot table");
  if ((s = ftm_expert_ffn(L, x, T, w.offsets, w.perm, soe, pool, W->shared_bank, W->act_scale, w.y, w.ffn_ws,
                          ffn_ws_bytes(L, T),
                          stream)))
    return s;  return ftm_combine(L, w.y, w.inv, w.gates, T, out, stream);
}

ftm_status ftm_moe_layers_forward(const ftm_layer_desc* L, int32_t n_layers, const ftm_layer_weights* W,
                                  ftm_slot_cache* C, const void* const* x, int32_t T, void* const* out,
                                  int32_t overlap, int32_t* overlapped, void* workspace, size_t ws_bytes,
                                  void* stream, void* copy_stream) {
  ftm_status s = check_desc(L);
  if (s || (s = check_T(T))) return s;
  if (n_layers < 1 || !W || !x || !out || !C) return fail(FTM_ERR_INVALID_ARG, "ftm_moe_layers_forward: NULL array");
  const int E = L->E;
  const int n_keys = C->n_keys ? C->n_keys : E;
  if (static_cast<int64_t>(n_layers) * E > n_keys)
    return fail(FTM_ERR_INVALID_ARG, "ftm_moe_layers_forward: %d layers of %d experts need %lld keys, the cache has %d",
                n_layers, E, static_cast<long long>(n_layers) * E, n_keys);
  for (int l = 0; l < n_layers; ++l)
    if (!W[l].w_router || (T > 0 && (!x[l] || !out[l])))
      return fail(FTM_ERR_INVALID_ARG, "ftm_moe_layers_forward: layer %d has a NULL router, input or output", l);
  LayerWs w = carve(L, T, static_cast<uint8_t*>(workspace));
  if ((s = check_ws(workspace, ws_bytes, w.total, "ftm_moe_layers_forward"))) return s;
  const bool on = overlap != 0 && L->S >= 2 * E;
  if (overlapped) *overlapped = on ? 1 : 0;
  g_warn[0] = 0;
  if (overlap && !on) {
    snprintf(g_warn, sizeof(g_warn),
             "WARNING Disabling MoE prefill overlap: the slot cache (%d slots) cannot hold two whole layers of "
             "experts (2 x %d); each layer's experts are copied before its compute",
             L->S, E);
    static std::atomic<bool> printed{false};
    if (!printed.exchange(true)) fprintf(stderr, "%s\n", g_warn);
  }
  if (T == 0) return ok();
  cudaStream_t cs = S_(stream);
  cudaEvent_t ev[5];
  for (int i = 0; i < 5; ++i)
    if (!(ev[i] = pipe_event(i))) return fail(FTM_ERR_CUDA, "could not create the pipeline events");
  cudaError_t e;
  if ((e = cudaEventRecord(ev[4], cs)) != cudaSuccess) return cuda_fail(e, "event record");
  const size_t lru_bytes = lru_workspace_bytes(E, L->S);
  // staging of layer l on the copy stream: a cache step for all its experts,
  // after `after` (the compute that reads the slots it may take); the copies
  // complete on ready[l % 2]
  auto stage = [&](int l, bool hold_previous, cudaEvent_t after) {
    return ftm_slot_stage_layer(L, C, l, hold_previous ? 1 : 0, after, w.lru_ws, lru_bytes, copy_stream, ev[l % 2]);
  };
  auto compute = [&](int l) -> ftm_status {
    cudaError_t ce;
    if ((ce = cudaStreamWaitEvent(cs, ev[l % 2], 0)) != cudaSuccess) return cuda_fail(ce, "ready event wait");
    ftm_layer_weights wl = W[l];
    wl.slot_pool = C->slot_pool;
    wl.slot_of_expert = C->slot_of_expert + static_cast<size_t>(l) * E;
    ftm_status st = ftm_moe_layer_forward(L, &wl, nullptr, x[l], T, out[l], workspace, ws_bytes, stream, nullptr);
    if (st) return st;
    if ((ce = cudaEventRecord(ev[2 + l % 2], cs)) != cudaSuccess) return cuda_fail(ce, "done event record");
    return FTM_OK;
  };
  if ((s = stage(0, false, ev[4]))) return s;
  for (int l = 0; l < n_layers; ++l) {
    if (!on && l > 0 && (s = stage(l, false, ev[2 + (l - 1) % 2]))) return s;
    if ((s = compute(l))) return s;
    // layer l+1's copies run while layer l computes; they may take the slots
    // of layer l-1 once its compute is over, never those of layer l
    if (on && l + 1 < n_layers && (s = stage(l + 1, true, l >= 1 ? ev[2 + (l - 1) % 2] : ev[4]))) return s;
  }
  return ok();
}

const char* ftm_last_warning(void) { return g_warn; }

int32_t ftm_hybrid_split(int32_t m, double pcie_gbs, double host_gbs) {
  if (m < 0 || !(pcie_gbs >= 0.0) || !(host_gbs >= 0.0) || !(pcie_gbs + host_gbs > 0.0) ||
      !std::isfinite(pcie_gbs + host_gbs))
    return -1;
  int q = static_cast<int>(floor(static_cast<double>(m) * pcie_gbs / (pcie_gbs + host_gbs) + 0.5));
  return q < 0 ? 0 : q > m ? m : q;
}

size_t ftm_hybrid_workspace_bytes(const ftm_layer_desc* L, int32_t T_max) {
  if (check_desc(L) || T_max < 0) return 0;
  return carve_hybrid(L, T_max, nullptr).total;
}

size_t ftm_hybrid_host_bytes(const ftm_layer_desc* L, int32_t T_max) {
  if (check_desc(L) || T_max < 0) return 0;
  return carve_host(L, T_max, nullptr).total;
}

size_t ftm_host_ffn_scratch_bytes(const ftm_layer_desc* L, int32_t n) {
  if (check_desc(L) || n < 0) return 0;
  return host_ffn_scratch_bytes(L, n);
}

ftm_status ftm_host_expert_ffn(const ftm_layer_desc* L, const void* bank, const void* x, int32_t n, void* y,
                               const float* act_scale, void* scratch, size_t scratch_bytes, int32_t threads) {
  ftm_status s = check_desc(L);
  if (s) return s;
  if (!host_ffn_supported(L->wdtype))
    return fail(FTM_ERR_UNSUPPORTED, "ftm_host_expert_ffn: no host FFN for wdtype %d", L->wdtype);
  if (n < 0) return fail(FTM_ERR_INVALID_ARG, "ftm_host_expert_ffn: n=%d is negative", n);
  if (n == 0) return ok();
  if (!bank || !x || !y || !scratch) return fail(FTM_ERR_INVALID_ARG, "ftm_host_expert_ffn: NULL pointer");
  if (scratch_bytes < host_ffn_scratch_bytes(L, n))
    return fail(FTM_ERR_INVALID_ARG, "ftm_host_expert_ffn: scratch %zu bytes < %zu needed", scratch_bytes,
                host_ffn_scratch_bytes(L, n));
  if (!aligned(bank, 16) || !aligned(scratch, 16))
    return fail(FTM_ERR_INVALID_ARG, "ftm_host_expert_ffn: bank / scratch not 16-byte aligned");
  ftm_bank_layout bl;
  bank_layout(L, &bl);
  const size_t row = static_cast<size_t>(L->d) * act_elt(L);
  std::vector<const uint8_t*> xr(n);
  std::vector<uint8_t*> yr(n);
  for (int r = 0; r < n; ++r) {
    xr[r] = static_cast<const uint8_t*>(x) + r * row;
    yr[r] = static_cast<uint8_t*>(y) + r * row;
  }
  HostGroup g{static_cast<const uint8_t*>(bank), n, xr.data(), yr.data()};
  host_ffn_groups(L, &bl, &g, 1, act_scale, static_cast<float*>(scratch), threads);
  return ok();
}

ftm_status ftm_moe_layer_forward_hybrid(const ftm_layer_desc* L, const ftm_layer_weights* W, ftm_slot_cache* C,
                                        ftm_hybrid* H, const void* x, int32_t T, void* out, void* workspace,
                                        size_t ws_bytes, void* stream, void* copy_stream) {
  static const char* who = "ftm_moe_layer_forward_hybrid";
  ftm_status s = check_desc(L);
  if (s || (s = check_T(T))) return s;
  if (!W || !W->w_router) return fail(FTM_ERR_INVALID_ARG, "%s: NULL weights", who);
  if (!H) return fail(FTM_ERR_INVALID_ARG, "%s: NULL split parameters", who);
  if (ftm_hybrid_split(0, H->pcie_gbs, H->host_gbs) < 0)
    return fail(FTM_ERR_INVALID_ARG, "%s: bandwidths must be finite, >= 0 and not both 0 (Bp=%g, Bh=%g)", who,
                H->pcie_gbs, H->host_gbs);
  if (!host_ffn_supported(L->wdtype)) return fail(FTM_ERR_UNSUPPORTED, "%s: no host FFN for wdtype %d", who, L->wdtype);
  // the fp32 GPU FFN (SIMT) maps every row to a group by searching the offsets,
  // so the host experts' rows cannot be left out of it: tensor-core dtypes only
  if (L->wdtype == FTM_F32)
    return fail(FTM_ERR_UNSUPPORTED, "%s: fp32 layers have no split (their GPU FFN computes every row)", who);
  if ((s = check_cache(L, C, who))) return s;
  if (T == 0) return ok();
  if (!x || !out) return fail(FTM_ERR_INVALID_ARG, "%s: NULL x / out", who);
  HybridWs hw = carve_hybrid(L, T, static_cast<uint8_t*>(workspace));
  if ((s = check_ws(workspace, ws_bytes, hw.total, who))) return s;
  HybridHost hh = carve_host(L, T, H->host_ws);
  if (!H->host_ws || H->host_ws_bytes < hh.total || !aligned(H->host_ws, 64))
    return fail(FTM_ERR_INVALID_ARG, "%s: host_ws needs %zu bytes, 64-byte aligned (have %zu)", who, hh.total,
                H->host_ws ? H->host_ws_bytes : static_cast<size_t>(0));
  cudaPointerAttributes pa;
  if (cudaPointerGetAttributes(&pa, H->host_ws) != cudaSuccess || pa.type != cudaMemoryTypeHost) {
    cudaGetLastError();
    return fail(FTM_ERR_INVALID_ARG, "%s: host_ws is not pinned host memory", who);
  }
  const int E = L->E, k = L->k, d = L->d, P = T * k;
  const size_t row = static_cast<size_t>(d) * act_elt(L);
  cudaStream_t cs = S_(stream), ps = S_(copy_stream);
  LayerWs& w = hw.w;
  cudaError_t e;
  if ((s = ftm_route(L, x, T, W->w_router, W->router_bias, w.ids, w.gates, stream))) return s;
  // the split (against the residency before this step), then the pairs by
  // expert with the host experts' pairs as one last group E
  if ((e = launch_hybrid_split(w.ids, P, E, C->slot_of_expert + C->key_base, H->pcie_gbs, H->host_gbs, w.ids2,
                               hw.skip, hw.split, cs)) != cudaSuccess)
    return cuda_fail(e, "split launch");
  prof_mark(FTM_K_PERMUTE, cs, false);
  e = launch_permute(w.ids2, P, 2 * E + 1, w.counts2, w.offsets2, w.perm, w.inv, w.perm_ws2, cs);
  prof_mark(FTM_K_PERMUTE, cs, true);
  if (e != cudaSuccess) return cuda_fail(e, "permute launch");
  // what the host needs, read back before the lookup's own read (same stream)
  const bool gscale = L->wdtype == FTM_NVFP4 && W->act_scale;   // the NVFP4 activation global scales
  struct { void* dst; const void* src; size_t n; } rd[6] = {
      {hh.split, hw.split, (4 + static_cast<size_t>(E)) * 4}, {hh.ids, w.ids, static_cast<size_t>(P) * 4},
      {hh.perm, w.perm, static_cast<size_t>(P) * 4}, {hh.offsets, w.offsets2, (2 * static_cast<size_t>(E) + 2) * 4},
      {hh.x, x, static_cast<size_t>(T) * row}, {hh.act, W->act_scale, gscale ? 2 * sizeof(float) : 0}};
  for (auto& c : rd)
    if (c.n && (e = cudaMemcpyAsync(c.dst, c.src, c.n, cudaMemcpyDeviceToHost, cs)) != cudaSuccess)
      return cuda_fail(e, "split read-back");
  // the cache step over the GPU's share: hits and the q copied misses (the
  // host waits here for the lookup, and with it for the reads above)
  int misses = 0;
  if ((s = cache_step(L, C, w.ids, P, C->step, w.lru_ws, cs, ps, nullptr, &misses, hw.skip))) return s;
  // the GPU's groups: hits while the copies run, the copied misses after them
  if ((s = ffn_hits_then_misses(L, W, C, x, T, w, misses, cs, ps))) return s;
  // meanwhile the host experts' pairs, positions offsets2[2E] .. P-1, on the host
  const int m = hh.split[0], Hn = hh.split[2], rows = hh.split[3], p0 = hh.offsets[2 * E];
  if (Hn < 0 || Hn > E || p0 < 0 || p0 + rows != P)
    return fail(FTM_ERR_CUDA, "%s: inconsistent split (H=%d, rows=%d, first host position %d, P=%d)", who, Hn, rows,
                p0, P);
  ftm_bank_layout bl;
  bank_layout(L, &bl);
  for (int i = 0; i < E; ++i) hh.gidx[i] = -1;
  for (int h = 0; h <= Hn; ++h) hh.gpos[h] = 0;
  for (int h = 0; h < Hn; ++h) {
    const int eh = hh.split[4 + h];
    if (eh < 0 || eh >= E || hh.gidx[eh] != -1)
      return fail(FTM_ERR_CUDA, "%s: host expert list entry %d (%d) out of range or repeated", who, h, eh);
    hh.gidx[eh] = h;
  }
  for (int p = p0; p < P; ++p) {
    const int q = hh.perm[p];
    const int g = (q >= 0 && q < P && hh.ids[q] >= 0 && hh.ids[q] < E) ? hh.gidx[hh.ids[q]] : -1;
    if (g < 0) return fail(FTM_ERR_CUDA, "%s: position %d of the host group maps to no host expert", who, p);
    hh.gpos[g + 1] += 1;
  }
  for (int h = 0; h < Hn; ++h) hh.gpos[h + 1] += hh.gpos[h];
  for (int h = 0; h < Hn; ++h) {
    const int key = C->key_base + hh.split[4 + h];
    hh.groups[h] = HostGroup{static_cast<const uint8_t*>(C->host_pool) + static_cast<size_t>(key) * bl.bank_bytes, 0,
                             hh.xrow + hh.gpos[h], hh.yrow + hh.gpos[h]};
  }
  for (int p = p0; p < P; ++p) {   // ascending positions: each group's rows in ascending pair order
    const int q = hh.perm[p], g = hh.gidx[hh.ids[q]];
    HostGroup& G = hh.groups[g];
    hh.xrow[hh.gpos[g] + G.n] = hh.x + static_cast<size_t>(q / k) * row;
    hh.yrow[hh.gpos[g] + G.n] = hh.y + static_cast<size_t>(p - p0) * row;
    G.n += 1;
  }
  const auto t0 = std::chrono::steady_clock::now();
  host_ffn_groups(L, &bl, hh.groups, Hn, gscale ? hh.act : nullptr, hh.scratch, H->threads);
  const auto t1 = std::chrono::steady_clock::now();
  if (rows > 0 && (e = cudaMemcpyAsync(static_cast<uint8_t*>(w.y) + static_cast<size_t>(p0) * row, hh.y,
                                       static_cast<size_t>(rows) * row, cudaMemcpyHostToDevice, cs)) != cudaSuccess)
    return cuda_fail(e, "host rows copy");
  H->last_misses = m;
  H->last_host = Hn;
  H->last_host_rows = rows;
  H->last_host_ms = std::chrono::duration<double, std::milli>(t1 - t0).count();
  return ftm_combine(L, w.y, w.inv, w.gates, T, out, stream);
}

}  // extern "C"
