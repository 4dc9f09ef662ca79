/*
 * ftm.h -- C ABI of a B200 (sm_100a) routed Mixture-of-Experts layer over a
 * slot-indexed expert cache.
 *
 * What the layer computes (FreeToken pages):
 *  - chenxutan.com FreeToken article, section "why the bottleneck is bandwidth,
 *    not capacity": every token activates a few routed experts; the full expert
 *    pool may live in host memory and experts are pulled into VRAM on demand.
 *  - same article, section "choosing among the five MoE backends", `offload`:
 *    experts in host RAM, LRU slots in VRAM, misses copied over PCIe.
 *  - claypier.com "FreeToken MoE edge runtime", first section: a global LRU
 *    cache evicts the expert weights unused for the longest time.
 *  - pomoai.com FreeToken hub, checkpoint list: BF16, FP8 and NVFP4 weights.
 * The pages print no formula; the layer is the plain top-k routed SwiGLU MoE:
 *   logits = x Wr^T + b;  ids = top-k(logits);  g = softmax(logits) restricted
 *   to the k picks and renormalised;  h = silu(x Wg_e^T) * (x Wu_e^T);
 *   y = h Wd_e^T;  out[t] = sum_j g[t][j] y[t,j]  (+ shared expert FFN(x[t])).
 *
 * Conventions for every entry point:
 *  - Pointers marked "device" are CUDA device pointers, "host" are host
 *    pointers.  The caller owns every buffer; the library never allocates device
 *    or host memory and keeps no per-call state beyond a thread-local error
 *    string and one cached CUDA event per thread for the miss-copy ordering.
 *    The one exception is the host FFN of the miss split
 *    (ftm_moe_layer_forward_hybrid, ftm_host_expert_ffn): it allocates small
 *    host buffers per call (row tables, and per work item the partial sums of
 *    its rows and one weight row's scales), and keeps a pool of host threads
 *    from its first call to process exit.
 *  - `stream` arguments are cudaStream_t values passed as void* (NULL = the
 *    legacy default stream).  Work is enqueued asynchronously; the entry
 *    points that synchronise the host are the cache steps
 *    (ftm_slot_lookup_update, ftm_slot_stage_layer, ftm_moe_layers_forward,
 *    ftm_moe_layer_forward with a cache, and ftm_moe_layer_forward_hybrid):
 *    each must read its miss list before it can issue the copies, and waits
 *    for that kernel alone.  ftm_moe_layer_forward_hybrid and
 *    ftm_host_expert_ffn also compute on the calling thread (and the library's
 *    host threads) before they return.
 *  - Arguments are validated before anything is enqueued; on error nothing is
 *    launched, the function returns a non-zero ftm_status and ftm_last_error()
 *    describes it.  No C++ exception crosses this boundary.
 *  - Device-side faults of the library's own kernels (a bounded wait that timed
 *    out) are recorded in a device status word read by ftm_device_status().
 *
 * Activation dtype: FTM_F32 layers take fp32 x, fp32 router weights and write
 * fp32 out; every other layer takes bf16 x (raw bits, row-major [T][d]), bf16
 * router weights and writes bf16 out.  Router bias and gates are fp32.
 */
#ifndef FTM_H_
#define FTM_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum ftm_status {
  FTM_OK = 0,
  FTM_ERR_INVALID_ARG = 1,   /* a size, pointer, alignment or layout is out of contract */
  FTM_ERR_UNSUPPORTED = 2,   /* valid layer, but no kernel for it (dtype/shape) */
  FTM_ERR_CAPACITY = 3,      /* more distinct experts in one step than cache slots */
  FTM_ERR_CUDA = 4           /* a CUDA call failed (message in ftm_last_error) */
} ftm_status;

typedef enum ftm_wdtype {
  FTM_F32 = 0,               /* fp32 expert weights */
  FTM_BF16 = 1,              /* bf16 expert weights */
  FTM_FP8_E4M3_B128 = 2,     /* e4m3 weights, one fp32 scale per 128x128 block */
  FTM_NVFP4 = 3,             /* e2m1 weights, one e4m3 scale per 16 elements + fp32 per-tensor scale */
  FTM_MXFP4 = 4              /* e2m1 weights, one E8M0 scale (power of two) per 32 elements (OCP MX) */
} ftm_wdtype;

/* One layer's shape.  Limits: d, I multiples of 128 (of 256 for NVFP4 and MXFP4);
 * 1 <= k <= min(E, 16); 1 <= E <= 512; 1 <= S. */
typedef struct ftm_layer_desc {
  int32_t d;            /* hidden size */
  int32_t E;            /* routed experts */
  int32_t k;            /* picks per token */
  int32_t I;            /* SwiGLU intermediate size */
  int32_t has_shared;   /* 1: one always-on shared expert (gate weight 1) */
  int32_t S;            /* expert slots in the HBM pool */
  int32_t wdtype;       /* ftm_wdtype */
  int32_t reserved;     /* must be 0 */
} ftm_layer_desc;

/* Layout of one expert "bank": the contiguous byte range holding all of one
 * expert's weights, so a cache miss is a single copy.  All offsets are from
 * the bank start and 256-byte aligned; bank_bytes is a multiple of 256.
 *   w_gu: [2I][d] row-major, rows 0..I-1 = gate projection, I..2I-1 = up
 *         (f32 / bf16 / e4m3 elements; NVFP4: [2I][d/2] bytes, two codes per
 *         byte, element 2j in the low nibble)
 *   w_d : [d][I] row-major (same element rules)
 *   s_gu: FP8: fp32 [2I/128][d/128]; NVFP4: the 2I x d/16 e4m3 scales in chunks (below),
 *         rows taken in paired order: gate rows 64b..64b+63 then up rows
 *         64b..64b+63 for b = 0..I/64-1 (chunk row block rb = b)
 *   s_d : FP8: fp32 [d/128][I/128];  NVFP4: the d x I/16 e4m3 scales in chunks
 *   s_t : NVFP4: fp32[4] = {gate, up, down, 0} per-tensor scales; else empty
 *   MXFP4: w_gu, w_d packed as NVFP4; s_gu: the 2I x d/32 E8M0 codes in chunks
 *          (rows in the paired order above), s_d: the d x I/32 codes in chunks;
 *          no s_t.
 * Scale chunks (the layout the block-scaled MMA reads): one 512-byte chunk per
 * (128-row block rb, column block kb of four scale groups: 64 columns for
 * NVFP4's 16-groups, 128 for MXFP4's 32-groups), ordered [rb][kb]; in a chunk
 * the scale of local row r (0..127) for its j-th group of the block (0..3) is
 * byte (r % 32) * 16 + (r / 32) * 4 + j. */
typedef struct ftm_bank_layout {
  uint64_t bank_bytes;
  uint64_t w_gu_off, w_gu_bytes;
  uint64_t w_d_off, w_d_bytes;
  uint64_t s_gu_off, s_gu_bytes;
  uint64_t s_d_off, s_d_bytes;
  uint64_t s_t_off, s_t_bytes;
} ftm_bank_layout;

ftm_status ftm_get_bank_layout(const ftm_layer_desc* L, ftm_bank_layout* out);

/* Router + gating (a1, a2).  chenxutan.com FreeToken article, section "why
 * the bottleneck is bandwidth, not capacity": each token activates only a few
 * of the routed experts (6 of them for the 284B model), picked per token by
 * the router; the gate reading (softmax over all E logits, then renormalised
 * over the k picks) is the plain top-k routed MoE.
 *   x        device [T][d] (fp32 or bf16, see above)
 *   w_router device [E][d] row-major (same dtype as x)
 *   bias     device fp32 [E] added to every logit, or NULL
 *   topk_ids device int32 [T][k]: picks in descending logit order, equal
 *            logits to the lower expert id
 *   topk_w   device fp32 [T][k]: softmax over all E logits, renormalised over
 *            the k picks (= softmax of the k picked logits)
 * Logits are accumulated in fp32.  T = 0 is a no-op. */
ftm_status ftm_route(const ftm_layer_desc* L, const void* x, int32_t T, const void* w_router,
                     const float* bias, int32_t* topk_ids, float* topk_w, void* stream);

/* Permutation of the P = T*k (token, pick) pairs by expert (a3).  chenxutan.com
 * FreeToken article, same section: in prefill a large batch routes to nearly
 * every expert at once, so the batch's pairs are grouped per expert and each
 * expert's weights are read once for all of its rows (the grouping a fused
 * MoE kernel performs; pomoai.com FreeToken hub, install paragraph, [accel]
 * fused kernels).
 *   counts  device int32 [E]     pairs per expert
 *   offsets device int32 [E+1]   exclusive prefix sum, offsets[E] = P
 *   perm    device int32 [P]     perm[pos] = q = t*k + j, stable: pairs of one
 *                                expert appear in ascending q
 *   inv     device int32 [P]     inv[q] = pos
 *   workspace device, >= ftm_permute_workspace_bytes(L, T) bytes, 256-aligned
 * Deterministic: identical results run to run.  Ids are range-checked on the
 * device: a pair whose id is outside [0, E) is not counted or placed, its
 * inv entry is -1, perm positions from offsets[E] to P-1 hold -1, and the
 * device status word (ftm_device_status) reads 2; no out-of-range access is
 * made. */
ftm_status ftm_permute(const ftm_layer_desc* L, const int32_t* topk_ids, int32_t T, int32_t* counts,
                       int32_t* offsets, int32_t* perm, int32_t* inv, void* workspace, size_t ws_bytes,
                       void* stream);
size_t ftm_permute_workspace_bytes(const ftm_layer_desc* L, int32_t T);

/* The LRU slot cache (a4).  State lives in caller-owned device arrays:
 *   slot_of_expert [n_keys] (-1: not resident), expert_of_slot [S] (the key
 *   held, -1: empty), last_use [S] int64 (-1: never).
 * A step s requests the distinct expert ids routed in that step (the shared
 * expert is not cached), as keys key_base + id.  Hits set last_use = s.
 * Misses, in ascending key, each take the slot with the smallest last_use
 * among slots not used in step s (ties: lowest slot index); the slot's
 * previous key is unmapped and the bank is copied host_pool[key] ->
 * slot_pool[slot]. */
typedef struct ftm_slot_cache {
  int32_t* slot_of_expert;      /* device [E] */
  int32_t* expert_of_slot;      /* device [S] */
  int64_t* last_use;            /* device [S] */
  int64_t step;                 /* host: index s of the next step; +1 per successful update */
  void* slot_pool;              /* device: S banks of bank_bytes, slot j at j*bank_bytes */
  const void* host_pool;        /* host, pinned (cudaHostAlloc/cudaHostRegister): E banks */
  int32_t* host_scratch;        /* host, pinned, >= ftm_slot_host_scratch_ints(L) int32 */
  int32_t last_distinct;        /* out: distinct experts requested by the last step */
  int32_t last_hits;            /* out: of which resident */
  int32_t last_misses;          /* out: of which copied in */
  int32_t fail_before_copy;     /* test hook: n >= 1 makes the next update with at least n
                                   misses fail as if its n-th copy could not be issued
                                   (copies 1..n-1 are issued); see the rollback rule of
                                   ftm_slot_lookup_update.  Cleared when it fires. */
  int32_t n_keys;               /* entries of slot_of_expert and banks of host_pool; 0 means E.
                                   A cache shared by several layers of E experts each (the
                                   pages' global LRU expert cache) has n_layers * E keys,
                                   layer l's expert e being key l*E + e */
  int32_t key_base;             /* first key of the layer a lookup serves (l*E; 0 for a cache
                                   of one layer); ftm_slot_stage_layer sets it */
} ftm_slot_cache;

size_t ftm_slot_host_scratch_ints(const ftm_layer_desc* L);
size_t ftm_slot_workspace_bytes(const ftm_layer_desc* L);

/* One cache step.  Runs the lookup/update kernel on `compute_stream`,
 * synchronises that stream to read the miss list (the one host sync of the
 * path), issues one cudaMemcpyAsync per miss on `copy_stream`, and makes
 * `compute_stream` wait for the copies, so work enqueued afterwards on
 * `compute_stream` sees the new slots.  Returns
 *   FTM_ERR_CAPACITY (state unchanged) when more than S distinct experts are
 *     requested;
 *   FTM_ERR_INVALID_ARG (state unchanged) when topk_ids holds an id outside
 *     [0, E) (found on the device, which also sets the device status word to 2);
 *   FTM_ERR_CUDA when a copy cannot be issued: the state is rolled back to
 *     before the call, except that every slot whose copy was already issued
 *     (it may hold part of the new bank) is left empty (expert_of_slot -1,
 *     last_use -1) with its previous expert unmapped, so no partly
 *     overwritten bank is ever taken for a hit.
 *   workspace device, >= ftm_slot_workspace_bytes(L) bytes */
ftm_status ftm_slot_lookup_update(const ftm_layer_desc* L, ftm_slot_cache* C, const int32_t* topk_ids,
                                  int32_t T, void* workspace, size_t ws_bytes, void* compute_stream,
                                  void* copy_stream);

/* Whole-layer staging (prefill double buffering).  pomoai.com FreeToken hub,
 * prefill-overlap paragraph: in prefill every MoE layer moves its experts from
 * host memory to the GPU; with overlap, layer n+1's copies run while layer n
 * computes, so a layer costs about max(copy, compute) instead of their sum,
 * which needs a cache that holds two whole layers (refft.com FreeToken guide:
 * full-layer double-buffered prefill over a global LRU expert cache).
 * One cache step that makes all E experts of `layer` resident (keys
 * layer*E .. layer*E+E-1; C->key_base is set to layer*E).  Everything runs on
 * `copy_stream`: after `after_event` (cudaEvent_t or NULL) the lookup/update
 * kernel, the miss-list read (the host waits for this kernel), then one copy
 * per miss; `ready_event` (cudaEvent_t or NULL) is recorded after the copies,
 * so compute that waits for it sees the layer in its slots.  hold_previous =
 * 1: the slots used by the previous step are kept (their layer may still be
 * computing): misses take only slots with last_use < step - 1, and more
 * misses than such slots gives FTM_ERR_CAPACITY (state unchanged).  The step
 * rewrites the entries of the keys it evicts, so `after_event` must mark the
 * end of every compute that reads those keys' slots.  Other errors as
 * ftm_slot_lookup_update.
 *   workspace device, >= ftm_slot_workspace_bytes(L) bytes */
ftm_status ftm_slot_stage_layer(const ftm_layer_desc* L, ftm_slot_cache* C, int32_t layer, int32_t hold_previous,
                                void* after_event, void* workspace, size_t ws_bytes, void* copy_stream,
                                void* ready_event);

/* Elastic slot-pool resize: move the cache to S_new slots at run time without
 * reloading weights from the host (pomoai.com FreeToken hub, two-level expert
 * memory: the expert cache's VRAM share changes while the engine runs;
 * freelamp.com FreeToken article, section 2.3 "elastic memory management",
 * `ftctl cache --moe <slots>`).  The pages give no rule for which experts stay;
 * this library keeps the min(S_new, resident) most recently used resident
 * experts (largest last_use first, ties to the lower old slot), compacted into
 * slots 0.. in their old slot order with their last_use, and evicts the rest.
 *   L          the layer with the OLD slot count (L->S = S_old)
 *   C          the current cache (read: state arrays and slot_pool)
 *   S_new      1 <= S_new <= 4096
 *   C_new      caller-owned new state: slot_of_expert [E], expert_of_slot
 *              [S_new], last_use [S_new] (device) and slot_pool (S_new banks),
 *              none overlapping C's; host_pool / host_scratch may be C's.  On
 *              success C_new->step = C->step and its counters are zeroed.
 *   workspace  device, >= ftm_slot_workspace_bytes(L) bytes, 256-aligned
 * Enqueues on `stream`, with no host synchronisation, one kernel that writes
 * the new state and the move list and one that copies the kept banks
 * device-to-device.  Afterwards use C_new with a layer desc whose S = S_new;
 * C's arrays and pool may be released once the stream has passed this call. */
ftm_status ftm_slot_resize(const ftm_layer_desc* L, const ftm_slot_cache* C, int32_t S_new, ftm_slot_cache* C_new,
                           void* workspace, size_t ws_bytes, void* stream);

/* Grouped SwiGLU expert FFN (a5, a6, a7).  chenxutan.com FreeToken article,
 * section "choosing among the five MoE backends": `fused` (every expert resident
 * in VRAM) and `offload` (experts computed on the GPU from LRU slots in VRAM);
 * pomoai.com FreeToken hub, checkpoint list: BF16, FP8 and NVFP4 expert weights.
 * The SwiGLU form and the shared expert (weight 1, configs with one) are the
 * plain reading of the DeepSeek/GLM/Qwen MoE layers the pages run.
 *   x              device [T][d] activations (token order)
 *   offsets, perm  from ftm_permute
 *   slot_of_expert device int32 [E]: bank of expert e is slot_pool[slot_of_expert[e]]
 *   slot_pool      device, S banks (layout from ftm_get_bank_layout)
 *   shared_bank    device, one bank, required iff L->has_shared
 *   act_scale      device fp32[2] or NULL (= {1, 1}); NVFP4 layers only (ignored
 *                  otherwise): the per-tensor global scales of the activations,
 *                  gx for x and gh for the SwiGLU output h, static values that
 *                  come with an NVFP4 checkpoint's calibration.  An activation
 *                  v is quantised per 16 consecutive elements as
 *                  s16 = e4m3(amax / (6 g)), code = e2m1(v / (s16 g)).  With
 *                  g = 1 a group whose amax / 6 is below 2^-10 (half the smallest
 *                  e4m3 subnormal) quantises to zero, so small activations need
 *                  a g near amax / (6 * 448) of their tensor.
 *   y              device [P + (has_shared ? T : 0)][d]: row pos = the FFN output of
 *                  pair perm[pos] (unweighted); rows P..P+T-1 = shared expert of token t
 *                  (bf16; fp32 for FTM_F32)
 *   workspace      device, >= ftm_ffn_workspace_bytes(L, T) bytes, 256-aligned
 * Every expert that has pairs must be resident (slot_of_expert[e] in [0,S)). */
ftm_status ftm_expert_ffn(const ftm_layer_desc* L, const void* x, int32_t T, const int32_t* offsets,
                          const int32_t* perm, const int32_t* slot_of_expert, const void* slot_pool,
                          const void* shared_bank, const float* act_scale, void* y, void* workspace,
                          size_t ws_bytes, void* stream);
size_t ftm_ffn_workspace_bytes(const ftm_layer_desc* L, int32_t T);

/* Weighted un-permute and combine (a8).  chenxutan.com FreeToken article,
 * section "why the bottleneck is bandwidth, not capacity": a token's output is
 * made from the few routed experts it activated; the gate-weighted sum (plus
 * the shared expert) is the plain reading:
 *   out[t] = sum_{j=0..k-1 ascending} topk_w[t][j] * y[inv[t*k+j]]  (+ y[P+t] if has_shared),
 * accumulated in fp32.  y, inv, topk_w device; out device [T][d].  A pair
 * whose inv entry is outside [0, P) (one ftm_permute skipped) is left out of
 * the sum and sets the device status word to 2. */
ftm_status ftm_combine(const ftm_layer_desc* L, const void* y, const int32_t* inv, const float* topk_w,
                       int32_t T, void* out, void* stream);

/* Weights of one layer for ftm_moe_layer_forward. */
typedef struct ftm_layer_weights {
  const void* w_router;            /* device [E][d] */
  const float* router_bias;        /* device [E] or NULL */
  const void* slot_pool;           /* device, S banks (resident layers; ignored with a cache) */
  const int32_t* slot_of_expert;   /* device [E] (resident layers; ignored with a cache) */
  const void* shared_bank;         /* device, one bank, or NULL */
  const float* act_scale;          /* device fp32[2] or NULL: NVFP4 activation global scales (see
                                      ftm_expert_ffn) */
} ftm_layer_weights;

/* The whole layer: route -> permute -> [cache step] -> expert FFN -> combine.
 * chenxutan.com FreeToken article, section "choosing among the five MoE
 * backends": `fused` (C = NULL, every expert resident) and `offload` (C set:
 * experts in host RAM, LRU slots in VRAM, misses copied over PCIe).
 *   C          NULL for a resident layer (every expert in W->slot_pool at
 *              W->slot_of_expert[e]); otherwise the LRU cache (its slot_pool and
 *              slot_of_expert are used, and the call synchronises once, see
 *              ftm_slot_lookup_update).  With a cache (bf16 / FP8 / FP4
 *              layers) the expert FFN runs in two launches: the experts that
 *              were resident (and the shared expert) right after the lookup,
 *              while the misses are copied on copy_stream, then the copied
 *              misses once their copies are done; fp32 layers run one FFN
 *              after the copies
 *   x, out     device [T][d]
 *   workspace  device, >= ftm_workspace_bytes(L, T) bytes, 256-aligned
 *   copy_stream  stream for the miss copies (only used with a cache) */
ftm_status ftm_moe_layer_forward(const ftm_layer_desc* L, const ftm_layer_weights* W, ftm_slot_cache* C,
                                 const void* x, int32_t T, void* out, void* workspace, size_t ws_bytes,
                                 void* stream, void* copy_stream);
size_t ftm_workspace_bytes(const ftm_layer_desc* L, int32_t T_max);

/* Several MoE layers in sequence over one slot cache shared by all of them,
 * with full-layer double buffering (see ftm_slot_stage_layer for the pages'
 * passages).  Layer l's experts are staged into the cache (one cache step per
 * layer, all E experts), then layer l runs as a resident layer on the staged
 * slots: route, permute, expert FFN, combine.
 *   L          one layer's shape (every layer has it); L->S = slots of C
 *   n_layers   >= 1; C->n_keys must be >= n_layers * E, host_pool holding
 *              layer l's expert banks at keys l*E ..
 *   W          host array [n_layers]: w_router, router_bias, shared_bank of
 *              each layer (slot_pool and slot_of_expert are ignored)
 *   x, out     host arrays [n_layers] of device pointers: layer l reads x[l]
 *              ([T][d]) and writes out[l]; x[l+1] may be out[l]
 *   overlap    1: stage layer l+1 on copy_stream while layer l computes on
 *              `stream` (the staging holds layer l's slots back, and may take
 *              layer l-1's once its compute is over); needs S >= 2E, else the
 *              overlap is switched off with a warning (ftm_last_warning, and
 *              once per process on stderr).  0: stage each layer after the
 *              previous layer's compute, then compute it.
 *   overlapped host, nullable: set to 1 when the overlap ran
 *   workspace  device, >= ftm_workspace_bytes(L, T) bytes, 256-aligned
 * The host waits once per layer for a staging kernel (its miss list).
 * C->step advances by n_layers. */
ftm_status ftm_moe_layers_forward(const ftm_layer_desc* L, int32_t n_layers, const ftm_layer_weights* W,
                                  ftm_slot_cache* C, const void* const* x, int32_t T, void* const* out,
                                  int32_t overlap, int32_t* overlapped, void* workspace, size_t ws_bytes,
                                  void* stream, void* copy_stream);

/* Bandwidth-adaptive miss split (the pages' q* policy: freelamp.com FreeToken
 * article, section 2.1 "bandwidth-adaptive execution"; chenxutan.com FreeToken
 * article, "choosing among the five MoE backends", `hybrid`, and the bandwidth
 * calibration `ft bench bw` that feeds it).  Of the m experts a step requests
 * that are not in the cache, q are copied over PCIe and computed on the GPU,
 * the other m - q are computed on the host CPU from host memory, both sides at
 * once.  With Bp the PCIe bandwidth and Bh the host FFN's (expert bytes per
 * second each side gets through), the two finish together when
 * q / Bp = (m - q) / Bh:  q = m Bp / (Bp + Bh), rounded to the nearest integer
 * (halves up), computed in fp64 as floor(m * Bp / (Bp + Bh) + 0.5).  (One page
 * prints q* = m Bp / Bh, which does not balance the two sides; this library
 * takes the balanced form the same pages describe in words.)  Bh = 0 gives
 * q = m (every miss over PCIe, the plain cache step); Bp = 0 gives q = 0.
 * Returns q, or -1 when m < 0 or the bandwidths are negative, not finite or
 * both 0.  Host-only, no CUDA call. */
int32_t ftm_hybrid_split(int32_t m, double pcie_gbs, double host_gbs);

/* Parameters, host buffer and per-call results of ftm_moe_layer_forward_hybrid. */
typedef struct ftm_hybrid {
  double pcie_gbs;          /* Bp >= 0 (GB/s of bank copies host -> GPU) */
  double host_gbs;          /* Bh >= 0 (GB/s of expert banks the host FFN gets through); Bp + Bh > 0 */
  int32_t threads;          /* host FFN threads (0: every hardware thread) */
  int32_t last_misses;      /* out: m, requested experts not in the cache */
  int32_t last_host;        /* out: m - q, of which computed on the host */
  int32_t last_host_rows;   /* out: (token, pick) pairs computed on the host */
  double last_host_ms;      /* out: wall time of the host FFN */
  void* host_ws;            /* host, pinned, 64-byte aligned, >= ftm_hybrid_host_bytes(L, T) bytes */
  size_t host_ws_bytes;
} ftm_hybrid;

/* Device workspace of ftm_moe_layer_forward_hybrid: ftm_workspace_bytes(L, T_max)
 * plus a few int32 arrays of P = T_max * k and E + 2 entries.  Pinned host
 * workspace: the read-back ids, permutation and activations, the host rows'
 * outputs, and the host FFN's fp32 scratch for up to P rows, about
 * P * (d + I) * 4 + (T_max + P) * d * 2 bytes: the split is meant for decode-sized
 * batches. */
size_t ftm_hybrid_workspace_bytes(const ftm_layer_desc* L, int32_t T_max);
size_t ftm_hybrid_host_bytes(const ftm_layer_desc* L, int32_t T_max);

/* The layer with a cache step split by ftm_hybrid_split (bf16, FP8, NVFP4 and
 * MXFP4 layers; fp32 layers return FTM_ERR_UNSUPPORTED, since their SIMT GPU FFN
 * computes every row and cannot leave the host's rows out).  Sequence:
 *  1. route on `stream`;
 *  2. one kernel counts each expert's pairs, finds the misses (against the
 *     cache state before this step), sets q, and gives the host the m - q
 *     misses with the fewest pairs (ties: the lower expert id); their pairs are
 *     relabelled E;
 *  3. the pairs are permuted over E + 1 groups (group E = the host's pairs, in
 *     ascending pair order, at positions P - rows .. P - 1);
 *  4. the cache step of ftm_slot_lookup_update over the remaining requests
 *     (hits and the q copied misses): the LRU state changes exactly as a plain
 *     step whose topk_ids held only those experts; the host experts are not
 *     inserted and their last use is not updated.  The host waits here once;
 *  5. the GPU expert FFN of every group but E, after the copies;
 *  6. meanwhile the host computes group E's rows from the banks in
 *     C->host_pool (the same FFN with the GPU path's activation quantisation,
 *     fp32 accumulation; ftm_host_expert_ffn; the NVFP4 global scales are read
 *     from W->act_scale) on H->threads threads, then copies them into place on
 *     `stream`;
 *  7. combine, as ftm_moe_layer_forward.
 * Output rows agree with ftm_moe_layer_forward within the dtype's tolerance
 * (bit-identical when m - q = 0).  Arguments as ftm_moe_layer_forward with a
 * cache, plus H; workspace >= ftm_hybrid_workspace_bytes(L, T).  H->host_ws
 * may be reused once `stream` has passed the call.  Errors as
 * ftm_slot_lookup_update (state unchanged on capacity / id errors). */
ftm_status ftm_moe_layer_forward_hybrid(const ftm_layer_desc* L, const ftm_layer_weights* W, ftm_slot_cache* C,
                                        ftm_hybrid* H, const void* x, int32_t T, void* out, void* workspace,
                                        size_t ws_bytes, void* stream, void* copy_stream);

/* The host half of the split on its own: one expert's SwiGLU FFN on the CPU.
 *   bank      host, one expert bank (layout from ftm_get_bank_layout), 16-byte aligned
 *   x, y      host [n][d] (bf16, fp32 for FTM_F32), row-major
 *   act_scale host fp32[2] = {gx, gh}, the NVFP4 activation global scales (see
 *             ftm_expert_ffn), or NULL (1, 1); ignored by other dtypes
 *   scratch   host, >= ftm_host_ffn_scratch_bytes(L, n) bytes, 16-byte aligned
 *   threads   0: every hardware thread
 * Every weight dtype, with the GPU path's activation quantisation of x and of
 * the SwiGLU output: FP8 per 128 elements (amax / 448, E4M3 nearest even),
 * NVFP4 per 16 (e4m3(amax / (6 g)) scales, E2M1 codes), MXFP4 per 32 (E8M0
 * scales); fp32 accumulation, outputs rounded to bf16 (fp32 for FTM_F32).  No
 * CUDA call: runs without a GPU. */
size_t ftm_host_ffn_scratch_bytes(const ftm_layer_desc* L, int32_t n);
ftm_status ftm_host_expert_ffn(const ftm_layer_desc* L, const void* bank, const void* x, int32_t n, void* y,
                               const float* act_scale, void* scratch, size_t scratch_bytes, int32_t threads);

/* Thread-local warning of the last ftm_moe_layers_forward call ("" if none). */
const char* ftm_last_warning(void);

/* The whole resident layer, for callers that cannot allocate device memory
 * (code running while a CUDA graph is being captured, allocator-free embedded
 * runtimes, engines whose memory is reserved up front).  The pages have no
 * counterpart of this entry point.
 *   Same computation and arguments as ftm_moe_layer_forward with C = NULL, but
 *   no workspace argument: the scratch is a static 16 MiB device array inside
 *   the library, which every GPU that loads the library keeps until exit.
 *   Calls whose ftm_workspace_bytes(L, T) exceeds 16 MiB are rejected with
 *   FTM_ERR_INVALID_ARG (decode-sized batches fit; large prefills do not).
 *   The first call on a device looks up the array's device address (with that
 *   device current); make that first call before any stream capture.
 *   All calls share the one array: calls that overlap on the GPU (on different
 *   streams, or from different host threads, without ordering) race on it.
 *   Nothing is allocated: no cudaMalloc/cudaFree and no allocating library call. */
ftm_status ftm_moe_layer_forward_noalloc(const ftm_layer_desc* L, const ftm_layer_weights* W, const void* x,
                                         int32_t T, void* out, void* stream);

/* Measurement hook.  Kernel ids of the path, in launch order. */
typedef enum ftm_kernel_id {
  FTM_K_ROUTE = 0,      /* router + gating */
  FTM_K_PERMUTE = 1,    /* histogram / scan / scatter (all launches of one call) */
  FTM_K_LRU = 2,        /* slot lookup/update */
  FTM_K_GATHER = 3,     /* X_p gather (+ activation quantisation) */
  FTM_K_GEMM1 = 4,      /* grouped gate/up GEMM + SwiGLU */
  FTM_K_GEMM2 = 5,      /* grouped down GEMM */
  FTM_K_COMBINE = 6,    /* weighted un-permute + shared expert */
  FTM_K_COUNT = 7
} ftm_kernel_id;

/* While set on the calling thread, every launch of kernel `which` is bracketed
 * by cudaEventRecord(start) / cudaEventRecord(stop) on the stream it is
 * launched on (events are cudaEvent_t passed as void*, created by the caller
 * with timing enabled).  NULL events clear the hook.  Nothing else changes.
 * In a layer call with a cache, the gather and GEMM events bracket the first
 * of the two FFN launches (the resident experts' and the shared expert's). */
ftm_status ftm_set_profile_events(int32_t which, void* start_event, void* stop_event);

/* Number of kernel launches the library has enqueued in this process so far
 * (all threads and devices; launches recorded into a CUDA graph under stream
 * capture count once, at capture).  A measurement hook: the difference across
 * one eager layer call is the number of kernels that call launches. */
uint64_t ftm_kernel_launches(void);

/* Thread-local description of the last error returned on this thread. */
const char* ftm_last_error(void);

/* Reads (and if reset != 0 clears) the device status word.  Synchronises the
 * device.  0 = no fault; 1 = a bounded wait of a tensor-core kernel gave up
 * (the kernel unwound and freed its tensor memory); 2 = a kernel met an index
 * outside its range (an expert id outside [0, E)) and skipped the access. */
int32_t ftm_device_status(int32_t reset);

/* Failure-detection self-test of the bounded waits: launches one block of one
 * thread that waits on a shared-memory mbarrier nothing ever completes, with
 * the wait every tensor-core kernel uses.  The wait gives up after its time
 * limit (about 2 s), sets the device status word to 1 and the kernel returns,
 * so the context stays usable.  Synchronises `stream`, then writes the status
 * word to *observed (1 expected) and clears it.  Allocates nothing; returns
 * FTM_ERR_CUDA if the launch or the synchronisation failed.  Not part of the
 * layer path: a test of the mechanism the layer kernels rely on. */
ftm_status ftm_selftest_bounded_wait(int32_t* observed, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* FTM_H_ */
