/*
 * ORACLE -- test infrastructure only.
 *
 * A plain, slow, obviously-correct CPU restatement of one routed
 * Mixture-of-Experts layer over a slot-indexed expert cache.  Only the tests,
 * the smoke check and the CPU-baseline leg of the benchmark load this file; the
 * product path never does, and it shares no code with the CUDA kernels.
 *
 * Sources (FreeToken web pages):
 *  - chenxutan.com FreeToken article, section "why the bottleneck is bandwidth,
 *    not capacity": each token activates a few routed experts (6 per token for
 *    the 284B model); the expert pool stays in host memory and experts are
 *    pulled into VRAM on demand.
 *  - same article, section "choosing among the five MoE backends", item
 *    `offload`: experts in host RAM, a set of LRU slots in VRAM, misses over PCIe.
 *  - claypier.com "FreeToken MoE edge runtime", first section: only the
 *    experts needed now are moved into VRAM and a global LRU cache evicts the
 *    ones unused for a while.
 *  - pomoai.com FreeToken hub, checkpoint list: MXFP4, NVFP4, FP8 and BF16
 *    weight formats.
 * The pages give no formula for the layer; the arithmetic below is the plain
 * reading of a top-k routed SwiGLU MoE layer (router logits + bias, softmax,
 * top-k, renormalise over the k picks, SwiGLU experts, gate-weighted sum).
 * Where the pages are silent, the reading taken is stated in the comment of
 * the function concerned: bias added to the logit before selection and
 * gating; picks in descending logit order with ties to the lower id; a stable
 * permutation by flat pair index; silu on the gate projection; the routing
 * gate applied after the down projection; the shared expert with weight 1.
 *
 * Precision: products and sums in double, results rounded to float.
 * Parallelism: OpenMP over independent tokens/rows only (no reordering of any
 * sum).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

int orc_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

/* Threads the calling thread's OpenMP regions use from now on (the setting
 * belongs to the calling thread). */
void orc_set_threads(int n) {
#ifdef _OPENMP
  omp_set_num_threads(n);
#else
  (void)n;
#endif
}

/* ---------------------------------------------------------------------------
 * Number formats (OCP 8-bit floating point spec, E4M3; OCP MX spec, E2M1).
 * ------------------------------------------------------------------------- */

float orc_bf16_to_f32(uint16_t v) {
  uint32_t u = (uint32_t)v << 16;
  float f;
  memcpy(&f, &u, 4);
  return f;
}

/* E4M3: 1 sign, 4 exponent bits (bias 7), 3 mantissa bits; exponent 0 is
 * subnormal (m * 2^-9); S.1111.111 is NaN; no infinities.  Max finite 448. */
double orc_e4m3_value(uint8_t q) {
  int sgn = (q >> 7) & 1, e = (q >> 3) & 15, m = q & 7;
  double v;
  if (e == 15 && m == 7) return NAN;
  if (e == 0) v = m * pow(2.0, -9);
  else v = (1.0 + m / 8.0) * pow(2.0, e - 7);
  return sgn ? -v : v;
}

/* E2M1: 1 sign, 2 exponent bits (bias 1), 1 mantissa bit; values
 * {0, 0.5, 1, 1.5, 2, 3, 4, 6}. */
double orc_e2m1_value(uint8_t nib) {
  int sgn = (nib >> 3) & 1, e = (nib >> 1) & 3, m = nib & 1;
  double v = (e == 0) ? 0.5 * m : (1.0 + 0.5 * m) * pow(2.0, e - 1);
  return sgn ? -v : v;
}

static double orc_e4m3_table[127];       /* values of codes 0x00 .. 0x7E */
static double orc_e4m3_all[256];         /* value of every code (decode lookup) */
static double orc_e2m1_all[16];

__attribute__((constructor)) static void orc_init_tables(void) {
  for (int c = 0; c < 127; ++c) orc_e4m3_table[c] = orc_e4m3_value((uint8_t)c);
  for (int c = 0; c < 256; ++c) orc_e4m3_all[c] = orc_e4m3_value((uint8_t)c);
  for (int c = 0; c < 16; ++c) orc_e2m1_all[c] = orc_e2m1_value((uint8_t)c);
}

/* Round to the nearest finite E4M3 value, ties to the code with an even
 * mantissa, magnitudes beyond 448 saturate to 448.  Done by exhaustive search
 * over the 127 non-negative finite codes. */
uint8_t orc_e4m3_encode(float v) {
  double a = fabs((double)v);
  int best = 0;
  double bd = INFINITY;
  for (int c = 0; c < 127; ++c) {         /* 0x00 .. 0x7E */
    double dd = fabs(a - orc_e4m3_table[c]);
    if (dd < bd || (dd == bd && (c & 1) == 0)) { bd = dd; best = c; }
  }
  if (best == 0) return 0;
  return (uint8_t)((v < 0.0f ? 0x80 : 0) | best);
}

/* Round to the nearest E2M1 value, ties to the even code, saturating at 6.
 * Magnitudes above 6 take code 7 outright: for huge ones the distances to 4
 * and to 6 round to the same double, and the tie rule would pick 4. */
uint8_t orc_e2m1_encode(float v) {
  double a = fabs((double)v);
  int best = 0;
  double bd = INFINITY;
  for (int c = 0; c < 8; ++c) {
    double dd = fabs(a - orc_e2m1_value((uint8_t)c));
    if (dd < bd || (dd == bd && (c & 1) == 0)) { bd = dd; best = c; }
  }
  if (a > 6.0) best = 7;
  if (best == 0) return 0;
  return (uint8_t)((v < 0.0f ? 0x8 : 0) | best);
}

/* ---------------------------------------------------------------------------
 * Weight dequantisation: the dequantised weight is the layer's ground truth.
 * ------------------------------------------------------------------------- */

void orc_dequant_bf16(const uint16_t* w, int64_t n, float* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = orc_bf16_to_f32(w[i]);
}

/* FP8 with one fp32 scale per 128x128 block: w[r][c] = e4m3(q[r][c]) * s[r/128][c/128]. */
void orc_dequant_fp8_b128(const uint8_t* q, const float* s, int R, int C, float* out) {
  int CB = C / 128;
#pragma omp parallel for schedule(static)
  for (int r = 0; r < R; ++r)
    for (int c = 0; c < C; ++c)
      out[(int64_t)r * C + c] =
          (float)(orc_e4m3_all[q[(int64_t)r * C + c]] * (double)s[(r / 128) * CB + c / 128]);
}

/* NVFP4: w[r][c] = e2m1(q) * e4m3(s16[r][c/16]) * s_t, two codes per byte
 * along c, element 2j in the low nibble. */
void orc_dequant_nvfp4(const uint8_t* qp, const uint8_t* s16, float s_t, int R, int C, float* out) {
#pragma omp parallel for schedule(static)
  for (int r = 0; r < R; ++r)
    for (int c = 0; c < C; ++c) {
      uint8_t byte = qp[(int64_t)r * (C / 2) + c / 2];
      uint8_t nib = (c & 1) ? (byte >> 4) : (byte & 15);
      double sc = orc_e4m3_all[s16[(int64_t)r * (C / 16) + c / 16]];
      out[(int64_t)r * C + c] = (float)(orc_e2m1_all[nib] * sc * (double)s_t);
    }
}

/* ---------------------------------------------------------------------------
 * Activation quantisation (the tensor-core FP8 / NVFP4 paths quantise the
 * hidden state and the SwiGLU output before their contractions; the oracle
 * applies the same declared quantiser).  In place: each value is replaced by
 * its quantised-then-dequantised value.  All scale arithmetic in fp32.
 * ------------------------------------------------------------------------- */

/* FP8: groups of 128 consecutive elements of a row; s = amax/448;
 * v <- e4m3(v / s) * s; an all-zero group stays zero. */
void orc_qa_fp8_g128(float* v, int rows, int K) {
  for (int r = 0; r < rows; ++r)
    for (int g = 0; g < K / 128; ++g) {
      float* p = v + (int64_t)r * K + g * 128;
      float amax = 0.0f;
      for (int j = 0; j < 128; ++j) if (fabsf(p[j]) > amax) amax = fabsf(p[j]);
      float s = amax / 448.0f;
      for (int j = 0; j < 128; ++j) {
        if (s == 0.0f) { p[j] = 0.0f; continue; }
        float qv = p[j] / s;
        p[j] = (float)(orc_e4m3_value(orc_e4m3_encode(qv)) * (double)s);
      }
    }
}

/* NVFP4 activations: groups of 16 consecutive elements of a row;
 * s16 = e4m3(amax/6) (per-tensor scale 1); v <- e2m1(v / s16) * s16. */
void orc_qa_nvfp4_g16(float* v, int rows, int K) {
  for (int r = 0; r < rows; ++r)
    for (int g = 0; g < K / 16; ++g) {
      float* p = v + (int64_t)r * K + g * 16;
      float amax = 0.0f;
      for (int j = 0; j < 16; ++j) if (fabsf(p[j]) > amax) amax = fabsf(p[j]);
      float s = (float)orc_e4m3_value(orc_e4m3_encode(amax / 6.0f));
      for (int j = 0; j < 16; ++j) {
        if (s == 0.0f) { p[j] = 0.0f; continue; }
        float qv = p[j] / s;
        p[j] = (float)(orc_e2m1_value(orc_e2m1_encode(qv)) * (double)s);
      }
    }
}

/* NVFP4 activations with a per-tensor global scale gs (fp32), the NVFP4
 * checkpoint convention of a static calibrated activation scale: groups of 16
 * consecutive elements of a row; s16 = e4m3(amax / (6 gs)); with
 * u = s16 * gs, v <- e2m1(v / u) * u.  gs = 1 is orc_qa_nvfp4_g16.  The global
 * scale keeps small activations in the e4m3 scale range (with gs = 1 a group
 * whose amax/6 is below half the smallest e4m3 subnormal, 2^-10, quantises to
 * zero). */
void orc_qa_nvfp4_g16_gs(float* v, int rows, int K, float gs) {
  const float six_gs = 6.0f * gs;
  for (int r = 0; r < rows; ++r)
    for (int g = 0; g < K / 16; ++g) {
      float* p = v + (int64_t)r * K + g * 16;
      float amax = 0.0f;
      for (int j = 0; j < 16; ++j) if (fabsf(p[j]) > amax) amax = fabsf(p[j]);
      float u = (float)orc_e4m3_value(orc_e4m3_encode(amax / six_gs)) * gs;
      for (int j = 0; j < 16; ++j) {
        if (u == 0.0f) { p[j] = 0.0f; continue; }
        float qv = p[j] / u;
        p[j] = (float)(orc_e2m1_value(orc_e2m1_encode(qv)) * (double)u);
      }
    }
}

/* ---------------------------------------------------------------------------
 * MXFP4 (pomoai.com FreeToken hub, checkpoint list: the engine loads MXFP4,
 * NVFP4, FP8 and BF16 checkpoints).  The format is the OCP Microscaling (MX)
 * v1.0 one: blocks of 32 consecutive elements along a row share one E8M0
 * scale X = 2^(e - 127) (code 255 is NaN) and each element is E2M1.
 * Quantisation of a block (the specification's conversion rule): the shared
 * exponent is floor(log2(max |v|)) minus the largest E2M1 exponent (2),
 * clamped to the E8M0 range [-127, 127]; each element is v / X rounded to
 * the nearest E2M1 value, ties to even, saturating at 6.  Reading for an
 * all-zero block (the specification leaves the exponent of zero open):
 * scale code 127 (X = 1) and zero elements.
 * ------------------------------------------------------------------------- */

double orc_e8m0_value(uint8_t c) { return c == 255 ? NAN : ldexp(1.0, (int)c - 127); }

/* Shared-scale code of one block of n values. */
uint8_t orc_mx_scale_code(const float* v, int n) {
  float amax = 0.0f;
  for (int j = 0; j < n; ++j) if (fabsf(v[j]) > amax) amax = fabsf(v[j]);
  if (amax == 0.0f) return 127;
  int e = (int)floor(log2((double)amax)) - 2;
  if (e < -127) e = -127;
  if (e > 127) e = 127;
  return (uint8_t)(e + 127);
}

/* w [R][C] -> packed codes q [R][C/2] (element 2j in the low nibble) and
 * scale codes s [R][C/32]. */
void orc_quant_mxfp4(const float* w, int R, int C, uint8_t* q, uint8_t* s) {
  for (int r = 0; r < R; ++r)
    for (int b = 0; b < C / 32; ++b) {
      const float* p = w + (int64_t)r * C + b * 32;
      uint8_t sc = orc_mx_scale_code(p, 32);
      s[(int64_t)r * (C / 32) + b] = sc;
      double X = orc_e8m0_value(sc);
      for (int j = 0; j < 32; j += 2) {
        uint8_t lo = orc_e2m1_encode((float)(p[j] / X)), hi = orc_e2m1_encode((float)(p[j + 1] / X));
        q[(int64_t)r * (C / 2) + (b * 32 + j) / 2] = (uint8_t)(lo | (hi << 4));
      }
    }
}

/* w[r][c] = e2m1(q) * 2^(s[r][c/32] - 127). */
void orc_dequant_mxfp4(const uint8_t* qp, const uint8_t* s, int R, int C, float* out) {
#pragma omp parallel for schedule(static)
  for (int r = 0; r < R; ++r)
    for (int c = 0; c < C; ++c) {
      uint8_t byte = qp[(int64_t)r * (C / 2) + c / 2];
      uint8_t nib = (c & 1) ? (byte >> 4) : (byte & 15);
      out[(int64_t)r * C + c] = (float)(orc_e2m1_all[nib] * orc_e8m0_value(s[(int64_t)r * (C / 32) + c / 32]));
    }
}

/* MXFP4 activations, in place: each 32-group of a row is replaced by its
 * quantised-then-dequantised values. */
void orc_qa_mxfp4_g32(float* v, int rows, int K) {
  for (int r = 0; r < rows; ++r)
    for (int b = 0; b < K / 32; ++b) {
      float* p = v + (int64_t)r * K + b * 32;
      double X = orc_e8m0_value(orc_mx_scale_code(p, 32));
      for (int j = 0; j < 32; ++j) p[j] = (float)(orc_e2m1_value(orc_e2m1_encode((float)(p[j] / X))) * X);
    }
}

/* ---------------------------------------------------------------------------
 * Router: logits, top-k, gates.
 * ------------------------------------------------------------------------- */

/* logits[t][e] = sum_i x[t][i] * Wr[e][i] + b[e]  (double sum, rounded to float). */
void orc_router_logits(const float* x, int T, int d, const float* Wr, const float* b, int E, float* logits) {
#pragma omp parallel for schedule(static)
  for (int t = 0; t < T; ++t)
    for (int e = 0; e < E; ++e) {
      double acc = 0.0;
      for (int i = 0; i < d; ++i) acc += (double)x[(int64_t)t * d + i] * (double)Wr[(int64_t)e * d + i];
      if (b) acc += (double)b[e];
      logits[(int64_t)t * E + e] = (float)acc;
    }
}

/* order[0..E) = expert ids sorted by logit descending, equal logits by id ascending. */
static void orc_sort_desc(const float* l, int E, int* order) {
  for (int e = 0; e < E; ++e) order[e] = e;
  for (int i = 1; i < E; ++i) {          /* insertion sort: stable on id */
    int v = order[i], j = i - 1;
    while (j >= 0 && l[order[j]] < l[v]) { order[j + 1] = order[j]; --j; }
    order[j + 1] = v;
  }
}

/* ok[t] = 1 iff every gap among the top-(k+1) sorted logits is >= margin
 * (the synthetic inputs are redrawn until this holds, so the pick set and
 * pick order are unique). */
void orc_margin_ok(const float* logits, int T, int E, int k, double margin, uint8_t* ok) {
  int* order = (int*)malloc(sizeof(int) * E);
  for (int t = 0; t < T; ++t) {
    const float* l = logits + (int64_t)t * E;
    orc_sort_desc(l, E, order);
    int last = (k < E) ? k : E - 1;
    ok[t] = 1;
    for (int r = 0; r < last; ++r)
      if ((double)l[order[r]] - (double)l[order[r + 1]] < margin) ok[t] = 0;
  }
  free(order);
}

/* ids[t][j] = j-th largest logit's expert; gates: softmax over all E experts,
 * then renormalised over the k picks: g_j = p[id_j] / sum_j' p[id_j']. */
void orc_topk_gates(const float* logits, int T, int E, int k, int32_t* ids, float* gates) {
  int* order = (int*)malloc(sizeof(int) * E);
  double* p = (double*)malloc(sizeof(double) * E);
  for (int t = 0; t < T; ++t) {
    const float* l = logits + (int64_t)t * E;
    orc_sort_desc(l, E, order);
    double m = l[order[0]], z = 0.0;
    for (int e = 0; e < E; ++e) { p[e] = exp((double)l[e] - m); z += p[e]; }
    for (int e = 0; e < E; ++e) p[e] /= z;
    double zk = 0.0;
    for (int j = 0; j < k; ++j) zk += p[order[j]];
    for (int j = 0; j < k; ++j) {
      ids[(int64_t)t * k + j] = order[j];
      gates[(int64_t)t * k + j] = (float)(p[order[j]] / zk);
    }
  }
  free(p);
  free(order);
}

/* ---------------------------------------------------------------------------
 * Permutation of the P = T*k (token, pick) pairs by expert.
 * counts[e] = #pairs routed to e; offsets[e] = exclusive prefix sum (offsets[E] = P);
 * pairs are visited in ascending flat index q = t*k + j and placed at
 * pos = offsets[e] + (number of earlier pairs with the same expert);
 * perm[pos] = q, inv[q] = pos.
 * ------------------------------------------------------------------------- */
void orc_permute(const int32_t* ids, int T, int k, int E, int32_t* counts, int32_t* offsets,
                 int32_t* perm, int32_t* inv) {
  int64_t P = (int64_t)T * k;
  for (int e = 0; e < E; ++e) counts[e] = 0;
  for (int64_t q = 0; q < P; ++q) counts[ids[q]]++;
  offsets[0] = 0;
  for (int e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + counts[e];
  int32_t* run = (int32_t*)calloc((size_t)E, sizeof(int32_t));
  for (int64_t q = 0; q < P; ++q) {
    int e = ids[q];
    int32_t pos = offsets[e] + run[e]++;
    perm[pos] = (int32_t)q;
    inv[q] = pos;
  }
  free(run);
}

/* ---------------------------------------------------------------------------
 * LRU slot cache step.
 * State: slot_of_expert[E] (-1: not resident), expert_of_slot[S] (-1: empty),
 * last_use[S] (-1: never).  Step s requests the distinct expert ids in
 * ids[0..n).  Hits: last_use = s.  Misses, in ascending expert id, each take
 * the slot with the smallest last_use among slots with last_use < s (ties: the
 * lowest slot index), unmapping its previous expert.  Returns 0 on success,
 * -1 (state untouched) when more distinct experts are requested than slots.
 * miss_expert/miss_slot list the misses in the order they were placed.
 * ------------------------------------------------------------------------- */
int orc_lru_step(int E, int S, int32_t* slot_of_expert, int32_t* expert_of_slot, int64_t* last_use,
                 int64_t s, const int32_t* ids, int n, int32_t* miss_expert, int32_t* miss_slot,
                 int32_t* n_distinct, int32_t* n_hits, int32_t* n_miss) {
  uint8_t* want = (uint8_t*)calloc((size_t)E, 1);
  for (int i = 0; i < n; ++i) want[ids[i]] = 1;
  int distinct = 0;
  for (int e = 0; e < E; ++e) distinct += want[e];
  *n_distinct = distinct;
  if (distinct > S) { free(want); *n_hits = 0; *n_miss = 0; return -1; }
  int hits = 0, misses = 0;
  for (int e = 0; e < E; ++e)
    if (want[e] && slot_of_expert[e] >= 0) { last_use[slot_of_expert[e]] = s; ++hits; }
  for (int e = 0; e < E; ++e) {
    if (!want[e] || slot_of_expert[e] >= 0) continue;
    int victim = -1;
    for (int j = 0; j < S; ++j)
      if (last_use[j] < s && (victim < 0 || last_use[j] < last_use[victim])) victim = j;
    /* victim >= 0 is guaranteed by distinct <= S */
    if (expert_of_slot[victim] >= 0) slot_of_expert[expert_of_slot[victim]] = -1;
    expert_of_slot[victim] = e;
    slot_of_expert[e] = victim;
    last_use[victim] = s;
    miss_expert[misses] = e;
    miss_slot[misses] = victim;
    ++misses;
  }
  *n_hits = hits;
  *n_miss = misses;
  free(want);
  return 0;
}

/* ---------------------------------------------------------------------------
 * Bandwidth-adaptive miss split (freelamp.com FreeToken article, section 2.1
 * "bandwidth-adaptive execution": the machine's measured PCIe bandwidth Bp and
 * host bandwidth Bh set how many of a step's m cache misses are copied to the
 * GPU and how many are computed on the CPU, the two running at once;
 * chenxutan.com FreeToken article, "choosing among the five MoE backends",
 * `hybrid`: the misses are split by the bandwidth ratio so that both sides
 * finish together).  Both sides move one expert bank per miss, so they finish
 * together when q / Bp = (m - q) / Bh:  q = m Bp / (Bp + Bh), taken to the
 * nearest integer, halves up, in fp64: floor(m * Bp / (Bp + Bh) + 0.5).  (The
 * printed formula q* = m Bp / Bh does not balance the two sides the text
 * describes; the balanced form is the reading.)  Which m - q misses go to the
 * host is not said: read as those with the fewest routed pairs (the host's
 * cost per expert grows with its rows, a copy's does not), ties to the lower
 * expert id.
 *   counts[E]   pairs routed to each expert this step
 *   resident[E] nonzero: expert in the cache (a hit)
 *   host[]      out: the host's experts, fewest pairs first (at most E)
 * Returns m - q; *m_out = m, *q_out = q.  Selection by repeated minimum.
 * ------------------------------------------------------------------------- */
int orc_hybrid_split(int E, const int32_t* counts, const int32_t* resident, double bp, double bh, int32_t* host,
                     int32_t* m_out, int32_t* q_out) {
  int m = 0;
  for (int e = 0; e < E; ++e)
    if (counts[e] > 0 && !resident[e]) ++m;
  int q = (int)floor((double)m * bp / (bp + bh) + 0.5);
  if (q < 0) q = 0;
  if (q > m) q = m;
  uint8_t* taken = (uint8_t*)calloc((size_t)E + 1, 1);
  for (int i = 0; i < m - q; ++i) {
    int best = -1;
    for (int e = 0; e < E; ++e)
      if (counts[e] > 0 && !resident[e] && !taken[e] && (best < 0 || counts[e] < counts[best])) best = e;
    taken[best] = 1;
    host[i] = best;
  }
  free(taken);
  *m_out = m;
  *q_out = q;
  return m - q;
}

/* ---------------------------------------------------------------------------
 * Cache step of a cache shared by several layers, with slots held back.
 * Keys: the cache holds n_keys entries; in a cache shared by several layers of
 * E experts each, layer l's expert e is key l*E + e.  Step s requests the
 * distinct keys in keys[0..n).  As in orc_lru_step, hits set last_use = s and
 * misses, in ascending key, each take the slot with the smallest last_use
 * (ties: lowest slot index) -- but only among slots with last_use < reserve
 * (reserve <= s): slots used in steps reserve..s-1 keep their experts, because
 * the compute of those steps may still be reading them while this step's
 * copies run (pomoai.com FreeToken hub, prefill-overlap paragraph: layer n+1's
 * experts are copied while layer n computes, which needs room for two whole
 * layers).  With reserve = s this is orc_lru_step.  Returns -1 with the state
 * untouched when the misses outnumber the slots they may take.
 * ------------------------------------------------------------------------- */
int orc_lru_step_reserve(int n_keys, int S, int32_t* slot_of_key, int32_t* key_of_slot, int64_t* last_use,
                         int64_t s, int64_t reserve, const int32_t* keys, int n, int32_t* miss_key,
                         int32_t* miss_slot, int32_t* n_distinct, int32_t* n_hits, int32_t* n_miss) {
  uint8_t* want = (uint8_t*)calloc((size_t)n_keys, 1);
  for (int i = 0; i < n; ++i) want[keys[i]] = 1;
  int distinct = 0, hits = 0, misses = 0, free_slots = 0;
  for (int key = 0; key < n_keys; ++key) {
    if (!want[key]) continue;
    ++distinct;
    if (slot_of_key[key] >= 0) ++hits; else ++misses;
  }
  /* slots a miss may take: not used since `reserve`, and not hit by this step */
  for (int j = 0; j < S; ++j) {
    int hit = key_of_slot[j] >= 0 && want[key_of_slot[j]];
    if (last_use[j] < reserve && !hit) ++free_slots;
  }
  *n_distinct = distinct;
  if (misses > free_slots) { free(want); *n_hits = 0; *n_miss = 0; return -1; }
  for (int key = 0; key < n_keys; ++key)
    if (want[key] && slot_of_key[key] >= 0) last_use[slot_of_key[key]] = s;
  int placed = 0;
  for (int key = 0; key < n_keys; ++key) {
    if (!want[key] || slot_of_key[key] >= 0) continue;
    int victim = -1;
    for (int j = 0; j < S; ++j)
      if (last_use[j] < reserve && (victim < 0 || last_use[j] < last_use[victim])) victim = j;
    if (key_of_slot[victim] >= 0) slot_of_key[key_of_slot[victim]] = -1;
    key_of_slot[victim] = key;
    slot_of_key[key] = victim;
    last_use[victim] = s;
    miss_key[placed] = key;
    miss_slot[placed] = victim;
    ++placed;
  }
  *n_hits = hits;
  *n_miss = placed;
  free(want);
  return 0;
}

/* ---------------------------------------------------------------------------
 * Elastic slot-pool resize.  The pages let the expert cache's share of VRAM
 * change at run time without restarting the engine or reloading weights
 * (pomoai.com FreeToken hub, the two-level expert memory paragraph; freelamp.com
 * FreeToken article, section 2.3 "elastic memory management": `ftctl cache
 * --moe <slots>`).  Reading taken here: the min(S_new, resident)
 * most recently used resident experts stay (largest last_use first, ties to the
 * lower old slot), in their old slot order, in slots 0..; the rest are evicted;
 * each kept expert keeps its last_use; the step counter does not move.
 * Written as the definition: S_new rounds of "take the most recent resident
 * slot not yet taken".  Returns the number of kept experts; move_from[i] ->
 * i is the bank move of the i-th kept expert.
 * ------------------------------------------------------------------------- */
int orc_lru_resize(int E, int S_old, const int32_t* slot_of_expert, const int32_t* expert_of_slot,
                   const int64_t* last_use, int S_new, int32_t* soe_new, int32_t* eos_new, int64_t* lu_new,
                   int32_t* move_from) {
  (void)slot_of_expert;
  uint8_t* kept = (uint8_t*)calloc((size_t)(S_old > 0 ? S_old : 1), 1);
  for (int r = 0; r < S_new; ++r) {
    int best = -1;
    for (int j = 0; j < S_old; ++j)
      if (expert_of_slot[j] >= 0 && !kept[j] && (best < 0 || last_use[j] > last_use[best])) best = j;
    if (best < 0) break;
    kept[best] = 1;
  }
  for (int e = 0; e < E; ++e) soe_new[e] = -1;
  for (int j = 0; j < S_new; ++j) { eos_new[j] = -1; lu_new[j] = -1; }
  int n = 0;
  for (int j = 0; j < S_old; ++j) {
    if (!kept[j]) continue;
    eos_new[n] = expert_of_slot[j];
    lu_new[n] = last_use[j];
    soe_new[expert_of_slot[j]] = n;
    move_from[n] = j;
    ++n;
  }
  free(kept);
  return n;
}

/* ---------------------------------------------------------------------------
 * Expert FFN (SwiGLU) over n rows, and the combine.
 * h[i] = silu(x . Wg[i]) * (x . Wu[i]),  silu(z) = z / (1 + exp(-z));
 * y[j] = h . Wd[j].
 * qa = 0: no activation quantisation; 1: FP8 (128-groups) on x and h;
 * 2: NVFP4 (16-groups) on x and h; 3: MXFP4 (32-groups, E8M0 scales) on x
 * and h -- the same activation reading as NVFP4, with MX's own block format.
 * ------------------------------------------------------------------------- */
void orc_expert_ffn_gs(const float* x, int n, int d, int I, const float* Wg, const float* Wu,
                       const float* Wd, int qa, float gx, float gh, float* y);

void orc_expert_ffn(const float* x, int n, int d, int I, const float* Wg, const float* Wu,
                    const float* Wd, int qa, float* y) {
  orc_expert_ffn_gs(x, n, d, I, Wg, Wu, Wd, qa, 1.0f, 1.0f, y);
}

/* As orc_expert_ffn; in NVFP4 mode (qa = 2) x is quantised with the global
 * scale gx and h with gh (orc_qa_nvfp4_g16_gs); other modes ignore them. */
void orc_expert_ffn_gs(const float* x, int n, int d, int I, const float* Wg, const float* Wu,
                       const float* Wd, int qa, float gx, float gh, float* y) {
#pragma omp parallel for schedule(dynamic)
  for (int r = 0; r < n; ++r) {
    float* xr = (float*)malloc(sizeof(float) * d);
    float* h = (float*)malloc(sizeof(float) * I);
    memcpy(xr, x + (int64_t)r * d, sizeof(float) * d);
    if (qa == 1) orc_qa_fp8_g128(xr, 1, d);
    if (qa == 2) orc_qa_nvfp4_g16_gs(xr, 1, d, gx);
    if (qa == 3) orc_qa_mxfp4_g32(xr, 1, d);
    for (int i = 0; i < I; ++i) {
      double g = 0.0, u = 0.0;
      for (int c = 0; c < d; ++c) {
        g += (double)xr[c] * (double)Wg[(int64_t)i * d + c];
        u += (double)xr[c] * (double)Wu[(int64_t)i * d + c];
      }
      h[i] = (float)(g / (1.0 + exp(-g)) * u);
    }
    if (qa == 1) orc_qa_fp8_g128(h, 1, I);
    if (qa == 2) orc_qa_nvfp4_g16_gs(h, 1, I, gh);
    if (qa == 3) orc_qa_mxfp4_g32(h, 1, I);
    for (int j = 0; j < d; ++j) {
      double acc = 0.0;
      for (int i = 0; i < I; ++i) acc += (double)h[i] * (double)Wd[(int64_t)j * I + i];
      y[(int64_t)r * d + j] = (float)acc;
    }
    free(h);
    free(xr);
  }
}

/* out[t] = sum_{j=0..k-1, ascending} g[t][j] * y[t*k + j]  (+ ysh[t] if given);
 * y rows here are in pair order q = t*k + j. */
void orc_combine(const float* y, const float* gates, int T, int k, int d, const float* ysh, float* out) {
  for (int t = 0; t < T; ++t)
    for (int c = 0; c < d; ++c) {
      double acc = 0.0;
      for (int j = 0; j < k; ++j)
        acc += (double)gates[(int64_t)t * k + j] * (double)y[((int64_t)t * k + j) * d + c];
      if (ysh) acc += (double)ysh[(int64_t)t * d + c];
      out[(int64_t)t * d + c] = (float)acc;
    }
}
