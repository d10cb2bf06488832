/*
 * oracle.c -- plain CPU oracle for the W4A16 mixture-of-experts layer.
 *
 * TEST INFRASTRUCTURE ONLY. Only the tests, the smoke check and the benchmark's CPU
 * baseline may load this library. It shares no code with the CUDA path.
 *
 * What it computes, and the passage each step follows (source: the Novita/vLLM blog
 * "vLLM x Novita AI: Chord W4A16 INT4 MoE Kernel fuer Kimi K2.x", German edition,
 * cited by section):
 *
 *   unpack   uint4 codes, eight per int32 along K, low nibble first (format named in
 *            "vLLM-Integration": uint4, group-32, BF16 scales, compressed-tensors
 *            pack-quantized INT4; the nibble order is the pack-quantized convention).
 *   dequant  w = bf16_rne( (q - 8) * s ), subtract first, then scale, rounded once to
 *            BF16 ("H200 und Blackwell indexierter Decode": subtract-then-scale keeps
 *            the unfused BF16 rounding order). Zero point 8 is the symmetric uint4
 *            convention of the layer's problem statement.
 *   align    block-padded sorted_ids / expert_ids / num_tokens_padded routing tensors
 *            ("Zwei Kernel-Familien": the indexed path consumes vLLM's sorted routing;
 *            Figure 3: activations stay unpadded, routing indices carry sentinels).
 *   gate_up  h = x . W13[e]^T, FP32 accumulation (F16 accumulation is not offered,
 *            "vLLM-Integration", last bullets).
 *   act      a = bf16_rne( silu(h[i]) * h[I+i] ), gate rows first, up rows second.
 *   down     y = a . W2[e]^T, FP32 accumulation.
 *   combine  out[t] = bf16_rne( sum over local slots j, ascending, of w[t,j] * y_j ).
 *   grouped  the grouped operator on the same dequant ("Gruppierte SM90-Kernel"): rows
 *            concatenated per expert with m_indices (-1 = padding), or a fixed row budget
 *            per expert with masked_m valid counts; out[m] = bf16_rne( x[m] . W[e_m]^T ),
 *            FP32 accumulation; rows without an expert are not written (consumers ignore
 *            them, same section).
 *   router   (the step upstream of align, for the fused routing entry point) per token
 *            the topk largest logits, ties to the lower expert id, and their softmax
 *            renormalised over the chosen ones: w_r = exp(l_r - l_0) / sum_j exp(l_j - l_0)
 *            (the layer's problem statement: top-k softmax routing, weights renormalised;
 *            the full softmax denominator cancels in the renormalisation).
 *
 * Every floating-point reduction runs in plain ascending order in FP32; this file is
 * built with -ffp-contract=off so no multiply-add is fused.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_GROUP 32

float oracle_bf16_to_f32(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return f;
}

/* IEEE round-to-nearest-even from binary32 to bfloat16 (keep the top 16 bits). */
uint16_t oracle_f32_to_bf16(float f) {
  uint32_t u;
  memcpy(&u, &f, sizeof u);
  if ((u & 0x7f800000u) == 0x7f800000u) {      /* inf or nan: no rounding */
    if (u & 0x007fffffu) return (uint16_t)((u >> 16) | 0x0040u);
    return (uint16_t)(u >> 16);
  }
  uint32_t keep_lsb = (u >> 16) & 1u;
  u += 0x7fffu + keep_lsb;                      /* carries into the exponent on overflow */
  return (uint16_t)(u >> 16);
}

static float round_bf16(float f) { return oracle_bf16_to_f32(oracle_f32_to_bf16(f)); }

/* Code of element (n, k) of one expert's packed matrix [N, K/8]. */
static int code_at(const int32_t* qweight, int64_t K, int64_t n, int64_t k) {
  uint32_t word = (uint32_t)qweight[n * (K / 8) + k / 8];
  return (int)((word >> (4 * (k % 8))) & 0xFu);
}

/* Dequantise one expert: w[n*K + k] = bf16((q - 8) * s[n, k/32]) as float. */
void oracle_dequant(const int32_t* qweight, const uint16_t* scales, int64_t N, int64_t K,
                    float* w) {
#pragma omp parallel for schedule(static)
  for (int64_t n = 0; n < N; ++n) {
    for (int64_t k = 0; k < K; ++k) {
      float s = oracle_bf16_to_f32(scales[n * (K / ORACLE_GROUP) + k / ORACLE_GROUP]);
      float qm8 = (float)(code_at(qweight, K, n, k) - 8);
      w[n * K + k] = round_bf16(qm8 * s);
    }
  }
}

/* Capacity of sorted_ids: every local pair plus at most BM-1 padding rows per expert. */
int64_t oracle_align_capacity(int64_t T, int64_t topk, int64_t E, int64_t BM) {
  return T * topk + E * (BM - 1);
}

int64_t oracle_align_blocks(int64_t T, int64_t topk, int64_t E, int64_t BM) {
  int64_t cap = oracle_align_capacity(T, topk, E, BM);
  return (cap + BM - 1) / BM;
}

/*
 * moe_align: flat index f = t*topk + j; a slot is local when 0 <= topk_ids[f] < E.
 * c_e = local slots of expert e; p_e = ceil(c_e / BM) * BM; off_e = sum_{e'<e} p_e'.
 * sorted_ids[off_e + r] = the r-th local flat index of expert e in increasing f;
 * every other slot of sorted_ids (capacity T*topk + E*(BM-1)) holds the sentinel T*topk.
 * expert_ids[b] = e for the p_e/BM blocks of e, -1 for blocks past num_tokens_padded.
 * expert_offsets (E+1 entries, may be NULL) receives off_0 .. off_E.
 * Returns 0, or -1 on invalid sizes.
 */
int oracle_moe_align(const int32_t* topk_ids, int64_t T, int64_t topk, int64_t E, int64_t BM,
                     int32_t* sorted_ids, int32_t* expert_ids, int32_t* num_tokens_padded,
                     int32_t* expert_offsets) {
  if (T < 0 || topk < 1 || E < 1 || BM < 1) return -1;
  int64_t n = T * topk;
  int64_t cap = oracle_align_capacity(T, topk, E, BM);
  int64_t nblocks = oracle_align_blocks(T, topk, E, BM);
  int64_t* count = (int64_t*)calloc((size_t)E, sizeof(int64_t));
  int64_t* off = (int64_t*)calloc((size_t)E + 1, sizeof(int64_t));
  int64_t* fill = (int64_t*)calloc((size_t)E, sizeof(int64_t));
  if (!count || !off || !fill) { free(count); free(off); free(fill); return -1; }

  for (int64_t f = 0; f < n; ++f) {
    int32_t e = topk_ids[f];
    if (e >= 0 && e < E) count[e] += 1;
  }
  for (int64_t e = 0; e < E; ++e) {
    int64_t padded = (count[e] + BM - 1) / BM * BM;
    off[e + 1] = off[e] + padded;
  }
  for (int64_t i = 0; i < cap; ++i) sorted_ids[i] = (int32_t)n;
  for (int64_t f = 0; f < n; ++f) {
    int32_t e = topk_ids[f];
    if (e >= 0 && e < E) {
      sorted_ids[off[e] + fill[e]] = (int32_t)f;
      fill[e] += 1;
    }
  }
  for (int64_t b = 0; b < nblocks; ++b) expert_ids[b] = -1;
  for (int64_t e = 0; e < E; ++e)
    for (int64_t b = off[e] / BM; b < off[e + 1] / BM; ++b) expert_ids[b] = (int32_t)e;
  *num_tokens_padded = (int32_t)off[E];
  if (expert_offsets)
    for (int64_t e = 0; e <= E; ++e) expert_offsets[e] = (int32_t)off[e];
  free(count); free(off); free(fill);
  return 0;
}

static float silu_f32(float g) { return g / (1.0f + expf(-g)); }

/*
 * The layer for the token rows listed in `rows` (n_rows of them; NULL = all T rows):
 * out[r, :] (bf16 bits, [n_rows, H]) for token rows[r].
 * x [T,H] bf16; topk_ids [T,topk]; topk_weights [T,topk] f32;
 * qw13 [E,2I,H/8], s13 [E,2I,H/32]; qw2 [E,H,I/8], s2 [E,H,I/32].
 * n_threads <= 0 keeps the OpenMP default. Returns 0, -1 on bad sizes, -2 on OOM.
 */
int oracle_moe_forward(const uint16_t* x, const int32_t* topk_ids, const float* topk_weights,
                       const int32_t* qw13, const uint16_t* s13, const int32_t* qw2,
                       const uint16_t* s2, int64_t T, int64_t H, int64_t I, int64_t E,
                       int64_t topk, const int64_t* rows, int64_t n_rows, uint16_t* out,
                       int n_threads) {
  if (T < 0 || H <= 0 || I <= 0 || E <= 0 || topk <= 0) return -1;
  if (H % ORACLE_GROUP || I % ORACLE_GROUP) return -1;
  if (!rows) n_rows = T;
#ifdef _OPENMP
  if (n_threads > 0) omp_set_num_threads(n_threads);
#else
  (void)n_threads;
#endif
  const int64_t N13 = 2 * I;
  float* w13 = (float*)malloc((size_t)(N13 * H) * sizeof(float));
  float* w2 = (float*)malloc((size_t)(H * I) * sizeof(float));
  float* y = (float*)malloc((size_t)(n_rows * topk * H) * sizeof(float) + 1);
  int64_t* pairs = (int64_t*)malloc((size_t)(n_rows * topk) * sizeof(int64_t) + 1);
  float* h = (float*)malloc((size_t)(n_rows * topk * N13) * sizeof(float) + 1);
  float* a = (float*)malloc((size_t)(n_rows * topk * I) * sizeof(float) + 1);
  float* xf = (float*)malloc((size_t)(n_rows * H) * sizeof(float) + 1);
  if (!w13 || !w2 || !y || !pairs || !h || !a || !xf) {
    free(w13); free(w2); free(y); free(pairs); free(h); free(a); free(xf);
    return -2;
  }
  for (int64_t r = 0; r < n_rows; ++r) {
    int64_t t = rows ? rows[r] : r;
    for (int64_t k = 0; k < H; ++k) xf[r * H + k] = oracle_bf16_to_f32(x[t * H + k]);
  }

  for (int64_t e = 0; e < E; ++e) {
    /* the (row, slot) pairs routed to expert e; slot index p = r*topk + j */
    int64_t np = 0;
    for (int64_t r = 0; r < n_rows; ++r) {
      int64_t t = rows ? rows[r] : r;
      for (int64_t j = 0; j < topk; ++j)
        if (topk_ids[t * topk + j] == e) pairs[np++] = r * topk + j;
    }
    if (np == 0) continue;
    oracle_dequant(qw13 + e * N13 * (H / 8), s13 + e * N13 * (H / ORACLE_GROUP), N13, H, w13);
    oracle_dequant(qw2 + e * H * (I / 8), s2 + e * H * (I / ORACLE_GROUP), H, I, w2);

    /* gate_up: h[n] = sum_k x[k] * w13[n, k], FP32, ascending k */
#pragma omp parallel for schedule(static)
    for (int64_t pn = 0; pn < np * N13; ++pn) {
      int64_t p = pairs[pn / N13], n = pn % N13;
      const float* xr = xf + (p / topk) * H;
      const float* wr = w13 + n * H;
      float acc = 0.0f;
      for (int64_t k = 0; k < H; ++k) acc += xr[k] * wr[k];
      h[p * N13 + n] = acc;
    }
    /* activation: a[i] = bf16(silu(gate_i) * up_i) */
    for (int64_t q = 0; q < np; ++q) {
      int64_t p = pairs[q];
      for (int64_t i = 0; i < I; ++i)
        a[p * I + i] = round_bf16(silu_f32(h[p * N13 + i]) * h[p * N13 + I + i]);
    }
    /* down: y[n] = sum_i a[i] * w2[n, i], FP32, ascending i */
#pragma omp parallel for schedule(static)
    for (int64_t pn = 0; pn < np * H; ++pn) {
      int64_t p = pairs[pn / H], n = pn % H;
      const float* ar = a + p * I;
      const float* wr = w2 + n * I;
      float acc = 0.0f;
      for (int64_t i = 0; i < I; ++i) acc += ar[i] * wr[i];
      y[p * H + n] = acc;
    }
  }

  /* combine: out = bf16( sum_{local j ascending} w[t,j] * y_j ), zero when no local slot */
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < n_rows; ++r) {
    int64_t t = rows ? rows[r] : r;
    for (int64_t n = 0; n < H; ++n) {
      float acc = 0.0f;
      for (int64_t j = 0; j < topk; ++j) {
        int32_t e = topk_ids[t * topk + j];
        if (e >= 0 && e < E) acc += topk_weights[t * topk + j] * y[(r * topk + j) * H + n];
      }
      out[r * H + n] = oracle_f32_to_bf16(acc);
    }
  }
  free(w13); free(w2); free(y); free(pairs); free(h); free(a); free(xf);
  return 0;
}

/* Router (see the header): topk_ids[t, r] = expert of rank r (descending logit, ties to
 * the lower id), topk_weights[t, r] = exp(l_r - l_0) / sum_j exp(l_j - l_0), in double,
 * summed in rank order, rounded once to float. Returns 0, or -1 for bad arguments. */
int oracle_router_topk(const float* logits, int64_t T, int64_t G, int64_t k, int32_t* topk_ids,
                       float* topk_weights) {
  if (T < 0 || G < 1 || k < 1 || k > G) return -1;
  unsigned char* taken = (unsigned char*)malloc((size_t)G);
  double* e = (double*)malloc((size_t)k * sizeof(double));
  if (!taken || !e) {
    free(taken);
    free(e);
    return -1;
  }
  for (int64_t t = 0; t < T; ++t) {
    const float* l = logits + t * G;
    memset(taken, 0, (size_t)G);
    for (int64_t r = 0; r < k; ++r) {
      int64_t best = -1;
      for (int64_t g = 0; g < G; ++g) {
        if (taken[g]) continue;
        if (best < 0 || l[g] > l[best]) best = g; /* strictly greater: ties keep the lower id */
      }
      taken[best] = 1;
      topk_ids[t * k + r] = (int32_t)best;
    }
    const double l0 = (double)l[topk_ids[t * k]];
    double sum = 0.0;
    for (int64_t r = 0; r < k; ++r) {
      e[r] = exp((double)l[topk_ids[t * k + r]] - l0);
      sum += e[r];
    }
    for (int64_t r = 0; r < k; ++r) topk_weights[t * k + r] = (float)(e[r] / sum);
  }
  free(taken);
  free(e);
  return 0;
}

/* Grouped GEMM (see the header). Weights: one expert after another, qweight [E, N, K/8],
 * scales [E, N, K/32]. Row m of x [M, K] belongs to expert e_m:
 *   contiguous (masked_m == NULL): e_m = m_indices[m] (negative: no expert);
 *   masked (m_indices == NULL): M = E * max_m, e_m = m / max_m when m % max_m < masked_m[e_m].
 * out [M, N] bf16: rows with an expert get bf16_rne(sum_k x[m,k] * w[e_m][n,k]) (FP32,
 * ascending k); other rows are left as they are. Experts are dequantised one at a time.
 * Returns 0, or -1 for bad arguments. */
static int64_t grouped_expert_of(int64_t m, const int32_t* m_indices, const int32_t* masked_m, int64_t max_m) {
  if (m_indices) return m_indices[m];
  const int64_t g = m / max_m;
  return (m % max_m < masked_m[g]) ? g : -1;
}

int oracle_grouped_gemm(const uint16_t* x, int64_t M, int64_t K, const int32_t* qweight, const uint16_t* scales,
                        int64_t E, int64_t N, const int32_t* m_indices, const int32_t* masked_m, int64_t max_m,
                        uint16_t* out, int n_threads) {
  if (M < 0 || K < 1 || N < 1 || E < 1 || (m_indices == NULL) == (masked_m == NULL)) return -1;
  if (masked_m && (max_m < 1 || M != E * max_m)) return -1;
#ifdef _OPENMP
  if (n_threads > 0) omp_set_num_threads(n_threads);
#else
  (void)n_threads;
#endif
  float* w = (float*)malloc((size_t)N * K * sizeof(float));
  if (!w) return -1;
  for (int64_t e = 0; e < E; ++e) {
    int used = 0;
    for (int64_t m = 0; m < M && !used; ++m) used = grouped_expert_of(m, m_indices, masked_m, max_m) == e;
    if (!used) continue;
    oracle_dequant(qweight + e * N * (K / 8), scales + e * N * (K / ORACLE_GROUP), N, K, w);
#pragma omp parallel for schedule(dynamic, 4)
    for (int64_t m = 0; m < M; ++m) {
      if (grouped_expert_of(m, m_indices, masked_m, max_m) != e) continue;
      for (int64_t n = 0; n < N; ++n) {
        float acc = 0.0f;
        for (int64_t k = 0; k < K; ++k) acc += oracle_bf16_to_f32(x[m * K + k]) * w[n * K + k];
        out[m * N + n] = oracle_f32_to_bf16(acc);
      }
    }
  }
  free(w);
  return 0;
}
