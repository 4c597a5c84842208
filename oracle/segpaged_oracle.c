/*
 * segpaged_oracle.c -- TEST INFRASTRUCTURE, not part of the product.
 *
 * A plain, slow fp64 CPU statement of what SegPagedAttention prefill computes. Only the
 * test suite, the smoke check and the benchmark's CPU-baseline leg may load this file's
 * library; the product path never does. It shares no code, header or table with the
 * CUDA library (head_sparse_paged_b200/csrc).
 *
 * What it computes, per sequence b, query head h and query position i in [L_b - Lq_b, L_b),
 * with KV head k = h / G (G = Hq / Hkv, contiguous grouping as in grouped-query attention):
 *
 *   V(i)  = { j : 0 <= j <= i }                              if KV head k of sequence b is global
 *         = { j : 0 <= j <= i  and ( j < S  or  j > i - W ) } if it is local (sink S, window W)
 *   s_j   = scale * sum_d q[i,h,d] * K[j,k,d]        (+ an optional test shift c, same for all j)
 *   LSE_i = ln sum_{j in V(i)} exp(s_j)
 *   O_i   = sum_{j in V(i)} exp(s_j - LSE_i) * V[j,k,:]
 *
 * Sources: global heads see the full causal context and local heads keep only their sink
 * tokens and recent window ("RedKnot" write-up on bjdmk.com.cn, section 二 "三大核心机制",
 * item 3 "SegPagedAttention"; shshi.cn "RedKnot技术原理" 1 "SegPagedAttention存储架构").
 * The pages name the sink and the window but print no boundaries; the sink-plus-window rule
 * above (window of W tokens ending at the query itself, sink = the first S tokens, never a
 * future token) is the reading this project takes. The kernel is exact attention over that
 * visible set, so this definition is the whole oracle: no paging, no tiling.
 *
 * V(i) is formed here by scanning every key j of the sequence and testing the predicate
 * directly (brute force). The numpy oracle (reference.py) builds the same set from index
 * ranges instead, and the tests require the two to agree.
 *
 * Inputs are float32 arrays that hold bf16-representable values; all arithmetic is double.
 * Softmax is the naive two-pass form: max, then sum of exponentials.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

static int oracle_visible(int is_global, int sink, int window, int64_t i, int64_t j) {
  if (j < 0 || j > i) return 0;
  if (is_global) return 1;
  return (j < sink) || (j > i - window);
}

/*
 * Attention rows. items[2*t] = global query row r (index into q's first dimension),
 * items[2*t+1] = query head h. For each item t: o_out[t*D + d], lse_out[t].
 * shift (nullable, one value per item) is added to every visible logit of that row
 * (a test hook for the softmax shift invariance).
 * Returns 0, or -1 on a malformed item.
 */
int oracle_attention(int B, int Hq, int Hkv, int D,
                     const int32_t* cu_q, const int32_t* cu_k,
                     const int32_t* cls_global, const int32_t* cls_sink, const int32_t* cls_window,
                     const float* q, const float* k, const float* v,
                     const int64_t* items, int64_t n_items, double scale, const double* shift,
                     double* o_out, double* lse_out) {
  const int G = Hq / Hkv;
  int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
  for (int64_t t = 0; t < n_items; ++t) {
    const int64_t r = items[2 * t], h = items[2 * t + 1];
    int b = -1;
    for (int bb = 0; bb < B; ++bb)
      if (r >= cu_q[bb] && r < cu_q[bb + 1]) { b = bb; break; }
    if (b < 0 || h < 0 || h >= Hq) { bad |= 1; continue; }
    const int64_t L = cu_k[b + 1] - cu_k[b];
    const int64_t Lq = cu_q[b + 1] - cu_q[b];
    const int64_t i = L - Lq + (r - cu_q[b]);
    const int kh = (int)(h / G);
    const int cg = cls_global[b * Hkv + kh], cs = cls_sink[b * Hkv + kh], cw = cls_window[b * Hkv + kh];
    const float* qrow = q + (r * Hq + h) * (int64_t)D;
    double* s = (double*)malloc(sizeof(double) * (size_t)(L > 0 ? L : 1));
    double mx = -INFINITY;
    for (int64_t j = 0; j < L; ++j) {
      if (!oracle_visible(cg, cs, cw, i, j)) { s[j] = -INFINITY; continue; }
      const float* krow = k + ((cu_k[b] + j) * Hkv + kh) * (int64_t)D;
      double acc = 0.0;
      for (int d = 0; d < D; ++d) acc += (double)qrow[d] * (double)krow[d];
      s[j] = scale * acc + (shift ? shift[t] : 0.0);
      if (s[j] > mx) mx = s[j];
    }
    double sum = 0.0;
    for (int64_t j = 0; j < L; ++j)
      if (s[j] != -INFINITY) sum += exp(s[j] - mx);
    const double lse = mx + log(sum);
    lse_out[t] = lse;
    double* orow = o_out + t * (int64_t)D;
    for (int d = 0; d < D; ++d) orow[d] = 0.0;
    for (int64_t j = 0; j < L; ++j) {
      if (s[j] == -INFINITY) continue;
      const double p = exp(s[j] - lse);
      const float* vrow = v + ((cu_k[b] + j) * Hkv + kh) * (int64_t)D;
      for (int d = 0; d < D; ++d) orow[d] += p * (double)vrow[d];
    }
    free(s);
  }
  return bad ? -1 : 0;
}

/*
 * Probability row of one item: p_out[j] for j in [0, L_b), zero outside V(i).
 * Returns |V(i)|, or -1 on a malformed item.
 */
int64_t oracle_probs(int B, int Hq, int Hkv, int D, const int32_t* cu_q, const int32_t* cu_k,
                     const int32_t* cls_global, const int32_t* cls_sink, const int32_t* cls_window,
                     const float* q, const float* k, int64_t r, int64_t h, double scale, double* p_out) {
  const int G = Hq / Hkv;
  int b = -1;
  for (int bb = 0; bb < B; ++bb)
    if (r >= cu_q[bb] && r < cu_q[bb + 1]) { b = bb; break; }
  if (b < 0 || h < 0 || h >= Hq) return -1;
  const int64_t L = cu_k[b + 1] - cu_k[b];
  const int64_t i = L - (cu_q[b + 1] - cu_q[b]) + (r - cu_q[b]);
  const int kh = (int)(h / G);
  const int cg = cls_global[b * Hkv + kh], cs = cls_sink[b * Hkv + kh], cw = cls_window[b * Hkv + kh];
  const float* qrow = q + (r * Hq + h) * (int64_t)D;
  double mx = -INFINITY;
  int64_t n = 0;
  for (int64_t j = 0; j < L; ++j) {
    if (!oracle_visible(cg, cs, cw, i, j)) { p_out[j] = -INFINITY; continue; }
    const float* krow = k + ((cu_k[b] + j) * Hkv + kh) * (int64_t)D;
    double acc = 0.0;
    for (int d = 0; d < D; ++d) acc += (double)qrow[d] * (double)krow[d];
    p_out[j] = scale * acc;
    if (p_out[j] > mx) mx = p_out[j];
    ++n;
  }
  double sum = 0.0;
  for (int64_t j = 0; j < L; ++j)
    if (p_out[j] != -INFINITY) sum += exp(p_out[j] - mx);
  for (int64_t j = 0; j < L; ++j) p_out[j] = (p_out[j] == -INFINITY) ? 0.0 : exp(p_out[j] - mx) / sum;
  return n;
}

/*
 * Attention mass each token of the query range receives in the prefill (the token score of the
 * sparse-FFN selection: "RedKnot技术原理" 3 "稀疏FFN动态调度", shshi.cn; the reading of "attention
 * score" as mass received is this project's, as the pages do not define it):
 *
 *   mass_out[r] = sum over query heads h and query rows r' of the same sequence, at position i,
 *                 with j in V_h(i), of exp(s_hij - LSE_hi),
 *
 * where j is the position of query row r. Every LSE is formed first (two-pass, brute-force visible
 * set), then every sum. Returns 0.
 */
int oracle_token_mass(int B, int Hq, int Hkv, int D, const int32_t* cu_q, const int32_t* cu_k,
                      const int32_t* cls_global, const int32_t* cls_sink, const int32_t* cls_window,
                      const float* q, const float* k, double scale, double* mass_out) {
  const int G = Hq / Hkv;
  for (int b = 0; b < B; ++b) {
    const int64_t L = cu_k[b + 1] - cu_k[b], Lq = cu_q[b + 1] - cu_q[b], q0 = L - Lq;
    if (Lq <= 0) continue;
    double* lse = (double*)malloc(sizeof(double) * (size_t)(Lq * Hq));
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t t = 0; t < Lq * Hq; ++t) {
      const int64_t rr = t / Hq, h = t % Hq, i = q0 + rr;
      const int kh = (int)(h / G);
      const int cg = cls_global[b * Hkv + kh], cs = cls_sink[b * Hkv + kh], cw = cls_window[b * Hkv + kh];
      const float* qrow = q + ((cu_q[b] + rr) * Hq + h) * (int64_t)D;
      double mx = -INFINITY, sum = 0.0;
      for (int pass = 0; pass < 2; ++pass)
        for (int64_t j = 0; j < L; ++j) {
          if (!oracle_visible(cg, cs, cw, i, j)) continue;
          const float* krow = k + ((cu_k[b] + j) * Hkv + kh) * (int64_t)D;
          double acc = 0.0;
          for (int d = 0; d < D; ++d) acc += (double)qrow[d] * (double)krow[d];
          const double s = scale * acc;
          if (pass == 0) {
            if (s > mx) mx = s;
          } else {
            sum += exp(s - mx);
          }
        }
      lse[t] = mx + log(sum);
    }
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < Lq; ++r) {
      const int64_t j = q0 + r;
      double m = 0.0;
      for (int64_t rr = 0; rr < Lq; ++rr) {
        const int64_t i = q0 + rr;
        for (int h = 0; h < Hq; ++h) {
          const int kh = h / G;
          if (!oracle_visible(cls_global[b * Hkv + kh], cls_sink[b * Hkv + kh], cls_window[b * Hkv + kh], i, j))
            continue;
          const float* qrow = q + ((cu_q[b] + rr) * Hq + h) * (int64_t)D;
          const float* krow = k + ((cu_k[b] + j) * Hkv + kh) * (int64_t)D;
          double acc = 0.0;
          for (int d = 0; d < D; ++d) acc += (double)qrow[d] * (double)krow[d];
          m += exp(scale * acc - lse[rr * Hq + h]);
        }
      }
      mass_out[cu_q[b] + r] = m;
    }
    free(lse);
  }
  return 0;
}
