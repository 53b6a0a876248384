/*
 * oracle/moe_oracle.cpp -- plain, slow CPU oracle of one MoE layer.
 *
 * TEST INFRASTRUCTURE. Only the tests, the smoke check and the benchmark's CPU
 * baseline load this library. It shares no code, header, table or helper with
 * the CUDA path (combine_warp_top_expert_b200/), and the CUDA path never calls it.
 *
 * Each function is the plain definition of one step, written as loops in the
 * order the tutorial page "Expert Parallelism" (learning-materials, inference
 * engineering IX.05) states the step, with fp64 arithmetic wherever floating
 * point is involved. bf16 inputs are upcast exactly (bits << 16). Readings of
 * points the page leaves open are marked [reading].
 *
 * Pins (tests/test_oracle_pins.py) tie every function to something other than
 * itself: brute-force top-k over all subsets, the page's worked imbalance
 * example (140/64), closed forms, the identity-expert and one-expert cases and
 * a numpy dense SwiGLU.
 */
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <limits>
#include <numeric>
#include <vector>

namespace {

double bf16_to_double(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  std::memcpy(&f, &u, sizeof f);
  return (double)f;
}

float bf16_to_float(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  std::memcpy(&f, &u, sizeof f);
  return f;
}

/* [reading] a NaN logit orders as -inf */
double order_key(float l) { return std::isnan(l) ? -std::numeric_limits<double>::infinity() : (double)l; }

}  // namespace

extern "C" {

/*
 * Router top-k and gates. Page "Expert Parallelism" §1: each token is routed to
 * k of the E experts; §4: the router's output names, per token, the experts it
 * goes to.
 *   Order the E experts of token t by (logit descending, index ascending): expert
 *   a comes before b iff l_a > l_b, or l_a == l_b and a < b (IEEE compare, so
 *   -0.0 == +0.0). topk_idx[t][j] is the j-th expert in that order.
 *   [reading] the page gives no gate formula, only that combine weights the k
 *   expert outputs: the gates are the softmax over the k selected logits,
 *   g_j = exp(l_j - l_0) / sum_i exp(l_i - l_0), in fp64, rounded to fp32;
 *   g_j = 1/k if l_0 = -inf.
 * Returns the number of NaN logits seen.
 */
int64_t oracle_route(int64_t T, int32_t E, int32_t k, const float* logits, int32_t* topk_idx, float* topk_gate) {
  int64_t nan_count = 0;
  std::vector<int32_t> order(E);
  for (int64_t t = 0; t < T; ++t) {
    const float* l = logits + t * E;
    for (int32_t e = 0; e < E; ++e) nan_count += std::isnan(l[e]) ? 1 : 0;
    std::iota(order.begin(), order.end(), 0);
    std::sort(order.begin(), order.end(), [&](int32_t a, int32_t b) {
      const double ka = order_key(l[a]), kb = order_key(l[b]);
      return ka > kb || (ka == kb && a < b);
    });
    for (int32_t j = 0; j < k; ++j) topk_idx[t * k + j] = order[j];
    const double l0 = order_key(l[order[0]]);
    if (l0 == -std::numeric_limits<double>::infinity()) {
      for (int32_t j = 0; j < k; ++j) topk_gate[t * k + j] = (float)(1.0 / (double)k);
      continue;
    }
    double s = 0.0;
    for (int32_t j = 0; j < k; ++j) s += std::exp(order_key(l[order[j]]) - l0);
    for (int32_t j = 0; j < k; ++j) topk_gate[t * k + j] = (float)(std::exp(order_key(l[order[j]]) - l0) / s);
  }
  return nan_count;
}

/*
 * Dispatch bookkeeping. Page "Expert Parallelism" §4 DISPATCH:
 *   step 1 orders the tokens by the expert they go to (and so by GPU),
 *   step 2 counts the tokens per GPU,
 *   step 4 leaves every GPU with one contiguous run of tokens per expert it owns
 * and §1 (experts placed on GPUs in contiguous blocks: GPU 0 holds 0-15, ...).
 *   Assignment a = t*k + j goes to expert e = topk_idx[a] (entries outside
 *   [0, E) are skipped, counted, and get assign_row = -1).
 *   Rows are handed out in assignment order: a takes row offsets[e] + (number of
 *   earlier assignments to e). [reading] the page asks for a sort without an order
 *   inside an expert; keeping assignment order is the plainest stable reading.
 *   Capacity, page §5 "Mitigations" 1 (capacity factor): when capacity > 0 an
 *   expert keeps only its first `capacity` assignments in that order; the rest
 *   are dropped (assign_row = -1: the dropped assignment skips its expert and
 *   only the residual path carries the token).
 *   counts[e] = assignments kept by e; offsets = exclusive scan of counts,
 *   offsets[E] = total kept.
 *   Logical rank r owns experts [r*E/R, (r+1)*E/R): rank_counts[r] = sum of its
 *   experts' counts, rank_offsets[r] = offsets[r*E/R].
 *   Imbalance, page §5: the most loaded GPU against the ideal, 140/64 in the
 *   worked example: imbalance[0] = max_r rank_counts[r] / (total / R),
 *   imbalance[1] = max_e counts[e] / (total / E), each computed as
 *   (double)(max * R) / (double)total rounded once to fp32 (exact integers, so
 *   this is the correctly rounded quotient for total < 2^28); {1, 1} if total = 0.
 * Returns the number of skipped (out-of-range) entries; *dropped (if not null)
 * receives the number of assignments dropped by the capacity.
 */
int64_t oracle_dispatch_capacity(int64_t T, int32_t E, int32_t k, int32_t R, int32_t capacity,
                                 const int32_t* topk_idx, int32_t* counts, int32_t* offsets, int32_t* rank_counts,
                                 int32_t* rank_offsets, int32_t* row_src, int32_t* assign_row, float* imbalance,
                                 int64_t* dropped) {
  const int64_t A = T * (int64_t)k;
  int64_t bad = 0, drop = 0;
  /* first pass: which assignments each expert keeps, in assignment order */
  std::vector<int32_t> seen(E, 0);
  std::vector<char> keep(A, 0);
  for (int64_t a = 0; a < A; ++a) {
    const int32_t e = topk_idx[a];
    if (e < 0 || e >= E) {
      ++bad;
      continue;
    }
    if (capacity > 0 && seen[e] >= capacity) {
      ++drop;
    } else {
      keep[a] = 1;
    }
    seen[e] += 1;
  }
  for (int32_t e = 0; e < E; ++e) counts[e] = 0;
  for (int64_t a = 0; a < A; ++a)
    if (keep[a]) counts[topk_idx[a]] += 1;
  offsets[0] = 0;
  for (int32_t e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + counts[e];
  std::vector<int32_t> cursor(E, 0);
  for (int64_t a = 0; a < A; ++a) {
    if (!keep[a]) {
      assign_row[a] = -1;
      continue;
    }
    const int32_t e = topk_idx[a];
    const int32_t p = offsets[e] + cursor[e]++;
    row_src[p] = (int32_t)a;
    assign_row[a] = p;
  }
  for (int64_t p = offsets[E]; p < A; ++p) row_src[p] = -1;
  const int32_t per_rank = E / R;
  for (int32_t r = 0; r < R; ++r) {
    rank_offsets[r] = offsets[r * per_rank];
    int32_t c = 0;
    for (int32_t e = r * per_rank; e < (r + 1) * per_rank; ++e) c += counts[e];
    rank_counts[r] = c;
  }
  rank_offsets[R] = offsets[E];
  const int64_t total = offsets[E];
  if (total == 0) {
    imbalance[0] = 1.0f;
    imbalance[1] = 1.0f;
  } else {
    int64_t max_r = 0, max_e = 0;
    for (int32_t r = 0; r < R; ++r) max_r = std::max<int64_t>(max_r, rank_counts[r]);
    for (int32_t e = 0; e < E; ++e) max_e = std::max<int64_t>(max_e, counts[e]);
    imbalance[0] = (float)((double)(max_r * R) / (double)total);
    imbalance[1] = (float)((double)(max_e * E) / (double)total);
  }
  if (dropped) *dropped = drop;
  return bad;
}

/* Dispatch with no capacity limit. */
int64_t oracle_dispatch(int64_t T, int32_t E, int32_t k, int32_t R, const int32_t* topk_idx, int32_t* counts,
                        int32_t* offsets, int32_t* rank_counts, int32_t* rank_offsets, int32_t* row_src,
                        int32_t* assign_row, float* imbalance) {
  return oracle_dispatch_capacity(T, E, k, R, 0, topk_idx, counts, offsets, rank_counts, rank_offsets, row_src,
                                  assign_row, imbalance, nullptr);
}

/* Dispatch data movement, page §4 DISPATCH step 3 (the token rows are exchanged):
 * x_perm[p] = x[row_src[p] / k] for every filled row p (bit copy). */
void oracle_permute_rows(int64_t n_rows, int32_t k, int32_t d, const uint16_t* x, const int32_t* row_src,
                         uint16_t* x_perm) {
  for (int64_t p = 0; p < n_rows; ++p) {
    if (row_src[p] < 0) continue;
    const int64_t t = row_src[p] / k;
    std::memcpy(x_perm + p * d, x + t * d, (size_t)d * sizeof(uint16_t));
  }
}

/*
 * One expert's SwiGLU FFN on n rows. Page §1 (a layer holds E expert FFNs);
 * [reading] the FFN is SwiGLU: with W_gate = w13[0:f], W_up = w13[f:2f],
 *   a = W_gate x, b = W_up x, h = silu(a) * b, silu(a) = a / (1 + e^-a), y = W2 h,
 * all in fp64 with no intermediate rounding.
 *   xrows [n, d] bf16, w13 [2f, d] bf16, w2 [d, f] bf16 -> y [n, d] fp64.
 */
void oracle_swiglu(int64_t n, int32_t d, int32_t f, const uint16_t* xrows, const uint16_t* w13, const uint16_t* w2,
                   double* y) {
  if (n <= 0) return;
  std::vector<float> w13f((size_t)2 * f * d), w2f((size_t)d * f);
  for (size_t i = 0; i < w13f.size(); ++i) w13f[i] = bf16_to_float(w13[i]);
  for (size_t i = 0; i < w2f.size(); ++i) w2f[i] = bf16_to_float(w2[i]);
#pragma omp parallel
  {
    std::vector<double> xr(d), h(f);
#pragma omp for schedule(dynamic, 1)
    for (int64_t r = 0; r < n; ++r) {
      for (int32_t i = 0; i < d; ++i) xr[i] = bf16_to_double(xrows[r * d + i]);
      for (int32_t j = 0; j < f; ++j) {
        const float* wg = &w13f[(size_t)j * d];
        const float* wu = &w13f[(size_t)(f + j) * d];
        double a = 0.0, b = 0.0;
        for (int32_t i = 0; i < d; ++i) {
          a += (double)wg[i] * xr[i];
          b += (double)wu[i] * xr[i];
        }
        h[j] = a / (1.0 + std::exp(-a)) * b;
      }
      for (int32_t o = 0; o < d; ++o) {
        const float* wd = &w2f[(size_t)o * f];
        double acc = 0.0;
        for (int32_t j = 0; j < f; ++j) acc += (double)wd[j] * h[j];
        y[r * d + o] = acc;
      }
    }
  }
}

/*
 * Expert compute, page §4 COMPUTE (every expert multiplies its own tokens): the rows
 * [offsets[e], offsets[e+1]) of x_perm go through expert e's FFN, written to the
 * same rows of y_perm. [reading] a shared expert (n_shared = 1) applies its own
 * SwiGLU FFN to every token of x, into y_shared.
 */
void oracle_expert_ffn(int64_t T, int32_t d, int32_t E, int32_t f, int32_t n_shared, const uint16_t* x_perm,
                       const int32_t* offsets, const uint16_t* w13, const uint16_t* w2, const uint16_t* x,
                       const uint16_t* w13s, const uint16_t* w2s, double* y_perm, double* y_shared) {
  for (int32_t e = 0; e < E; ++e) {
    const int64_t r0 = offsets[e], r1 = offsets[e + 1];
    oracle_swiglu(r1 - r0, d, f, x_perm + r0 * d, w13 + (size_t)e * 2 * f * d, w2 + (size_t)e * d * f,
                  y_perm + r0 * d);
  }
  if (n_shared) oracle_swiglu(T, d, f, x, w13s, w2s, y_shared);
}

/*
 * Combine, page §4 COMBINE: expert outputs return in the original token order
 * and each token's k outputs are summed with its gate weights.
 *   out[t] = sum_{j<k} gate[t][j] * y_perm[assign_row[t*k+j]] (+ y_shared[t]), fp64,
 *   j in increasing order; a skipped assignment (assign_row < 0) adds nothing.
 */
void oracle_combine(int64_t T, int32_t k, int32_t d, const double* y_perm, const int32_t* assign_row,
                    const float* gate, const double* y_shared, double* out) {
  for (int64_t t = 0; t < T; ++t) {
    double* o = out + t * d;
    for (int32_t c = 0; c < d; ++c) o[c] = 0.0;
    for (int32_t j = 0; j < k; ++j) {
      const int64_t p = assign_row[t * k + j];
      if (p < 0) continue;
      const double g = (double)gate[t * k + j];
      for (int32_t c = 0; c < d; ++c) o[c] += g * y_perm[p * d + c];
    }
    if (y_shared)
      for (int32_t c = 0; c < d; ++c) o[c] += y_shared[t * d + c];
  }
}

/* The unsorted per-token loop of the page's hands-on exercise C (§10): no sort,
 * each token visits its k experts directly. Same result as dispatch -> FFN ->
 * combine; used as an independent cross-check of the sorted path. */
void oracle_naive_token_loop(int64_t T, int32_t d, int32_t E, int32_t k, int32_t f, int32_t n_shared,
                             const uint16_t* x, const int32_t* topk_idx, const float* gate, const uint16_t* w13,
                             const uint16_t* w2, const uint16_t* w13s, const uint16_t* w2s, double* out) {
  std::vector<double> y(d);
  for (int64_t t = 0; t < T; ++t) {
    double* o = out + t * d;
    for (int32_t c = 0; c < d; ++c) o[c] = 0.0;
    for (int32_t j = 0; j < k; ++j) {
      const int32_t e = topk_idx[t * k + j];
      if (e < 0 || e >= E) continue;
      oracle_swiglu(1, d, f, x + t * d, w13 + (size_t)e * 2 * f * d, w2 + (size_t)e * d * f, y.data());
      for (int32_t c = 0; c < d; ++c) o[c] += (double)gate[t * k + j] * y[c];
    }
    if (n_shared) {
      oracle_swiglu(1, d, f, x + t * d, w13s, w2s, y.data());
      for (int32_t c = 0; c < d; ++c) o[c] += y[c];
    }
  }
}

}  // extern "C"
