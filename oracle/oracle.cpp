/*
 * oracle.cpp - plain, slow CPU oracle of the gated Indexer + Top-K sparse-attention layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the benchmark's
 * CPU-baseline leg may load this library.  It shares no code with the CUDA path
 * (no headers, helpers or tables); it reads the same seeded inputs.
 *
 * Pages cited (web articles on one model release):
 *   [HSA] "Hybrid Sparse Attention for Long-Context LLMs: How Linear Attention and
 *          Indexer + Top-K Work Together"
 *   [ITK] "Optimizing LLM Long-Context Inference with Indexed Top-K Sparse Attention"
 *   [FGS] "How Fine-Grained Sparse Attention Reshapes Long-Context Architecture in
 *          Large Models"
 *   [SAE] "Sparse Attention in Long-Context LLM Inference: Engineering Trade-offs and
 *          Architecture Choices"
 *   [GSA] "From Linear Attention to Gated Sparse Attention: Dissecting a Hybrid LLM
 *          Architecture Trade-off"
 *
 * Every step is the plain definition, written out in fp64:
 *   1. indexer score  s[t,j] = sum_h w_h * max(0, q_idx[t,h,:] . k_idx[j,h,:]),  j <= p(t)
 *      ([HSA] "Indexer + Top-K: How Fine-Grained Sparse Attention Works", step 1;
 *       [ITK] "Two Engineering Considerations", 1. Indexer Computational Cost.  The pages
 *       call the indexer lightweight and low-dimensional but give no formula; the
 *       per-head ReLU dot product with a weighted head sum is the reading used here.)
 *   2. Top-K: the K largest scores of the row, ties to the lower position; all
 *      positions when the row has <= K ([HSA] same section, step 2; [ITK]
 *      "Introducing Indexed Top-K Sparse Attention", Top-K Selection Stage).
 *      Block granularity ([HSA] same section, steps 1-2: positions "or blocks"): the
 *      score of block m (positions mB .. mB+B-1 up to p) is the largest score of its
 *      positions, the K blocks with the largest scores are kept (ties to the lower block;
 *      all blocks when the row has <= K), and their positions are the selection.
 *   3. exact softmax attention over the selected rows only, scale 1/sqrt(d)
 *      ([HSA] same section, step 3 and its pseudocode; [SAE] "5. Abstract
 *       Implementation Sketch of Indexer + Top-K").
 *   4. sigmoid output gate, per head and dimension: out = sigmoid(g) * o
 *      ([HSA] same section, step 4; [GSA] "2. The Core Change", pseudocode), or, with
 *      the layer's second branch o2 (the linear / compressed-context output),
 *      out = sigmoid(g) * o + (1 - sigmoid(g)) * o2 ([HSA] same section, step 4 and the
 *      last line of its pseudocode; [FGS] "How Indexer + Top-K Works at Runtime",
 *      step 3 "Fuse" of its pseudocode).
 * Parity is pinned by the tests against brute force, closed forms and library
 * routines (dense causal attention when K covers the whole history).
 */
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <thread>
#include <utility>
#include <vector>

extern "C" {

typedef struct {
  int32_t batch;
  const int64_t* q_off;   /* [batch+1] host prefix offsets of query rows        */
  const int64_t* kv_off;  /* [batch+1] host prefix offsets of cache rows        */
  int32_t n_idx_heads;    /* H_i */
  int32_t idx_dim;        /* D_i */
  int32_t n_q_heads;      /* Hq  */
  int32_t n_kv_heads;     /* Hkv */
  int32_t head_dim;       /* d   */
  int32_t top_k;          /* K   */
  int32_t idx_is_fp8;     /* indexer tensors are e4m3 bytes instead of bf16 bits */
  double idx_scale_q;     /* dequantisation scales of the indexer tensors */
  double idx_scale_k;
  double attn_scale;      /* <= 0 means 1/sqrt(d) */
  int32_t w_row_stride;   /* 0: w[h] shared by all rows; else w[row*stride + h] */
} oracle_problem;

}  // extern "C"

namespace {

double bf16_value(uint16_t bits) {
  uint32_t u = (uint32_t)bits << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return (double)f;
}

/* OCP fp8 e4m3: 1 sign, 4 exponent (bias 7), 3 mantissa bits; no infinities. */
double e4m3_value(uint8_t c) {
  int sign = c >> 7, e = (c >> 3) & 15, m = c & 7;
  double mag;
  if (e == 0) mag = std::ldexp((double)m / 8.0, -6);
  else if (e == 15 && m == 7) mag = NAN;
  else mag = std::ldexp(1.0 + (double)m / 8.0, e - 7);
  return sign ? -mag : mag;
}

int seq_of_row(const oracle_problem* P, int64_t r) {
  int b = 0;
  while (b + 1 <= P->batch && P->q_off[b + 1] <= r) ++b;
  return b;
}

/* absolute position of packed query row r inside its sequence */
int64_t position_of_row(const oracle_problem* P, int64_t r, int* seq) {
  int b = seq_of_row(P, r);
  int64_t L = P->kv_off[b + 1] - P->kv_off[b];
  int64_t Q = P->q_off[b + 1] - P->q_off[b];
  if (seq) *seq = b;
  return L - Q + (r - P->q_off[b]);
}

double idx_elem(const oracle_problem* P, const void* base, int64_t i, double scale) {
  if (P->idx_is_fp8) return e4m3_value(((const uint8_t*)base)[i]) * scale;
  return bf16_value(((const uint16_t*)base)[i]) * scale;
}

}  // namespace

extern "C" {

/* Step 1: indexer scores of packed query row r, s[j] for j = 0..p (returns n = p+1). */
int64_t oracle_index_scores_row(const oracle_problem* P, const void* q_idx, const void* k_idx,
                                const float* w, int64_t r, double* s) {
  int b = 0;
  int64_t p = position_of_row(P, r, &b);
  const int Hi = P->n_idx_heads, Di = P->idx_dim;
  for (int64_t j = 0; j <= p; ++j) {
    double total = 0.0;
    for (int h = 0; h < Hi; ++h) {
      double dot = 0.0;
      for (int e = 0; e < Di; ++e) {
        double a = idx_elem(P, q_idx, (r * Hi + h) * (int64_t)Di + e, P->idx_scale_q);
        double c = idx_elem(P, k_idx, ((P->kv_off[b] + j) * Hi + h) * (int64_t)Di + e,
                            P->idx_scale_k);
        dot += a * c;
      }
      double wh = P->w_row_stride ? (double)w[r * P->w_row_stride + h] : (double)w[h];
      total += wh * (dot > 0.0 ? dot : 0.0);
    }
    s[j] = total;
  }
  return p + 1;
}

/* Step 2: the K best (score desc, position asc) of s[0..n), written in ascending
 * position order, padded with -1 up to K.  Returns the number selected. */
int32_t oracle_topk_row(const double* s, int64_t n, int32_t K, int32_t* idx) {
  std::vector<std::pair<double, int64_t>> items((size_t)n);
  for (int64_t j = 0; j < n; ++j) items[(size_t)j] = {s[j] == 0.0 ? 0.0 : s[j], j};
  std::sort(items.begin(), items.end(), [](const auto& a, const auto& b) {
    if (a.first != b.first) return a.first > b.first;
    return a.second < b.second;
  });
  int64_t take = n < (int64_t)K ? n : (int64_t)K;
  std::vector<int32_t> chosen((size_t)take);
  for (int64_t i = 0; i < take; ++i) chosen[(size_t)i] = (int32_t)items[(size_t)i].second;
  std::sort(chosen.begin(), chosen.end());
  for (int32_t i = 0; i < K; ++i) idx[i] = i < take ? chosen[(size_t)i] : -1;
  return (int32_t)take;
}

/* Step 2 at block granularity: s[0..n) one row's scores, blocks of B positions (the last
 * one partial), Kb blocks kept.  idx receives the selected positions in ascending order,
 * then -1 up to Kb * B.  Returns the number of positions selected. */
int32_t oracle_block_topk_row(const double* s, int64_t n, int32_t B, int32_t Kb, int32_t* idx) {
  const int64_t nb = (n + B - 1) / B;
  std::vector<std::pair<double, int64_t>> blocks((size_t)nb);
  for (int64_t m = 0; m < nb; ++m) {
    double best = s[m * B];
    for (int64_t j = m * B + 1; j < n && j < (m + 1) * B; ++j)
      if (s[j] > best) best = s[j];
    blocks[(size_t)m] = {best == 0.0 ? 0.0 : best, m};  // -0.0 counts as +0.0
  }
  std::sort(blocks.begin(), blocks.end(), [](const std::pair<double, int64_t>& x,
                                             const std::pair<double, int64_t>& y) {
    if (x.first != y.first) return x.first > y.first;
    return x.second < y.second;
  });
  const int64_t take = nb < (int64_t)Kb ? nb : (int64_t)Kb;
  std::vector<int64_t> chosen((size_t)take);
  for (int64_t i = 0; i < take; ++i) chosen[(size_t)i] = blocks[(size_t)i].second;
  std::sort(chosen.begin(), chosen.end());
  int32_t w = 0;
  for (int64_t m : chosen)
    for (int64_t j = m * B; j < n && j < (m + 1) * B; ++j) idx[w++] = (int32_t)j;
  const int32_t total = w;
  while (w < Kb * B) idx[w++] = -1;
  return total;
}

/* Steps 3-4: gated exact softmax attention of packed query row r over the cache rows
 * idx[0..K) (entries < 0 are padding).  out is [Hq, d]; lse (nullable) is [Hq] and
 * holds log(sum_j exp(scale * q.k_j)).  gate may be NULL (no gate). */
void oracle_sparse_attn_row(const oracle_problem* P, const uint16_t* q, const uint16_t* k,
                            const uint16_t* v, const uint16_t* gate, const int32_t* idx,
                            int64_t r, double* out, double* lse) {
  int b = 0;
  position_of_row(P, r, &b);
  const int Hq = P->n_q_heads, Hkv = P->n_kv_heads, d = P->head_dim, K = P->top_k;
  const int G = Hq / Hkv;
  const double scale = P->attn_scale > 0 ? P->attn_scale : 1.0 / std::sqrt((double)d);
  std::vector<int64_t> rows;
  for (int i = 0; i < K; ++i)
    if (idx[i] >= 0) rows.push_back(P->kv_off[b] + idx[i]);
  std::vector<double> logit(rows.size());
  for (int h = 0; h < Hq; ++h) {
    const int g = h / G;
    const uint16_t* qh = q + (r * Hq + h) * (int64_t)d;
    double m = -INFINITY;
    for (size_t i = 0; i < rows.size(); ++i) {
      const uint16_t* kr = k + (rows[i] * Hkv + g) * (int64_t)d;
      double dot = 0.0;
      for (int e = 0; e < d; ++e) dot += bf16_value(qh[e]) * bf16_value(kr[e]);
      logit[i] = scale * dot;
      if (logit[i] > m) m = logit[i];
    }
    std::vector<double> prob(rows.size());
    double l = 0.0;
    for (size_t i = 0; i < rows.size(); ++i) {
      prob[i] = std::exp(logit[i] - m);
      l += prob[i];
    }
    for (int e = 0; e < d; ++e) {
      double acc = 0.0;
      for (size_t i = 0; i < rows.size(); ++i)
        acc += prob[i] * bf16_value(v[(rows[i] * Hkv + g) * (int64_t)d + e]);
      double o = rows.empty() ? 0.0 : acc / l;
      if (gate) {
        double gl = bf16_value(gate[(r * Hq + h) * (int64_t)d + e]);
        o = o * (1.0 / (1.0 + std::exp(-gl)));
      }
      out[(int64_t)h * d + e] = o;
    }
    if (lse) lse[h] = rows.empty() ? -INFINITY : m + std::log(l);
  }
}

/* Step 4 with the second branch: out[e] = s * o[e] + (1 - s) * o2[e], s = sigmoid(gate[e]),
 * over the n elements of one query row ([Hq, d]): o is the row's ungated attention output
 * (oracle_sparse_attn_row with gate NULL), gate and o2 the row's bf16 logits and second-
 * branch values. */
void oracle_gate_mix(const double* o, const uint16_t* gate, const uint16_t* o2, int64_t n,
                     double* out) {
  for (int64_t e = 0; e < n; ++e) {
    const double s = 1.0 / (1.0 + std::exp(-bf16_value(gate[e])));
    out[e] = s * o[e] + (1.0 - s) * bf16_value(o2[e]);
  }
}

/* The whole layer for a list of packed query rows, one thread per row at a time.
 * idx_out [nrows, K], out [nrows, Hq, d], lse [nrows, Hq] (nullable). */
void oracle_layer_rows(const oracle_problem* P, const void* q_idx, const void* k_idx,
                       const float* w, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                       const uint16_t* gate, const int64_t* rows, int64_t nrows,
                       int32_t nthreads, int32_t* idx_out, double* out, double* lse) {
  const int K = P->top_k, Hq = P->n_q_heads, d = P->head_dim;
  if (nthreads < 1) nthreads = 1;
  auto work = [&](int tid) {
    std::vector<double> s;
    for (int64_t i = tid; i < nrows; i += nthreads) {
      int64_t r = rows[i];
      int b = 0;
      int64_t p = position_of_row(P, r, &b);
      s.assign((size_t)(p + 1), 0.0);
      int64_t n = oracle_index_scores_row(P, q_idx, k_idx, w, r, s.data());
      oracle_topk_row(s.data(), n, K, idx_out + i * K);
      oracle_sparse_attn_row(P, q, k, v, gate, idx_out + i * K, r, out + i * (int64_t)Hq * d,
                             lse ? lse + i * Hq : nullptr);
    }
  };
  std::vector<std::thread> pool;
  for (int t = 1; t < nthreads; ++t) pool.emplace_back(work, t);
  work(0);
  for (auto& th : pool) th.join();
}

int32_t oracle_hardware_threads(void) {
  unsigned n = std::thread::hardware_concurrency();
  return n ? (int32_t)n : 1;
}

}  // extern "C"
