// Reference oracle for the DSA (sparse-attention) layer: lightning-indexer
// score, top-k token selection, attention over the selected cache rows.
//
// TEST INFRASTRUCTURE ONLY. Nothing in the product library calls, links or
// loads this file; only the tests, the package's smoke check and the CPU
// baseline leg of the benchmark do. It shares no code, header, table or helper
// with the CUDA path.
//
// It is written as the plain definition of what the layer computes, in double
// precision, one query at a time, with no blocking, fusion or reordering:
//
//   * "Lightning indexer" scoring of every earlier cached token
//     (llama.cpp b12180 news, aiaulis.com, paragraph 2; aiunderstanding.org,
//     "What happened"; devotd.net section 1 and its configuration table:
//     32 indexer heads, key length 128, no RoPE).  The pages do not print the
//     formula; the form used here is the usual lightning-indexer form
//         I[q,s] = sum_h w[q,h] * ReLU( sum_j q_idx[q,h,j] * k_idx[s,j] )
//     taken as an assumption (parity of this form against the real model is
//     unpinned: no weights and no published scores exist).
//   * Top-k selection of the highest-scoring tokens, k = 2048 in the released
//     checkpoint (devotd.net configuration table; aiaulis.com paragraph 3).
//     Ties are broken by score descending, then position ascending.
//   * Attention only over the selected rows of the key-only latent cache
//     (aiaulis.com paragraph 4; devotd.net section 2): K is the whole 576-wide
//     row, V is its first 512 entries, scale 1/sqrt(576) supplied by the caller.
//   * With top_k >= the number of causal positions the layer is full causal
//     attention (aiaulis.com paragraph 7; aiunderstanding.org "What happened";
//     devotd.net section 4).  oracle_full_causal_attn states that case with no
//     indexer code at all.
//   * The indexer's input step: the three indexer tensors named on the pages
//     (q_b, k and the head-weight projection; aiunderstanding.org "What
//     happened"; devotd.net section 3 -- kept out of quantization, so bf16
//     here) are plain linear maps of each new token: q_idx = c_q . W_q_b^T
//     from the token's query latent c_q, k = x . W_k^T and w = x . W_proj^T
//     from its hidden state x; k is appended to the indexer key cache at the
//     token's own row (devotd.net section 2: the indexer keeps a key cache).
//     The pages give no widths for x and c_q, and no normalisation or
//     scaling; none is applied.
//
// Conventions shared with the header of the product library (restated here,
// not included): sequence b owns query rows [q_off[b], q_off[b+1]) and cache
// rows starting at kv_off[b]; its context holds L_b = ctx_lens[b] rows, and the
// j-th query of the sequence sits at position p = L_b - nq_b + j and sees
// positions 0..p (its own row included).  bf16 values arrive as raw uint16
// bit patterns.  Outputs outside the computed rows are left untouched.

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <vector>
#ifdef _OPENMP
#include <omp.h>
#endif

namespace {

// Planted-mistake switch used only by the oracle's own mutation tests, which
// check that the pins catch each kind of error.  0 = the oracle as written.
int g_fault = 0;

double bf16_to_double(uint16_t bits) {
  uint32_t u = static_cast<uint32_t>(bits) << 16;
  float f;
  std::memcpy(&f, &u, sizeof f);
  return static_cast<double>(f);
}

struct Row {
  int64_t row;     // global query row
  int b;           // sequence
  int64_t pos;     // position p of the query inside its sequence
  int64_t kv0;     // first cache row of the sequence
};

// Lists the query rows to compute: all rows, or the caller's sample.
std::vector<Row> plan_rows(int B, const int32_t* q_off, const int64_t* kv_off,
                           const int32_t* ctx_lens, const int64_t* sample,
                           int64_t n_sample) {
  std::vector<Row> all;
  for (int b = 0; b < B; ++b) {
    const int64_t nq = q_off[b + 1] - q_off[b];
    for (int64_t j = 0; j < nq; ++j) {
      all.push_back({q_off[b] + j, b, ctx_lens[b] - nq + j, kv_off[b]});
    }
  }
  if (!sample) return all;
  std::vector<Row> out;
  out.reserve(static_cast<size_t>(n_sample));
  for (int64_t i = 0; i < n_sample; ++i) {
    for (const Row& r : all) {
      if (r.row == sample[i]) { out.push_back(r); break; }
    }
  }
  return out;
}

// Number of positions a query at position p sees: 0..p, its own row included.
int64_t causal_count(const Row& r) {
  return (g_fault == 3) ? r.pos : r.pos + 1;  // fault 3: strictly earlier rows only
}

// Index score of one query against positions 0..p, rounded once to fp32.
void score_row(const Row& r, int Hi, int Di, const uint16_t* q_idx, const float* w,
               const uint16_t* k_idx, float* out /* [p+1] */) {
  const int64_t n_pos = causal_count(r);
  for (int64_t s = 0; s < n_pos; ++s) {
    const uint16_t* k = k_idx + (r.kv0 + s) * Di;
    double I = 0.0;
    for (int h = 0; h < Hi; ++h) {
      const uint16_t* qh = q_idx + (r.row * Hi + h) * Di;
      double dot = 0.0;
      for (int j = 0; j < Di; ++j) dot += bf16_to_double(qh[j]) * bf16_to_double(k[j]);
      const double act = (g_fault == 1) ? dot : std::max(0.0, dot);  // fault 1: no ReLU
      I += static_cast<double>(w[r.row * Hi + h]) * act;
    }
    float f = static_cast<float>(I);  // round to nearest even
    if (f == 0.0f) f = 0.0f;          // -0 is the same score as +0
    out[s] = f;
  }
}

// The n_sel = min(k, p+1) positions that are largest by (score desc, pos asc),
// written in ascending position order and padded with -1 up to k.
void select_row(const float* sc, int64_t n_pos, int top_k, int32_t* idx) {
  std::vector<int32_t> order(static_cast<size_t>(n_pos));
  for (int64_t s = 0; s < n_pos; ++s) order[s] = static_cast<int32_t>(s);
  std::sort(order.begin(), order.end(), [&](int32_t a, int32_t b) {
    if (sc[a] != sc[b]) return sc[a] > sc[b];
    return (g_fault == 2) ? a > b : a < b;  // fault 2: ties to the later position
  });
  const int64_t n_sel = std::min<int64_t>(top_k, n_pos);
  std::sort(order.begin(), order.begin() + n_sel);
  for (int64_t i = 0; i < top_k; ++i) idx[i] = (i < n_sel) ? order[i] : -1;
}

// Softmax attention of one query (all heads) over an explicit list of
// sequence positions.  Logits, weights and the weighted sum stay in double.
void attend_row(const Row& r, int H, int D, int Dv, const uint16_t* q, const uint16_t* kv,
                const int32_t* pos, int64_t n, double scale, float* out, float* lse) {
  std::vector<double> logit(static_cast<size_t>(n));
  std::vector<double> acc(static_cast<size_t>(Dv));
  const double c = (g_fault == 4) ? 1.0 : scale;      // fault 4: scale dropped
  const int v0 = (g_fault == 5) ? D - Dv : 0;          // fault 5: V taken from the tail
  for (int g = 0; g < H; ++g) {
    const uint16_t* qg = q + (r.row * H + g) * D;
    double m = -INFINITY;
    for (int64_t i = 0; i < n; ++i) {
      const uint16_t* k = kv + (r.kv0 + pos[i]) * D;
      double dot = 0.0;
      for (int j = 0; j < D; ++j) dot += bf16_to_double(qg[j]) * bf16_to_double(k[j]);
      logit[i] = c * dot;
      m = std::max(m, logit[i]);
    }
    double denom = 0.0;
    std::fill(acc.begin(), acc.end(), 0.0);
    for (int64_t i = 0; i < n; ++i) {
      const double e = std::exp(logit[i] - m);
      denom += e;
      const uint16_t* v = kv + (r.kv0 + pos[i]) * D + v0;
      for (int j = 0; j < Dv; ++j) acc[j] += e * bf16_to_double(v[j]);
    }
    float* o = out + (r.row * H + g) * Dv;
    for (int j = 0; j < Dv; ++j) o[j] = static_cast<float>(acc[j] / denom);
    if (lse) lse[r.row * H + g] = static_cast<float>(m + std::log(denom));
  }
}

// bf16 bit pattern of a double, rounded to nearest even through fp32 (the
// precision in which a projection's sum is formed before it is stored).
uint16_t double_to_bf16(double v) {
  const float f = static_cast<float>(v);
  uint32_t u;
  std::memcpy(&u, &f, sizeof u);
  if ((u & 0x7FFFFFFFu) > 0x7F800000u) return static_cast<uint16_t>((u >> 16) | 0x40u);  // NaN
  u += 0x7FFFu + ((u >> 16) & 1u);
  return static_cast<uint16_t>(u >> 16);
}

// sum_j a[j] * W[f, j] in double for one output feature f; W is [n_out, n_in].
double linear_one(const uint16_t* a, const uint16_t* W, int64_t n_in, int64_t f) {
  double acc = 0.0;
  const uint16_t* wf = W + f * n_in;
  for (int64_t j = 0; j < n_in; ++j) acc += bf16_to_double(a[j]) * bf16_to_double(wf[j]);
  return acc;
}

}  // namespace

extern "C" {

void oracle_set_threads(int n) {
#ifdef _OPENMP
  if (n > 0) omp_set_num_threads(n);
#else
  (void)n;
#endif
}

int oracle_max_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

void oracle_set_fault(int f) { g_fault = f; }

// Index scores I[row, s] for s = 0..p of every (sampled) query row.
void oracle_indexer_scores(int B, const int32_t* q_off, const int64_t* kv_off,
                           const int32_t* ctx_lens, int Hi, int Di, const uint16_t* q_idx,
                           const float* w, const uint16_t* k_idx, float* scores, int64_t ld,
                           const int64_t* sample, int64_t n_sample) {
  const std::vector<Row> rows = plan_rows(B, q_off, kv_off, ctx_lens, sample, n_sample);
  const int64_t n = static_cast<int64_t>(rows.size());
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t i = 0; i < n; ++i) {
    score_row(rows[i], Hi, Di, q_idx, w, k_idx, scores + rows[i].row * ld);
  }
}

// Top-k of precomputed scores: idx[row, 0..k) per the selection rule above.
void oracle_topk(int B, const int32_t* q_off, const int64_t* kv_off, const int32_t* ctx_lens,
                 const float* scores, int64_t ld, int top_k, int32_t* idx,
                 const int64_t* sample, int64_t n_sample) {
  const std::vector<Row> rows = plan_rows(B, q_off, kv_off, ctx_lens, sample, n_sample);
  const int64_t n = static_cast<int64_t>(rows.size());
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t i = 0; i < n; ++i) {
    select_row(scores + rows[i].row * ld, causal_count(rows[i]), top_k,
               idx + rows[i].row * top_k);
  }
}

// Attention of each (sampled) query over the positions listed in idx (-1 = none).
void oracle_sparse_attn(int B, const int32_t* q_off, const int64_t* kv_off,
                        const int32_t* ctx_lens, int H, int D, int Dv, const uint16_t* q,
                        const uint16_t* kv, const int32_t* idx, int top_k, double scale,
                        float* out, float* lse, const int64_t* sample, int64_t n_sample) {
  const std::vector<Row> rows = plan_rows(B, q_off, kv_off, ctx_lens, sample, n_sample);
  const int64_t n = static_cast<int64_t>(rows.size());
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t i = 0; i < n; ++i) {
    std::vector<int32_t> pos;
    const int32_t* ir = idx + rows[i].row * top_k;
    for (int t = 0; t < top_k; ++t) {
      if (ir[t] >= 0) pos.push_back(ir[t]);
    }
    attend_row(rows[i], H, D, Dv, q, kv, pos.data(), static_cast<int64_t>(pos.size()), scale,
               out, lse);
  }
}

// Full causal attention over positions 0..p: no indexer, no selection.
void oracle_full_causal_attn(int B, const int32_t* q_off, const int64_t* kv_off,
                             const int32_t* ctx_lens, int H, int D, int Dv, const uint16_t* q,
                             const uint16_t* kv, double scale, float* out, float* lse,
                             const int64_t* sample, int64_t n_sample) {
  const std::vector<Row> rows = plan_rows(B, q_off, kv_off, ctx_lens, sample, n_sample);
  const int64_t n = static_cast<int64_t>(rows.size());
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t i = 0; i < n; ++i) {
    const int64_t n_pos = causal_count(rows[i]);
    std::vector<int32_t> pos(static_cast<size_t>(n_pos));
    for (int64_t s = 0; s < n_pos; ++s) pos[s] = static_cast<int32_t>(s);
    attend_row(rows[i], H, D, Dv, q, kv, pos.data(), n_pos, scale, out, lse);
  }
}

// The whole layer for each (sampled) query: score, select, attend.  Scores and
// idx are also returned (scores rows need ld >= max context length).
void oracle_dsa_layer(int B, const int32_t* q_off, const int64_t* kv_off,
                      const int32_t* ctx_lens, int Hi, int Di, const uint16_t* q_idx,
                      const float* w, const uint16_t* k_idx, int H, int D, int Dv,
                      const uint16_t* q, const uint16_t* kv, int top_k, double scale,
                      float* scores, int64_t ld, int32_t* idx, float* out, float* lse,
                      const int64_t* sample, int64_t n_sample) {
  const std::vector<Row> rows = plan_rows(B, q_off, kv_off, ctx_lens, sample, n_sample);
  const int64_t n = static_cast<int64_t>(rows.size());
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t i = 0; i < n; ++i) {
    const Row& r = rows[i];
    float* sc = scores + r.row * ld;
    int32_t* ir = idx + r.row * top_k;
    score_row(r, Hi, Di, q_idx, w, k_idx, sc);
    select_row(sc, causal_count(r), top_k, ir);
    std::vector<int32_t> pos;
    for (int t = 0; t < top_k; ++t) {
      if (ir[t] >= 0) pos.push_back(ir[t]);
    }
    attend_row(r, H, D, Dv, q, kv, pos.data(), static_cast<int64_t>(pos.size()), scale, out,
               lse);
  }
}

// The indexer's input step for every (sampled) query row t (a new token of
// sequence b at position p): q_idx[t] = c_q[t] . W_q_b^T (Hi*Di outputs, bf16),
// k = x[t] . W_k^T (Di outputs, bf16) written to cache row kv_off[b] + p of
// k_idx, w[t] = x[t] . W_proj^T (Hi outputs, fp32).  Weights are [out, in].
void oracle_indexer_project(int B, const int32_t* q_off, const int64_t* kv_off,
                            const int32_t* ctx_lens, int Hi, int Di, int64_t d_model,
                            int64_t d_q, const uint16_t* x, const uint16_t* c_q,
                            const uint16_t* w_q_b, const uint16_t* w_k, const uint16_t* w_proj,
                            uint16_t* q_idx, uint16_t* k_idx, float* w, const int64_t* sample,
                            int64_t n_sample) {
  const std::vector<Row> rows = plan_rows(B, q_off, kv_off, ctx_lens, sample, n_sample);
  const int64_t n = static_cast<int64_t>(rows.size());
  const int64_t nq_out = static_cast<int64_t>(Hi) * Di;
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t i = 0; i < n; ++i) {
    const Row& r = rows[i];
    const uint16_t* xr = x + r.row * d_model;
    const uint16_t* cr = c_q + r.row * d_q;
    for (int64_t f = 0; f < nq_out; ++f) {
      q_idx[r.row * nq_out + f] = double_to_bf16(linear_one(cr, w_q_b, d_q, f));
    }
    const int64_t cache_row = (g_fault == 6) ? r.kv0 + r.pos + 1 : r.kv0 + r.pos;  // fault 6
    for (int64_t f = 0; f < Di; ++f) {
      double v = 0.0;
      if (g_fault == 7) {  // fault 7: the key map read transposed (W_k taken as [in, out])
        for (int64_t j = 0; j < d_model; ++j) {
          v += bf16_to_double(xr[j]) * bf16_to_double(w_k[j * Di + f]);
        }
      } else {
        v = linear_one(xr, w_k, d_model, f);
      }
      k_idx[cache_row * Di + f] = double_to_bf16(v);
    }
    for (int h = 0; h < Hi; ++h) {
      w[r.row * Hi + h] = static_cast<float>(linear_one(xr, w_proj, d_model, h));
    }
  }
}

}  // extern "C"
