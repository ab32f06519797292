// fp64 CPU oracle for exact scaled-dot-product attention, forward and backward.
//
// TEST INFRASTRUCTURE ONLY. Only tests/, the smoke check of the package entry
// file and the cpu_baseline / reference legs of bench.py may load this library.
// The CUDA path never calls it, and it shares no code with the CUDA path.
//
// What it computes is the plain definition of standard attention, because the
// tiled method reaches that result exactly up to rounding order:
//   * "FlashAttention (v2)" glossary page, definition paragraph: the method
//     works through attention tile by tile and makes no approximation;
//     results paragraph: what it returns is standard attention's result.
//   * "FlashAttention-2" summary page, "How It Works": the work is only
//     re-partitioned and the scaling moved to the end; the function computed is
//     unchanged.
// For each head (b, h), with query rows i in [0, Nq) and key columns j in
// [0, Nk) (Nq = Nk = N in every configuration of the pages):
//   s_ij  = scale * sum_c q_ic k_jc          (-inf where causal and j > i + Nk - Nq)
//   m_i   = max_j s_ij,  l_i = sum_j exp(s_ij - m_i)
//   p_ij  = exp(s_ij - m_i) / l_i
//   O_i   = sum_j p_ij v_j,  LSE_i = m_i + ln l_i   (natural log)
// Backward (the pages plot the backward pass -- paper reproduction page,
// Figure 6a-d -- but print no equations; these are the chain-rule gradients of
// the definition above for a loss L with dL/dO = dO):
//   dP_ij = dO_i . v_j,   D_i = sum_c dO_ic O_ic,   dS_ij = p_ij (dP_ij - D_i)
//   dQ_i  = scale * sum_j dS_ij k_j
//   dK_j  = scale * sum_i dS_ij q_i
//   dV_j  = sum_i p_ij dO_i
//
// Arithmetic is fp64 on inputs that the caller widened exactly from bf16.
// Every sum runs over its index in increasing order. The only restructuring is
// where loops are nested so that an inner loop over an independent index
// (j for the dot products, c for the row sums) runs contiguously; each
// individual sum still adds its terms in the same order as the formula.
// Threads split rows or heads; no sum is split between threads.
//
// Causal masking with Nq != Nk is aligned to the bottom-right corner of the
// score matrix (the last query sees every key); the pages only use Nq = Nk, so
// this is our reading. Causal with Nq > Nk would leave rows without keys and is
// rejected.
//
// Layout: q, o, dq, dout are contiguous [n_heads][Nq][d] arrays of doubles, k, v,
// dk, dv [n_heads][Nk][d] (one head = one (b, h) pair); LSE and D are [n_heads][Nq].
//
// parity: pinned by tests/test_oracle.py (pure-Python brute force on tiny
// inputs, central finite differences of the forward, closed forms at N = 1,
// uniform scores, causal row 0, shift invariance, gradient-sum identities and an
// independent tiled online-softmax recurrence).

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <limits>
#include <thread>
#include <vector>

namespace {

constexpr double kNegInf = -std::numeric_limits<double>::infinity();
constexpr int64_t kJBlock = 256;  // columns of the score row computed together

int resolve_threads(int nthreads) {
  if (nthreads > 0) return nthreads;
  unsigned hc = std::thread::hardware_concurrency();
  return hc ? (int)hc : 1;
}

// Runs body(t) for t in [0, count) on up to nthreads threads (dynamic split).
template <class F>
void parallel_for(int64_t count, int nthreads, F body) {
  nthreads = (int)std::min<int64_t>(resolve_threads(nthreads), std::max<int64_t>(count, 1));
  if (nthreads <= 1) {
    for (int64_t t = 0; t < count; ++t) body(t);
    return;
  }
  std::atomic<int64_t> next{0};
  std::vector<std::thread> pool;
  pool.reserve(nthreads);
  for (int w = 0; w < nthreads; ++w) {
    pool.emplace_back([&]() {
      for (int64_t t = next.fetch_add(1); t < count; t = next.fetch_add(1)) body(t);
    });
  }
  for (auto& th : pool) th.join();
}

// K transposed to [d][N] so that the dot products for a block of columns j can
// run with j innermost; each s_ij still sums c = 0, 1, ..., d-1 in order.
std::vector<double> transpose(const double* k, int64_t N, int64_t d) {
  std::vector<double> kt((size_t)(N * d));
  for (int64_t j = 0; j < N; ++j)
    for (int64_t c = 0; c < d; ++c) kt[(size_t)(c * N + j)] = k[j * d + c];
  return kt;
}

// Number of key columns query row i may see: causal rows see j <= i + Nk - Nq.
inline int64_t n_allowed(int64_t i, int64_t Nq, int64_t Nk, int causal) {
  return causal ? std::min(Nk, i + 1 + Nk - Nq) : Nk;
}

// s[j] = scale * sum_c q_ic k_jc for j < ncols (row i of the score matrix).
void score_row(const double* qi, const double* kt, int64_t N, int64_t d, int64_t ncols,
               double scale, double* s) {
  for (int64_t j0 = 0; j0 < ncols; j0 += kJBlock) {
    const int64_t j1 = std::min(ncols, j0 + kJBlock);
    double* acc = s + j0;
    for (int64_t j = j0; j < j1; ++j) acc[j - j0] = 0.0;
    for (int64_t c = 0; c < d; ++c) {
      const double qc = qi[c];
      const double* kc = kt + c * N;
      for (int64_t j = j0; j < j1; ++j) acc[j - j0] += qc * kc[j];
    }
    for (int64_t j = j0; j < j1; ++j) acc[j - j0] *= scale;
  }
}

// Softmax of one score row over its first ncols entries: writes p (ncols
// entries) and returns LSE = m + ln l.
double softmax_row(const double* s, int64_t ncols, double* p) {
  double m = kNegInf;
  for (int64_t j = 0; j < ncols; ++j) m = std::max(m, s[j]);
  double l = 0.0;
  for (int64_t j = 0; j < ncols; ++j) l += std::exp(s[j] - m);
  for (int64_t j = 0; j < ncols; ++j) p[j] = std::exp(s[j] - m) / l;
  return m + std::log(l);
}

// out[c] = sum_j p[j] * rows[j][c] for j < ncols (j in order, c innermost).
void weighted_row_sum(const double* p, const double* rows, int64_t ncols, int64_t d, double* out) {
  for (int64_t c = 0; c < d; ++c) out[c] = 0.0;
  for (int64_t j = 0; j < ncols; ++j) {
    const double pj = p[j];
    const double* r = rows + j * d;
    for (int64_t c = 0; c < d; ++c) out[c] += pj * r[c];
  }
}

double dot(const double* a, const double* b, int64_t d) {
  double acc = 0.0;
  for (int64_t c = 0; c < d; ++c) acc += a[c] * b[c];
  return acc;
}

}  // namespace

extern "C" {

// Forward of standard attention for n_heads independent heads.
// rows: optional list of n_rows query rows (NULL = all Nq rows, n_rows ignored).
// o: [n_heads][n_rows][d], lse: [n_heads][n_rows] (natural log).
// Returns 0, or -1 on bad sizes.
int oracle_attention_forward_qk(const double* q, const double* k, const double* v, int64_t n_heads,
                                int64_t Nq, int64_t Nk, int64_t d, int causal, double scale,
                                const int64_t* rows, int64_t n_rows, double* o, double* lse,
                                int nthreads) {
  if (n_heads < 0 || Nq < 1 || Nk < 1 || d < 1 || (causal && Nq > Nk)) return -1;
  if (!rows) n_rows = Nq;
  for (int64_t r = 0; rows && r < n_rows; ++r)
    if (rows[r] < 0 || rows[r] >= Nq) return -1;
  for (int64_t h = 0; h < n_heads; ++h) {
    const double* qh = q + h * Nq * d;
    const double* kh = k + h * Nk * d;
    const double* vh = v + h * Nk * d;
    const std::vector<double> kt = transpose(kh, Nk, d);
    parallel_for(n_rows, nthreads, [&](int64_t r) {
      const int64_t i = rows ? rows[r] : r;
      const int64_t nc = n_allowed(i, Nq, Nk, causal);
      std::vector<double> s((size_t)Nk), p((size_t)Nk);
      score_row(qh + i * d, kt.data(), Nk, d, nc, scale, s.data());
      lse[h * n_rows + r] = softmax_row(s.data(), nc, p.data());
      weighted_row_sum(p.data(), vh, nc, d, o + (h * n_rows + r) * d);
    });
  }
  return 0;
}

int oracle_attention_forward(const double* q, const double* k, const double* v, int64_t n_heads,
                             int64_t N, int64_t d, int causal, double scale, const int64_t* rows,
                             int64_t n_rows, double* o, double* lse, int nthreads) {
  return oracle_attention_forward_qk(q, k, v, n_heads, N, N, d, causal, scale, rows, n_rows, o, lse,
                                     nthreads);
}

// Full backward for n_heads heads (also returns the oracle's own O and LSE).
// o, dq: [n_heads][Nq][d], lse: [n_heads][Nq], dk, dv: [n_heads][Nk][d]. Memory:
// two Nq x Nk double matrices per head (P and dS), so keep them moderate.
int oracle_attention_backward_qk(const double* q, const double* k, const double* v,
                                 const double* dout, int64_t n_heads, int64_t Nq, int64_t Nk,
                                 int64_t d, int causal, double scale, double* o, double* lse,
                                 double* dq, double* dk, double* dv, int nthreads) {
  if (n_heads < 0 || Nq < 1 || Nk < 1 || d < 1 || (causal && Nq > Nk)) return -1;
  std::vector<double> P((size_t)(Nq * Nk)), dS((size_t)(Nq * Nk)), D((size_t)Nq);
  for (int64_t h = 0; h < n_heads; ++h) {
    const double* qh = q + h * Nq * d;
    const double* kh = k + h * Nk * d;
    const double* vh = v + h * Nk * d;
    const double* doh = dout + h * Nq * d;
    double* oh = o + h * Nq * d;
    double* lseh = lse + h * Nq;
    double* dqh = dq + h * Nq * d;
    double* dkh = dk + h * Nk * d;
    double* dvh = dv + h * Nk * d;
    const std::vector<double> kt = transpose(kh, Nk, d);
    const std::vector<double> vt = transpose(vh, Nk, d);
    // forward rows, then D_i, dP_i and dS_i, then dQ_i = scale * sum_j dS_ij k_j
    parallel_for(Nq, nthreads, [&](int64_t i) {
      const int64_t nc = n_allowed(i, Nq, Nk, causal);
      std::vector<double> s((size_t)Nk), dp((size_t)Nk);
      double* pi = P.data() + i * Nk;
      score_row(qh + i * d, kt.data(), Nk, d, nc, scale, s.data());
      lseh[i] = softmax_row(s.data(), nc, pi);
      for (int64_t j = nc; j < Nk; ++j) pi[j] = 0.0;
      weighted_row_sum(pi, vh, nc, d, oh + i * d);
      D[(size_t)i] = dot(doh + i * d, oh + i * d, d);
      score_row(doh + i * d, vt.data(), Nk, d, nc, 1.0, dp.data());  // dP_ij = dO_i . v_j
      double* dsi = dS.data() + i * Nk;
      for (int64_t j = 0; j < nc; ++j) dsi[j] = pi[j] * (dp[j] - D[(size_t)i]);
      for (int64_t j = nc; j < Nk; ++j) dsi[j] = 0.0;
      weighted_row_sum(dsi, kh, nc, d, dqh + i * d);
      for (int64_t c = 0; c < d; ++c) dqh[i * d + c] *= scale;
    });
    // dK_j = scale * sum_i dS_ij q_i and dV_j = sum_i p_ij dO_i over the queries
    // that see key j (i in order)
    parallel_for(Nk, nthreads, [&](int64_t j) {
      double* dkj = dkh + j * d;
      double* dvj = dvh + j * d;
      for (int64_t c = 0; c < d; ++c) dkj[c] = 0.0, dvj[c] = 0.0;
      for (int64_t i = causal ? std::max<int64_t>(0, j - (Nk - Nq)) : 0; i < Nq; ++i) {
        const double ds = dS[(size_t)(i * Nk + j)];
        const double p = P[(size_t)(i * Nk + j)];
        const double* qi = qh + i * d;
        const double* doi = doh + i * d;
        for (int64_t c = 0; c < d; ++c) dkj[c] += ds * qi[c];
        for (int64_t c = 0; c < d; ++c) dvj[c] += p * doi[c];
      }
      for (int64_t c = 0; c < d; ++c) dkj[c] *= scale;
    });
  }
  return 0;
}

int oracle_attention_backward(const double* q, const double* k, const double* v, const double* dout,
                              int64_t n_heads, int64_t N, int64_t d, int causal, double scale,
                              double* o, double* lse, double* dq, double* dk, double* dv,
                              int nthreads) {
  return oracle_attention_backward_qk(q, k, v, dout, n_heads, N, N, d, causal, scale, o, lse, dq, dk,
                                      dv, nthreads);
}

// Backward restricted to chosen rows, for heads too long to hold Nq x Nk.
// Computes the full forward of each head (every LSE_i and O_i, hence every
// D_i), then dQ for the query rows qrows and dK, dV for the key rows krows
// straight from the definitions. Outputs: dq [n_heads][n_q][d],
// dk and dv [n_heads][n_k][d].
int oracle_attention_backward_rows_qk(const double* q, const double* k, const double* v,
                                      const double* dout, int64_t n_heads, int64_t Nq, int64_t Nk,
                                      int64_t d, int causal, double scale, const int64_t* qrows,
                                      int64_t n_q, const int64_t* krows, int64_t n_k, double* dq,
                                      double* dk, double* dv, int nthreads) {
  if (n_heads < 0 || Nq < 1 || Nk < 1 || d < 1 || n_q < 0 || n_k < 0 || (causal && Nq > Nk))
    return -1;
  for (int64_t r = 0; r < n_q; ++r)
    if (qrows[r] < 0 || qrows[r] >= Nq) return -1;
  for (int64_t r = 0; r < n_k; ++r)
    if (krows[r] < 0 || krows[r] >= Nk) return -1;
  std::vector<double> O((size_t)(Nq * d)), L((size_t)Nq), D((size_t)Nq);
  for (int64_t h = 0; h < n_heads; ++h) {
    const double* qh = q + h * Nq * d;
    const double* kh = k + h * Nk * d;
    const double* vh = v + h * Nk * d;
    const double* doh = dout + h * Nq * d;
    const std::vector<double> kt = transpose(kh, Nk, d);
    const std::vector<double> vt = transpose(vh, Nk, d);
    parallel_for(Nq, nthreads, [&](int64_t i) {
      const int64_t nc = n_allowed(i, Nq, Nk, causal);
      std::vector<double> s((size_t)Nk), p((size_t)Nk);
      score_row(qh + i * d, kt.data(), Nk, d, nc, scale, s.data());
      L[(size_t)i] = softmax_row(s.data(), nc, p.data());
      weighted_row_sum(p.data(), vh, nc, d, O.data() + i * d);
      D[(size_t)i] = dot(doh + i * d, O.data() + i * d, d);
    });
    parallel_for(n_q, nthreads, [&](int64_t r) {
      const int64_t i = qrows[r];
      const int64_t nc = n_allowed(i, Nq, Nk, causal);
      std::vector<double> s((size_t)Nk), dp((size_t)Nk), ds((size_t)Nk);
      score_row(qh + i * d, kt.data(), Nk, d, nc, scale, s.data());
      score_row(doh + i * d, vt.data(), Nk, d, nc, 1.0, dp.data());
      for (int64_t j = 0; j < nc; ++j) ds[j] = std::exp(s[j] - L[(size_t)i]) * (dp[j] - D[(size_t)i]);
      double* out = dq + (h * n_q + r) * d;
      weighted_row_sum(ds.data(), kh, nc, d, out);
      for (int64_t c = 0; c < d; ++c) out[c] *= scale;
    });
    parallel_for(n_k, nthreads, [&](int64_t r) {
      const int64_t j = krows[r];
      double* dkj = dk + (h * n_k + r) * d;
      double* dvj = dv + (h * n_k + r) * d;
      for (int64_t c = 0; c < d; ++c) dkj[c] = 0.0, dvj[c] = 0.0;
      const double* kj = kh + j * d;
      const double* vj = vh + j * d;
      for (int64_t i = causal ? std::max<int64_t>(0, j - (Nk - Nq)) : 0; i < Nq; ++i) {
        const double* qi = qh + i * d;
        const double* doi = doh + i * d;
        const double p = std::exp(scale * dot(qi, kj, d) - L[(size_t)i]);
        const double ds = p * (dot(doi, vj, d) - D[(size_t)i]);
        for (int64_t c = 0; c < d; ++c) dkj[c] += ds * qi[c];
        for (int64_t c = 0; c < d; ++c) dvj[c] += p * doi[c];
      }
      for (int64_t c = 0; c < d; ++c) dkj[c] *= scale;
    });
  }
  return 0;
}

int oracle_attention_backward_rows(const double* q, const double* k, const double* v,
                                   const double* dout, int64_t n_heads, int64_t N, int64_t d,
                                   int causal, double scale, const int64_t* qrows, int64_t n_q,
                                   const int64_t* krows, int64_t n_k, double* dq, double* dk,
                                   double* dv, int nthreads) {
  return oracle_attention_backward_rows_qk(q, k, v, dout, n_heads, N, N, d, causal, scale, qrows, n_q,
                                           krows, n_k, dq, dk, dv, nthreads);
}

int oracle_default_threads(void) { return resolve_threads(0); }

}  // extern "C"
