// Candidate-to-history cross attention (the two branches of STCA), fp64 CPU oracle.
//
// TEST INFRASTRUCTURE ONLY, like sa_oracle.cpp: only tests/, __graft_entry__.smoke() and
// bench.py's cpu_baseline leg may load it. It shares no code with the CUDA library.
//
// What it computes. User u has a sketch S_u (k rows of length d, the output of Sketch
// Attention) and a ragged group of candidates c in [coff[u], coff[u+1]) with embeddings
// Q_c (length d). Every candidate of the user reads the same sketch (the one sketch read
// per user that multi-request user-level batching buys):
//   q_c  = Q_c W_q,   K_j = S_uj W_K,   V_j = S_uj W_V       (row vectors of length d)
//   z_cj = (q_c . K_j) / sqrt(d)                            (the candidate scores every row)
//   a_cj = exp(z_cj) / sum_i exp(z_ci)                      (softmax over the k sketch rows)
//   O_c  = sum_j a_cj V_j,   lse_c = log sum_j exp(z_cj)
// The *_keys entry points take each user's key rows as a ragged list instead (k_u rows
// for user u), which covers the other branch: the candidate attending over the user's
// most recent tokens (the last min(n_u, L) rows of the history).
// Sources: "100,000 videos in your pocket" blog (danielsamfdo.github.io), section
// "2. STCA reasons at two time scales" (the sketch branch: the candidate attends over
// the fixed-size sketch; the recent branch: over the recent 10K suffix) and section
// "3. The system makes it cheap enough to matter" (multi-request user-level batching: a
// user's candidates share one sketch read). The pages give no equations for STCA;
// single-head scaled dot-product attention with square, bias-free projections W_q,
// W_K, W_V, one layer (stacking repeats it), no mask, is the plainest reading and is
// what this file computes for both branches.
//
// Candidate sums over a user's candidates (dK, dV and the weight gradients of the
// backward) are taken over fixed chunks of candidates whose partials are added in
// chunk order, so results do not depend on the number of OpenMP threads.
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <vector>
#ifdef _OPENMP
#include <omp.h>
#endif

namespace {

constexpr int64_t kCandChunk = 64;  // candidates per fixed summation chunk

int threads_or_default(int nthreads) {
#ifdef _OPENMP
  return nthreads > 0 ? nthreads : omp_get_max_threads();
#else
  (void)nthreads;
  return 1;
#endif
}

int check_args(const int64_t* coff, int R, int64_t n_cand, int d, int k) {
  if (R < 0 || n_cand < 0 || d <= 0 || k <= 0) return 1;
  if (coff[0] != 0 || coff[R] != n_cand) return 2;
  for (int u = 0; u < R; ++u) if (coff[u + 1] < coff[u]) return 2;
  return 0;
}

// y = x W for a row vector x of length d and W [d, d] row-major.
void row_times(const double* x, const double* W, int d, double* y) {
  for (int e = 0; e < d; ++e) y[e] = 0.0;
  for (int c = 0; c < d; ++c) {
    const double xc = x[c];
    const double* w = W + (int64_t)c * d;
    for (int e = 0; e < d; ++e) y[e] += xc * w[e];
  }
}

// K = S_u W_K and V = S_u W_V for the k rows of one user's sketch.
void project_rows(const double* Su, int k, int d, const double* WK, const double* WV,
                  double* K, double* V) {
  for (int j = 0; j < k; ++j) {
    row_times(Su + (int64_t)j * d, WK, d, K + (int64_t)j * d);
    row_times(Su + (int64_t)j * d, WV, d, V + (int64_t)j * d);
  }
}

// One candidate: q (length d) against K, V [k, d]. Fills a (k) and O (d), returns lse.
double candidate_forward(const double* q, const double* K, const double* V, int k, int d,
                         double* a, double* O) {
  const double inv_sqrt_d = 1.0 / std::sqrt((double)d);
  double m = -INFINITY;
  for (int j = 0; j < k; ++j) {
    const double* kj = K + (int64_t)j * d;
    double z = 0.0;
    for (int e = 0; e < d; ++e) z += q[e] * kj[e];
    z *= inv_sqrt_d;
    a[j] = z;
    m = std::max(m, z);
  }
  double Z = 0.0;
  for (int j = 0; j < k; ++j) { a[j] = std::exp(a[j] - m); Z += a[j]; }
  for (int j = 0; j < k; ++j) a[j] /= Z;
  for (int e = 0; e < d; ++e) O[e] = 0.0;
  for (int j = 0; j < k; ++j) {
    const double* vj = V + (int64_t)j * d;
    for (int e = 0; e < d; ++e) O[e] += a[j] * vj[e];
  }
  return m + std::log(Z);
}

}  // namespace

extern "C" {

// Forward over a ragged batch of users whose key rows are ragged too.
//   Q     [n_cand, d]   candidate embeddings, users' groups concatenated
//   coff  [R+1]         coff[0] = 0, non-decreasing, coff[R] = n_cand
//   Kx    [n_keys, d]   the rows each user's candidates attend over, users concatenated
//                       (a sketch: k rows per user; the recent suffix: the last tokens)
//   koff  [R+1]         koff[0] = 0, non-decreasing, koff[R] = n_keys
//   Wq, WK, WV [d, d]
// Outputs: O [n_cand, d]; lse [n_cand] (may be null). A user with candidates but no key
// rows gives O = 0 and lse = -inf (the attention has nothing to read).
// Returns 0 on success, 1 on bad sizes, 2 on bad offsets.
int stca_oracle_forward_keys(const double* Q, const int64_t* coff, int R, int64_t n_cand, int d,
                             const double* Kx, const int64_t* koff, int64_t n_keys,
                             const double* Wq, const double* WK, const double* WV, double* O,
                             double* lse, int nthreads) {
  if (int rc = check_args(coff, R, n_cand, d, 1)) return rc;
  if (int rc = check_args(koff, R, n_keys, d, 1)) return rc;
  const int nt = threads_or_default(nthreads);
  std::vector<double> K, V;
  for (int u = 0; u < R; ++u) {
    const int64_t c0 = coff[u], c1 = coff[u + 1];
    if (c1 == c0) continue;
    const int k = (int)(koff[u + 1] - koff[u]);
    K.assign((size_t)k * d, 0.0);
    V.assign((size_t)k * d, 0.0);
    project_rows(Kx + koff[u] * d, k, d, WK, WV, K.data(), V.data());
#pragma omp parallel for schedule(dynamic, 16) num_threads(nt)
    for (int64_t c = c0; c < c1; ++c) {
      std::vector<double> q(d), a(k);
      row_times(Q + c * d, Wq, d, q.data());
      const double l = candidate_forward(q.data(), K.data(), V.data(), k, d, a.data(), O + c * d);
      if (lse) lse[c] = l;
    }
  }
  return 0;
}

// The sketch case: every user has k key rows, S [R, k, d].
int stca_oracle_forward(const double* Q, const int64_t* coff, int R, int64_t n_cand, int d,
                        const double* S, int k, const double* Wq, const double* WK,
                        const double* WV, double* O, double* lse, int nthreads) {
  if (R < 0 || k <= 0) return 1;
  std::vector<int64_t> koff((size_t)R + 1);
  for (int u = 0; u <= R; ++u) koff[u] = (int64_t)u * k;
  return stca_oracle_forward_keys(Q, coff, R, n_cand, d, S, koff.data(), (int64_t)R * k, Wq, WK,
                                  WV, O, lse, nthreads);
}

// Backward: gradients of a loss L given dO = dL/dO [n_cand, d].
// Outputs: dQ [n_cand, d]; dS [n_keys, d] (per user: the gradient that flows into its
// key rows; for a sketch, into Sketch Attention's backward); dWq, dWK, dWV [d, d] summed
// over users (all overwritten, not accumulated into).
//
// Derivation (per user, chain rule through the forward above):
//   dV_j  = sum_c a_cj dO_c
//   da_cj = dO_c . V_j,   D_c = sum_j a_cj da_cj,   dz_cj = a_cj (da_cj - D_c)
//   dq_c  = sum_j dz_cj K_j / sqrt(d),   dK_j = sum_c dz_cj q_c / sqrt(d)
//   dQ_c  = dq_c W_q^T,   dS_uj = dK_j W_K^T + dV_j W_V^T
//   dW_q += sum_c Q_c^T dq_c,   dW_K += sum_j S_uj^T dK_j,   dW_V += sum_j S_uj^T dV_j
// A user without candidates gets dS = 0. Returns 0 / 1 / 2 as the forward.
int stca_oracle_backward_keys(const double* Q, const int64_t* coff, int R, int64_t n_cand, int d,
                              const double* Kx, const int64_t* koff, int64_t n_keys,
                              const double* Wq, const double* WK, const double* WV,
                              const double* dO, double* dQ, double* dS, double* dWq,
                              double* dWK, double* dWV, int nthreads) {
  if (int rc = check_args(coff, R, n_cand, d, 1)) return rc;
  if (int rc = check_args(koff, R, n_keys, d, 1)) return rc;
  const int nt = threads_or_default(nthreads);
  const int64_t dd = (int64_t)d * d;
  const double inv_sqrt_d = 1.0 / std::sqrt((double)d);
  std::memset(dS, 0, sizeof(double) * (size_t)n_keys * d);
  std::memset(dWq, 0, sizeof(double) * dd);
  std::memset(dWK, 0, sizeof(double) * dd);
  std::memset(dWV, 0, sizeof(double) * dd);
  std::vector<double> K, V;
  for (int u = 0; u < R; ++u) {
    const int64_t c0 = coff[u], c1 = coff[u + 1];
    if (c1 == c0) continue;
    const int k = (int)(koff[u + 1] - koff[u]);
    const int64_t kd = (int64_t)k * d;
    const int64_t acc_len = 2 * kd + dd;  // [dK | dV | dWq] per chunk of candidates
    const double* Su = Kx + koff[u] * d;
    K.assign((size_t)kd, 0.0);
    V.assign((size_t)kd, 0.0);
    project_rows(Su, k, d, WK, WV, K.data(), V.data());
    const int64_t nchunks = (c1 - c0 + kCandChunk - 1) / kCandChunk;
    std::vector<double> part(nchunks * acc_len, 0.0);
#pragma omp parallel for schedule(dynamic, 1) num_threads(nt)
    for (int64_t ch = 0; ch < nchunks; ++ch) {
      std::vector<double> q(d), a(k), da(k), O(d), dq(d);
      double* aK = part.data() + ch * acc_len;
      double* aV = aK + kd;
      double* aWq = aK + 2 * kd;
      const int64_t b0 = c0 + ch * kCandChunk, b1 = std::min(c1, b0 + kCandChunk);
      for (int64_t c = b0; c < b1; ++c) {
        const double* Qc = Q + c * d;
        const double* g = dO + c * d;
        row_times(Qc, Wq, d, q.data());
        candidate_forward(q.data(), K.data(), V.data(), k, d, a.data(), O.data());
        double D = 0.0;
        for (int j = 0; j < k; ++j) {
          const double* vj = V.data() + (int64_t)j * d;
          double s = 0.0;
          for (int e = 0; e < d; ++e) s += g[e] * vj[e];
          da[j] = s;
          D += a[j] * s;
        }
        for (int e = 0; e < d; ++e) dq[e] = 0.0;
        for (int j = 0; j < k; ++j) {
          const double dz = a[j] * (da[j] - D);
          const double* kj = K.data() + (int64_t)j * d;
          double* dkj = aK + (int64_t)j * d;
          double* dvj = aV + (int64_t)j * d;
          for (int e = 0; e < d; ++e) {
            dq[e] += dz * kj[e] * inv_sqrt_d;
            dkj[e] += dz * q[e] * inv_sqrt_d;
            dvj[e] += a[j] * g[e];
          }
        }
        double* dQc = dQ + c * d;
        for (int r = 0; r < d; ++r) {  // dQ_c[r] = sum_e dq[e] Wq[r][e]
          const double* w = Wq + (int64_t)r * d;
          double s = 0.0;
          for (int e = 0; e < d; ++e) s += dq[e] * w[e];
          dQc[r] = s;
          double* wq = aWq + (int64_t)r * d;
          for (int e = 0; e < d; ++e) wq[e] += Qc[r] * dq[e];
        }
      }
    }
    std::vector<double> dK(kd, 0.0), dV(kd, 0.0);
    for (int64_t ch = 0; ch < nchunks; ++ch) {
      const double* p = part.data() + ch * acc_len;
      for (int64_t i = 0; i < kd; ++i) { dK[i] += p[i]; dV[i] += p[kd + i]; }
      for (int64_t i = 0; i < dd; ++i) dWq[i] += p[2 * kd + i];
    }
    double* dSu = dS + koff[u] * d;
    for (int j = 0; j < k; ++j) {
      const double* dkj = dK.data() + (int64_t)j * d;
      const double* dvj = dV.data() + (int64_t)j * d;
      const double* sj = Su + (int64_t)j * d;
      for (int r = 0; r < d; ++r) {
        const double* wk = WK + (int64_t)r * d;
        const double* wv = WV + (int64_t)r * d;
        double s = 0.0;
        for (int e = 0; e < d; ++e) s += dkj[e] * wk[e] + dvj[e] * wv[e];
        dSu[(int64_t)j * d + r] = s;
        double* gk = dWK + (int64_t)r * d;
        double* gv = dWV + (int64_t)r * d;
        for (int e = 0; e < d; ++e) { gk[e] += sj[r] * dkj[e]; gv[e] += sj[r] * dvj[e]; }
      }
    }
  }
  return 0;
}

// The sketch case: every user has k key rows, S and dS [R, k, d].
int stca_oracle_backward(const double* Q, const int64_t* coff, int R, int64_t n_cand, int d,
                         const double* S, int k, const double* Wq, const double* WK,
                         const double* WV, const double* dO, double* dQ, double* dS,
                         double* dWq, double* dWK, double* dWV, int nthreads) {
  if (R < 0 || k <= 0) return 1;
  std::vector<int64_t> koff((size_t)R + 1);
  for (int u = 0; u <= R; ++u) koff[u] = (int64_t)u * k;
  return stca_oracle_backward_keys(Q, coff, R, n_cand, d, S, koff.data(), (int64_t)R * k, Wq,
                                   WK, WV, dO, dQ, dS, dWq, dWK, dWV, nthreads);
}

}  // extern "C"
