// Sketch Attention fp64 CPU oracle.
//
// TEST INFRASTRUCTURE ONLY. This file is the slow, plain reference that the CUDA
// path is checked against. Only tests/, __graft_entry__.smoke() and bench.py's
// cpu_baseline leg may load it. It shares no code, header, table or helper with
// the CUDA library, and the CUDA library never calls it.
//
// What it computes (single user u, tokens t in [offsets[u], offsets[u+1])):
//   K_t = X_t W_k,  V_t = X_t W_v                       (row vectors of length d)
//   s_jt = (P_j . K_t) / sqrt(d)                         (k prototypes score every token)
//   A_jt = exp(s_jt) / sum_i exp(s_it)                   (normalised over prototypes, so
//                                                         every token spreads unit mass)
//   mass_j   = sum_t A_jt
//   sketch_j = (sum_t A_jt V_t) / mass_j                 (mass-weighted mean of values)
//   xsketch_j = sum_t A_jt X_t                           (un-normalised, kept for backward)
//   lse_t    = log sum_j exp(s_jt)
// Sources: "100,000 videos in your pocket" blog (danielsamfdo.github.io), section
// "1. Sketch Attention compresses the history" (prototypes score every item, items
// distribute their mass over prototypes, k x d output, differentiable); evolve.pub
// review of arXiv 2609.08443, "Summary" and FAQ "How is Sketch Attention different
// from standard attention?" (normalisation across prototypes, fixed total mass per
// token, deployed 1K x 128). The pages give no equations; the projections K = X W_k,
// V = X W_v, the 1/sqrt(d) scale, the softmax as the normaliser and the
// mass-weighted mean are the plainest reading, taken as stated above.
//
// The oracle uses the UNFOLDED definition (it forms K_t and V_t explicitly) in fp64,
// with std::exp / std::log. Token sums are taken over fixed chunks of tokens whose
// partial sums are added in chunk order, so results do not depend on the number of
// OpenMP threads.
#include <cmath>
#include <cstdint>
#include <cstring>
#include <vector>
#include <algorithm>
#ifdef _OPENMP
#include <omp.h>
#endif

namespace {

constexpr int64_t kChunk = 1024;  // tokens per fixed summation chunk

// Forward quantities of one token: fills K (d), V (d), A (k) and returns lse.
double token_forward(const double* Xt, int d, const double* P, int k,
                     const double* Wk, const double* Wv,
                     double* K, double* V, double* A) {
  for (int e = 0; e < d; ++e) { K[e] = 0.0; V[e] = 0.0; }
  for (int c = 0; c < d; ++c) {
    const double x = Xt[c];
    const double* wk = Wk + (int64_t)c * d;
    const double* wv = Wv + (int64_t)c * d;
    for (int e = 0; e < d; ++e) { K[e] += x * wk[e]; V[e] += x * wv[e]; }
  }
  const double inv_sqrt_d = 1.0 / std::sqrt((double)d);
  double m = -INFINITY;
  for (int j = 0; j < k; ++j) {
    const double* pj = P + (int64_t)j * d;
    double s = 0.0;
    for (int e = 0; e < d; ++e) s += pj[e] * K[e];
    s *= inv_sqrt_d;
    A[j] = s;
    m = std::max(m, s);
  }
  double Z = 0.0;
  for (int j = 0; j < k; ++j) { A[j] = std::exp(A[j] - m); Z += A[j]; }
  for (int j = 0; j < k; ++j) A[j] /= Z;
  return m + std::log(Z);
}

int check_args(const int64_t* offsets, int R, int64_t n_total, int d, int k) {
  if (R < 0 || n_total < 0 || d <= 0 || k <= 0) return 1;
  if (offsets[0] != 0 || offsets[R] != n_total) return 2;
  for (int u = 0; u < R; ++u) if (offsets[u + 1] < offsets[u]) return 2;
  return 0;
}

int nthreads_or_default(int nthreads) {
#ifdef _OPENMP
  return nthreads > 0 ? nthreads : omp_get_max_threads();
#else
  (void)nthreads;
  return 1;
#endif
}

}  // namespace

extern "C" {

// Forward pass over a ragged batch.
//   X        [n_total, d]   row-major, users concatenated
//   offsets  [R+1]          offsets[0] = 0, non-decreasing, offsets[R] = n_total
//   P        [k, d], Wk [d, d], Wv [d, d]
// Outputs (any may be null except sketch and mass):
//   sketch [R, k, d], mass [R, k], lse [n_total], xsketch [R, k, d]
// A user with no tokens gets sketch = 0, mass = 0, xsketch = 0.
// Returns 0 on success, 1 on bad sizes, 2 on bad offsets.
int sa_oracle_forward(const double* X, const int64_t* offsets, int R, int64_t n_total,
                      int d, const double* P, int k, const double* Wk, const double* Wv,
                      double* sketch, double* mass, double* lse, double* xsketch,
                      int nthreads) {
  if (int rc = check_args(offsets, R, n_total, d, k)) return rc;
  const int nt = nthreads_or_default(nthreads);
  const int64_t acc_len = (int64_t)k * (2 * d + 1);  // [mass | sum A V | sum A X]
  for (int u = 0; u < R; ++u) {
    const int64_t t0 = offsets[u], n = offsets[u + 1] - offsets[u];
    const int64_t nchunks = (n + kChunk - 1) / kChunk;
    std::vector<double> total(acc_len, 0.0);
    // Process chunks in batches so memory stays bounded; add batch partials in order.
    const int64_t batch = std::max<int64_t>(1, 2 * nt);
    for (int64_t cb = 0; cb < nchunks; cb += batch) {
      const int64_t ce = std::min(nchunks, cb + batch);
      std::vector<double> part((ce - cb) * acc_len, 0.0);
#pragma omp parallel for schedule(dynamic, 1) num_threads(nt)
      for (int64_t c = cb; c < ce; ++c) {
        std::vector<double> K(d), V(d), A(k);
        double* acc = part.data() + (c - cb) * acc_len;
        double* acc_mass = acc;
        double* acc_av = acc + k;
        double* acc_ax = acc + k + (int64_t)k * d;
        const int64_t a = c * kChunk, b = std::min(n, a + kChunk);
        for (int64_t i = a; i < b; ++i) {
          const int64_t t = t0 + i;
          const double* Xt = X + t * d;
          const double l = token_forward(Xt, d, P, k, Wk, Wv, K.data(), V.data(), A.data());
          if (lse) lse[t] = l;
          for (int j = 0; j < k; ++j) {
            const double aj = A[j];
            acc_mass[j] += aj;
            double* av = acc_av + (int64_t)j * d;
            double* ax = acc_ax + (int64_t)j * d;
            for (int e = 0; e < d; ++e) { av[e] += aj * V[e]; ax[e] += aj * Xt[e]; }
          }
        }
      }
      for (int64_t c = cb; c < ce; ++c) {
        const double* p = part.data() + (c - cb) * acc_len;
        for (int64_t i = 0; i < acc_len; ++i) total[i] += p[i];
      }
    }
    const double* tm = total.data();
    const double* tav = tm + k;
    const double* tax = tm + k + (int64_t)k * d;
    for (int j = 0; j < k; ++j) {
      const double mj = tm[j];
      mass[(int64_t)u * k + j] = mj;
      for (int e = 0; e < d; ++e) {
        const int64_t o = ((int64_t)u * k + j) * d + e;
        sketch[o] = mj > 0.0 ? tav[(int64_t)j * d + e] / mj : 0.0;
        if (xsketch) xsketch[o] = tax[(int64_t)j * d + e];
      }
    }
  }
  return 0;
}

// Backward pass: gradients of a loss L given G = dL/dsketch [R, k, d] and an
// optional Gm = dL/dmass [R, k] (null means zero).
// Outputs: dX [n_total, d]; dP [k, d], dWk [d, d], dWv [d, d] summed over users
// (overwritten, not accumulated into).
//
// Derivation (unfolded, per user, chain rule through the forward above):
//   Gt_j    = G_j / mass_j
//   dmass_j = -Gt_j . sketch_j + Gm_j            (sketch_j = Y_j / mass_j, Y_j = sum_t A_jt V_t)
//   dA_jt   = Gt_j . V_t + dmass_j
//   dS_jt   = A_jt (dA_jt - sum_i A_it dA_it)     (softmax over prototypes)
//   dK_t    = sum_j dS_jt P_j / sqrt(d)
//   dV_t    = sum_j A_jt Gt_j
//   dX_t    = dK_t W_k^T + dV_t W_v^T
//   dP_j   += sum_t dS_jt K_t / sqrt(d)
//   dW_k   += X_t^T dK_t,   dW_v += X_t^T dV_t
// A user with no tokens contributes nothing. Returns 0 / 1 / 2 as the forward.
int sa_oracle_backward(const double* X, const int64_t* offsets, int R, int64_t n_total,
                       int d, const double* P, int k, const double* Wk, const double* Wv,
                       const double* G, const double* Gm,
                       double* dX, double* dP, double* dWk, double* dWv, int nthreads) {
  if (int rc = check_args(offsets, R, n_total, d, k)) return rc;
  const int nt = nthreads_or_default(nthreads);
  const int64_t kd = (int64_t)k * d, dd = (int64_t)d * d;
  std::memset(dP, 0, sizeof(double) * kd);
  std::memset(dWk, 0, sizeof(double) * dd);
  std::memset(dWv, 0, sizeof(double) * dd);
  std::vector<double> sk((int64_t)R * kd), ms((int64_t)R * k);
  if (int rc = sa_oracle_forward(X, offsets, R, n_total, d, P, k, Wk, Wv, sk.data(),
                                 ms.data(), nullptr, nullptr, nthreads))
    return rc;
  const double inv_sqrt_d = 1.0 / std::sqrt((double)d);
  const int64_t acc_len = kd + 2 * dd;  // [dP | dWk | dWv]
  for (int u = 0; u < R; ++u) {
    const int64_t t0 = offsets[u], n = offsets[u + 1] - offsets[u];
    std::vector<double> Gt(kd), dmass(k);
    for (int j = 0; j < k; ++j) {
      const double mj = ms[(int64_t)u * k + j];
      double dot = 0.0;
      for (int e = 0; e < d; ++e) {
        const int64_t o = ((int64_t)u * k + j) * d + e;
        Gt[(int64_t)j * d + e] = mj > 0.0 ? G[o] / mj : 0.0;
        dot += Gt[(int64_t)j * d + e] * sk[o];
      }
      dmass[j] = -dot + (Gm ? Gm[(int64_t)u * k + j] : 0.0);
    }
    const int64_t nchunks = (n + kChunk - 1) / kChunk;
    const int64_t batch = std::max<int64_t>(1, 2 * nt);
    for (int64_t cb = 0; cb < nchunks; cb += batch) {
      const int64_t ce = std::min(nchunks, cb + batch);
      std::vector<double> part((ce - cb) * acc_len, 0.0);
#pragma omp parallel for schedule(dynamic, 1) num_threads(nt)
      for (int64_t c = cb; c < ce; ++c) {
        std::vector<double> K(d), V(d), A(k), dA(k), dK(d), dV(d);
        double* acc = part.data() + (c - cb) * acc_len;
        double* aP = acc;
        double* aWk = acc + kd;
        double* aWv = acc + kd + dd;
        const int64_t a = c * kChunk, b = std::min(n, a + kChunk);
        for (int64_t i = a; i < b; ++i) {
          const int64_t t = t0 + i;
          const double* Xt = X + t * d;
          token_forward(Xt, d, P, k, Wk, Wv, K.data(), V.data(), A.data());
          double D = 0.0;
          for (int j = 0; j < k; ++j) {
            const double* g = Gt.data() + (int64_t)j * d;
            double s = 0.0;
            for (int e = 0; e < d; ++e) s += g[e] * V[e];
            dA[j] = s + dmass[j];
            D += A[j] * dA[j];
          }
          for (int e = 0; e < d; ++e) { dK[e] = 0.0; dV[e] = 0.0; }
          for (int j = 0; j < k; ++j) {
            const double dS = A[j] * (dA[j] - D);
            const double* pj = P + (int64_t)j * d;
            const double* g = Gt.data() + (int64_t)j * d;
            double* dpj = aP + (int64_t)j * d;
            for (int e = 0; e < d; ++e) {
              dK[e] += dS * pj[e] * inv_sqrt_d;
              dV[e] += A[j] * g[e];
              dpj[e] += dS * K[e] * inv_sqrt_d;
            }
          }
          double* dXt = dX + t * d;
          for (int c2 = 0; c2 < d; ++c2) {
            const double* wk = Wk + (int64_t)c2 * d;
            const double* wv = Wv + (int64_t)c2 * d;
            double s = 0.0;
            for (int e = 0; e < d; ++e) s += dK[e] * wk[e] + dV[e] * wv[e];
            dXt[c2] = s;
            double* rk = aWk + (int64_t)c2 * d;
            double* rv = aWv + (int64_t)c2 * d;
            for (int e = 0; e < d; ++e) { rk[e] += Xt[c2] * dK[e]; rv[e] += Xt[c2] * dV[e]; }
          }
        }
      }
      for (int64_t c = cb; c < ce; ++c) {
        const double* p = part.data() + (c - cb) * acc_len;
        for (int64_t i = 0; i < kd; ++i) dP[i] += p[i];
        for (int64_t i = 0; i < dd; ++i) { dWk[i] += p[kd + i]; dWv[i] += p[kd + dd + i]; }
      }
    }
  }
  return 0;
}

}  // extern "C"
