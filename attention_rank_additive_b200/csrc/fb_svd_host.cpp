// fb_svd_host.cpp -- truncated SVD of a static dense bias on the host, the
// "SVD decomposition" of FlashBias (rebuttal, reply to Reviewer xU4x, Q6: the
// rank of each head is chosen from its singular values; decomposing once is
// fine for a static bias, while per-inference SVD of a dynamic bias is not
// an efficient design).
//
// Algorithm (randomized range finder, Halko-Martinsson-Tropp 2011, then an
// exact SVD of the small projected matrix by one-sided Jacobi rotations,
// Hestenes 1958):
//   1. Omega: N x l Gaussian, l = R + oversample (clamped to N).
//   2. Y = B Omega; orthonormalise -> Qm.  power_iters times:
//      Z = B^T Qm, orthonormalise; Y = B Z, orthonormalise -> Qm.
//   3. M = B^T Qm (N x l), so Qm^T B = M^T.
//   4. One-sided Jacobi on the columns of M: M J = W with orthogonal columns,
//      sigma_c = |W_c|, so Qm^T B = J Sigma Vhat^T with Vhat = W / sigma.
//   5. B ~ (Qm J) Sigma Vhat^T; keep the R largest: phi_q = U_R sqrt(S_R),
//      phi_k = V_R sqrt(S_R).
// The relative Frobenius error is then computed exactly against B.
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <thread>
#include <vector>

#include "../../include/flashbias.h"

namespace {

// splitmix64 (Steele, Lea, Flood 2014) for the seeded Gaussian test matrix.
struct SplitMix64 {
  uint64_t s;
  uint64_t next() {
    uint64_t z = (s += 0x9E3779B97F4A7C15ull);
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
  }
  double uniform() { return (double((next() >> 11)) + 0.5) * (1.0 / 9007199254740992.0); }
};

int worker_count() {
  unsigned n = std::thread::hardware_concurrency();
  return int(std::max(1u, std::min(n, 64u)));
}

template <class F>
void parallel_rows(int64_t n, F f) {
  const int nt = worker_count();
  if (nt <= 1 || n < 64) {
    f(int64_t(0), n);
    return;
  }
  std::vector<std::thread> th;
  const int64_t chunk = (n + nt - 1) / nt;
  for (int t = 0; t < nt; ++t) {
    const int64_t a = t * chunk, e = std::min(n, a + chunk);
    if (a >= e) break;
    th.emplace_back([=]() { f(a, e); });
  }
  for (auto &x : th) x.join();
}

// Y[N, l] = A[N, N] X[N, l]   (A row-major)
void mat_mul(const double *A, const double *X, double *Y, int64_t N, int l) {
  parallel_rows(N, [&](int64_t r0, int64_t r1) {
    for (int64_t i = r0; i < r1; ++i) {
      double *y = Y + i * l;
      std::fill(y, y + l, 0.0);
      const double *a = A + i * N;
      for (int64_t k = 0; k < N; ++k) {
        const double s = a[k];
        const double *x = X + k * l;
        for (int c = 0; c < l; ++c) y[c] += s * x[c];
      }
    }
  });
}

// Y[N, l] = A^T X   (A row-major N x N): accumulate per thread, then reduce.
void mat_mul_t(const double *A, const double *X, double *Y, int64_t N, int l) {
  const int nt = worker_count();
  std::vector<std::vector<double>> part(nt, std::vector<double>(size_t(N) * l, 0.0));
  std::vector<std::thread> th;
  const int64_t chunk = (N + nt - 1) / nt;
  for (int t = 0; t < nt; ++t) {
    th.emplace_back([&, t]() {
      const int64_t a0 = t * chunk, a1 = std::min(N, a0 + chunk);
      double *py = part[t].data();
      for (int64_t k = a0; k < a1; ++k) {  // row k of A contributes A[k, i] * X[k, :] to Y[i, :]
        const double *a = A + k * N;
        const double *x = X + k * l;
        for (int64_t i = 0; i < N; ++i) {
          const double s = a[i];
          double *y = py + i * l;
          for (int c = 0; c < l; ++c) y[c] += s * x[c];
        }
      }
    });
  }
  for (auto &x : th) x.join();
  parallel_rows(N, [&](int64_t r0, int64_t r1) {
    for (int64_t i = r0; i < r1; ++i)
      for (int c = 0; c < l; ++c) {
        double s = 0.0;
        for (int t = 0; t < nt; ++t) s += part[t][i * l + c];
        Y[i * l + c] = s;
      }
  });
}

// Orthonormalise the l columns of Y [N, l] (row-major) by modified
// Gram-Schmidt, done twice. Columns that vanish are replaced by zeros.
void orthonormalise(double *Y, int64_t N, int l) {
  for (int pass = 0; pass < 2; ++pass)
    for (int c = 0; c < l; ++c) {
      for (int p = 0; p < c; ++p) {
        double dot = 0.0;
        for (int64_t i = 0; i < N; ++i) dot += Y[i * l + p] * Y[i * l + c];
        for (int64_t i = 0; i < N; ++i) Y[i * l + c] -= dot * Y[i * l + p];
      }
      double nrm = 0.0;
      for (int64_t i = 0; i < N; ++i) nrm += Y[i * l + c] * Y[i * l + c];
      nrm = std::sqrt(nrm);
      const double inv = nrm > 0.0 ? 1.0 / nrm : 0.0;
      for (int64_t i = 0; i < N; ++i) Y[i * l + c] *= inv;
    }
}

}  // namespace

extern "C" int fb_svd_factors_host(const double *B, int N, int R, int oversample, int power_iters, uint64_t seed,
                                   float *phi_q, float *phi_k, double *rel_fro_err, double *energy) {
  if (!B || !phi_q || !phi_k || N < 1 || R < 1 || R > 128 || R > N || oversample < 0 || power_iters < 0 ||
      power_iters > 64)
    return FB_ERR_INVALID_ARG;
  try {
    const int64_t n = N;
    const int l = int(std::min<int64_t>(n, int64_t(R) + oversample));
    std::vector<double> Om(size_t(n) * l), Y(size_t(n) * l), Z(size_t(n) * l);
    SplitMix64 rng{seed};
    for (size_t i = 0; i < Om.size(); i += 2) {  // Box-Muller pairs
      const double u1 = rng.uniform(), u2 = rng.uniform();
      const double rad = std::sqrt(-2.0 * std::log(u1)), th = 6.283185307179586 * u2;
      Om[i] = rad * std::cos(th);
      if (i + 1 < Om.size()) Om[i + 1] = rad * std::sin(th);
    }
    mat_mul(B, Om.data(), Y.data(), n, l);
    orthonormalise(Y.data(), n, l);
    for (int it = 0; it < power_iters; ++it) {
      mat_mul_t(B, Y.data(), Z.data(), n, l);
      orthonormalise(Z.data(), n, l);
      mat_mul(B, Z.data(), Y.data(), n, l);
      orthonormalise(Y.data(), n, l);
    }
    // M = B^T Qm  (N x l), column-major copy for the rotations.
    mat_mul_t(B, Y.data(), Z.data(), n, l);
    std::vector<double> Mc(size_t(n) * l), J(size_t(l) * l, 0.0);
    for (int64_t i = 0; i < n; ++i)
      for (int c = 0; c < l; ++c) Mc[size_t(c) * n + i] = Z[i * l + c];
    for (int c = 0; c < l; ++c) J[size_t(c) * l + c] = 1.0;  // column-major l x l
    for (int sweep = 0; sweep < 80; ++sweep) {
      bool rotated = false;
      for (int p = 0; p < l - 1; ++p)
        for (int q = p + 1; q < l; ++q) {
          double *mp = &Mc[size_t(p) * n], *mq = &Mc[size_t(q) * n];
          double a = 0.0, bb = 0.0, g = 0.0;
          for (int64_t i = 0; i < n; ++i) {
            a += mp[i] * mp[i];
            bb += mq[i] * mq[i];
            g += mp[i] * mq[i];
          }
          if (std::fabs(g) <= 1e-12 * std::sqrt(a * bb) || g == 0.0) continue;
          rotated = true;
          const double zeta = (bb - a) / (2.0 * g);
          const double t = (zeta >= 0 ? 1.0 : -1.0) / (std::fabs(zeta) + std::sqrt(1.0 + zeta * zeta));
          const double cs = 1.0 / std::sqrt(1.0 + t * t), sn = cs * t;
          for (int64_t i = 0; i < n; ++i) {
            const double x = mp[i], y = mq[i];
            mp[i] = cs * x - sn * y;
            mq[i] = sn * x + cs * y;
          }
          double *jp = &J[size_t(p) * l], *jq = &J[size_t(q) * l];
          for (int i = 0; i < l; ++i) {
            const double x = jp[i], y = jq[i];
            jp[i] = cs * x - sn * y;
            jq[i] = sn * x + cs * y;
          }
        }
      if (!rotated) break;
    }
    std::vector<double> sig(l);
    std::vector<int> order(l);
    for (int c = 0; c < l; ++c) {
      double s = 0.0;
      for (int64_t i = 0; i < n; ++i) s += Mc[size_t(c) * n + i] * Mc[size_t(c) * n + i];
      sig[c] = std::sqrt(s);
      order[c] = c;
    }
    std::stable_sort(order.begin(), order.end(), [&](int x, int y) { return sig[x] > sig[y]; });
    // Left vectors U = Qm J (N x l), right vectors V = W / sigma.
    std::vector<double> pq(size_t(n) * R), pk(size_t(n) * R);
    for (int r = 0; r < R; ++r) {
      const int c = order[r];
      const double s = sig[c], root = std::sqrt(s);
      const double *jc = &J[size_t(c) * l];
      const double *wc = &Mc[size_t(c) * n];
      for (int64_t i = 0; i < n; ++i) {
        double u = 0.0;
        for (int k = 0; k < l; ++k) u += Y[i * l + k] * jc[k];
        pq[i * R + r] = u * root;
        pk[i * R + r] = s > 0.0 ? wc[i] / s * root : 0.0;
      }
    }
    // Exact error of the truncation, and the captured energy.
    std::vector<double> err_part(size_t(worker_count()) + 1, 0.0), tot_part(size_t(worker_count()) + 1, 0.0);
    {
      const int nt = worker_count();
      std::vector<std::thread> th;
      const int64_t chunk = (n + nt - 1) / nt;
      for (int t = 0; t < nt; ++t)
        th.emplace_back([&, t]() {
          const int64_t r0 = t * chunk, r1 = std::min(n, r0 + chunk);
          double e = 0.0, tt = 0.0;
          for (int64_t i = r0; i < r1; ++i)
            for (int64_t j = 0; j < n; ++j) {
              double a = 0.0;
              for (int r = 0; r < R; ++r) a += pq[i * R + r] * pk[j * R + r];
              const double bij = B[i * n + j];
              e += (bij - a) * (bij - a);
              tt += bij * bij;
            }
          err_part[t] = e;
          tot_part[t] = tt;
        });
      for (auto &x : th) x.join();
    }
    double err2 = 0.0, tot2 = 0.0;
    for (size_t t = 0; t < err_part.size(); ++t) {
      err2 += err_part[t];
      tot2 += tot_part[t];
    }
    double cap = 0.0;
    for (int r = 0; r < R; ++r) cap += sig[order[r]] * sig[order[r]];
    if (rel_fro_err) *rel_fro_err = tot2 > 0.0 ? std::sqrt(err2 / tot2) : 0.0;
    if (energy) *energy = tot2 > 0.0 ? std::min(1.0, cap / tot2) : 1.0;
    for (size_t i = 0; i < pq.size(); ++i) {
      phi_q[i] = float(pq[i]);
      phi_k[i] = float(pk[i]);
    }
    return FB_OK;
  } catch (...) {
    return FB_ERR_INVALID_ARG;
  }
}
