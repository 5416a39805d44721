// fb_svd_device.cu -- truncated SVD of dense biases on the GPU, for biases
// that are only known at call time (the "SVD decomposition" of FlashBias
// made per call; the rebuttal, reply to Reviewer xU4x, Q6, notes that online
// SVD of a dynamic bias is not an efficient design -- this makes its cost
// measurable).
//
// Algorithm per head (randomized range finder, Halko-Martinsson-Tropp 2011):
//   Omega: N x l Gaussian (l = R + oversample, <= 32);
//   Y = B Omega, Q = orth(Y); power_iters times: Z = orth(B^T Q), Q = orth(B Z);
//   M = B^T Q (so Q^T B = M^T); M^T M = W diag(sigma^2) W^T (Jacobi, fp64);
//   B ~ (Q W) diag(sigma) (M W diag(1/sigma))^T; the R largest give the
//   balanced factors phi_q = Q W_R diag(sqrt sigma), phi_k = M W_R diag(1/sqrt sigma).
// orth() is shifted CholeskyQR3 (Fukaya et al. 2020): three Gram / Cholesky /
// triangular-solve passes in fp64, the first with a diagonal shift so that
// the Gram matrix of an ill-conditioned Y stays positive definite.
// The tall N x l matrices are stored column-major ([l][N]) so that column
// sweeps are coalesced. The relative Frobenius error is computed exactly.
#include <algorithm>
#include <cmath>
#include <cstdint>

#include "fb_internal.h"

namespace fb {
namespace {

constexpr int kMaxL = 32;

// ------------------------------------------------------------------ kernels

// Counter-based Gaussian: splitmix64 at state seed + c * gamma (Steele, Lea
// and Flood 2014) for two uniforms, then Box-Muller.
__device__ __forceinline__ uint64_t splitmix(uint64_t s) {
  uint64_t z = s + 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

__global__ void gauss_kernel(int H, int N, int l, uint64_t seed, float *__restrict__ out) {
  const long long total = (long long)H * l * N;
  for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < total;
       idx += (long long)gridDim.x * blockDim.x) {
    const uint64_t a = splitmix(seed + uint64_t(2 * idx) * 0x9E3779B97F4A7C15ull);
    const uint64_t b = splitmix(seed + uint64_t(2 * idx + 1) * 0x9E3779B97F4A7C15ull);
    const double u1 = (double(a >> 11) + 0.5) * (1.0 / 9007199254740992.0);
    const double u2 = (double(b >> 11) + 0.5) * (1.0 / 9007199254740992.0);
    out[idx] = float(sqrt(-2.0 * log(u1)) * cos(6.283185307179586 * u2));
  }
}

// Y[h] = B[h] X[h]: B [N, N] row-major, X and Y [l][N]. One warp per row of
// B (16 rows per CTA); X is staged in shared memory 256 columns at a time.
__global__ void __launch_bounds__(512) bx_kernel(int N, int l, const float *__restrict__ B,
                                                 const float *__restrict__ X, float *__restrict__ Y) {
  __shared__ float xs[kMaxL][256];
  const int h = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long i = (long long)blockIdx.x * 16 + warp;
  const float *Bh = B + (long long)h * N * N;
  const float *Xh = X + (long long)h * l * N;
  float acc[kMaxL];
#pragma unroll
  for (int j = 0; j < kMaxL; ++j) acc[j] = 0.f;
  for (int c0 = 0; c0 < N; c0 += 256) {
    for (int e = threadIdx.x; e < l * 256; e += blockDim.x) {
      const int j = e / 256, t = e - j * 256;
      xs[j][t] = c0 + t < N ? Xh[(long long)j * N + c0 + t] : 0.f;
    }
    __syncthreads();
    if (i < N) {
#pragma unroll
      for (int m = 0; m < 8; ++m) {
        const int t = lane + 32 * m;
        const float bv = c0 + t < N ? Bh[i * N + c0 + t] : 0.f;
#pragma unroll
        for (int j = 0; j < kMaxL; ++j)
          if (j < l) acc[j] = fmaf(bv, xs[j][t], acc[j]);
      }
    }
    __syncthreads();
  }
  if (i < N) {
#pragma unroll
    for (int j = 0; j < kMaxL; ++j) {
      if (j >= l) break;
      float v = acc[j];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      if (lane == 0) Y[(long long)h * l * N + (long long)j * N + i] = v;
    }
  }
}

// Z[h] += B[h]^T X[h] over one slice of 512 rows of B (Z zeroed beforehand):
// one thread per column of B (128 per CTA), X staged in shared memory 64 rows
// at a time; grid (column blocks, H, row slices), partial sums added with
// atomics.
__global__ void __launch_bounds__(128) btx_kernel(int N, int l, const float *__restrict__ B,
                                                  const float *__restrict__ X, float *__restrict__ Z) {
  __shared__ float xs[kMaxL][64];
  const int h = blockIdx.y;
  const long long c = (long long)blockIdx.x * 128 + threadIdx.x;
  const float *Bh = B + (long long)h * N * N;
  const float *Xh = X + (long long)h * l * N;
  float acc[kMaxL];
#pragma unroll
  for (int j = 0; j < kMaxL; ++j) acc[j] = 0.f;
  const int i_end = min(N, int(blockIdx.z + 1) * 512);
  for (int i0 = int(blockIdx.z) * 512; i0 < i_end; i0 += 64) {
    for (int e = threadIdx.x; e < l * 64; e += blockDim.x) {
      const int j = e / 64, r = e - j * 64;
      xs[j][r] = i0 + r < N ? Xh[(long long)j * N + i0 + r] : 0.f;
    }
    __syncthreads();
    if (c < N) {
      const int rmax = min(64, i_end - i0);
      for (int r = 0; r < rmax; ++r) {
        const float bv = Bh[(long long)(i0 + r) * N + c];
#pragma unroll
        for (int j = 0; j < kMaxL; ++j)
          if (j < l) acc[j] = fmaf(bv, xs[j][r], acc[j]);
      }
    }
    __syncthreads();
  }
  if (c < N) {
    for (int j = 0; j < l; ++j) atomicAdd(&Z[(long long)h * l * N + (long long)j * N + c], acc[j]);
  }
}

// G[h] += A[h]^T A[h] over one chunk of 256 rows (A [l][N]); fp64 sums of
// exact fp64 products, added into G (zeroed beforehand) with atomics. Grid
// (row chunks, H); one thread per (a, b) pair with a <= b.
__global__ void __launch_bounds__(512) gram_kernel(int N, int l, const float *__restrict__ A,
                                                   double *__restrict__ G) {
  __shared__ float as[kMaxL][256];
  const int h = blockIdx.y;
  const long long i0 = (long long)blockIdx.x * 256;
  const float *Ah = A + (long long)h * l * N;
  for (int e = threadIdx.x; e < l * 256; e += blockDim.x) {
    const int j = e / 256, t = e - j * 256;
    as[j][t] = i0 + t < N ? Ah[(long long)j * N + i0 + t] : 0.f;
  }
  __syncthreads();
  const int npairs = l * (l + 1) / 2;
  for (int p = threadIdx.x; p < npairs; p += blockDim.x) {
    int a = 0, rem = p;
    while (rem >= l - a) {
      rem -= l - a;
      ++a;
    }
    const int b = a + rem;
    double s = 0.0;
    for (int t = 0; t < 256; ++t) s += double(as[a][t]) * double(as[b][t]);
    atomicAdd(&G[(long long)h * l * l + a * l + b], s);
    if (a != b) atomicAdd(&G[(long long)h * l * l + b * l + a], s);
  }
}

// T[h] = R^{-1} with R^T R = G + shift I (R upper triangular, Cholesky in
// fp64), so that A T has orthonormal columns. A pivot that is not positive
// (a column dependent on the previous ones) zeroes that column of T.
// One warp per head: lane i updates entry i of the current row of R, and
// lane j solves column j of the inverse.
__global__ void chol_kernel(int H, int N, int l, double shift_coef, const double *__restrict__ G,
                            double *__restrict__ T) {
  __shared__ double Rm[kMaxL][kMaxL];
  __shared__ bool dead[kMaxL];
  const int h = blockIdx.x, lane = threadIdx.x;
  if (h >= H) return;
  const double *g = G + (long long)h * l * l;
  double *t = T + (long long)h * l * l;
  double tr = 0.0;
  for (int a = 0; a < l; ++a) tr += g[a * l + a];
  const double shift = shift_coef * tr;
  for (int i = 0; i < l; ++i) Rm[i][lane] = 0.0;
  __syncwarp();
  for (int j = 0; j < l; ++j) {
    double dj = g[j * l + j] + shift;
    for (int k = 0; k < j; ++k) dj -= Rm[k][j] * Rm[k][j];
    const bool dj_dead = !(dj > 1e-300 && dj > 1e-14 * (g[j * l + j] + shift));
    const double rjj = dj_dead ? 0.0 : sqrt(dj);
    const int i = lane;  // row j of R, entry i > j
    double v = 0.0;
    if (i > j && i < l) {
      v = g[j * l + i];
      for (int k = 0; k < j; ++k) v -= Rm[k][j] * Rm[k][i];
    }
    __syncwarp();
    if (lane == 0) {
      dead[j] = dj_dead;
      Rm[j][j] = rjj;
    }
    if (i > j && i < l) Rm[j][i] = dj_dead ? 0.0 : v / rjj;
    __syncwarp();
  }
  // inverse of the upper triangular Rm: lane j back-substitutes column j
  const int j = lane;
  if (j < l) {
    for (int i = l - 1; i >= 0; --i) {
      if (i > j || dead[i]) {
        t[i * l + j] = 0.0;
        continue;
      }
      double v = (i == j) ? 1.0 : 0.0;
      for (int k = i + 1; k <= j; ++k) v -= Rm[i][k] * t[k * l + j];
      t[i * l + j] = v / Rm[i][i];
    }
  }
  (void)N;
}

// Out[h] = A[h] T[h] (A, Out [l][N], T [l][l] fp64); one thread per row.
__global__ void apply_kernel(int N, int l, const float *__restrict__ A, const double *__restrict__ T,
                             float *__restrict__ Out) {
  const int h = blockIdx.y;
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= N) return;
  const float *Ah = A + (long long)h * l * N;
  const double *t = T + (long long)h * l * l;
  double a[kMaxL];
#pragma unroll
  for (int k = 0; k < kMaxL; ++k) a[k] = k < l ? double(Ah[(long long)k * N + i]) : 0.0;
  for (int j = 0; j < l; ++j) {
    double s = 0.0;
#pragma unroll
    for (int k = 0; k < kMaxL; ++k)
      if (k <= j) s += a[k] * t[k * l + j];  // T is upper triangular
    Out[(long long)h * l * N + (long long)j * N + i] = float(s);
  }
}

// Symmetric eigen-decomposition of M = Z^T Z (fp64 cyclic Jacobi), then the
// coefficient matrices of the balanced factors: Cq = W_R diag(sqrt sigma),
// Ck = W_R diag(1 / sqrt sigma), sigma^2 the R largest eigenvalues;
// sig2[h] = sum of those sigma^2. One warp per head: every lane forms the
// rotation, lane k updates entry k of the two columns, rows and V columns.
__global__ void eig_kernel(int H, int l, int R, const double *__restrict__ Mg, double *__restrict__ Cq,
                           double *__restrict__ Ck, double *__restrict__ sig2) {
  __shared__ double A[kMaxL][kMaxL], V[kMaxL][kMaxL];
  __shared__ int order[kMaxL];
  const int h = blockIdx.x, k = threadIdx.x;
  if (h >= H) return;
  for (int i = 0; i < l; ++i) {
    if (k < l) {
      A[i][k] = Mg[(long long)h * l * l + i * l + k];
      V[i][k] = i == k ? 1.0 : 0.0;
    }
  }
  __syncwarp();
  for (int sweep = 0; sweep < 60; ++sweep) {
    double off = 0.0, diag = 0.0;
    if (k < l) {
      diag = A[k][k] * A[k][k];
      for (int j = k + 1; j < l; ++j) off += A[k][j] * A[k][j];
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      off += __shfl_xor_sync(0xffffffffu, off, o);
      diag += __shfl_xor_sync(0xffffffffu, diag, o);
    }
    if (off <= 1e-26 * diag || off == 0.0) break;
    for (int p = 0; p < l - 1; ++p) {
      for (int q = p + 1; q < l; ++q) {
        const double apq = A[p][q];
        if (fabs(apq) < 1e-300) continue;
        const double theta = (A[q][q] - A[p][p]) / (2.0 * apq);
        const double tt = (theta >= 0 ? 1.0 : -1.0) / (fabs(theta) + sqrt(theta * theta + 1.0));
        const double cs = 1.0 / sqrt(tt * tt + 1.0), sn = tt * cs;
        __syncwarp();
        if (k < l) {  // columns p, q
          const double akp = A[k][p], akq = A[k][q];
          A[k][p] = cs * akp - sn * akq;
          A[k][q] = sn * akp + cs * akq;
        }
        __syncwarp();
        if (k < l) {  // rows p, q
          const double apk = A[p][k], aqk = A[q][k];
          A[p][k] = cs * apk - sn * aqk;
          A[q][k] = sn * apk + cs * aqk;
          const double vkp = V[k][p], vkq = V[k][q];
          V[k][p] = cs * vkp - sn * vkq;
          V[k][q] = sn * vkp + cs * vkq;
        }
        __syncwarp();
      }
    }
  }
  // the R largest eigenvalues, in decreasing order (lane 0 picks them)
  if (k == 0) {
    bool used[kMaxL];
    for (int i = 0; i < l; ++i) used[i] = false;
    double s2 = 0.0;
    for (int r = 0; r < R; ++r) {
      int best = -1;
      for (int i = 0; i < l; ++i)
        if (!used[i] && (best < 0 || A[i][i] > A[best][best])) best = i;
      order[r] = best;
      if (best >= 0) {
        used[best] = true;
        s2 += fmax(A[best][best], 0.0);
      }
    }
    sig2[h] = s2;
  }
  __syncwarp();
  if (k < l) {
    for (int r = 0; r < R; ++r) {
      const int best = order[r];
      const double lam = best >= 0 ? fmax(A[best][best], 0.0) : 0.0;
      const double sigma = sqrt(lam);
      const double sq = sqrt(sigma), isq = sigma > 0.0 ? 1.0 / sqrt(sigma) : 0.0;
      const double w = best >= 0 ? V[k][best] : 0.0;
      Cq[((long long)h * l + k) * R + r] = w * sq;
      Ck[((long long)h * l + k) * R + r] = w * isq;
    }
  }
}

// phi[h, i, r] = sum_k A[h][k][i] C[h][k][r] (A [l][N], C [l][R] fp64,
// phi [H, N, R] fp32 row-major); one thread per row.
__global__ void rows_kernel(int N, int l, int R, const float *__restrict__ A, const double *__restrict__ C,
                            float *__restrict__ phi) {
  const int h = blockIdx.y;
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= N) return;
  const float *Ah = A + (long long)h * l * N;
  const double *ch = C + (long long)h * l * R;
  double a[kMaxL];
#pragma unroll
  for (int k = 0; k < kMaxL; ++k) a[k] = k < l ? double(Ah[(long long)k * N + i]) : 0.0;
  for (int r = 0; r < R; ++r) {
    double s = 0.0;
#pragma unroll
    for (int k = 0; k < kMaxL; ++k)
      if (k < l) s += a[k] * ch[k * R + r];
    phi[((long long)h * N + i) * R + r] = float(s);
  }
}

// sums[h] += (||B - phi_q phi_k^T||_F^2, ||B||_F^2), fp64; one warp per row,
// phi_k staged 256 rows at a time.
__global__ void __launch_bounds__(512) err_kernel(int N, int R, const float *__restrict__ B,
                                                  const float *__restrict__ pq, const float *__restrict__ pk,
                                                  double *__restrict__ sums) {
  __shared__ float ks[kMaxL][257];
  const int h = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long i = (long long)blockIdx.x * 16 + warp;
  const float *Bh = B + (long long)h * N * N;
  float q[kMaxL];
#pragma unroll
  for (int r = 0; r < kMaxL; ++r) q[r] = (i < N && r < R) ? pq[((long long)h * N + i) * R + r] : 0.f;
  double e2 = 0.0, f2 = 0.0;
  for (int c0 = 0; c0 < N; c0 += 256) {
    for (int e = threadIdx.x; e < 256 * R; e += blockDim.x) {
      const int t = e / R, r = e - t * R;
      ks[r][t] = c0 + t < N ? pk[((long long)h * N + c0 + t) * R + r] : 0.f;
    }
    __syncthreads();
    if (i < N) {
      for (int m = 0; m < 8; ++m) {
        const int t = lane + 32 * m;
        if (c0 + t >= N) break;
        float pred = 0.f;
#pragma unroll
        for (int r = 0; r < kMaxL; ++r)
          if (r < R) pred = fmaf(q[r], ks[r][t], pred);
        const float bv = Bh[i * N + c0 + t];
        const double dv = double(bv) - double(pred);
        e2 += dv * dv;
        f2 += double(bv) * double(bv);
      }
    }
    __syncthreads();
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    e2 += __shfl_xor_sync(0xffffffffu, e2, o);
    f2 += __shfl_xor_sync(0xffffffffu, f2, o);
  }
  if (lane == 0 && i < N) {
    atomicAdd(&sums[2 * h], e2);
    atomicAdd(&sums[2 * h + 1], f2);
  }
}

__global__ void finish_kernel(int H, const double *__restrict__ sums, const double *__restrict__ sig2,
                              double *__restrict__ out) {
  const int h = blockIdx.x * blockDim.x + threadIdx.x;
  if (h >= H) return;
  const double fro2 = sums[2 * h + 1];
  out[2 * h] = fro2 > 0.0 ? sqrt(sums[2 * h] / fro2) : 0.0;
  out[2 * h + 1] = fro2 > 0.0 ? fmin(sig2[h] / fro2, 1.0) : 1.0;
}

// ------------------------------------------------------------------ host side

struct SvdWs {
  size_t tall, small, total;  // bytes: one [H][l][N] fp32 buffer; the fp64 block
};

int svd_l(int N, int R, int oversample) {
  int l = R + (oversample > 0 ? oversample : 0);
  if (l > kMaxL) l = kMaxL;
  if (l > N) l = N;
  return l;
}

SvdWs svd_layout(int H, int N, int l, int R) {
  SvdWs w;
  w.tall = (size_t(H) * l * N * 4 + 255) & ~size_t(255);
  // G, T (l x l), Cq, Ck (l x R), sig2 (1), sums (2), out (2) per head, fp64
  w.small = (size_t(H) * (2 * l * l + 2 * l * R + 5) * 8 + 255) & ~size_t(255);
  w.total = 3 * w.tall + w.small;
  return w;
}

}  // namespace
}  // namespace fb

using namespace fb;

extern "C" size_t fb_svd_device_workspace_bytes(int H, int N, int R, int oversample) {
  if (H < 1 || N < 1 || R < 1 || R > kMaxL || R > N) return 0;
  return svd_layout(H, N, svd_l(N, R, oversample), R).total;
}

extern "C" int fb_svd_factors_device(int H, int N, int R, int oversample, int power_iters, uint64_t seed,
                                     const float *bias, float *phi_q, float *phi_k, double *err_energy,
                                     void *workspace, size_t workspace_bytes, void *stream) {
  if (!bias || !phi_q || !phi_k) return FB_ERR_INVALID_ARG;
  if (H < 1 || N < 1 || R < 1 || R > kMaxL || R > N || oversample < 0 || power_iters < 0 || power_iters > 16)
    return FB_ERR_UNSUPPORTED;
  if ((long long)N * N > (1ll << 40) || (long long)H * N > (1ll << 31)) return FB_ERR_UNSUPPORTED;
  if (((reinterpret_cast<uintptr_t>(bias) | reinterpret_cast<uintptr_t>(phi_q) |
        reinterpret_cast<uintptr_t>(phi_k)) & 3u) != 0)
    return FB_ERR_INVALID_ARG;
  if (err_energy && (reinterpret_cast<uintptr_t>(err_energy) & 7u) != 0) return FB_ERR_INVALID_ARG;
  const int l = svd_l(N, R, oversample);
  const SvdWs w = svd_layout(H, N, l, R);
  if (!workspace || workspace_bytes < w.total || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return FB_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t *ws = static_cast<uint8_t *>(workspace);
  float *P0 = reinterpret_cast<float *>(ws), *P1 = reinterpret_cast<float *>(ws + w.tall),
        *P2 = reinterpret_cast<float *>(ws + 2 * w.tall);
  double *G = reinterpret_cast<double *>(ws + 3 * w.tall);
  double *T = G + size_t(H) * l * l;
  double *Cq = T + size_t(H) * l * l;
  double *Ck = Cq + size_t(H) * l * R;
  double *sig2 = Ck + size_t(H) * l * R;
  double *sums = sig2 + H;
  double *out = sums + 2 * H;

  const dim3 rows16((N + 15) / 16, H), cols128((N + 127) / 128, H, (N + 511) / 512), rows256((N + 255) / 256, H);
  const double u = 1.1102230246251565e-16;  // 2^-53: unit roundoff of the fp64 Gram matrices
  const double shift_coef = 11.0 * (double(N) * l + double(l) * (l + 1)) * u;
  const int hb = (H + 31) / 32;
  // orth(A) -> out via shifted CholeskyQR3; A and tmp are clobbered
  const dim3 chunks256((N + 255) / 256, H);
  auto gram = [&](const float *A) {
    cudaMemsetAsync(G, 0, size_t(H) * l * l * sizeof(double), st);
    gram_kernel<<<chunks256, 512, 0, st>>>(N, l, A, G);
  };
  auto orth = [&](float *A, float *tmp, float *outp) {
    gram(A);
    chol_kernel<<<H, 32, 0, st>>>(H, N, l, shift_coef, G, T);
    apply_kernel<<<rows256, 256, 0, st>>>(N, l, A, T, tmp);
    gram(tmp);
    chol_kernel<<<H, 32, 0, st>>>(H, N, l, 0.0, G, T);
    apply_kernel<<<rows256, 256, 0, st>>>(N, l, tmp, T, A);
    gram(A);
    chol_kernel<<<H, 32, 0, st>>>(H, N, l, 0.0, G, T);
    apply_kernel<<<rows256, 256, 0, st>>>(N, l, A, T, outp);
  };
  const long long ng = (long long)H * l * N;
  gauss_kernel<<<int(std::min<long long>((ng + 255) / 256, 148 * 16)), 256, 0, st>>>(H, N, l, seed, P1);
  bx_kernel<<<rows16, 512, 0, st>>>(N, l, bias, P1, P0);  // Y = B Omega
  orth(P0, P1, P2);                                         // Q in P2
  for (int it = 0; it < power_iters; ++it) {
    cudaMemsetAsync(P0, 0, size_t(H) * l * N * sizeof(float), st);
    btx_kernel<<<cols128, 128, 0, st>>>(N, l, bias, P2, P0);  // Z = B^T Q
    orth(P0, P2, P1);                                         // Z orthonormal in P1
    bx_kernel<<<rows16, 512, 0, st>>>(N, l, bias, P1, P0);   // Y = B Z
    orth(P0, P1, P2);                                         // Q in P2
  }
  cudaMemsetAsync(P0, 0, size_t(H) * l * N * sizeof(float), st);
  btx_kernel<<<cols128, 128, 0, st>>>(N, l, bias, P2, P0);  // M = B^T Q
  gram(P0);                                                 // M^T M
  eig_kernel<<<H, 32, 0, st>>>(H, l, R, G, Cq, Ck, sig2);
  rows_kernel<<<rows256, 256, 0, st>>>(N, l, R, P2, Cq, phi_q);
  rows_kernel<<<rows256, 256, 0, st>>>(N, l, R, P0, Ck, phi_k);
  if (err_energy) {
    if (cudaMemsetAsync(sums, 0, size_t(2) * H * sizeof(double), st) != cudaSuccess) return FB_ERR_CUDA;
    err_kernel<<<rows16, 512, 0, st>>>(N, R, bias, phi_q, phi_k, sums);
    finish_kernel<<<hb, 32, 0, st>>>(H, sums, sig2, out);
    if (cudaMemcpyAsync(err_energy, out, size_t(2) * H * sizeof(double), cudaMemcpyDeviceToDevice, st) !=
        cudaSuccess)
      return FB_ERR_CUDA;
  }
  return cudaGetLastError() == cudaSuccess ? FB_OK : FB_ERR_CUDA;
}
