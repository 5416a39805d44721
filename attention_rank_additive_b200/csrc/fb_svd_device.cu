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

// Stage columns c0 .. c0+W-1 of the l rows of a [l][N] fp32 matrix into
// shared memory (row pitch W), zero outside the matrix. Each of the NT
// threads owns whole 16-byte pieces and issues all of its loads before its
// stores, so a chunk costs one memory latency, not one per element. Needs
// NT * 4 * K == kMaxL * W for some K.
template <int W, int NT>
__device__ __forceinline__ void stage_rows(float (*xs)[W], const float *__restrict__ A, int l, int N, long long c0,
                                           long long c_end) {
  constexpr int PIECES = kMaxL * W / 4;  // 16-byte pieces of a full kMaxL x W tile
  constexpr int K = PIECES / NT;
  static_assert(K * NT == PIECES, "staging split");
  const bool vec = (N & 3) == 0 && (reinterpret_cast<uintptr_t>(A) & 15u) == 0;
  float4 v[K];
#pragma unroll
  for (int k = 0; k < K; ++k) {
    const int piece = k * NT + int(threadIdx.x);
    const int j = piece / (W / 4), t = (piece - j * (W / 4)) * 4;
    const long long c = c0 + t;
    if (j < l && vec && c + 3 < c_end) {
      v[k] = *reinterpret_cast<const float4 *>(A + (long long)j * N + c);
    } else {
      float e[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) e[q] = (j < l && c + q < c_end) ? A[(long long)j * N + c + q] : 0.f;
      v[k] = make_float4(e[0], e[1], e[2], e[3]);
    }
  }
#pragma unroll
  for (int k = 0; k < K; ++k) {
    const int piece = k * NT + int(threadIdx.x);
    const int j = piece / (W / 4), t = (piece - j * (W / 4)) * 4;
    *reinterpret_cast<float4 *>(&xs[j][t]) = v[k];
  }
}

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

// Y[h] = B[h] X[h]: B [N, N] row-major, X and Y [l][N]. A CTA of 8 warps
// takes 8 kBxRows rows of B, each warp kBxRows of them; X is staged in shared
// memory 256 columns at a time and each lane works on 4 consecutive columns,
// so one 16-byte shared load of X feeds 4 kBxRows FMAs and each row's 16-byte
// loads of B are coalesced across the warp. The per-lane partial sums are
// reduced across the warp at the end.
// Rows of B per warp (B X) and columns of B per thread (B^T X): 2 each keeps
// a thread under 128 registers, so that two CTAs share an SM (4 each: one
// CTA of 8 warps per SM, about 4 % slower over the whole SVD).
#ifndef FB_SVD_BX_ROWS
#define FB_SVD_BX_ROWS 2
#endif
#ifndef FB_SVD_BTX_COLS
#define FB_SVD_BTX_COLS 2
#endif
constexpr int kBxRows = FB_SVD_BX_ROWS;  // rows per warp
constexpr int kBtxCols = FB_SVD_BTX_COLS;  // columns per thread
__global__ void __launch_bounds__(256, kBxRows <= 2 ? 2 : 1) bx_kernel(int N, int l, const float *__restrict__ B,
                                                                      const float *__restrict__ X,
                                                                      float *__restrict__ Y) {
  __shared__ __align__(16) float xs[kMaxL][256];
  const int h = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long i0 = (long long)blockIdx.x * (8 * kBxRows) + warp * kBxRows;
  const float *Bh = B + (long long)h * N * N;
  const float *Xh = X + (long long)h * l * N;
  // rows of B start on 16-byte boundaries: 16-byte loads
  const bool vec = (N & 3) == 0 && (reinterpret_cast<uintptr_t>(B) & 15u) == 0;
  float acc[kBxRows][kMaxL];
#pragma unroll
  for (int r = 0; r < kBxRows; ++r)
#pragma unroll
    for (int j = 0; j < kMaxL; ++j) acc[r][j] = 0.f;
  for (int c0 = 0; c0 < N; c0 += 256) {
    // this chunk's B values first (they stream from HBM while X is staged)
    float bv2[2][kBxRows][4];
#pragma unroll
    for (int m = 0; m < 2; ++m) {
      const int t = 128 * m + 4 * lane;  // this lane's 4 columns of the chunk
#pragma unroll
      for (int r = 0; r < kBxRows; ++r) {
        const long long i = i0 + r;
        const long long c = c0 + t;
        if (i < N && vec && c + 3 < N) {
          const float4 b4 = *reinterpret_cast<const float4 *>(Bh + i * N + c);
          bv2[m][r][0] = b4.x, bv2[m][r][1] = b4.y, bv2[m][r][2] = b4.z, bv2[m][r][3] = b4.w;
        } else {
#pragma unroll
          for (int q = 0; q < 4; ++q) bv2[m][r][q] = (i < N && c + q < N) ? Bh[i * N + c + q] : 0.f;
        }
      }
    }
    stage_rows<256, 256>(xs, Xh, l, N, c0, N);
    __syncthreads();
#pragma unroll
    for (int m = 0; m < 2; ++m) {
      const int t = 128 * m + 4 * lane;  // this lane's 4 columns of the chunk
      const float(&bv)[kBxRows][4] = bv2[m];
#pragma unroll
      for (int j = 0; j < kMaxL; ++j) {
        if (j < l) {
          const float4 x4 = *reinterpret_cast<const float4 *>(&xs[j][t]);
#pragma unroll
          for (int r = 0; r < kBxRows; ++r) {
            float a = acc[r][j];
            a = fmaf(bv[r][0], x4.x, a);
            a = fmaf(bv[r][1], x4.y, a);
            a = fmaf(bv[r][2], x4.z, a);
            a = fmaf(bv[r][3], x4.w, a);
            acc[r][j] = a;
          }
        }
      }
    }
    __syncthreads();
  }
#pragma unroll
  for (int r = 0; r < kBxRows; ++r) {
    const long long i = i0 + r;
#pragma unroll
    for (int j = 0; j < kMaxL; ++j) {
      if (j >= l) break;
      float v = acc[r][j];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      if (lane == 0 && i < N) Y[(long long)h * l * N + (long long)j * N + i] = v;
    }
  }
}

// Z[h] += B[h]^T X[h] over one slice of 512 rows of B (Z zeroed beforehand):
// each thread takes kBtxCols consecutive columns of B (256 threads per CTA)
// and walks the slice 4 rows at a time, X staged in shared memory 64 rows at
// a time, so that one 16-byte broadcast load of X (4 rows of one column of X)
// feeds 4 kBtxCols FMAs; grid (column blocks, H, row slices), partial sums
// added with atomics.
__global__ void __launch_bounds__(256, kBtxCols <= 2 ? 2 : 1) btx_kernel(int N, int l, const float *__restrict__ B,
                                                                         const float *__restrict__ X,
                                                                         float *__restrict__ Z) {
  constexpr int CQ = kBtxCols;
  __shared__ __align__(16) float xs[kMaxL][64];
  const int h = blockIdx.y;
  const long long c = ((long long)blockIdx.x * 256 + threadIdx.x) * CQ;  // first of this thread's CQ columns
  const float *Bh = B + (long long)h * N * N;
  const float *Xh = X + (long long)h * l * N;
  const bool vec = (N % CQ) == 0 && (reinterpret_cast<uintptr_t>(B) % (4 * CQ)) == 0;
  float acc[CQ][kMaxL];
#pragma unroll
  for (int q = 0; q < CQ; ++q)
#pragma unroll
    for (int j = 0; j < kMaxL; ++j) acc[q][j] = 0.f;
  const int i_end = min(N, int(blockIdx.z + 1) * 512);
  for (int i0 = int(blockIdx.z) * 512; i0 < i_end; i0 += 64) {
    stage_rows<64, 256>(xs, Xh, l, N, i0, i_end);
    __syncthreads();
    if (c < N) {
      const int rmax = min(64, i_end - i0);
      // B values of 4 rows x this thread's 4 columns; the next group's are
      // loaded before the current group's FMAs
      auto load4 = [&](int r, float (&bv)[4][CQ]) {
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const long long i = i0 + r + u;
          if (r + u < rmax && vec && c + CQ - 1 < N) {
            if constexpr (CQ == 4) {
              const float4 b4 = *reinterpret_cast<const float4 *>(Bh + i * N + c);
              bv[u][0] = b4.x, bv[u][1] = b4.y, bv[u][2] = b4.z, bv[u][3] = b4.w;
            } else {
              const float2 b2 = *reinterpret_cast<const float2 *>(Bh + i * N + c);
              bv[u][0] = b2.x, bv[u][1] = b2.y;
            }
          } else {
#pragma unroll
            for (int q = 0; q < CQ; ++q) bv[u][q] = (r + u < rmax && c + q < N) ? Bh[i * N + c + q] : 0.f;
          }
        }
      };
      float nb[4][CQ];
      load4(0, nb);
      for (int r = 0; r < rmax; r += 4) {
        float bv[4][CQ];  // [row][column]
#pragma unroll
        for (int u = 0; u < 4; ++u)
#pragma unroll
          for (int q = 0; q < CQ; ++q) bv[u][q] = nb[u][q];
        if (r + 4 < rmax) load4(r + 4, nb);
#pragma unroll
        for (int j = 0; j < kMaxL; ++j) {
          if (j < l) {
            const float4 x4 = *reinterpret_cast<const float4 *>(&xs[j][r]);  // rows r .. r+3 (zero past the slice)
#pragma unroll
            for (int q = 0; q < CQ; ++q) {
              float a = acc[q][j];
              a = fmaf(bv[0][q], x4.x, a);
              a = fmaf(bv[1][q], x4.y, a);
              a = fmaf(bv[2][q], x4.z, a);
              a = fmaf(bv[3][q], x4.w, a);
              acc[q][j] = a;
            }
          }
        }
      }
    }
    __syncthreads();
  }
#pragma unroll
  for (int q = 0; q < CQ; ++q) {
#pragma unroll
    for (int j = 0; j < kMaxL; ++j)  // compile-time indices keep acc in registers
      if (j < l && c + q < N) atomicAdd(&Z[(long long)h * l * N + (long long)j * N + c + q], acc[q][j]);
  }
}

// G[h] += A[h]^T A[h] over one chunk of 256 rows (A [l][N]); fp64 sums of
// exact fp64 products, added into G (zeroed beforehand) with atomics. Grid
// (row chunks, H); one thread per (a, b) pair with a <= b.
__global__ void __launch_bounds__(512) gram_kernel(int N, int l, const float *__restrict__ A,
                                                   double *__restrict__ G) {
  __shared__ float as[kMaxL][257];  // padded: threads of one warp read different rows at the same t
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
    double s4[4] = {0.0, 0.0, 0.0, 0.0};  // independent chains
    for (int t = 0; t < 256; t += 4) {
#pragma unroll
      for (int u = 0; u < 4; ++u) s4[u] += double(as[a][t + u]) * double(as[b][t + u]);
    }
    const double s = (s4[0] + s4[1]) + (s4[2] + s4[3]);
    atomicAdd(&G[(long long)h * l * l + a * l + b], s);
    if (a != b) atomicAdd(&G[(long long)h * l * l + b * l + a], s);
  }
}

// T[h] = R^{-1} with R^T R = G + shift I (R upper triangular, Cholesky in
// fp64), so that A T has orthonormal columns. A pivot that is not positive
// (a column dependent on the previous ones) zeroes that column of T.
// One warp per head, all in registers: lane i holds row i of the (trailing)
// matrix and, after step j, R[j][i]; each step broadcasts row j of R with
// shuffles and updates the trailing rows (right-looking). Then lane j
// back-substitutes column j of the inverse.
__device__ __forceinline__ double shfl_d(double v, int src) { return __shfl_sync(0xffffffffu, v, src); }
__global__ void __launch_bounds__(32) chol_kernel(int H, int N, int l, double shift_coef,
                                                  const double *__restrict__ G, double *__restrict__ T) {
  const int h = blockIdx.x, lane = threadIdx.x;
  if (h >= H) return;
  const double *g = G + (long long)h * l * l;
  double a[kMaxL];  // row `lane` of G + shift I, then of the trailing matrix
#pragma unroll
  for (int k = 0; k < kMaxL; ++k) a[k] = (lane < l && k < l) ? g[lane * l + k] : 0.0;
  double diag = 0.0;
#pragma unroll
  for (int k = 0; k < kMaxL; ++k)
    if (k == lane) diag = a[k];
  double tr = diag;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) tr += __shfl_xor_sync(0xffffffffu, tr, o);
  const double shift = shift_coef * tr;
  const double gdiag = diag + shift;  // this row's pivot before elimination
#pragma unroll
  for (int k = 0; k < kMaxL; ++k)
    if (k == lane) a[k] += shift;
  double r[kMaxL];  // r[j] = R[j][lane]
  uint32_t dead = 0u;  // bit j: pivot j not positive (the same in every lane)
#pragma unroll
  for (int j = 0; j < kMaxL; ++j) {
    r[j] = 0.0;
    if (j < l) {
      const double ajj = shfl_d(a[j], j);
      const double gjj = shfl_d(gdiag, j);
      const bool dj_dead = !(ajj > 1e-300 && ajj > 1e-14 * gjj);
      if (dj_dead) dead |= 1u << j;
      const double rjj = dj_dead ? 0.0 : sqrt(ajj);
      // lane i > j holds A[i][j] = A[j][i]
      const double rji = lane == j ? rjj : ((lane > j && lane < l && !dj_dead) ? a[j] / rjj : 0.0);
      r[j] = rji;
#pragma unroll
      for (int k = j + 1; k < kMaxL; ++k) {
        const double rjk = shfl_d(rji, k);
        if (lane > j) a[k] -= rji * rjk;
      }
    }
  }
  // inverse of R: lane j back-substitutes column j (t[i] = T[i][lane])
  double t[kMaxL];
#pragma unroll
  for (int i = 0; i < kMaxL; ++i) t[i] = 0.0;
#pragma unroll
  for (int i = kMaxL - 1; i >= 0; --i) {
    if (i < l) {
      const double rii = shfl_d(r[i], i);
      double v = (i == lane) ? 1.0 : 0.0;
#pragma unroll
      for (int k = i + 1; k < kMaxL; ++k) v -= shfl_d(r[i], k) * t[k];  // R[i][k], zero past l
      t[i] = (i <= lane && !((dead >> i) & 1u)) ? v / rii : 0.0;
    }
  }
  if (lane < l) {
    double *out = T + (long long)h * l * l;
#pragma unroll
    for (int i = 0; i < kMaxL; ++i)
      if (i < l) out[i * l + lane] = t[i];
  }
  (void)N;
}

// Out[h] = A[h] T[h] (A, Out [l][N], T [l][l] fp64); one thread per row.
__global__ void apply_kernel(int N, int l, const float *__restrict__ A, const double *__restrict__ T,
                             float *__restrict__ Out) {
  __shared__ double t[kMaxL * kMaxL];
  const int h = blockIdx.y;
  for (int e = threadIdx.x; e < l * l; e += blockDim.x) t[e] = T[(long long)h * l * l + e];
  __syncthreads();
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= N) return;
  const float *Ah = A + (long long)h * l * N;
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

// Symmetric eigen-decomposition of M = Z^T Z (fp64 Jacobi), then the
// coefficient matrices of the balanced factors: Cq = W_R diag(sqrt sigma),
// Ck = W_R diag(1 / sqrt sigma), sigma^2 the R largest eigenvalues;
// sig2[h] = sum of those sigma^2. One warp per head, parallel ordering: the
// matrix is padded to an even size n and each sweep is n - 1 rounds of the
// round-robin pairing (index 0 fixed, the others rotating), whose n / 2
// pairs are disjoint, so their rotations commute: all angles are taken from
// the current matrix, then every column pair is rotated (lane k: row k),
// then every row pair (lane k: column k), and the eigenvector columns.
__global__ void eig_kernel(int H, int l, int R, const double *__restrict__ Mg, double *__restrict__ Cq,
                           double *__restrict__ Ck, double *__restrict__ sig2) {
  // rows padded by one entry: lane k walking row k of A or V then hits its own bank
  __shared__ double A[kMaxL][kMaxL + 1], V[kMaxL][kMaxL + 1];
  __shared__ double cs_s[kMaxL / 2], sn_s[kMaxL / 2];
  __shared__ int pp_s[kMaxL / 2], qq_s[kMaxL / 2];
  __shared__ int order[kMaxL];
  const int h = blockIdx.x, k = threadIdx.x;
  if (h >= H) return;
  const int n = (l + 1) & ~1;  // padded size (the pad row and column stay zero)
  for (int i = 0; i < n; ++i) {
    if (k < n) {
      A[i][k] = (i < l && k < l) ? Mg[(long long)h * l * l + i * l + k] : 0.0;
      V[i][k] = i == k ? 1.0 : 0.0;
    }
  }
  __syncwarp();
  // A rotation is skipped when |a_pq| is at rounding level next to the
  // largest diagonal entry (the leading eigenpairs, the only ones used, are
  // then converged); the iteration stops after a sweep without one.
  for (int sweep = 0; sweep < 40; ++sweep) {
    bool rotated = false;
    double dmax = k < n ? fabs(A[k][k]) : 0.0;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) dmax = fmax(dmax, __shfl_xor_sync(0xffffffffu, dmax, o));
    const double tol = 1e-15 * dmax;
    for (int round = 0; round < n - 1; ++round) {
      // pair m of this round: positions m and n-1-m of the sequence
      // [0, (round + 0) .. (round + n - 2) mod (n - 1) + 1]
      if (k < n / 2) {
        auto member = [&](int pos) { return pos == 0 ? 0 : ((pos - 1 + round) % (n - 1)) + 1; };
        int p = member(k), q = member(n - 1 - k);
        if (p > q) {
          const int t = p;
          p = q;
          q = t;
        }
        const double apq = A[p][q];
        double c = 1.0, sn = 0.0;
        if (fabs(apq) >= 1e-300 && fabs(apq) > tol) {
          rotated = true;
          const double theta = (A[q][q] - A[p][p]) / (2.0 * apq);
          const double tt = (theta >= 0 ? 1.0 : -1.0) / (fabs(theta) + sqrt(theta * theta + 1.0));
          c = 1.0 / sqrt(tt * tt + 1.0);
          sn = tt * c;
        }
        pp_s[k] = p;
        qq_s[k] = q;
        cs_s[k] = c;
        sn_s[k] = sn;
      }
      __syncwarp();
      if (k < n) {  // columns p, q of row k; eigenvector columns of row k
        for (int m = 0; m < n / 2; ++m) {
          const int p = pp_s[m], q = qq_s[m];
          const double c = cs_s[m], sn = sn_s[m];
          const double akp = A[k][p], akq = A[k][q];
          A[k][p] = c * akp - sn * akq;
          A[k][q] = sn * akp + c * akq;
          const double vkp = V[k][p], vkq = V[k][q];
          V[k][p] = c * vkp - sn * vkq;
          V[k][q] = sn * vkp + c * vkq;
        }
      }
      __syncwarp();
      if (k < n) {  // rows p, q of column k
        for (int m = 0; m < n / 2; ++m) {
          const int p = pp_s[m], q = qq_s[m];
          const double c = cs_s[m], sn = sn_s[m];
          const double apk = A[p][k], aqk = A[q][k];
          A[p][k] = c * apk - sn * aqk;
          A[q][k] = sn * apk + c * aqk;
        }
      }
      __syncwarp();
    }
    if (!__any_sync(0xffffffffu, rotated)) break;
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

// sums[h] += (||B - phi_q phi_k^T||_F^2, ||B||_F^2). A CTA takes 32 rows and
// 256 * CPT columns of B: each thread keeps its CPT columns of phi_k in
// registers and walks the rows (phi_q rows from shared memory, broadcast
// 16-byte loads), 4 rows' loads of B in flight at a time. The squares of a
// thread's CPT columns are summed in fp32 (at most 4 terms), everything
// above in fp64.
constexpr int kErrRows = 32;
template <int RT, int CPT>
__global__ void __launch_bounds__(256) err_kernel(int N, int R, const float *__restrict__ B,
                                                  const float *__restrict__ pq, const float *__restrict__ pk,
                                                  double *__restrict__ sums) {
  __shared__ __align__(16) float qs[kErrRows][RT];
  const int h = blockIdx.z;
  const long long i0 = (long long)blockIdx.y * kErrRows;
  const long long c = ((long long)blockIdx.x * 256 + threadIdx.x) * CPT;  // this thread's first column
  const float *Bh = B + (long long)h * N * N;
  for (int e = threadIdx.x; e < kErrRows * RT; e += 256) {
    const int rr = e / RT, r = e - rr * RT;
    const long long i = i0 + rr;
    qs[rr][r] = (i < N && r < R) ? pq[((long long)h * N + i) * R + r] : 0.f;
  }
  float k[CPT][RT];
#pragma unroll
  for (int q = 0; q < CPT; ++q)
#pragma unroll
    for (int r = 0; r < RT; ++r) k[q][r] = (c + q < N && r < R) ? pk[((long long)h * N + c + q) * R + r] : 0.f;
  __syncthreads();
  const bool vec = (N % CPT) == 0 && (reinterpret_cast<uintptr_t>(B) % (CPT * 4)) == 0 && c + CPT <= N;
  double e2 = 0.0, f2 = 0.0;
  for (int rb = 0; rb < kErrRows; rb += 4) {
    float bv[4][CPT];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const long long i = i0 + rb + u;
      if (i < N && vec) {
        if constexpr (CPT == 4) {
          const float4 b4 = *reinterpret_cast<const float4 *>(Bh + i * N + c);
          bv[u][0] = b4.x, bv[u][1] = b4.y, bv[u][2] = b4.z, bv[u][3] = b4.w;
        } else {
          const float2 b2 = *reinterpret_cast<const float2 *>(Bh + i * N + c);
          bv[u][0] = b2.x, bv[u][1] = b2.y;
        }
      } else {
#pragma unroll
        for (int q = 0; q < CPT; ++q) bv[u][q] = (i < N && c + q < N) ? Bh[i * N + c + q] : 0.f;
      }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      float pred[CPT];
#pragma unroll
      for (int q = 0; q < CPT; ++q) pred[q] = 0.f;
#pragma unroll
      for (int r = 0; r < RT; r += 4) {
        const float4 q4 = *reinterpret_cast<const float4 *>(&qs[rb + u][r]);
#pragma unroll
        for (int q = 0; q < CPT; ++q) {
          pred[q] = fmaf(q4.x, k[q][r], pred[q]);
          pred[q] = fmaf(q4.y, k[q][r + 1], pred[q]);
          pred[q] = fmaf(q4.z, k[q][r + 2], pred[q]);
          pred[q] = fmaf(q4.w, k[q][r + 3], pred[q]);
        }
      }
      float ee = 0.f, ff = 0.f;  // rows or columns past N hold zeros
#pragma unroll
      for (int q = 0; q < CPT; ++q) {
        const float dv = bv[u][q] - pred[q];
        ee = fmaf(dv, dv, ee);
        ff = fmaf(bv[u][q], bv[u][q], ff);
      }
      e2 += double(ee);
      f2 += double(ff);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    e2 += __shfl_xor_sync(0xffffffffu, e2, o);
    f2 += __shfl_xor_sync(0xffffffffu, f2, o);
  }
  if ((threadIdx.x & 31u) == 0) {
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

  const dim3 rows32((N + 8 * kBxRows - 1) / (8 * kBxRows), H),
      cols1024((N + 256 * kBtxCols - 1) / (256 * kBtxCols), H, (N + 511) / 512),
      rows256((N + 255) / 256, H);
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
  bx_kernel<<<rows32, 256, 0, st>>>(N, l, bias, P1, P0);  // Y = B Omega
  orth(P0, P1, P2);                                         // Q in P2
  for (int it = 0; it < power_iters; ++it) {
    cudaMemsetAsync(P0, 0, size_t(H) * l * N * sizeof(float), st);
    btx_kernel<<<cols1024, 256, 0, st>>>(N, l, bias, P2, P0);  // Z = B^T Q
    orth(P0, P2, P1);                                         // Z orthonormal in P1
    bx_kernel<<<rows32, 256, 0, st>>>(N, l, bias, P1, P0);   // Y = B Z
    orth(P0, P1, P2);                                         // Q in P2
  }
  cudaMemsetAsync(P0, 0, size_t(H) * l * N * sizeof(float), st);
  btx_kernel<<<cols1024, 256, 0, st>>>(N, l, bias, P2, P0);  // M = B^T Q
  gram(P0);                                                 // M^T M
  eig_kernel<<<H, 32, 0, st>>>(H, l, R, G, Cq, Ck, sig2);
  rows_kernel<<<rows256, 256, 0, st>>>(N, l, R, P2, Cq, phi_q);
  rows_kernel<<<rows256, 256, 0, st>>>(N, l, R, P0, Ck, phi_k);
  if (err_energy) {
    if (cudaMemsetAsync(sums, 0, size_t(2) * H * sizeof(double), st) != cudaSuccess) return FB_ERR_CUDA;
    const int rows_err = (N + kErrRows - 1) / kErrRows;
    if (R <= 8)
      err_kernel<8, 4><<<dim3((N + 1023) / 1024, rows_err, H), 256, 0, st>>>(N, R, bias, phi_q, phi_k, sums);
    else if (R <= 16)
      err_kernel<16, 4><<<dim3((N + 1023) / 1024, rows_err, H), 256, 0, st>>>(N, R, bias, phi_q, phi_k, sums);
    else
      err_kernel<32, 2><<<dim3((N + 511) / 512, rows_err, H), 256, 0, st>>>(N, R, bias, phi_q, phi_k, sums);
    finish_kernel<<<hb, 32, 0, st>>>(H, sums, sig2, out);
    if (cudaMemcpyAsync(err_energy, out, size_t(2) * H * sizeof(double), cudaMemcpyDeviceToDevice, st) !=
        cudaSuccess)
      return FB_ERR_CUDA;
  }
  return cudaGetLastError() == cudaSuccess ? FB_OK : FB_ERR_CUDA;
}
