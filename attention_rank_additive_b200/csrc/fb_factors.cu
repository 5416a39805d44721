// fb_factors.cu -- exact factor generators (Sandwich, ALiBi), the factor
// preparation step that feeds the tensor-core kernels, the multiplicative-bias
// reweighting, the neural decomposition's linear layers and their gradients,
// the small row and reduction steps of the backward, and the wait self-test.
#include <atomic>
#include <cmath>

#include "fb_internal.h"
#include "fb_ptx.cuh"

namespace fb {

// Sandwich factors (FlashBias rebuttal, reply to Reviewer UJUf, Q1 (2)):
// phi(n)[2(k-1)] = cos(n w_k), phi(n)[2k-1] = sin(n w_k), w_k = 10000^(-2k/C).
// Evaluated in fp64, rounded once to fp32.
__global__ void sandwich_kernel(int N, int C, float *__restrict__ phi_q, float *__restrict__ phi_k) {
  const int half = C / 2;
  const long long total = (long long)N * half;
  for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < total;
       idx += (long long)gridDim.x * blockDim.x) {
    const long long n = idx / half;
    const int k = int(idx - n * half) + 1;
    const double w = pow(10000.0, -2.0 * double(k) / double(C));
    double sv, cv;
    sincos(double(n) * w, &sv, &cv);
    const size_t o = size_t(n) * C + 2 * (k - 1);
    phi_q[o] = float(cv);
    phi_q[o + 1] = float(sv);
    if (phi_k != nullptr && phi_k != phi_q) {
      phi_k[o] = float(cv);
      phi_k[o + 1] = float(sv);
    }
  }
}

// ALiBi factors (FlashBias Example 3.4; rebuttal, reply to Reviewer BRmd, Q2
// (2)): m_h = 2^(-8(h+1)/H), phi_q = [-m_h n, 1], phi_k = [1, m_h n].
__global__ void alibi_kernel(int H, int N, float *__restrict__ phi_q, float *__restrict__ phi_k) {
  const long long total = (long long)H * N;
  for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < total;
       idx += (long long)gridDim.x * blockDim.x) {
    const int h = int(idx / N);
    const long long n = idx - (long long)h * N;
    const double m = exp2(-8.0 * double(h + 1) / double(H));
    const double v = m * double(n);
    phi_q[2 * idx] = float(-v);
    phi_q[2 * idx + 1] = 1.0f;
    phi_k[2 * idx] = 1.0f;
    phi_k[2 * idx + 1] = float(v);
  }
}

// Preparation for the tensor-core path (fp16, R < RP zero-padded):
//   out_q[f, n, r] = fp16(phi_q[b', h', n, r] / scale),  out_k = fp16(phi_k).
// Values beyond the fp16 range are saturated and raise kFlagRange.
__global__ void prep_mma_kernel(int N, int R, int RP, int fac_H, const float *__restrict__ pq,
                                const float *__restrict__ pk, long long bs, long long hs, float inv_scale,
                                __half *__restrict__ oq, __half *__restrict__ ok, int *flags, long long total,
                                unsigned int *sched) {
  if (sched != nullptr && blockIdx.x == 0 && threadIdx.x == 0) sched[0] = sched[1] = 0u;  // the work counter
  bool overflow = false;
  griddep_launch_dependents();  // the fused kernel may start its set-up now
  for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < total;
       idx += (long long)gridDim.x * blockDim.x) {
    const int r = int(idx % RP);
    const long long rest = idx / RP;
    const long long n = rest % N;
    const long long f = rest / N;
    const long long fb = f / fac_H, fh = f - (f / fac_H) * fac_H;
    float vq = 0.f, vk = 0.f;
    if (r < R) {
      const long long src = fb * bs + fh * hs + n * R + r;
      vq = pq[src] * inv_scale;
      vk = pk[src];
    }
    if (fabsf(vq) > 65504.f) { vq = copysignf(65504.f, vq); overflow = true; }
    if (fabsf(vk) > 65504.f) { vk = copysignf(65504.f, vk); overflow = true; }
    if (!(vq == vq) || !(vk == vk)) overflow = true;
    oq[idx] = __float2half_rn(vq);
    ok[idx] = __float2half_rn(vk);
  }
  if (overflow) atomicOr(flags, kFlagRange);
}

// Rank <= 4: the factors enter the tensor cores as tf32 (kind::tf32 MMA),
// split so that the product keeps fp32 accuracy: x = hi + lo with hi = x with
// its 13 low mantissa bits cleared (what a tf32 operand holds) and lo = x - hi
// (exact). Row layouts, KT = 8 or 16 columns, zero-padded:
//   q' = [qh_0..qh_{R-1}, qh_0..qh_{R-1}, ql_0..ql_{R-1}]   (phi_q / scale)
//   k' = [kh_0..kh_{R-1}, kl_0..kl_{R-1}, kh_0..kh_{R-1}]
// so q'.k' = qh.kh + qh.kl + ql.kh; the dropped ql.kl and the tf32 rounding
// of the lo parts are about 2^-22 of each product.
__device__ __forceinline__ float tf32_hi(float x) { return __uint_as_float(__float_as_uint(x) & 0xFFFFE000u); }

__global__ void prep_tf32_kernel(int N, int R, int KT, int fac_H, const float *__restrict__ pq,
                                 const float *__restrict__ pk, long long bs, long long hs, float inv_scale,
                                 float *__restrict__ oq, float *__restrict__ ok, long long total,
                                 unsigned int *sched) {
  if (sched != nullptr && blockIdx.x == 0 && threadIdx.x == 0) sched[0] = sched[1] = 0u;  // the work counter
  griddep_launch_dependents();  // the fused kernel may start its set-up now
  for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < total;
       idx += (long long)gridDim.x * blockDim.x) {
    const long long n = idx % N;
    const long long f = idx / N;
    const long long fb = f / fac_H, fh = f - (f / fac_H) * fac_H;
    const long long src = fb * bs + fh * hs + n * R;
    float q[16], k[16];
#pragma unroll
    for (int c = 0; c < 16; ++c) q[c] = k[c] = 0.f;
    for (int r = 0; r < R; ++r) {
      const float x = pq[src + r] * inv_scale, y = pk[src + r];
      const float xh = tf32_hi(x), yh = tf32_hi(y);
      q[r] = xh;
      q[R + r] = xh;
      q[2 * R + r] = x - xh;
      k[r] = yh;
      k[R + r] = y - yh;
      k[2 * R + r] = yh;
    }
    float4 *dq = reinterpret_cast<float4 *>(oq + idx * KT);
    float4 *dk = reinterpret_cast<float4 *>(ok + idx * KT);
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      if (4 * v < KT) {
        dq[v] = make_float4(q[4 * v], q[4 * v + 1], q[4 * v + 2], q[4 * v + 3]);
        dk[v] = make_float4(k[4 * v], k[4 * v + 1], k[4 * v + 2], k[4 * v + 3]);
      }
    }
  }
}

// Multiplicative bias b = phi_q phi_k^T (rebuttal, reply to Reviewer BRmd,
// Q1 (2), Eq. (3)): (q k^T) * b = sum_r (q phi_q,r)(k phi_k,r)^T. The first
// term becomes the kernel's Q and K (bf16, [BH, N, d]); the others become its
// factor tiles, fp16 [BH, N, RP] with column (r-1) d + c = q_c phi_q,r (not
// divided by scale: the kernel's scale multiplies every term), zero-padded
// from d (R-1) to RP. One thread per (row, group of 8 columns), 16-byte
// loads and stores (d, d (R-1) and RP are multiples of 8); values beyond the
// fp16 range are saturated and raise kFlagRange.
__global__ void prep_mul_bias_kernel(int H, int N, int d, int R, int RP, const __nv_bfloat16 *__restrict__ Q,
                                     const __nv_bfloat16 *__restrict__ K, const float *__restrict__ pq,
                                     const float *__restrict__ pk, long long bs, long long hs,
                                     __nv_bfloat16 *__restrict__ q1, __nv_bfloat16 *__restrict__ k1,
                                     __half *__restrict__ fq, __half *__restrict__ fk, int *flags, int width,
                                     long long total, unsigned int *sched) {
  if (sched != nullptr && blockIdx.x == 0 && threadIdx.x == 0) sched[0] = sched[1] = 0u;  // the work counter
  griddep_launch_dependents();  // the fused kernel may start its set-up now
  bool overflow = false;
  const int used = d * (R - 1);
  for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < total;
       idx += (long long)gridDim.x * blockDim.x) {
    const int c = int(idx % width) * 8;  // first of 8 columns
    const long long row = idx / width;   // bh * N + n
    const long long n = row % N, bh = row / N;
    const long long b = bh / H, h = bh - (bh / H) * H;
    if (c < d) {
      const uint4 uq = *reinterpret_cast<const uint4 *>(Q + row * d + c);
      const uint4 uk = *reinterpret_cast<const uint4 *>(K + row * d + c);
      const __nv_bfloat162 *hq = reinterpret_cast<const __nv_bfloat162 *>(&uq);
      const __nv_bfloat162 *hk = reinterpret_cast<const __nv_bfloat162 *>(&uk);
      float qv[8], kv[8];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 fqv = __bfloat1622float2(hq[e]), fkv = __bfloat1622float2(hk[e]);
        qv[2 * e] = fqv.x, qv[2 * e + 1] = fqv.y, kv[2 * e] = fkv.x, kv[2 * e + 1] = fkv.y;
      }
      const long long src = b * bs + h * hs + n * R;
      for (int r = 0; r < R; ++r) {
        const float a = pq[src + r], g = pk[src + r];
        if (r == 0) {
          uint4 oq, ok;
          __nv_bfloat162 *bq = reinterpret_cast<__nv_bfloat162 *>(&oq);
          __nv_bfloat162 *bk = reinterpret_cast<__nv_bfloat162 *>(&ok);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            bq[e] = __floats2bfloat162_rn(qv[2 * e] * a, qv[2 * e + 1] * a);
            bk[e] = __floats2bfloat162_rn(kv[2 * e] * g, kv[2 * e + 1] * g);
          }
          *reinterpret_cast<uint4 *>(q1 + row * d + c) = oq;
          *reinterpret_cast<uint4 *>(k1 + row * d + c) = ok;
        } else {
          uint4 oq, ok;
          __half2 *hq2 = reinterpret_cast<__half2 *>(&oq);
          __half2 *hk2 = reinterpret_cast<__half2 *>(&ok);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            float v0 = qv[2 * e] * a, v1 = qv[2 * e + 1] * a, w0 = kv[2 * e] * g, w1 = kv[2 * e + 1] * g;
            overflow |= !(fabsf(v0) <= 65504.f) || !(fabsf(v1) <= 65504.f) || !(fabsf(w0) <= 65504.f) ||
                        !(fabsf(w1) <= 65504.f);
            v0 = fminf(fmaxf(v0, -65504.f), 65504.f), v1 = fminf(fmaxf(v1, -65504.f), 65504.f);
            w0 = fminf(fmaxf(w0, -65504.f), 65504.f), w1 = fminf(fmaxf(w1, -65504.f), 65504.f);
            hq2[e] = __floats2half2_rn(v0, v1);
            hk2[e] = __floats2half2_rn(w0, w1);
          }
          *reinterpret_cast<uint4 *>(fq + row * RP + (r - 1) * d + c) = oq;
          *reinterpret_cast<uint4 *>(fk + row * RP + (r - 1) * d + c) = ok;
        }
      }
    }
    if (RP > 0 && used + c < RP) {  // zero padding of the factor rows
      *reinterpret_cast<uint4 *>(fq + row * RP + used + c) = make_uint4(0u, 0u, 0u, 0u);
      *reinterpret_cast<uint4 *>(fk + row * RP + used + c) = make_uint4(0u, 0u, 0u, 0u);
    }
  }
  if (overflow) atomicOr(flags, kFlagRange);
}

// Neural decomposition (rebuttal, reply to Reviewer xU4x, Q4: the factors
// of a dynamic bias come from lightweight networks, "simple linear layers"):
// phi_q[b, h] = X_q[b] W_q[h], phi_k[b, h] = X_k[b] W_k[h]; X [B, N, F],
// W [H, F, R], phi [B, H, N, R], all fp32 (fp32 products and sums). Grid
// (row blocks of 64, B H); the CTA holds W_q[h] and W_k[h] in shared memory
// (F R <= 8192 each) and one thread computes one (row, column) pair of both.
__global__ void __launch_bounds__(256) neural_factor_kernel(int H, int N, int F, int R,
                                                            const float *__restrict__ Xq,
                                                            const float *__restrict__ Xk,
                                                            const float *__restrict__ Wq,
                                                            const float *__restrict__ Wk, float *__restrict__ pq,
                                                            float *__restrict__ pk) {
  extern __shared__ float wsm[];  // [2][F][R]
  const int bh = blockIdx.y, b = bh / H, h = bh - (bh / H) * H;
  for (int e = threadIdx.x; e < F * R; e += blockDim.x) {
    wsm[e] = Wq[(long long)h * F * R + e];
    wsm[F * R + e] = Wk[(long long)h * F * R + e];
  }
  __syncthreads();
  const long long n0 = (long long)blockIdx.x * 64;
  for (int e = threadIdx.x; e < 64 * R; e += blockDim.x) {
    const int rr = e / R, r = e - rr * R;
    const long long n = n0 + rr;
    if (n >= N) break;
    const float *xq = Xq + ((long long)b * N + n) * F;
    const float *xk = Xk + ((long long)b * N + n) * F;
    float sq = 0.f, sk = 0.f;
    for (int f = 0; f < F; ++f) {
      sq = fmaf(xq[f], wsm[f * R + r], sq);
      sk = fmaf(xk[f], wsm[F * R + f * R + r], sk);
    }
    pq[((long long)bh * N + n) * R + r] = sq;
    pk[((long long)bh * N + n) * R + r] = sk;
  }
}

// The neural decomposition made straight into the fused kernel's factor
// layout, in one launch (the linear layers and the preparation step fused):
// phi_q = X_q[b] W_q[h], phi_k = X_k[b] W_k[h] in fp32, each sum in the order
// f = 0, 1, ..., F-1 (as neural_factor_kernel), then as the preparation step
// makes them: fp16 [B*H, N, RP] with phi_q / scale (R > 4), or the tf32 hi/lo
// split rows of KT = RP columns (R <= 4). Also zeroes the fused kernel's work
// counter.
//
// R > 4: a 64-row x TW-column tile of phi per CTA (TW = 32, or 16 when
// RP = 16), X and W staged in shared memory 32 features at a time (X
// transposed), each thread a 4 x 4 block of both products.
template <int TW>
__global__ void __launch_bounds__(64 * TW / 16) neural_prep_mma_kernel(
    int H, int N, int F, int R, int RP, const float *__restrict__ Xq, const float *__restrict__ Xk,
    const float *__restrict__ Wq, const float *__restrict__ Wk, float inv_scale, __half *__restrict__ oq,
    __half *__restrict__ ok, int *flags, unsigned int *sched) {
  constexpr int NT = 64 * TW / 16;  // threads
  constexpr int FC = 32;            // features per stage
  __shared__ __align__(16) float xs[2][FC][68];   // [side][f][row], rows padded against bank conflicts
  __shared__ __align__(16) float ws[2][FC][TW];   // [side][f][col]
  if (sched != nullptr && blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0 && threadIdx.x == 0)
    sched[0] = sched[1] = 0u;
  griddep_launch_dependents();  // the fused kernel may start its set-up now
  const int bh = blockIdx.y, b = bh / H, h = bh - (bh / H) * H;
  const long long n0 = (long long)blockIdx.x * 64;
  const int c0 = blockIdx.z * TW;
  const int tr = threadIdx.x % 16, tc = threadIdx.x / 16;  // rows 4 tr .. 4 tr + 3, cols 4 tc .. 4 tc + 3
  float aq[4][4], ak[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) aq[i][j] = ak[i][j] = 0.f;
  // each thread's share of a stage: all of its loads are issued before its
  // shared-memory stores, so a stage costs one memory latency, not one per
  // element
  constexpr int XK = 64 * FC / NT, WK = FC * TW / NT;
  static_assert(XK * NT == 64 * FC && WK * NT == FC * TW, "staging split");
  for (int f0 = 0; f0 < F; f0 += FC) {
    const int fc = min(FC, F - f0);
    float xv[2][XK], wv[2][WK];
#pragma unroll
    for (int u = 0; u < XK; ++u) {
      const int e = int(threadIdx.x) + u * NT;
      const int rr = e / FC, f = e - rr * FC;  // consecutive threads: consecutive features of one row
      const long long n = n0 + rr;
      const bool in = n < N && f < fc;
      xv[0][u] = in ? Xq[((long long)b * N + n) * F + f0 + f] : 0.f;
      xv[1][u] = in ? Xk[((long long)b * N + n) * F + f0 + f] : 0.f;
    }
#pragma unroll
    for (int u = 0; u < WK; ++u) {
      const int e = int(threadIdx.x) + u * NT;
      const int f = e / TW, c = e - f * TW;
      const int r = c0 + c;
      const bool in = f < fc && r < R;
      wv[0][u] = in ? Wq[((long long)h * F + f0 + f) * R + r] : 0.f;
      wv[1][u] = in ? Wk[((long long)h * F + f0 + f) * R + r] : 0.f;
    }
#pragma unroll
    for (int u = 0; u < XK; ++u) {
      const int e = int(threadIdx.x) + u * NT;
      const int rr = e / FC, f = e - rr * FC;
      xs[0][f][rr] = xv[0][u];
      xs[1][f][rr] = xv[1][u];
    }
#pragma unroll
    for (int u = 0; u < WK; ++u) {
      const int e = int(threadIdx.x) + u * NT;
      const int f = e / TW, c = e - f * TW;
      ws[0][f][c] = wv[0][u];
      ws[1][f][c] = wv[1][u];
    }
    __syncthreads();
    for (int f = 0; f < fc; ++f) {
      const float4 xq4 = *reinterpret_cast<const float4 *>(&xs[0][f][4 * tr]);
      const float4 xk4 = *reinterpret_cast<const float4 *>(&xs[1][f][4 * tr]);
      const float4 wq4 = *reinterpret_cast<const float4 *>(&ws[0][f][4 * tc]);
      const float4 wk4 = *reinterpret_cast<const float4 *>(&ws[1][f][4 * tc]);
      const float xq[4] = {xq4.x, xq4.y, xq4.z, xq4.w}, xk[4] = {xk4.x, xk4.y, xk4.z, xk4.w};
      const float wq[4] = {wq4.x, wq4.y, wq4.z, wq4.w}, wk[4] = {wk4.x, wk4.y, wk4.z, wk4.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          aq[i][j] = fmaf(xq[i], wq[j], aq[i][j]);
          ak[i][j] = fmaf(xk[i], wk[j], ak[i][j]);
        }
    }
    __syncthreads();
  }
  bool overflow = false;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const long long n = n0 + 4 * tr + i;
    if (n >= N) break;
    __half hq[4], hk[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      float vq = aq[i][j] * inv_scale, vk = ak[i][j];
      if (fabsf(vq) > 65504.f) { vq = copysignf(65504.f, vq); overflow = true; }
      if (fabsf(vk) > 65504.f) { vk = copysignf(65504.f, vk); overflow = true; }
      if (!(vq == vq) || !(vk == vk)) overflow = true;
      hq[j] = __float2half_rn(vq);
      hk[j] = __float2half_rn(vk);
    }
    const long long o = ((long long)bh * N + n) * RP + c0 + 4 * tc;  // 8-byte aligned: RP, c0, 4 tc multiples of 4
    *reinterpret_cast<uint2 *>(oq + o) = *reinterpret_cast<const uint2 *>(hq);
    *reinterpret_cast<uint2 *>(ok + o) = *reinterpret_cast<const uint2 *>(hk);
  }
  if (overflow) atomicOr(flags, kFlagRange);
}

// R <= 4: one thread per row, the few products as plain loops, then the tf32
// hi/lo split of the preparation step.
__global__ void __launch_bounds__(128) neural_prep_tf32_kernel(int H, int N, int F, int R, int KT,
                                                               const float *__restrict__ Xq,
                                                               const float *__restrict__ Xk,
                                                               const float *__restrict__ Wq,
                                                               const float *__restrict__ Wk, float inv_scale,
                                                               float *__restrict__ oq, float *__restrict__ ok,
                                                               unsigned int *sched) {
  if (sched != nullptr && blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0) sched[0] = sched[1] = 0u;
  griddep_launch_dependents();  // the fused kernel may start its set-up now
  const int bh = blockIdx.y, b = bh / H, h = bh - (bh / H) * H;
  const long long n = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (n >= N) return;
  const float *xq = Xq + ((long long)b * N + n) * F;
  const float *xk = Xk + ((long long)b * N + n) * F;
  float q[16], k[16];
#pragma unroll
  for (int c = 0; c < 16; ++c) q[c] = k[c] = 0.f;
  for (int r = 0; r < R; ++r) {
    float sq = 0.f, sk = 0.f;
    for (int f = 0; f < F; ++f) {
      sq = fmaf(xq[f], Wq[((long long)h * F + f) * R + r], sq);
      sk = fmaf(xk[f], Wk[((long long)h * F + f) * R + r], sk);
    }
    const float x = sq * inv_scale, y = sk;
    const float xh = tf32_hi(x), yh = tf32_hi(y);
    q[r] = xh;
    q[R + r] = xh;
    q[2 * R + r] = x - xh;
    k[r] = yh;
    k[R + r] = y - yh;
    k[2 * R + r] = yh;
  }
  float4 *dq = reinterpret_cast<float4 *>(oq + ((long long)bh * N + n) * KT);
  float4 *dk = reinterpret_cast<float4 *>(ok + ((long long)bh * N + n) * KT);
#pragma unroll
  for (int v = 0; v < 4; ++v) {
    if (4 * v < KT) {
      dq[v] = make_float4(q[4 * v], q[4 * v + 1], q[4 * v + 2], q[4 * v + 3]);
      dk[v] = make_float4(k[4 * v], k[4 * v + 1], k[4 * v + 2], k[4 * v + 3]);
    }
  }
}

cudaError_t launch_neural_prep(int B, int H, int N, int F, int R, int RP, int tf32, const float *Xq, const float *Xk,
                               const float *Wq, const float *Wk, float scale, void *out_q, void *out_k, int *flags,
                               unsigned int *sched, cudaStream_t s) {
  if (tf32) {
    const dim3 grid((N + 127) / 128, B * H);
    neural_prep_tf32_kernel<<<grid, 128, 0, s>>>(H, N, F, R, RP, Xq, Xk, Wq, Wk, 1.0f / scale,
                                                 static_cast<float *>(out_q), static_cast<float *>(out_k), sched);
  } else if (RP == 16) {
    const dim3 grid((N + 63) / 64, B * H, 1);
    neural_prep_mma_kernel<16><<<grid, 64, 0, s>>>(H, N, F, R, RP, Xq, Xk, Wq, Wk, 1.0f / scale,
                                                   static_cast<__half *>(out_q), static_cast<__half *>(out_k), flags,
                                                   sched);
  } else {
    const dim3 grid((N + 63) / 64, B * H, RP / 32);
    neural_prep_mma_kernel<32><<<grid, 128, 0, s>>>(H, N, F, R, RP, Xq, Xk, Wq, Wk, 1.0f / scale,
                                                    static_cast<__half *>(out_q), static_cast<__half *>(out_k), flags,
                                                    sched);
  }
  return cudaGetLastError();
}

cudaError_t launch_neural_factors(int B, int H, int N, int F, int R, const float *Xq, const float *Xk,
                                  const float *Wq, const float *Wk, float *pq, float *pk, cudaStream_t s) {
  const size_t smem = size_t(2) * F * R * sizeof(float);
  if (smem > 48 * 1024) {  // the opt-in above the default, once per device (64 KB covers F R <= 8192)
    static std::atomic<int> done[64];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!done[dev].load(std::memory_order_acquire)) {
      e = cudaFuncSetAttribute(neural_factor_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 64 * 1024);
      if (e != cudaSuccess) return e;
      done[dev].store(1, std::memory_order_release);
    }
  }
  const dim3 grid((N + 63) / 64, B * H);
  neural_factor_kernel<<<grid, 256, smem, s>>>(H, N, F, R, Xq, Xk, Wq, Wk, pq, pk);
  return cudaGetLastError();
}

static int grid_for(long long total, int block);

cudaError_t launch_prep_mul_bias(int B, int H, int N, int d, int R, int RP, const void *Q, const void *K,
                                 const float *phi_q, const float *phi_k, int64_t bs, int64_t hs, void *q1, void *k1,
                                 void *fq, void *fk, int *flags, unsigned int *sched, cudaStream_t s) {
  const int width = (d > RP - d * (R - 1) ? d : RP - d * (R - 1)) / 8;  // groups of 8 columns
  const long long total = (long long)B * H * N * width;
  prep_mul_bias_kernel<<<grid_for(total, 256), 256, 0, s>>>(
      H, N, d, R, RP, static_cast<const __nv_bfloat16 *>(Q), static_cast<const __nv_bfloat16 *>(K), phi_q, phi_k,
      bs, hs, static_cast<__nv_bfloat16 *>(q1), static_cast<__nv_bfloat16 *>(k1), static_cast<__half *>(fq),
      static_cast<__half *>(fk), flags, width, total, sched);
  return cudaGetLastError();
}

// One CTA waits on an mbarrier that nothing completes, with a short limit,
// then records a timeout and exits: exercises the failure path of the bounded
// waits without faulting or hanging the GPU.
__global__ void wait_selftest_kernel(unsigned long long limit_ns, int *flags) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    if (!mbar_wait_for(&bar, 0, limit_ns)) atomicOr(flags, kFlagTimeout);
  }
  __syncthreads();
}

static int grid_for(long long total, int block) {
  long long g = (total + block - 1) / block;
  if (g < 1) g = 1;
  if (g > 148 * 16) g = 148 * 16;
  return int(g);
}

cudaError_t launch_sandwich(int N, int C, float *phi_q, float *phi_k, cudaStream_t s) {
  const long long total = (long long)N * (C / 2);
  sandwich_kernel<<<grid_for(total, 256), 256, 0, s>>>(N, C, phi_q, phi_k);
  return cudaGetLastError();
}

cudaError_t launch_alibi(int H, int N, float *phi_q, float *phi_k, cudaStream_t s) {
  const long long total = (long long)H * N;
  alibi_kernel<<<grid_for(total, 256), 256, 0, s>>>(H, N, phi_q, phi_k);
  return cudaGetLastError();
}

cudaError_t launch_prep_factors(int mode, int B, int H, int N, int R, int RP, const float *phi_q, const float *phi_k,
                                int64_t bs, int64_t hs, int fac_B, int fac_H, float scale, void *out_q, void *out_k,
                                int *flags, unsigned int *sched, cudaStream_t s) {
  (void)B;
  (void)H;
  if (mode == kBiasMma) {
    const long long total = (long long)fac_B * fac_H * N * RP;
    prep_mma_kernel<<<grid_for(total, 256), 256, 0, s>>>(N, R, RP, fac_H, phi_q, phi_k, bs, hs, 1.0f / scale,
                                                         static_cast<__half *>(out_q), static_cast<__half *>(out_k),
                                                         flags, total, sched);
  } else {
    const long long total = (long long)fac_B * fac_H * N;
    prep_tf32_kernel<<<grid_for(total, 256), 256, 0, s>>>(N, R, RP, fac_H, phi_q, phi_k, bs, hs, 1.0f / scale,
                                                          static_cast<float *>(out_q), static_cast<float *>(out_k),
                                                          total, sched);
  }
  return cudaGetLastError();
}

// Backward rows: nlse2 = -LSE log2(e) and delta = rowsum(dO * O) (fp32 sum of
// the bf16 products). Eight threads per row, 16 bytes of O and dO each per
// step (d % 8 == 0); rows N .. Npad-1 get -inf and 0, so the kernels' padded
// queries carry P = 0 without a bounds test.
__global__ void __launch_bounds__(256) bwd_rows_kernel(long long rows, int N, int Npad, int d,
                                                       const __nv_bfloat16 *__restrict__ O,
                                                       const __nv_bfloat16 *__restrict__ dO,
                                                       const float *__restrict__ LSE, float *__restrict__ nlse2,
                                                       float *__restrict__ delta, float *__restrict__ dq_acc,
                                                       int dqw, unsigned int *__restrict__ sched) {
  griddep_launch_dependents();  // the gradient kernel may start its set-up now
  if (sched && blockIdx.x == 0 && threadIdx.x == 0) *sched = 0u;
  const long long w = (blockIdx.x * (long long)blockDim.x + threadIdx.x) >> 3;  // row
  const int sub = threadIdx.x & 7;
  if (w >= rows) return;  // whole 8-thread groups leave together
  if (dq_acc) {
    float4 *dst = reinterpret_cast<float4 *>(dq_acc + w * dqw);
    for (int c = sub; c < dqw / 4; c += 8) dst[c] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
  const long long bh = w / Npad;
  const int n = int(w - bh * Npad);
  float acc = 0.f;
  if (n < N) {
    const size_t base = (size_t(bh) * N + n) * d;
    for (int c = sub * 8; c < d; c += 64) {
      const uint4 a = *reinterpret_cast<const uint4 *>(O + base + c);
      const uint4 g = *reinterpret_cast<const uint4 *>(dO + base + c);
      const uint32_t av[4] = {a.x, a.y, a.z, a.w}, gv[4] = {g.x, g.y, g.z, g.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        acc = fmaf(__uint_as_float(av[e] << 16), __uint_as_float(gv[e] << 16), acc);
        acc = fmaf(__uint_as_float(av[e] & 0xFFFF0000u), __uint_as_float(gv[e] & 0xFFFF0000u), acc);
      }
    }
  }
  acc += __shfl_xor_sync(0xffffffffu, acc, 4);
  acc += __shfl_xor_sync(0xffffffffu, acc, 2);
  acc += __shfl_xor_sync(0xffffffffu, acc, 1);
  if (sub == 0) {
    nlse2[w] = n < N ? -LSE[size_t(bh) * N + n] * 1.4426950408889634f : -INFINITY;
    delta[w] = acc;
  }
}

// bf16 copies of the factors for the gradient products, [FB, N, RG] with
// zero padding.
__global__ void prep_grad_factors_kernel(int N, int R, int RG, int fac_H, const float *__restrict__ pq,
                                         const float *__restrict__ pk, long long bs, long long hs,
                                         __nv_bfloat16 *__restrict__ gq, __nv_bfloat16 *__restrict__ gk,
                                         long long total) {
  for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < total;
       idx += (long long)gridDim.x * blockDim.x) {
    const int r = int(idx % RG);
    const long long rest = idx / RG;
    const long long n = rest % N;
    const long long f = rest / N;
    const long long fb = f / fac_H, fh = f - (f / fac_H) * fac_H;
    float vq = 0.f, vk = 0.f;
    if (r < R) {
      const long long src = fb * bs + fh * hs + n * R + r;
      vq = pq[src];
      vk = pk[src];
    }
    gq[idx] = __float2bfloat16_rn(vq);
    gk[idx] = __float2bfloat16_rn(vk);
  }
}

cudaError_t launch_bwd_rows(int BH, int N, int Npad, int d, const void *O, const void *dO, const float *LSE,
                            float *nlse2, float *delta, float *acc, int dqw, unsigned int *sched, cudaStream_t s) {
  const long long rows = (long long)BH * Npad;  // a multiple of 128: full warps
  const long long blocks = (rows * 8 + 255) / 256;
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
  bwd_rows_kernel<<<unsigned(blocks), 256, 0, s>>>(rows, N, Npad, d, static_cast<const __nv_bfloat16 *>(O),
                                                   static_cast<const __nv_bfloat16 *>(dO), LSE, nlse2, delta, acc,
                                                   dqw, sched);
  return cudaGetLastError();
}

// The fused backward's accumulator [BH, Npad, dqw] (fp32; columns [0, 64):
// dQ / scale, columns [64, 64 + R): dphi_q of the head) to dQ (bf16, times the
// scale) and, where every head has its own factor slice, to dphi_q. One
// 8-thread group per row; a thread takes 8 consecutive columns.
__global__ void __launch_bounds__(256) bwd_dq_convert_kernel(long long rows, int H, int N, int Npad, int d, int R,
                                                             int dqw, float scale, const float *__restrict__ acc,
                                                             __nv_bfloat16 *__restrict__ dQ,
                                                             float *__restrict__ dphi_q, long long bs, long long hs,
                                                             int fac_B, int fac_H) {
  griddep_launch_dependents();
  griddep_wait();  // the fused kernel's accumulator is complete
  const long long w = (blockIdx.x * (long long)blockDim.x + threadIdx.x) >> 3;  // row (bh, n), n < N
  const int sub = threadIdx.x & 7;
  if (w >= rows) return;
  const long long bh = w / N;
  const int n = int(w - bh * N);
  const float *src = acc + (bh * Npad + n) * dqw;
  const int c0 = sub * 8;
  if (c0 < d) {
    const float4 a = *reinterpret_cast<const float4 *>(src + c0);
    const float4 b = *reinterpret_cast<const float4 *>(src + c0 + 4);
    const float v[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
    __nv_bfloat16 *dst = dQ + w * d + c0;
    if (c0 + 8 <= d && (d & 7) == 0) {
      uint32_t p[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const __nv_bfloat162 t = __floats2bfloat162_rn(v[2 * e] * scale, v[2 * e + 1] * scale);
        p[e] = *reinterpret_cast<const uint32_t *>(&t);
      }
      *reinterpret_cast<uint4 *>(dst) = make_uint4(p[0], p[1], p[2], p[3]);
    } else {
      for (int e = 0; e < 8 && c0 + e < d; ++e) dst[e] = __float2bfloat16_rn(v[e] * scale);
    }
  }
  if (dphi_q) {
    const int b = int(bh / H), h = int(bh - (bh / H) * H);
    float *row = dphi_q + (fac_B > 1 ? b * bs : 0) + (fac_H > 1 ? h * hs : 0) + (long long)n * R;
    for (int r = sub; r < R; r += 8) row[r] = src[64 + r];
  }
}

cudaError_t launch_bwd_dq_convert(int B, int H, int N, int Npad, int d, int R, int dqw, float scale,
                                  const float *acc, void *dQ, float *dphi_q, int64_t bs, int64_t hs, int fac_B,
                                  int fac_H, cudaStream_t s) {
  const long long rows = (long long)B * H * N;
  const long long blocks = (rows * 8 + 255) / 256;
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
  return launch_programmatic(bwd_dq_convert_kernel, dim3(unsigned(blocks)), dim3(256), 0, s, rows, H, N, Npad, d, R,
                             dqw, scale, acc, static_cast<__nv_bfloat16 *>(dQ), dphi_q, (long long)bs,
                             (long long)hs, fac_B, fac_H);
}

cudaError_t launch_prep_grad_factors(int N, int R, int RG, const float *phi_q, const float *phi_k, int64_t bs,
                                     int64_t hs, int fac_B, int fac_H, void *gq, void *gk, cudaStream_t s) {
  const long long total = (long long)fac_B * fac_H * N * RG;
  prep_grad_factors_kernel<<<grid_for(total, 256), 256, 0, s>>>(
      N, R, RG, fac_H, phi_q, phi_k, bs, hs, static_cast<__nv_bfloat16 *>(gq), static_cast<__nv_bfloat16 *>(gk),
      total);
  return cudaGetLastError();
}

// dphi[fb, fh, n, r] = sum over the heads (b, h) that share slice (fb, fh)
// of part[b H + h, n, r]: one thread per output element, fp32 in head order.
// The q-side rows may sit in a wider buffer: row n of head bh at
// pq + bh q_head + n q_row + q_off.
__global__ void reduce_factor_grads_kernel(int B, int H, int N, int R, int fac_B, int fac_H, long long bs,
                                           long long hs, const float *__restrict__ pq, long long q_head, int q_row,
                                           int q_off, const float *__restrict__ pk, float *__restrict__ dq,
                                           float *__restrict__ dk, long long total) {
  griddep_wait();  // the gradient kernels' partial rows are complete
  const long long NR = (long long)N * R;
  for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < total;
       idx += (long long)gridDim.x * blockDim.x) {
    const long long f = idx / NR, e = idx - f * NR;
    const int fb = int(f / fac_H), fh = int(f - (f / fac_H) * fac_H);
    const int b0 = fac_B > 1 ? fb : 0, b1 = fac_B > 1 ? fb + 1 : B;
    const int h0 = fac_H > 1 ? fh : 0, h1 = fac_H > 1 ? fh + 1 : H;
    const long long n = e / R, r = e - (e / R) * R;
    const long long oq = n * q_row + q_off + r;
    float aq = 0.f, ak = 0.f;
    for (int b = b0; b < b1; ++b)
      for (int h = h0; h < h1; ++h) {
        const long long hb = (long long)b * H + h;
        aq += pq[hb * q_head + oq];
        ak += pk[hb * NR + e];
      }
    const long long dst = fb * bs + fh * hs + n * R + r;
    dq[dst] = aq;
    dk[dst] = ak;
  }
}

cudaError_t launch_reduce_factor_grads(int B, int H, int N, int R, int fac_B, int fac_H, int64_t bs, int64_t hs,
                                       const float *part_q, int64_t q_head, int q_row, int q_off, const float *part_k,
                                       float *dphi_q, float *dphi_k, cudaStream_t s) {
  const long long total = (long long)fac_B * fac_H * N * R;
  return launch_programmatic(reduce_factor_grads_kernel, dim3(grid_for(total, 256)), dim3(256), 0, s, B, H, N, R,
                             fac_B, fac_H, (long long)bs, (long long)hs, part_q, (long long)q_head, q_row, q_off,
                             part_k, dphi_q, dphi_k, total);
}

// Gradients of the neural decomposition's linear layers from the factor
// gradients dphi [B, H, N, R]: dW[h, f, r] = sum_b sum_n X[b, n, f] dphi[b, h, n, r]
// (one thread per weight; the warp's lanes run along r, so the dphi loads
// coalesce and the X load is a broadcast) and dX[b, n, f] = sum_h sum_r
// dphi[b, h, n, r] W[h, f, r] (one thread per feature). fp32, fixed order.
__global__ void neural_grad_w_kernel(int B, int H, int N, int F, int R, const float *__restrict__ X,
                                     const float *__restrict__ dphi, float *__restrict__ dW, long long total) {
  for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < total;
       idx += (long long)gridDim.x * blockDim.x) {
    const int r = int(idx % R);
    const int f = int((idx / R) % F);
    const int h = int(idx / ((long long)R * F));
    float acc = 0.f;
    for (int b = 0; b < B; ++b) {
      const float *xb = X + (long long)b * N * F + f;
      const float *gb = dphi + ((long long)b * H + h) * N * R + r;
      for (int n = 0; n < N; ++n) acc = fmaf(xb[(long long)n * F], gb[(long long)n * R], acc);
    }
    dW[idx] = acc;
  }
}

__global__ void neural_grad_x_kernel(int B, int H, int N, int F, int R, const float *__restrict__ W,
                                     const float *__restrict__ dphi, float *__restrict__ dX, long long total) {
  for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < total;
       idx += (long long)gridDim.x * blockDim.x) {
    const int f = int(idx % F);
    const long long bn = idx / F;
    const int n = int(bn % N);
    const int b = int(bn / N);
    float acc = 0.f;
    for (int h = 0; h < H; ++h) {
      const float *g = dphi + (((long long)b * H + h) * N + n) * R;
      const float *w = W + ((long long)h * F + f) * R;
      for (int r = 0; r < R; ++r) acc = fmaf(g[r], w[r], acc);
    }
    dX[idx] = acc;
  }
}

cudaError_t launch_neural_grads(int B, int H, int N, int F, int R, const float *Xq, const float *Xk,
                                const float *Wq, const float *Wk, const float *dpq, const float *dpk, float *dWq,
                                float *dWk, float *dXq, float *dXk, cudaStream_t s) {
  const long long nw = (long long)H * F * R;
  neural_grad_w_kernel<<<grid_for(nw, 128), 128, 0, s>>>(B, H, N, F, R, Xq, dpq, dWq, nw);
  neural_grad_w_kernel<<<grid_for(nw, 128), 128, 0, s>>>(B, H, N, F, R, Xk, dpk, dWk, nw);
  if (dXq != nullptr && dXk != nullptr) {
    const long long nx = (long long)B * N * F;
    neural_grad_x_kernel<<<grid_for(nx, 256), 256, 0, s>>>(B, H, N, F, R, Wq, dpq, dXq, nx);
    neural_grad_x_kernel<<<grid_for(nx, 256), 256, 0, s>>>(B, H, N, F, R, Wk, dpk, dXk, nx);
  }
  return cudaGetLastError();
}

cudaError_t launch_wait_selftest(int limit_ms, int *flags, cudaStream_t s) {
  wait_selftest_kernel<<<1, 32, 0, s>>>((unsigned long long)limit_ms * 1000000ull, flags);
  return cudaGetLastError();
}

}  // namespace fb
