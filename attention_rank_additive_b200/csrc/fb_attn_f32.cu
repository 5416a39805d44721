// fb_attn_f32.cu -- fp32 forward of attention with an additive bias on the
// CUDA cores (the fp32 workload; the tensor cores have no fp32 path that
// holds 1e-5). Same mathematics as the tensor-core kernel: scores
// scale * q.k plus the bias (low-rank phi_q . phi_k in fp32, or a dense fp32
// bias), online softmax over 32-key tiles, O / l and the log-sum-exp.
//
// A CTA of 128 threads owns 32 query rows; four threads share a row, each
// holding every fourth head-dim element and every fourth factor rank, and the
// row's partial dot products meet through two xor-shuffles.
#include <cfloat>

#include "fb_internal.h"

namespace fb {

constexpr int kF32Rows = 32;
constexpr int kF32Keys = 32;
constexpr int kF32MaxD = 128;
constexpr int kF32MaxR = 128;

__global__ void __launch_bounds__(128) attn_fwd_f32_kernel(int B, int H, int N, int d, const float *__restrict__ Q,
                                                           const float *__restrict__ K, const float *__restrict__ V,
                                                           int R, const float *__restrict__ phi_q,
                                                           const float *__restrict__ phi_k, long long phi_bs,
                                                           long long phi_hs, const float *__restrict__ bias,
                                                           long long bias_bs, long long bias_hs, float scale,
                                                           int causal, float *__restrict__ O, float *__restrict__ LSE) {
  __shared__ float sK[kF32Keys][kF32MaxD];
  __shared__ float sV[kF32Keys][kF32MaxD];
  __shared__ float sF[kF32Keys][kF32MaxR];

  const int bh = blockIdx.y;
  const int b = bh / H, h = bh - (bh / H) * H;
  const int sub = threadIdx.x & 3;
  const int row = blockIdx.x * kF32Rows + (threadIdx.x >> 2);
  const bool row_ok = row < N;
  const size_t head = size_t(bh) * N * d;
  const float *phq = phi_q ? phi_q + b * phi_bs + h * phi_hs : nullptr;
  const float *phk = phi_k ? phi_k + b * phi_bs + h * phi_hs : nullptr;
  const float *brow = bias ? bias + b * bias_bs + h * bias_hs + (size_t)(row_ok ? row : 0) * N : nullptr;

  float q[kF32MaxD / 4], o[kF32MaxD / 4], fq[kF32MaxR / 4];
#pragma unroll
  for (int u = 0; u < kF32MaxD / 4; ++u) {
    const int c = sub + 4 * u;
    q[u] = (row_ok && c < d) ? Q[head + size_t(row) * d + c] : 0.f;
    o[u] = 0.f;
  }
#pragma unroll
  for (int u = 0; u < kF32MaxR / 4; ++u) {
    const int r = sub + 4 * u;
    fq[u] = (row_ok && phq && r < R) ? phq[size_t(row) * R + r] : 0.f;
  }

  float m = -INFINITY, l = 0.f;
  const int kmax = causal ? min(N, (blockIdx.x + 1) * kF32Rows) : N;  // keys any row of this CTA can see
  for (int k0 = 0; k0 < kmax; k0 += kF32Keys) {
    __syncthreads();
    for (int e = threadIdx.x; e < kF32Keys * d; e += blockDim.x) {
      const int j = e / d, c = e - (e / d) * d;
      const bool ok = k0 + j < N;
      sK[j][c] = ok ? K[head + size_t(k0 + j) * d + c] : 0.f;
      sV[j][c] = ok ? V[head + size_t(k0 + j) * d + c] : 0.f;
    }
    if (phk)
      for (int e = threadIdx.x; e < kF32Keys * R; e += blockDim.x) {
        const int j = e / R, r = e - (e / R) * R;
        sF[j][r] = (k0 + j < N) ? phk[size_t(k0 + j) * R + r] : 0.f;
      }
    __syncthreads();

    float s[kF32Keys];
    float mt = -INFINITY;
#pragma unroll
    for (int j = 0; j < kF32Keys; ++j) {
      float dot = 0.f, fb = 0.f;
#pragma unroll
      for (int u = 0; u < kF32MaxD / 4; ++u) {
        const int c = sub + 4 * u;
        if (c < d) dot = fmaf(q[u], sK[j][c], dot);
      }
      if (phk) {
#pragma unroll
        for (int u = 0; u < kF32MaxR / 4; ++u) {
          const int r = sub + 4 * u;
          if (r < R) fb = fmaf(fq[u], sF[j][r], fb);
        }
      }
      dot += __shfl_xor_sync(0xffffffffu, dot, 1);
      dot += __shfl_xor_sync(0xffffffffu, dot, 2);
      fb += __shfl_xor_sync(0xffffffffu, fb, 1);
      fb += __shfl_xor_sync(0xffffffffu, fb, 2);
      const int key = k0 + j;
      float x = scale * dot + fb;
      if (brow && key < N && row_ok) x += brow[key];
      const bool visible = key < N && (!causal || key <= row);
      s[j] = visible ? x : -INFINITY;
      mt = fmaxf(mt, s[j]);
    }
    const float m_new = fmaxf(m, mt);
    if (m_new == -INFINITY) continue;  // nothing visible yet in this row
    const float alpha = expf(m - m_new);
    l *= alpha;
#pragma unroll
    for (int u = 0; u < kF32MaxD / 4; ++u) o[u] *= alpha;
#pragma unroll
    for (int j = 0; j < kF32Keys; ++j) {
      const float p = expf(s[j] - m_new);
      l += p;
#pragma unroll
      for (int u = 0; u < kF32MaxD / 4; ++u) {
        const int c = sub + 4 * u;
        if (c < d) o[u] = fmaf(p, sV[j][c], o[u]);
      }
    }
    m = m_new;
  }

  if (row_ok) {
    const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
    for (int u = 0; u < kF32MaxD / 4; ++u) {
      const int c = sub + 4 * u;
      if (c < d) O[head + size_t(row) * d + c] = o[u] * inv;
    }
    if (sub == 0) LSE[size_t(bh) * N + row] = l > 0.f ? m + logf(l) : -INFINITY;
  }
}

cudaError_t f32_launch(int B, int H, int N, int d, const float *Q, const float *K, const float *V, int R,
                       const float *phi_q, const float *phi_k, int64_t phi_bs, int64_t phi_hs, const float *bias,
                       int64_t bias_bs, int64_t bias_hs, float scale, int causal, float *O, float *LSE,
                       cudaStream_t stream) {
  dim3 grid((N + kF32Rows - 1) / kF32Rows, B * H);
  attn_fwd_f32_kernel<<<grid, 128, 0, stream>>>(B, H, N, d, Q, K, V, R, R > 0 ? phi_q : nullptr,
                                                 R > 0 ? phi_k : nullptr, phi_bs, phi_hs, bias, bias_bs, bias_hs,
                                                 scale, causal, O, LSE);
  return cudaGetLastError();
}

}  // namespace fb
