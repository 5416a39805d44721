// fb_attn_f32.cu -- fp32 forward of attention with an additive bias on the
// CUDA cores (the fp32 workload; the tensor cores have no fp32 path that
// holds 1e-5). Same mathematics as the tensor-core kernel: scores
// scale * q.k plus the bias (low-rank phi_q . phi_k in fp32, or a dense fp32
// bias), online softmax over 32-key tiles, O / l and the log-sum-exp.
//
// A CTA of 128 threads owns 32 query rows; four threads share a row, each
// holding every fourth float4 column of q, o and the factors, and the row's
// partial dot products meet through two xor-shuffles.
// Key, value and factor tiles are staged in shared memory with all of a
// tile's global loads in flight before the first store.
#include <cfloat>

#include "fb_internal.h"

namespace fb {

constexpr int kF32Rows = 32;
constexpr int kF32Keys = 32;

// DQ: float4 columns of q/k/v per row after padding (4, 8, 16 or 32; d <= 4 DQ).
// FR: float4 columns of the factors after padding (0, 4, 8 or 32; R <= 4 FR).
template <int DQ, int FR>
__global__ void __launch_bounds__(128) attn_fwd_f32_kernel(int B, int H, int N, int d, const float *__restrict__ Q,
                                                           const float *__restrict__ K, const float *__restrict__ V,
                                                           int R, const float *__restrict__ phi_q,
                                                           const float *__restrict__ phi_k, long long phi_bs,
                                                           long long phi_hs, const float *__restrict__ bias,
                                                           long long bias_bs, long long bias_hs, float scale,
                                                           int causal, float *__restrict__ O, float *__restrict__ LSE) {
  constexpr int U = DQ / 4;   // q/k/v float4 columns per thread
  constexpr int UF = FR / 4;  // factor float4 columns per thread
  constexpr int FRS = FR > 0 ? FR : 1;
  __shared__ float4 sK[kF32Keys][DQ];
  __shared__ float4 sV[kF32Keys][DQ];
  __shared__ float4 sF[kF32Keys][FRS];

  const int bh = blockIdx.y;
  const int b = bh / H, h = bh - (bh / H) * H;
  const int tid = threadIdx.x;
  const int sub = tid & 3;
  const int row = blockIdx.x * kF32Rows + (tid >> 2);
  const bool row_ok = row < N;
  const int d4 = d >> 2;
  const size_t head = size_t(bh) * N * d;
  const float4 *Q4 = reinterpret_cast<const float4 *>(Q + head);
  const float4 *K4 = reinterpret_cast<const float4 *>(K + head);
  const float4 *V4 = reinterpret_cast<const float4 *>(V + head);
  const float *phq = phi_q ? phi_q + b * phi_bs + h * phi_hs : nullptr;
  const float *phk = phi_k ? phi_k + b * phi_bs + h * phi_hs : nullptr;
  const float *brow = bias ? bias + b * bias_bs + h * bias_hs + (size_t)(row_ok ? row : 0) * N : nullptr;
  const float4 zero4 = make_float4(0.f, 0.f, 0.f, 0.f);

  float4 q[U], o[U];
#pragma unroll
  for (int u = 0; u < U; ++u) {
    const int c4 = sub + 4 * u;
    q[u] = (row_ok && c4 < d4) ? Q4[size_t(row) * d4 + c4] : zero4;
    o[u] = zero4;
  }
  float4 fq[UF > 0 ? UF : 1];
#pragma unroll
  for (int u = 0; u < UF; ++u) {
    const int r = 4 * (sub + 4 * u);
    float v[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) v[e] = (row_ok && phq && r + e < R) ? phq[size_t(row) * R + r + e] : 0.f;
    fq[u] = make_float4(v[0], v[1], v[2], v[3]);
  }

  float m = -INFINITY, l = 0.f;
  const int kmax = causal ? min(N, (blockIdx.x + 1) * kF32Rows) : N;  // keys any row of this CTA can see
  for (int k0 = 0; k0 < kmax; k0 += kF32Keys) {
    __syncthreads();
    {
      constexpr int PER = kF32Keys * DQ / 128;  // float4 per thread per tensor
      float4 kr[PER], vr[PER];
#pragma unroll
      for (int it = 0; it < PER; ++it) {
        const int e = tid + 128 * it;
        const int j = e / DQ, c4 = e % DQ;
        const bool ok = (k0 + j < N) && (c4 < d4);
        kr[it] = ok ? K4[size_t(k0 + j) * d4 + c4] : zero4;
        vr[it] = ok ? V4[size_t(k0 + j) * d4 + c4] : zero4;
      }
#pragma unroll
      for (int it = 0; it < PER; ++it) {
        const int e = tid + 128 * it;
        sK[e / DQ][e % DQ] = kr[it];
        sV[e / DQ][e % DQ] = vr[it];
      }
    }
    if (FR > 0) {
      constexpr int PERF = kF32Keys * FR * 4 / 128;  // floats per thread
      float fr[PERF > 0 ? PERF : 1];
#pragma unroll
      for (int it = 0; it < PERF; ++it) {
        const int e = tid + 128 * it;
        const int j = e / (FRS * 4), r = e % (FRS * 4);
        fr[it] = (k0 + j < N && r < R) ? phk[size_t(k0 + j) * R + r] : 0.f;
      }
#pragma unroll
      for (int it = 0; it < PERF; ++it) {
        const int e = tid + 128 * it;
        reinterpret_cast<float *>(&sF[0][0])[e] = fr[it];
      }
    }
    __syncthreads();

    float s[kF32Keys];
    float mt = -INFINITY;
#pragma unroll
    for (int j = 0; j < kF32Keys; ++j) {
      float dot = 0.f, fb = 0.f;
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const float4 kv = sK[j][sub + 4 * u];
        dot = fmaf(q[u].x, kv.x, fmaf(q[u].y, kv.y, fmaf(q[u].z, kv.z, fmaf(q[u].w, kv.w, dot))));
      }
#pragma unroll
      for (int u = 0; u < UF; ++u) {
        const float4 f = sF[j][sub + 4 * u];
        fb = fmaf(fq[u].x, f.x, fmaf(fq[u].y, f.y, fmaf(fq[u].z, f.z, fmaf(fq[u].w, f.w, fb))));
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
    for (int u = 0; u < U; ++u) {
      o[u].x *= alpha;
      o[u].y *= alpha;
      o[u].z *= alpha;
      o[u].w *= alpha;
    }
#pragma unroll
    for (int j = 0; j < kF32Keys; ++j) {
      const float p = expf(s[j] - m_new);
      l += p;
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const float4 vv = sV[j][sub + 4 * u];
        o[u].x = fmaf(p, vv.x, o[u].x);
        o[u].y = fmaf(p, vv.y, o[u].y);
        o[u].z = fmaf(p, vv.z, o[u].z);
        o[u].w = fmaf(p, vv.w, o[u].w);
      }
    }
    m = m_new;
  }

  if (row_ok) {
    const float inv = l > 0.f ? 1.f / l : 0.f;
    float4 *O4 = reinterpret_cast<float4 *>(O + head);
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int c4 = sub + 4 * u;
      if (c4 < d4) O4[size_t(row) * d4 + c4] = make_float4(o[u].x * inv, o[u].y * inv, o[u].z * inv, o[u].w * inv);
    }
    if (sub == 0) LSE[size_t(bh) * N + row] = l > 0.f ? m + logf(l) : -INFINITY;
  }
}

cudaError_t f32_launch(int B, int H, int N, int d, const float *Q, const float *K, const float *V, int R,
                       const float *phi_q, const float *phi_k, int64_t phi_bs, int64_t phi_hs, const float *bias,
                       int64_t bias_bs, int64_t bias_hs, float scale, int causal, float *O, float *LSE,
                       cudaStream_t stream) {
  dim3 grid((N + kF32Rows - 1) / kF32Rows, B * H);
  const float *pq = R > 0 ? phi_q : nullptr, *pk = R > 0 ? phi_k : nullptr;
  const int d4 = d / 4;
  const int rr = R > 0 ? R : 0;
#define FB_F32_LAUNCH(DQv, FRv)                                                                                    \
  attn_fwd_f32_kernel<DQv, FRv><<<grid, 128, 0, stream>>>(B, H, N, d, Q, K, V, R, pq, pk, phi_bs, phi_hs, bias,     \
                                                           bias_bs, bias_hs, scale, causal, O, LSE)
#define FB_F32_BY_R(DQv)            \
  if (rr == 0)                      \
    FB_F32_LAUNCH(DQv, 0);          \
  else if (rr <= 16)                \
    FB_F32_LAUNCH(DQv, 4);          \
  else if (rr <= 32)                \
    FB_F32_LAUNCH(DQv, 8);          \
  else                              \
    FB_F32_LAUNCH(DQv, 32);
  if (d4 <= 4) {
    FB_F32_BY_R(4)
  } else if (d4 <= 8) {
    FB_F32_BY_R(8)
  } else if (d4 <= 16) {
    FB_F32_BY_R(16)
  } else {
    FB_F32_BY_R(32)
  }
#undef FB_F32_BY_R
#undef FB_F32_LAUNCH
  return cudaGetLastError();
}

}  // namespace fb
