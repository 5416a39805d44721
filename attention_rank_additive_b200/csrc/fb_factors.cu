// fb_factors.cu -- exact factor generators (Sandwich, ALiBi), the factor
// preparation step that feeds the tensor-core kernel, and the wait self-test.
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
                                __half *__restrict__ oq, __half *__restrict__ ok, int *flags, long long total) {
  bool overflow = false;
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

// Preparation for the CUDA-core factor path (R <= 4, fp32):
//   out_q[f, n, 0..3] = phi_q * log2(e) (zero padded), out_k[f, n, 0..3] = phi_k.
// Rank <= 4 (factors applied on the CUDA cores, fp32): phi_q / scale per
// row as [slice][N] float4, and phi_k by key pairs, so that one 16-byte load
// gives a factor column for two adjacent keys: pair j (keys 2j, 2j+1) holds
// (f0[2j], f0[2j+1], f1[2j], f1[2j+1]) and, for RP = 4, a second float4 with
// f2, f3. A missing key 2j+1 (odd N) has zero factors.
__global__ void prep_reg_kernel(int N, int R, int RP, int fac_H, const float *__restrict__ pq,
                                const float *__restrict__ pk, long long bs, long long hs, float inv_scale,
                                float4 *__restrict__ oq, float4 *__restrict__ ok, long long total) {
  const long long NP = (N + 1) / 2;
  for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < total;
       idx += (long long)gridDim.x * blockDim.x) {
    const long long j = idx % NP;
    const long long f = idx / NP;
    const long long fb = f / fac_H, fh = f - (f / fac_H) * fac_H;
    float k[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
    for (int e = 0; e < 2; ++e) {
      const long long n = 2 * j + e;
      if (n >= N) break;
      const long long src = fb * bs + fh * hs + n * R;
      float q[4] = {0.f, 0.f, 0.f, 0.f};
      for (int r = 0; r < R; ++r) {
        q[r] = pq[src + r] * inv_scale;
        k[e][r] = pk[src + r];
      }
      oq[f * N + n] = make_float4(q[0], q[1], q[2], q[3]);
    }
    float4 *dst = ok + (f * NP + j) * (RP / 2);
    dst[0] = make_float4(k[0][0], k[1][0], k[0][1], k[1][1]);
    if (RP > 2) dst[1] = make_float4(k[0][2], k[1][2], k[0][3], k[1][3]);
  }
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
                                int *flags, cudaStream_t s) {
  (void)B;
  (void)H;
  if (mode == kBiasMma) {
    const long long total = (long long)fac_B * fac_H * N * RP;
    prep_mma_kernel<<<grid_for(total, 256), 256, 0, s>>>(N, R, RP, fac_H, phi_q, phi_k, bs, hs, 1.0f / scale,
                                                         static_cast<__half *>(out_q), static_cast<__half *>(out_k),
                                                         flags, total);
  } else {
    const long long total = (long long)fac_B * fac_H * ((N + 1) / 2);
    prep_reg_kernel<<<grid_for(total, 256), 256, 0, s>>>(N, R, RP, fac_H, phi_q, phi_k, bs, hs, 1.0f / scale,
                                                         static_cast<float4 *>(out_q), static_cast<float4 *>(out_k),
                                                         total);
  }
  return cudaGetLastError();
}

cudaError_t launch_wait_selftest(int limit_ms, int *flags, cudaStream_t s) {
  wait_selftest_kernel<<<1, 32, 0, s>>>((unsigned long long)limit_ms * 1000000ull, flags);
  return cudaGetLastError();
}

}  // namespace fb
