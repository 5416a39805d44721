// fb_internal.h -- declarations shared by the translation units of
// libflashbias (host side). Not part of the public ABI.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/flashbias.h"

namespace fb {

// Bits of the library's device flag word.
constexpr int kFlagTimeout = 1;
constexpr int kFlagRange = 2;

// Bias handling inside the tensor-core kernel.
enum BiasMode : int {
  kBiasNone = 0,   // plain attention (R == 0)
  kBiasMma = 1,    // fp16 factors, second tcgen05 MMA into the score accumulator
  kBiasTf32 = 2,   // R <= 4: fp32 factors split hi/lo, second MMA (kind::tf32) into the score accumulator
  kBiasDense = 3,  // materialised bf16 bias tile streamed by TMA (comparison path)
};

// Runtime arguments of the tensor-core forward kernel.
struct FwdArgs {
  int B, H, N, d;
  int n_kv;          // number of 128-key tiles
  int n_cta_q;       // number of CTA row groups along N
  float scale_log2;  // scale * log2(e)
  float scale;       // the score scale itself (the dense path adds its bias to scale * QK^T)
  int causal;
  void *O;
  float *LSE;
  int fac_B, fac_H;       // factor slices: B or 1, H or 1 (1 = broadcast)
  int bias_B, bias_H;     // dense bias slices, same convention
  int *flags;             // device flag word
  unsigned int *sched;    // work counter [2] (zero at launch), or null: a fixed item order
  int head_group;         // work items are numbered in groups of this many heads (B*H: one group)
};

// Launch description chosen by the host for one call.
struct FwdPlan {
  int DP;    // padded head dim: 16, 32, 64, 128
  int RP;    // kBiasMma: padded factor rank (16..128); kBiasTf32: split-factor columns 8 or 16; else 0
  int mode;  // BiasMode
  int QT;    // 128-row query tiles per CTA: 1 or 2
};

struct FwdMaps {
  CUtensorMap q, k, v;  // bf16 [BH, N, d] with box (min(DP,64), 128, 1)
  CUtensorMap fq, fk;   // factors: fp16 [FB, N, RP] (mma) or fp32 [FB, N, RP] (tf32)
  CUtensorMap bias;     // dense bias bf16 [B', H', N, N] with box (64, 128, 1, 1)
  CUtensorMap o;        // O bf16 [BH, N, d] with box (min(DP,32), 32, 1): the epilogue's TMA stores
};

// Shared-memory bytes the kernel needs for a plan, or 0 if it does not fit.
size_t sm100_smem_bytes(const FwdPlan &p);
// Columns of O per epilogue TMA store (the O tensor map's box width) for a plan.
int sm100_epi_cols(const FwdPlan &p);
// Launches the tcgen05 kernel; returns a cudaError_t.
cudaError_t sm100_launch(const FwdPlan &p, const FwdMaps &maps, const FwdArgs &a, cudaStream_t stream);

// CUDA-core fp32 path (also the oracle-precision path of the bf16-free workload).
cudaError_t f32_launch(int B, int H, int N, int d, const float *Q, const float *K, const float *V, int R,
                       const float *phi_q, const float *phi_k, int64_t phi_bs, int64_t phi_hs, const float *bias,
                       int64_t bias_bs, int64_t bias_hs, float scale, int causal, float *O, float *LSE,
                       cudaStream_t stream);

// Factor generators and preparation.
cudaError_t launch_sandwich(int N, int C, float *phi_q, float *phi_k, cudaStream_t s);
cudaError_t launch_alibi(int H, int N, float *phi_q, float *phi_k, cudaStream_t s);
// kBiasMma: fp16 [FB, N, RP], phi_q / scale. kBiasTf32: fp32 [FB, N, RP] hi/lo split, phi_q / scale.
// Also zeroes the fused kernel's work counter sched[2] when sched is not null.
cudaError_t launch_prep_factors(int mode, int B, int H, int N, int R, int RP, const float *phi_q, const float *phi_k,
                                int64_t bs, int64_t hs, int fac_B, int fac_H, float scale, void *out_q, void *out_k,
                                int *flags, unsigned int *sched, cudaStream_t s);
cudaError_t launch_wait_selftest(int limit_ms, int *flags, cudaStream_t s);
// Multiplicative bias: q1 = q phi_q,0 and k1 = k phi_k,0 (bf16 [BH, N, d]);
// fp16 factor rows [BH, N, RP] with the terms r >= 1.
// Neural decomposition: phi_q[b, h] = X_q[b] W_q[h], phi_k[b, h] = X_k[b] W_k[h] (fp32).
cudaError_t launch_neural_factors(int B, int H, int N, int F, int R, const float *Xq, const float *Xk,
                                  const float *Wq, const float *Wk, float *pq, float *pk, cudaStream_t s);
// The same factors made straight into the fused kernel's prepared layout (fp16
// [B*H, N, RP] with phi_q / scale, or tf32 hi/lo rows of RP columns when tf32),
// zeroing the work counter: the linear layers and the preparation in one launch.
cudaError_t launch_neural_prep(int B, int H, int N, int F, int R, int RP, int tf32, const float *Xq, const float *Xk,
                               const float *Wq, const float *Wk, float scale, void *out_q, void *out_k, int *flags,
                               unsigned int *sched, cudaStream_t s);
// Gradients of the neural decomposition's linear layers: dW [H, F, R] from X and
// dphi [B, H, N, R]; dX [B, N, F] from W and dphi (skipped when dXq or dXk is null).
cudaError_t launch_neural_grads(int B, int H, int N, int F, int R, const float *Xq, const float *Xk,
                                const float *Wq, const float *Wk, const float *dpq, const float *dpk, float *dWq,
                                float *dWk, float *dXq, float *dXk, cudaStream_t s);
cudaError_t launch_prep_mul_bias(int B, int H, int N, int d, int R, int RP, const void *Q, const void *K,
                                 const float *phi_q, const float *phi_k, int64_t bs, int64_t hs, void *q1, void *k1,
                                 void *fq, void *fk, int *flags, unsigned int *sched, cudaStream_t s);

// Backward (gradients of O for dO).
struct BwdArgs {
  int B, H, N, d, R;
  int n_kv;                // 128-row tiles along N
  int Npad;                // n_kv * 128: row stride of lse2 / delta
  float scale, scale_log2;
  int causal;
  const float *nlse2;      // [BH, Npad] -LSE * log2(e); -inf past N
  const float *delta;      // [BH, Npad] rowsum(dO * O); 0 past N
  void *dQ, *dK, *dV;      // bf16 [BH, N, d]
  float *dphi_q, *dphi_k;  // fp32, laid out like phi_q / phi_k
  float *dphi_q_part, *dphi_k_part;  // per-head partial rows [BH, N, R] (shared factor slices)
  int dphi_direct;         // 1: every head has its own factor slice, rows go straight to dphi
  int64_t phi_bs, phi_hs;  // element strides of the factor tensors
  int fac_B, fac_H;        // factor slices: B or 1, H or 1
  float *dqacc;            // fused kernel: fp32 [BH, Npad, 64 + RG] accumulator of dq' = dS [K | phi_k]
  unsigned int *sched;     // fused kernel: work counter (zeroed by the per-row pass)
  int *flags;
};

struct BwdPlan {
  int DP;    // padded head dim
  int RP;    // S-side factor width (as FwdPlan)
  int mode;  // kBiasNone, kBiasMma or kBiasTf32
  int RG;    // bf16 gradient factor width: pad_rank(R), 16 for R <= 4, 0 for R = 0
};

struct BwdMaps {
  CUtensorMap q, dO, fq;                         // dQ kernel, fixed tiles: box rows 128
  CUtensorMap k, v, fk;                          // dK/dV kernel, fixed tiles: box rows 128
  CUtensorMap q_blk, do_blk, fq_blk, gq_blk;     // dK/dV kernel, streamed query blocks
  CUtensorMap k_blk, v_blk, fk_blk, gk_blk;      // dQ kernel, streamed key blocks
  CUtensorMap gk;                                // fused kernel: fixed bf16 gradient factor tile, box rows 128
  CUtensorMap acc;                               // fused kernel: fp32 dq' accumulator, box (64 + RG, 16 or 32, 1)
  // Q, K, V, dO: bf16 [BH, N, d], box (min(DP,64), rows, 1); fq/fk: the forward's
  // factor tiles; gq/gk: bf16 gradient factors [FB, N, RG].
};

// Rows of the dK/dV kernel's query block and of the dQ kernel's key block
// for a plan (0: unsupported).
int bwd_query_block_rows(const BwdPlan &p);
int bwd_key_block_rows(const BwdPlan &p);
// Whether the plan runs as the single fused kernel (dq' accumulated in the
// workspace, then converted) instead of the dK/dV and dQ kernels.
bool bwd_fused(const BwdPlan &p);
// dQ = scale acc[:, :d] (bf16) and, where every head has its own factor slice,
// dphi_q = acc[:, 64:64+R], from the fused kernel's accumulator.
cudaError_t launch_bwd_dq_convert(int B, int H, int N, int Npad, int d, int R, int dqw, float scale,
                                  const float *acc, void *dQ, float *dphi_q, int64_t bs, int64_t hs, int fac_B,
                                  int fac_H, cudaStream_t s);
cudaError_t bwd_launch(const BwdPlan &p, const BwdMaps &maps, const BwdArgs &a, cudaStream_t stream);
// nlse2 = -LSE * log2(e) and delta = rowsum(dO * O) per row, padded to Npad.
// With acc != nullptr, also zeroes the fused kernel's accumulator rows [BH, Npad, dqw]
// and its work counter *sched.
cudaError_t launch_bwd_rows(int BH, int N, int Npad, int d, const void *O, const void *dO, const float *LSE,
                            float *nlse2, float *delta, float *acc, int dqw, unsigned int *sched, cudaStream_t s);
// bf16 copies of the factors [FB, N, RG] (zero-padded).
cudaError_t launch_prep_grad_factors(int N, int R, int RG, const float *phi_q, const float *phi_k, int64_t bs,
                                     int64_t hs, int fac_B, int fac_H, void *gq, void *gk, cudaStream_t s);
// Factor gradients of shared slices: dphi[f] = sum over the heads of slice f of
// the per-head partial rows: [B*H, N, R] for k; for q, row n of head bh at
// part_q + bh q_head + n q_row + q_off (the partial rows, or the fused
// kernel's accumulator).
cudaError_t launch_reduce_factor_grads(int B, int H, int N, int R, int fac_B, int fac_H, int64_t bs, int64_t hs,
                                       const float *part_q, int64_t q_head, int q_row, int q_off, const float *part_k,
                                       float *dphi_q, float *dphi_k, cudaStream_t s);

// Launch with programmatic stream serialization: the kernel may start while
// the previous kernel in the stream finishes, and must call griddep_wait()
// before it reads anything that kernel writes.
template <typename... KArgs, typename... Args>
cudaError_t launch_programmatic(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                                Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
  return e != cudaSuccess ? e : cudaGetLastError();
}

// Per-device flag word (allocated once per device as a module global).
int *device_flags();

// fb_attn_fwd's argument checks other than the workspace (FB_OK or the status
// fb_attn_fwd returns), for entry points that must report the same errors.
int fwd_arg_status(int dt, int B, int H, int N, int d, const void *Q, const void *K, const void *V, int R,
                   const float *phi_q, const float *phi_k, int64_t phi_bstride, int64_t phi_hstride, float scale,
                   const void *O, const float *LSE);

}  // namespace fb
