/*
 * flashbias.h -- C ABI of libflashbias: attention with a low-rank additive
 * bias on NVIDIA B200 (sm_100a).
 *
 * The method is "FlashBias: Fast Computation of Attention with Bias" (Wu et
 * al., arXiv 2505.12044). Attention with bias adds an N x N matrix b to the
 * query-key scores (FlashBias abstract; Figure 1). FlashBias replaces b by
 * per-token factors phi_q, phi_k of rank R, b = phi_q phi_k^T (Figure 2), and
 * joins them to the QK^T tile product by concatenating them with the queries
 * and keys (rebuttal, reply to Reviewer UJUf, Q2: "Eq. (3) of main text").
 * The N x N bias is never materialised; only heads x N x R factor values are
 * read (reply to Reviewer BRmd, Q3).
 *
 * Conventions shared by every entry point:
 *  - Tensor pointers are DEVICE pointers unless the name ends in _host.
 *  - Q, K, V, O are [B, H, N, d] row-major (d innermost, contiguous).
 *  - Calls are asynchronous on `stream` (a cudaStream_t passed as void*;
 *    NULL = the legacy default stream).
 *  - The caller owns all memory. Besides caller-provided workspace the
 *    library allocates no device memory at run time; its only device
 *    storage is module globals (a flag word per device and the fixed 8 MiB
 *    scratch array of fb_attn_fwd_noalloc), reserved when the library's
 *    module is loaded on a device.
 *  - Argument, shape, alignment and range errors are reported synchronously,
 *    before anything is launched. A launch failure returns FB_ERR_CUDA.
 *  - Kernel-side conditions (a pipeline wait that ran out, a factor that
 *    overflowed fp16) set a library-wide device flag that
 *    fb_check_device_error() reads back; the kernels never trap.
 *  - Entry points declared to return int return an fb_status value.
 *  - No C++ exception crosses this interface. Entry points may be called
 *    from several host threads, except that fb_attn_fwd_noalloc calls that
 *    can overlap on one device must be serialised by the caller (they share
 *    one scratch array; see there).
 */
#ifndef FLASHBIAS_H_
#define FLASHBIAS_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  FB_OK = 0,
  FB_ERR_INVALID_ARG = 1, /* null or misaligned pointer, empty shape (a size
                             below 1), bad stride, bad scale                 */
  FB_ERR_UNSUPPORTED = 2, /* valid but outside what the library implements
                             (a head dim, rank, dtype or size it does not take) */
  FB_ERR_RANGE = 3,       /* a factor value does not fit the kernel's type    */
  FB_ERR_WORKSPACE = 4,   /* workspace missing, too small or misaligned       */
  FB_ERR_CUDA = 5,        /* CUDA runtime/driver call or launch failed        */
  FB_ERR_TIMEOUT = 6      /* a kernel's bounded pipeline wait ran out         */
} fb_status;

/* Element type of Q, K, V, O (and of a dense bias). fp16 inputs are not
 * implemented: every entry point returns FB_ERR_UNSUPPORTED for FB_F16. */
typedef enum { FB_F32 = 0, FB_BF16 = 1, FB_F16 = 2 } fb_dtype;

/* Human-readable name of a status code (static string, never NULL). */
const char *fb_status_str(int status);

/* Library version as major*10000 + minor*100 + patch. */
int fb_version(void);

/*
 * Workspace for fb_attn_fwd with the bf16 path: the factor tensors after the
 * preparation step (scaled, converted and padded so the tensor cores can read
 * them), followed by a 256-byte block holding the fused kernel's work counter
 * (the preparation step zeroes it and every fused launch leaves it at zero;
 * the counter lets the CTAs take work items in order as they become free).
 * Depends on which factor dimensions are broadcast (stride 0).
 * Returns 0 when R == 0 (the kernel then deals out its work items in a fixed
 * order). The fp32 path needs no workspace.
 */
size_t fb_attn_workspace_bytes(int B, int H, int N, int R,
                               int64_t phi_bstride, int64_t phi_hstride);

/*
 * Fused forward of attention with a low-rank additive bias:
 *
 *   O = softmax(scale * Q K^T + phi_q phi_k^T [+ causal mask]) V
 *   LSE[b,h,i] = ln sum_j exp(scale * q_i.k_j + b_ij)   (over visible j)
 *
 * (FlashBias abstract and Figure 2; rebuttal, reply to Reviewer UJUf, Q2, the
 * concatenation q' = [q, phi_q], k' = [k, phi_k]. The bias is not scaled:
 * scale multiplies QK^T only.)
 *
 *  dt          FB_BF16: Q, K, V, O are bf16, tensor-core path (tcgen05).
 *              FB_F32 : Q, K, V, O are fp32, CUDA-core path, fp32 throughout.
 *  B, H, N, d  batch, heads, sequence length, head dim. bf16: d % 8 == 0,
 *              8 <= d <= 128. fp32: d % 4 == 0, 4 <= d <= 128. N >= 1.
 *  Q, K, V     [B, H, N, d] device, 16-byte aligned.
 *  R           bias rank, 0 <= R <= 128. R == 0 is plain attention.
 *  phi_q/phi_k fp32 device factors; element (b, h, n, r) sits at
 *              b*phi_bstride + h*phi_hstride + n*R + r. A stride of 0
 *              broadcasts that dimension (the Sandwich and ALiBi factors do
 *              not depend on the batch). May be NULL when R == 0.
 *  scale       multiplies QK^T; finite and > 0 (usually 1/sqrt(d)).
 *  causal      nonzero: key j is visible to query i iff j <= i.
 *  O           [B, H, N, d] device output (dtype dt).
 *  LSE         [B, H, N] fp32 device output, natural log.
 *  workspace   device scratch of at least fb_attn_workspace_bytes(...) bytes,
 *              256-byte aligned; may be NULL when that is 0 or dt == FB_F32.
 *              It must not be shared by calls that can run concurrently.
 *  stream      cudaStream_t.
 *
 * bf16 path numerics: QK^T in bf16 x bf16 -> fp32; the factors enter the same
 * fp32 accumulator as a second MMA in fp16 (phi_q pre-divided by scale) when
 * R > 4, or as a tf32 MMA of hi/lo split fp32 factors when R <= 4 (fp32-level
 * accuracy: q'.k' = qh.kh + qh.kl + ql.kh); softmax in fp32;
 * P rounded to bf16 for the PV MMA; O rounded to bf16. A factor that does not
 * fit fp16 is saturated and flags FB_ERR_RANGE for fb_check_device_error().
 */
int fb_attn_fwd(int dt, int B, int H, int N, int d,
                const void *Q, const void *K, const void *V,
                int R, const float *phi_q, const float *phi_k,
                int64_t phi_bstride, int64_t phi_hstride,
                float scale, int causal,
                void *O, float *LSE,
                void *workspace, size_t workspace_bytes, void *stream);

/*
 * The two halves of fb_attn_fwd's bf16 path, for factors that are reused
 * across calls (the Sandwich and ALiBi factors depend only on N, H and the
 * bias parameters, not on the inputs): fb_attn_prepare_factors writes the
 * prepared factors into the workspace once, and fb_attn_fwd_prepared runs
 * the fused kernel alone, as often as needed. fb_attn_fwd is exactly
 * prepare-then-run on one stream. (FlashBias rebuttal, reply to Reviewer
 * xU4x, Q6: the decomposition of a static bias is done once, not at every
 * inference; only dynamic biases need factors per call.)
 *
 * fb_attn_prepare_factors: B, H, N, R, phi_q, phi_k, the strides and scale
 *   as for fb_attn_fwd (scale is folded into the prepared factors). R == 0
 *   does nothing and returns FB_OK. The workspace (fb_attn_workspace_bytes,
 *   256-byte aligned) is written on `stream`; the fp32 factors may be freed
 *   or changed once that work has run.
 * fb_attn_fwd_prepared: dt must be FB_BF16; every argument as for
 *   fb_attn_fwd, and B, H, N, R, the strides and scale equal to those of
 *   the fb_attn_prepare_factors call that filled `workspace` (the library
 *   cannot check this: other values read the workspace under the wrong
 *   layout). The workspace is only read, so concurrent calls may share it.
 * Errors as fb_attn_fwd; both return before launching anything on an
 * argument error.
 */
int fb_attn_prepare_factors(int B, int H, int N, int R,
                            const float *phi_q, const float *phi_k,
                            int64_t phi_bstride, int64_t phi_hstride, float scale,
                            void *workspace, size_t workspace_bytes, void *stream);

int fb_attn_fwd_prepared(int dt, int B, int H, int N, int d,
                         const void *Q, const void *K, const void *V,
                         int R, int64_t phi_bstride, int64_t phi_hstride,
                         float scale, int causal,
                         void *O, float *LSE,
                         const void *workspace, size_t workspace_bytes, void *stream);

/*
 * Attention with a multiplicative low-rank bias (FlashBias rebuttal, reply
 * to Reviewer BRmd, Q1 (2), Eq. (1) and (3)):
 *
 *   O = softmax(scale * (Q K^T) o (phi_q phi_k^T) [+ causal mask]) V
 *
 * (o: elementwise product), computed as (Q K^T) o b = sum_r (Q phi_q,r)
 * (K phi_k,r)^T: the repeated, reweighted q and k of the rebuttal's Eq. (3).
 * The first term runs as the fused kernel's bf16 Q K^T, the other R - 1 as
 * its fp16 factor MMA (a factor rank of d (R - 1) <= 128). Reading of Eq. (3):
 * the printed sqrt(C) in q' would cancel the 1/sqrt(C) of Eq. (1), so it is
 * taken as a typo and `scale` multiplies the whole product, as in Eq. (1).
 *
 *  dt          FB_BF16 only.
 *  R           1 <= R and d (R - 1) <= 128 (R = 1 is a rank-1 bias).
 *  phi_q/phi_k fp32 device factors, layout and strides as for fb_attn_fwd.
 *  workspace   fb_attn_mul_bias_workspace_bytes(B, H, N, d, R) bytes,
 *              256-byte aligned: the reweighted q, k and the fp16 factor rows.
 *  Other arguments and errors as fb_attn_fwd. A product q_c phi_q,r beyond
 *  the fp16 range is saturated and flags FB_ERR_RANGE.
 */
size_t fb_attn_mul_bias_workspace_bytes(int B, int H, int N, int d, int R);

int fb_attn_mul_bias_fwd(int dt, int B, int H, int N, int d,
                         const void *Q, const void *K, const void *V,
                         int R, const float *phi_q, const float *phi_k,
                         int64_t phi_bstride, int64_t phi_hstride,
                         float scale, int causal,
                         void *O, float *LSE,
                         void *workspace, size_t workspace_bytes, void *stream);

/*
 * Attention with a bias from the neural decomposition (FlashBias rebuttal,
 * reply to Reviewer xU4x, Q4: the factors of a dynamic bias come from
 * "lightweight networks", simple linear layers added to the block):
 *
 *   phi_q[b, h] = X_q[b] W_q[h],  phi_k[b, h] = X_k[b] W_k[h],
 *   O = softmax(scale Q K^T + phi_q phi_k^T [+ causal]) V
 *
 *  X_q, X_k    [B, N, F] fp32 device token features.
 *  W_q, W_k    [H, F, R] fp32 device weights of the two linear layers.
 *              1 <= F <= 256, 1 <= R <= 128, F R <= 8192.
 *  workspace   fb_attn_neural_workspace_bytes(B, H, N, F, R) bytes, 256-byte
 *              aligned: the factors in the form the fused kernel reads (as
 *              fb_attn_prepare_factors writes them for per-head factors) and
 *              the work counter.
 *  Other arguments and errors as fb_attn_fwd (dt = FB_BF16 only). Two
 *  launches: the linear layers run in fp32 and write the prepared factors
 *  directly (the preparation step fused into them), then the fused kernel.
 */
size_t fb_attn_neural_workspace_bytes(int B, int H, int N, int F, int R);

int fb_attn_neural_fwd(int dt, int B, int H, int N, int d,
                       const void *Q, const void *K, const void *V,
                       int F, int R, const float *X_q, const float *X_k,
                       const float *W_q, const float *W_k,
                       float scale, int causal,
                       void *O, float *LSE,
                       void *workspace, size_t workspace_bytes, void *stream);

/*
 * Backward of fb_attn_fwd: the gradients of O for an upstream gradient dO.
 * FlashBias trains with a factorised bias by concatenating the factors to the
 * queries and keys (rebuttal, reply to Reviewer UJUf, Q2, and its training
 * speedup in Q1 (3); reply to Reviewer Bp2x, Q3), so the factor gradients are
 * the extra columns of the concatenated query and key gradients:
 *
 *   P = softmax(scale Q K^T + phi_q phi_k^T [+ causal]),  dP = dO V^T,
 *   dS = P o (dP - rowsum(dO o O)),
 *   dQ = scale dS K, dK = scale dS^T Q, dV = P^T dO,
 *   dphi_q = dS phi_k, dphi_k = dS^T phi_q.
 *
 *  dt          FB_BF16 only.
 *  Q..phi_k    the forward's inputs, same layouts and strides.
 *  O, LSE      the forward's outputs for these inputs (O bf16 [B,H,N,d],
 *              LSE fp32 [B,H,N], natural log).
 *  dO          bf16 [B,H,N,d] device.
 *  dQ, dK, dV  bf16 [B,H,N,d] device outputs, 16-byte aligned.
 *  dphi_q/k    fp32 device outputs laid out like phi_q / phi_k (the same
 *              strides; a broadcast factor, stride 0, gets the gradient
 *              summed over the batches or heads sharing it). Overwritten
 *              (no accumulation into the caller's values). Both NULL: the factors
 *              are fixed (e.g. the exact Sandwich or ALiBi factors) and their
 *              gradient products are skipped; one NULL is an argument error.
 *              Unused when R = 0. They must not alias any input.
 *  workspace   fb_attn_bwd_workspace_bytes(B, H, N, R, phi_bstride,
 *              phi_hstride) bytes, 256-byte aligned (never 0).
 * Arithmetic: S and P are recomputed as the forward computes them; the
 * products with dO, Q, K and the factors run on the tensor cores in bf16 with
 * fp32 accumulation. Launches: the factor preparation and the bf16 factor
 * copies (R > 0), the per-row terms, then the gradient kernels, and for a
 * factor shared by several heads one reduction of the per-head factor
 * gradients (kept in the workspace). The gradient kernels: for head dims 33
 * to 64 with fixed factors (or R = 0) or with 33 <= R <= 64, one tcgen05
 * kernel per key tile that also adds each query block's dS [K | phi_k] into
 * an fp32 accumulator in the workspace (TMA reduce-adds at L2), then a
 * conversion to dQ and dphi_q; the order of those fp32 additions varies
 * between runs, so dQ and dphi_q may differ in the last bits from run to run.
 * Otherwise two tcgen05 kernels (dK, dV, dphi_k per key tile; dQ, dphi_q per
 * query tile), bitwise reproducible. Argument errors return before any
 * launch; other errors as fb_attn_fwd.
 */
size_t fb_attn_bwd_workspace_bytes(int B, int H, int N, int R,
                                   int64_t phi_bstride, int64_t phi_hstride);

int fb_attn_bwd(int dt, int B, int H, int N, int d,
                const void *Q, const void *K, const void *V,
                int R, const float *phi_q, const float *phi_k,
                int64_t phi_bstride, int64_t phi_hstride,
                float scale, int causal,
                const void *O, const float *LSE, const void *dO,
                void *dQ, void *dK, void *dV, float *dphi_q, float *dphi_k,
                void *workspace, size_t workspace_bytes, void *stream);

/*
 * Backward of fb_attn_neural_fwd: the gradients of O for an upstream
 * gradient dO, down to the features and the weights of the two linear
 * layers of the neural decomposition (rebuttal, reply to Reviewer xU4x, Q4):
 *
 *   dphi_q, dphi_k     as fb_attn_bwd, per (b, h)
 *   dW_q[h] = sum_b X_q[b]^T dphi_q[b, h],  dX_q[b] = sum_h dphi_q[b, h] W_q[h]^T
 *   (and the same for k)
 *
 *  Q..W_k      the forward's inputs; O, LSE its outputs; dO bf16 [B,H,N,d].
 *  dQ, dK, dV  bf16 [B,H,N,d] device outputs, 16-byte aligned.
 *  dW_q, dW_k  fp32 [H, F, R] device outputs.
 *  dX_q, dX_k  fp32 [B, N, F] device outputs, or both NULL (fixed features).
 *  workspace   fb_attn_neural_bwd_workspace_bytes(B, H, N, F, R) bytes,
 *              256-byte aligned.
 * The factors are recomputed as the forward made them; the attention part is
 * fb_attn_bwd's; the linear-layer gradients run in fp32 on the CUDA cores.
 * Limits, arguments and errors as fb_attn_neural_fwd and fb_attn_bwd.
 */
size_t fb_attn_neural_bwd_workspace_bytes(int B, int H, int N, int F, int R);

int fb_attn_neural_bwd(int dt, int B, int H, int N, int d,
                       const void *Q, const void *K, const void *V,
                       int F, int R, const float *X_q, const float *X_k,
                       const float *W_q, const float *W_k,
                       float scale, int causal,
                       const void *O, const float *LSE, const void *dO,
                       void *dQ, void *dK, void *dV,
                       float *dX_q, float *dX_k, float *dW_q, float *dW_k,
                       void *workspace, size_t workspace_bytes, void *stream);

/*
 * Truncated SVD of H dense biases on the GPU, for biases known only at call
 * time (the SVD decomposition of the rebuttal, reply to Reviewer xU4x, Q6,
 * done per call; the rebuttal calls this inefficient for dynamic biases,
 * and this entry point makes it measurable). Randomized range finder with
 * l = min(R + oversample, 32, N) columns and `power_iters` subspace
 * iterations (orthonormalised by shifted CholeskyQR3 in fp64), then the
 * eigen-decomposition of the l x l Gram matrix of the projected bias.
 * Balanced split: phi_q = U_R sqrt(S_R), phi_k = V_R sqrt(S_R).
 *
 *  bias        [H, N, N] fp32 device, row-major, 4-byte aligned.
 *  R           1 <= R <= min(N, 32).
 *  phi_q/phi_k [H, N, R] fp32 device outputs.
 *  err_energy  optional [H, 2] fp64 device output, 8-byte aligned:
 *              ||B - phi_q phi_k^T||_F / ||B||_F (computed exactly) and
 *              sum_{r<R} s_r^2 / ||B||_F^2.
 *  workspace   fb_svd_device_workspace_bytes(H, N, R, oversample) bytes,
 *              256-byte aligned.
 * Asynchronous on `stream`; returns before any launch on an argument error.
 */
size_t fb_svd_device_workspace_bytes(int H, int N, int R, int oversample);

int fb_svd_factors_device(int H, int N, int R, int oversample, int power_iters,
                          uint64_t seed, const float *bias,
                          float *phi_q, float *phi_k, double *err_energy,
                          void *workspace, size_t workspace_bytes, void *stream);

/*
 * fb_attn_fwd for callers that cannot allocate device memory. (The FlashBias
 * paper has no counterpart: this is an interface convenience.)
 *
 * Who needs it: code that only receives the tensors it works on and has no
 * allocator of its own to call (a plugin or operator interface whose
 * signature carries inputs and outputs only, a host framework that owns every
 * device buffer through its own pool), and code that must not call
 * cudaMalloc on its path (it synchronises the device and can fail under
 * memory pressure). Such callers cannot supply fb_attn_fwd's workspace.
 *
 * Same arguments and results as fb_attn_fwd, without workspace and
 * workspace_bytes. The prepared factors live instead in a fixed 8 MiB array
 * in the library's device memory, reserved on every device that loads the
 * library until the process exits. A call whose prepared factors need more
 * than 8 MiB (fb_attn_workspace_bytes(...) > 8 MiB) returns FB_ERR_WORKSPACE
 * before anything is launched; fb_attn_fwd with a caller workspace has no
 * such limit. The function allocates nothing.
 *
 * The first call on a device looks up the array's device address (with that
 * device current) and caches it; make that first call before capturing the
 * stream into a graph. All calls on a device share the one array and it
 * keeps the last call's contents; the preparation step rewrites every byte a
 * call reads, so nothing needs clearing, but calls that can overlap on the
 * GPU (on different streams, or from different host threads) race on it and
 * must be serialised by the caller.
 */
int fb_attn_fwd_noalloc(int dt, int B, int H, int N, int d,
                        const void *Q, const void *K, const void *V,
                        int R, const float *phi_q, const float *phi_k,
                        int64_t phi_bstride, int64_t phi_hstride,
                        float scale, int causal,
                        void *O, float *LSE, void *stream);

/*
 * Comparison path, "FlashAttention w/ Bias" (FlashBias Figure 1(c)): the same
 * attention with a materialised dense bias that is streamed from HBM tile by
 * tile (the quadratic bias IO that FlashBias avoids, Figure 2).
 *
 *  Bias        [., ., N, N] device, dtype dt; element (b, h, i, j) sits at
 *              b*bias_bstride + h*bias_hstride + i*N + j (strides in
 *              elements, 0 = broadcast, otherwise multiples of 8).
 *              bf16 path: N % 8 == 0 (TMA row pitch) and 16-byte alignment.
 *  Other arguments as fb_attn_fwd. No workspace.
 */
int fb_attn_dense_bias_fwd(int dt, int B, int H, int N, int d,
                           const void *Q, const void *K, const void *V,
                           const void *Bias, int64_t bias_bstride,
                           int64_t bias_hstride, float scale, int causal,
                           void *O, float *LSE, void *stream);

/*
 * Exact Sandwich factors (rebuttal, reply to Reviewer UJUf, Q1 (1)-(2)):
 *   b_ij = sum_{k=1}^{C/2} cos((i-j) / 10000^{2k/C}) = phi(i) . phi(j),
 *   phi(i) = [cos(i w_1), sin(i w_1), ..., cos(i w_{C/2}), sin(i w_{C/2})],
 *   w_k = 10000^{-2k/C}.
 * Writes phi_q and phi_k, each [N, C] fp32 device (rank R = C), computed in
 * fp64. phi_k may be NULL or equal phi_q (the two factors are identical).
 * C even, 2 <= C <= 128.
 */
int fb_factors_sandwich(int N, int C, float *phi_q, float *phi_k, void *stream);

/*
 * Exact rank-2 ALiBi factors (FlashBias Example 3.4; rebuttal, reply to
 * Reviewer BRmd, Q2 (2): Block x 2 factor tiles in place of the
 * Block x Block bias): for head h of H, m_h = 2^{-8(h+1)/H},
 *   phi_q(i) = [-m_h i, 1],  phi_k(j) = [1, m_h j],  phi_q(i).phi_k(j) = -m_h (i-j).
 * Writes phi_q, phi_k as [H, N, 2] fp32 device (use phi_bstride = 0,
 * phi_hstride = 2N). Products are formed in fp64 and rounded once.
 */
int fb_factors_alibi(int H, int N, float *phi_q, float *phi_k, void *stream);

/*
 * Truncated SVD of one head's static dense bias on the host (rebuttal, reply
 * to Reviewer xU4x, Q6: SVD decomposition, rank chosen per head; computed
 * once, not per inference). Randomized range finder with `oversample` extra
 * columns and `power_iters` subspace iterations, then a one-sided Jacobi SVD
 * of the projected matrix. Balanced split: phi_q = U_R sqrt(S_R),
 * phi_k = V_R sqrt(S_R).
 *
 *  bias_host     [N, N] fp64 host, row-major.
 *  R             rank, 1 <= R <= min(N, 128); R + oversample <= N is clamped.
 *  seed          seeds the Gaussian test matrix.
 *  phi_q_host, phi_k_host   [N, R] fp32 host outputs.
 *  rel_fro_err   optional: ||B - phi_q phi_k^T||_F / ||B||_F (exact, fp64).
 *  energy        optional: sum_{r<R} s_r^2 / ||B||_F^2.
 * Synchronous; uses the host's cores. Allocates host memory internally.
 */
int fb_svd_factors_host(const double *bias_host, int N, int R, int oversample,
                        int power_iters, uint64_t seed, float *phi_q_host,
                        float *phi_k_host, double *rel_fro_err, double *energy);

/*
 * Synchronises `stream`, then reads and clears the library's device flag:
 * FB_ERR_TIMEOUT if a kernel's bounded wait ran out, FB_ERR_RANGE if a factor
 * overflowed fp16 in the preparation step, FB_OK otherwise (FB_ERR_CUDA if
 * the synchronisation itself failed). The flag is per device and shared by
 * all calls on that device.
 */
int fb_check_device_error(void *stream);

/*
 * Self-test of the failure path: launches one CTA whose pipeline wait is on
 * a barrier that nothing completes, with a limit of `limit_ms` milliseconds
 * (1 <= limit_ms <= 2000). The kernel gives up, records FB_ERR_TIMEOUT in
 * the device flag and exits normally; the context stays usable. Returns the
 * launch status; read the outcome with fb_check_device_error().
 */
int fb_selftest_wait_timeout(int limit_ms, void *stream);

#ifdef __cplusplus
}
#endif
#endif /* FLASHBIAS_H_ */
