// fb_api.cu -- the extern "C" entry points of libflashbias: argument
// validation, the launch plan, TMA tensor maps and the launches. Every check
// that can fail does so before anything is launched.
#include <algorithm>
#include <cmath>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "fb_internal.h"

namespace fb {

__device__ int g_device_flags;  // one word per device; see fb_check_device_error

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_mu;
int *g_flag_ptr[kMaxDevices] = {nullptr};

using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                   const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, []() {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int pad_dim(int d) { return d <= 16 ? 16 : (d <= 32 ? 32 : (d <= 64 ? 64 : 128)); }
int pad_rank(int r) { return r <= 16 ? 16 : (r <= 32 ? 32 : (r <= 64 ? 64 : 128)); }

CUtensorMapSwizzle swizzle_for(int row_bytes) {
  return row_bytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                          : (row_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                             : (row_bytes == 32 ? CU_TENSOR_MAP_SWIZZLE_32B
                                                                : CU_TENSOR_MAP_SWIZZLE_NONE));
}

// Tiled map over a tensor of `rank` dims (innermost first), strides in bytes
// for dims 1..rank-1.
bool encode(CUtensorMap *m, CUtensorMapDataType dt, int rank, const void *ptr, const uint64_t *dims,
            const uint64_t *strides, const uint32_t *box, CUtensorMapSwizzle swz) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t gd[5], gs[4];
  cuuint32_t bx[5], es[5];
  for (int i = 0; i < rank; ++i) {
    gd[i] = dims[i];
    bx[i] = box[i];
    es[i] = 1;
  }
  for (int i = 0; i < rank - 1; ++i) gs[i] = strides[i];
  CUresult r = fn(m, dt, cuuint32_t(rank), const_cast<void *>(ptr), gd, gs, bx, es, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Q/K/V: bf16 [BH, N, d] with a box of (min(DP, 64), 128, 1).
// Heads per group of the fused kernel's item order (read by the head-dim-128
// kernels): all of them when every head's K and V (bf16) fit in a 64 MiB
// share of the 126 MB L2, else as many as do (ALiBi N8192 d128: 16 of 64
// heads; 6 % faster than one group there).
int head_group(int BH, int N, int DP) {
  const long long per_head = (long long)N * DP * 2 * 2;
  const long long budget = 64ll << 20;
  if ((long long)BH * per_head <= budget) return BH;
  return int(std::max<long long>(1, std::min<long long>(BH, budget / per_head)));
}

bool encode_qkv(CUtensorMap *m, const void *ptr, int BH, int N, int d, int DP) {
  const int ch = DP > 64 ? 64 : DP;
  const uint64_t dims[3] = {uint64_t(d), uint64_t(N), uint64_t(BH)};
  const uint64_t strides[2] = {uint64_t(d) * 2, uint64_t(N) * d * 2};
  const uint32_t box[3] = {uint32_t(ch), 128u, 1u};
  return encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, ptr, dims, strides, box, swizzle_for(ch * 2));
}

// O: bf16 [BH, N, d] with a box of (e, 32, 1), e the plan's epilogue chunk
// width: the per-warp TMA store (columns and rows past the tensor are not
// written).
bool encode_o(CUtensorMap *m, void *ptr, int BH, int N, int d, int e) {
  if (e != 16 && e != 32 && e != 64) return false;
  const uint64_t dims[3] = {uint64_t(d), uint64_t(N), uint64_t(BH)};
  const uint64_t strides[2] = {uint64_t(d) * 2, uint64_t(N) * d * 2};
  const uint32_t box[3] = {uint32_t(e), 32u, 1u};
  return encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, ptr, dims, strides, box, swizzle_for(e * 2));
}

int *flags_for_current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_flag_ptr[dev]) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_device_flags) != cudaSuccess) return nullptr;
    g_flag_ptr[dev] = static_cast<int *>(p);
  }
  return g_flag_ptr[dev];
}

struct WsLayout {
  size_t q_off, k_off, sched_off, total;
};

// Rank <= 4 factors go to the tensor cores as tf32 hi/lo parts: q' = [qh, qh, ql],
// k' = [kh, kl, kh] (3R columns, zero-padded to 8 or 16).
int tf32_cols(int R) { return R <= 2 ? 8 : 16; }

WsLayout workspace_layout(int B, int H, int N, int R, int64_t bs, int64_t hs) {
  WsLayout w{0, 0, 0, 0};
  if (R <= 0) return w;
  const size_t fb = size_t(bs == 0 ? 1 : B) * size_t(hs == 0 ? 1 : H);
  // rank <= 4: fp32 hi/lo split factors, 8 or 16 columns; else fp16 padded to 16..128
  const size_t per = R <= 4 ? fb * size_t(N) * size_t(tf32_cols(R)) * 4 : fb * size_t(N) * size_t(pad_rank(R)) * 2;
  const size_t per_al = (per + 255) & ~size_t(255);
  w.q_off = 0;
  w.k_off = per_al;
  // the fused kernel's work counter (two words; zeroed by the preparation
  // step, reset by the kernel itself at the end of every launch)
  w.sched_off = 2 * per_al;
  w.total = 2 * per_al + 256;
  return w;
}

bool valid_shape_bf16(int B, int H, int N, int d) {
  // the kernel numbers its work items (B * H * query-tile groups) in int
  return B >= 1 && H >= 1 && N >= 1 && d >= 8 && d <= 128 && d % 8 == 0 && (long long)B * H <= (1ll << 31) - 1 &&
         (long long)N <= (1ll << 31) - 256 && ((long long)N + 255) / 256 <= 65535 &&
         (long long)B * H * (((long long)N + 127) / 128) <= (1ll << 30);
}

bool valid_scale(float s) { return std::isfinite(s) && s > 0.f; }

// FB_ERR_INVALID_ARG for an empty batch, head count or sequence, else
// FB_ERR_UNSUPPORTED for a shape the tensor-core kernels do not take, else FB_OK.
int shape_status_bf16(int B, int H, int N, int d) {
  if (B < 1 || H < 1 || N < 1) return FB_ERR_INVALID_ARG;
  return valid_shape_bf16(B, H, N, d) ? FB_OK : FB_ERR_UNSUPPORTED;
}

// Pick query tiles per CTA: two (the K/V tiles serve 256 rows) when there are
// enough CTAs to fill the GPU at one CTA per SM and the ring keeps >= 2 stages.
// FLASHBIAS_QUERY_TILES=1|2 pins the choice (a tuning and test knob).
int forced_query_tiles() {
  const char *e = std::getenv("FLASHBIAS_QUERY_TILES");
  if (!e) return 0;
  const int v = std::atoi(e);
  return (v == 1 || v == 2) ? v : 0;
}

FwdPlan choose_plan(int DP, int RP, int mode, int BH, int N, int num_sms) {
  const FwdPlan p2{DP, RP, mode, 2}, p1{DP, RP, mode, 1};
  const int forced = forced_query_tiles();
  if (forced == 2 && sm100_smem_bytes(p2) > 0) return p2;
  if (forced == 1 && sm100_smem_bytes(p1) > 0) return p1;
  // One query tile per CTA when two such CTAs fit on an SM (small head dim
  // and rank): the two CTAs run independently and their softmax phases
  // interleave, which beats two tiles sharing one pipeline (measured on the
  // d = 16 workload: 194 vs 215 us). Head dim 128 uses the key-split plan at
  // one tile per CTA, which needs a whole SM.
  const size_t smem1 = sm100_smem_bytes(p1);
  if (DP < 128 && smem1 > 0 && 2 * (smem1 + 1024) <= 228 * 1024) return p1;
  const long long ctas2 = (long long)BH * ((N + 255) / 256);
  if (sm100_smem_bytes(p2) > 0 && ctas2 >= 2ll * num_sms) return p2;
  if (sm100_smem_bytes(p1) > 0) return p1;
  return p2;
}

int sm_count() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n;
}

}  // namespace

int *device_flags() { return flags_for_current_device(); }

// Every argument check of fb_attn_fwd except the workspace, in its order.
int fwd_arg_status(int dt, int B, int H, int N, int d, const void *Q, const void *K, const void *V, int R,
                   const float *phi_q, const float *phi_k, int64_t phi_bstride, int64_t phi_hstride, float scale,
                   const void *O, const float *LSE) {
  if (!Q || !K || !V || !O || !LSE) return FB_ERR_INVALID_ARG;
  if (R < 0 || R > 128) return FB_ERR_UNSUPPORTED;
  if (R > 0 && (!phi_q || !phi_k || phi_bstride < 0 || phi_hstride < 0)) return FB_ERR_INVALID_ARG;
  if (!valid_scale(scale)) return FB_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O) || !aligned16(LSE)) return FB_ERR_INVALID_ARG;
  if (R > 0 && (((reinterpret_cast<uintptr_t>(phi_q) | reinterpret_cast<uintptr_t>(phi_k)) & 3u) != 0))
    return FB_ERR_INVALID_ARG;
  if (dt == FB_F32) {
    if (B < 1 || H < 1 || N < 1) return FB_ERR_INVALID_ARG;
    if (d < 4 || d > 128 || d % 4 != 0 || (N + 31) / 32 > (1 << 30) || (long long)B * H > 65535)
      return FB_ERR_UNSUPPORTED;
    return FB_OK;
  }
  if (dt != FB_BF16) return FB_ERR_UNSUPPORTED;
  return shape_status_bf16(B, H, N, d);
}

}  // namespace fb

using namespace fb;

extern "C" {

const char *fb_status_str(int s) {
  switch (s) {
    case FB_OK: return "FB_OK";
    case FB_ERR_INVALID_ARG: return "FB_ERR_INVALID_ARG";
    case FB_ERR_UNSUPPORTED: return "FB_ERR_UNSUPPORTED";
    case FB_ERR_RANGE: return "FB_ERR_RANGE";
    case FB_ERR_WORKSPACE: return "FB_ERR_WORKSPACE";
    case FB_ERR_CUDA: return "FB_ERR_CUDA";
    case FB_ERR_TIMEOUT: return "FB_ERR_TIMEOUT";
    default: return "FB_ERR_UNKNOWN";
  }
}

int fb_version(void) { return 100; }

size_t fb_attn_workspace_bytes(int B, int H, int N, int R, int64_t phi_bstride, int64_t phi_hstride) {
  if (B < 1 || H < 1 || N < 1 || R < 0 || R > 128) return 0;
  return workspace_layout(B, H, N, R, phi_bstride, phi_hstride).total;
}

int fb_attn_prepare_factors(int B, int H, int N, int R, const float *phi_q, const float *phi_k, int64_t phi_bstride,
                            int64_t phi_hstride, float scale, void *workspace, size_t workspace_bytes, void *stream) {
  if (B < 1 || H < 1 || N < 1) return FB_ERR_INVALID_ARG;
  if (R < 0 || R > 128) return FB_ERR_UNSUPPORTED;
  if (R == 0) return FB_OK;
  if (!phi_q || !phi_k || phi_bstride < 0 || phi_hstride < 0) return FB_ERR_INVALID_ARG;
  if (((reinterpret_cast<uintptr_t>(phi_q) | reinterpret_cast<uintptr_t>(phi_k)) & 3u) != 0) return FB_ERR_INVALID_ARG;
  if (!valid_scale(scale)) return FB_ERR_INVALID_ARG;
  if ((long long)N > (1ll << 31) - 256) return FB_ERR_UNSUPPORTED;
  const WsLayout ws = workspace_layout(B, H, N, R, phi_bstride, phi_hstride);
  if (!workspace || workspace_bytes < ws.total || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return FB_ERR_WORKSPACE;
  int *flags = device_flags();
  if (!flags) return FB_ERR_CUDA;
  const int mode = R <= 4 ? kBiasTf32 : kBiasMma;
  const int RP = mode == kBiasMma ? pad_rank(R) : tf32_cols(R);
  const int fac_B = phi_bstride == 0 ? 1 : B, fac_H = phi_hstride == 0 ? 1 : H;
  uint8_t *wsb = static_cast<uint8_t *>(workspace);
  const cudaError_t e = launch_prep_factors(mode, B, H, N, R, RP, phi_q, phi_k, phi_bstride, phi_hstride, fac_B,
                                            fac_H, scale, wsb + ws.q_off, wsb + ws.k_off, flags,
                                            reinterpret_cast<unsigned int *>(wsb + ws.sched_off),
                                            static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? FB_OK : FB_ERR_CUDA;
}

int fb_attn_fwd_prepared(int dt, int B, int H, int N, int d, const void *Q, const void *K, const void *V, int R,
                         int64_t phi_bstride, int64_t phi_hstride, float scale, int causal, void *O, float *LSE,
                         const void *workspace, size_t workspace_bytes, void *stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (!Q || !K || !V || !O || !LSE) return FB_ERR_INVALID_ARG;
  if (dt != FB_BF16) return FB_ERR_UNSUPPORTED;
  if (R < 0 || R > 128) return FB_ERR_UNSUPPORTED;
  if (R > 0 && (phi_bstride < 0 || phi_hstride < 0)) return FB_ERR_INVALID_ARG;
  if (!valid_scale(scale)) return FB_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O) || !aligned16(LSE)) return FB_ERR_INVALID_ARG;
  if (const int sh = shape_status_bf16(B, H, N, d)) return sh;

  const WsLayout ws = workspace_layout(B, H, N, R, phi_bstride, phi_hstride);
  if (ws.total > 0) {
    if (!workspace || workspace_bytes < ws.total) return FB_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return FB_ERR_WORKSPACE;
  }
  const int DP = pad_dim(d);
  const int mode = R == 0 ? kBiasNone : (R <= 4 ? kBiasTf32 : kBiasMma);
  const int RP = mode == kBiasMma ? pad_rank(R) : (mode == kBiasTf32 ? tf32_cols(R) : 0);
  const int fac_B = phi_bstride == 0 ? 1 : B, fac_H = phi_hstride == 0 ? 1 : H;
  const FwdPlan plan = choose_plan(DP, RP, mode, B * H, N, sm_count());
  if (sm100_smem_bytes(plan) == 0) return FB_ERR_UNSUPPORTED;

  int *flags = device_flags();
  if (!flags) return FB_ERR_CUDA;

  FwdMaps maps;
  std::memset(&maps, 0, sizeof(maps));
  const int BH = B * H;
  if (!encode_qkv(&maps.q, Q, BH, N, d, DP) || !encode_qkv(&maps.k, K, BH, N, d, DP) ||
      !encode_qkv(&maps.v, V, BH, N, d, DP) || !encode_o(&maps.o, O, BH, N, d, sm100_epi_cols(plan)))
    return FB_ERR_CUDA;
  const uint8_t *wsb = static_cast<const uint8_t *>(workspace);
  void *wq = ws.total ? const_cast<uint8_t *>(wsb) + ws.q_off : nullptr;
  void *wk = ws.total ? const_cast<uint8_t *>(wsb) + ws.k_off : nullptr;
  const int FB = fac_B * fac_H;
  if (mode == kBiasMma) {
    const int ch = RP > 64 ? 64 : RP;
    const uint64_t dims[3] = {uint64_t(RP), uint64_t(N), uint64_t(FB)};
    const uint64_t strides[2] = {uint64_t(RP) * 2, uint64_t(N) * RP * 2};
    const uint32_t box[3] = {uint32_t(ch), 128u, 1u};
    if (!encode(&maps.fq, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, wq, dims, strides, box, swizzle_for(ch * 2)) ||
        !encode(&maps.fk, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, wk, dims, strides, box, swizzle_for(ch * 2)))
      return FB_ERR_CUDA;
  } else if (mode == kBiasTf32) {
    const uint64_t dims[3] = {uint64_t(RP), uint64_t(N), uint64_t(FB)};
    const uint64_t strides[2] = {uint64_t(RP) * 4, uint64_t(N) * RP * 4};
    const uint32_t box[3] = {uint32_t(RP), 128u, 1u};
    if (!encode(&maps.fq, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, wq, dims, strides, box, swizzle_for(RP * 4)) ||
        !encode(&maps.fk, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, wk, dims, strides, box, swizzle_for(RP * 4)))
      return FB_ERR_CUDA;
  }

  FwdArgs a;
  std::memset(&a, 0, sizeof(a));
  a.B = B, a.H = H, a.N = N, a.d = d;
  a.n_kv = (N + 127) / 128;
  a.n_cta_q = (a.n_kv + plan.QT - 1) / plan.QT;
  a.head_group = head_group(B * H, N, plan.DP);
  a.scale_log2 = scale * 1.4426950408889634f;
  a.scale = scale;
  a.causal = causal ? 1 : 0;
  a.O = O;
  a.LSE = LSE;
  a.fac_B = fac_B, a.fac_H = fac_H;
  a.bias_B = 1, a.bias_H = 1;
  a.flags = flags;
  a.sched = ws.total ? reinterpret_cast<unsigned int *>(const_cast<uint8_t *>(wsb) + ws.sched_off) : nullptr;
  const cudaError_t e = sm100_launch(plan, maps, a, st);
  return e == cudaSuccess ? FB_OK : FB_ERR_CUDA;
}


int fb_attn_fwd(int dt, int B, int H, int N, int d, const void *Q, const void *K, const void *V, int R,
                const float *phi_q, const float *phi_k, int64_t phi_bstride, int64_t phi_hstride, float scale,
                int causal, void *O, float *LSE, void *workspace, size_t workspace_bytes, void *stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (const int a = fwd_arg_status(dt, B, H, N, d, Q, K, V, R, phi_q, phi_k, phi_bstride, phi_hstride, scale, O,
                                   LSE))
    return a;

  if (dt == FB_F32) {
    int *flags = device_flags();
    if (!flags) return FB_ERR_CUDA;
    cudaError_t e = f32_launch(B, H, N, d, static_cast<const float *>(Q), static_cast<const float *>(K),
                               static_cast<const float *>(V), R, phi_q, phi_k, phi_bstride, phi_hstride, nullptr, 0, 0,
                               scale, causal, static_cast<float *>(O), LSE, st);
    return e == cudaSuccess ? FB_OK : FB_ERR_CUDA;
  }
  const WsLayout ws = workspace_layout(B, H, N, R, phi_bstride, phi_hstride);
  if (ws.total > 0) {
    if (!workspace || workspace_bytes < ws.total) return FB_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return FB_ERR_WORKSPACE;
  }
  // the preparation step, then the fused kernel, in stream order
  int rc = fb_attn_prepare_factors(B, H, N, R, phi_q, phi_k, phi_bstride, phi_hstride, scale, workspace,
                                   workspace_bytes, stream);
  if (rc != FB_OK) return rc;
  return fb_attn_fwd_prepared(dt, B, H, N, d, Q, K, V, R, phi_bstride, phi_hstride, scale, causal, O, LSE, workspace,
                              workspace_bytes, stream);
}

namespace {
struct MulLayout {
  size_t q1_off, k1_off, fac_off, fac_bytes, total;
  int Rf;  // rank of the factor part: d (R - 1)
};
size_t align256(size_t x) { return (x + 255) & ~size_t(255); }
MulLayout mul_layout(int B, int H, int N, int d, int R) {
  MulLayout m{};
  const size_t qk = size_t(B) * H * N * d * 2;
  m.Rf = d * (R - 1);
  m.q1_off = 0;
  m.k1_off = align256(qk);
  m.fac_off = m.k1_off + align256(qk);
  const int64_t hs = int64_t(N) * m.Rf, bs = int64_t(H) * hs;
  m.fac_bytes = m.Rf > 0 ? workspace_layout(B, H, N, m.Rf, bs, hs).total : 0;
  m.total = m.fac_off + m.fac_bytes;
  return m;
}
}  // namespace

size_t fb_attn_mul_bias_workspace_bytes(int B, int H, int N, int d, int R) {
  if (B < 1 || H < 1 || N < 1 || R < 1 || d < 8 || d * (R - 1) > 128) return 0;
  return mul_layout(B, H, N, d, R).total;
}

int fb_attn_mul_bias_fwd(int dt, int B, int H, int N, int d, const void *Q, const void *K, const void *V, int R,
                         const float *phi_q, const float *phi_k, int64_t phi_bstride, int64_t phi_hstride, float scale,
                         int causal, void *O, float *LSE, void *workspace, size_t workspace_bytes, void *stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (!Q || !K || !V || !O || !LSE || !phi_q || !phi_k) return FB_ERR_INVALID_ARG;
  if (dt != FB_BF16) return FB_ERR_UNSUPPORTED;
  if (R < 1 || d * (R - 1) > 128) return FB_ERR_UNSUPPORTED;
  if (phi_bstride < 0 || phi_hstride < 0) return FB_ERR_INVALID_ARG;
  if (!valid_scale(scale)) return FB_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O) || !aligned16(LSE)) return FB_ERR_INVALID_ARG;
  if (((reinterpret_cast<uintptr_t>(phi_q) | reinterpret_cast<uintptr_t>(phi_k)) & 3u) != 0) return FB_ERR_INVALID_ARG;
  if (const int sh = shape_status_bf16(B, H, N, d)) return sh;
  const MulLayout m = mul_layout(B, H, N, d, R);
  if (!workspace || workspace_bytes < m.total || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return FB_ERR_WORKSPACE;
  int *flags = device_flags();
  if (!flags) return FB_ERR_CUDA;
  uint8_t *ws = static_cast<uint8_t *>(workspace);
  const int64_t hs = int64_t(N) * m.Rf, bs = int64_t(H) * hs;
  const WsLayout fl = workspace_layout(B, H, N, m.Rf, bs, hs);
  const int RP = m.Rf > 0 ? pad_rank(m.Rf) : 0;
  void *fq = m.Rf > 0 ? ws + m.fac_off + fl.q_off : nullptr;
  void *fk = m.Rf > 0 ? ws + m.fac_off + fl.k_off : nullptr;
  unsigned int *sched = m.Rf > 0 ? reinterpret_cast<unsigned int *>(ws + m.fac_off + fl.sched_off) : nullptr;
  if (launch_prep_mul_bias(B, H, N, d, R, RP, Q, K, phi_q, phi_k, phi_bstride, phi_hstride, ws + m.q1_off,
                           ws + m.k1_off, fq, fk, flags, sched, st) != cudaSuccess)
    return FB_ERR_CUDA;
  return fb_attn_fwd_prepared(FB_BF16, B, H, N, d, ws + m.q1_off, ws + m.k1_off, V, m.Rf, bs, hs, scale, causal, O, LSE,
                              m.Rf > 0 ? ws + m.fac_off : nullptr, m.fac_bytes, stream);
}

namespace {
// The forward's workspace is the prepared per-head factors (as fb_attn_fwd's
// with strides bs = H N R, hs = N R): the linear layers write them directly.
WsLayout neural_layout(int B, int H, int N, int R) {
  const int64_t hs = int64_t(N) * R, bs = int64_t(H) * hs;
  return workspace_layout(B, H, N, R, bs, hs);
}
bool neural_ok(int F, int R) { return F >= 1 && F <= 256 && R >= 1 && R <= 128 && F * R <= 8192; }
}  // namespace

size_t fb_attn_neural_workspace_bytes(int B, int H, int N, int F, int R) {
  if (B < 1 || H < 1 || N < 1 || !neural_ok(F, R)) return 0;
  return neural_layout(B, H, N, R).total;
}

int fb_attn_neural_fwd(int dt, int B, int H, int N, int d, const void *Q, const void *K, const void *V, int F,
                       int R, const float *X_q, const float *X_k, const float *W_q, const float *W_k, float scale,
                       int causal, void *O, float *LSE, void *workspace, size_t workspace_bytes, void *stream) {
  if (!Q || !K || !V || !O || !LSE || !X_q || !X_k || !W_q || !W_k) return FB_ERR_INVALID_ARG;
  if (dt != FB_BF16) return FB_ERR_UNSUPPORTED;
  if (!neural_ok(F, R)) return FB_ERR_UNSUPPORTED;
  if (!valid_scale(scale)) return FB_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O) || !aligned16(LSE)) return FB_ERR_INVALID_ARG;
  if (((reinterpret_cast<uintptr_t>(X_q) | reinterpret_cast<uintptr_t>(X_k) | reinterpret_cast<uintptr_t>(W_q) |
        reinterpret_cast<uintptr_t>(W_k)) & 3u) != 0)
    return FB_ERR_INVALID_ARG;
  if (const int sh = shape_status_bf16(B, H, N, d)) return sh;
  const WsLayout m = neural_layout(B, H, N, R);
  if (!workspace || workspace_bytes < m.total || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return FB_ERR_WORKSPACE;
  int *flags = device_flags();
  if (!flags) return FB_ERR_CUDA;
  uint8_t *ws = static_cast<uint8_t *>(workspace);
  // one launch makes the factors in the layout the fused kernel reads, the
  // fused kernel follows in stream order
  const bool tf32 = R <= 4;
  if (launch_neural_prep(B, H, N, F, R, tf32 ? tf32_cols(R) : pad_rank(R), tf32 ? 1 : 0, X_q, X_k, W_q, W_k, scale,
                         ws + m.q_off, ws + m.k_off, flags, reinterpret_cast<unsigned int *>(ws + m.sched_off),
                         static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return FB_ERR_CUDA;
  const int64_t hs = int64_t(N) * R, bs = int64_t(H) * hs;
  return fb_attn_fwd_prepared(FB_BF16, B, H, N, d, Q, K, V, R, bs, hs, scale, causal, O, LSE, ws, m.total, stream);
}

size_t fb_attn_neural_bwd_workspace_bytes(int B, int H, int N, int F, int R) {
  if (B < 1 || H < 1 || N < 1 || !neural_ok(F, R)) return 0;
  const size_t phi = align256(size_t(B) * H * N * R * 4);
  const int64_t hs = int64_t(N) * R, bs = int64_t(H) * hs;
  const size_t bwd = fb_attn_bwd_workspace_bytes(B, H, N, R, bs, hs);
  return bwd == 0 ? 0 : 4 * phi + bwd;
}

int fb_attn_neural_bwd(int dt, int B, int H, int N, int d, const void *Q, const void *K, const void *V, int F,
                       int R, const float *X_q, const float *X_k, const float *W_q, const float *W_k, float scale,
                       int causal, const void *O, const float *LSE, const void *dO, void *dQ, void *dK, void *dV,
                       float *dX_q, float *dX_k, float *dW_q, float *dW_k, void *workspace, size_t workspace_bytes,
                       void *stream) {
  if (!Q || !K || !V || !O || !LSE || !dO || !dQ || !dK || !dV || !X_q || !X_k || !W_q || !W_k || !dW_q || !dW_k)
    return FB_ERR_INVALID_ARG;
  if ((dX_q == nullptr) != (dX_k == nullptr)) return FB_ERR_INVALID_ARG;  // both or neither
  if (dt != FB_BF16) return FB_ERR_UNSUPPORTED;
  if (!neural_ok(F, R)) return FB_ERR_UNSUPPORTED;
  if (!valid_scale(scale)) return FB_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O) || !aligned16(LSE) || !aligned16(dO) ||
      !aligned16(dQ) || !aligned16(dK) || !aligned16(dV))
    return FB_ERR_INVALID_ARG;
  if (((reinterpret_cast<uintptr_t>(X_q) | reinterpret_cast<uintptr_t>(X_k) | reinterpret_cast<uintptr_t>(W_q) |
        reinterpret_cast<uintptr_t>(W_k) | reinterpret_cast<uintptr_t>(dW_q) | reinterpret_cast<uintptr_t>(dW_k) |
        reinterpret_cast<uintptr_t>(dX_q) | reinterpret_cast<uintptr_t>(dX_k)) & 3u) != 0)
    return FB_ERR_INVALID_ARG;
  if (const int sh = shape_status_bf16(B, H, N, d)) return sh;
  const size_t need = fb_attn_neural_bwd_workspace_bytes(B, H, N, F, R);
  if (need == 0) return FB_ERR_UNSUPPORTED;
  if (!workspace || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return FB_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t *ws = static_cast<uint8_t *>(workspace);
  const size_t phi = align256(size_t(B) * H * N * R * 4);
  float *pq = reinterpret_cast<float *>(ws), *pk = reinterpret_cast<float *>(ws + phi);
  float *dpq = reinterpret_cast<float *>(ws + 2 * phi), *dpk = reinterpret_cast<float *>(ws + 3 * phi);
  // the factors again (as the forward made them), the attention backward with
  // per-head factors, then the chain rule through the linear layers
  if (launch_neural_factors(B, H, N, F, R, X_q, X_k, W_q, W_k, pq, pk, st) != cudaSuccess) return FB_ERR_CUDA;
  const int64_t hs = int64_t(N) * R, bs = int64_t(H) * hs;
  const int rc = fb_attn_bwd(FB_BF16, B, H, N, d, Q, K, V, R, pq, pk, bs, hs, scale, causal, O, LSE, dO, dQ, dK, dV,
                             dpq, dpk, ws + 4 * phi, need - 4 * phi, stream);
  if (rc != FB_OK) return rc;
  return launch_neural_grads(B, H, N, F, R, X_q, X_k, W_q, W_k, dpq, dpk, dW_q, dW_k, dX_q, dX_k, st) ==
                 cudaSuccess
             ? FB_OK
             : FB_ERR_CUDA;
}

int fb_attn_dense_bias_fwd(int dt, int B, int H, int N, int d, const void *Q, const void *K, const void *V,
                           const void *Bias, int64_t bias_bstride, int64_t bias_hstride, float scale, int causal,
                           void *O, float *LSE, void *stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (!Q || !K || !V || !O || !LSE || !Bias) return FB_ERR_INVALID_ARG;
  if (bias_bstride < 0 || bias_hstride < 0) return FB_ERR_INVALID_ARG;
  if (!valid_scale(scale)) return FB_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O) || !aligned16(LSE) || !aligned16(Bias))
    return FB_ERR_INVALID_ARG;
  if (dt == FB_F32) {
    if (B < 1 || H < 1 || N < 1) return FB_ERR_INVALID_ARG;
    if (d < 4 || d > 128 || d % 4 != 0 || (long long)B * H > 65535) return FB_ERR_UNSUPPORTED;
    if (!device_flags()) return FB_ERR_CUDA;
    cudaError_t e = f32_launch(B, H, N, d, static_cast<const float *>(Q), static_cast<const float *>(K),
                               static_cast<const float *>(V), 0, nullptr, nullptr, 0, 0,
                               static_cast<const float *>(Bias), bias_bstride, bias_hstride, scale, causal,
                               static_cast<float *>(O), LSE, st);
    return e == cudaSuccess ? FB_OK : FB_ERR_CUDA;
  }
  if (dt != FB_BF16) return FB_ERR_UNSUPPORTED;
  if (const int sh = shape_status_bf16(B, H, N, d)) return sh;
  if (N % 8 != 0 || bias_bstride % 8 != 0 || bias_hstride % 8 != 0) return FB_ERR_UNSUPPORTED;
  const int DP = pad_dim(d);
  // The dense path keeps a two-deep ring: one query tile per CTA when two do not leave room for it.
  FwdPlan plan{DP, 0, kBiasDense, 2};
  {
    const long long ctas2 = (long long)B * H * ((N + 255) / 256);
    const size_t s2 = sm100_smem_bytes(plan);
    FwdPlan p1{DP, 0, kBiasDense, 1};
    const bool deep2 = s2 > 0 && DP <= 64;
    const int forced = forced_query_tiles();
    if (forced == 1 || (forced != 2 && !(deep2 && ctas2 >= 2ll * sm_count()))) plan = p1;
    if (forced == 2 && s2 == 0) plan = p1;
    if (sm100_smem_bytes(plan) == 0) return FB_ERR_UNSUPPORTED;
  }
  int *flags = device_flags();
  if (!flags) return FB_ERR_CUDA;
  FwdMaps maps;
  std::memset(&maps, 0, sizeof(maps));
  const int BH = B * H;
  if (!encode_qkv(&maps.q, Q, BH, N, d, DP) || !encode_qkv(&maps.k, K, BH, N, d, DP) ||
      !encode_qkv(&maps.v, V, BH, N, d, DP) || !encode_o(&maps.o, O, BH, N, d, sm100_epi_cols(plan)))
    return FB_ERR_CUDA;
  const int bias_B = bias_bstride == 0 ? 1 : B, bias_H = bias_hstride == 0 ? 1 : H;
  {
    const uint64_t nn2 = uint64_t(N) * uint64_t(N) * 2;
    const uint64_t dims[4] = {uint64_t(N), uint64_t(N), uint64_t(bias_H), uint64_t(bias_B)};
    const uint64_t strides[3] = {uint64_t(N) * 2, bias_H > 1 ? uint64_t(bias_hstride) * 2 : nn2,
                                 bias_B > 1 ? uint64_t(bias_bstride) * 2 : nn2};
    const uint32_t box[4] = {64u, 128u, 1u, 1u};
    if (!encode(&maps.bias, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, Bias, dims, strides, box,
                CU_TENSOR_MAP_SWIZZLE_128B))
      return FB_ERR_CUDA;
  }
  FwdArgs a;
  std::memset(&a, 0, sizeof(a));
  a.B = B, a.H = H, a.N = N, a.d = d;
  a.n_kv = (N + 127) / 128;
  a.n_cta_q = (a.n_kv + plan.QT - 1) / plan.QT;
  a.head_group = head_group(B * H, N, plan.DP);
  a.scale_log2 = scale * 1.4426950408889634f;
  a.scale = scale;
  a.causal = causal ? 1 : 0;
  a.O = O;
  a.LSE = LSE;
  a.fac_B = 1, a.fac_H = 1;
  a.bias_B = bias_B, a.bias_H = bias_H;
  a.flags = flags;
  cudaError_t e = sm100_launch(plan, maps, a, st);
  return e == cudaSuccess ? FB_OK : FB_ERR_CUDA;
}

int fb_factors_sandwich(int N, int C, float *phi_q, float *phi_k, void *stream) {
  if (N < 1 || C < 2 || C > 128 || C % 2 != 0 || !phi_q) return FB_ERR_INVALID_ARG;
  return launch_sandwich(N, C, phi_q, phi_k, static_cast<cudaStream_t>(stream)) == cudaSuccess ? FB_OK : FB_ERR_CUDA;
}

int fb_factors_alibi(int H, int N, float *phi_q, float *phi_k, void *stream) {
  if (H < 1 || N < 1 || !phi_q || !phi_k) return FB_ERR_INVALID_ARG;
  return launch_alibi(H, N, phi_q, phi_k, static_cast<cudaStream_t>(stream)) == cudaSuccess ? FB_OK : FB_ERR_CUDA;
}

namespace {
struct BwdLayout {
  WsLayout f;  // the S-side factor tiles (as the forward's workspace)
  // acc_off: the fused kernel's fp32 dq' accumulator [BH, Npad, up to 128]; the
  // two-kernel path keeps its per-head dphi_q rows there instead (pq_off).
  size_t gq_off, gk_off, l_off, d_off, acc_off, pq_off, pk_off, sched_off, total;
  int RG, Npad;
  bool shared_slices;  // some factor slice serves several heads: per-head partial gradients
};
size_t al256(size_t x) { return (x + 255) & ~size_t(255); }
BwdLayout bwd_layout(int B, int H, int N, int R, int64_t bs, int64_t hs) {
  BwdLayout w{};
  w.f = workspace_layout(B, H, N, R, bs, hs);
  w.RG = R == 0 ? 0 : (R <= 4 ? 16 : pad_rank(R));
  w.Npad = int(((long long)N + 127) / 128 * 128);
  const size_t fb = size_t(bs == 0 ? 1 : B) * size_t(hs == 0 ? 1 : H);
  const size_t g = al256(fb * size_t(N) * size_t(w.RG) * 2);
  const size_t rows = al256(size_t(B) * H * size_t(w.Npad) * 4);
  w.gq_off = w.f.total;
  w.gk_off = w.gq_off + g;
  w.l_off = w.gk_off + g;
  w.d_off = w.l_off + rows;
  w.shared_slices = R > 0 && fb < size_t(B) * H;
  const size_t part = w.shared_slices ? al256(size_t(B) * H * size_t(N) * size_t(R) * 4) : 0;
  const size_t acc = al256(size_t(B) * H * size_t(w.Npad) * 128 * 4);  // >= part (R <= 128, N <= Npad)
  w.acc_off = w.d_off + rows;
  w.pq_off = w.acc_off;
  w.pk_off = w.acc_off + acc;
  w.sched_off = w.pk_off + part;  // the fused kernel's work counter
  w.total = w.sched_off + 256;
  return w;
}
bool encode_rows_bf16(CUtensorMap *m, const void *ptr, int slices, int N, int cols, int width, int rows) {
  const int ch = width > 64 ? 64 : width;
  const uint64_t dims[3] = {uint64_t(cols), uint64_t(N), uint64_t(slices)};
  const uint64_t strides[2] = {uint64_t(cols) * 2, uint64_t(N) * cols * 2};
  const uint32_t box[3] = {uint32_t(ch), uint32_t(rows), 1u};
  return encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, ptr, dims, strides, box, swizzle_for(ch * 2));
}
bool encode_fac(CUtensorMap *m, int mode, const void *ptr, int FB, int N, int RP, int rows) {
  const uint64_t dims[3] = {uint64_t(RP), uint64_t(N), uint64_t(FB)};
  if (mode == kBiasMma) {
    const int ch = RP > 64 ? 64 : RP;
    const uint64_t strides[2] = {uint64_t(RP) * 2, uint64_t(N) * RP * 2};
    const uint32_t box[3] = {uint32_t(ch), uint32_t(rows), 1u};
    return encode(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, ptr, dims, strides, box, swizzle_for(ch * 2));
  }
  const uint64_t strides[2] = {uint64_t(RP) * 4, uint64_t(N) * RP * 4};
  const uint32_t box[3] = {uint32_t(RP), uint32_t(rows), 1u};
  return encode(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, ptr, dims, strides, box, swizzle_for(RP * 4));
}
}  // namespace

size_t fb_attn_bwd_workspace_bytes(int B, int H, int N, int R, int64_t phi_bstride, int64_t phi_hstride) {
  if (B < 1 || H < 1 || N < 1 || R < 0 || R > 128 || phi_bstride < 0 || phi_hstride < 0) return 0;
  if (!valid_shape_bf16(B, H, N, 16)) return 0;
  return bwd_layout(B, H, N, R, phi_bstride, phi_hstride).total;
}

int fb_attn_bwd(int dt, int B, int H, int N, int d, const void *Q, const void *K, const void *V, int R,
                const float *phi_q, const float *phi_k, int64_t phi_bstride, int64_t phi_hstride, float scale,
                int causal, const void *O, const float *LSE, const void *dO, void *dQ, void *dK, void *dV,
                float *dphi_q, float *dphi_k, void *workspace, size_t workspace_bytes, void *stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (!Q || !K || !V || !O || !LSE || !dO || !dQ || !dK || !dV) return FB_ERR_INVALID_ARG;
  if (dt != FB_BF16) return FB_ERR_UNSUPPORTED;
  if (R < 0 || R > 128) return FB_ERR_UNSUPPORTED;
  // factor gradients: both or neither (neither: fixed factors, their products skipped)
  const bool want_dphi = dphi_q != nullptr && dphi_k != nullptr;
  if (R > 0 && (!phi_q || !phi_k || phi_bstride < 0 || phi_hstride < 0)) return FB_ERR_INVALID_ARG;
  if (R > 0 && !want_dphi && (dphi_q || dphi_k)) return FB_ERR_INVALID_ARG;
  if (R > 0 && (((reinterpret_cast<uintptr_t>(phi_q) | reinterpret_cast<uintptr_t>(phi_k) |
                  reinterpret_cast<uintptr_t>(dphi_q) | reinterpret_cast<uintptr_t>(dphi_k)) &
                 3u) != 0))
    return FB_ERR_INVALID_ARG;
  if (!valid_scale(scale)) return FB_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O) || !aligned16(dO) || !aligned16(dQ) ||
      !aligned16(dK) || !aligned16(dV) || !aligned16(LSE))
    return FB_ERR_INVALID_ARG;
  if (const int sh = shape_status_bf16(B, H, N, d)) return sh;
  const BwdLayout L = bwd_layout(B, H, N, R, phi_bstride, phi_hstride);
  if (!workspace || workspace_bytes < L.total || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return FB_ERR_WORKSPACE;
  BwdPlan plan;
  plan.DP = pad_dim(d);
  plan.mode = R == 0 ? kBiasNone : (R <= 4 ? kBiasTf32 : kBiasMma);
  plan.RP = plan.mode == kBiasMma ? pad_rank(R) : (plan.mode == kBiasTf32 ? tf32_cols(R) : 0);
  plan.RG = want_dphi ? L.RG : 0;
  const int BQ = bwd_query_block_rows(plan), BK = bwd_key_block_rows(plan);
  if (BQ == 0 || BK == 0) return FB_ERR_UNSUPPORTED;
  int *flags = device_flags();
  if (!flags) return FB_ERR_CUDA;

  uint8_t *wsb = static_cast<uint8_t *>(workspace);
  const int fac_B = phi_bstride == 0 ? 1 : B, fac_H = phi_hstride == 0 ? 1 : H;
  const int FB = fac_B * fac_H;
  const int BH = B * H;
  float *nlse2 = reinterpret_cast<float *>(wsb + L.l_off);
  float *delta = reinterpret_cast<float *>(wsb + L.d_off);

  // tensor maps first: a failure here returns before anything is launched
  BwdMaps maps;
  std::memset(&maps, 0, sizeof(maps));
  const int DP = plan.DP;
  if (!encode_rows_bf16(&maps.q, Q, BH, N, d, DP, 128) || !encode_rows_bf16(&maps.k, K, BH, N, d, DP, 128) ||
      !encode_rows_bf16(&maps.v, V, BH, N, d, DP, 128) || !encode_rows_bf16(&maps.dO, dO, BH, N, d, DP, 128) ||
      !encode_rows_bf16(&maps.q_blk, Q, BH, N, d, DP, BQ) || !encode_rows_bf16(&maps.do_blk, dO, BH, N, d, DP, BQ) ||
      !encode_rows_bf16(&maps.k_blk, K, BH, N, d, DP, BK) || !encode_rows_bf16(&maps.v_blk, V, BH, N, d, DP, BK))
    return FB_ERR_CUDA;
  if (R > 0) {
    void *wq = wsb + L.f.q_off, *wk = wsb + L.f.k_off;
    if (!encode_fac(&maps.fq, plan.mode, wq, FB, N, plan.RP, 128) ||
        !encode_fac(&maps.fk, plan.mode, wk, FB, N, plan.RP, 128) ||
        !encode_fac(&maps.fq_blk, plan.mode, wq, FB, N, plan.RP, BQ) ||
        !encode_fac(&maps.fk_blk, plan.mode, wk, FB, N, plan.RP, BK))
      return FB_ERR_CUDA;
    if (want_dphi && (!encode_rows_bf16(&maps.gq_blk, wsb + L.gq_off, FB, N, L.RG, L.RG, BQ) ||
                      !encode_rows_bf16(&maps.gk_blk, wsb + L.gk_off, FB, N, L.RG, L.RG, BK) ||
                      !encode_rows_bf16(&maps.gk, wsb + L.gk_off, FB, N, L.RG, L.RG, 128)))
      return FB_ERR_CUDA;
  }
  const bool fused = bwd_fused(plan);
  const int dqw = 64 + plan.RG;  // fused: accumulator columns (dQ | dphi_q)
  float *acc = reinterpret_cast<float *>(wsb + L.acc_off);
  if (fused) {
    const uint64_t dims[3] = {uint64_t(dqw), uint64_t(L.Npad), uint64_t(BH)};
    const uint64_t strides[2] = {uint64_t(dqw) * 4, uint64_t(L.Npad) * dqw * 4};
    const uint32_t box[3] = {uint32_t(dqw), dqw == 128 ? 16u : 32u, 1u};  // the kernel's staging pieces
    if (!encode(&maps.acc, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, acc, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_NONE))
      return FB_ERR_CUDA;
  }

  // 1. the forward's factor tiles (S is recomputed as the forward computed it)
  if (R > 0) {
    const int rc = fb_attn_prepare_factors(B, H, N, R, phi_q, phi_k, phi_bstride, phi_hstride, scale, workspace,
                                           workspace_bytes, stream);
    if (rc != FB_OK) return rc;
    // 2. bf16 factor copies for the gradient products
    if (want_dphi && launch_prep_grad_factors(N, R, L.RG, phi_q, phi_k, phi_bstride, phi_hstride, fac_B, fac_H,
                                              wsb + L.gq_off, wsb + L.gk_off, st) != cudaSuccess)
      return FB_ERR_CUDA;
  }
  // 3. per-row -LSE in log2 units and rowsum(dO * O)
  //    (and, fused, the zeroed accumulator)
  unsigned int *sched = reinterpret_cast<unsigned int *>(wsb + L.sched_off);
  if (launch_bwd_rows(BH, N, L.Npad, d, O, dO, LSE, nlse2, delta, fused ? acc : nullptr, dqw,
                      fused ? sched : nullptr, st) != cudaSuccess)
    return FB_ERR_CUDA;

  // 4. the gradient kernels: the fused kernel, or the dK/dV and dQ kernels
  BwdArgs a;
  std::memset(&a, 0, sizeof(a));
  a.B = B, a.H = H, a.N = N, a.d = d, a.R = R;
  a.n_kv = (N + 127) / 128;
  a.Npad = L.Npad;
  a.scale = scale;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.scale = scale;
  a.causal = causal ? 1 : 0;
  a.nlse2 = nlse2;
  a.delta = delta;
  a.dQ = dQ, a.dK = dK, a.dV = dV;
  a.dphi_q = dphi_q, a.dphi_k = dphi_k;
  a.dphi_direct = L.shared_slices ? 0 : 1;
  a.dphi_q_part = L.shared_slices ? reinterpret_cast<float *>(wsb + L.pq_off) : nullptr;
  a.dphi_k_part = L.shared_slices ? reinterpret_cast<float *>(wsb + L.pk_off) : nullptr;
  a.phi_bs = phi_bstride, a.phi_hs = phi_hstride;
  a.fac_B = fac_B, a.fac_H = fac_H;
  a.dqacc = fused ? acc : nullptr;
  a.sched = fused ? sched : nullptr;
  a.flags = flags;
  if (bwd_launch(plan, maps, a, st) != cudaSuccess) return FB_ERR_CUDA;
  // 5. fused: dQ (and per-head dphi_q) from the accumulator
  if (fused && launch_bwd_dq_convert(B, H, N, L.Npad, d, want_dphi ? R : 0, dqw, scale, acc, dQ,
                                     want_dphi && !L.shared_slices ? dphi_q : nullptr, phi_bstride, phi_hstride,
                                     fac_B, fac_H, st) != cudaSuccess)
    return FB_ERR_CUDA;
  // 6. factor slices shared by several heads: sum the per-head rows
  if (want_dphi && L.shared_slices) {
    const cudaError_t e =
        fused ? launch_reduce_factor_grads(B, H, N, R, fac_B, fac_H, phi_bstride, phi_hstride, acc,
                                           int64_t(L.Npad) * dqw, dqw, 64, a.dphi_k_part, dphi_q, dphi_k, st)
              : launch_reduce_factor_grads(B, H, N, R, fac_B, fac_H, phi_bstride, phi_hstride, a.dphi_q_part,
                                           int64_t(N) * R, R, 0, a.dphi_k_part, dphi_q, dphi_k, st);
    if (e != cudaSuccess) return FB_ERR_CUDA;
  }
  return FB_OK;
}

int fb_check_device_error(void *stream) {
  int *flags = device_flags();
  if (!flags) return FB_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return FB_ERR_CUDA;
  int host = 0;
  if (cudaMemcpyFromSymbol(&host, g_device_flags, sizeof(int)) != cudaSuccess) return FB_ERR_CUDA;
  const int zero = 0;
  if (cudaMemcpyToSymbol(g_device_flags, &zero, sizeof(int)) != cudaSuccess) return FB_ERR_CUDA;
  if (host & kFlagTimeout) return FB_ERR_TIMEOUT;
  if (host & kFlagRange) return FB_ERR_RANGE;
  return FB_OK;
}

int fb_selftest_wait_timeout(int limit_ms, void *stream) {
  if (limit_ms < 1 || limit_ms > 2000) return FB_ERR_INVALID_ARG;
  int *flags = device_flags();
  if (!flags) return FB_ERR_CUDA;
  return launch_wait_selftest(limit_ms, flags, static_cast<cudaStream_t>(stream)) == cudaSuccess ? FB_OK
                                                                                                 : FB_ERR_CUDA;
}

}  // extern "C"
