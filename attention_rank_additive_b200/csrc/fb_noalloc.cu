// fb_noalloc.cu -- fb_attn_fwd_noalloc: the fused forward for callers that
// cannot allocate device memory.
//
// fb_attn_fwd needs a caller-provided workspace for the prepared factors
// (phi_q / scale and phi_k converted to the type the tensor cores read,
// padded to the MMA width). Some callers have no way to provide it: code
// running where every allocation is owned by someone else (a host framework
// with its own pool that exposes only the tensors it passes in, a plugin
// interface whose signature has inputs and outputs only), or code that must
// not allocate at all on its path (cudaMalloc synchronises the device and
// can fail under memory pressure). For them this entry point keeps the
// workspace in a fixed array in the library's own device memory.
//
// The array below is allocated when the module is loaded on a device and
// stays reserved on every device that loads the library until the process
// exits. Its size is the limit: calls whose prepared factors need more are
// rejected before anything runs.
#include <mutex>

#include "fb_internal.h"

namespace fb {
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(8) << 20;  // 8 MiB per device

// File-scope device scratch. Host code may not use this name as an address:
// on the host it is only a stand-in for the symbol, so the device address is
// looked up with cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void *g_scratch_ptr[kMaxDevices] = {nullptr};

// Device address of the scratch array on the current device, looked up once
// per device (with that device current) and cached. Returns nullptr on error.
void *scratch_for_current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_scratch_ptr[dev] == nullptr) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return nullptr;
    g_scratch_ptr[dev] = p;
  }
  return g_scratch_ptr[dev];
}

}  // namespace
}  // namespace fb

extern "C" int fb_attn_fwd_noalloc(int dt, int B, int H, int N, int d, const void *Q, const void *K, const void *V,
                                   int R, const float *phi_q, const float *phi_k, int64_t phi_bstride,
                                   int64_t phi_hstride, float scale, int causal, void *O, float *LSE, void *stream) {
  // fb_attn_fwd's own argument checks come first, so that both entry points
  // report the same status for the same bad argument; the size limit of the
  // fixed array is checked after them.
  if (const int a = fb::fwd_arg_status(dt, B, H, N, d, Q, K, V, R, phi_q, phi_k, phi_bstride, phi_hstride, scale, O,
                                       LSE))
    return a;
  size_t need = 0;
  if (dt == FB_BF16) {
    need = fb_attn_workspace_bytes(B, H, N, R, phi_bstride, phi_hstride);
    if (need > fb::kNoAllocScratchBytes) return FB_ERR_WORKSPACE;  // beyond the fixed scratch
  }
  void *scratch = nullptr;
  if (need > 0) {
    scratch = fb::scratch_for_current_device();
    if (scratch == nullptr) return FB_ERR_CUDA;
  }
  // The factor preparation inside overwrites every scratch byte the kernel
  // reads, so nothing has to be cleared between calls.
  return fb_attn_fwd(dt, B, H, N, d, Q, K, V, R, phi_q, phi_k, phi_bstride, phi_hstride, scale, causal, O, LSE,
                     scratch, need, stream);
}
