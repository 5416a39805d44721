"""attention_rank_additive_b200 -- attention with a low-rank additive bias on B200.

Python binding of libflashbias (the C ABI in include/flashbias.h). The
functions named ``fb_*`` mirror the C entry points one to one and take raw
integers for pointers; the helpers below them (``attn``, ``attn_dense_bias``,
``factors_sandwich``, ``factors_alibi``, ``svd_factors``) only marshal torch
tensors: every step of the computation runs in the library's kernels.

There is no fallback: importing works without a GPU, but the first call that
needs the library raises if ``libflashbias.so`` has not been built
(``python -m attention_rank_additive_b200.build``).
"""
from __future__ import annotations

import ctypes
import math
import os

__all__ = [
    "FB_OK", "FB_ERR_INVALID_ARG", "FB_ERR_UNSUPPORTED", "FB_ERR_RANGE", "FB_ERR_WORKSPACE", "FB_ERR_CUDA",
    "FB_ERR_TIMEOUT", "FB_F32", "FB_BF16", "FB_F16", "FlashBiasError", "lib", "lib_path", "EXPORTED",
    "fb_status_str", "fb_version", "fb_attn_workspace_bytes", "fb_attn_fwd", "fb_attn_dense_bias_fwd",
    "fb_factors_sandwich", "fb_factors_alibi", "fb_svd_factors_host", "fb_check_device_error",
    "fb_selftest_wait_timeout", "fb_attn_fwd_noalloc", "fb_attn_prepare_factors", "fb_attn_fwd_prepared",
    "fb_attn_mul_bias_workspace_bytes", "fb_attn_mul_bias_fwd", "attn_mul_bias", "attn",
    "fb_svd_device_workspace_bytes", "fb_svd_factors_device", "svd_factors_device",
    "fb_attn_neural_workspace_bytes", "fb_attn_neural_fwd", "attn_neural",
    "PreparedBias", "attn_dense_bias", "factors_sandwich", "factors_alibi", "svd_factors",
    "attn_flops",
]

FB_OK, FB_ERR_INVALID_ARG, FB_ERR_UNSUPPORTED, FB_ERR_RANGE, FB_ERR_WORKSPACE, FB_ERR_CUDA, FB_ERR_TIMEOUT = range(7)
FB_F32, FB_BF16, FB_F16 = 0, 1, 2

_HERE = os.path.dirname(os.path.abspath(__file__))
lib_path = os.path.join(_HERE, "libflashbias.so")

# Every symbol include/flashbias.h declares.
EXPORTED = (
    "fb_status_str", "fb_version", "fb_attn_workspace_bytes", "fb_attn_fwd", "fb_attn_dense_bias_fwd",
    "fb_factors_sandwich", "fb_factors_alibi", "fb_svd_factors_host", "fb_check_device_error",
    "fb_selftest_wait_timeout", "fb_attn_fwd_noalloc", "fb_attn_prepare_factors", "fb_attn_fwd_prepared",
    "fb_attn_mul_bias_workspace_bytes", "fb_attn_mul_bias_fwd", "fb_svd_device_workspace_bytes",
    "fb_svd_factors_device", "fb_attn_neural_workspace_bytes", "fb_attn_neural_fwd", "fb_attn_bwd_workspace_bytes",
    "fb_attn_bwd", "fb_attn_neural_bwd_workspace_bytes", "fb_attn_neural_bwd",
)


class FlashBiasError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {fb_status_str(status)} ({status})")


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded libflashbias; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(lib_path):
            raise RuntimeError(f"libflashbias.so is missing at {lib_path}; build it with "
                               "`python -m attention_rank_additive_b200.build`")
        L = ctypes.CDLL(lib_path)
        i32, i64, sz, vp, f32 = ctypes.c_int, ctypes.c_int64, ctypes.c_size_t, ctypes.c_void_p, ctypes.c_float
        L.fb_status_str.argtypes, L.fb_status_str.restype = [i32], ctypes.c_char_p
        L.fb_version.argtypes, L.fb_version.restype = [], i32
        L.fb_attn_workspace_bytes.argtypes = [i32, i32, i32, i32, i64, i64]
        L.fb_attn_workspace_bytes.restype = sz
        L.fb_attn_fwd.argtypes = [i32, i32, i32, i32, i32, vp, vp, vp, i32, vp, vp, i64, i64, f32, i32, vp, vp, vp,
                                  sz, vp]
        L.fb_attn_fwd.restype = i32
        L.fb_attn_fwd_noalloc.argtypes = [i32, i32, i32, i32, i32, vp, vp, vp, i32, vp, vp, i64, i64, f32, i32, vp,
                                          vp, vp]
        L.fb_attn_fwd_noalloc.restype = i32
        L.fb_attn_prepare_factors.argtypes = [i32, i32, i32, i32, vp, vp, i64, i64, f32, vp, sz, vp]
        L.fb_attn_prepare_factors.restype = i32
        L.fb_attn_fwd_prepared.argtypes = [i32, i32, i32, i32, i32, vp, vp, vp, i32, i64, i64, f32, i32, vp, vp, vp,
                                           sz, vp]
        L.fb_attn_fwd_prepared.restype = i32
        L.fb_attn_mul_bias_workspace_bytes.argtypes = [i32, i32, i32, i32, i32]
        L.fb_attn_mul_bias_workspace_bytes.restype = sz
        L.fb_attn_mul_bias_fwd.argtypes = [i32, i32, i32, i32, i32, vp, vp, vp, i32, vp, vp, i64, i64, f32, i32, vp,
                                           vp, vp, sz, vp]
        L.fb_attn_mul_bias_fwd.restype = i32
        L.fb_svd_device_workspace_bytes.argtypes = [i32, i32, i32, i32]
        L.fb_svd_device_workspace_bytes.restype = sz
        L.fb_svd_factors_device.argtypes = [i32, i32, i32, i32, i32, ctypes.c_uint64, vp, vp, vp, vp, vp, sz, vp]
        L.fb_svd_factors_device.restype = i32
        L.fb_attn_neural_workspace_bytes.argtypes = [i32, i32, i32, i32, i32]
        L.fb_attn_neural_workspace_bytes.restype = sz
        L.fb_attn_neural_fwd.argtypes = [i32, i32, i32, i32, i32, vp, vp, vp, i32, i32, vp, vp, vp, vp, f32, i32, vp,
                                         vp, vp, sz, vp]
        L.fb_attn_neural_fwd.restype = i32
        L.fb_attn_bwd_workspace_bytes.argtypes = [i32, i32, i32, i32, i64, i64]
        L.fb_attn_bwd_workspace_bytes.restype = sz
        L.fb_attn_bwd.argtypes = [i32, i32, i32, i32, i32, vp, vp, vp, i32, vp, vp, i64, i64, f32, i32, vp, vp, vp,
                                  vp, vp, vp, vp, vp, vp, sz, vp]
        L.fb_attn_bwd.restype = i32
        L.fb_attn_neural_bwd_workspace_bytes.argtypes = [i32, i32, i32, i32, i32]
        L.fb_attn_neural_bwd_workspace_bytes.restype = sz
        L.fb_attn_neural_bwd.argtypes = [i32, i32, i32, i32, i32, vp, vp, vp, i32, i32, vp, vp, vp, vp, f32, i32, vp,
                                         vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
        L.fb_attn_neural_bwd.restype = i32
        L.fb_attn_dense_bias_fwd.argtypes = [i32, i32, i32, i32, i32, vp, vp, vp, vp, i64, i64, f32, i32, vp, vp, vp]
        L.fb_attn_dense_bias_fwd.restype = i32
        L.fb_factors_sandwich.argtypes, L.fb_factors_sandwich.restype = [i32, i32, vp, vp, vp], i32
        L.fb_factors_alibi.argtypes, L.fb_factors_alibi.restype = [i32, i32, vp, vp, vp], i32
        L.fb_svd_factors_host.argtypes = [vp, i32, i32, i32, i32, ctypes.c_uint64, vp, vp, vp, vp]
        L.fb_svd_factors_host.restype = i32
        L.fb_check_device_error.argtypes, L.fb_check_device_error.restype = [vp], i32
        L.fb_selftest_wait_timeout.argtypes, L.fb_selftest_wait_timeout.restype = [i32, vp], i32
        _lib = L
    return _lib


# ---------------------------------------------------------------- raw C ABI

def fb_status_str(status: int) -> str:
    return lib().fb_status_str(int(status)).decode()


def fb_version() -> int:
    return lib().fb_version()


def fb_attn_workspace_bytes(B, H, N, R, phi_bstride, phi_hstride) -> int:
    return lib().fb_attn_workspace_bytes(B, H, N, R, phi_bstride, phi_hstride)


def fb_attn_fwd(dt, B, H, N, d, Q, K, V, R, phi_q, phi_k, phi_bstride, phi_hstride, scale, causal, O, LSE,
                workspace, workspace_bytes, stream) -> int:
    return lib().fb_attn_fwd(dt, B, H, N, d, Q, K, V, R, phi_q, phi_k, phi_bstride, phi_hstride, scale, causal, O,
                             LSE, workspace, workspace_bytes, stream)


def fb_attn_prepare_factors(B, H, N, R, phi_q, phi_k, phi_bstride, phi_hstride, scale, workspace, workspace_bytes,
                            stream) -> int:
    return lib().fb_attn_prepare_factors(B, H, N, R, phi_q, phi_k, phi_bstride, phi_hstride, scale, workspace,
                                         workspace_bytes, stream)


def fb_attn_fwd_prepared(dt, B, H, N, d, Q, K, V, R, phi_bstride, phi_hstride, scale, causal, O, LSE, workspace,
                         workspace_bytes, stream) -> int:
    return lib().fb_attn_fwd_prepared(dt, B, H, N, d, Q, K, V, R, phi_bstride, phi_hstride, scale, causal, O, LSE,
                                      workspace, workspace_bytes, stream)


def fb_attn_mul_bias_workspace_bytes(B, H, N, d, R) -> int:
    return lib().fb_attn_mul_bias_workspace_bytes(B, H, N, d, R)


def fb_attn_mul_bias_fwd(dt, B, H, N, d, Q, K, V, R, phi_q, phi_k, phi_bstride, phi_hstride, scale, causal, O, LSE,
                         workspace, workspace_bytes, stream) -> int:
    return lib().fb_attn_mul_bias_fwd(dt, B, H, N, d, Q, K, V, R, phi_q, phi_k, phi_bstride, phi_hstride, scale,
                                      causal, O, LSE, workspace, workspace_bytes, stream)


def fb_svd_device_workspace_bytes(H, N, R, oversample) -> int:
    return lib().fb_svd_device_workspace_bytes(H, N, R, oversample)


def fb_svd_factors_device(H, N, R, oversample, power_iters, seed, bias, phi_q, phi_k, err_energy, workspace,
                          workspace_bytes, stream) -> int:
    return lib().fb_svd_factors_device(H, N, R, oversample, power_iters, seed, bias, phi_q, phi_k, err_energy,
                                       workspace, workspace_bytes, stream)


def svd_factors_device(bias, R: int, oversample: int = 16, power_iters: int = 2, seed: int = 0):
    """Truncated SVD of dense biases on the GPU (fb_svd_factors_device).

    bias: fp32 CUDA tensor [N, N] or [H, N, N]. Returns (phi_q, phi_k, err_energy)
    with phi [.., N, R] fp32 on the device and err_energy a [H, 2] fp64 device
    tensor (relative Frobenius error, captured energy per head)."""
    import torch
    squeeze = bias.dim() == 2
    b = bias[None] if squeeze else bias
    assert b.is_cuda and b.dtype == torch.float32 and b.is_contiguous()
    H, N, _ = b.shape
    pq = torch.empty((H, N, R), device=b.device, dtype=torch.float32)
    pk = torch.empty_like(pq)
    ee = torch.empty((H, 2), device=b.device, dtype=torch.float64)
    nb = fb_svd_device_workspace_bytes(H, N, R, oversample)
    ws = torch.empty(max(nb, 1), device=b.device, dtype=torch.uint8)
    _check(fb_svd_factors_device(H, N, R, oversample, power_iters, seed, b.data_ptr(), pq.data_ptr(), pk.data_ptr(),
                                 ee.data_ptr(), ws.data_ptr(), nb, _stream(b.device)), "fb_svd_factors_device")
    if squeeze:
        return pq[0], pk[0], ee
    return pq, pk, ee


def fb_attn_neural_workspace_bytes(B, H, N, F, R) -> int:
    return lib().fb_attn_neural_workspace_bytes(B, H, N, F, R)


def fb_attn_neural_fwd(dt, B, H, N, d, Q, K, V, F, R, X_q, X_k, W_q, W_k, scale, causal, O, LSE, workspace,
                       workspace_bytes, stream) -> int:
    return lib().fb_attn_neural_fwd(dt, B, H, N, d, Q, K, V, F, R, X_q, X_k, W_q, W_k, scale, causal, O, LSE,
                                    workspace, workspace_bytes, stream)


def attn_neural(q, k, v, x_q, x_k, w_q, w_k, scale=None, causal=False, out=None, lse=None):
    """Attention whose bias factors come from linear layers on token features
    (fb_attn_neural_fwd): phi_q[b, h] = x_q[b] w_q[h], phi_k[b, h] = x_k[b] w_k[h].

    q, k, v: bf16 CUDA [B, H, N, d]; x_q, x_k: fp32 [B, N, F]; w_q, w_k: fp32
    [H, F, R]. Returns (O, LSE)."""
    import torch
    assert q.is_cuda and q.dtype == torch.bfloat16 and q.is_contiguous() and k.is_contiguous() \
        and v.is_contiguous()
    for t in (x_q, x_k, w_q, w_k):
        assert t.is_cuda and t.dtype == torch.float32 and t.is_contiguous()
    B, H, N, d = q.shape
    F, R = w_q.shape[1], w_q.shape[2]
    assert x_q.shape == (B, N, F) and x_k.shape == (B, N, F) and w_k.shape == (H, F, R)
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    o = torch.empty_like(q) if out is None else out
    l = torch.empty((B, H, N), device=q.device, dtype=torch.float32) if lse is None else lse
    nb = fb_attn_neural_workspace_bytes(B, H, N, F, R)
    ws = torch.empty(max(nb, 1), device=q.device, dtype=torch.uint8)
    _check(fb_attn_neural_fwd(FB_BF16, B, H, N, d, q.data_ptr(), k.data_ptr(), v.data_ptr(), F, R, x_q.data_ptr(),
                              x_k.data_ptr(), w_q.data_ptr(), w_k.data_ptr(), scale, int(bool(causal)), o.data_ptr(),
                              l.data_ptr(), ws.data_ptr(), nb, _stream(q.device)), "fb_attn_neural_fwd")
    return o, l


def fb_attn_bwd_workspace_bytes(B, H, N, R, phi_bstride, phi_hstride) -> int:
    return lib().fb_attn_bwd_workspace_bytes(B, H, N, R, phi_bstride, phi_hstride)


def fb_attn_bwd(dt, B, H, N, d, Q, K, V, R, phi_q, phi_k, phi_bstride, phi_hstride, scale, causal, O, LSE, dO,
                dQ, dK, dV, dphi_q, dphi_k, workspace, workspace_bytes, stream) -> int:
    return lib().fb_attn_bwd(dt, B, H, N, d, Q, K, V, R, phi_q, phi_k, phi_bstride, phi_hstride, scale, causal, O,
                             LSE, dO, dQ, dK, dV, dphi_q, dphi_k, workspace, workspace_bytes, stream)


def attn_bwd(q, k, v, phi_q, phi_k, o, lse, do, scale=None, causal=False, workspace=None, factor_grads=True):
    """Gradients of attn's O for an upstream gradient do (fb_attn_bwd).

    q, k, v, o, do: bf16 CUDA [B, H, N, d] contiguous; lse: fp32 [B, H, N]
    from the forward; phi_q, phi_k as for attn (or None). Returns
    (dq, dk, dv, dphi_q, dphi_k): bf16 [B, H, N, d] and fp32 gradients shaped
    like phi_q, phi_k (None without factors, or with factor_grads=False for
    fixed factors, whose gradient products are then skipped)."""
    import torch
    for t in (q, k, v, o, do):
        assert t.is_cuda and t.dtype == torch.bfloat16 and t.is_contiguous()
    B, H, N, d = q.shape
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    R, bs, hs, pq, pk, gq, gk = 0, 0, 0, 0, 0, 0, 0
    dpq = dpk = None
    if phi_q is not None:
        assert phi_q.dtype == torch.float32 and phi_k.dtype == torch.float32
        assert phi_q.shape == phi_k.shape and phi_q.stride() == phi_k.stride() and phi_q.is_contiguous()
        R = phi_q.shape[-1]
        bs, hs = _factor_strides(phi_q, B, H, N, R)
        pq, pk = phi_q.data_ptr(), phi_k.data_ptr()
        if factor_grads:
            dpq, dpk = torch.empty_like(phi_q), torch.empty_like(phi_k)
            gq, gk = dpq.data_ptr(), dpk.data_ptr()
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    nb = fb_attn_bwd_workspace_bytes(B, H, N, R, bs, hs)
    if workspace is None:
        workspace = torch.empty(max(nb, 1), device=q.device, dtype=torch.uint8)
    _check(fb_attn_bwd(FB_BF16, B, H, N, d, q.data_ptr(), k.data_ptr(), v.data_ptr(), R, pq, pk, bs, hs, scale,
                       int(bool(causal)), o.data_ptr(), lse.data_ptr(), do.data_ptr(), dq.data_ptr(), dk.data_ptr(),
                       dv.data_ptr(), gq, gk, workspace.data_ptr(), nb, _stream(q.device)), "fb_attn_bwd")
    return dq, dk, dv, dpq, dpk


def fb_attn_neural_bwd_workspace_bytes(B, H, N, F, R) -> int:
    return lib().fb_attn_neural_bwd_workspace_bytes(B, H, N, F, R)


def fb_attn_neural_bwd(dt, B, H, N, d, Q, K, V, F, R, X_q, X_k, W_q, W_k, scale, causal, O, LSE, dO, dQ, dK, dV,
                       dX_q, dX_k, dW_q, dW_k, workspace, workspace_bytes, stream) -> int:
    return lib().fb_attn_neural_bwd(dt, B, H, N, d, Q, K, V, F, R, X_q, X_k, W_q, W_k, scale, causal, O, LSE, dO, dQ,
                                    dK, dV, dX_q, dX_k, dW_q, dW_k, workspace, workspace_bytes, stream)


def attn_neural_bwd(q, k, v, x_q, x_k, w_q, w_k, o, lse, do, scale=None, causal=False, feature_grads=True):
    """Gradients of attn_neural's O for an upstream gradient do
    (fb_attn_neural_bwd). Returns (dq, dk, dv, dx_q, dx_k, dw_q, dw_k); dx
    are None with feature_grads=False."""
    import torch
    for t in (q, k, v, o, do):
        assert t.is_cuda and t.dtype == torch.bfloat16 and t.is_contiguous()
    for t in (x_q, x_k, w_q, w_k):
        assert t.is_cuda and t.dtype == torch.float32 and t.is_contiguous()
    B, H, N, d = q.shape
    F, R = w_q.shape[1], w_q.shape[2]
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    dwq, dwk = torch.empty_like(w_q), torch.empty_like(w_k)
    dxq = torch.empty_like(x_q) if feature_grads else None
    dxk = torch.empty_like(x_k) if feature_grads else None
    nb = fb_attn_neural_bwd_workspace_bytes(B, H, N, F, R)
    ws = torch.empty(max(nb, 1), device=q.device, dtype=torch.uint8)
    _check(fb_attn_neural_bwd(FB_BF16, B, H, N, d, q.data_ptr(), k.data_ptr(), v.data_ptr(), F, R, x_q.data_ptr(),
                              x_k.data_ptr(), w_q.data_ptr(), w_k.data_ptr(), scale, int(bool(causal)), o.data_ptr(),
                              lse.data_ptr(), do.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(),
                              dxq.data_ptr() if dxq is not None else 0, dxk.data_ptr() if dxk is not None else 0,
                              dwq.data_ptr(), dwk.data_ptr(), ws.data_ptr(), nb, _stream(q.device)),
           "fb_attn_neural_bwd")
    return dq, dk, dv, dxq, dxk, dwq, dwk


def fb_attn_fwd_noalloc(dt, B, H, N, d, Q, K, V, R, phi_q, phi_k, phi_bstride, phi_hstride, scale, causal, O, LSE,
                        stream) -> int:
    """fb_attn_fwd without a caller workspace, for callers that cannot allocate
    device memory: the prepared factors go to the library's fixed 8 MiB device
    array (larger needs return FB_ERR_WORKSPACE). Calls that overlap on the GPU
    share that array and must be serialised by the caller."""
    return lib().fb_attn_fwd_noalloc(dt, B, H, N, d, Q, K, V, R, phi_q, phi_k, phi_bstride, phi_hstride, scale,
                                     causal, O, LSE, stream)


def fb_attn_dense_bias_fwd(dt, B, H, N, d, Q, K, V, Bias, bias_bstride, bias_hstride, scale, causal, O, LSE,
                           stream) -> int:
    return lib().fb_attn_dense_bias_fwd(dt, B, H, N, d, Q, K, V, Bias, bias_bstride, bias_hstride, scale, causal, O,
                                        LSE, stream)


def fb_factors_sandwich(N, C, phi_q, phi_k, stream) -> int:
    return lib().fb_factors_sandwich(N, C, phi_q, phi_k, stream)


def fb_factors_alibi(H, N, phi_q, phi_k, stream) -> int:
    return lib().fb_factors_alibi(H, N, phi_q, phi_k, stream)


def fb_svd_factors_host(bias_host, N, R, oversample, power_iters, seed, phi_q_host, phi_k_host, rel_fro_err,
                        energy) -> int:
    return lib().fb_svd_factors_host(bias_host, N, R, oversample, power_iters, seed, phi_q_host, phi_k_host,
                                     rel_fro_err, energy)


def fb_check_device_error(stream) -> int:
    return lib().fb_check_device_error(stream)


def fb_selftest_wait_timeout(limit_ms, stream) -> int:
    return lib().fb_selftest_wait_timeout(limit_ms, stream)


# ------------------------------------------------- torch-tensor marshalling

def _check(status: int, where: str):
    if status != FB_OK:
        raise FlashBiasError(status, where)


def _stream(device=None) -> int:
    import torch
    return torch.cuda.current_stream(device).cuda_stream


def _dtype_code(t) -> int:
    import torch
    if t.dtype == torch.bfloat16:
        return FB_BF16
    if t.dtype == torch.float32:
        return FB_F32
    raise TypeError(f"unsupported dtype {t.dtype}; use bfloat16 or float32")


def _factor_strides(phi, B, H, N, R):
    """Element strides (b, h) of a factor tensor broadcastable to [B, H, N, R]."""
    if phi.dim() == 2:  # [N, R]: shared by every head and batch
        return 0, 0
    if phi.dim() == 3:  # [H, N, R]: shared by the batch
        return 0, (phi.stride(0) if phi.shape[0] == H and H > 1 else 0)
    bs = phi.stride(0) if phi.shape[0] == B and B > 1 else 0
    hs = phi.stride(1) if phi.shape[1] == H and H > 1 else 0
    return bs, hs


def attn(q, k, v, phi_q=None, phi_k=None, scale=None, causal=False, out=None, lse=None, workspace=None):
    """O, LSE = softmax(scale q k^T + phi_q phi_k^T [+ causal]) v through fb_attn_fwd.

    q, k, v: CUDA tensors [B, H, N, d] (bf16 or fp32, contiguous).
    phi_q, phi_k: fp32 factors [N, R], [H, N, R] or [B, H, N, R] (last two dims
    contiguous), or None for plain attention. Returns (O, LSE).
    """
    import torch
    assert q.is_cuda and q.is_contiguous() and k.is_contiguous() and v.is_contiguous()
    B, H, N, d = q.shape
    dt = _dtype_code(q)
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    R, bs, hs, pq, pk = 0, 0, 0, 0, 0
    if phi_q is not None:
        assert phi_q.dtype == torch.float32 and phi_k.dtype == torch.float32
        assert phi_q.shape == phi_k.shape and phi_q.stride() == phi_k.stride()
        assert phi_q.stride(-1) == 1 and phi_q.stride(-2) == phi_q.shape[-1]
        R = phi_q.shape[-1]
        bs, hs = _factor_strides(phi_q, B, H, N, R)
        pq, pk = phi_q.data_ptr(), phi_k.data_ptr()
    o = torch.empty_like(q) if out is None else out
    l = torch.empty((B, H, N), device=q.device, dtype=torch.float32) if lse is None else lse
    ws_bytes = fb_attn_workspace_bytes(B, H, N, R, bs, hs) if dt == FB_BF16 else 0
    if ws_bytes and workspace is None:
        workspace = torch.empty(ws_bytes, device=q.device, dtype=torch.uint8)
    ws_ptr = workspace.data_ptr() if (workspace is not None and ws_bytes) else 0
    _check(fb_attn_fwd(dt, B, H, N, d, q.data_ptr(), k.data_ptr(), v.data_ptr(), R, pq, pk, bs, hs, scale,
                       int(bool(causal)), o.data_ptr(), l.data_ptr(), ws_ptr, ws_bytes, _stream(q.device)),
           "fb_attn_fwd")
    return o, l


def attn_mul_bias(q, k, v, phi_q, phi_k, scale=None, causal=False, out=None, lse=None, workspace=None):
    """O, LSE = softmax(scale (q k^T) o (phi_q phi_k^T) [+ causal]) v through
    fb_attn_mul_bias_fwd (multiplicative low-rank bias; bf16 q, k, v).

    phi_q, phi_k: fp32 [N, R], [H, N, R] or [B, H, N, R] (last two dims
    contiguous). Returns (O, LSE)."""
    import torch
    assert q.is_cuda and q.dtype == torch.bfloat16 and q.is_contiguous() and k.is_contiguous() \
        and v.is_contiguous()
    assert phi_q.dtype == torch.float32 and phi_k.dtype == torch.float32
    assert phi_q.shape == phi_k.shape and phi_q.stride() == phi_k.stride()
    assert phi_q.stride(-1) == 1 and phi_q.stride(-2) == phi_q.shape[-1]
    B, H, N, d = q.shape
    R = phi_q.shape[-1]
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    bs, hs = _factor_strides(phi_q, B, H, N, R)
    o = torch.empty_like(q) if out is None else out
    l = torch.empty((B, H, N), device=q.device, dtype=torch.float32) if lse is None else lse
    ws_bytes = fb_attn_mul_bias_workspace_bytes(B, H, N, d, R)
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 1), device=q.device, dtype=torch.uint8)
    _check(fb_attn_mul_bias_fwd(FB_BF16, B, H, N, d, q.data_ptr(), k.data_ptr(), v.data_ptr(), R, phi_q.data_ptr(),
                                phi_k.data_ptr(), bs, hs, scale, int(bool(causal)), o.data_ptr(), l.data_ptr(),
                                workspace.data_ptr(), ws_bytes, _stream(q.device)), "fb_attn_mul_bias_fwd")
    return o, l


class PreparedBias:
    """Factors prepared once (fb_attn_prepare_factors) for many bf16 calls.

    phi_q, phi_k as for attn(); B, H, N the shape of the q tensors it will be
    used with; scale the softmax scale (it is folded into the prepared
    factors). Call it as attn(q, k, v, causal=...) -> (O, LSE)."""

    def __init__(self, phi_q, phi_k, B: int, H: int, N: int, d: int, scale=None):
        import torch
        assert phi_q.dtype == torch.float32 and phi_k.dtype == torch.float32
        assert phi_q.shape == phi_k.shape and phi_q.stride() == phi_k.stride()
        assert phi_q.stride(-1) == 1 and phi_q.stride(-2) == phi_q.shape[-1]
        self.B, self.H, self.N, self.d = B, H, N, d
        self.R = phi_q.shape[-1]
        self.scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
        self.bs, self.hs = _factor_strides(phi_q, B, H, N, self.R)
        self.ws_bytes = fb_attn_workspace_bytes(B, H, N, self.R, self.bs, self.hs)
        self.workspace = torch.empty(max(self.ws_bytes, 1), device=phi_q.device, dtype=torch.uint8)
        _check(fb_attn_prepare_factors(B, H, N, self.R, phi_q.data_ptr(), phi_k.data_ptr(), self.bs, self.hs,
                                       self.scale, self.workspace.data_ptr(), self.ws_bytes,
                                       _stream(phi_q.device)), "fb_attn_prepare_factors")

    def attn(self, q, k, v, causal=False, out=None, lse=None):
        import torch
        assert q.is_cuda and q.dtype == torch.bfloat16 and q.is_contiguous() and k.is_contiguous() \
            and v.is_contiguous()
        B, H, N, d = q.shape
        assert (B, H, N, d) == (self.B, self.H, self.N, self.d)
        o = torch.empty_like(q) if out is None else out
        l = torch.empty((B, H, N), device=q.device, dtype=torch.float32) if lse is None else lse
        _check(fb_attn_fwd_prepared(FB_BF16, B, H, N, d, q.data_ptr(), k.data_ptr(), v.data_ptr(), self.R, self.bs,
                                    self.hs, self.scale, int(bool(causal)), o.data_ptr(), l.data_ptr(),
                                    self.workspace.data_ptr(), self.ws_bytes, _stream(q.device)),
               "fb_attn_fwd_prepared")
        return o, l


def attn_dense_bias(q, k, v, bias, scale=None, causal=False, out=None, lse=None):
    """The dense-bias comparison path through fb_attn_dense_bias_fwd.

    bias: [N, N], [H, N, N] or [B, H, N, N] tensor of q's dtype (last two dims
    contiguous). Returns (O, LSE).
    """
    import torch
    B, H, N, d = q.shape
    dt = _dtype_code(q)
    assert bias.dtype == q.dtype and bias.stride(-1) == 1 and bias.stride(-2) == N
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    if bias.dim() == 2:
        bs, hs = 0, 0
    elif bias.dim() == 3:
        bs, hs = 0, (bias.stride(0) if H > 1 else 0)
    else:
        bs = bias.stride(0) if (bias.shape[0] == B and B > 1) else 0
        hs = bias.stride(1) if (bias.shape[1] == H and H > 1) else 0
    o = torch.empty_like(q) if out is None else out
    l = torch.empty((B, H, N), device=q.device, dtype=torch.float32) if lse is None else lse
    _check(fb_attn_dense_bias_fwd(dt, B, H, N, d, q.data_ptr(), k.data_ptr(), v.data_ptr(), bias.data_ptr(), bs, hs,
                                  scale, int(bool(causal)), o.data_ptr(), l.data_ptr(), _stream(q.device)),
           "fb_attn_dense_bias_fwd")
    return o, l


def factors_sandwich(N: int, C: int, device="cuda"):
    """Exact Sandwich factors phi [N, C] fp32 (phi_q = phi_k); one kernel."""
    import torch
    phi = torch.empty((N, C), device=device, dtype=torch.float32)
    _check(fb_factors_sandwich(N, C, phi.data_ptr(), phi.data_ptr(), _stream(phi.device)), "fb_factors_sandwich")
    return phi


def factors_alibi(H: int, N: int, device="cuda"):
    """Exact rank-2 ALiBi factors (phi_q, phi_k), each [H, N, 2] fp32; one kernel."""
    import torch
    pq = torch.empty((H, N, 2), device=device, dtype=torch.float32)
    pk = torch.empty((H, N, 2), device=device, dtype=torch.float32)
    _check(fb_factors_alibi(H, N, pq.data_ptr(), pk.data_ptr(), _stream(pq.device)), "fb_factors_alibi")
    return pq, pk


def svd_factors(bias, R: int, oversample: int = 16, power_iters: int = 2, seed: int = 0):
    """Host truncated SVD of one head's bias (numpy float64 [N, N]).

    Returns (phi_q [N, R] fp32, phi_k [N, R] fp32, rel_fro_err, energy) as numpy.
    """
    import numpy as np
    b = np.ascontiguousarray(bias, dtype=np.float64)
    N = b.shape[0]
    assert b.shape == (N, N)
    pq = np.empty((N, R), dtype=np.float32)
    pk = np.empty((N, R), dtype=np.float32)
    err, en = ctypes.c_double(), ctypes.c_double()
    _check(fb_svd_factors_host(b.ctypes.data, N, R, oversample, power_iters, seed, pq.ctypes.data, pk.ctypes.data,
                               ctypes.addressof(err), ctypes.addressof(en)), "fb_svd_factors_host")
    return pq, pk, err.value, en.value


def attn_flops(B: int, H: int, N: int, d: int, R: int, causal: bool) -> float:
    """Counted FLOPs: 4 N^2 d + 2 N^2 R per head, halved when causal."""
    f = float(B) * H * (4.0 * N * N * d + 2.0 * N * N * R)
    return f / 2.0 if causal else f
