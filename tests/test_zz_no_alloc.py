"""fb_attn_fwd_noalloc, the fused forward for callers that cannot allocate
device memory (plugin or operator interfaces that only hand over their input
and output tensors, frameworks that own every device buffer, paths that must
not call cudaMalloc). It keeps the prepared factors in the library's fixed
8 MiB device array instead of a caller workspace.

The check: two calls in a row through the C ABI give the same result as
fb_attn_fwd with a caller workspace, within the bf16 tolerance of the other
tests; and a problem whose prepared factors exceed the array is refused
before launch. This file is collected last so that a run stopping at the
first failure has already run every other test."""
import math

import numpy as np
import pytest

import seeded_inputs as si

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
import attention_rank_additive_b200 as fb  # noqa: E402

TOL_MAX, TOL_MEAN = 2e-2, 2e-3  # the bf16 tolerance the parity tests use
LIMIT = 8 << 20


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from attention_rank_additive_b200 import build
    build.build()
    fb.lib()


def _inputs(B, H, N, d, R, layout, seed):
    q, k, v = si.qkv(B, H, N, d, seed, "bf16")
    dev = lambda x, dt: torch.from_numpy(x).cuda().to(dt)  # noqa: E731
    Q, K, V = (dev(x, torch.bfloat16) for x in (q, k, v))
    pq = pk = None
    bs = hs = 0
    if R > 0:
        shape = (N, R) if layout == "nr" else (B, H, N, R)
        a, b = si.random_factors(shape, math.sqrt(1.0 / R), seed + 1)
        pq, pk = dev(a, torch.float32), dev(b, torch.float32)
        if layout != "nr":
            bs, hs = H * N * R, N * R
    return Q, K, V, pq, pk, bs, hs


@pytest.mark.parametrize("B,H,N,d,R,layout,causal", [
    (2, 3, 300, 64, 64, "bhnr", True),   # fp16 factor MMA path
    (1, 4, 513, 128, 2, "bhnr", False),  # rank <= 4 CUDA-core factor path
    (4, 8, 1024, 32, 32, "nr", True),    # broadcast factors
])
def test_noalloc_matches_workspace_entry_twice(B, H, N, d, R, layout, causal):
    Q, K, V, pq, pk, bs, hs = _inputs(B, H, N, d, R, layout, seed=900 + N)
    scale = 1.0 / math.sqrt(d)
    stream = torch.cuda.current_stream().cuda_stream
    ptr = lambda t: 0 if t is None else t.data_ptr()  # noqa: E731
    # reference: the workspace entry point with a caller-allocated workspace
    ws_bytes = fb.fb_attn_workspace_bytes(B, H, N, R, bs, hs)
    assert 0 < ws_bytes <= LIMIT
    ws = torch.empty(ws_bytes, device="cuda", dtype=torch.uint8)
    O_ref = torch.empty_like(Q)
    L_ref = torch.empty((B, H, N), device="cuda", dtype=torch.float32)
    assert fb.fb_attn_fwd(fb.FB_BF16, B, H, N, d, Q.data_ptr(), K.data_ptr(), V.data_ptr(), R, ptr(pq), ptr(pk), bs,
                          hs, scale, int(causal), O_ref.data_ptr(), L_ref.data_ptr(), ws.data_ptr(), ws_bytes,
                          stream) == fb.FB_OK
    for call in range(2):
        O = torch.full_like(Q, float("nan"))
        L = torch.full((B, H, N), float("nan"), device="cuda", dtype=torch.float32)
        st = fb.fb_attn_fwd_noalloc(fb.FB_BF16, B, H, N, d, Q.data_ptr(), K.data_ptr(), V.data_ptr(), R, ptr(pq),
                                    ptr(pk), bs, hs, scale, int(causal), O.data_ptr(), L.data_ptr(), stream)
        assert st == fb.FB_OK, fb.fb_status_str(st)
        torch.cuda.synchronize()
        assert fb.fb_check_device_error(stream) == fb.FB_OK
        d_o = (O.float() - O_ref.float()).abs()
        assert torch.isfinite(O.float()).all(), f"call {call}: non-finite output"
        assert d_o.max().item() <= TOL_MAX and d_o.mean().item() <= TOL_MEAN, f"call {call}"
        assert (L - L_ref).abs().max().item() <= TOL_MAX, f"call {call}"


def test_noalloc_refuses_problems_beyond_its_scratch():
    B, H, N, d, R = 4, 16, 8192, 64, 64  # per-head fp16 factors: 2 x 64 x 8192 x 64 x 2 B = 128 MiB
    assert fb.fb_attn_workspace_bytes(B, H, N, R, H * N * R, N * R) > LIMIT
    x = torch.empty((1,), device="cuda", dtype=torch.bfloat16)
    p = torch.empty((1,), device="cuda", dtype=torch.float32)
    st = fb.fb_attn_fwd_noalloc(fb.FB_BF16, B, H, N, d, x.data_ptr(), x.data_ptr(), x.data_ptr(), R, p.data_ptr(),
                                p.data_ptr(), H * N * R, N * R, 0.125, 1, x.data_ptr(), p.data_ptr(),
                                torch.cuda.current_stream().cuda_stream)
    assert st == fb.FB_ERR_WORKSPACE
