"""fb_attn_fwd_noalloc, the fused forward for callers that cannot allocate
device memory (plugin or operator interfaces that only hand over their input
and output tensors, frameworks that own every device buffer, paths that must
not call cudaMalloc). It keeps the prepared factors in the library's fixed
8 MiB device array instead of a caller workspace.

The check: two calls in a row through the C ABI give the same result as
fb_attn_fwd with a caller workspace. Both run the same preparation and fused
kernels on the same inputs, so the results must be bit-identical (a
tolerance could hide stale scratch); before each checked call a no-alloc
call of another shape and factor path leaves its own contents in the shared
array. A problem whose prepared factors exceed the array is refused before
launch, and bad arguments get fb_attn_fwd's status. This file is collected
last so that a run stopping at the first failure has already run every other
test."""
import math

import numpy as np
import pytest

import seeded_inputs as si

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
import attention_rank_additive_b200 as fb  # noqa: E402

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


def _ptr(t):
    return 0 if t is None else t.data_ptr()


def _noalloc(B, H, N, d, R, causal, Q, K, V, pq, pk, bs, hs, O, L, stream):
    return fb.fb_attn_fwd_noalloc(fb.FB_BF16, B, H, N, d, Q.data_ptr(), K.data_ptr(), V.data_ptr(), R, _ptr(pq),
                                  _ptr(pk), bs, hs, 1.0 / math.sqrt(d), int(causal), O.data_ptr(), L.data_ptr(),
                                  stream)


def _other_call(shape, stream):
    """One no-alloc call of a different shape and factor path, which leaves
    its own prepared factors in the shared array."""
    B, H, N, d, R, layout, causal = shape
    Q, K, V, pq, pk, bs, hs = _inputs(B, H, N, d, R, layout, seed=77 + R)
    O = torch.empty_like(Q)
    L = torch.empty((B, H, N), device="cuda", dtype=torch.float32)
    assert _noalloc(B, H, N, d, R, causal, Q, K, V, pq, pk, bs, hs, O, L, stream) == fb.FB_OK


CASES = [
    (2, 3, 300, 64, 64, "bhnr", True),   # fp16 factor MMA path, per-head factors
    (1, 4, 513, 128, 2, "bhnr", False),  # rank <= 4 split-tf32 factor MMA path
    (4, 8, 1024, 32, 32, "nr", True),    # broadcast factors
]


@pytest.mark.parametrize("case", range(len(CASES)))
def test_noalloc_matches_workspace_entry_twice(case):
    B, H, N, d, R, layout, causal = CASES[case]
    other = CASES[(case + 1) % len(CASES)]
    Q, K, V, pq, pk, bs, hs = _inputs(B, H, N, d, R, layout, seed=900 + N)
    scale = 1.0 / math.sqrt(d)
    stream = torch.cuda.current_stream().cuda_stream
    ptr = _ptr
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
        _other_call(other, stream)  # the shared array now holds another call's factors
        O = torch.full_like(Q, float("nan"))
        L = torch.full((B, H, N), float("nan"), device="cuda", dtype=torch.float32)
        st = _noalloc(B, H, N, d, R, causal, Q, K, V, pq, pk, bs, hs, O, L, stream)
        assert st == fb.FB_OK, fb.fb_status_str(st)
        torch.cuda.synchronize()
        assert fb.fb_check_device_error(stream) == fb.FB_OK
        assert torch.equal(O, O_ref), f"call {call}: O differs from fb_attn_fwd"
        assert torch.equal(L, L_ref), f"call {call}: LSE differs from fb_attn_fwd"


def test_noalloc_refuses_problems_beyond_its_scratch():
    B, H, N, d, R = 4, 16, 8192, 64, 64  # per-head fp16 factors: 2 x 64 x 8192 x 64 x 2 B = 128 MiB
    assert fb.fb_attn_workspace_bytes(B, H, N, R, H * N * R, N * R) > LIMIT
    x = torch.empty((1,), device="cuda", dtype=torch.bfloat16)
    p = torch.empty((1,), device="cuda", dtype=torch.float32)
    st = fb.fb_attn_fwd_noalloc(fb.FB_BF16, B, H, N, d, x.data_ptr(), x.data_ptr(), x.data_ptr(), R, p.data_ptr(),
                                p.data_ptr(), H * N * R, N * R, 0.125, 1, x.data_ptr(), p.data_ptr(),
                                torch.cuda.current_stream().cuda_stream)
    assert st == fb.FB_ERR_WORKSPACE


def test_noalloc_reports_the_argument_errors_of_fb_attn_fwd():
    """A bad argument gets the status fb_attn_fwd gives it, also when the
    problem would not fit the fixed array (argument checks come first)."""
    x = torch.empty((1,), device="cuda", dtype=torch.bfloat16)
    p = torch.empty((1,), device="cuda", dtype=torch.float32)
    big = dict(B=4, H=16, N=8192, d=64, R=64)  # prepared factors beyond the array
    stream = torch.cuda.current_stream().cuda_stream

    def both(B, H, N, d, R, Q, scale):
        bs, hs = H * N * R, N * R
        a = fb.fb_attn_fwd_noalloc(fb.FB_BF16, B, H, N, d, Q, x.data_ptr(), x.data_ptr(), R, p.data_ptr(),
                                   p.data_ptr(), bs, hs, scale, 1, x.data_ptr(), p.data_ptr(), stream)
        b = fb.fb_attn_fwd(fb.FB_BF16, B, H, N, d, Q, x.data_ptr(), x.data_ptr(), R, p.data_ptr(), p.data_ptr(), bs,
                           hs, scale, 1, x.data_ptr(), p.data_ptr(), 0, 0, stream)
        return a, b

    assert both(Q=0, scale=0.125, **big) == (fb.FB_ERR_INVALID_ARG,) * 2
    assert both(Q=x.data_ptr(), scale=0.0, **big) == (fb.FB_ERR_INVALID_ARG,) * 2
    assert both(Q=x.data_ptr(), scale=0.125, B=0, H=2, N=64, d=64, R=8) == (fb.FB_ERR_INVALID_ARG,) * 2
    assert both(Q=x.data_ptr(), scale=0.125, B=1, H=2, N=64, d=12, R=8) == (fb.FB_ERR_UNSUPPORTED,) * 2
