"""GPU parity of every kernel against the fp64 oracle on small seeded inputs
that still span several 128-row tiles and a ragged tail, plus the edge cases
(one row, d not a multiple of 16, every factor path, broadcast layouts) and
the failure-path checks (fp16 range flag, bounded-wait timeout)."""
import math

import numpy as np
import pytest

import oracle
from oracle import HeadBias
import seeded_inputs as si
from gpu_util import compare, dev, grad_close, host

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
import attention_rank_additive_b200 as fb  # noqa: E402


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from attention_rank_additive_b200 import build
    build.build()
    fb.lib()
    yield
    torch.cuda.synchronize()


def _no_device_error():
    assert fb.fb_check_device_error(torch.cuda.current_stream().cuda_stream) == fb.FB_OK


# ---------------------------------------------------------------- factors

@pytest.mark.parametrize("N,C", [(2048, 64), (5, 8), (300, 2), (1, 128)])
def test_sandwich_factors_match_oracle(N, C):
    phi = fb.factors_sandwich(N, C)
    torch.cuda.synchronize()
    ref = oracle.sandwich_factors(N, C)
    np.testing.assert_allclose(host(phi), ref, rtol=0, atol=1e-6)


@pytest.mark.parametrize("H,N", [(16, 8192), (3, 100)])
def test_alibi_factors_match_oracle(H, N):
    pq, pk = fb.factors_alibi(H, N)
    torch.cuda.synchronize()
    pq, pk = host(pq), host(pk)
    for h in range(H):
        rq, rk = oracle.alibi_factors(N, oracle.alibi_slope(h, H))
        np.testing.assert_allclose(pq[h], rq, rtol=1e-7, atol=0)
        np.testing.assert_allclose(pk[h], rk, rtol=1e-7, atol=0)


# ------------------------------------------------------- fused bf16 sweeps

def _run_fused(B, H, N, d, R, causal, seed, std=None, layout="bhnr", dtype="bf16"):
    q, k, v = si.qkv(B, H, N, d, seed, dtype)
    scale = 1.0 / math.sqrt(d)
    pq = pk = None
    if R > 0:
        std = std if std is not None else math.sqrt(1.0 / R)
        shape = {"nr": (N, R), "hnr": (H, N, R), "bhnr": (B, H, N, R)}[layout]
        pq, pk = si.random_factors(shape, std, seed + 7)
    o, l = fb.attn(dev(q, dtype), dev(k, dtype), dev(v, dtype),
                   None if pq is None else dev(pq, "f32"), None if pk is None else dev(pk, "f32"),
                   scale=scale, causal=causal)
    torch.cuda.synchronize()
    _no_device_error()

    def bias_of(b, h):
        if R == 0:
            return HeadBias.none()
        if layout == "nr":
            return HeadBias.lowrank(pq, pk)
        if layout == "hnr":
            return HeadBias.lowrank(pq[h], pk[h])
        return HeadBias.lowrank(pq[b, h], pk[b, h])

    heads = [(0, 0), (B - 1, H - 1)] if B * H > 2 else [(b, h) for b in range(B) for h in range(H)]
    ro, rl = oracle.attention(q, k, v, bias_of, scale, causal, heads=heads)
    og, lg = host(o), host(l)
    for (b, h) in heads:
        compare(og[b, h], lg[b, h], ro[(b, h)], rl[(b, h)], dtype, f"B{B} H{H} N{N} d{d} R{R} c{causal} ({b},{h})")


SWEEP = [
    # B, H, N, d, R, causal
    (1, 1, 1, 64, 0, False),
    (1, 1, 1, 64, 8, True),
    (1, 2, 17, 16, 8, False),
    (1, 2, 128, 64, 64, True),
    (2, 1, 129, 64, 64, True),
    (1, 2, 255, 24, 32, False),
    (1, 1, 256, 128, 2, True),
    (1, 2, 300, 128, 2, False),
    (1, 1, 300, 8, 3, True),
    (1, 1, 384, 32, 1, True),
    (1, 2, 513, 40, 4, False),
    (1, 1, 513, 72, 5, True),
    (1, 1, 400, 96, 100, False),
    (1, 1, 260, 120, 128, True),
    (1, 1, 640, 128, 16, True),
    (1, 2, 700, 64, 0, True),
    (2, 2, 1000, 16, 8, False),
]


@pytest.mark.parametrize("qt", ["1", "2"])
@pytest.mark.parametrize("B,H,N,d,R,causal", SWEEP)
def test_fused_bf16_matches_oracle(monkeypatch, qt, B, H, N, d, R, causal):
    monkeypatch.setenv("FLASHBIAS_QUERY_TILES", qt)
    _run_fused(B, H, N, d, R, causal, seed=100 + N + d + R)


@pytest.mark.parametrize("layout", ["nr", "hnr", "bhnr"])
@pytest.mark.parametrize("R", [2, 16])
def test_fused_factor_layouts(layout, R):
    _run_fused(2, 3, 200, 64, R, True, seed=7, layout=layout)


def test_fused_default_plan_many_heads():
    # enough (batch, head) pairs for the two-tile plan on its own
    _run_fused(4, 40, 512, 64, 32, True, seed=11)


@pytest.mark.parametrize("qt", ["1", "2"])
def test_fused_persistent_many_items(monkeypatch, qt):
    # more work items than resident CTAs, ragged last tile: every CTA walks
    # several items, so barrier phases carry across items
    monkeypatch.setenv("FLASHBIAS_QUERY_TILES", qt)
    _run_fused(3, 50, 300, 64, 16, True, seed=13)


@pytest.mark.parametrize("R,layout", [(2, "hnr"), (3, "bhnr"), (32, "nr"), (64, "bhnr")])
def test_prepared_factors_equal_fused_and_reuse(R, layout):
    """fb_attn_prepare_factors once + fb_attn_fwd_prepared per call gives
    bit-identical results to fb_attn_fwd, for several inputs, and does not
    read the fp32 factors after the preparation."""
    B, H, N, d = 2, 3, 300, 64
    shape = {"nr": (N, R), "hnr": (H, N, R), "bhnr": (B, H, N, R)}[layout]
    pq, pk = si.random_factors(shape, math.sqrt(1.0 / R), 31 + R)
    pq_d, pk_d = dev(pq, "f32"), dev(pk, "f32")
    prep = fb.PreparedBias(pq_d, pk_d, B, H, N, d)
    ref = []
    for seed in (3, 4):
        q, k, v = (dev(x, "bf16") for x in si.qkv(B, H, N, d, seed, "bf16"))
        o1, l1 = fb.attn(q, k, v, pq_d, pk_d, causal=True)
        o2, l2 = prep.attn(q, k, v, causal=True)
        torch.cuda.synchronize()
        assert torch.equal(o1, o2) and torch.equal(l1, l2)
        ref.append((q, k, v, o1, l1))
    pq_d.zero_()
    pk_d.zero_()
    for q, k, v, o1, l1 in ref:
        o3, l3 = prep.attn(q, k, v, causal=True)
        torch.cuda.synchronize()
        assert torch.equal(o1, o3) and torch.equal(l1, l3)
    _no_device_error()


def test_fused_f32_matches_oracle_tight():
    for (B, H, N, d, R, causal) in [(1, 2, 256, 64, 8, False), (1, 1, 1, 4, 0, True), (2, 1, 300, 128, 5, True),
                                    (1, 3, 33, 12, 128, False)]:
        _run_fused(B, H, N, d, R, causal, seed=5, dtype="f32")


# ------------------------------------------------------------ dense path

def _run_dense(B, H, N, d, causal, layout, dtype, seed):
    q, k, v = si.qkv(B, H, N, d, seed, dtype)
    scale = 1.0 / math.sqrt(d)
    rng = si.generator(seed + 3)
    shape = {"nn": (N, N), "hnn": (H, N, N), "bhnn": (B, H, N, N)}[layout]
    bias = (rng.standard_normal(size=shape) * 2.0).astype(np.float32)
    if dtype == "bf16":
        bias = si.round_to_bf16(bias)
    o, l = fb.attn_dense_bias(dev(q, dtype), dev(k, dtype), dev(v, dtype), dev(bias, dtype), scale=scale,
                              causal=causal)
    torch.cuda.synchronize()
    _no_device_error()

    def bias_of(b, h):
        return HeadBias.dense({"nn": bias, "hnn": bias[h] if layout == "hnn" else None,
                               "bhnn": bias[b, h] if layout == "bhnn" else None}[layout])

    heads = [(0, 0), (B - 1, H - 1)] if B * H > 2 else [(b, h) for b in range(B) for h in range(H)]
    ro, rl = oracle.attention(q, k, v, bias_of, scale, causal, heads=heads)
    og, lg = host(o), host(l)
    for (b, h) in heads:
        compare(og[b, h], lg[b, h], ro[(b, h)], rl[(b, h)], dtype, f"dense N{N} d{d} c{causal} {layout} ({b},{h})")


@pytest.mark.parametrize("qt", ["1", "2"])
@pytest.mark.parametrize("B,H,N,d,causal,layout", [
    (1, 1, 8, 64, False, "nn"),
    (1, 2, 136, 16, True, "hnn"),
    (2, 2, 256, 24, False, "bhnn"),
    (1, 1, 264, 128, True, "nn"),
    (1, 2, 520, 64, True, "bhnn"),
    (1, 1, 384, 40, False, "hnn"),
])
def test_dense_bf16_matches_oracle(monkeypatch, qt, B, H, N, d, causal, layout):
    monkeypatch.setenv("FLASHBIAS_QUERY_TILES", qt)
    _run_dense(B, H, N, d, causal, layout, "bf16", seed=200 + N)


@pytest.mark.parametrize("B,H,N,d,causal,layout", [(1, 2, 256, 64, False, "hnn"), (2, 1, 77, 8, True, "bhnn")])
def test_dense_f32_matches_oracle(B, H, N, d, causal, layout):
    _run_dense(B, H, N, d, causal, layout, "f32", seed=300 + N)


# ------------------------------------------------------ failure paths

def test_fp16_range_flag():
    N, d, R = 128, 64, 8
    q, k, v = si.qkv(1, 1, N, d, 9, "bf16")
    pq = np.full((N, R), 1.0e6, dtype=np.float32)  # / scale overflows fp16
    fb.attn(dev(q, "bf16"), dev(k, "bf16"), dev(v, "bf16"), dev(pq, "f32"), dev(pq, "f32"), causal=False)
    assert fb.fb_check_device_error(torch.cuda.current_stream().cuda_stream) == fb.FB_ERR_RANGE
    _no_device_error()  # the flag was cleared by the read


def test_bounded_wait_times_out_and_context_survives():
    s = torch.cuda.current_stream().cuda_stream
    assert fb.fb_selftest_wait_timeout(20, s) == fb.FB_OK
    assert fb.fb_check_device_error(s) == fb.FB_ERR_TIMEOUT
    _no_device_error()
    _run_fused(1, 1, 200, 64, 8, True, seed=3)  # the context is still usable


def test_unsupported_dense_pitch_returns_before_launch():
    x = torch.zeros((1, 1, 130, 64), device="cuda", dtype=torch.bfloat16)
    b = torch.zeros((130, 130), device="cuda", dtype=torch.bfloat16)
    with pytest.raises(fb.FlashBiasError) as e:
        fb.attn_dense_bias(x, x, x, b)
    assert e.value.status == fb.FB_ERR_UNSUPPORTED


# ------------------------------------------------- multiplicative low-rank bias

MUL_CASES = [
    # B, H, N, d, R, causal, factors ("cos": the rebuttal's cos(i - j) example; else N(0, std) per layout)
    (1, 2, 300, 64, 2, True, "cos"),
    (2, 2, 257, 32, 3, False, "bhnr"),
    (1, 2, 200, 128, 2, True, "hnr"),
    (1, 1, 384, 16, 9, True, "nr"),
    (1, 2, 130, 64, 1, False, "nr"),
]


@pytest.mark.parametrize("B,H,N,d,R,causal,kind", MUL_CASES)
def test_mul_bias_matches_oracle(B, H, N, d, R, causal, kind):
    """fb_attn_mul_bias_fwd against the oracle's multiplicative definition
    (rebuttal, reply to Reviewer BRmd, Q1 (2)); ragged tails, every head."""
    q, k, v = si.qkv(B, H, N, d, 400 + N + R, "bf16")
    if kind == "cos":
        i = np.arange(N, dtype=np.float64)
        pq = pk = np.stack([np.cos(i), np.sin(i)], 1).astype(np.float32)
    else:
        shape = {"nr": (N, R), "hnr": (H, N, R), "bhnr": (B, H, N, R)}[kind]
        pq, pk = si.random_factors(shape, 0.6, 500 + R)
    scale = 1.0 / math.sqrt(d)
    o, l = fb.attn_mul_bias(dev(q, "bf16"), dev(k, "bf16"), dev(v, "bf16"), dev(pq, "f32"), dev(pk, "f32"),
                            scale=scale, causal=causal)
    torch.cuda.synchronize()
    _no_device_error()
    og, lg = host(o), host(l)
    for b in range(B):
        for h in range(H):
            fq = pq if pq.ndim == 2 else (pq[h] if pq.ndim == 3 else pq[b, h])
            fk = pk if pk.ndim == 2 else (pk[h] if pk.ndim == 3 else pk[b, h])
            ro, rl = oracle.attention_mul_head(q[b, h], k[b, h], v[b, h], fq, fk, scale, causal)
            compare(og[b, h], lg[b, h], ro, rl, "bf16", f"mul B{B} H{H} N{N} d{d} R{R} {kind} ({b},{h})")


# -------------------------------------------------- truncated SVD on the device

def _known_spectrum(N, sigma, seed):
    rng = np.random.Generator(np.random.PCG64(seed))
    U, _ = np.linalg.qr(rng.standard_normal((N, len(sigma))))
    V, _ = np.linalg.qr(rng.standard_normal((N, len(sigma))))
    return U @ np.diag(sigma) @ V.T


def test_svd_device_known_spectrum():
    """Randomized SVD on the GPU against matrices with known singular values:
    error and energy match the Eckart-Young values, and the rank-R product
    matches the oracle's library SVD."""
    sigma = np.array([40.0, 15.0, 7.0, 3.0, 1.0, 0.3, 0.1, 0.03, 0.01, 0.003])
    Bm = np.stack([_known_spectrum(300, sigma, 61), _known_spectrum(300, sigma * 2.0, 62)])
    Bd = torch.from_numpy(Bm.astype(np.float32)).cuda()
    for R in (1, 4, 8):
        pq, pk, ee = fb.svd_factors_device(Bd, R, oversample=16, power_iters=2, seed=R)
        torch.cuda.synchronize()
        ee = ee.cpu().numpy()
        pq, pk = host(pq), host(pk)
        want_rel = math.sqrt(np.sum(sigma[R:] ** 2) / np.sum(sigma ** 2))
        want_en = np.sum(sigma[:R] ** 2) / np.sum(sigma ** 2)
        for h in range(2):
            assert abs(ee[h, 0] - want_rel) <= 1e-5 + 0.01 * want_rel, (R, h, ee[h, 0], want_rel)
            assert abs(ee[h, 1] - want_en) <= 1e-5, (R, h, ee[h, 1], want_en)
            opq, opk, _, _ = oracle.truncated_svd_factors(Bm[h], R)
            diff = pq[h] @ pk[h].T - opq @ opk.T
            assert np.linalg.norm(diff) <= 1e-4 * np.linalg.norm(Bm[h]), (R, h)
    _no_device_error()


def test_svd_device_rbf_field_near_optimal():
    """The vision workload's RBF field (2 heads, 24 x 24 grid): the GPU's
    rank-8 error is within 2 % of the optimum the oracle's exact SVD gives."""
    grid, R = 24, 8
    om, ph = si.rbf_params(2, 32)
    dense = si.rbf_dense(si.rbf_offset_table(om, ph, grid), grid)
    Bd = torch.from_numpy(dense.astype(np.float32)).cuda()
    pq, pk, ee = fb.svd_factors_device(Bd, R, oversample=16, power_iters=2, seed=5)
    torch.cuda.synchronize()
    ee = ee.cpu().numpy()
    for h in range(2):
        _, _, orel, oen = oracle.truncated_svd_factors(dense[h], R)
        assert ee[h, 0] <= orel * 1.02 + 1e-5, (h, ee[h, 0], orel)
        assert ee[h, 1] >= oen - 1e-3, (h, ee[h, 1], oen)
    _no_device_error()


def test_svd_device_exact_low_rank():
    """A bias of exact rank 3 asked for rank 8: reproduced to fp32 accuracy
    (the dependent columns of the range finder must not break it)."""
    rng = np.random.Generator(np.random.PCG64(71))
    X, Y = rng.standard_normal((200, 3)), rng.standard_normal((200, 3))
    Bm = (X @ Y.T)[None]
    pq, pk, ee = fb.svd_factors_device(torch.from_numpy(Bm.astype(np.float32)).cuda(), 8, oversample=8,
                                       power_iters=1, seed=3)
    torch.cuda.synchronize()
    ee = ee.cpu().numpy()
    assert ee[0, 0] <= 1e-5 and abs(ee[0, 1] - 1.0) <= 1e-5
    pq, pk = host(pq), host(pk)
    assert np.linalg.norm(pq[0] @ pk[0].T - Bm[0]) <= 2e-6 * np.linalg.norm(Bm[0]) + 1e-6
    _no_device_error()


# ------------------------------------------------------- neural decomposition

@pytest.mark.parametrize("B,H,N,d,F,R,causal", [(2, 3, 200, 64, 32, 16, True), (1, 4, 300, 24, 64, 32, False),
                                                (1, 2, 257, 128, 16, 2, True), (1, 1, 129, 32, 8, 128, False)])
def test_neural_bias_matches_oracle(B, H, N, d, F, R, causal):
    """fb_attn_neural_fwd against the oracle: factors x w in fp64, then the
    low-rank biased attention."""
    rng = np.random.Generator(np.random.PCG64(900 + F + R))
    xq, xk = rng.standard_normal((B, N, F)).astype(np.float32), rng.standard_normal((B, N, F)).astype(np.float32)
    wq = (rng.standard_normal((H, F, R)) / math.sqrt(F * R)).astype(np.float32)
    wk = (rng.standard_normal((H, F, R)) / math.sqrt(F)).astype(np.float32)
    q, k, v = si.qkv(B, H, N, d, 950 + N, "bf16")
    scale = 1.0 / math.sqrt(d)
    o, l = fb.attn_neural(dev(q, "bf16"), dev(k, "bf16"), dev(v, "bf16"), dev(xq, "f32"), dev(xk, "f32"),
                          dev(wq, "f32"), dev(wk, "f32"), scale=scale, causal=causal)
    torch.cuda.synchronize()
    _no_device_error()
    pq, pk = oracle.neural_factors(xq, xk, wq, wk)
    ro, rl = oracle.attention(q, k, v, lambda b, h: HeadBias.lowrank(pq[b, h], pk[b, h]), scale, causal)
    og, lg = host(o), host(l)
    for b in range(B):
        for h in range(H):
            compare(og[b, h], lg[b, h], ro[b, h], rl[b, h], "bf16", f"neural F{F} R{R} ({b},{h})")


# ---------------------------------------------------------------- backward

BWD_SWEEP = [
    # B, H, N, d, R, causal, factor layout
    (1, 2, 200, 64, 64, True, "bhnr"),
    (1, 1, 1, 64, 8, True, "bhnr"),
    (2, 1, 257, 128, 2, True, "bhnr"),
    (1, 2, 300, 128, 128, False, "hnr"),
    (1, 1, 384, 32, 1, True, "bhnr"),
    (1, 2, 130, 16, 8, False, "nr"),
    (1, 2, 255, 24, 32, True, "bhnr"),
    (1, 1, 513, 40, 4, False, "bhnr"),
    (1, 2, 700, 64, 0, True, "bhnr"),
    (1, 1, 400, 96, 100, False, "bhnr"),
    (2, 3, 129, 8, 4, True, "hnr"),      # d = 8 (head dim 16 padded), ragged by one row, head-shared factors
    (1, 1, 640, 128, 16, True, "bhnr"),  # head dim 128 with 32-row query blocks, several diagonal blocks
    (3, 2, 96, 64, 64, False, "nr"),     # one factor slice for all six heads, N below one tile
    (1, 1, 1024, 32, 0, False, "bhnr"),  # plain attention, many blocks
]


@pytest.mark.parametrize("B,H,N,d,R,causal,layout", BWD_SWEEP)
def test_backward_matches_oracle(B, H, N, d, R, causal, layout):
    seed = 900 + N + d + R
    q, k, v = si.qkv(B, H, N, d, seed, "bf16")
    g = si.round_to_bf16(si.normal((B, H, N, d), seed + 3))
    scale = 1.0 / math.sqrt(d)
    pq = pk = None
    if R > 0:
        shape = {"nr": (N, R), "hnr": (H, N, R), "bhnr": (B, H, N, R)}[layout]
        pq, pk = si.random_factors(shape, math.sqrt(1.0 / R), seed + 7)
    tq, tk, tv, tg = (dev(x, "bf16") for x in (q, k, v, g))
    tpq = None if pq is None else dev(pq, "f32")
    tpk = None if pk is None else dev(pk, "f32")
    o, lse = fb.attn(tq, tk, tv, tpq, tpk, scale=scale, causal=causal)
    dq, dk, dv, dpq, dpk = fb.attn_bwd(tq, tk, tv, tpq, tpk, o, lse, tg, scale=scale, causal=causal)
    torch.cuda.synchronize()
    _no_device_error()

    def fac(x, b, h):
        if x is None:
            return np.zeros((N, 0))
        return {"nr": lambda: x, "hnr": lambda: x[h], "bhnr": lambda: x[b, h]}[layout]()

    ref_pq = None if pq is None else np.zeros(pq.shape)
    ref_pk = None if pk is None else np.zeros(pk.shape)
    got = {n: host(t) for n, t in (("dq", dq), ("dk", dk), ("dv", dv))}
    for b in range(B):
        for h in range(H):
            r = oracle.attention_lowrank_bwd_head(q[b, h], k[b, h], v[b, h], fac(pq, b, h), fac(pk, b, h),
                                                  g[b, h], scale, causal)
            for n in ("dq", "dk", "dv"):
                grad_close(got[n][b, h], r[n], f"{n} ({b},{h}) B{B} H{H} N{N} d{d} R{R} c{causal}")
            if R > 0:
                for acc, key in ((ref_pq, "dphi_q"), (ref_pk, "dphi_k")):
                    if layout == "nr":
                        acc += r[key]
                    elif layout == "hnr":
                        acc[h] += r[key]
                    else:
                        acc[b, h] += r[key]
    if R > 0:
        grad_close(host(dpq), ref_pq, f"dphi_q B{B} H{H} N{N} d{d} R{R} {layout}")
        grad_close(host(dpk), ref_pk, f"dphi_k B{B} H{H} N{N} d{d} R{R} {layout}")


@pytest.mark.parametrize("B,H,N,d,R,causal", [(1, 2, 200, 64, 64, True), (1, 1, 257, 128, 2, False),
                                               (1, 2, 300, 32, 100, True)])
def test_backward_fixed_factors_matches_oracle(B, H, N, d, R, causal):
    """Fixed factors (no factor gradients requested): dQ, dK, dV still match."""
    seed = 1900 + N + R
    q, k, v = si.qkv(B, H, N, d, seed, "bf16")
    g = si.round_to_bf16(si.normal((B, H, N, d), seed + 3))
    pq, pk = si.random_factors((B, H, N, R), math.sqrt(1.0 / R), seed + 7)
    scale = 1.0 / math.sqrt(d)
    tq, tk, tv, tg = (dev(x, "bf16") for x in (q, k, v, g))
    tpq, tpk = dev(pq, "f32"), dev(pk, "f32")
    o, lse = fb.attn(tq, tk, tv, tpq, tpk, scale=scale, causal=causal)
    dq, dk, dv, dpq, dpk = fb.attn_bwd(tq, tk, tv, tpq, tpk, o, lse, tg, scale=scale, causal=causal,
                                       factor_grads=False)
    torch.cuda.synchronize()
    _no_device_error()
    assert dpq is None and dpk is None
    got = {n: host(t) for n, t in (("dq", dq), ("dk", dk), ("dv", dv))}
    for b in range(B):
        for h in range(H):
            r = oracle.attention_lowrank_bwd_head(q[b, h], k[b, h], v[b, h], pq[b, h], pk[b, h], g[b, h], scale,
                                                  causal)
            for n in ("dq", "dk", "dv"):
                grad_close(got[n][b, h], r[n], f"{n} ({b},{h}) fixed factors N{N} d{d} R{R}")


@pytest.mark.parametrize("B,H,N,d,F,R,causal", [(2, 3, 200, 64, 16, 8, True), (1, 2, 130, 24, 64, 32, False)])
def test_neural_backward_matches_oracle(B, H, N, d, F, R, causal):
    """The neural decomposition's backward (fb_attn_neural_bwd) down to the
    linear layers' features and weights."""
    seed = 2900 + N + F
    q, k, v = si.qkv(B, H, N, d, seed, "bf16")
    g = si.round_to_bf16(si.normal((B, H, N, d), seed + 3))
    xq, xk, wq, wk = si.neural_inputs(B, H, N, F, R, seed + 5)
    scale = 1.0 / math.sqrt(d)
    tq, tk, tv, tg = (dev(x, "bf16") for x in (q, k, v, g))
    txq, txk, twq, twk = (dev(x, "f32") for x in (xq, xk, wq, wk))
    o, lse = fb.attn_neural(tq, tk, tv, txq, txk, twq, twk, scale=scale, causal=causal)
    dq, dk, dv, dxq, dxk, dwq, dwk = fb.attn_neural_bwd(tq, tk, tv, txq, txk, twq, twk, o, lse, tg, scale=scale,
                                                        causal=causal)
    torch.cuda.synchronize()
    _no_device_error()
    ref = oracle.neural_bwd(xq, xk, wq, wk, q, k, v, g, scale, causal)
    for name, t in (("dq", dq), ("dk", dk), ("dv", dv), ("dx_q", dxq), ("dx_k", dxk), ("dw_q", dwq), ("dw_k", dwk)):
        grad_close(host(t), ref[name], f"{name} B{B} H{H} N{N} d{d} F{F} R{R} c{causal}")
