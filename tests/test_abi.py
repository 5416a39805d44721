"""Host-side checks of libflashbias (no GPU): the library loads, exports every
symbol the header declares, rejects bad arguments before any launch, and its
host truncated SVD matches the oracle's library SVD."""
import ctypes
import math
import os
import re

import numpy as np
import pytest

import attention_rank_additive_b200 as fb
import oracle
import seeded_inputs as si

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def _built():
    from attention_rank_additive_b200 import build
    build.build()


def _declared():
    text = open(os.path.join(ROOT, "include", "flashbias.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(fb_[a-z0-9_]+)\s*\(", text)))


def test_header_symbols_exported():
    declared = _declared()
    assert set(declared) == set(fb.EXPORTED)
    L = ctypes.CDLL(fb.lib_path)
    for name in declared:
        assert hasattr(L, name), name


def test_status_strings_and_version():
    assert fb.fb_status_str(fb.FB_OK) == "FB_OK"
    assert fb.fb_status_str(fb.FB_ERR_TIMEOUT) == "FB_ERR_TIMEOUT"
    assert fb.fb_status_str(99) == "FB_ERR_UNKNOWN"
    assert fb.fb_version() >= 100


def test_workspace_bytes():
    # Every nonzero size ends in the fused kernel's 256-byte work-counter block.
    C = 256
    assert fb.fb_attn_workspace_bytes(8, 12, 2048, 0, 0, 0) == 0
    # broadcast Sandwich factors: one [N, 64] fp16 slice per side
    assert fb.fb_attn_workspace_bytes(8, 12, 2048, 64, 0, 0) == 2 * 2048 * 64 * 2 + C
    # rank 8 pads to 16 columns; per-head factors
    assert fb.fb_attn_workspace_bytes(4, 8, 4096, 8, 0, 4096 * 8) == 2 * 8 * 4096 * 16 * 2 + C
    # rank <= 4: fp32 hi/lo split factors, 3R columns padded to 8 (R <= 2) or 16
    assert fb.fb_attn_workspace_bytes(4, 16, 8192, 2, 0, 8192 * 2) == 2 * 16 * 8192 * 8 * 4 + C
    assert fb.fb_attn_workspace_bytes(1, 1, 17, 3, 0, 0) == 2 * 1280 + C  # 17 rows x 64 B, rounded to 256 B
    assert fb.fb_attn_workspace_bytes(1, 1, 16, 129, 0, 0) == 0  # out of range -> 0


FAKE = 1 << 20  # a 16-byte aligned address; never dereferenced by the checks below


def _fwd(**kw):
    a = dict(dt=fb.FB_BF16, B=1, H=1, N=128, d=64, Q=FAKE, K=FAKE, V=FAKE, R=0, phi_q=0, phi_k=0, phi_bstride=0,
             phi_hstride=0, scale=0.125, causal=0, O=FAKE, LSE=FAKE, workspace=0, workspace_bytes=0, stream=None)
    a.update(kw)
    return fb.fb_attn_fwd(**a)


def test_noalloc_reports_fb_attn_fwd_argument_errors_first():
    """fb_attn_fwd_noalloc runs fb_attn_fwd's argument checks before its own
    size limit, so a bad argument gets the same status from both, even for a
    problem whose prepared factors would not fit its fixed array."""
    def na(**kw):
        a = dict(dt=fb.FB_BF16, B=4, H=16, N=8192, d=64, Q=FAKE, K=FAKE, V=FAKE, R=64, phi_q=FAKE, phi_k=FAKE,
                 phi_bstride=16 * 8192 * 64, phi_hstride=8192 * 64, scale=0.125, causal=1, O=FAKE, LSE=FAKE,
                 stream=None)
        a.update(kw)
        return fb.fb_attn_fwd_noalloc(**a)

    for bad in (dict(Q=0), dict(O=FAKE + 4), dict(scale=0.0), dict(phi_hstride=-1), dict(d=12), dict(N=0),
                dict(dt=fb.FB_F16), dict(R=200)):
        full = dict(B=4, H=16, N=8192, d=64, R=64, phi_q=FAKE, phi_k=FAKE, phi_bstride=16 * 8192 * 64,
                    phi_hstride=8192 * 64, causal=1)
        full.update(bad)
        assert na(**bad) == _fwd(**full) != fb.FB_OK, bad
    assert na() == fb.FB_ERR_WORKSPACE  # valid, but beyond the 8 MiB array


def test_forward_rejects_bad_arguments_before_launch():
    assert _fwd(Q=0) == fb.FB_ERR_INVALID_ARG
    assert _fwd(LSE=0) == fb.FB_ERR_INVALID_ARG
    assert _fwd(Q=FAKE + 8) == fb.FB_ERR_INVALID_ARG  # misaligned
    assert _fwd(scale=0.0) == fb.FB_ERR_INVALID_ARG
    assert _fwd(scale=-1.0) == fb.FB_ERR_INVALID_ARG
    assert _fwd(scale=float("nan")) == fb.FB_ERR_INVALID_ARG
    assert _fwd(R=129) == fb.FB_ERR_UNSUPPORTED
    assert _fwd(R=-1) == fb.FB_ERR_UNSUPPORTED
    assert _fwd(R=8) == fb.FB_ERR_INVALID_ARG  # factors missing
    assert _fwd(R=8, phi_q=FAKE, phi_k=FAKE, phi_bstride=-1) == fb.FB_ERR_INVALID_ARG
    assert _fwd(d=12) == fb.FB_ERR_UNSUPPORTED
    assert _fwd(d=136) == fb.FB_ERR_UNSUPPORTED
    assert _fwd(N=0) == fb.FB_ERR_INVALID_ARG
    assert _fwd(B=0) == fb.FB_ERR_INVALID_ARG
    assert _fwd(dt=7) == fb.FB_ERR_UNSUPPORTED
    assert _fwd(dt=fb.FB_F16) == fb.FB_ERR_UNSUPPORTED  # fp16 inputs are not implemented
    assert _fwd(dt=fb.FB_F32, d=6) == fb.FB_ERR_UNSUPPORTED
    # workspace missing / too small / misaligned
    assert _fwd(R=8, phi_q=FAKE, phi_k=FAKE) == fb.FB_ERR_WORKSPACE
    need = fb.fb_attn_workspace_bytes(1, 1, 128, 8, 0, 0)
    assert _fwd(R=8, phi_q=FAKE, phi_k=FAKE, workspace=FAKE, workspace_bytes=need - 1) == fb.FB_ERR_WORKSPACE
    assert _fwd(R=8, phi_q=FAKE, phi_k=FAKE, workspace=FAKE + 16, workspace_bytes=need) == fb.FB_ERR_WORKSPACE


def _dense(**kw):
    a = dict(dt=fb.FB_BF16, B=1, H=1, N=128, d=64, Q=FAKE, K=FAKE, V=FAKE, Bias=FAKE, bias_bstride=0, bias_hstride=0,
             scale=0.125, causal=0, O=FAKE, LSE=FAKE, stream=None)
    a.update(kw)
    return fb.fb_attn_dense_bias_fwd(**a)


def test_dense_rejects_bad_arguments_before_launch():
    assert _dense(Bias=0) == fb.FB_ERR_INVALID_ARG
    assert _dense(Bias=FAKE + 2) == fb.FB_ERR_INVALID_ARG
    assert _dense(bias_hstride=-8) == fb.FB_ERR_INVALID_ARG
    assert _dense(N=130) == fb.FB_ERR_UNSUPPORTED  # bias row pitch must be 16-byte aligned
    assert _dense(bias_hstride=12, H=2) == fb.FB_ERR_UNSUPPORTED
    assert _dense(scale=0.0) == fb.FB_ERR_INVALID_ARG


def test_factor_generators_reject_bad_arguments():
    assert fb.fb_factors_sandwich(16, 7, FAKE, FAKE, None) == fb.FB_ERR_INVALID_ARG
    assert fb.fb_factors_sandwich(0, 8, FAKE, FAKE, None) == fb.FB_ERR_INVALID_ARG
    assert fb.fb_factors_sandwich(16, 130, FAKE, FAKE, None) == fb.FB_ERR_INVALID_ARG
    assert fb.fb_factors_alibi(0, 16, FAKE, FAKE, None) == fb.FB_ERR_INVALID_ARG
    assert fb.fb_factors_alibi(4, 16, 0, FAKE, None) == fb.FB_ERR_INVALID_ARG
    assert fb.fb_selftest_wait_timeout(0, None) == fb.FB_ERR_INVALID_ARG
    assert fb.fb_selftest_wait_timeout(5000, None) == fb.FB_ERR_INVALID_ARG


# --- host truncated SVD (product) against the oracle's library SVD ----------

def _known_spectrum(N, sigma, seed):
    rng = np.random.Generator(np.random.PCG64(seed))
    U, _ = np.linalg.qr(rng.standard_normal((N, len(sigma))))
    V, _ = np.linalg.qr(rng.standard_normal((N, len(sigma))))
    return U @ np.diag(sigma) @ V.T


def test_svd_host_known_spectrum():
    sigma = np.array([40.0, 15.0, 7.0, 3.0, 1.0, 0.3, 0.1, 0.03, 0.01, 0.003])
    Bm = _known_spectrum(257, sigma, 5)
    for R in (1, 4, 8):
        pq, pk, rel, energy = fb.svd_factors(Bm, R, oversample=16, power_iters=2, seed=3)
        want_rel = math.sqrt(np.sum(sigma[R:] ** 2) / np.sum(sigma ** 2))
        assert abs(rel - want_rel) < 1e-6
        assert abs(energy - np.sum(sigma[:R] ** 2) / np.sum(sigma ** 2)) < 1e-6
        opq, opk, orel, _ = oracle.truncated_svd_factors(Bm, R)
        np.testing.assert_allclose(pq.astype(np.float64) @ pk.T.astype(np.float64), opq @ opk.T, atol=2e-5)


def test_svd_host_rbf_field_matches_oracle():
    grid, M, R = 24, 32, 8
    om, ph = si.rbf_params(2, M)
    dense = si.rbf_dense(si.rbf_offset_table(om, ph, grid), grid)
    for h in range(2):
        pq, pk, rel, energy = fb.svd_factors(dense[h], R, oversample=64, power_iters=1, seed=11)
        opq, opk, orel, oen = oracle.truncated_svd_factors(dense[h], R)
        assert abs(rel - orel) < 1e-6 and abs(energy - oen) < 1e-6
        np.testing.assert_allclose(pq.astype(np.float64) @ pk.T.astype(np.float64), opq @ opk.T,
                                   atol=1e-5 * np.abs(dense[h]).max())


def test_svd_host_rejects_bad_arguments():
    b = np.zeros((4, 4))
    out = np.zeros((4, 8), dtype=np.float32)
    assert fb.fb_svd_factors_host(b.ctypes.data, 4, 0, 4, 1, 0, out.ctypes.data, out.ctypes.data, None, None) \
        == fb.FB_ERR_INVALID_ARG
    assert fb.fb_svd_factors_host(b.ctypes.data, 4, 5, 4, 1, 0, out.ctypes.data, out.ctypes.data, None, None) \
        == fb.FB_ERR_INVALID_ARG
    assert fb.fb_svd_factors_host(None, 4, 2, 4, 1, 0, out.ctypes.data, out.ctypes.data, None, None) \
        == fb.FB_ERR_INVALID_ARG


def test_fma_pipe_exp2_polynomial_error_bound():
    """The FMA-pipe exp2 of the softmax (range reduction + fitted cubic),
    restated in numpy float32 and checked against fp64 exp2: relative error
    below 1e-4 on the range the softmax uses, so it is invisible after P is
    rounded to bf16 (relative step 2^-8)."""
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "fit", os.path.join(ROOT, "attention_rank_additive_b200", "csrc", "fit_exp2_poly.py"))
    fit = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(fit)
    c, err = fit.fit(samples=4001, iters=150)
    assert err < 1e-4
    want = [0.9999252, 0.6958336, 0.22606726, 0.078024276]  # the constants in fb_ptx.cuh
    np.testing.assert_allclose(np.float32(c), np.float32(want), rtol=2e-4)
    x = np.concatenate([np.linspace(-126.0, 8.0, 200001), -np.arange(0, 127, dtype=np.float64)]).astype(np.float32)
    n = np.floor(x)
    f = (x - n).astype(np.float32)
    w = np.float32(want)
    p = ((w[3] * f + w[2]) * f + w[1]) * f + w[0]
    got = p.astype(np.float64) * np.exp2(n.astype(np.float64))
    rel = np.abs(got / np.exp2(x.astype(np.float64)) - 1.0)
    assert rel.max() < 1e-4


def test_prepared_entry_points_reject_bad_arguments_before_launch():
    need = fb.fb_attn_workspace_bytes(1, 1, 128, 8, 0, 0)
    prep = dict(B=1, H=1, N=128, R=8, phi_q=FAKE, phi_k=FAKE, phi_bstride=0, phi_hstride=0, scale=0.125,
                workspace=FAKE, workspace_bytes=need, stream=None)

    def p(**kw):
        a = dict(prep)
        a.update(kw)
        return fb.fb_attn_prepare_factors(**a)

    assert p(R=0, phi_q=0, phi_k=0, workspace=0, workspace_bytes=0) == fb.FB_OK  # nothing to prepare
    assert p(R=129) == fb.FB_ERR_UNSUPPORTED
    assert p(N=0) == fb.FB_ERR_INVALID_ARG
    assert p(phi_q=0) == fb.FB_ERR_INVALID_ARG
    assert p(phi_k=FAKE + 2) == fb.FB_ERR_INVALID_ARG
    assert p(phi_hstride=-1) == fb.FB_ERR_INVALID_ARG
    assert p(scale=0.0) == fb.FB_ERR_INVALID_ARG
    assert p(workspace=0) == fb.FB_ERR_WORKSPACE
    assert p(workspace_bytes=need - 1) == fb.FB_ERR_WORKSPACE
    assert p(workspace=FAKE + 16) == fb.FB_ERR_WORKSPACE

    run = dict(dt=fb.FB_BF16, B=1, H=1, N=128, d=64, Q=FAKE, K=FAKE, V=FAKE, R=8, phi_bstride=0, phi_hstride=0,
               scale=0.125, causal=0, O=FAKE, LSE=FAKE, workspace=FAKE, workspace_bytes=need, stream=None)

    def r(**kw):
        a = dict(run)
        a.update(kw)
        return fb.fb_attn_fwd_prepared(**a)

    assert r(dt=fb.FB_F32) == fb.FB_ERR_UNSUPPORTED  # the prepared form is the tensor-core path
    assert r(Q=0) == fb.FB_ERR_INVALID_ARG
    assert r(O=FAKE + 8) == fb.FB_ERR_INVALID_ARG
    assert r(d=12) == fb.FB_ERR_UNSUPPORTED
    assert r(R=129) == fb.FB_ERR_UNSUPPORTED
    assert r(scale=-1.0) == fb.FB_ERR_INVALID_ARG
    assert r(workspace=0) == fb.FB_ERR_WORKSPACE
    assert r(workspace_bytes=need - 1) == fb.FB_ERR_WORKSPACE


def test_shape_limit_on_work_items():
    # B * H * ceil(N / 128) work items must stay below 2^30 (the kernel counts them in int)
    assert _fwd(B=65536, H=128, N=16512) == fb.FB_ERR_UNSUPPORTED


def test_mul_bias_workspace_and_argument_errors():
    # q1, k1 bf16 [BH, N, d] each, then fp16 factor rows of rank d (R - 1) padded to 16..128
    B, H, N, d, R = 2, 3, 130, 64, 2
    qk = B * H * N * d * 2
    al = lambda x: (x + 255) // 256 * 256
    fac = fb.fb_attn_workspace_bytes(B, H, N, d * (R - 1), H * N * d, N * d)
    assert fb.fb_attn_mul_bias_workspace_bytes(B, H, N, d, R) == 2 * al(qk) + fac
    assert fb.fb_attn_mul_bias_workspace_bytes(B, H, N, d, 1) == 2 * al(qk)  # rank 1: no factor part
    assert fb.fb_attn_mul_bias_workspace_bytes(B, H, N, 64, 4) == 0  # d (R - 1) > 128
    need = fb.fb_attn_mul_bias_workspace_bytes(1, 1, 128, 64, 2)
    run = dict(dt=fb.FB_BF16, B=1, H=1, N=128, d=64, Q=FAKE, K=FAKE, V=FAKE, R=2, phi_q=FAKE, phi_k=FAKE,
               phi_bstride=0, phi_hstride=0, scale=0.125, causal=1, O=FAKE, LSE=FAKE, workspace=FAKE,
               workspace_bytes=need, stream=None)

    def m(**kw):
        a = dict(run)
        a.update(kw)
        return fb.fb_attn_mul_bias_fwd(**a)

    assert m(dt=fb.FB_F32) == fb.FB_ERR_UNSUPPORTED
    assert m(R=0) == fb.FB_ERR_UNSUPPORTED
    assert m(R=4) == fb.FB_ERR_UNSUPPORTED  # 64 * 3 > 128
    assert m(phi_q=0) == fb.FB_ERR_INVALID_ARG
    assert m(phi_k=FAKE + 2) == fb.FB_ERR_INVALID_ARG
    assert m(phi_hstride=-1) == fb.FB_ERR_INVALID_ARG
    assert m(Q=FAKE + 8) == fb.FB_ERR_INVALID_ARG
    assert m(scale=0.0) == fb.FB_ERR_INVALID_ARG
    assert m(d=12) == fb.FB_ERR_UNSUPPORTED
    assert m(workspace=0) == fb.FB_ERR_WORKSPACE
    assert m(workspace_bytes=need - 1) == fb.FB_ERR_WORKSPACE
    assert m(workspace=FAKE + 16) == fb.FB_ERR_WORKSPACE


def test_svd_device_workspace_and_argument_errors():
    # three [H, l, N] fp32 buffers (l = min(R + oversample, 32, N)) + fp64 small matrices, each 256-aligned
    al = lambda x: (x + 255) // 256 * 256
    H, N, R, p = 3, 500, 8, 16
    l = 24
    assert fb.fb_svd_device_workspace_bytes(H, N, R, p) == 3 * al(H * l * N * 4) + al(H * (2 * l * l + 2 * l * R + 5) * 8)
    assert fb.fb_svd_device_workspace_bytes(1, 10, 8, 40) == 3 * al(10 * 10 * 4) + al((2 * 100 + 2 * 10 * 8 + 5) * 8)
    assert fb.fb_svd_device_workspace_bytes(1, 100, 33, 0) == 0  # R > 32
    need = fb.fb_svd_device_workspace_bytes(2, 64, 4, 8)
    a = dict(H=2, N=64, R=4, oversample=8, power_iters=1, seed=1, bias=FAKE, phi_q=FAKE, phi_k=FAKE, err_energy=0,
             workspace=FAKE, workspace_bytes=need, stream=None)

    def s(**kw):
        b = dict(a)
        b.update(kw)
        return fb.fb_svd_factors_device(**b)

    assert s(bias=0) == fb.FB_ERR_INVALID_ARG
    assert s(phi_k=FAKE + 2) == fb.FB_ERR_INVALID_ARG
    assert s(err_energy=FAKE + 4) == fb.FB_ERR_INVALID_ARG
    assert s(R=0) == fb.FB_ERR_UNSUPPORTED
    assert s(R=33) == fb.FB_ERR_UNSUPPORTED
    assert s(R=65, N=64) == fb.FB_ERR_UNSUPPORTED
    assert s(power_iters=-1) == fb.FB_ERR_UNSUPPORTED
    assert s(workspace=0) == fb.FB_ERR_WORKSPACE
    assert s(workspace_bytes=need - 1) == fb.FB_ERR_WORKSPACE
    assert s(workspace=FAKE + 16) == fb.FB_ERR_WORKSPACE


def test_neural_workspace_and_argument_errors():
    B, H, N, F, R = 2, 4, 100, 16, 8
    # the linear layers write the prepared per-head factors directly: the
    # workspace is fb_attn_fwd's for per-head factors, nothing more
    prep = fb.fb_attn_workspace_bytes(B, H, N, R, H * N * R, N * R)
    assert fb.fb_attn_neural_workspace_bytes(B, H, N, F, R) == prep
    assert fb.fb_attn_neural_workspace_bytes(B, H, N, 128, 128) == 0  # F R > 8192
    need = fb.fb_attn_neural_workspace_bytes(1, 2, 128, F, R)
    run = dict(dt=fb.FB_BF16, B=1, H=2, N=128, d=64, Q=FAKE, K=FAKE, V=FAKE, F=F, R=R, X_q=FAKE, X_k=FAKE,
               W_q=FAKE, W_k=FAKE, scale=0.125, causal=0, O=FAKE, LSE=FAKE, workspace=FAKE, workspace_bytes=need,
               stream=None)

    def n(**kw):
        a = dict(run)
        a.update(kw)
        return fb.fb_attn_neural_fwd(**a)

    assert n(dt=fb.FB_F32) == fb.FB_ERR_UNSUPPORTED
    assert n(F=0) == fb.FB_ERR_UNSUPPORTED
    assert n(R=129) == fb.FB_ERR_UNSUPPORTED
    assert n(F=257) == fb.FB_ERR_UNSUPPORTED
    assert n(W_k=0) == fb.FB_ERR_INVALID_ARG
    assert n(X_q=FAKE + 2) == fb.FB_ERR_INVALID_ARG
    assert n(scale=-1.0) == fb.FB_ERR_INVALID_ARG
    assert n(d=20) == fb.FB_ERR_UNSUPPORTED
    assert n(workspace=0) == fb.FB_ERR_WORKSPACE
    assert n(workspace_bytes=need - 1) == fb.FB_ERR_WORKSPACE


def test_backward_workspace_and_argument_errors():
    """fb_attn_bwd: the workspace covers the forward's factor tiles, the bf16
    factor copies, two fp32 rows per (b, h, padded query) and a 128-column
    fp32 accumulator row per (b, h, padded query) (the fused kernel's dq', or
    the two-kernel path's per-head dphi_q rows) and the fused kernel's work
    counter; every argument error returns before a launch."""
    al = lambda x: (x + 255) // 256 * 256
    B, H, N, R = 2, 3, 200, 8
    Npad = 256
    acc = al(B * H * Npad * 128 * 4)
    fwd = fb.fb_attn_workspace_bytes(B, H, N, R, H * N * R, N * R)
    sched = 256  # the fused kernel's work counter
    assert fb.fb_attn_bwd_workspace_bytes(B, H, N, R, H * N * R, N * R) == \
        fwd + 2 * al(B * H * N * 16 * 2) + 2 * al(B * H * Npad * 4) + acc + sched
    # broadcast factors: one factor slice, plus per-head partial dphi_k rows
    assert fb.fb_attn_bwd_workspace_bytes(B, H, N, R, 0, 0) == \
        fb.fb_attn_workspace_bytes(B, H, N, R, 0, 0) + 2 * al(N * 16 * 2) + 2 * al(B * H * Npad * 4) + \
        acc + al(B * H * N * R * 4) + sched
    assert fb.fb_attn_bwd_workspace_bytes(B, H, N, 0, 0, 0) == 2 * al(B * H * Npad * 4) + acc + sched
    assert fb.fb_attn_bwd_workspace_bytes(B, H, N, 129, 0, 0) == 0
    assert fb.fb_attn_bwd_workspace_bytes(0, H, N, R, 0, 0) == 0
    need = fb.fb_attn_bwd_workspace_bytes(1, 2, 128, R, 2 * 128 * R, 128 * R)
    run = dict(dt=fb.FB_BF16, B=1, H=2, N=128, d=64, Q=FAKE, K=FAKE, V=FAKE, R=R, phi_q=FAKE, phi_k=FAKE,
               phi_bstride=2 * 128 * R, phi_hstride=128 * R, scale=0.125, causal=1, O=FAKE, LSE=FAKE, dO=FAKE,
               dQ=FAKE, dK=FAKE, dV=FAKE, dphi_q=FAKE, dphi_k=FAKE, workspace=FAKE, workspace_bytes=need,
               stream=None)

    def b(**kw):
        a = dict(run)
        a.update(kw)
        return fb.fb_attn_bwd(**a)

    assert b(dt=fb.FB_F32) == fb.FB_ERR_UNSUPPORTED
    assert b(R=129) == fb.FB_ERR_UNSUPPORTED
    assert b(d=20) == fb.FB_ERR_UNSUPPORTED
    assert b(dO=0) == fb.FB_ERR_INVALID_ARG
    assert b(dphi_k=0) == fb.FB_ERR_INVALID_ARG  # one factor gradient without the other
    assert b(dphi_q=FAKE + 2) == fb.FB_ERR_INVALID_ARG
    assert b(dK=FAKE + 8) == fb.FB_ERR_INVALID_ARG
    assert b(phi_hstride=-1) == fb.FB_ERR_INVALID_ARG
    assert b(scale=float("nan")) == fb.FB_ERR_INVALID_ARG
    assert b(workspace=0) == fb.FB_ERR_WORKSPACE
    assert b(workspace_bytes=need - 1) == fb.FB_ERR_WORKSPACE
    assert b(workspace=FAKE + 16) == fb.FB_ERR_WORKSPACE


def test_neural_backward_workspace_and_argument_errors():
    """fb_attn_neural_bwd: the workspace holds the factors, their gradients and
    fb_attn_bwd's own (per-head factor slices); argument errors return before a
    launch."""
    al = lambda x: (x + 255) // 256 * 256
    B, H, N, F, R = 2, 3, 100, 16, 8
    phi = al(B * H * N * R * 4)
    assert fb.fb_attn_neural_bwd_workspace_bytes(B, H, N, F, R) == \
        4 * phi + fb.fb_attn_bwd_workspace_bytes(B, H, N, R, H * N * R, N * R)
    assert fb.fb_attn_neural_bwd_workspace_bytes(B, H, N, 128, 128) == 0  # F R > 8192
    need = fb.fb_attn_neural_bwd_workspace_bytes(1, 2, 128, F, R)
    run = dict(dt=fb.FB_BF16, B=1, H=2, N=128, d=64, Q=FAKE, K=FAKE, V=FAKE, F=F, R=R, X_q=FAKE, X_k=FAKE,
               W_q=FAKE, W_k=FAKE, scale=0.125, causal=1, O=FAKE, LSE=FAKE, dO=FAKE, dQ=FAKE, dK=FAKE, dV=FAKE,
               dX_q=FAKE, dX_k=FAKE, dW_q=FAKE, dW_k=FAKE, workspace=FAKE, workspace_bytes=need, stream=None)

    def n(**kw):
        a = dict(run)
        a.update(kw)
        return fb.fb_attn_neural_bwd(**a)

    assert n(dt=fb.FB_F32) == fb.FB_ERR_UNSUPPORTED
    assert n(F=0) == fb.FB_ERR_UNSUPPORTED
    assert n(R=129) == fb.FB_ERR_UNSUPPORTED
    assert n(dW_k=0) == fb.FB_ERR_INVALID_ARG
    assert n(dX_q=0) == fb.FB_ERR_INVALID_ARG  # one feature gradient without the other
    assert n(W_q=FAKE + 2) == fb.FB_ERR_INVALID_ARG
    assert n(dV=FAKE + 8) == fb.FB_ERR_INVALID_ARG
    assert n(scale=0.0) == fb.FB_ERR_INVALID_ARG
    assert n(d=20) == fb.FB_ERR_UNSUPPORTED
    assert n(workspace=0) == fb.FB_ERR_WORKSPACE
    assert n(workspace_bytes=need - 1) == fb.FB_ERR_WORKSPACE
