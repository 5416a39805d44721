"""GPU parity on the five benchmark workloads at their full sizes, in the
launch configuration the benchmark uses. The oracle evaluates sampled query
rows of sampled heads one by one (always the first and last row)."""
import concurrent.futures
import math
import os

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


def _check_rows(o, l, q, k, v, heads, rows, bias_of, scale, causal, dtype, what):
    og, lg = host(o), host(l)
    ro, rl = oracle.attention(q, k, v, bias_of, scale, causal, rows=rows, heads=heads)
    errs = []
    for (b, h) in heads:
        errs.append(compare(og[b, h][rows], lg[b, h][rows], ro[(b, h)], rl[(b, h)], dtype, f"{what} ({b},{h})"))
    return errs


def _stream():
    return torch.cuda.current_stream().cuda_stream


def test_config0_fp32_lowrank_all_rows():
    c = si.CONFIGS[0]
    B, H, N, d, R = c["B"], c["H"], c["N"], c["d"], c["R"]
    q, k, v = si.qkv(B, H, N, d, si.QKV_SEED_BASE + 0, "f32")
    pq, pk = si.random_factors((B, H, N, R), c["factor_std"], si.FACTOR_SEED_BASE + 0)
    scale = 1.0 / math.sqrt(d)
    o, l = fb.attn(dev(q, "f32"), dev(k, "f32"), dev(v, "f32"), dev(pq, "f32"), dev(pk, "f32"), scale=scale)
    torch.cuda.synchronize()
    assert fb.fb_check_device_error(_stream()) == fb.FB_OK
    _check_rows(o, l, q, k, v, [(b, h) for b in range(B) for h in range(H)], np.arange(N),
                lambda b, h: HeadBias.lowrank(pq[b, h], pk[b, h]), scale, False, "f32", "c0")


def test_config1_sandwich_fused_and_dense():
    c = si.CONFIGS[1]
    B, H, N, d, R = c["B"], c["H"], c["N"], c["d"], c["R"]
    q, k, v = si.qkv(B, H, N, d, si.QKV_SEED_BASE + 1, "bf16")
    scale = 1.0 / math.sqrt(d)
    Q, K, V = dev(q, "bf16"), dev(k, "bf16"), dev(v, "bf16")
    phi = fb.factors_sandwich(N, R)
    o, l = fb.attn(Q, K, V, phi, phi, scale=scale, causal=True)
    torch.cuda.synchronize()
    assert fb.fb_check_device_error(_stream()) == fb.FB_OK
    heads = [(0, 0), (3, 7), (7, 11)]
    rows = si.sample_rows(N, 40, 1)
    _check_rows(o, l, q, k, v, heads, rows, lambda b, h: HeadBias.sandwich(R), scale, True, "bf16", "c1 fused")
    # dense comparison path: the same bias materialised as [B, H, N, N] bf16
    tab = si.round_to_bf16(si.sandwich_offset_table(N, R).astype(np.float32))
    bias = si.toeplitz_device(tab, N, "cuda").expand(B, H, N, N).contiguous()
    od, ld = fb.attn_dense_bias(Q, K, V, bias, scale=scale, causal=True)
    torch.cuda.synchronize()
    _check_rows(od, ld, q, k, v, heads, rows, lambda b, h: HeadBias.toeplitz(tab, N), scale, True, "bf16", "c1 dense")


def test_config2_alibi_fused_and_dense():
    c = si.CONFIGS[2]
    B, H, N, d = c["B"], c["H"], c["N"], c["d"]
    q, k, v = si.qkv(B, H, N, d, si.QKV_SEED_BASE + 2, "bf16")
    scale = 1.0 / math.sqrt(d)
    Q, K, V = dev(q, "bf16"), dev(k, "bf16"), dev(v, "bf16")
    pq, pk = fb.factors_alibi(H, N)
    o, l = fb.attn(Q, K, V, pq, pk, scale=scale, causal=True)
    torch.cuda.synchronize()
    assert fb.fb_check_device_error(_stream()) == fb.FB_OK
    heads = [(0, 0), (1, 5), (3, 15)]
    rows = si.sample_rows(N, 24, 2)
    _check_rows(o, l, q, k, v, heads, rows, lambda b, h: HeadBias.alibi(oracle.alibi_slope(h, H)), scale, True,
                "bf16", "c2 fused")
    del o, l
    # dense comparison path: per-head bias [H, N, N] bf16, shared by the batch
    tabs = [si.round_to_bf16(si.alibi_offset_table(N, oracle.alibi_slope(h, H)).astype(np.float32)) for h in range(H)]
    bias = torch.stack([si.toeplitz_device(t, N, "cuda") for t in tabs])
    od, ld = fb.attn_dense_bias(Q, K, V, bias, scale=scale, causal=True)
    torch.cuda.synchronize()
    _check_rows(od, ld, q, k, v, heads, rows, lambda b, h: HeadBias.toeplitz(tabs[h], N), scale, True, "bf16",
                "c2 dense")


def test_config3_rbf_svd_fused_and_dense():
    c = si.CONFIGS[3]
    B, H, N, d, R, g = c["B"], c["H"], c["N"], c["d"], c["R"], c["grid"]
    q, k, v = si.qkv(B, H, N, d, si.QKV_SEED_BASE + 3, "bf16")
    scale = 1.0 / math.sqrt(d)
    om, ph = si.rbf_params(H, c["rbf_terms"])
    table = si.rbf_offset_table(om, ph, g)
    pq = np.empty((H, N, R), np.float32)
    pk = np.empty((H, N, R), np.float32)
    errs = []
    for h in range(H):
        dense_h = si.rbf_dense(table, g, heads=[h])[0]
        pq[h], pk[h], rel, energy = fb.svd_factors(dense_h, R, oversample=64, power_iters=1, seed=h)
        errs.append((rel, energy))
    print("c3 SVD rank-8 relative Frobenius error / energy per head:", errs)
    Q, K, V = dev(q, "bf16"), dev(k, "bf16"), dev(v, "bf16")
    o, l = fb.attn(Q, K, V, dev(pq, "f32"), dev(pk, "f32"), scale=scale, causal=False)
    torch.cuda.synchronize()
    assert fb.fb_check_device_error(_stream()) == fb.FB_OK
    heads = [(0, 0), (3, 7)]
    rows = si.sample_rows(N, 32, 3)
    oracle_factors = {}
    for (_, h) in heads:
        opq, opk, orel, _ = oracle.truncated_svd_factors(si.rbf_dense(table, g, heads=[h])[0], R)
        assert abs(orel - errs[h][0]) < 1e-6
        oracle_factors[h] = (opq, opk)
    _check_rows(o, l, q, k, v, heads, rows, lambda b, h: HeadBias.lowrank(*oracle_factors[h]), scale, False, "bf16",
                "c3 fused")
    # dense comparison path: the field itself, bf16, materialised [H, N, N]
    tab16 = si.round_to_bf16(table.astype(np.float32))
    ix, iy = si.grid_offset_index(g)
    tdev = si.bf16_tensor(tab16, "cuda")
    ixd = torch.from_numpy(ix).cuda()
    iyd = torch.from_numpy(iy).cuda()
    bias = torch.stack([tdev[h][ixd, iyd] for h in range(H)])
    del ixd, iyd
    od, ld = fb.attn_dense_bias(Q, K, V, bias, scale=scale, causal=False)
    torch.cuda.synchronize()
    _check_rows(od, ld, q, k, v, heads, rows, lambda b, h: HeadBias.grid(tab16[h], g), scale, False, "bf16",
                "c3 dense")


def test_config4_pair_bias_fused_and_dense():
    c = si.CONFIGS[4]
    B, H, N, d, R = c["B"], c["H"], c["N"], c["d"], c["R"]
    q, k, v = si.qkv(B, H, N, d, si.QKV_SEED_BASE + 4, "bf16")
    pq, pk = si.random_factors((B, H, N, R), c["factor_std"], si.FACTOR_SEED_BASE + 4)
    scale = 1.0 / math.sqrt(d)
    Q, K, V = dev(q, "bf16"), dev(k, "bf16"), dev(v, "bf16")
    o, l = fb.attn(Q, K, V, dev(pq, "f32"), dev(pk, "f32"), scale=scale, causal=False)
    torch.cuda.synchronize()
    assert fb.fb_check_device_error(_stream()) == fb.FB_OK
    heads = [(0, 0), (0, 9), (0, 15)]
    rows = si.sample_rows(N, 64, 4)
    _check_rows(o, l, q, k, v, heads, rows, lambda b, h: HeadBias.lowrank(pq[b, h], pk[b, h]), scale, False, "bf16",
                "c4 fused")
    # dense comparison path: bf16(phi_q phi_k^T) per head
    dense = np.stack([si.round_to_bf16((pq[0, h].astype(np.float64) @ pk[0, h].T.astype(np.float64))
                                       .astype(np.float32)) for h in range(H)])
    od, ld = fb.attn_dense_bias(Q, K, V, dev(dense, "bf16")[None], scale=scale, causal=False)
    torch.cuda.synchronize()
    _check_rows(od, ld, q, k, v, heads, rows, lambda b, h: HeadBias.dense(dense[h]), scale, False, "bf16",
                "c4 dense")


def test_config5_multiplicative_cos_full_size():
    """The multiplicative cos(i - j) bias at the GPT-2 shape of the widening
    case (bench.py --config 5), sampled rows of three heads against the oracle."""
    c = si.CONFIGS[5]
    B, H, N, d, R = c["B"], c["H"], c["N"], c["d"], c["R"]
    q, k, v = si.qkv(B, H, N, d, si.QKV_SEED_BASE + 5, "bf16")
    scale = 1.0 / math.sqrt(d)
    i = np.arange(N, dtype=np.float64)
    f = np.stack([np.cos(i), np.sin(i)], 1).astype(np.float32)
    o, l = fb.attn_mul_bias(dev(q, "bf16"), dev(k, "bf16"), dev(v, "bf16"), dev(f, "f32"), dev(f, "f32"),
                            scale=scale, causal=True)
    torch.cuda.synchronize()
    assert fb.fb_check_device_error(_stream()) == fb.FB_OK
    og, lg = host(o), host(l)
    rows = si.sample_rows(N, 40, 5)
    for (b, h) in [(0, 0), (5, 6), (7, 11)]:
        ro, rl = oracle.attention_mul_head(q[b, h], k[b, h], v[b, h], f, f, scale, True, rows)
        compare(og[b, h][rows], lg[b, h][rows], ro, rl, "bf16", f"c5 ({b},{h})")


def test_config6_neural_full_size():
    """The neural-decomposition widening case (bench.py --config 6) at full
    size: sampled rows of three heads against the oracle."""
    c = si.CONFIGS[6]
    B, H, N, d, R, F = c["B"], c["H"], c["N"], c["d"], c["R"], c["F"]
    q, k, v = si.qkv(B, H, N, d, si.QKV_SEED_BASE + 6, "bf16")
    xq, xk, wq, wk = si.neural_inputs(B, H, N, F, R, si.FACTOR_SEED_BASE + 6)
    scale = 1.0 / math.sqrt(d)
    o, l = fb.attn_neural(dev(q, "bf16"), dev(k, "bf16"), dev(v, "bf16"), dev(xq, "f32"), dev(xk, "f32"),
                          dev(wq, "f32"), dev(wk, "f32"), scale=scale, causal=False)
    torch.cuda.synchronize()
    assert fb.fb_check_device_error(_stream()) == fb.FB_OK
    pq, pk = oracle.neural_factors(xq, xk, wq, wk)
    rows = si.sample_rows(N, 40, 6)
    _check_rows(o, l, q, k, v, [(0, 0), (0, 7), (0, 15)], rows, lambda b, h: HeadBias.lowrank(pq[b, h], pk[b, h]),
                scale, False, "bf16", "c6")


def test_config7_backward_full_size():
    """The backward workload (bench.py --config 7: GPT-2 Sandwich shape) at
    full size through fb_attn_bwd. Every gradient of two whole heads against
    the oracle; dphi_q (the Sandwich factor is shared by all 96 heads, so its
    gradient sums over them) on sampled rows through the oracle's
    row-restricted backward of every head, and dphi_k on sampled rows through
    its key-restricted backward of every head; also the zero column sums of
    dphi_k that rows of dS summing to zero imply."""
    c = si.CONFIGS[7]
    B, H, N, d, R = c["B"], c["H"], c["N"], c["d"], c["R"]
    q, k, v = si.qkv(B, H, N, d, si.QKV_SEED_BASE + 7, "bf16")
    g = si.upstream_grad(B, H, N, d, si.DO_SEED_BASE + 7)
    scale = 1.0 / math.sqrt(d)
    Q, K, V, G = (dev(x, "bf16") for x in (q, k, v, g))
    phi = fb.factors_sandwich(N, R)
    o, l = fb.attn(Q, K, V, phi, phi, scale=scale, causal=True)
    dq, dk, dv, dpq, dpk = fb.attn_bwd(Q, K, V, phi, phi, o, l, G, scale=scale, causal=True)
    torch.cuda.synchronize()
    assert fb.fb_check_device_error(_stream()) == fb.FB_OK
    ph = oracle.sandwich_factors(N, R)
    got = {"dq": host(dq), "dk": host(dk), "dv": host(dv)}
    for (b, h) in [(0, 0), (B - 1, H - 1)]:
        r = oracle.attention_lowrank_bwd_head(q[b, h], k[b, h], v[b, h], ph, ph, g[b, h], scale, True)
        for n in ("dq", "dk", "dv"):
            grad_close(got[n][b, h], r[n], f"c7 {n} ({b},{h})")
    rows = si.sample_rows(N, 12, 7)
    ref = np.zeros((len(rows), R))
    for b in range(B):
        for h in range(H):
            ref += oracle.attention_lowrank_bwd_head(q[b, h], k[b, h], v[b, h], ph, ph, g[b, h], scale, True,
                                                     rows=rows)["dphi_q"]
    grad_close(host(dpq)[rows], ref, "c7 dphi_q rows")
    keys = si.sample_rows(N, 12, 17)

    def key_part(bh):  # one head's contribution (its whole score matrix, in fp64)
        b, h = divmod(bh, H)
        return oracle.attention_lowrank_bwd_head(q[b, h], k[b, h], v[b, h], ph, ph, g[b, h], scale, True,
                                                 key_rows=keys)["dphi_k"]

    with concurrent.futures.ThreadPoolExecutor(max_workers=os.cpu_count() or 4) as pool:
        refk = sum(pool.map(key_part, range(B * H)))
    grad_close(host(dpk)[keys], refk, "c7 dphi_k rows")
    gk = host(dpk)
    assert np.all(np.isfinite(gk))
    assert np.abs(gk.sum(axis=0)).max() <= 2e-2 * np.abs(gk).max() * math.sqrt(N), "c7 dphi_k column sums"
