"""Pins for the fp64 oracle: each check compares it with something other than itself.

- a library attention routine (torch SDPA, fp64 CPU) and torch.logsumexp;
- a 50-digit mpmath evaluation on tiny inputs;
- invariants of the definition (row-constant bias, zero bias, rows of P sum to
  one, key permutation, saturating scores, the first causal row);
- the closed-form identities the pages state (Sandwich bias = product of its
  exact factors; ALiBi = product of its rank-2 factors) and golden constants;
- the truncated SVD against matrices with known singular values;
- the backward against central finite differences of the forward (the C
  definition), and the invariants that rows of dS sum to zero and rows of P
  to one.
"""
import json
import math
import os

import mpmath
import numpy as np
import pytest
import torch

import oracle
from oracle import HeadBias
import seeded_inputs as si

GOLDEN = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "closed_forms.json")))


def _rand(shape, seed, std=1.0):
    return np.random.Generator(np.random.PCG64(seed)).standard_normal(shape) * std


def _sdpa(q, k, v, bias, scale, causal):
    """Library attention with an additive float mask (fp64, CPU)."""
    Q, K, V = (torch.from_numpy(np.ascontiguousarray(x))[None, None] for x in (q, k, v))
    mask = torch.from_numpy(np.ascontiguousarray(bias)).clone()
    if causal:
        N = q.shape[0]
        mask = mask.masked_fill(torch.triu(torch.ones(N, N, dtype=torch.bool), 1), float("-inf"))
    o = torch.nn.functional.scaled_dot_product_attention(Q, K, V, attn_mask=mask[None, None], scale=scale)
    scores = scale * (torch.from_numpy(q) @ torch.from_numpy(k).T) + mask
    lse = torch.logsumexp(scores, dim=-1)
    return o[0, 0].numpy(), lse.numpy()


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N,d", [(1, 4), (37, 8), (64, 16), (130, 24)])
def test_dense_bias_matches_library_attention(N, d, causal):
    q, k, v = (_rand((N, d), s) for s in (1, 2, 3))
    bias = _rand((N, N), 4, 2.0)  # asymmetric: a transposed bias would not match
    scale = 1.0 / math.sqrt(d)
    o, lse = oracle.attention_head(q, k, v, HeadBias.dense(bias), scale, causal)
    o_ref, lse_ref = _sdpa(q, k, v, bias, scale, causal)
    np.testing.assert_allclose(o, o_ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, lse_ref, rtol=0, atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_lowrank_bias_matches_library_matmul(causal):
    N, d, R = 50, 8, 5
    q, k, v = (_rand((N, d), s) for s in (5, 6, 7))
    pq, pk = _rand((N, R), 8, 0.7), _rand((N, R), 9, 0.7)
    scale = 0.3
    o, lse = oracle.attention_head(q, k, v, HeadBias.lowrank(pq, pk), scale, causal)
    o_ref, lse_ref = _sdpa(q, k, v, torch.from_numpy(pq) @ torch.from_numpy(pk).T, scale, causal)
    np.testing.assert_allclose(o, o_ref, atol=1e-12)
    np.testing.assert_allclose(lse, lse_ref, atol=1e-12)
    # the LOWRANK definition element by element against a library matmul
    dense = HeadBias.lowrank(pq, pk).dense_matrix(N)
    np.testing.assert_allclose(dense, pq @ pk.T, atol=1e-13)


def test_zero_bias_is_plain_attention():
    N, d = 40, 16
    q, k, v = (_rand((N, d), s) for s in (11, 12, 13))
    for causal in (False, True):
        o0, l0 = oracle.attention_head(q, k, v, HeadBias.none(), 0.25, causal)
        Q, K, V = (torch.from_numpy(x)[None, None] for x in (q, k, v))
        o_ref = torch.nn.functional.scaled_dot_product_attention(Q, K, V, is_causal=causal, scale=0.25)[0, 0]
        np.testing.assert_allclose(o0, o_ref.numpy(), atol=1e-12)
        od, ld = oracle.attention_head(q, k, v, HeadBias.dense(np.zeros((N, N))), 0.25, causal)
        np.testing.assert_array_equal(o0, od)
        np.testing.assert_array_equal(l0, ld)


def _mp_attention_row(q, k, v, bias, scale, i, causal):
    jmax = i + 1 if causal else k.shape[0]
    s = [mpmath.mpf(scale) * mpmath.fsum(mpmath.mpf(q[i, c]) * mpmath.mpf(k[j, c]) for c in range(q.shape[1]))
         + mpmath.mpf(bias[i, j]) for j in range(jmax)]
    e = [mpmath.exp(x) for x in s]
    z = mpmath.fsum(e)
    o = [mpmath.fsum(e[j] * mpmath.mpf(v[j, c]) for j in range(jmax)) / z for c in range(v.shape[1])]
    return o, mpmath.log(z)


@pytest.mark.parametrize("causal", [False, True])
def test_fifty_digit_bruteforce(causal):
    mpmath.mp.dps = 50
    N, d = 12, 4
    q, k, v = (_rand((N, d), s) for s in (21, 22, 23))
    bias = _rand((N, N), 24, 3.0)
    o, lse = oracle.attention_head(q, k, v, HeadBias.dense(bias), 0.7, causal)
    for i in range(N):
        o_mp, l_mp = _mp_attention_row(q, k, v, bias, 0.7, i, causal)
        for c in range(d):
            assert abs(o[i, c] - float(o_mp[c])) < 1e-13
        assert abs(lse[i] - float(l_mp)) < 1e-13 * max(1.0, abs(float(l_mp)))


def test_row_constant_bias_leaves_output_and_shifts_lse():
    N, d = 33, 8
    q, k, v = (_rand((N, d), s) for s in (31, 32, 33))
    c = _rand((N,), 34, 5.0)
    for causal in (False, True):
        o0, l0 = oracle.attention_head(q, k, v, HeadBias.none(), 0.5, causal)
        o1, l1 = oracle.attention_head(q, k, v, HeadBias.dense(np.repeat(c[:, None], N, 1)), 0.5, causal)
        np.testing.assert_allclose(o1, o0, atol=1e-14)
        np.testing.assert_allclose(l1 - l0, c, atol=1e-12)


def test_rows_of_p_sum_to_one_and_first_causal_row():
    N, d = 29, 6
    q, k = _rand((N, d), 41), _rand((N, d), 42)
    v = np.ones((N, d))
    bias = _rand((N, N), 43, 4.0)
    o, _ = oracle.attention_head(q, k, v, HeadBias.dense(bias), 1.0, False)
    np.testing.assert_allclose(o, 1.0, atol=1e-14 * N)
    v = _rand((N, d), 44)
    o, lse = oracle.attention_head(q, k, v, HeadBias.dense(bias), 1.0, True)
    np.testing.assert_array_equal(o[0], v[0])  # causal row 0 sees key 0 only
    assert abs(lse[0] - (q[0] @ k[0] + bias[0, 0])) < 1e-14


def test_key_permutation_equivariance():
    N, d = 31, 8
    q, k, v = (_rand((N, d), s) for s in (51, 52, 53))
    bias = _rand((N, N), 54)
    perm = np.random.Generator(np.random.PCG64(55)).permutation(N)
    o, l = oracle.attention_head(q, k, v, HeadBias.dense(bias), 0.4, False)
    op, lp = oracle.attention_head(q, k[perm], v[perm], HeadBias.dense(bias[:, perm]), 0.4, False)
    np.testing.assert_allclose(op, o, atol=1e-13)
    np.testing.assert_allclose(lp, l, atol=1e-13)


def test_saturating_scores_pick_one_key():
    N, d = 20, 4
    q, k, v = (_rand((N, d), s) for s in (61, 62, 63))
    bias = np.zeros((N, N))
    bias[:, 7] = 1.0e4  # exp would overflow without the max shift
    o, lse = oracle.attention_head(q, k, v, HeadBias.dense(bias), 1.0, False)
    np.testing.assert_allclose(o, np.repeat(v[7:8], N, 0), atol=1e-300)
    np.testing.assert_allclose(lse, q @ k[7] + 1.0e4, rtol=1e-15)


# --- Sandwich ---------------------------------------------------------------

def test_sandwich_identity_bias_equals_factor_product():
    """The pages state b = phi_q phi_k^T for the exact Sandwich factors."""
    C, N = 64, 2048
    phi = oracle.sandwich_factors(N, C)
    bias = HeadBias.sandwich(C)
    rng = np.random.Generator(np.random.PCG64(70))
    pairs = [(0, 0), (N - 1, 0), (0, N - 1), (N - 1, N - 1)] + [tuple(x) for x in rng.integers(0, N, (300, 2))]
    for i, j in pairs:
        assert abs(bias.value(i, j) - float(phi[i] @ phi[j])) < 1e-11
    # whole small block through the dense builder as well
    Bd = HeadBias.sandwich(16).dense_matrix(300)
    f16 = oracle.sandwich_factors(300, 16)
    np.testing.assert_allclose(Bd, f16 @ f16.T, atol=1e-12)


def test_sandwich_golden_values():
    g = GOLDEN
    b = HeadBias.sandwich(g["sandwich_diagonal"]["C"])
    for i in (0, 5, 4095):
        assert b.value(i, i) == g["sandwich_diagonal"]["value"]
    for delta, val in g["sandwich_delta"]["points"]:
        assert abs(b.value(delta + 3, 3) - val) < 1e-12
        assert abs(b.value(3, delta + 3) - val) < 1e-12  # even in i - j
    phi = oracle.sandwich_factors(2, 64)
    assert abs(math.acos(phi[1, 0]) - g["sandwich_w1"]["value"]) < 1e-14
    assert abs(math.atan2(phi[1, 63], phi[1, 62]) - g["sandwich_w_last"]["value"]) < 1e-16
    np.testing.assert_array_equal(oracle.sandwich_factors(1, 8)[0], g["sandwich_phi_at_zero"]["value"])


# --- ALiBi ------------------------------------------------------------------

def test_alibi_slopes_golden():
    for key in ("alibi_slopes_H8", "alibi_slopes_H16"):
        H = GOLDEN[key]["H"]
        got = [oracle.alibi_slope(h, H) for h in range(H)]
        np.testing.assert_allclose(got, GOLDEN[key]["value"], rtol=1e-15)


def test_alibi_factor_product_is_distance_bias():
    N = 8192
    for h, H in ((0, 16), (7, 16), (15, 16), (3, 8)):
        m = oracle.alibi_slope(h, H)
        pq, pk = oracle.alibi_factors(N, m)
        bias = HeadBias.alibi(m)
        rng = np.random.Generator(np.random.PCG64(80 + h))
        for i, j in [(0, 0), (N - 1, 0), (N - 1, N - 1), (5, 9)] + [tuple(x) for x in rng.integers(0, N, (200, 2))]:
            want = -m * (i - j)
            assert abs(float(pq[i] @ pk[j]) - want) <= 1e-9 * max(1.0, abs(want))
            assert bias.value(i, j) == want


def test_multiplicative_example_rank2():
    """cos(i-j) = [cos i, sin i].[cos j, sin j] (the pages' rank-2 example)."""
    n = np.arange(64, dtype=np.float64)
    f = np.stack([np.cos(n), np.sin(n)], 1)
    np.testing.assert_allclose(f @ f.T, np.cos(n[:, None] - n[None, :]), atol=1e-13)
    assert np.linalg.matrix_rank(np.cos(n[:, None] - n[None, :])) == GOLDEN["multiplicative_cos_rank2"]["R"]


# --- truncated SVD ----------------------------------------------------------

def _known_spectrum(N, sigma, seed):
    rng = np.random.Generator(np.random.PCG64(seed))
    U, _ = np.linalg.qr(rng.standard_normal((N, len(sigma))))
    V, _ = np.linalg.qr(rng.standard_normal((N, len(sigma))))
    return U @ np.diag(sigma) @ V.T


def test_svd_truncation_against_known_spectrum():
    sigma = np.array([50.0, 20.0, 9.0, 4.0, 2.0, 1.0, 0.5, 0.25])
    Bm = _known_spectrum(200, sigma, 90)
    for R in (1, 3, 8):
        pq, pk, rel, energy = oracle.truncated_svd_factors(Bm, R)
        want_rel = math.sqrt(np.sum(sigma[R:] ** 2) / np.sum(sigma ** 2))
        want_energy = np.sum(sigma[:R] ** 2) / np.sum(sigma ** 2)
        assert abs(rel - want_rel) < 1e-12
        assert abs(energy - want_energy) < 1e-12
        # balanced split: phi_q^T phi_q = phi_k^T phi_k = diag(sigma_R)
        np.testing.assert_allclose(pq.T @ pq, np.diag(sigma[:R]), atol=1e-10)
        np.testing.assert_allclose(pk.T @ pk, np.diag(sigma[:R]), atol=1e-10)
    pq, pk, rel, _ = oracle.truncated_svd_factors(Bm, 8)
    np.testing.assert_allclose(pq @ pk.T, Bm, atol=1e-11)
    assert rel < 1e-12


# --- seeded inputs (the workload definitions both sides receive) ------------

def test_rbf_field_rank_and_gather():
    grid, M = 12, 6
    om, ph = si.rbf_params(2, M)
    tab = si.rbf_offset_table(om, ph, grid)
    dense = si.rbf_dense(tab, grid)
    assert dense.shape == (2, grid * grid, grid * grid)
    for h in range(2):
        assert np.linalg.matrix_rank(dense[h], tol=1e-9 * np.abs(dense[h]).max()) <= 2 * M
        for (i, j) in [(0, 0), (5, 77), (143, 3)]:
            dx = i % grid - j % grid
            dy = i // grid - j // grid
            want = math.sqrt(2.0 / M) * sum(math.cos(om[h, m, 0] * dx + om[h, m, 1] * dy + ph[h, m]) for m in range(M))
            assert abs(dense[h, i, j] - want) < 1e-12


def test_bf16_rounding_is_round_to_nearest_even():
    x = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.5, 1e-3, 65504.0], dtype=np.float32)
    r = si.round_to_bf16(x)
    t = torch.from_numpy(x).to(torch.bfloat16).to(torch.float32).numpy()
    np.testing.assert_array_equal(r, t)
    y = si.normal((4096,), 5)
    np.testing.assert_array_equal(si.round_to_bf16(y), torch.from_numpy(y).to(torch.bfloat16).float().numpy())


def test_offset_table_kinds():
    """TOEPLITZ and GRID biases: the offset-table forms of the dense inputs."""
    N, C = 200, 16
    tab = si.sandwich_offset_table(N, C)
    tb = HeadBias.toeplitz(tab, N)
    sw = HeadBias.sandwich(C)
    for i, j in [(0, 0), (199, 0), (0, 199), (57, 123)]:
        assert abs(tb.value(i, j) - sw.value(i, j)) < 1e-12
    np.testing.assert_array_equal(tb.dense_matrix(N), si.toeplitz_rows(tab, N, np.arange(N)))
    m = oracle.alibi_slope(2, 8)
    ta = HeadBias.toeplitz(si.alibi_offset_table(N, m), N)
    for i, j in [(0, 0), (199, 0), (5, 9)]:
        assert ta.value(i, j) == HeadBias.alibi(m).value(i, j)
    g = 9
    om, ph = si.rbf_params(1, 4)
    t2 = si.rbf_offset_table(om, ph, g)
    np.testing.assert_array_equal(HeadBias.grid(t2[0], g).dense_matrix(g * g), si.rbf_dense(t2, g)[0])


# --- multiplicative bias (rebuttal, reply to Reviewer BRmd, Q1 (2)) ---------

@pytest.mark.parametrize("causal", [False, True])
def test_multiplicative_unit_bias_is_plain_attention(causal):
    """b = 1 (phi_q = phi_k = [1]): the multiplicative form is plain attention,
    checked against torch SDPA; an additive reading would shift the LSE by 1."""
    N, d = 40, 8
    q, k, v = (_rand((N, d), s) for s in (31, 32, 33))
    ones = np.ones((N, 1))
    o, lse = oracle.attention_mul_head(q, k, v, ones, ones, 0.35, causal)
    o_ref, lse_ref = _sdpa(q, k, v, np.zeros((N, N)), 0.35, causal)
    np.testing.assert_allclose(o, o_ref, atol=1e-12)
    np.testing.assert_allclose(lse, lse_ref, atol=1e-12)


def _mp_mul_row(q, k, v, pq, pk, scale, i, causal):
    jmax = i + 1 if causal else q.shape[0]
    s = [mpmath.mpf(scale) * mpmath.fsum(mpmath.mpf(q[i, c]) * mpmath.mpf(k[j, c]) for c in range(q.shape[1]))
         * mpmath.fsum(mpmath.mpf(pq[i, r]) * mpmath.mpf(pk[j, r]) for r in range(pq.shape[1])) for j in range(jmax)]
    m = max(s)
    e = [mpmath.exp(x - m) for x in s]
    z = mpmath.fsum(e)
    o = [mpmath.fsum(e[j] * mpmath.mpf(v[j, c]) for j in range(jmax)) / z for c in range(v.shape[1])]
    return o, m + mpmath.log(z)


@pytest.mark.parametrize("causal", [False, True])
def test_multiplicative_fifty_digit_bruteforce(causal):
    """Loops over i, j, c, r at 50 digits, with phi_q != phi_k so that b_ij and
    b_ji differ (a transposed bias fails)."""
    mpmath.mp.dps = 50
    N, d, R = 10, 4, 3
    q, k, v = (_rand((N, d), s) for s in (41, 42, 43))
    pq, pk = _rand((N, R), 44), _rand((N, R), 45)
    o, lse = oracle.attention_mul_head(q, k, v, pq, pk, 0.6, causal)
    for i in range(N):
        o_mp, l_mp = _mp_mul_row(q, k, v, pq, pk, 0.6, i, causal)
        for c in range(d):
            assert abs(o[i, c] - float(o_mp[c])) < 1e-13
        assert abs(lse[i] - float(l_mp)) < 1e-13 * max(1.0, abs(float(l_mp)))


def test_multiplicative_cos_example_closed_form():
    """The pages' example b_ij = cos(i - j) from its rank-2 factors, against the
    scores built from np.cos(i - j) directly and a library softmax."""
    N, d = 50, 8
    q, k, v = (_rand((N, d), s) for s in (51, 52, 53))
    f = oracle.cos_factors(N)
    o, lse = oracle.attention_mul_head(q, k, v, f, f, 0.5, True)
    n = np.arange(N, dtype=np.float64)
    s = 0.5 * (q @ k.T) * np.cos(n[:, None] - n[None, :])
    s = np.where(n[None, :] <= n[:, None], s, -np.inf)
    st = torch.from_numpy(s)
    np.testing.assert_allclose(lse, torch.logsumexp(st, dim=-1).numpy(), atol=1e-12)
    np.testing.assert_allclose(o, (torch.softmax(st, dim=-1) @ torch.from_numpy(v)).numpy(), atol=1e-12)


def test_neural_factors_are_the_linear_layers():
    """phi = x w per (batch, head), against explicit loops over n, f, r."""
    rng = np.random.Generator(np.random.PCG64(81))
    B, H, N, F, R = 2, 3, 5, 4, 2
    xq, xk = rng.standard_normal((B, N, F)), rng.standard_normal((B, N, F))
    wq, wk = rng.standard_normal((H, F, R)), rng.standard_normal((H, F, R))
    pq, pk = oracle.neural_factors(xq, xk, wq, wk)
    for b in range(B):
        for h in range(H):
            for n in range(N):
                for r in range(R):
                    assert abs(pq[b, h, n, r] - sum(xq[b, n, f] * wq[h, f, r] for f in range(F))) < 1e-12
                    assert abs(pk[b, h, n, r] - sum(xk[b, n, f] * wk[h, f, r] for f in range(F))) < 1e-12


def _fd_loss(q, k, v, pq, pk, g, scale, causal):
    o, _ = oracle.attention_head(q, k, v, HeadBias.lowrank(pq, pk), scale, causal)
    return float(np.sum(o * g))


@pytest.mark.parametrize("causal", [False, True])
def test_backward_matches_finite_differences(causal):
    """Every gradient against a central difference of the forward definition
    (the C oracle, not the numpy backward): a dropped term, a transposed
    operand or a wrong scale in any of the five gradients fails here."""
    N, d, R = 6, 3, 2
    q, k, v = (_rand((N, d), s) for s in (41, 42, 43))
    pq, pk = _rand((N, R), 44, 0.8), _rand((N, R), 45, 0.8)
    g = _rand((N, d), 46)
    scale = 0.7
    grads = oracle.attention_lowrank_bwd_head(q, k, v, pq, pk, g, scale, causal)
    args = {"dq": q, "dk": k, "dv": v, "dphi_q": pq, "dphi_k": pk}
    h = 1e-6
    for name, x in args.items():
        fd = np.empty_like(x)
        for idx in np.ndindex(x.shape):
            x0 = x[idx]
            x[idx] = x0 + h
            up = _fd_loss(q, k, v, pq, pk, g, scale, causal)
            x[idx] = x0 - h
            dn = _fd_loss(q, k, v, pq, pk, g, scale, causal)
            x[idx] = x0
            fd[idx] = (up - dn) / (2 * h)
        np.testing.assert_allclose(grads[name], fd, rtol=0, atol=2e-8, err_msg=name)


@pytest.mark.parametrize("causal", [False, True])
def test_backward_invariants(causal):
    """Rows of dS sum to zero (the softmax is invariant to a per-row shift),
    so the key and phi_k gradients sum to zero over the keys and a constant
    phi_k column gets a zero phi_q gradient; rows of P sum to one, so the
    value gradients sum to the sum of dO."""
    N, d, R = 40, 8, 4
    q, k, v = (_rand((N, d), s) for s in (51, 52, 53))
    pq, pk = _rand((N, R), 54), _rand((N, R), 55)
    pk[:, 2] = 1.5
    g = _rand((N, d), 56)
    out = oracle.attention_lowrank_bwd_head(q, k, v, pq, pk, g, 0.35, causal)
    np.testing.assert_allclose(out["dk"].sum(axis=0), 0.0, atol=1e-12)
    np.testing.assert_allclose(out["dphi_k"].sum(axis=0), 0.0, atol=1e-12)
    np.testing.assert_allclose(out["dphi_q"][:, 2], 0.0, atol=1e-12)
    np.testing.assert_allclose(out["dv"].sum(axis=0), g.sum(axis=0), atol=1e-12)
    o, _ = oracle.attention_head(q, k, v, HeadBias.lowrank(pq, pk), 0.35, causal)
    np.testing.assert_allclose(out["delta"], np.sum(o * g, axis=1), atol=1e-12)
    if causal:  # the first query sees only key 0: its dS row is zero
        np.testing.assert_allclose(out["dq"][0], 0.0, atol=1e-15)


@pytest.mark.parametrize("causal", [False, True])
def test_backward_row_subset_matches_whole_head(causal):
    """The row-restricted backward (dq, dphi_q, delta of chosen queries) is the
    same computation on fewer score rows, and the key-restricted one (dk, dv,
    dphi_k of chosen keys) takes rowsum(P dP) as rowsum(dO O): both must agree
    with the whole head."""
    N, d, R = 70, 8, 3
    q, k, v = (_rand((N, d), s) for s in (61, 62, 63))
    pq, pk = _rand((N, R), 64), _rand((N, R), 65)
    g = _rand((N, d), 66)
    full = oracle.attention_lowrank_bwd_head(q, k, v, pq, pk, g, 0.4, causal)
    rows = np.array([0, 5, 33, 69])
    part = oracle.attention_lowrank_bwd_head(q, k, v, pq, pk, g, 0.4, causal, rows=rows)
    for key in ("dq", "dphi_q", "delta"):
        np.testing.assert_allclose(part[key], full[key][rows], rtol=0, atol=1e-13)
    # the key-row form (its rowsum term through rowsum(dO * O)) against the whole head
    keys = np.array([0, 4, 33, 69])
    kpart = oracle.attention_lowrank_bwd_head(q, k, v, pq, pk, g, 0.4, causal, key_rows=keys)
    for key in ("dk", "dv", "dphi_k"):
        np.testing.assert_allclose(kpart[key], full[key][keys], rtol=0, atol=1e-12)


def test_neural_backward_matches_finite_differences():
    """Gradients of the linear layers of the neural decomposition against a
    central difference of the forward definition (the factors as library
    matmuls of the features and weights, attention by the C oracle)."""
    B, H, N, d, F, R = 1, 2, 5, 3, 3, 2
    xq, xk = _rand((B, N, F), 71, 0.7), _rand((B, N, F), 72, 0.7)
    wq, wk = _rand((H, F, R), 73, 0.7), _rand((H, F, R), 74, 0.7)
    q, k, v = (_rand((B, H, N, d), s) for s in (75, 76, 77))
    g = _rand((B, H, N, d), 78)
    scale = 0.6

    def loss():
        pq, pk = np.einsum("bnf,hfr->bhnr", xq, wq), np.einsum("bnf,hfr->bhnr", xk, wk)
        tot = 0.0
        for b in range(B):
            for h in range(H):
                o, _ = oracle.attention_head(q[b, h], k[b, h], v[b, h], HeadBias.lowrank(pq[b, h], pk[b, h]),
                                             scale, True)
                tot += float(np.sum(o * g[b, h]))
        return tot

    out = oracle.neural_bwd(xq, xk, wq, wk, q, k, v, g, scale, True)
    step = 1e-6
    for name, x in (("dx_q", xq), ("dx_k", xk), ("dw_q", wq), ("dw_k", wk)):
        fd = np.empty_like(x)
        for idx in np.ndindex(x.shape):
            x0 = x[idx]
            x[idx] = x0 + step
            up = loss()
            x[idx] = x0 - step
            dn = loss()
            x[idx] = x0
            fd[idx] = (up - dn) / (2 * step)
        np.testing.assert_allclose(out[name], fd, rtol=0, atol=5e-8, err_msg=name)


def test_backward_single_key_closed_form():
    """One key: P = 1 whatever the scores, so dV = dO and every score
    gradient (dq, dk, dphi_q, dphi_k) is exactly zero."""
    q, k, v = (_rand((1, 4), s) for s in (81, 82, 83))
    pq, pk = _rand((1, 2), 84), _rand((1, 2), 85)
    g = _rand((1, 4), 86)
    out = oracle.attention_lowrank_bwd_head(q, k, v, pq, pk, g, 0.5, True)
    np.testing.assert_array_equal(out["dv"], g)
    for name in ("dq", "dk", "dphi_q", "dphi_k"):
        np.testing.assert_array_equal(out[name], 0.0)


@pytest.mark.parametrize("causal", [False, True])
def test_backward_uniform_attention_by_loops(causal):
    """q = 0 and a zero bias give uniform attention over the visible keys,
    P_ij = 1 / n_i. The gradients then follow from the definition alone,
    written here as plain loops: dv_j = sum_i dO_i / n_i, and with
    dP_ij = dO_i . v_j, dS_ij = (dP_ij - mean_j dP_ij) / n_i,
    dq_i = scale sum_j dS_ij k_j, dk_j = scale sum_i dS_ij q_i = 0."""
    N, d, R = 7, 3, 2
    q = np.zeros((N, d))
    k, v = _rand((N, d), 91), _rand((N, d), 92)
    pq, pk = np.zeros((N, R)), _rand((N, R), 93)
    g = _rand((N, d), 94)
    scale = 0.8
    out = oracle.attention_lowrank_bwd_head(q, k, v, pq, pk, g, scale, causal)
    dv = np.zeros((N, d))
    dq = np.zeros((N, d))
    dphi_q = np.zeros((N, R))
    for i in range(N):
        vis = list(range(i + 1)) if causal else list(range(N))
        n = len(vis)
        dp = [float(np.dot(g[i], v[j])) for j in vis]
        mean = sum(dp) / n
        for t, j in enumerate(vis):
            dv[j] += g[i] / n
            ds = (dp[t] - mean) / n
            dq[i] += scale * ds * k[j]
            dphi_q[i] += ds * pk[j]
    np.testing.assert_allclose(out["dv"], dv, rtol=0, atol=1e-13)
    np.testing.assert_allclose(out["dq"], dq, rtol=0, atol=1e-13)
    np.testing.assert_allclose(out["dphi_q"], dphi_q, rtol=0, atol=1e-13)
    np.testing.assert_allclose(out["dk"], 0.0, atol=1e-15)
    np.testing.assert_allclose(out["dphi_k"], 0.0, atol=1e-15)


@pytest.mark.parametrize("mistake", ["dk_without_scale", "delta_dropped", "factor_grads_swapped", "dv_untransposed"])
def test_backward_pin_catches_planted_mistakes(mistake, monkeypatch):
    """Each plausible slip in the backward (a dropped scale, the rowsum term
    left out, the two factor gradients exchanged, P instead of P^T for dV),
    planted in the oracle on the CPU, fails the finite-difference pin."""
    true_bwd = oracle.attention_lowrank_bwd_head

    def planted(q, k, v, pq, pk, do, scale, causal, rows=None):
        r = true_bwd(q, k, v, pq, pk, do, scale, causal)
        if mistake == "dk_without_scale":
            r["dk"] = r["dk"] / scale
        elif mistake == "delta_dropped":
            N = np.shape(q)[0]
            s = scale * (np.asarray(q) @ np.asarray(k).T) + np.asarray(pq) @ np.asarray(pk).T
            if causal:
                s = np.where(np.arange(N)[None, :] <= np.arange(N)[:, None], s, -np.inf)
            p = np.exp(s - s.max(axis=1, keepdims=True))
            p /= p.sum(axis=1, keepdims=True)
            ds = p * (np.asarray(do) @ np.asarray(v).T)  # the - rowsum(P dP) term left out
            r["dq"] = scale * ds @ np.asarray(k)
        elif mistake == "factor_grads_swapped":
            r["dphi_q"], r["dphi_k"] = r["dphi_k"], r["dphi_q"]
        else:
            N = np.shape(q)[0]
            s = scale * (np.asarray(q) @ np.asarray(k).T) + np.asarray(pq) @ np.asarray(pk).T
            if causal:
                s = np.where(np.arange(N)[None, :] <= np.arange(N)[:, None], s, -np.inf)
            p = np.exp(s - s.max(axis=1, keepdims=True))
            p /= p.sum(axis=1, keepdims=True)
            r["dv"] = p @ np.asarray(do)
        return r

    monkeypatch.setattr(oracle, "attention_lowrank_bwd_head", planted)
    with pytest.raises(AssertionError):
        test_backward_matches_finite_differences(True)
