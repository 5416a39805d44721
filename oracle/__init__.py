"""fp64 CPU oracle for attention with an additive bias (FlashBias, arXiv 2505.12044).

TEST INFRASTRUCTURE ONLY: the test suite, the smoke check and the CPU-baseline
leg of the benchmark are the only callers. The product path never imports this
package, and this package imports nothing from the product.

The arithmetic lives in ``fb_oracle.c`` (the definition of biased attention,
the Sandwich and ALiBi biases and their exact factors). This module marshals
numpy arrays for it, and adds two things in plain numpy fp64: the truncated
SVD of a static bias (FlashBias rebuttal, reply to Reviewer xU4x, Q6: SVD
decomposition with a per-head rank), done with ``numpy.linalg.svd``;
attention with a multiplicative bias (rebuttal, reply to Reviewer BRmd, Q1
(2), its Eq. (1): the scaled scores are multiplied elementwise by b); and the
factors of the neural decomposition (rebuttal, reply to Reviewer xU4x, Q4:
linear layers on token features), a library matmul; and the gradients of
attention with a low-rank bias (the backward of the concatenated form
q' = [q, phi_q], k' = [k, phi_k], rebuttal, reply to Reviewer UJUf, Q2, used
for training in Q1 (3) and in the reply to Reviewer Bp2x, Q3).
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build as _build

BIAS_NONE, BIAS_DENSE, BIAS_LOWRANK, BIAS_SANDWICH, BIAS_ALIBI, BIAS_TOEPLITZ, BIAS_GRID = range(7)


class _Bias(ctypes.Structure):
    _fields_ = [
        ("kind", ctypes.c_int),
        ("dense", ctypes.c_void_p),
        ("ld", ctypes.c_int64),
        ("phi_q", ctypes.c_void_p),
        ("phi_k", ctypes.c_void_p),
        ("R", ctypes.c_int),
        ("C", ctypes.c_int),
        ("slope", ctypes.c_double),
        ("table", ctypes.c_void_p),
        ("n", ctypes.c_int64),
    ]


_lib = None


def _load():
    global _lib
    if _lib is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        P = ctypes.c_void_p
        lib.fbo_attention_rows.argtypes = [ctypes.c_int64, ctypes.c_int, P, P, P,
                                           ctypes.POINTER(_Bias), ctypes.c_double,
                                           ctypes.c_int, P, ctypes.c_int64, P, P]
        lib.fbo_attention_rows.restype = ctypes.c_int
        lib.fbo_bias_dense.argtypes = [ctypes.c_int64, ctypes.POINTER(_Bias), P]
        lib.fbo_bias_dense.restype = ctypes.c_int
        lib.fbo_bias_value.argtypes = [ctypes.POINTER(_Bias), ctypes.c_int64, ctypes.c_int64]
        lib.fbo_bias_value.restype = ctypes.c_double
        lib.fbo_sandwich_factors.argtypes = [ctypes.c_int64, ctypes.c_int, P]
        lib.fbo_sandwich_factors.restype = ctypes.c_int
        lib.fbo_alibi_slope.argtypes = [ctypes.c_int, ctypes.c_int]
        lib.fbo_alibi_slope.restype = ctypes.c_double
        lib.fbo_alibi_factors.argtypes = [ctypes.c_int64, ctypes.c_double, P, P]
        lib.fbo_alibi_factors.restype = ctypes.c_int
        lib.fbo_num_threads.argtypes = []
        lib.fbo_num_threads.restype = ctypes.c_int
        _lib = lib
    return _lib


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


class HeadBias:
    """The bias of one head, by kind. Keeps its arrays alive for the C call."""

    def __init__(self, kind: int, dense=None, phi_q=None, phi_k=None, C: int = 0,
                 slope: float = 0.0, table=None, n: int = 0):
        self.kind = kind
        self._keep = []
        self.s = _Bias()
        self.s.kind = kind
        if kind == BIAS_DENSE:
            dense = _f64(dense)
            self._keep.append(dense)
            self.s.dense = dense.ctypes.data
            self.s.ld = dense.shape[1]
        elif kind == BIAS_LOWRANK:
            phi_q, phi_k = _f64(phi_q), _f64(phi_k)
            assert phi_q.shape[1] == phi_k.shape[1]
            self._keep += [phi_q, phi_k]
            self.s.phi_q = phi_q.ctypes.data
            self.s.phi_k = phi_k.ctypes.data
            self.s.R = phi_q.shape[1]
        elif kind == BIAS_SANDWICH:
            self.s.C = int(C)
        elif kind == BIAS_ALIBI:
            self.s.slope = float(slope)
        elif kind in (BIAS_TOEPLITZ, BIAS_GRID):
            table = _f64(table).ravel()
            want = 2 * n - 1 if kind == BIAS_TOEPLITZ else (2 * n - 1) ** 2
            assert table.size == want
            self._keep.append(table)
            self.s.table = table.ctypes.data
            self.s.n = int(n)

    @staticmethod
    def none():
        return HeadBias(BIAS_NONE)

    @staticmethod
    def dense(b):
        return HeadBias(BIAS_DENSE, dense=b)

    @staticmethod
    def lowrank(phi_q, phi_k):
        return HeadBias(BIAS_LOWRANK, phi_q=phi_q, phi_k=phi_k)

    @staticmethod
    def sandwich(C: int):
        return HeadBias(BIAS_SANDWICH, C=C)

    @staticmethod
    def alibi(slope: float):
        return HeadBias(BIAS_ALIBI, slope=slope)

    @staticmethod
    def toeplitz(table, N: int):
        """b_ij = table[i - j + N - 1] (table over the 2N-1 offsets)."""
        return HeadBias(BIAS_TOEPLITZ, table=table, n=N)

    @staticmethod
    def grid(table, g: int):
        """b_ij = table[dx + g - 1, dy + g - 1] for tokens on a g x g grid (n = g*y + x)."""
        return HeadBias(BIAS_GRID, table=table, n=g)

    def value(self, i: int, j: int) -> float:
        return _load().fbo_bias_value(ctypes.byref(self.s), int(i), int(j))

    def dense_matrix(self, N: int) -> np.ndarray:
        out = np.empty((N, N), dtype=np.float64)
        rc = _load().fbo_bias_dense(N, ctypes.byref(self.s), _ptr(out))
        assert rc == 0
        return out


def attention_head(q, k, v, bias: HeadBias, scale: float, causal: bool, rows=None):
    """One head: q, k, v [N, d]. Returns (o [len(rows), d], lse [len(rows)]) in fp64."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    N, d = q.shape
    assert k.shape == (N, d) and v.shape == (N, d)
    rows = np.arange(N, dtype=np.int64) if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    o = np.empty((rows.shape[0], d), dtype=np.float64)
    lse = np.empty((rows.shape[0],), dtype=np.float64)
    rc = _load().fbo_attention_rows(N, d, _ptr(q), _ptr(k), _ptr(v), ctypes.byref(bias.s),
                                    float(scale), int(bool(causal)), _ptr(rows), rows.shape[0],
                                    _ptr(o), _ptr(lse))
    if rc != 0:
        raise ValueError("oracle rejected its arguments")
    return o, lse


def attention(q, k, v, bias_of, scale: float, causal: bool, rows=None, heads=None):
    """q, k, v [B, H, N, d]. ``bias_of(b, h)`` returns the HeadBias of head (b, h).

    rows: optional query indices evaluated for every head (default: all).
    heads: optional list of (b, h) pairs to evaluate (default: all).
    Returns (o, lse) as dicts keyed by (b, h) when ``heads`` is given, else as
    arrays [B, H, len(rows), d] and [B, H, len(rows)].
    """
    B, H, N, d = q.shape
    pairs = heads if heads is not None else [(b, h) for b in range(B) for h in range(H)]
    out_o, out_l = {}, {}
    for (b, h) in pairs:
        o, l = attention_head(q[b, h], k[b, h], v[b, h], bias_of(b, h), scale, causal, rows)
        out_o[(b, h)], out_l[(b, h)] = o, l
    if heads is not None:
        return out_o, out_l
    nr = N if rows is None else len(rows)
    O = np.empty((B, H, nr, d))
    L = np.empty((B, H, nr))
    for (b, h) in pairs:
        O[b, h], L[b, h] = out_o[(b, h)], out_l[(b, h)]
    return O, L


def num_threads() -> int:
    """Host threads the oracle's parallel loops use."""
    return _load().fbo_num_threads()


def sandwich_factors(N: int, C: int) -> np.ndarray:
    """Exact Sandwich factors phi [N, C] (phi_q = phi_k = phi)."""
    out = np.empty((N, C), dtype=np.float64)
    assert _load().fbo_sandwich_factors(N, C, _ptr(out)) == 0
    return out


def alibi_slope(h: int, H: int) -> float:
    return _load().fbo_alibi_slope(h, H)


def alibi_factors(N: int, slope: float):
    """Exact rank-2 ALiBi factors (phi_q [N, 2], phi_k [N, 2]) of one head."""
    pq = np.empty((N, 2), dtype=np.float64)
    pk = np.empty((N, 2), dtype=np.float64)
    assert _load().fbo_alibi_factors(N, float(slope), _ptr(pq), _ptr(pk)) == 0
    return pq, pk


def truncated_svd_factors(bias, R: int):
    """Rank-R truncation of one head's bias by SVD, split evenly between the sides.

    phi_q = U_R sqrt(S_R), phi_k = V_R sqrt(S_R), so phi_q phi_k^T is the best
    rank-R approximation (Eckart-Young). Returns (phi_q, phi_k, rel_fro_err,
    energy) with rel_fro_err = ||B - phi_q phi_k^T||_F / ||B||_F and energy =
    sum_{r<R} s_r^2 / sum_r s_r^2 (the "95% energy" criterion of the rebuttal,
    reply to Reviewer Bp2x, Q2 (2), is reported, not enforced).
    """
    Bm = _f64(bias)
    U, S, Vt = np.linalg.svd(Bm, full_matrices=False)
    root = np.sqrt(S[:R])
    phi_q = U[:, :R] * root[None, :]
    phi_k = Vt[:R, :].T * root[None, :]
    approx = phi_q @ phi_k.T
    nrm = np.linalg.norm(Bm)
    rel = float(np.linalg.norm(Bm - approx) / nrm) if nrm > 0 else 0.0
    tot = float(np.sum(S * S))
    energy = float(np.sum(S[:R] ** 2) / tot) if tot > 0 else 1.0
    return phi_q, phi_k, rel, energy


def lowrank_dense(phi_q, phi_k) -> np.ndarray:
    """phi_q phi_k^T in fp64 (the dense bias a set of factors stands for)."""
    return _f64(phi_q) @ _f64(phi_k).T


def attention_mul_head(q, k, v, phi_q, phi_k, scale: float, causal: bool, rows=None):
    """One head with a multiplicative bias b = phi_q phi_k^T (rebuttal, reply to
    Reviewer BRmd, Q1 (2), Eq. (1)): s_ij = scale * (q_i . k_j) * b_ij, then the
    softmax over the visible j (j <= i when causal) and O = P v; LSE = ln sum_j
    exp(s_ij). q, k, v [N, d]; phi_q, phi_k [N, R]. The plain definition in
    fp64, the whole score row at once. Returns (o [len(rows), d], lse)."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    N = q.shape[0]
    rows = np.arange(N, dtype=np.int64) if rows is None else np.asarray(rows, dtype=np.int64)
    b = _f64(phi_q)[rows] @ _f64(phi_k).T                    # [rows, N]
    s = float(scale) * (q[rows] @ k.T) * b
    if causal:
        s = np.where(np.arange(N)[None, :] <= rows[:, None], s, -np.inf)
    m = np.max(s, axis=1, keepdims=True)
    e = np.exp(s - m)
    l = np.sum(e, axis=1, keepdims=True)
    return (e @ v) / l, (m + np.log(l))[:, 0]


def cos_factors(N: int) -> np.ndarray:
    """The rebuttal's multiplicative example b_ij = cos(i - j): phi_q = phi_k =
    [cos i, sin i] (reply to Reviewer BRmd, Q1 (2), Example), [N, 2] fp64."""
    i = np.arange(N, dtype=np.float64)
    return np.stack([np.cos(i), np.sin(i)], axis=1)


def neural_factors(x_q, x_k, w_q, w_k):
    """Factors of the neural decomposition (rebuttal, reply to Reviewer xU4x,
    Q4: "simple linear layers"): phi_q[b, h] = x_q[b] w_q[h] and phi_k[b, h] =
    x_k[b] w_k[h] in fp64. x [B, N, F], w [H, F, R] -> phi [B, H, N, R]."""
    xq, xk, wq, wk = _f64(x_q), _f64(x_k), _f64(w_q), _f64(w_k)
    return np.einsum("bnf,hfr->bhnr", xq, wq), np.einsum("bnf,hfr->bhnr", xk, wk)


def attention_lowrank_bwd_head(q, k, v, phi_q, phi_k, do, scale: float, causal: bool, rows=None, key_rows=None):
    """Gradients of one head of O = softmax(scale q k^T + phi_q phi_k^T [causal]) v
    for an upstream gradient dO, in fp64 (the chain rule through the softmax,
    whole rows at once; library matmuls).

    The pages train with the factorised bias by concatenating the factors to
    the queries and keys (rebuttal, reply to Reviewer UJUf, Q2 and Q1 (3);
    reply to Reviewer Bp2x, Q3), so the factor gradients are the extra columns
    of the concatenated query and key gradients:
        P = softmax(s) row-wise over the visible keys, O = P v
        dV = P^T dO,  dP = dO v^T,  dS = P * (dP - rowsum(P * dP))
        dq = scale dS k,  dk = scale dS^T q,  dphi_q = dS phi_k,  dphi_k = dS^T phi_q.
    q, k, v, do [N, d]; phi_q, phi_k [N, R]. Returns a dict with dq, dk, dv,
    dphi_q, dphi_k and the intermediate rowsum(P * dP) as ``delta``. With
    ``rows`` (query indices) only the row-wise results dq, dphi_q and delta
    of those queries are computed (a query row of dS needs only its own
    score row). With ``key_rows`` (key indices) only the key-wise results dk,
    dv and dphi_k of those keys are computed: a key column of dS needs every
    row's softmax normaliser and rowsum(P * dP), taken here as rowsum(dO * O)
    (equal, since O = P v), and only the dP columns of those keys."""
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
    pq, pk = _f64(phi_q), _f64(phi_k)
    N = q.shape[0]
    if key_rows is not None:
        kr = np.asarray(key_rows, dtype=np.int64)
        s = float(scale) * (q @ k.T) + pq @ pk.T
        if causal:
            s = np.where(np.arange(N)[None, :] <= np.arange(N)[:, None], s, -np.inf)
        m = np.max(s, axis=1, keepdims=True)
        e = np.exp(s - m)
        lsum = np.sum(e, axis=1, keepdims=True)
        o = (e @ v) / lsum
        delta = np.sum(do * o, axis=1, keepdims=True)
        p_cols = e[:, kr] / lsum
        ds_cols = p_cols * (do @ v[kr].T - delta)
        return {"dk": float(scale) * (ds_cols.T @ q), "dv": p_cols.T @ do, "dphi_k": ds_cols.T @ pq}
    if rows is not None:
        rows = np.asarray(rows, dtype=np.int64)
        s = float(scale) * (q[rows] @ k.T) + pq[rows] @ pk.T
        if causal:
            s = np.where(np.arange(N)[None, :] <= rows[:, None], s, -np.inf)
        m = np.max(s, axis=1, keepdims=True)
        e = np.exp(s - m)
        p = e / np.sum(e, axis=1, keepdims=True)
        dp = do[rows] @ v.T
        delta = np.sum(p * dp, axis=1, keepdims=True)
        ds = p * (dp - delta)
        return {"dq": float(scale) * (ds @ k), "dphi_q": ds @ pk, "delta": delta[:, 0]}
    s = float(scale) * (q @ k.T) + pq @ pk.T
    if causal:
        s = np.where(np.arange(N)[None, :] <= np.arange(N)[:, None], s, -np.inf)
    m = np.max(s, axis=1, keepdims=True)
    e = np.exp(s - m)
    p = e / np.sum(e, axis=1, keepdims=True)
    dp = do @ v.T
    delta = np.sum(p * dp, axis=1, keepdims=True)
    ds = p * (dp - delta)
    return {
        "dq": float(scale) * (ds @ k),
        "dk": float(scale) * (ds.T @ q),
        "dv": p.T @ do,
        "dphi_q": ds @ pk,
        "dphi_k": ds.T @ pq,
        "delta": delta[:, 0],
    }


def neural_bwd(x_q, x_k, w_q, w_k, q, k, v, do, scale: float, causal: bool):
    """Gradients of the neural-decomposition attention (rebuttal, reply to
    Reviewer xU4x, Q4: phi_q[b, h] = x_q[b] w_q[h], phi_k[b, h] = x_k[b] w_k[h])
    for an upstream gradient do, in fp64: the factor gradients of every head
    from ``attention_lowrank_bwd_head``, then the chain rule through the linear
    layers, dw[h] = sum_b x[b]^T dphi[b, h] and dx[b] = sum_h dphi[b, h] w[h]^T.
    x [B, N, F], w [H, F, R], q, k, v, do [B, H, N, d]. Returns a dict with
    dq, dk, dv [B, H, N, d], dx_q, dx_k [B, N, F] and dw_q, dw_k [H, F, R]."""
    xq, xk, wq, wk = _f64(x_q), _f64(x_k), _f64(w_q), _f64(w_k)
    B, H, N, d = np.shape(q)
    pq, pk = neural_factors(xq, xk, wq, wk)
    out = {n: np.zeros((B, H, N, d)) for n in ("dq", "dk", "dv")}
    dpq = np.zeros(pq.shape)
    dpk = np.zeros(pk.shape)
    for b in range(B):
        for h in range(H):
            r = attention_lowrank_bwd_head(q[b, h], k[b, h], v[b, h], pq[b, h], pk[b, h], do[b, h], scale, causal)
            for n in ("dq", "dk", "dv"):
                out[n][b, h] = r[n]
            dpq[b, h], dpk[b, h] = r["dphi_q"], r["dphi_k"]
    out["dw_q"] = np.einsum("bnf,bhnr->hfr", xq, dpq)
    out["dw_k"] = np.einsum("bnf,bhnr->hfr", xk, dpk)
    out["dx_q"] = np.einsum("bhnr,hfr->bnf", dpq, wq)
    out["dx_k"] = np.einsum("bhnr,hfr->bnf", dpk, wk)
    return out
