"""Seeded synthetic inputs shared by the tests, the smoke check and the benchmark.

This module holds no step of the attention method: it only draws random
numbers, rounds them to the storage type the GPU path reads, and lays out the
synthetic biases that the workloads define (the smooth spatial field of the
vision-style workload is a workload definition, not a step of FlashBias).
Both the oracle and the CUDA path receive exactly these values.

Workloads (restated from the benchmark definitions; the FlashBias pages use
GPT-2, Swin, AlphaFold 3 and PDE solvers, which need trained models and
datasets, so these seeded shapes stand in for them):

  0  fp32, B=1,  H=2,  N=256,  d=64,  no mask, random rank-8 factors ~ N(0, 1/8)
  1  bf16, B=8,  H=12, N=2048, d=64,  causal, Sandwich bias, exact rank 64
  2  bf16, B=4,  H=16, N=8192, d=128, causal, ALiBi, exact rank 2
  3  bf16, B=4,  H=8,  N=4096, d=16,  no mask, RBF random-Fourier spatial field
     on a 64 x 64 token grid, truncated by SVD to rank 8
  4  bf16, B=1,  H=16, N=1536, d=24,  no mask, random rank-32 factors ~ N(0, 1/32)
"""
from __future__ import annotations

import math

import numpy as np

CONFIGS = [
    dict(index=0, name="fp32_lowrank8_N256", dtype="f32", B=1, H=2, N=256, d=64, R=8,
         causal=False, bias="lowrank", factor_std=math.sqrt(1.0 / 8.0)),
    dict(index=1, name="gpt2_sandwich_N2048", dtype="bf16", B=8, H=12, N=2048, d=64, R=64,
         causal=True, bias="sandwich"),
    dict(index=2, name="alibi_N8192_d128", dtype="bf16", B=4, H=16, N=8192, d=128, R=2,
         causal=True, bias="alibi"),
    dict(index=3, name="vision_rbf_svd_N4096_d16", dtype="bf16", B=4, H=8, N=4096, d=16, R=8,
         causal=False, bias="rbf_svd", grid=64, rbf_terms=32),
    dict(index=4, name="af3_pair_lowrank32_N1536_d24", dtype="bf16", B=1, H=16, N=1536, d=24,
         R=32, causal=False, bias="lowrank", factor_std=math.sqrt(1.0 / 32.0)),
    # multiplicative bias b_ij = cos(i - j) (rank 2) on the GPT-2 shape: a widening case, not a headline
    dict(index=5, name="gpt2_mulcos_N2048", dtype="bf16", B=8, H=12, N=2048, d=64, R=2,
         causal=True, bias="mulcos"),
    # neural decomposition: factors from per-head linear layers on token features (F = 64) on the
    # pair-bias shape: a widening case, not a headline
    dict(index=6, name="af3_neural_F64_R32_N1536_d24", dtype="bf16", B=1, H=16, N=1536, d=24, R=32,
         causal=False, bias="neural", F=64),
    # the backward (training) pass on the GPT-2 Sandwich shape: a widening case, not a headline
    dict(index=7, name="gpt2_sandwich_bwd_N2048", dtype="bf16", B=8, H=12, N=2048, d=64, R=64,
         causal=True, bias="sandwich", bwd=True),
]

QKV_SEED_BASE = 1000
FACTOR_SEED_BASE = 2000
RBF_SEED_BASE = 3000
DO_SEED_BASE = 4000


def generator(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed))


def round_to_bf16(x: np.ndarray) -> np.ndarray:
    """Round fp32 values to the nearest bf16 (ties to even); returns fp32 holding them."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    r = (u + np.uint32(0x7FFF) + lsb) & np.uint32(0xFFFF0000)
    return r.view(np.float32)


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """uint16 bf16 encodings of values that are already bf16-representable."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    assert not np.any(u & np.uint32(0xFFFF)), "values are not bf16-representable"
    return (u >> np.uint32(16)).astype(np.uint16)


def normal(shape, seed: int, std: float = 1.0) -> np.ndarray:
    g = generator(seed)
    x = g.standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        x *= np.float32(std)
    return x


def qkv(B: int, H: int, N: int, d: int, seed: int, dtype: str):
    """Q, K, V ~ N(0, 1), fp32 arrays [B, H, N, d]; rounded to bf16 values for bf16."""
    g = generator(seed)
    out = []
    for _ in range(3):
        x = g.standard_normal(size=(B, H, N, d), dtype=np.float32)
        out.append(round_to_bf16(x) if dtype == "bf16" else x)
    return tuple(out)


def random_factors(shape, std: float, seed: int):
    """Two independent fp32 factor tensors ~ N(0, std^2) of the given shape."""
    g = generator(seed)
    pq = g.standard_normal(size=shape, dtype=np.float32) * np.float32(std)
    pk = g.standard_normal(size=shape, dtype=np.float32) * np.float32(std)
    return pq, pk


def neural_inputs(B: int, H: int, N: int, F: int, R: int, seed: int):
    """Token features x_q, x_k ~ N(0, 1) [B, N, F] and linear-layer weights
    w_q ~ N(0, 1/(F R)), w_k ~ N(0, 1/F) [H, F, R], fp32 (synthetic weights;
    the bias phi_q phi_k^T then has entries of order 1)."""
    g = generator(seed)
    xq = g.standard_normal(size=(B, N, F), dtype=np.float32)
    xk = g.standard_normal(size=(B, N, F), dtype=np.float32)
    wq = g.standard_normal(size=(H, F, R), dtype=np.float32) * np.float32(1.0 / math.sqrt(F * R))
    wk = g.standard_normal(size=(H, F, R), dtype=np.float32) * np.float32(1.0 / math.sqrt(F))
    return xq, xk, wq, wk


# --- vision-style smooth spatial bias (workload 3) -------------------------
#
# Tokens sit on a g x g grid, token n = g*y + x. Head h has the random Fourier
# field  f_h(dx, dy) = sqrt(2/M) sum_m cos(w_{h,m} . (dx, dy) + u_{h,m}),
# w ~ N(0, I / l_h^2), u ~ U[0, 2 pi), l_h = 4 + 2h grid units, M terms, seed
# 3000 + h. Its covariance over draws is a Gaussian RBF kernel of the offset,
# which is why the workload calls it an RBF field. b_ij = f_h(x_i - x_j,
# y_i - y_j). It has exact rank <= 2M.

def rbf_params(H: int, M: int = 32, seed_base: int = RBF_SEED_BASE):
    omega = np.empty((H, M, 2), dtype=np.float64)
    phase = np.empty((H, M), dtype=np.float64)
    for h in range(H):
        g = generator(seed_base + h)
        ell = 4.0 + 2.0 * h
        omega[h] = g.standard_normal(size=(M, 2)) / ell
        phase[h] = g.uniform(0.0, 2.0 * math.pi, size=M)
    return omega, phase


def rbf_offset_table(omega: np.ndarray, phase: np.ndarray, grid: int) -> np.ndarray:
    """f_h on every offset: [H, 2g-1, 2g-1], index [h, dx + g - 1, dy + g - 1]."""
    H, M, _ = omega.shape
    off = np.arange(-(grid - 1), grid, dtype=np.float64)
    dx, dy = np.meshgrid(off, off, indexing="ij")
    tab = np.zeros((H, off.size, off.size), dtype=np.float64)
    for h in range(H):
        for m in range(M):
            tab[h] += np.cos(omega[h, m, 0] * dx + omega[h, m, 1] * dy + phase[h, m])
    return tab * math.sqrt(2.0 / M)


def grid_offset_index(grid: int):
    """Per token pair (i, j) of the g*g tokens: table indices (dx+g-1, dy+g-1)."""
    n = np.arange(grid * grid)
    x, y = n % grid, n // grid
    ix = x[:, None] - x[None, :] + grid - 1
    iy = y[:, None] - y[None, :] + grid - 1
    return ix, iy


def rbf_dense(table: np.ndarray, grid: int, heads=None) -> np.ndarray:
    """Dense per-head field [H, N, N] (fp64) gathered from the offset table."""
    ix, iy = grid_offset_index(grid)
    hs = range(table.shape[0]) if heads is None else heads
    return np.stack([table[h][ix, iy] for h in hs])


def sample_rows(N: int, count: int, seed: int) -> np.ndarray:
    """Sorted distinct query rows, always including the first and last row."""
    g = generator(seed)
    count = min(count, N)
    rows = set([0, N - 1])
    if count > 2:
        rows.update(g.choice(N, size=count - 2, replace=False).tolist())
    return np.array(sorted(rows), dtype=np.int64)


# --- dense biases for the comparison path -----------------------------------
#
# The dense-bias path reads a materialised bias. For biases that depend only
# on i - j (Sandwich, ALiBi) the workload builds a table over the 2N-1
# offsets, rounds it to bf16 once, and lays the N x N matrix out on the device
# by pure data movement (a strided view and a copy), so host and device hold
# bit-identical values.

def sandwich_offset_table(N: int, C: int) -> np.ndarray:
    """f(delta) = sum_{k=1}^{C/2} cos(delta / 10000^{2k/C}) for delta = -(N-1)..N-1 (fp64)."""
    delta = np.arange(-(N - 1), N, dtype=np.float64)
    k = np.arange(1, C // 2 + 1, dtype=np.float64)
    w = np.power(10000.0, -2.0 * k / C)
    return np.cos(delta[:, None] * w[None, :]).sum(axis=1)


def alibi_offset_table(N: int, slope: float) -> np.ndarray:
    """f(delta) = -m * delta for delta = -(N-1)..N-1 (fp64)."""
    return -slope * np.arange(-(N - 1), N, dtype=np.float64)


def toeplitz_rows(table: np.ndarray, N: int, rows) -> np.ndarray:
    """Rows of the N x N matrix M[i, j] = table[i - j + N - 1] (host)."""
    rows = np.asarray(rows)
    j = np.arange(N)
    return table[rows[:, None] - j[None, :] + N - 1]


def toeplitz_device(table_bf16: np.ndarray, N: int, device):
    """N x N bf16 device matrix M[i, j] = table[i - j + N - 1] by data movement only."""
    import torch
    bits = torch.from_numpy(bf16_bits(table_bf16).view(np.int16)).to(device)
    t = bits.view(torch.bfloat16)
    w = torch.flip(t, dims=[0])  # w[k] = table[2N-2-k]
    # row i' = N-1-i of the strided view reads w[i' + j] = table[i - j + N - 1]
    v = torch.as_strided(w, size=(N, N), stride=(1, 1))
    return torch.flip(v, dims=[0]).contiguous()


def bf16_tensor(x: np.ndarray, device):
    """Device bf16 tensor holding the bf16-representable fp32 values x exactly."""
    import torch
    return torch.from_numpy(bf16_bits(x).view(np.int16)).to(device).view(torch.bfloat16)


def alibi_slope(h: int, H: int) -> float:
    """Slope of head h (0-based) of H in the ALiBi workload: 2^(-8(h+1)/H)."""
    return 2.0 ** (-8.0 * (h + 1) / H)


def upstream_grad(B: int, H: int, N: int, d: int, seed: int) -> np.ndarray:
    """dO ~ N(0, 1) rounded to bf16 values, fp32 [B, H, N, d] (the gradient a
    loss hands to the attention output in the backward workload)."""
    return round_to_bf16(normal((B, H, N, d), seed))
