"""Helpers shared by the GPU parity tests: device upload of seeded inputs,
the tolerances, and the comparison against the oracle."""
from __future__ import annotations

import numpy as np

# Tolerances on O against the fp64 oracle, as the benchmark definition states
# them (fp32 path: max 1e-5; bf16 inputs with fp32 accumulation: max 2e-2,
# mean 2e-3). LSE has no stated bound; these are our reading (relative for the
# fp32 path, absolute for bf16).
TOL = {
    "f32": dict(o_max=1e-5, o_mean=None, lse=1e-5),
    "bf16": dict(o_max=2e-2, o_mean=2e-3, lse=2e-2),
}


def dev(x: np.ndarray, dtype: str, device="cuda"):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(device)
    return t.to(torch.bfloat16) if dtype == "bf16" else t


def host(t) -> np.ndarray:
    return t.float().cpu().numpy().astype(np.float64)


def compare(o_gpu, lse_gpu, o_ref, lse_ref, dtype: str, what: str = ""):
    """Assert the GPU result matches the oracle within the tolerance; return the errors."""
    tol = TOL[dtype]
    do = np.abs(np.asarray(o_gpu, np.float64) - o_ref)
    dl = np.abs(np.asarray(lse_gpu, np.float64) - lse_ref)
    if dtype == "f32":
        dl = dl / np.maximum(1.0, np.abs(lse_ref))
    err = dict(o_max=float(do.max()), o_mean=float(do.mean()), lse_max=float(dl.max()))
    assert np.all(np.isfinite(o_gpu)), f"{what}: non-finite output"
    assert err["o_max"] <= tol["o_max"], f"{what}: max|dO| {err['o_max']:.3e} > {tol['o_max']}"
    if tol["o_mean"] is not None:
        assert err["o_mean"] <= tol["o_mean"], f"{what}: mean|dO| {err['o_mean']:.3e} > {tol['o_mean']}"
    assert err["lse_max"] <= tol["lse"], f"{what}: |dLSE| {err['lse_max']:.3e} > {tol['lse']}"
    return err


def grad_close(g, ref, what):
    """Gradient tolerance: the forward's bf16 bound on O (max 2e-2, mean 2e-3
    for values of order one) applied to the gradient scaled by its largest
    reference magnitude, floored at 1e-3 for gradients that vanish exactly
    (a single visible key makes dS zero; the kernel then returns rounding
    noise of D = rowsum(dO * O) from the bf16 O)."""
    g = np.asarray(g, np.float64)
    assert np.all(np.isfinite(g)), f"{what}: non-finite gradient"
    m = max(float(np.abs(ref).max()) if ref.size else 0.0, 1e-3)
    err = np.abs(g - ref) / m
    assert err.max() <= 2e-2, f"{what}: max rel {err.max():.3e}"
    assert err.mean() <= 2e-3, f"{what}: mean rel {err.mean():.3e}"
    return float(err.max()), float(err.mean())
