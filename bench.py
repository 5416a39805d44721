"""Benchmark: fused forward of attention with a low-rank additive bias on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config C] [--impl ours|reference]

One step is one pass of the hot path over one batch of the workload: the
factor preparation and the fused tcgen05 attention kernel. The exact
Sandwich/ALiBi factors depend only on N and H, so they are generated once on
the device before timing. The default workload is the GPT-2-small-shaped
causal attention with the Sandwich bias (B=8, H=12, N=2048, d=64, exact rank
64); --config selects another workload (0..7) for measurement. The default
single-GPU run also times the fused and the dense-bias kernels of the four
bf16 workloads (1..4) on their own and reports them under "per_config".

Prints one JSON line (rank 0). Under torchrun every rank runs its own batch
(independent problems, weak scaling, no data-path collective); timing is on
the device with CUDA events, the max over ranks.

--impl reference times the fp64 CPU oracle as the reference arm on a bounded
sample of the same workload (rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import seeded_inputs as si  # noqa: E402

METRIC = "biased-attn fwd TFLOP/s & ms at 1 B200 (% of bf16 TC peak) vs dense-bias path"
UNIT = "TFLOP/s"
L2_FLUSH_BYTES = 256 << 20
KERNEL_SOURCES = ("attention_rank_additive_b200/csrc/fb_attn_sm100.cu", "attention_rank_additive_b200/csrc/fb_ptx.cuh")
BWD_KERNEL_SOURCES = ("attention_rank_additive_b200/csrc/fb_attn_bwd_sm100.cu",
                      "attention_rank_additive_b200/csrc/fb_ptx.cuh")


def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--config", type=int, default=1, choices=[0, 1, 2, 3, 4, 5, 6, 7])
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-dense", action="store_true", help="skip the dense-bias comparison leg")
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU oracle baseline leg")
    ap.add_argument("--batch", type=int, default=0, help="override the workload's B (a smaller case, e.g. to profile)")
    ap.add_argument("--heads", type=int, default=0, help="override the workload's H (a smaller case, e.g. to profile)")
    ap.add_argument("--no-per-config", action="store_true",
                    help="skip the per-workload leg (fused and dense kernels of workloads 1..4)")
    return ap.parse_args(argv)


def workload(cfg_idx: int, batch: int = 0, heads: int = 0) -> dict:
    """The seeded workload cfg_idx, optionally with fewer batches or heads (a
    smaller case of the same kernel, for profiling); counted FLOPs follow."""
    c = dict(si.CONFIGS[cfg_idx])
    if batch > 0:
        c["B"] = batch
    if heads > 0:
        c["H"] = heads
    c["flops"] = flops(c["B"], c["H"], c["N"], c["d"], c["R"], c["causal"], c["bias"] == "mulcos")
    if c.get("bwd"):
        c["flops"] = bwd_flops(c["B"], c["H"], c["N"], c["d"], c["R"], c["causal"])
    if c["bias"] == "neural":  # plus the two linear layers, per (batch, head)
        c["flops"] += 2.0 * 2.0 * c["B"] * c["H"] * c["N"] * c["F"] * c["R"]
    return c


def flops(B, H, N, d, R, causal, multiplicative=False) -> float:
    """Counted FLOPs per head: additive 4 N^2 d + 2 N^2 R; multiplicative
    2 N^2 d R (the scores over the R reweighted copies of q and k) + 2 N^2 d
    (PV); halved when causal."""
    per = 2.0 * N * N * d * R + 2.0 * N * N * d if multiplicative else 4.0 * N * N * d + 2.0 * N * N * R
    f = float(B) * H * per
    return f / 2.0 if causal else f


def bwd_flops(B, H, N, d, R, causal, factor_grads=True) -> float:
    """Counted FLOPs of the backward per head: the five products of the
    concatenated form, 2 N^2 (d + R) each for S, dQ' = dS K' and dK' =
    dS^T Q', 2 N^2 d each for dP and dV (the dQ kernel's recomputation of S
    and dP is not counted); without factor gradients dQ and dK are 2 N^2 d
    each; halved when causal."""
    f = float(B) * H * 2.0 * N * N * ((5.0 * d + 3.0 * R) if factor_grads else (5.0 * d + R))
    return f / 2.0 if causal else f


def config_json(c: dict, l2: str) -> dict:
    return {"workload": f"{c['name']} (B={c['B']},H={c['H']},N={c['N']},d={c['d']},R={c['R']},"
                        f"{'causal' if c['causal'] else 'no mask'},{c['bias']} bias)",
            "B": c["B"], "H": c["H"], "N": c["N"], "d": c["d"], "R": c["R"], "causal": c["causal"],
            "bias": c["bias"], "dtype": c["dtype"], "l2": l2,
            "pass": "backward (dQ, dK, dV, dphi_q, dphi_k for a given dO)" if c.get("bwd") else "forward",
            "factors": ("static (the exact Sandwich/ALiBi decomposition depends on N, H only), generated once "
                        "before timing; prepared (scaled, fp16/paired) and consumed every step"
                        if c["bias"] in ("sandwich", "alibi") else
                        "given fp32 factors, prepared (scaled, fp16/paired) and consumed every step")}


# ---------------------------------------------------------------- distributed

def dist_init(n_gpus: int):
    """(rank, world, local_rank); initialises NCCL when launched by torchrun."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=torch.device("cuda", local))
    return rank, world, local


def reduce_max(value: float, world: int, device=None) -> float:
    """Max of a scalar over ranks (identity for one rank)."""
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_value(flops_per_rank: float, world: int, ms_max: float) -> float:
    """Whole-job TFLOP/s: every rank ran its own batch; time is the max over ranks."""
    return flops_per_rank * world / (ms_max * 1e-3) / 1e12


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ------------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "20"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        time.sleep(0.05)
        self.lines = []
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [ln for ln in out.splitlines() if ln.strip()]
        return False

    def summary(self):
        rows = []
        for ln in self.lines:
            p = [x.strip() for x in ln.split(",")]
            if len(p) < 9:
                continue
            try:
                rows.append(dict(sm=float(p[1]), smax=float(p[2]), power=float(p[3]), hw=p[5], hwt=p[6], swt=p[7],
                                 swp=p[8]))
            except ValueError:
                continue
        if not rows:
            return None
        peak_power = max(r["power"] for r in rows)
        loaded = [r for r in rows if r["power"] >= 0.5 * peak_power] or rows
        reasons = set()
        for r in rows:
            for key, name in (("hw", "hw_slowdown"), ("hwt", "hw_thermal_slowdown"), ("swt", "sw_thermal_slowdown"),
                              ("swp", "sw_power_cap")):
                if r[key].lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(r["sm"] for r in loaded), "sm_max_mhz": max(r["smax"] for r in rows),
                "samples": len(rows), "reasons": sorted(reasons)}


# ---------------------------------------------------------------- profiles

def kernel_source_sha(sources=KERNEL_SOURCES) -> str:
    h = hashlib.sha256()
    for rel in sources:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic(cfg_idx: int):
    """dram bytes per launch of the fused kernel (of the fused backward kernel
    for the backward) from the committed ncu summary, if it was taken on the
    current kernel source and this workload; else None."""
    c = si.CONFIGS[cfg_idx]
    bwd = bool(c.get("bwd"))
    path = os.path.join(ROOT, "profiles", f"attn_{'bwd' if bwd else 'fwd'}_sm100_{c['name']}.md")
    if not os.path.exists(path):
        return None
    text = open(path).read()
    sha = re.search(r"kernel_source_sha:\s*([0-9a-f]+)", text)
    val = re.search(r"traffic_bytes_per_launch:\s*([0-9.eE+]+)", text)
    if not sha or not val or sha.group(1) != kernel_source_sha(BWD_KERNEL_SOURCES if bwd else KERNEL_SOURCES):
        return None
    return float(val.group(1))


def fp32_fma_peak_tflops(clk_sum) -> float:
    """fp32 FMA peak of the GPU from its unit counts and clock: 148 SMs x 128
    FMA lanes per clock x 2 FLOP, at the maximum SM clock the run reported."""
    mhz = clk_sum["sm_max_mhz"] if clk_sum else 1965.0
    return 148 * 128 * 2 * mhz * 1e6 / 1e12


def measured_peaks():
    """(bf16 burst TF/s, bf16 sustained TF/s, HBM GB/s, 'measured' | 'fallback')."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        burst = float(p["bf16_tflops"])
        return burst, float(p.get("bf16_tflops_sustained", burst)), float(p["hbm_gbs"]), "measured"
    return 1590.0, 1400.0, 6650.0, "fallback"


# ------------------------------------------------------------ GPU workload

class GpuWorkload:
    """Device-resident inputs of one workload and the step that runs the hot path."""

    def __init__(self, c: dict, device, with_dense: bool):
        import torch

        import attention_rank_additive_b200 as fb
        self.fb, self.torch, self.c, self.device = fb, torch, c, device
        B, H, N, d, R = c["B"], c["H"], c["N"], c["d"], c["R"]
        self.dt = torch.bfloat16 if c["dtype"] == "bf16" else torch.float32
        q, k, v = si.qkv(B, H, N, d, si.QKV_SEED_BASE + c["index"], c["dtype"])
        self.host_q, self.host_k, self.host_v = (torch.from_numpy(x).to(self.dt).pin_memory() for x in (q, k, v))
        self.Q = self.host_q.to(device)
        self.K = self.host_k.to(device)
        self.V = self.host_v.to(device)
        self.O = torch.empty_like(self.Q)
        self.LSE = torch.empty((B, H, N), device=device, dtype=torch.float32)
        self.scale = 1.0 / math.sqrt(d)
        self.stream = torch.cuda.current_stream(device).cuda_stream
        # factors: generated on the device inside the step for the exact kinds
        self.pq = self.pk = None
        if c["bias"] == "sandwich":
            self.pq = torch.empty((N, R), device=device, dtype=torch.float32)
            self.pk = self.pq
        elif c["bias"] == "alibi":
            self.pq = torch.empty((H, N, 2), device=device, dtype=torch.float32)
            self.pk = torch.empty((H, N, 2), device=device, dtype=torch.float32)
        elif c["bias"] == "lowrank":
            pq, pk = si.random_factors((B, H, N, R), c["factor_std"], si.FACTOR_SEED_BASE + c["index"])
            self.pq, self.pk = torch.from_numpy(pq).to(device), torch.from_numpy(pk).to(device)
        elif c["bias"] == "mulcos":
            # the multiplicative example's exact rank-2 factors [cos i, sin i] (static input)
            i = np.arange(N, dtype=np.float64)
            f = np.stack([np.cos(i), np.sin(i)], 1).astype(np.float32)
            self.pq = torch.from_numpy(f).to(device)
            self.pk = self.pq
        elif c["bias"] == "neural":
            xq, xk, wq, wk = si.neural_inputs(B, H, N, c["F"], R, si.FACTOR_SEED_BASE + c["index"])
            self.nx = [torch.from_numpy(a).to(device) for a in (xq, xk, wq, wk)]
            self.pq = self.pk = None
        elif c["bias"] == "rbf_svd":
            om, ph = si.rbf_params(H, c["rbf_terms"])
            table = si.rbf_offset_table(om, ph, c["grid"])
            pq = np.empty((H, N, R), np.float32)
            pk = np.empty((H, N, R), np.float32)
            self.svd_err = []
            t0 = time.perf_counter()
            for h in range(H):
                pq[h], pk[h], err, en = fb.svd_factors(si.rbf_dense(table, c["grid"], heads=[h])[0], R,
                                                       oversample=64, power_iters=1, seed=h)
                self.svd_err.append((round(err, 4), round(en, 4)))
            self.svd_host_s = time.perf_counter() - t0  # includes building each dense field on the host
            self.pq, self.pk = torch.from_numpy(pq).to(device), torch.from_numpy(pk).to(device)
            self.rbf_table = table
        if self.pq is not None:
            self.bs, self.hs = fb._factor_strides(self.pq, B, H, N, R)
        else:
            self.bs = self.hs = 0
        Rk = self.pq.shape[-1] if self.pq is not None else (R if c["bias"] == "neural" else 0)
        self.R = Rk
        self.mul = c["bias"] == "mulcos"
        self.neural = c["bias"] == "neural"
        if self.neural:
            self.ws_bytes = fb.fb_attn_neural_workspace_bytes(B, H, N, c["F"], Rk)
        elif self.mul:
            self.ws_bytes = fb.fb_attn_mul_bias_workspace_bytes(B, H, N, d, Rk)
        else:
            self.ws_bytes = fb.fb_attn_workspace_bytes(B, H, N, Rk, self.bs, self.hs) if c["dtype"] == "bf16" else 0
        self.ws = torch.empty(max(self.ws_bytes, 256), device=device, dtype=torch.uint8)
        self.flush_buf = torch.empty(L2_FLUSH_BYTES, device=device, dtype=torch.uint8)
        self.dense = None
        if with_dense and c["dtype"] == "bf16":
            self.dense = self._dense_bias()
        # fused kernel, plus the preparation launch (bf16 with a bias); the multiplicative case has its
        # reweighting launch instead, the neural case its linear layers (which write the prepared factors)
        self.launches_per_step = (2 if self.neural else
                                  (2 if self.mul or (Rk > 0 and c["dtype"] == "bf16") else 1))
        self.bwd = bool(c.get("bwd"))
        if self.bwd:  # factor preparation, bf16 factor copies, per-row terms, the gradient kernels (the
            # fused kernel and its dQ conversion at head dim 64; else the dK/dV and dQ kernels), and the
            # reduction of per-head factor gradients when a factor slice serves several heads
            shared = Rk > 0 and (self.bs == 0 and B > 1 or self.hs == 0 and H > 1)
            self.launches_per_step = (5 + (1 if shared else 0)) if Rk > 0 else 3

    def setup_bwd(self):
        """Forward outputs O, LSE for the backward workload (once, untimed),
        the seeded upstream gradient dO, and the gradient buffers."""
        torch, fb, c = self.torch, self.fb, self.c
        B, H, N, d = c["B"], c["H"], c["N"], c["d"]
        self.attn()
        self.host_o = self.O.cpu().pin_memory()
        self.host_lse = self.LSE.cpu().pin_memory()
        g = si.upstream_grad(B, H, N, d, si.DO_SEED_BASE + c["index"])
        self.host_do = torch.from_numpy(g).to(torch.bfloat16).pin_memory()
        self.dO = self.host_do.to(self.device)
        self.dQ, self.dK, self.dV = (torch.empty_like(self.Q) for _ in range(3))
        self.dpq = torch.empty_like(self.pq) if self.R else None
        self.dpk = torch.empty_like(self.pk) if self.R else None
        self.bws_bytes = fb.fb_attn_bwd_workspace_bytes(B, H, N, self.R, self.bs, self.hs)
        self.bws = torch.empty(self.bws_bytes, device=self.device, dtype=torch.uint8)

    def run_bwd(self, factor_grads=True):
        fb, c = self.fb, self.c
        fg = factor_grads and self.R > 0
        st = fb.fb_attn_bwd(fb.FB_BF16, c["B"], c["H"], c["N"], c["d"], self.Q.data_ptr(), self.K.data_ptr(),
                            self.V.data_ptr(), self.R, self.pq.data_ptr() if self.R else 0,
                            self.pk.data_ptr() if self.R else 0, self.bs, self.hs, self.scale, int(c["causal"]),
                            self.O.data_ptr(), self.LSE.data_ptr(), self.dO.data_ptr(), self.dQ.data_ptr(),
                            self.dK.data_ptr(), self.dV.data_ptr(), self.dpq.data_ptr() if fg else 0,
                            self.dpk.data_ptr() if fg else 0, self.bws.data_ptr(), self.bws_bytes, self.stream)
        assert st == fb.FB_OK, fb.fb_status_str(st)

    def _dense_bias(self):
        """The same bias materialised as [B, H, N, N] bf16 (the comparison path's input)."""
        torch, c = self.torch, self.c
        B, H, N, R = c["B"], c["H"], c["N"], c["R"]
        if c["bias"] == "sandwich":
            tab = si.round_to_bf16(si.sandwich_offset_table(N, R).astype(np.float32))
            return si.toeplitz_device(tab, N, self.device).expand(B, H, N, N).contiguous()
        if c["bias"] == "alibi":
            per_head = torch.stack([si.toeplitz_device(
                si.round_to_bf16(si.alibi_offset_table(N, si.alibi_slope(h, H)).astype(np.float32)), N, self.device)
                for h in range(H)])
            return per_head.expand(B, H, N, N).contiguous()
        if c["bias"] == "rbf_svd":
            g = c["grid"]
            tdev = si.bf16_tensor(si.round_to_bf16(self.rbf_table.astype(np.float32)), self.device)
            ix, iy = si.grid_offset_index(g)
            ixd, iyd = torch.from_numpy(ix).to(self.device), torch.from_numpy(iy).to(self.device)
            per_head = torch.stack([tdev[h][ixd, iyd] for h in range(H)])
            return per_head.expand(B, H, N, N).contiguous()
        if c["bias"] == "lowrank":
            pq = self.pq.double().cpu().numpy()
            pk = self.pk.double().cpu().numpy()
            dense = np.einsum("bhnr,bhmr->bhnm", pq, pk).astype(np.float32)
            return si.bf16_tensor(si.round_to_bf16(dense), self.device)
        return None

    def gen_factors(self):
        fb, c = self.fb, self.c
        if c["bias"] == "sandwich":
            st = fb.fb_factors_sandwich(c["N"], c["R"], self.pq.data_ptr(), self.pq.data_ptr(), self.stream)
            assert st == fb.FB_OK, fb.fb_status_str(st)
        elif c["bias"] == "alibi":
            st = fb.fb_factors_alibi(c["H"], c["N"], self.pq.data_ptr(), self.pk.data_ptr(), self.stream)
            assert st == fb.FB_OK, fb.fb_status_str(st)

    def prepare(self):
        """The factor preparation launch (bf16 path with a bias); fb_attn_fwd's first half."""
        fb, c = self.fb, self.c
        if c["dtype"] != "bf16" or self.R == 0 or self.mul or self.neural or getattr(self, "bwd_active", False):
            return
        st = fb.fb_attn_prepare_factors(c["B"], c["H"], c["N"], self.R, self.pq.data_ptr(), self.pk.data_ptr(),
                                        self.bs, self.hs, self.scale, self.ws.data_ptr(), self.ws_bytes, self.stream)
        assert st == fb.FB_OK, fb.fb_status_str(st)

    def run(self):
        """The fused kernel alone (bf16), or the whole fp32 call."""
        fb, c = self.fb, self.c
        if getattr(self, "bwd_active", False):  # the whole backward call (its preparation included)
            self.run_bwd()
            return
        if self.neural:  # linear layers writing the prepared factors + fused kernel (one C-ABI call)
            xq, xk, wq, wk = self.nx
            st = fb.fb_attn_neural_fwd(fb.FB_BF16, c["B"], c["H"], c["N"], c["d"], self.Q.data_ptr(),
                                       self.K.data_ptr(), self.V.data_ptr(), c["F"], self.R, xq.data_ptr(),
                                       xk.data_ptr(), wq.data_ptr(), wk.data_ptr(), self.scale, int(c["causal"]),
                                       self.O.data_ptr(), self.LSE.data_ptr(), self.ws.data_ptr(), self.ws_bytes,
                                       self.stream)
        elif self.mul:  # reweighting launch + fused kernel (one C-ABI call)
            st = fb.fb_attn_mul_bias_fwd(fb.FB_BF16, c["B"], c["H"], c["N"], c["d"], self.Q.data_ptr(),
                                         self.K.data_ptr(), self.V.data_ptr(), self.R, self.pq.data_ptr(),
                                         self.pk.data_ptr(), self.bs, self.hs, self.scale, int(c["causal"]),
                                         self.O.data_ptr(), self.LSE.data_ptr(), self.ws.data_ptr(), self.ws_bytes,
                                         self.stream)
        elif c["dtype"] == "bf16":
            st = fb.fb_attn_fwd_prepared(fb.FB_BF16, c["B"], c["H"], c["N"], c["d"], self.Q.data_ptr(),
                                         self.K.data_ptr(), self.V.data_ptr(), self.R, self.bs, self.hs, self.scale,
                                         int(c["causal"]), self.O.data_ptr(), self.LSE.data_ptr(), self.ws.data_ptr(),
                                         self.ws_bytes, self.stream)
        else:
            st = fb.fb_attn_fwd(fb.FB_F32, c["B"], c["H"], c["N"], c["d"], self.Q.data_ptr(), self.K.data_ptr(),
                                self.V.data_ptr(), self.R, self.pq.data_ptr() if self.R else 0,
                                self.pk.data_ptr() if self.R else 0, self.bs, self.hs, self.scale, int(c["causal"]),
                                self.O.data_ptr(), self.LSE.data_ptr(), 0, 0, self.stream)
        assert st == fb.FB_OK, fb.fb_status_str(st)

    def attn(self):
        """One fb_attn_fwd: preparation, then the fused kernel."""
        self.prepare()
        self.run()

    def dense_attn(self):
        fb, c = self.fb, self.c
        B, H, N = c["B"], c["H"], c["N"]
        st = fb.fb_attn_dense_bias_fwd(fb.FB_BF16, B, H, N, c["d"], self.Q.data_ptr(), self.K.data_ptr(),
                                       self.V.data_ptr(), self.dense.data_ptr(), H * N * N, N * N, self.scale,
                                       int(c["causal"]), self.O.data_ptr(), self.LSE.data_ptr(), self.stream)
        assert st == fb.FB_OK, fb.fb_status_str(st)

    def flush_l2(self):
        self.flush_buf.zero_()


def svd_device_leg(torch, fb, w, c, stream):
    """The same truncation on the GPU (fb_svd_factors_device) from the fp32
    dense fields, timed with CUDA events; its per-head error and energy."""
    H, N, R = c["H"], c["N"], c["R"]
    dense = torch.from_numpy(si.rbf_dense(w.rbf_table, c["grid"]).astype(np.float32)).to(w.device)
    pq = torch.empty((H, N, R), device=w.device, dtype=torch.float32)
    pk = torch.empty_like(pq)
    ee = torch.empty((H, 2), device=w.device, dtype=torch.float64)
    nb = fb.fb_svd_device_workspace_bytes(H, N, R, 24)
    ws = torch.empty(nb, device=w.device, dtype=torch.uint8)

    def run():
        st = fb.fb_svd_factors_device(H, N, R, 24, 2, 7, dense.data_ptr(), pq.data_ptr(), pk.data_ptr(),
                                      ee.data_ptr(), ws.data_ptr(), nb, stream.cuda_stream)
        assert st == fb.FB_OK, fb.fb_status_str(st)

    run()
    torch.cuda.synchronize()
    ms = statistics.median(time_steps(torch, run, None, 5, stream))
    e = ee.cpu().numpy()
    return {"ms": round(ms, 3), "heads": H, "N": N, "R": R, "oversample": 24, "power_iters": 2,
            "rank_error_energy_per_head": [(round(float(a), 4), round(float(b), 4)) for a, b in e],
            "host_s_same_heads": round(w.svd_host_s, 2),
            "host_settings": "fb_svd_factors_host, oversample 64, power_iters 1, fp64"}


# ------------------------------------------------------------ per workload

PER_CONFIG_STEPS = {1: 100, 2: 30, 3: 60, 4: 200}
MUFU_EXP2_PER_CLK_PER_SM = 16  # B200 special-function unit rate for exp2


def exp2_elements(c: dict) -> float:
    """Scores that need an exponential: B H N^2, halved when causal (as counted FLOPs)."""
    e = float(c["B"]) * c["H"] * c["N"] * c["N"]
    return e / 2.0 if c["causal"] else e


def per_config_leg(torch, fb, device, stream):
    """The fused kernel alone and the dense-bias kernel alone on each bf16
    workload (1..4), L2 flushed between launches, CUDA events on the launching
    stream, clocks sampled during the fused timing: the roofline fraction
    against the peak the clock record calls for, the exp2 (special-function
    unit) floor, and the dense kernel's bias stream against the HBM peak."""
    burst_tf, sustained_tf, peak_hbm, peak_src = measured_peaks()
    out = {}
    for ci in (1, 2, 3, 4):
        c = workload(ci)
        w = GpuWorkload(c, device, with_dense=True)
        w.gen_factors()
        for _ in range(3):
            w.attn()
        torch.cuda.synchronize()
        st = fb.fb_check_device_error(stream.cuda_stream)
        assert st == fb.FB_OK, fb.fb_status_str(st)
        w.prepare()
        steps = PER_CONFIG_STEPS[ci]
        with ClockSampler(device.index or 0) as clk:
            ms = time_steps(torch, w.run, w.flush_l2, steps, stream)
        clk_sum = clk.summary()
        kms = statistics.median(ms)
        capped = bool(clk_sum) and "sw_power_cap" in clk_sum.get("reasons", [])
        peak_tf = sustained_tf if capped else burst_tf
        achieved = c["flops"] / (kms * 1e-3) / 1e12
        sm_max_hz = 1e6 * (clk_sum["sm_max_mhz"] if clk_sum else 1965.0)
        floor_ms = exp2_elements(c) / (MUFU_EXP2_PER_CLK_PER_SM * 148 * sm_max_hz) * 1e3
        entry = {"workload": config_json(c, "")["workload"], "steps": steps, "kernel_ms": round(kms, 5),
                 "kernel_ms_mean": round(statistics.mean(ms), 5), "tflops": round(achieved, 2),
                 "peak": peak_tf, "peak_kind": f"{peak_src} bf16 {'sustained (power-capped)' if capped else 'burst'}",
                 "frac": round(achieved / peak_tf, 4), "traffic": profiled_traffic(ci),
                 "exp2_floor_ms": round(floor_ms, 5), "exp2_floor_frac": round(floor_ms / kms, 4),
                 "clocks": clk_sum}
        if w.dense is not None:
            for _ in range(3):
                w.dense_attn()
            d_ms = statistics.median(time_steps(torch, w.dense_attn, w.flush_l2, max(10, steps // 2), stream))
            n_kv = (c["N"] + 127) // 128
            tiles = c["B"] * c["H"] * (n_kv * (n_kv + 1) // 2 if c["causal"] else n_kv * n_kv)
            bias_bytes = tiles * 128 * 128 * 2
            entry["dense"] = {"ms": round(d_ms, 5), "bias_bytes_read": bias_bytes,
                              "bias_gbs": round(bias_bytes / (d_ms * 1e-3) / 1e9, 1),
                              "hbm_frac": round(bias_bytes / (d_ms * 1e-3) / 1e9 / peak_hbm, 4),
                              "fused_speedup": round(d_ms / kms, 3)}
        st = fb.fb_check_device_error(stream.cuda_stream)
        assert st == fb.FB_OK, fb.fb_status_str(st)
        out[f"c{ci}"] = entry
        del w
        torch.cuda.synchronize()
        torch.cuda.empty_cache()
    return out


# ------------------------------------------------------------------ timing

def time_steps(torch, fn, before, steps: int, stream):
    """Run `steps` iterations; `before` (untimed, e.g. an L2 flush) precedes each.
    Returns the per-step device times in ms (CUDA events on the launching stream)."""
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for a, b in evs:
        if before is not None:
            before()
        a.record(stream)
        fn()
        b.record(stream)
    torch.cuda.synchronize()
    return [a.elapsed_time(b) for a, b in evs]


def run_ours(args, rank: int, world: int, local: int):
    import torch

    import attention_rank_additive_b200 as fb
    c = workload(args.config, args.batch, args.heads)
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    fb.lib()
    # (no dense counterpart for the multiplicative bias: the comparison kernel adds its bias)
    w = GpuWorkload(c, device, with_dense=not args.no_dense and c["dtype"] == "bf16"
                    and c["bias"] not in ("mulcos", "neural") and not c.get("bwd"))
    stream = torch.cuda.current_stream(device)

    attn_ms = []

    w.gen_factors()  # static factors: once, outside the timed steps
    if w.bwd:
        w.setup_bwd()
        w.bwd_active = True

    def step():
        w.prepare()
        e1 = torch.cuda.Event(enable_timing=True)
        e2 = torch.cuda.Event(enable_timing=True)
        e1.record(stream)
        w.run()  # the fused kernel alone, bracketed for the roofline
        e2.record(stream)
        attn_ms.append((e1, e2))

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    st = fb.fb_check_device_error(stream.cuda_stream)
    assert st == fb.FB_OK, fb.fb_status_str(st)
    attn_ms.clear()

    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        step_ms = time_steps(torch, step, w.flush_l2, args.steps, stream)
    torch.cuda.synchronize()
    barrier(world)
    st = fb.fb_check_device_error(stream.cuda_stream)
    assert st == fb.FB_OK, fb.fb_status_str(st)
    kern_ms = statistics.mean(a.elapsed_time(b) for a, b in attn_ms)
    ms_local = statistics.mean(step_ms)
    ms = reduce_max(ms_local, world, device)
    kern_ms = reduce_max(kern_ms, world, device)
    value = weak_scaling_value(c["flops"], world, ms)

    # end to end through the C ABI with host buffers: H2D of Q, K, V from
    # pinned memory, the step, D2H of O and LSE, every step.
    host_o = torch.empty(w.O.shape, dtype=w.O.dtype, pin_memory=True)
    host_l = torch.empty(w.LSE.shape, dtype=torch.float32, pin_memory=True)

    def e2e_step():
        w.Q.copy_(w.host_q, non_blocking=True)
        w.K.copy_(w.host_k, non_blocking=True)
        w.V.copy_(w.host_v, non_blocking=True)
        w.attn()
        host_o.copy_(w.O, non_blocking=True)
        host_l.copy_(w.LSE, non_blocking=True)

    if w.bwd:  # inputs Q, K, V, O, LSE, dO up; dQ, dK, dV (and the factor gradients) down
        host_g = [torch.empty(w.Q.shape, dtype=w.Q.dtype, pin_memory=True) for _ in range(3)]
        host_gf = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in (w.dpq, w.dpk) if t is not None]

        def e2e_step():
            w.Q.copy_(w.host_q, non_blocking=True)
            w.K.copy_(w.host_k, non_blocking=True)
            w.V.copy_(w.host_v, non_blocking=True)
            w.O.copy_(w.host_o, non_blocking=True)
            w.LSE.copy_(w.host_lse, non_blocking=True)
            w.dO.copy_(w.host_do, non_blocking=True)
            w.run_bwd()
            for hb, t in zip(host_g, (w.dQ, w.dK, w.dV)):
                hb.copy_(t, non_blocking=True)
            for hb, t in zip(host_gf, [t for t in (w.dpq, w.dpk) if t is not None]):
                hb.copy_(t, non_blocking=True)

    for _ in range(3):
        e2e_step()
    e2e_steps = max(5, min(args.steps, 50))
    barrier(world)
    e2e_ms = reduce_max(statistics.mean(time_steps(torch, e2e_step, None, e2e_steps, stream)), world, device)
    barrier(world)
    h2d = 3 * w.Q.numel() * w.Q.element_size()
    d2h = w.O.numel() * w.O.element_size() + w.LSE.numel() * 4
    if w.bwd:
        h2d = 5 * w.Q.numel() * w.Q.element_size() + w.LSE.numel() * 4
        d2h = 3 * w.Q.numel() * w.Q.element_size() + sum(t.numel() * 4 for t in (w.dpq, w.dpk) if t is not None)

    dense = None
    if w.dense is not None:
        for _ in range(3):
            w.dense_attn()
        d_steps = max(5, min(args.steps, 100))
        barrier(world)
        d_ms = reduce_max(statistics.mean(time_steps(torch, w.dense_attn, w.flush_l2, d_steps, stream)), world,
                          device)
        barrier(world)
        n_kv = (c["N"] + 127) // 128
        tiles = c["B"] * c["H"] * (n_kv * (n_kv + 1) // 2 if c["causal"] else n_kv * n_kv)
        bias_bytes = tiles * 128 * 128 * 2
        dense = {"ms": round(d_ms, 5), "tflops": round(c["flops"] / (d_ms * 1e-3) / 1e12, 2),
                 "bias_bytes_read": bias_bytes, "bias_gbs": round(bias_bytes / (d_ms * 1e-3) / 1e9, 1),
                 "fused_speedup": round(d_ms / kern_ms, 3),
                 "layout": "[B,H,N,N] bf16 materialised, L2 flushed between steps"}

    clk_sum = clk.summary()
    burst_tf, sustained_tf, peak_hbm, peak_src = measured_peaks()
    # the burst peak for a kernel timed alone; the sustained one when the run
    # itself was held at the power cap (the clock record says so)
    capped = bool(clk_sum) and "sw_power_cap" in clk_sum.get("reasons", [])
    peak_tf = sustained_tf if capped else burst_tf
    peak_kind = f"{peak_src} bf16 {'sustained (run power-capped)' if capped else 'burst'}"
    bound = "tensor"
    if c["dtype"] == "f32":  # the fp32 path runs on the CUDA cores' FMA pipe
        bound, peak_tf = "alu", fp32_fma_peak_tflops(clk_sum)
        peak_kind = "derived: 148 SMs x 128 fp32 FMA/clk x 2 FLOP x max SM clock"
    achieved = c["flops"] / (kern_ms * 1e-3) / 1e12
    traffic = profiled_traffic(args.config)
    out = {
        "metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": max(3, args.warmup), "ms_per_step": round(ms, 5), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": c["dtype"], "data": "synthetic (seeded; see seeded_inputs)",
        "config": config_json(c, "flushed: 256 MiB memset between timed steps (untimed)"),
        "roofline": {"bound": bound, "achieved": round(achieved, 2), "peak": round(peak_tf, 1), "unit": "TFLOP/s",
                     "frac": round(achieved / peak_tf, 4), "traffic": traffic,
                     "kernel": ("prep_mul_bias + attn_fwd_sm100" if w.mul else
                                ("neural_prep + attn_fwd_sm100" if w.neural else
                                 ("bwd preparation (3) + attn_bwd_fused_sm100 + dQ conversion + factor-gradient "
                                  "reduction" if w.bwd and c["d"] > 32 and c["d"] <= 64
                                  else "bwd preparation (3) + attn_bwd_dkdv_sm100 + attn_bwd_dq_sm100 + "
                                       "factor-gradient reduction" if w.bwd
                                  else "attn_fwd_sm100"))),
                     "peak_kind": peak_kind,
                     "kernel_ms": round(kern_ms, 5)},
        "e2e": {"value": round(c["flops"] * world / (e2e_ms * 1e-3) / 1e12, 3), "unit": UNIT,
                "ms_per_step": round(e2e_ms, 4), "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": w.launches_per_step * args.steps,
        "dense_bias": dense,
    }
    if w.bwd and w.R > 0:
        # the same backward with fixed factors (the exact Sandwich factors are not
        # trained): no factor gradients, FLOPs counted without their products
        for _ in range(3):
            w.run_bwd(factor_grads=False)
        f_steps = max(5, min(args.steps, 100))
        barrier(world)
        f_ms = reduce_max(statistics.mean(time_steps(torch, lambda: w.run_bwd(factor_grads=False), w.flush_l2,
                                                     f_steps, stream)), world, device)
        barrier(world)
        f_flops = bwd_flops(c["B"], c["H"], c["N"], c["d"], c["R"], c["causal"], factor_grads=False)
        out["bwd_fixed_factors"] = {"ms": round(f_ms, 5), "tflops": round(f_flops / (f_ms * 1e-3) / 1e12, 2),
                                    "launches_per_step": 4}
    if hasattr(w, "svd_err"):
        out["svd_rank_error_energy_per_head"] = w.svd_err
        out["svd_device"] = svd_device_leg(torch, fb, w, c, stream)
    if world > 1:
        # every rank sampled its own GPU; rank 0 reports its own
        pass
    out["clocks"] = clk_sum
    if world == 1 and args.config == 1 and not args.no_per_config:
        del w
        torch.cuda.empty_cache()
        out["per_config"] = per_config_leg(torch, fb, device, stream)
    if rank == 0 and not args.no_cpu:
        out["cpu_baseline"] = cpu_baseline(c, budget_s=12.0)
    return out


# ------------------------------------------------------------- CPU oracle

def oracle_sample(c: dict, step: int, rows_per_head: int):
    """A bounded sample of the workload for the oracle: `rows_per_head` query
    rows of one (b, h) head, rotating over heads with `step`. Returns
    (callable that runs it, counted FLOPs of the sample, description)."""
    import oracle
    B, H, N, d, R = c["B"], c["H"], c["N"], c["d"], c["R"]
    b, h = (step // H) % B, step % H
    if c.get("bwd"):
        # the causal prefix of n tokens of one head is a complete causal
        # problem of its own: every gradient of it, by the oracle's backward
        n = min(N, rows_per_head)
        q, k, v = (x[:n] for x in _head_inputs(c, b, h))
        phi = oracle.sandwich_factors(n, R)
        g = si.upstream_grad(B, H, N, d, si.DO_SEED_BASE + c["index"])[b, h, :n].astype(np.float64)
        scale = 1.0 / math.sqrt(d)

        def run_bwd():
            oracle.attention_lowrank_bwd_head(q, k, v, phi, phi, g, scale, c["causal"])

        return run_bwd, bwd_flops(1, 1, n, d, R, c["causal"]), f"causal prefix of {n} tokens of head (b={b}, h={h})"
    rng = si.generator(7000 + step)
    rows = np.sort(rng.choice(N, size=min(rows_per_head, N), replace=False)).astype(np.int64)
    q, k, v = _head_inputs(c, b, h)
    scale = 1.0 / math.sqrt(d)
    if c["bias"] == "sandwich":
        bias = oracle.HeadBias.sandwich(R)
    elif c["bias"] == "alibi":
        bias = oracle.HeadBias.alibi(oracle.alibi_slope(h, H))
    elif c["bias"] == "lowrank":
        pq, pk = si.random_factors((B, H, N, R), c["factor_std"], si.FACTOR_SEED_BASE + c["index"])
        bias = oracle.HeadBias.lowrank(pq[b, h], pk[b, h])
    elif c["bias"] == "neural":
        xq, xk, wq, wk = si.neural_inputs(B, H, N, c["F"], R, si.FACTOR_SEED_BASE + c["index"])
        pq, pk = oracle.neural_factors(xq[b:b + 1], xk[b:b + 1], wq[h:h + 1], wk[h:h + 1])
        bias = oracle.HeadBias.lowrank(pq[0, 0], pk[0, 0])
    elif c["bias"] == "mulcos":
        f = oracle.cos_factors(N)
        keys = (rows + 1).astype(np.float64) if c["causal"] else np.full(rows.shape, float(N))

        def run_mul():
            oracle.attention_mul_head(q, k, v, f, f, scale, c["causal"], rows)

        return run_mul, float(np.sum(keys * (2.0 * d * R + 2.0 * d))), f"{len(rows)} query rows of head (b={b}, h={h})"
    else:  # rbf_svd: the dense field truncated by the oracle's own SVD
        om, ph = si.rbf_params(H, c["rbf_terms"])
        dense = si.rbf_dense(si.rbf_offset_table(om, ph, c["grid"]), c["grid"], heads=[h])[0]
        pq, pk, _, _ = oracle.truncated_svd_factors(dense, R)
        bias = oracle.HeadBias.lowrank(pq, pk)
    keys = (rows + 1).astype(np.float64) if c["causal"] else np.full(rows.shape, float(N))
    fl = float(np.sum(keys * (4.0 * d + 2.0 * R)))

    def run():
        oracle.attention_head(q, k, v, bias, scale, c["causal"], rows)

    return run, fl, f"{len(rows)} query rows of head (b={b}, h={h})"


_HEAD_CACHE = {}


def _head_inputs(c, b, h):
    key = (c["index"], b, h)
    if key not in _HEAD_CACHE:
        q, k, v = si.qkv(c["B"], c["H"], c["N"], c["d"], si.QKV_SEED_BASE + c["index"], c["dtype"]) \
            if "all" not in _HEAD_CACHE or _HEAD_CACHE["all"][0] != c["index"] else _HEAD_CACHE["all"][1]
        _HEAD_CACHE["all"] = (c["index"], (q, k, v))
        _HEAD_CACHE[key] = (q[b, h].astype(np.float64), k[b, h].astype(np.float64), v[b, h].astype(np.float64))
    return _HEAD_CACHE[key]


def cpu_baseline(c: dict, budget_s: float):
    """The oracle, as it stands, on the host cores over ~budget_s of a bounded sample."""
    import oracle
    total_fl, total_s, step, parts = 0.0, 0.0, 0, []
    while total_s < budget_s and step < 1024:
        run, fl, desc = oracle_sample(c, step, rows_per_head=256)
        t0 = time.perf_counter()
        run()
        total_s += time.perf_counter() - t0
        total_fl += fl
        parts.append(desc)
        step += 1
    what = ("causal prefixes of 256 tokens (every gradient, fp64 oracle backward, counted FLOPs of the prefix)"
            if c.get("bwd") else "256 sampled query rows (fp64 oracle, counted FLOPs of those rows)")
    return {"value": total_fl / total_s / 1e12, "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"{step} heads x {what}, {total_s:.1f} s"}


def run_reference(args, rank: int, world: int):
    """Reference arm: the fp64 CPU oracle on a bounded sample per step."""
    import oracle
    if rank != 0:
        return None
    c = workload(args.config)
    rows = 32
    for s in range(max(3, args.warmup)):
        oracle_sample(c, s, rows)[0]()
    times, fls = [], []
    for s in range(args.steps):
        run, fl, _ = oracle_sample(c, 1000 + s, rows)
        t0 = time.perf_counter()
        run()
        times.append(time.perf_counter() - t0)
        fls.append(fl)
    tot_s, tot_fl = sum(times), sum(fls)
    value = tot_fl / tot_s / 1e12
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": max(3, args.warmup), "ms_per_step": round(1e3 * tot_s / args.steps, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded; see seeded_inputs)",
        "config": config_json(c, "n/a (host)"),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
                         "sample": (f"per step every gradient of the causal prefix of {rows} tokens of one head "
                                    "(rotating over heads; the oracle backward on a complete sub-problem)"
                                    if c.get("bwd") else
                                    f"per step {rows} sampled query rows of one head (rotating over heads)")},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main(argv=None):
    args = parse_args(argv)
    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        world = int(os.environ.get("WORLD_SIZE", "1"))
        out = run_reference(args, rank, world)
        if out is not None:
            print(json.dumps(out), flush=True)
        return 0
    rank, world, local = dist_init(args.gpus)
    try:
        out = run_ours(args, rank, world, local)
        if rank == 0:
            print(json.dumps(out), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
