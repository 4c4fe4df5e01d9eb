#!/usr/bin/env python
"""Benchmark: fused alpha-entmax attention forward + backward on B200.

One step = one forward and one backward over one batch of the workload
(default: B4 H16 N4096 d128 bf16, causal, alpha 1.5, beta 1).  Prints one JSON
line (rank 0).  ``--impl reference`` times the float64 CPU oracle instead, on a
bounded sample of the same workload, on the host cores.

Multi-GPU (torchrun): every rank runs its own independent batch (heads are
independent problems; no data-path collective), the step time is the max over
ranks, and ``value`` counts the work of all ranks (weak scaling).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from adaptive_sparse_flash_entmax_b200 import inputs  # noqa: E402

METRIC = "entmax attn fwd+bwd ms & TFLOP/s (executed, % BF16 peak) vs block sparsity"
UNIT = "TFLOP/s"


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=100)
    p.add_argument("--warmup", type=int, default=3)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--workload", default="iid", choices=sorted(inputs.WORKLOADS))
    p.add_argument("--beta", type=float, default=None)
    p.add_argument("--alpha", type=float, default=None)
    p.add_argument("--span", type=int, default=None,
                   help="cluster span in keys (clustered workloads; block-sparsity sweep)")
    p.add_argument("--no-comparator", action="store_true",
                   help="skip timing the dense softmax comparator (torch SDPA)")
    p.add_argument("--no-rowop", action="store_true",
                   help="skip timing the row-wise entmax op")
    p.add_argument("--hist-budget", type=int, default=None,
                   help="ablation: histogram insert budget per forward tile (0: no histogram, "
                        "i.e. every row from the plain bracket; -1: no limit)")
    p.add_argument("--delta", choices=["auto", "otilde", "recompute", "lists"], default="auto",
                   help="backward path: delta from the forward's otilde (ent_attn_fwd_otilde + "
                        "ent_attn_bwd_otilde), recomputed by a pass over the keys, the support "
                        "lists (ent_attn_fwd_lists + ent_attn_bwd_lists), or auto: lists when an "
                        "untimed forward gives >= 90%% of the query tiles a list for every row, "
                        "else otilde below 50%% empty blocks, else recompute")
    p.add_argument("--seed", type=int, default=0)
    p.add_argument("--B", type=int, default=None, help="override the batch (profiling cases)")
    p.add_argument("--H", type=int, default=None, help="override the head count")
    p.add_argument("--e2e-steps", type=int, default=10)
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--cpu-heads", type=int, default=24,
                   help="heads in the oracle sample of the cpu_baseline leg")
    p.add_argument("--ref-heads-per-step", type=int, default=4,
                   help="heads per step in the --impl reference arm")
    p.add_argument("--no-sweep", action="store_true",
                   help="skip the block-sparsity / alpha sweep over the other workloads")
    p.add_argument("--sweep-steps", type=int, default=10,
                   help="timed steps per sweep point (after 3 warm-up steps)")
    p.add_argument("--sustained-s", type=float, default=2.0,
                   help="seconds of back-to-back steps for the sustained-clock measurement "
                        "(0: skip)")
    return p.parse_args()


def workload(args) -> inputs.Workload:
    w = inputs.WORKLOADS[args.workload]
    kw = {}
    if args.beta is not None:
        kw["beta"] = args.beta
    if args.alpha is not None:
        kw["alpha"] = args.alpha
    if args.B is not None:
        kw["B"] = args.B
    if args.H is not None:
        kw["H"] = args.H
    if args.span is not None:
        kw["span"] = args.span
    return w.replace(**kw) if kw else w


def config_of(w, n_gpus, extra=None):
    c = {"workload": f"{w.name}: B{w.B} H{w.H} N{w.N} d{w.d} {w.dtype} "
                     f"{'causal' if w.causal else 'non-causal'} alpha={w.alpha} beta={w.beta} "
                     f"({w.kind} inputs)",
         "B": w.B, "H": w.H, "N": w.N, "d": w.d, "alpha": w.alpha, "beta": w.beta,
         "causal": w.causal, "global_batch": w.B * n_gpus, "seq_len": w.N,
         "parallelism": f"replicas x{n_gpus} (independent batches per GPU)",
         "l2": "inputs larger than L2: q, k, v, dO = %d MiB per GPU" % (
             4 * w.B * w.H * w.N * w.d * (2 if w.dtype == 'bf16' else 4) >> 20)}
    if w.kind == "clustered":
        c["cluster_span"] = w.span
    hb = os.environ.get("ENTATTN_HIST_BUDGET")
    calib = (w.dtype == "bf16" and -(-w.N // 128) >= 64
             and os.environ.get("ENTATTN_CALIB", "1") != "0")
    c["tau_start"] = (f"histogram (insert budget {hb})" if hb and int(hb) != 0 else
                      "plain bracket, calibrated (8 sampled rows per head)" if calib else
                      "plain bracket midpoint")
    if hb:
        c["hist_budget"] = int(hb)
    if extra:
        c.update(extra)
    return c


def dense_flops(w) -> float:
    """Algorithmic (dense, FlashAttention convention) fwd+bwd flops: 14 B H N^2 d (/2 causal)."""
    f = 14.0 * w.B * w.H * w.N * w.N * w.d
    return f / 2 if w.causal else f


# --------------------------------------------------------------------- clocks
class ClockSampler:
    """Samples nvidia-smi clocks and throttle reasons while running."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
            # the timed region starts once the sampler is producing (at most 3 s)
            t0 = time.time()
            while not self.lines and time.time() - t0 < 3.0 and self.proc.poll() is None:
                time.sleep(0.01)
            self.skip = len(self.lines)
        except (OSError, ValueError):
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines[getattr(self, "skip", 0):]:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, val in zip(names, f[5:9]):
                if val.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": ["unsampled"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return json.load(f), "measured"
    except (OSError, ValueError):
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                "sm_max_mhz": 1965.0}, "fallback"


def profiled_traffic(w, kernel, variant="plain"):
    """DRAM bytes per launch of `kernel` (variant "plain" or "otilde") on this workload
    from the committed ncu summary (profiles/traffic.json), or None when the kernel
    source changed since the capture (the summary stores a hash of its source files)."""
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            rec = json.load(f)
    except (OSError, ValueError):
        return None
    for r in rec.get("captures", []):
        if r.get("kernel") != kernel or r.get("workload") != w.name:
            continue
        if r.get("variant", "plain") != variant:
            continue
        if any(r.get(k) != getattr(w, k) for k in ("B", "H", "N", "d", "alpha", "beta")):
            continue
        if sources_digest(r.get("sources") or [r["source"]]) == r.get("sha256"):
            return r["dram_bytes_per_launch"]
    return None


def sources_digest(paths):
    """sha256 over the bytes of the given repository files, in order (None if one is
    missing): the kernel file and the headers it includes."""
    import hashlib
    h = hashlib.sha256()
    for rel in paths:
        try:
            with open(os.path.join(ROOT, rel), "rb") as f:
                h.update(f.read())
        except OSError:
            return None
    return h.hexdigest()


# --------------------------------------------------------------------- oracle
def oracle_sample(w, heads, seed):
    """Time the oracle (fwd + bwd) on `heads` heads of the workload (host cores)."""
    import oracle
    oracle.build()
    q, k, v, do = inputs.make_inputs(w.replace(B=1, H=max(1, heads)), seed)
    cores = os.cpu_count() or 1
    t0 = time.perf_counter()
    oracle.attn_fwd(q, k, v, w.alpha, w.causal, nthreads=cores)
    oracle.attn_bwd(q, k, v, do, w.alpha, w.causal, nthreads=cores)
    dt = time.perf_counter() - t0
    return dt, cores


def run_reference(args):
    """The float64 oracle on the host cores: each step is fwd + bwd of a bounded sample
    of the workload (``--ref-heads-per-step`` heads).  ``value`` counts the sample's
    dense-equivalent flops (14 N^2 d / 2 per causal head, the same definition as the
    GPU line's ``cpu_baseline`` and ``effective_dense_tflops``); ``ms_per_step`` is the
    measured time of one sample step, and the time the whole batch would take is
    reported beside it as an extrapolation."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    w = workload(args)
    heads = min(args.ref_heads_per_step, w.B * w.H)
    frac = heads / (w.B * w.H)
    for _ in range(args.warmup):
        oracle_sample(w, heads, args.seed)
    times = []
    for _ in range(args.steps):
        dt, cores = oracle_sample(w, heads, args.seed)
        times.append(dt)
    tot = sum(times)
    value = dense_flops(w) * frac * args.steps / tot / 1e12
    sample_ms = 1e3 * tot / args.steps
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": sample_ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_of(w, 1, {"sample_per_step": f"{heads} of {w.B * w.H} heads"}),
            "sample_ms_per_step": sample_ms,
            "extrapolated_full_batch_ms_per_step": sample_ms / frac,
            "flop_definition": "dense-equivalent: 14 B H N^2 d (/2 causal), as effective_dense_tflops",
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": f"float64 oracle fwd+bwd on {heads} of {w.B * w.H} heads "
                                       f"per step ({sample_ms:.0f} ms measured per sample step); "
                                       "dense-equivalent flops (14 N^2 d / 2 per causal head)"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# --------------------------------------------------------------------- ours
NOMINAL_BF16_TFLOPS = 2250.0   # dense bf16 tensor peak, nominal


def element_density(q, k, tau, alpha, causal, heads=2, chunk=512):
    """Fraction of admissible (query, key) pairs with p > 0 over the first `heads` heads
    (scores recomputed in float32 with torch from the same inputs; measurement only)."""
    import torch
    B, H, N, d = q.shape
    cx = (alpha - 1.0) / d ** 0.5
    cols = torch.arange(N, device=q.device)
    nnz = adm = 0
    for bh in range(min(heads, B * H)):
        b, h = divmod(bh, H)
        K = k[b, h].float()
        for r0 in range(0, N, chunk):
            r1 = min(N, r0 + chunk)
            rows = torch.arange(r0, r1, device=q.device)
            x = cx * (q[b, h, r0:r1].float() @ K.T)
            live = x > tau[b, h, r0:r1, None]
            if causal:
                live &= cols[None, :] <= rows[:, None]
            nnz += int(live.sum().item())
            adm += int(((rows + 1).sum().item()) if causal else (r1 - r0) * N)
    return nnz / adm


def time_dense_comparator(q, k, v, do, causal, steps):
    """Softmax attention forward + backward with torch SDPA on the same tensors
    (flash and cuDNN backends, the faster counts): measurement context only, not
    part of the method.  Returns {"flash_ms", "cudnn_ms", "ms_per_step", "backend"}."""
    import torch
    import torch.nn.functional as F
    from torch.nn.attention import SDPBackend, sdpa_kernel
    out = {}
    for name, backend in (("flash", SDPBackend.FLASH_ATTENTION), ("cudnn", SDPBackend.CUDNN_ATTENTION)):
        try:
            qq, kk, vv = (x.detach().requires_grad_() for x in (q, k, v))

            def step():
                qq.grad = kk.grad = vv.grad = None
                with sdpa_kernel(backend):
                    o = F.scaled_dot_product_attention(qq, kk, vv, is_causal=causal)
                o.backward(do)

            for _ in range(3):
                step()
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            for _ in range(steps):
                step()
            e1.record()
            torch.cuda.synchronize()
            out[name + "_ms"] = e0.elapsed_time(e1) / steps
        except Exception:   # backend unavailable for this shape or build
            out[name + "_ms"] = None
    done = {k: v for k, v in out.items() if v is not None}
    if done:
        best = min(done, key=done.get)
        out["ms_per_step"] = done[best]
        out["backend"] = best[:-3]
    return out


def time_row_entmax(dev, seed, hbm_gbs, rows=16384, n=4096, alpha=1.5):
    """The row-wise entmax op on a [rows, n] bf16 score matrix, per root finder:
    ms per call, solver passes, and HBM throughput (z read once, p written once)."""
    import torch
    from adaptive_sparse_flash_entmax_b200 import attention as A
    z = torch.from_numpy(inputs.row_scores(rows, n, seed)).to(torch.bfloat16).to(dev)
    p = torch.empty_like(z)
    tau = torch.empty(rows, dtype=torch.float32, device=dev)
    it = torch.empty(rows, dtype=torch.uint8, device=dev)
    nbytes = 2 * rows * n * 2 + rows * 5
    out = {"shape": f"[{rows}, {n}] bf16 N(0,1) scores, alpha {alpha}",
           "bytes_per_call": nbytes}
    for solver in ("hist", "halley", "bisect"):
        for _ in range(3):
            A.entmax_rows_fwd(z, alpha, solver, out=(p, tau, it))
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(20):
            A.entmax_rows_fwd(z, alpha, solver, out=(p, tau, it))
        e1.record()
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1) / 20
        itf = it.float()
        out[solver] = {"ms": ms, "passes_mean": itf.mean().item(), "passes_max": int(itf.max().item()),
                       "gbs": nbytes / (ms * 1e-3) / 1e9,
                       "hbm_frac": nbytes / (ms * 1e-3) / 1e9 / hbm_gbs}
    out["bisect_over_halley_passes"] = out["bisect"]["passes_mean"] / out["halley"]["passes_mean"]
    out["bisect_over_hist_ms"] = out["bisect"]["ms"] / out["hist"]["ms"]
    return out


def combine_ranks(ms: float, units: float, world: int, device) -> tuple:
    """(max over ranks of the device time `ms`, sum over ranks of the work `units`).

    Every rank calls it at the same point of the run (two all-reduces: MAX, then
    SUM), so ``value = units / ms`` counts the work of all ranks against the slowest
    rank's clock."""
    if world == 1:
        return ms, units
    import torch
    import torch.distributed as dist
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    u = torch.tensor([units], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    dist.all_reduce(u, op=dist.ReduceOp.SUM)
    return t.item(), u.item()


def launches_per_step(dtype, delta, T):
    """Kernels of this library launched per step.  bf16: the key-block statistics and the
    two kernels of the calibrated start (each at least 64 query tiles, unless
    ENTATTN_BOUND=0 / ENTATTN_CALIB=0 or the histogram start is selected), the forward
    (whose free CTAs also re-solve any tile that failed the check of its unevaluated
    stops), the support-list backward (lists only), dq and dkv.  float32: the forward and
    three backward kernels."""
    if dtype != "bf16":
        return 4
    hb = os.environ.get("ENTATTN_HIST_BUDGET")
    plain = (not hb or int(hb) == 0) and T >= 64
    bound = os.environ.get("ENTATTN_BOUND", "1") != "0" and plain
    calib = os.environ.get("ENTATTN_CALIB", "1") != "0" and plain
    return int(bound) + 2 * int(calib) + 1 + (1 if delta == "lists" else 0) + 2


SWEEP = ([("iid", {"beta": b}) for b in (1.0, 2.0, 4.0, 8.0)]
         + [("alpha", {"alpha": a}) for a in (1.25, 1.5, 2.0)]
         + [("long", {}), ("lm", {})]
         + [("clustered4k", {"span": sp}) for sp in (2048, 512, 128)])


class Case:
    """Device buffers of one workload and the fwd + bwd step that the bench times."""

    def __init__(self, w, seed, dev, delta="auto", keep_host=False):
        import torch
        from adaptive_sparse_flash_entmax_b200 import attention as A
        from adaptive_sparse_flash_entmax_b200 import capi
        self.w, self.dev = w, dev
        B, H, N, d = w.shape
        tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
        q, k, v, do = inputs.make_inputs(w, seed)
        host = [torch.from_numpy(a).to(tdt) for a in (q, k, v, do)]
        if keep_host:
            host = [h.pin_memory() for h in host]
            self.host = host
        self.qd, self.kd, self.vd, self.dod = (h.to(dev) for h in host)
        del q, k, v, do
        dt_code = capi.ENT_BF16 if w.dtype == "bf16" else capi.ENT_F32
        self.T = T = -(-N // 128)
        self.o = torch.empty_like(self.qd)
        self.tau = torch.empty((B, H, N), dtype=torch.float32, device=dev)
        self.mask = torch.empty((B, H, T, T), dtype=torch.uint8, device=dev)
        self.dq, self.dk, self.dv = (torch.empty_like(self.qd) for _ in range(3))
        self.wsf = A.workspace(capi.ent_attn_fwd_workspace_size(B, H, N, d, dt_code), dev)
        self.wsb = A.workspace(capi.ent_attn_bwd_workspace_size(B, H, N, d, dt_code), dev)
        self.admissible = B * H * (T * (T + 1) // 2 if w.causal else T * T)
        self.delta_why = "requested"
        if delta == "auto":
            # Measured on B200: delta from otilde makes the dense-block workloads 2-4 %
            # faster per step (the backward drops S and dP of every live block, the
            # forward adds one G V product per live block); at 95 % block sparsity the
            # saving no longer pays for the forward's extra work.  Where nearly every row
            # has at most 16 nonzeros the support lists replace the block backward.  One
            # untimed forward of each kind measures the sparsity and the list coverage.
            A.entmax_attn_fwd(self.qd, self.kd, self.vd, w.alpha, w.causal, ws=self.wsf,
                              out=(self.o, self.tau, self.mask, None))
            sp0 = 1.0 - int(self.mask.sum().item()) / self.admissible
            cover = 0.0
            if w.dtype == "bf16":
                lists = A.alloc_lists(self.qd)
                A.entmax_attn_fwd(self.qd, self.kd, self.vd, w.alpha, w.causal, ws=self.wsf,
                                  out=(self.o, self.tau, self.mask, None), lists=lists)
                # fraction of query tiles whose rows all have lists (the list kernel's tiles)
                ln = lists[2]
                T_ = -(-N // 128)
                pad = torch.full((B, H, T_ * 128), 0, dtype=torch.uint8, device=dev)
                pad[:, :, :N] = ln
                cover = (pad.view(B, H, T_, 128) != 255).all(dim=3).float().mean().item()
                del lists
            delta = "lists" if cover >= 0.9 else "otilde" if sp0 < 0.5 else "recompute"
            self.delta_why = (f"auto: block sparsity {sp0:.3f}, query tiles with every row's "
                              f"support list {cover:.3f}, of untimed forwards")
        self.delta = delta
        # otilde = G V / sum g (float32, like q) when the backward takes delta from it
        self.ot = (torch.empty(self.qd.shape, dtype=torch.float32, device=dev)
                   if delta == "otilde" else None)
        self.lists = A.alloc_lists(self.qd) if delta == "lists" else None
        if delta == "lists":
            self.wsb = A.workspace(capi.ent_attn_bwd_lists_workspace_size(B, H, N, d, dt_code), dev)

    def fwd(self, iters=None):
        from adaptive_sparse_flash_entmax_b200 import attention as A
        w = self.w
        A.entmax_attn_fwd(self.qd, self.kd, self.vd, w.alpha, w.causal, ws=self.wsf,
                          out=(self.o, self.tau, self.mask, iters), otilde=self.ot, lists=self.lists)

    def bwd(self):
        from adaptive_sparse_flash_entmax_b200 import attention as A
        w = self.w
        A.entmax_attn_bwd(self.qd, self.kd, self.vd, self.o, self.dod, self.tau, self.mask,
                          w.alpha, w.causal, ws=self.wsb, out=(self.dq, self.dk, self.dv),
                          otilde=self.ot, lists=self.lists)

    def step(self):
        self.fwd()
        self.bwd()

    def work(self):
        """Counters, block sparsity, element density and solver passes of one untimed step."""
        import torch
        from adaptive_sparse_flash_entmax_b200 import attention as A
        w = self.w
        B, H, N, d = w.shape
        it = torch.empty((B, H, N), dtype=torch.uint8, device=self.dev)
        self.fwd(iters=it)
        cf = A.read_status(self.wsf)
        self.bwd()
        cb = A.read_status(self.wsb)
        blk = 2.0 * 128 * 128 * d
        fwd_flops = blk * (cf[0] + 2 * cf[1] + cf[5])
        # block products of the backward kernels, plus 8 d flops per support-list entry
        # (dP, dQ, dK and dV terms of one nonzero)
        bwd_flops = blk * cb[4] + 8.0 * d * cb[7]
        live = int(self.mask.sum().item())
        itf = it.float()
        hist = torch.bincount(it.reshape(-1).long(), minlength=1).tolist()
        return {"fwd_flops": fwd_flops, "bwd_flops": bwd_flops, "exec_flops": fwd_flops + bwd_flops,
                "counters_fwd": cf, "counters_bwd": cb,
                "block_sparsity": 1.0 - live / self.admissible,
                "element_density": element_density(self.qd, self.kd, self.tau, w.alpha, w.causal),
                "tau_passes": {"row_mean": itf.mean().item(), "row_max": int(itf.max().item()),
                               "tile_mean": cf[2] / max(1, cf[3]),
                               "row_histogram": {str(k): c for k, c in enumerate(hist) if c}}}

    def time_steps(self, steps, stream):
        """Device time of `steps` back-to-back steps: (total ms, mean fwd ms, mean bwd ms)."""
        import torch
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for s in range(steps):
            ev[s][0].record(stream)
            self.fwd()
            ev[s][1].record(stream)
            self.bwd()
            ev[s][2].record(stream)
        t1.record(stream)
        torch.cuda.synchronize()
        return (t0.elapsed_time(t1), statistics.mean(e[0].elapsed_time(e[1]) for e in ev),
                statistics.mean(e[1].elapsed_time(e[2]) for e in ev))


def sweep_point(name, change, seed, dev, steps, peaks):
    """One point of the sweep: the fwd + bwd step of a workload, its work, and the
    dense softmax comparator on the same tensors.  Step time and effective-dense
    TFLOP/s lead; executed TFLOP/s (which counts the method's own recomputation)
    follows."""
    import torch
    w = inputs.WORKLOADS[name].replace(**change) if change else inputs.WORKLOADS[name]
    c = Case(w, seed, dev)
    for _ in range(3):
        c.step()
    torch.cuda.synchronize()
    wk = c.work()
    stream = torch.cuda.current_stream(dev)
    tot, ms_f, ms_b = c.time_steps(steps, stream)
    ms = tot / steps
    comp = time_dense_comparator(c.qd, c.kd, c.vd, c.dod, w.causal, steps)
    exec_tf = wk["exec_flops"] / (ms * 1e-3) / 1e12
    out = {"workload": f"{w.name} B{w.B} H{w.H} N{w.N} d{w.d} alpha {w.alpha} beta {w.beta}"
                       + (f" span {w.span}" if w.kind == "clustered" else ""),
           "ms_per_step": ms, "ms_fwd": ms_f, "ms_bwd": ms_b,
           "effective_dense_tflops": dense_flops(w) / (ms * 1e-3) / 1e12,
           "ms_over_dense_softmax": (ms / comp["ms_per_step"]) if "ms_per_step" in comp else None,
           "dense_softmax_ms": comp.get("ms_per_step"),
           "block_sparsity": wk["block_sparsity"],
           "element_density": wk["element_density"],
           "executed_tflops": exec_tf,
           "executed_frac_of_bf16_peak": exec_tf / peaks["bf16_tflops"],
           "fwd_executed_tflops": wk["fwd_flops"] / (ms_f * 1e-3) / 1e12,
           "bwd_executed_tflops": wk["bwd_flops"] / (ms_b * 1e-3) / 1e12,
           "target_regime": wk["block_sparsity"] >= 0.6,
           "tau_passes": wk["tau_passes"],
           "delta": c.delta}
    del c
    torch.cuda.empty_cache()
    return out


def run_ours(args):
    if args.hist_budget is not None:   # read by the library at each forward call
        os.environ["ENTATTN_HIST_BUDGET"] = str(args.hist_budget)
    import torch
    import torch.distributed as dist

    from adaptive_sparse_flash_entmax_b200 import attention as A
    from adaptive_sparse_flash_entmax_b200 import capi

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
    capi.load()
    w = workload(args)
    B, H, N, d = w.shape
    c = Case(w, args.seed + rank, dev, delta=args.delta, keep_host=True)
    for _ in range(max(3, args.warmup)):
        c.step()
    torch.cuda.synchronize()
    wk = c.work()
    exec_flops = wk["exec_flops"]

    stream = torch.cuda.current_stream(dev)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        elapsed, ms_fwd, ms_bwd = c.time_steps(args.steps, stream)
    if world > 1:
        dist.barrier()
    ms_total, flops_all = combine_ranks(elapsed, exec_flops, world, dev)
    ms_step = ms_total / args.steps
    timed_region_s = elapsed * 1e-3

    peaks, peak_kind = measured_peaks()
    sustained = None
    if world == 1 and args.sustained_s > 0:
        # the same step back to back for seconds, clocks sampled throughout: the
        # forward's rate there is compared with the sustained (power-capped) peak
        n_sus = max(1, int(math.ceil(args.sustained_s * 1e3 / ms_step)))
        with ClockSampler(local) as clk2:
            tot2, f2, b2 = c.time_steps(n_sus, stream)
        fwd_tf2 = wk["fwd_flops"] / (f2 * 1e-3) / 1e12
        sus_peak = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])
        sustained = {"seconds": tot2 * 1e-3, "steps": n_sus, "ms_per_step": tot2 / n_sus,
                     "ms_fwd": f2, "ms_bwd": b2, "fwd_executed_tflops": fwd_tf2,
                     "fwd_frac_of_sustained_peak": fwd_tf2 / sus_peak,
                     "sustained_peak": sus_peak, "clocks": clk2.summary()}

    # end to end through the public API from pinned host memory: every step copies its
    # inputs (Q, K, V, dO) in, runs forward + backward and copies O, dQ, dK, dV out.
    # Consecutive steps overlap: copy-in, compute and copy-out run on three streams with
    # two buffer sets, so step i+1's inputs travel while step i computes (the copies of
    # a step still happen inside the timed region, each exactly once).
    tdt = c.qd.dtype
    host = c.host
    T_ = c.T
    outs_host = [[torch.empty(c.qd.shape, dtype=tdt).pin_memory() for _ in range(4)] for _ in range(2)]
    h2d = sum(h.numel() * h.element_size() for h in host)
    d2h = sum(x.numel() * x.element_size() for x in outs_host[0])
    s_in, s_cmp, s_out = (torch.cuda.Stream(dev) for _ in range(3))
    din = [[torch.empty_like(x) for x in (c.qd, c.kd, c.vd, c.dod)] for _ in range(2)]
    dout = [(torch.empty_like(c.qd), torch.empty((B, H, N), dtype=torch.float32, device=dev),
             torch.empty((B, H, T_, T_), dtype=torch.uint8, device=dev),
             torch.empty_like(c.qd), torch.empty_like(c.kd), torch.empty_like(c.vd)) for _ in range(2)]
    ot = c.ot

    def e2e_run(n):
        done_cmp, done_out = [], []
        for i in range(n):
            bset = i % 2
            e_in = torch.cuda.Event()
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(done_cmp[i - 2])   # inputs of this buffer set consumed
                for dst, src in zip(din[bset], host):
                    dst.copy_(src, non_blocking=True)
                e_in.record(s_in)
            with torch.cuda.stream(s_cmp):
                s_cmp.wait_event(e_in)
                if i >= 2:
                    s_cmp.wait_event(done_out[i - 2])  # outputs of this buffer set copied out
                qq, kk, vv, dd = din[bset]
                oo, tt, mm, g1, g2, g3 = dout[bset]
                A.entmax_attn_fwd(qq, kk, vv, w.alpha, w.causal, ws=c.wsf, out=(oo, tt, mm, None),
                                  otilde=ot, lists=c.lists)
                A.entmax_attn_bwd(qq, kk, vv, oo, dd, tt, mm, w.alpha, w.causal, ws=c.wsb, otilde=ot,
                                  lists=c.lists, out=(g1, g2, g3))
                done_cmp.append(torch.cuda.Event())
                done_cmp[-1].record(s_cmp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(done_cmp[i])
                for dst, src in zip(outs_host[bset], (oo, g1, g2, g3)):
                    dst.copy_(src, non_blocking=True)
                done_out.append(torch.cuda.Event(enable_timing=True))
                done_out[-1].record(s_out)
        return done_out[-1]

    e2e_run(2)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    e1 = e2e_run(args.e2e_steps)
    torch.cuda.synchronize()
    ms_e2e, _ = combine_ranks(e0.elapsed_time(e1) / args.e2e_steps, exec_flops, world, dev)
    del din, dout, outs_host

    comparator = None
    if not args.no_comparator and w.dtype == "bf16":
        comparator = time_dense_comparator(c.qd, c.kd, c.vd, c.dod, w.causal, min(args.steps, 20))
        if "ms_per_step" in comparator:
            comparator["ours_over_dense"] = ms_step / comparator["ms_per_step"]
        comparator["what"] = ("torch SDPA softmax attention fwd+bwd on the same tensors "
                              "(measurement context, not the method)")

    sm_max = peaks.get("sm_max_mhz", 1965.0)
    rowop = None
    if not args.no_rowop:
        rowop = time_row_entmax(dev, args.seed, peaks["hbm_gbs"])
    fwd_tflops = wk["fwd_flops"] / (ms_fwd * 1e-3) / 1e12
    if w.dtype == "bf16":
        # tcgen05 forward: executed MMA flops against the measured bf16 tensor peak; the
        # burst figure, because the timed region lasts well under the seconds it takes
        # the 1 kW power cap to pull the clock down (the sustained run above is compared
        # with the sustained figure)
        use_sus = timed_region_s >= 5.0
        roof = {"kernel": "tc_fwd_kernel: statistics + solver + P.V passes (tcgen05/TMEM/TMA)"
                          + ("; G.V for otilde" if ot is not None else ""),
                "bound": "tensor", "achieved": fwd_tflops,
                "peak": peaks["bf16_tflops_sustained"] if use_sus else peaks["bf16_tflops"],
                "unit": "TFLOP/s",
                "peak_source": f"{peak_kind} " + (
                    "bf16_tflops_sustained" if use_sus else
                    f"bf16_tflops (burst; the timed region lasts {timed_region_s:.2f} s)"),
                "achieved_what": "executed MMA flops of the forward (2*128*128*d per block "
                                 "product, counted by the kernel) / mean forward launch time "
                                 "over the timed region"}
    else:
        alu_peak = 148 * 128 * 2 * sm_max * 1e6 / 1e12   # FP32 FMA, all SMs, max clock
        roof = {"kernel": "simt_fwd_kernel: FP32 CUDA-core forward", "bound": "alu",
                "achieved": fwd_tflops, "peak": alu_peak, "unit": "TFLOP/s",
                "peak_source": "148 SMs x 128 FP32 lanes x 2 flop x %.0f MHz" % sm_max}
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["traffic"] = profiled_traffic(w, roof["kernel"].split(":")[0],
                                       "otilde" if ot is not None else "plain")
    value = flops_all / (ms_step * 1e-3) / 1e12
    c_why, c_delta = c.delta_why, c.delta
    del c
    torch.cuda.empty_cache()
    sweep = None
    if world == 1 and not args.no_sweep and w.dtype == "bf16":
        sweep = [sweep_point(n, ch, args.seed, dev, args.sweep_steps, peaks) for n, ch in SWEEP]
    line = None
    if rank == 0:
        clocks = clk.summary()
        cpu = None
        if world == 1 and not args.no_cpu_baseline:
            heads = min(args.cpu_heads, B * H)
            dt_cpu, cores = oracle_sample(w, heads, args.seed)
            frac = heads / (B * H)
            cpu = {"value": dense_flops(w) * frac / dt_cpu / 1e12, "unit": UNIT, "cores": cores,
                   "kind": "oracle",
                   "sample": f"float64 oracle fwd+bwd on {heads} of {B * H} heads of the same "
                             f"workload ({dt_cpu:.1f} s measured); value = dense-equivalent "
                             "flops of those heads (14 N^2 d / 2 per causal head, as "
                             "effective_dense_tflops and the reference arm) / oracle time"}
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f32" if w.dtype == "f32" else "bf16 inputs, f32 accumulate",
            "data": "synthetic",
            "config": config_of(w, world, {"delta": {
                "otilde": "from the forward's otilde = G V / sum g (ent_attn_fwd_otilde, "
                          "ent_attn_bwd_otilde)",
                "recompute": "recomputed by a pass over the live keys",
                "lists": "per row from the support lists (ent_attn_fwd_lists, ent_attn_bwd_lists) "
                         "where every row of the query tile has one, else block kernels"}[c_delta]
                + f" [{c_why}]"}),
            "ms_fwd": ms_fwd, "ms_bwd": ms_bwd,
            "executed_tflop_per_step": flops_all / 1e12,
            "effective_dense_tflops": world * dense_flops(w) / (ms_step * 1e-3) / 1e12,
            "pct_bf16_peak_executed": 100 * value / world / peaks["bf16_tflops"],
            "pct_bf16_nominal_executed": 100 * value / world / NOMINAL_BF16_TFLOPS,
            "block_sparsity": wk["block_sparsity"],
            "element_density": {"value": wk["element_density"],
                                "what": "fraction of admissible pairs with p > 0, first 2 heads"},
            "tau_passes": wk["tau_passes"],
            "dense_softmax_comparator": comparator,
            "rowwise_entmax": rowop,
            "roofline": roof,
            "sustained": sustained,
            "sweep": sweep,
            "cpu_baseline": cpu,
            "e2e": {"value": flops_all / (ms_e2e * 1e-3) / 1e12, "unit": UNIT,
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": ms_e2e},
            "gpu_launches": launches_per_step(w.dtype, c_delta, -(-N // 128)) * args.steps,
            "clocks": clocks,
            "timed_region_s": timed_region_s,
            "peaks": {"source": peak_kind, "bf16_tflops": peaks["bf16_tflops"],
                      "bf16_tflops_sustained": peaks.get("bf16_tflops_sustained"),
                      "hbm_gbs": peaks["hbm_gbs"]},
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return line


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
