#!/usr/bin/env python3
"""Attention forward throughput on B200: one JSON line.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

A step is one attention forward pass (attn_fwd through the C ABI) over the
headline workload: B=4, H=16, N=8192, d=128, bf16, non-causal, seeded N(0,1)
inputs.  ``value`` is TFLOP/s (4*B*H*N^2*d per step, halved for causal) over
all ranks, with the inputs resident in HBM; ``e2e`` is the same metric when
every step copies Q, K, V from pinned host memory and reads O and LSE back.
The same line carries the causal and FP8 variants, the roofline of the
kernel, clock samples taken during the timed region and (rank 0, one GPU) the
CPU oracle timed on a bounded sample of the same workload.

``--impl reference`` times the CPU oracle alone (fp64 definition, numpy) on a
bounded sample of the workload and prints its line in the same metric.

Multi-GPU (torchrun): every rank runs the same per-rank workload on its own
GPU with no data exchange (weak scaling); the timed region is bracketed by a
barrier and device synchronisation and the time is the max over ranks.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from io_aware_attention_02_b200 import inputs  # noqa: E402

WORKLOAD = dict(B=4, H=16, N=8192, d=128)
SPEC_BF16_TFLOPS = 2250.0
SPEC_FP8_TFLOPS = 4500.0
FALLBACK_BF16_TFLOPS = 1590.0
METRIC = "attention fwd TFLOP/s on 1 B200 and % of dense BF16/FP8 tensor peak"

# DRAM bytes per launch of the bf16 d=128 non-causal kernel on the workload
# above, from the ncu DRAM capture of this kernel (`ncu --metrics
# dram__bytes_read.sum,dram__bytes_write.sum`), keyed by the sha256 of the
# kernel source it was measured on: reported only while the source is unchanged.
TRAFFIC = {"94b24a8bc775b81d": 518538496}


def flops(B, H, N, d, causal):
    f = 4.0 * B * H * N * N * d
    return f / 2 if causal else f


def quant_roofline(B, H, N, d, n_tensors, ms, hbm_gbs):
    """HBM roofline of the FP8 quantiser over `n_tensors` [B, H, N, d] bf16
    tensors: algorithmic bytes = 2 read + 1 written per element plus one fp32
    scale per 128-row block, over the measured time."""
    nbytes = n_tensors * (3.0 * B * H * N * d + 4.0 * B * H * ((N + 127) // 128))
    gbs = nbytes / (ms * 1e-3) / 1e9
    return {"quant_bytes": nbytes, "quant_GBs": gbs, "quant_frac_of_measured_hbm": gbs / hbm_gbs}


def kernel_source_hash():
    h = hashlib.sha256()
    for f in ("fwd_sm100.cuh", "ptx.cuh"):
        with open(os.path.join(ROOT, "io_aware_attention_02_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return json.load(f), "measured"
    except (OSError, ValueError):
        return {"bf16_tflops": FALLBACK_BF16_TFLOPS, "hbm_gbs": 6650.0}, "fallback"


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled during the timed region."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int, period_ms: int = 100):
        self.index, self.period_ms, self.proc = index, period_ms, None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", f"-lms={self.period_ms}"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [l for l in out.splitlines() if l.strip()]
        return False

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in getattr(self, "lines", []):
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for name, val in zip(names, f[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------------------
# distributed plumbing
# ---------------------------------------------------------------------------

def dist_setup(n_gpus, backend="nccl"):
    """One process per GPU: (world, rank, local rank) from the torchrun env.

    The process group only carries barriers and the one-scalar max of the
    timings: the per-rank workloads are independent (no data exchange).
    """
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        kw = {}
        if backend == "nccl":
            torch.cuda.set_device(local)
            kw["device_id"] = torch.device("cuda", local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120), **kw)
    elif backend == "nccl":
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x, world):
    """Max of a per-rank scalar over all ranks (the job time is the slowest rank's)."""
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_seed(rank):
    """Each rank draws its own batch (weak scaling: same per-rank work)."""
    return rank


def job_throughput(per_rank_flops, world, max_ms):
    """Whole-job TFLOP/s: all ranks' work over the slowest rank's time."""
    return world * per_rank_flops / (max_ms * 1e-3) / 1e12


def timed(fn, steps, warmup, world):
    """Device time of `steps` calls of fn (ms), max over ranks."""
    for _ in range(warmup):
        fn()
    barrier(world)
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    for _ in range(steps):
        fn()
    e.record()
    torch.cuda.synchronize()
    barrier(world)
    return max_over_ranks(s.elapsed_time(e), world)


# ---------------------------------------------------------------------------
# CPU oracle baseline (rank 0, one GPU only)
# ---------------------------------------------------------------------------

def oracle_sample(q, k, v, causal, budget_s=15.0, gpu_out=None, single_thread=True):
    """Time the fp64 oracle on a bounded sample of the workload.

    Whole heads (every query row) while the budget allows more than four of
    them, else sampled rows of four heads; sized so the work takes roughly
    `budget_s`.  With `single_thread`, also times 64 rows on one thread.  Returns the cpu_baseline
    dict (value in TFLOP/s, same convention as the GPU figure, counted on the
    rows computed).
    """
    from oracle import attention as A
    try:
        from threadpoolctl import threadpool_info, threadpool_limits
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:  # pragma: no cover
        threadpool_limits = None
        cores = len(os.sched_getaffinity(0))
    B, H, N, d = q.shape
    scale = 1.0 / math.sqrt(d)
    # calibrate (after one warm call) on 256 rows of one head
    rows = inputs.sample_rows(N, 256, seed=11)
    A.attention_head(q[0, 0], k[0, 0], v[0, 0], scale, causal, rows[:16])
    t0 = time.perf_counter()
    A.attention_head(q[0, 0], k[0, 0], v[0, 0], scale, causal, rows)
    per_row = (time.perf_counter() - t0) / len(rows)
    per_head = per_row * N
    if 4 * per_head <= budget_s:
        n_heads = int(min(B * H, max(4, budget_s // per_head)))
        rows = np.arange(N, dtype=np.int64)
    else:
        n_heads = 4
        rows = inputs.sample_rows(N, int(max(64, min(N, budget_s / per_row / 4))), seed=12)
    heads = [(i % B, (i * 5 + i // B) % H) for i in range(n_heads)]
    errs = []
    t0 = time.perf_counter()
    for b, h in heads:
        o, l = A.attention_head(q[b, h], k[b, h], v[b, h], scale, causal, rows)
        if gpu_out is not None:
            og = gpu_out[0][b, h][rows].double().cpu().numpy()
            lg = gpu_out[1][b, h][rows].double().cpu().numpy()
            errs.append((np.abs(og - o).max(), np.mean((og - o) ** 2), np.abs(lg - l).max()))
    dt = time.perf_counter() - t0
    # flops of the rows computed: 4*N*d per row (non-causal), halved for causal
    # exactly as the throughput convention does
    f = len(heads) * len(rows) * 4.0 * N * d / (2 if causal else 1)
    out = {"value": f / dt / 1e12, "unit": "TFLOP/s", "cores": int(cores), "kind": "oracle",
           "sample": f"{len(rows)} query rows x {len(heads)} heads of B={B},H={H},N={N},d={d} "
                     f"{'causal' if causal else 'non-causal'} (numpy fp64, full keys)",
           "seconds": dt,
           # every row costs the same here (all keys scored, then masked), so the
           # whole workload's time is the per-row time times all B*H*N rows
           "extrapolated_full_workload_s": dt / (len(heads) * len(rows)) * B * H * N}
    if single_thread and threadpool_limits is not None:
        rows1 = inputs.sample_rows(N, 64, seed=13)
        with threadpool_limits(limits=1):
            t1 = time.perf_counter()
            A.attention_head(q[0, 0], k[0, 0], v[0, 0], scale, causal, rows1)
            dt1 = time.perf_counter() - t1
        out["single_thread"] = {"value": len(rows1) * 4.0 * N * d / (2 if causal else 1) / dt1 / 1e12,
                                "unit": "TFLOP/s", "sample": f"{len(rows1)} rows of one head"}
    if errs:
        e = np.array(errs)
        out["parity_sample"] = {"max_abs_dO": float(e[:, 0].max()),
                                "rmse_dO": float(math.sqrt(e[:, 1].mean())),
                                "max_abs_dLSE": float(e[:, 2].max())}
    return out


# ---------------------------------------------------------------------------
# arms
# ---------------------------------------------------------------------------

def run_reference(args, world, rank):
    if rank != 0:
        return
    W = WORKLOAD
    q, k, v = inputs.qkv(W["B"], W["H"], W["N"], W["d"], seed=0)
    per_step = []
    cb = None
    # each step is a bounded sample, sized so that the whole run stays within
    # about --ref-total seconds of CPU work
    budget = max(0.05, min(args.ref_budget, args.ref_total / (args.steps + args.warmup)))
    for _ in range(args.warmup):
        oracle_sample(q, k, v, False, budget_s=budget, single_thread=False)
    for _ in range(args.steps):
        cb = oracle_sample(q, k, v, False, budget_s=budget, single_thread=False)
        per_step.append(cb["seconds"])
    val = cb["value"]
    line = {"impl": "reference", "metric": METRIC, "value": val, "unit": "TFLOP/s", "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1000 * statistics.mean(per_step), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": "B=4,H=16,N=8192,d=128 bf16 inputs, non-causal", **W,
                       "causal": False},
            "cpu_baseline": {k2: cb[k2] for k2 in ("value", "unit", "cores", "kind", "sample")},
            "e2e": {"value": val, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def time_shape(B, H, N, d, causal, dev, steps, warmup, world):
    """TFLOP/s of attn_fwd on one shape with timing-only inputs (torch.randn
    bf16 on the device): a few steps, enough for a stable device time."""
    from io_aware_attention_02_b200 import binding
    g = torch.Generator(device=dev).manual_seed(0)
    q, k, v = (torch.randn(B, H, N, d, device=dev, dtype=torch.bfloat16, generator=g) for _ in range(3))
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
    f = flops(B, H, N, d, causal)
    n = max(3, min(steps, int(2e13 / f)))
    ms = timed(lambda: binding.fwd(q, k, v, causal=causal, out=o, lse=lse), n, warmup, world) / n
    return {"tflops": f / (ms * 1e-3) / 1e12, "ms": ms, "steps": n,
            "pct_of_spec_bf16_peak": 100 * f / (ms * 1e-3) / 1e12 / SPEC_BF16_TFLOPS,
            "shape": f"B={B},H={H},N={N},d={d},{'causal' if causal else 'non-causal'}",
            "inputs": "torch.randn bf16 (timing only)"}


def time_fp8_shape(B, H, N, d, causal, dev, steps, warmup, world):
    """TFLOP/s of attn_fwd_fp8 on one shape, the e4m3 operands resident:
    timing-only inputs (torch.randn bf16 with 0.1 % of the entries scaled by
    10), Q and K rotated, 128 x d block scales."""
    from io_aware_attention_02_b200 import binding
    g = torch.Generator(device=dev).manual_seed(0)
    xs = []
    for _ in range(3):
        x = torch.randn(B, H, N, d, device=dev, dtype=torch.float32, generator=g)
        hit = torch.rand(B, H, N, d, device=dev, generator=g) < 1e-3
        xs.append(torch.where(hit, x * 10.0, x).to(torch.bfloat16))
        del x, hit
    signs = torch.from_numpy(inputs.hadamard_signs(d, seed=0)).to(dev)
    q8, qs = binding.quant_fp8(xs[0], hadamard=True, signs=signs)
    k8, ks = binding.quant_fp8(xs[1], hadamard=True, signs=signs)
    v8, vs = binding.quant_fp8(xs[2])
    o = torch.empty_like(xs[0])
    del xs
    lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
    f = flops(B, H, N, d, causal)
    n = max(3, min(steps, int(2e13 / f)))
    ms = timed(lambda: binding.fwd_fp8(q8, k8, v8, qs, ks, vs, causal=causal, out=o, lse=lse), n, warmup,
               world) / n
    return {"tflops": f / (ms * 1e-3) / 1e12, "ms": ms, "steps": n,
            "pct_of_spec_fp8_peak": 100 * f / (ms * 1e-3) / 1e12 / SPEC_FP8_TFLOPS,
            "shape": f"B={B},H={H},N={N},d={d},{'causal' if causal else 'non-causal'}",
            "inputs": "torch.randn bf16 with 0.1% entries x10, quantised once (timing only)"}


def run_ours(args, world, rank, local):
    from io_aware_attention_02_b200 import binding
    binding.load()
    W = WORKLOAD
    B, H, N, d = W["B"], W["H"], W["N"], W["d"]
    dev = torch.device("cuda", local)
    q, k, v = inputs.qkv(B, H, N, d, seed=rank_seed(rank))
    qd, kd, vd = (t.to(dev) for t in (q, k, v))
    o = torch.empty_like(qd)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
    f_nc = flops(B, H, N, d, False)

    if args.only == "decode":
        DB, DH, DNk = 8, 32, args.decode_nk
        qdec = torch.randn(DB, DH, 1, d, device=dev, dtype=torch.bfloat16)
        kdec = torch.randn(DB, DH, DNk, d, device=dev, dtype=torch.bfloat16)
        vdec = torch.randn_like(kdec)
        odec = torch.empty_like(qdec)
        ldec = torch.empty((DB, DH, 1), dtype=torch.float32, device=dev)
        nsd = int(binding.lib().attn_fwd_splitkv_auto_splits(DB, DH, 1, DNk))
        wsd = torch.empty(int(binding.lib().attn_fwd_splitkv_workspace_bytes(DB, DH, 1, d, nsd)),
                          dtype=torch.uint8, device=dev)
        ms_dec = timed(lambda: binding.fwd_splitkv(qdec, kdec, vdec, causal=True, n_splits=nsd, out=odec,
                                                   lse=ldec, workspace=wsd), args.steps, args.warmup, world) / args.steps
        code, where = binding.last_status()
        if code != 0:
            raise RuntimeError(f"kernel status {code} at {where}")
        if rank == 0:
            print(json.dumps({"metric": "split-KV decode K/V read GB/s", "unit": "GB/s",
                              "value": world * 2 * DB * DH * DNk * d * 2 / (ms_dec * 1e-3) / 1e9,
                              "ms_per_step": ms_dec, "splits": nsd, "steps": args.steps, "only": "decode"}),
                  flush=True)
        return

    if args.only == "bwd":
        dod = inputs.grad_out(B, H, N, d, seed=rank_seed(rank)).to(dev)
        binding.fwd(qd, kd, vd, out=o, lse=lse)
        grads = [torch.empty_like(qd) for _ in range(3)]
        ws = torch.empty(binding.bwd_workspace_bytes(B, H, N, d, False), dtype=torch.uint8, device=dev)

        def step_b():
            binding.bwd(qd, kd, vd, o, dod, lse, dq=grads[0], dk=grads[1], dv=grads[2], workspace=ws)
        ms_b = timed(step_b, args.steps, args.warmup, world) / args.steps
        code, where = binding.last_status()
        if code != 0:
            raise RuntimeError(f"kernel status {code} at {where}")
        if rank == 0:
            print(json.dumps({"metric": "attention bwd TFLOP/s (5 products, 10*B*H*N^2*d)",
                              "value": job_throughput(2.5 * f_nc, world, ms_b), "unit": "TFLOP/s",
                              "ms_per_step": ms_b, "steps": args.steps, "only": "bwd"}), flush=True)
        return

    if args.only in ("fp8", "quant"):
        # profiler runs of the FP8 path at the headline shape: outlier inputs,
        # Q and K rotated, 128 x d block scales
        qo, ko, vo = (t.to(dev) for t in inputs.qkv(B, H, N, d, seed=rank_seed(rank), outliers=True))
        signs = torch.from_numpy(inputs.hadamard_signs(d, seed=0)).to(dev)
        q8, qs = binding.quant_fp8(qo, hadamard=True, signs=signs)
        k8, ks = binding.quant_fp8(ko, hadamard=True, signs=signs)
        v8, vs = binding.quant_fp8(vo)
        if args.only == "fp8":
            def step_p():
                binding.fwd_fp8(q8, k8, v8, qs, ks, vs, out=o, lse=lse)
            fl = f_nc
        else:
            def step_p():
                binding.quant_fp8(qo, hadamard=True, signs=signs, out=q8, descale=qs)
                binding.quant_fp8(ko, hadamard=True, signs=signs, out=k8, descale=ks)
                binding.quant_fp8(vo, out=v8, descale=vs)
            fl = 0.0
        ms_p = timed(step_p, args.steps, args.warmup, world) / args.steps
        code, where = binding.last_status()
        if code != 0:
            raise RuntimeError(f"kernel status {code} at {where}")
        if rank == 0:
            print(json.dumps({"only": args.only, "ms_per_step": ms_p, "steps": args.steps,
                              "tflops": fl / (ms_p * 1e-3) / 1e12 if fl else None,
                              "quant_GBs": None if fl else 3 * (3.0 * B * H * N * d) / (ms_p * 1e-3) / 1e9}),
                  flush=True)
        return

    if args.only in ("d64", "d256", "causal", "long", "fp8d64", "fp8d256"):
        SB, SH, SN, Sd, sc = {"d64": (8, 16, 8192, 64, False), "d256": (2, 16, 8192, 256, False),
                              "causal": (B, H, N, d, True), "long": (1, 32, 65536, 128, True),
                              "fp8d64": (8, 16, 8192, 64, False), "fp8d256": (2, 16, 8192, 256, False)}[args.only]
        timer = time_fp8_shape if args.only.startswith("fp8") else time_shape
        r = timer(SB, SH, SN, Sd, sc, dev, args.steps, args.warmup, world)
        code, where = binding.last_status()
        if code != 0:
            raise RuntimeError(f"kernel status {code} at {where}")
        if rank == 0:
            print(json.dumps({"only": args.only, **r}), flush=True)
        return

    def step():
        binding.fwd(qd, kd, vd, causal=False, out=o, lse=lse)

    with ClockSampler(local) as clk:
        ms = timed(step, args.steps, args.warmup, world)
    ms_step = ms / args.steps
    value = job_throughput(f_nc, world, ms_step)
    code, where = binding.last_status()
    if code != 0:
        raise RuntimeError(f"kernel status {code} at {where}")

    if args.only == "main":
        if rank == 0:
            print(json.dumps({"metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
                              "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
                              "only": "main"}), flush=True)
        return

    # causal variant, same shape
    def step_c():
        binding.fwd(qd, kd, vd, causal=True, out=o, lse=lse)
    ms_c = timed(step_c, max(3, args.steps // 2), args.warmup, world) / max(3, args.steps // 2)
    tf_c = flops(B, H, N, d, True) / (ms_c * 1e-3) / 1e12

    # backward (attn_bwd: dQ, dK, dV from dO, O and LSE), same shape; the
    # nominal count is five N x N x d products, 2.5x the forward's
    dod = inputs.grad_out(B, H, N, d, seed=rank_seed(rank)).to(dev)
    dq, dk, dv = (torch.empty_like(qd) for _ in range(3))
    bwd_ms = {}
    for causal, det in ((False, False), (True, False), (False, True)):
        ws = torch.empty(binding.bwd_workspace_bytes(B, H, N, d, det), dtype=torch.uint8, device=dev)
        o_b, lse_b = torch.empty_like(qd), torch.empty_like(lse)
        binding.fwd(qd, kd, vd, causal=causal, out=o_b, lse=lse_b)

        def step_bwd():
            binding.bwd(qd, kd, vd, o_b, dod, lse_b, causal=causal, dq=dq, dk=dk, dv=dv, workspace=ws,
                        deterministic=det)
        nb = max(3, args.steps // 8)
        bwd_ms[(causal, det)] = timed(step_bwd, nb, args.warmup, world) / nb
        del o_b, lse_b, ws
    code, where = binding.last_status()
    if code != 0:
        raise RuntimeError(f"backward kernel status {code} at {where}")
    del dq, dk, dv, dod

    # decode shape through the split-KV path: one query per (b, h) against a
    # 32K-token KV cache; HBM-bound (K and V read once)
    DB, DH, DNk = 8, 32, 32768
    qdec = torch.randn(DB, DH, 1, d, device=dev, dtype=torch.bfloat16)
    kdec = torch.randn(DB, DH, DNk, d, device=dev, dtype=torch.bfloat16)
    vdec = torch.randn_like(kdec)
    odec = torch.empty_like(qdec)
    ldec = torch.empty((DB, DH, 1), dtype=torch.float32, device=dev)
    nsd = int(binding.lib().attn_fwd_splitkv_auto_splits(DB, DH, 1, DNk))
    wsd = torch.empty(int(binding.lib().attn_fwd_splitkv_workspace_bytes(DB, DH, 1, d, nsd)), dtype=torch.uint8,
                      device=dev)

    def step_dec():
        binding.fwd_splitkv(qdec, kdec, vdec, causal=True, n_splits=nsd, out=odec, lse=ldec, workspace=wsd)
    nd = max(3, args.steps // 4)
    ms_dec = timed(step_dec, nd, args.warmup, world) / nd
    code, where = binding.last_status()
    if code != 0:
        raise RuntimeError(f"split-KV kernel status {code} at {where}")
    kv_bytes_dec = 2 * DB * DH * DNk * d * 2
    del qdec, kdec, vdec, odec, ldec, wsd

    # sequence-sweep points at 8K tokens (B*N = 16K, H = 16) for head dims 64
    # and 256, and the long-context case; timing-only inputs (torch.randn)
    shape_var = {}
    for name, (SB, SH, SN, Sd, sc) in {
            "bf16_d64_B2H16N8192": (2, 16, 8192, 64, False), "bf16_d64_B2H16N8192_causal": (2, 16, 8192, 64, True),
            "bf16_d256_B2H16N8192": (2, 16, 8192, 256, False),
            "bf16_d256_B2H16N8192_causal": (2, 16, 8192, 256, True),
            "bf16_long_B1H32N65536_d128_causal": (1, 32, 65536, 128, True)}.items():
        shape_var[name] = time_shape(SB, SH, SN, Sd, sc, dev, args.steps, args.warmup, world)
    for name, (SB, SH, SN, Sd, sc) in {
            "fp8_e4m3_d64_B2H16N8192": (2, 16, 8192, 64, False),
            "fp8_e4m3_d256_B2H16N8192": (2, 16, 8192, 256, False)}.items():
        shape_var[name] = time_fp8_shape(SB, SH, SN, Sd, sc, dev, args.steps, args.warmup, world)
    code, where = binding.last_status()
    if code != 0:
        raise RuntimeError(f"kernel status {code} at {where}")

    # FP8 variant: outlier inputs, Hadamard rotation of Q and K, 128 x d block scales
    qo, ko, vo = (t.to(dev) for t in inputs.qkv(B, H, N, d, seed=rank_seed(rank), outliers=True))
    signs = torch.from_numpy(inputs.hadamard_signs(d, seed=0)).to(dev)
    q8, qs = binding.quant_fp8(qo, hadamard=True, signs=signs)
    k8, ks = binding.quant_fp8(ko, hadamard=True, signs=signs)
    v8, vs = binding.quant_fp8(vo)
    o8 = torch.empty_like(qo)

    def step_fp8():
        binding.fwd_fp8(q8, k8, v8, qs, ks, vs, causal=False, out=o8, lse=lse)
    n8 = max(3, args.steps // 2)
    ms_8 = timed(step_fp8, n8, args.warmup, world) / n8

    def step_fp8_vt():
        binding.fwd_fp8(q8, k8, v8, qs, ks, vs, causal=False, v_transpose=True, out=o8, lse=lse)
    ms_8t = timed(step_fp8_vt, n8, args.warmup, world) / n8

    def step_quant():
        binding.quant_fp8(qo, hadamard=True, signs=signs, out=q8, descale=qs)
        binding.quant_fp8(ko, hadamard=True, signs=signs, out=k8, descale=ks)
        binding.quant_fp8(vo, out=v8, descale=vs)
    ms_q = timed(step_quant, n8, args.warmup, world) / n8
    tf_8 = f_nc / (ms_8 * 1e-3) / 1e12

    # e2e: pinned host inputs in, O and LSE out, every step, through
    # attn_fwd_host (head chunks: copies in, compute and copies out overlap)
    qh, kh, vh = (t.pin_memory() for t in (q, k, v))
    oh = torch.empty(q.shape, dtype=q.dtype).pin_memory()
    lh = torch.empty((B, H, N), dtype=torch.float32).pin_memory()
    ws_h = torch.empty(int(binding.lib().attn_fwd_host_workspace_bytes(B, H, N, d)), dtype=torch.uint8, device=dev)

    def step_e2e():
        binding.fwd_host(qh, kh, vh, causal=False, out=oh, lse=lh, workspace=ws_h, device=dev)
    n_e = max(3, args.steps // 4)
    ms_e = timed(step_e2e, n_e, min(args.warmup, 3), world) / n_e
    e2e_val = job_throughput(f_nc, world, ms_e)
    h2d = 3 * q.numel() * q.element_size()
    d2h = o.numel() * o.element_size() + lse.numel() * 4

    peaks, src = measured_peaks()
    peak = float(peaks.get("bf16_tflops", FALLBACK_BF16_TFLOPS))
    achieved = f_nc / (ms_step * 1e-3) / 1e12
    khash = kernel_source_hash()
    traffic = TRAFFIC.get(khash)

    if rank != 0:
        return
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic: seeded N(0,1) fp32 rounded to bf16",
        "config": {"workload": "B=4,H=16,N=8192,d=128 bf16 non-causal", **W, "causal": False,
                   "parallelism": f"replicas x{world} (independent batches, no exchange)",
                   "l2": "inputs 384 MiB + output 128 MiB per step exceed the 126 MB L2; no flush"},
        "pct_of_spec_bf16_peak": 100.0 * value / world / SPEC_BF16_TFLOPS,
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak, "traffic": traffic,
                     "peak_source": f"{src} bf16_tflops (burst cuBLAS 8192^3)",
                     "algorithmic_flops_per_launch": f_nc, "kernel_source": khash},
        "variants": {
            **shape_var,
            "bf16_causal": {"tflops": tf_c, "ms": ms_c,
                            "pct_of_spec_bf16_peak": 100 * tf_c / SPEC_BF16_TFLOPS},
            "bf16_backward_noncausal": {"tflops": 2.5 * f_nc / (bwd_ms[(False, False)] * 1e-3) / 1e12,
                                        "ms": bwd_ms[(False, False)], "kernels_per_call": 3,
                                        "path": "fused, dQ summed by fp32 TMA reduce-add"},
            "bf16_backward_causal": {"tflops": 2.5 * flops(B, H, N, d, True) / (bwd_ms[(True, False)] * 1e-3) / 1e12,
                                     "ms": bwd_ms[(True, False)], "kernels_per_call": 3,
                                     "path": "fused, dQ summed by fp32 TMA reduce-add"},
            "bf16_backward_noncausal_deterministic": {
                "tflops": 2.5 * f_nc / (bwd_ms[(False, True)] * 1e-3) / 1e12, "ms": bwd_ms[(False, True)],
                "kernels_per_call": 2, "path": "dQ kernel then dK/dV kernel, no atomics"},
            "bf16_decode_splitkv": {
                "shape": f"B={DB},H={DH},Nq=1,Nk={DNk},d={d} causal (inputs torch.randn)",
                "splits": nsd, "ms": ms_dec, "kv_read_GBs": kv_bytes_dec / (ms_dec * 1e-3) / 1e9,
                "frac_of_measured_hbm": kv_bytes_dec / (ms_dec * 1e-3) / 1e9 / float(peaks.get("hbm_gbs", 6650.0)),
                "kernels_per_call": 2},
            "fp8_e4m3_hadamard_noncausal": {
                "tflops": tf_8, "ms": ms_8, "pct_of_spec_fp8_peak": 100 * tf_8 / SPEC_FP8_TFLOPS,
                "quant_ms_qkv": ms_q,
                **quant_roofline(B, H, N, d, 3, ms_q, float(peaks.get("hbm_gbs", 6650.0))),
                "tflops_incl_quant": f_nc / ((ms_8 + ms_q) * 1e-3) / 1e12,
                "tflops_v_transpose": f_nc / (ms_8t * 1e-3) / 1e12,
                "inputs": "N(0,1) with 0.1% entries replaced by N(0,10^2)"},
        },
        "e2e": {"value": e2e_val, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": ms_e},
        "gpu_launches": args.steps,
        "clocks": clk.summary(),
    }
    if world == 1 and not args.no_cpu_baseline:
        # oh / lh hold the last e2e step's result for these same inputs
        line["cpu_baseline"] = oracle_sample(q, k, v, False, budget_s=args.ref_budget, gpu_out=(oh, lh))
    print(json.dumps(line), flush=True)


def run_sweep(args):
    """TFLOP/s of attn_fwd over the sequence sweep (total tokens B*N = 16K,
    H = 16, d in {64, 128, 256}, causal and not) and the long-context case
    (B=1, H=32, N=65536, d=128, causal); one JSON line per configuration."""
    from io_aware_attention_02_b200 import binding
    torch.cuda.set_device(0)
    cases = [(16384 // n, 16, n, d, c) for d in (64, 128, 256) for n in (512, 1024, 2048, 4096, 8192, 16384)
             for c in (False, True)]
    cases.append((1, 32, 65536, 128, True))
    for B, H, N, d, causal in cases:
        g = torch.Generator(device="cuda").manual_seed(0)
        q, k, v = (torch.randn(B, H, N, d, device="cuda", dtype=torch.bfloat16, generator=g) for _ in range(3))
        o = torch.empty_like(q)
        lse = torch.empty((B, H, N), dtype=torch.float32, device="cuda")
        steps = max(5, min(200, int(2e13 / flops(B, H, N, d, causal))))
        ms = timed(lambda: binding.fwd(q, k, v, causal=causal, out=o, lse=lse), steps, 5, 1) / steps
        tf = flops(B, H, N, d, causal) / (ms * 1e-3) / 1e12
        print(json.dumps({"sweep": True, "B": B, "H": H, "N": N, "d": d, "causal": causal, "ms": ms,
                          "tflops": tf, "pct_of_spec_bf16_peak": 100 * tf / SPEC_BF16_TFLOPS,
                          "data": "torch.randn bf16 (timing only)"}), flush=True)
        del q, k, v, o, lse
    code, where = binding.last_status()
    if code != 0:
        raise RuntimeError(f"kernel status {code} at {where}")


def run_ablation(args):
    """The pages' ablation shape {B=4, N=8448, H=16, d=128}, non-causal, bf16:
    one kernel (attn_fwd) with its two query tiles in ping-pong (the tensor
    core works on one tile while the other tile's softmax runs) and with the
    tiles serialised by attn_debug_set_ablation(1) (no product overlaps a
    softmax).  Runs alternate A/B/A/B in one process; one JSON line with the
    medians."""
    from io_aware_attention_02_b200 import binding
    torch.cuda.set_device(0)
    B, H, N, d = 4, 16, 8448, 128
    g = torch.Generator(device="cuda").manual_seed(0)
    q, k, v = (torch.randn(B, H, N, d, device="cuda", dtype=torch.bfloat16, generator=g) for _ in range(3))
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device="cuda")

    def arm(mode):
        def fn():
            binding.fwd(q, k, v, out=o, lse=lse)
        def run():
            binding.debug_set_ablation(mode)
            try:
                return timed(fn, steps, 3, 1) / steps
            finally:
                binding.debug_set_ablation(0)
        return run
    arms = {"pingpong_two_tiles": arm(0), "serialised_tiles": arm(1)}
    res = {name: [] for name in arms}
    steps = max(5, args.steps // 20)
    for _ in range(4):
        for name, run in arms.items():
            res[name].append(run())
    code, where = binding.last_status()
    if code != 0:
        raise RuntimeError(f"kernel status {code} at {where}")
    f = flops(B, H, N, d, False)
    print(json.dumps({"ablation": True, "B": B, "H": H, "N": N, "d": d, "causal": False,
                      **{name: {"ms": statistics.median(v), "tflops": f / (statistics.median(v) * 1e-3) / 1e12}
                         for name, v in res.items()},
                      "data": "torch.randn bf16 (timing only)"}), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=600)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--ref-budget", type=float, default=30.0,
                    help="seconds of CPU work per oracle sample")
    ap.add_argument("--ref-total", type=float, default=150.0,
                    help="seconds of CPU work for the whole reference arm")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--only", choices=["all", "main", "bwd", "decode", "fp8", "quant", "d64", "d256", "causal",
                                       "long", "fp8d64", "fp8d256"], default="all",
                    help="main: time only the bf16 non-causal step; bwd: only the fused bf16 "
                         "non-causal backward of the same workload; decode: only the split-KV decode "
                         "variant; fp8 / quant: only the FP8 forward / the FP8 quantisation of Q, K, V; "
                         "d64 (B=8, N=8K), d256 (B=2, N=8K), causal, long (B=1, H=32, N=64K causal): "
                         "only that bf16 forward; fp8d64 (B=8, N=8K), fp8d256 (B=2, N=8K): only that FP8 "
                         "forward (for profiler runs)")
    ap.add_argument("--decode-nk", type=int, default=32768,
                    help="KV length of the --only decode run (smaller for profiler captures)")
    ap.add_argument("--sweep", action="store_true",
                    help="print TFLOP/s for the sequence sweep and the long-context case instead")
    ap.add_argument("--ablation", action="store_true",
                    help="print the ping-pong ablation at the pages' {4, 8448, 16, 128} shape instead")
    args = ap.parse_args()
    if args.sweep:
        run_sweep(args)
        return
    if args.ablation:
        run_ablation(args)
        return
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        # the CPU oracle: rank 0 alone works, other ranks exit without work
        run_reference(args, 1, int(os.environ.get("RANK", "0")))
        return
    world, rank, local = dist_setup(args.gpus)
    try:
        run_ours(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
