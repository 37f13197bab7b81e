#!/usr/bin/env python
"""Throughput of the dynamic block-sparse attention pipeline on B200.

One step = the whole path on one batch: pooled block scores + row softmax
(dsa_pool_score), Top-p selection to CSR (dsa_select_topp), block-sparse
attention forward (dsa_attn_fwd) and exact block mass (dsa_block_mass), on
seeded synthetic Q/K/V already resident in HBM.

Metric: executed attention TFLOP/s, 4 * sum over selected (i, j) of
|B_i| |B_j| D, divided by the whole step's device time; the attention kernel
alone is reported against the measured bf16 tensor peak, and the step is
compared with a dense p = 1 run of the same kernel (all blocks selected).

Multi-GPU (torchrun): every rank runs its own batch (seed + rank), with no
collective on the data path; the JSON value is the sum of executed FLOPs
over the max step time across ranks ("weak" scaling).

--impl reference times the fp64 CPU oracle on a bounded sample of the same
workload (rank 0 only).
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time
from typing import Tuple

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch  # noqa: E402

from dynamic_block_sparse_pool_b200 import ops, synth  # noqa: E402

METRIC = "block-sparse attn fwd TFLOP/s (executed) & % bf16 peak; speedup vs p=1"
# pool_means, block_scores, select, csr_scan, compact, row_order, attn_fwd, block_mass
LAUNCHES_PER_STEP = 8
ATTN_SOURCE = os.path.join(ROOT, "dynamic_block_sparse_pool_b200", "csrc", "attn_sm100.cu")
# DRAM bytes per attention launch from an ncu capture, keyed by the sha256
# prefix of attn_sm100.cu at capture time: (workload, p, seed, heads of the
# capture, bytes read + written).  Reported only for that workload, p and
# seed, scaled by the number of heads (traffic grows with the heads); stale
# entries are ignored.
ATTN_TRAFFIC = {
    # 8-head Wan2.1-like capture: 539.2 MB read + 500.2 MB written
    "2de04737e0c4a4a4": ("wan2.1-14b-like", 0.9, 0, 8, 539209728 + 500218880),
}


def parse_args():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=("dsa", "reference"), default="dsa")
    ap.add_argument("--workload", default=synth.WAN21.name, choices=sorted(synth.WORKLOADS))
    ap.add_argument("--p", type=float, default=0.9)
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--heads", type=int, default=0,
                    help="use only this many heads of the workload (profiling captures)")
    ap.add_argument("--no-dense", action="store_true", help="skip the p=1 reference run")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer end-to-end run")
    ap.add_argument("--no-cpu", action="store_true", help="skip the oracle cpu_baseline")
    ap.add_argument("--sweep", action="store_true",
                    help="instead of the bench line: one JSON line per point of the "
                         "p-sweep, reduced search, HunyuanVideo schedule and CogVideoX runs")
    ap.add_argument("--profile-rows", action="store_true",
                    help="instead of the bench line: run the kernels of the step policy, "
                         "token reordering, two-level estimate and backward once each on "
                         "a moderate case (for an ncu launch list)")
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="target CPU time of the oracle sample")
    return ap.parse_args()


# --------------------------------------------------------------------- utils --

def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return dict(bf16_burst=float(d["bf16_tflops"]),
                    bf16_sustained=float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                    sustained_sm_mhz=d.get("clocks_under_load", {}).get("sm_mhz_median"),
                    hbm=float(d["hbm_gbs"]), source="measured")
    return dict(bf16_burst=1590.0, bf16_sustained=1400.0, hbm=6650.0, source="fallback")


def attn_source_hash():
    with open(ATTN_SOURCE, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def executed_flops(row_ptr, col_idx, N, block, D, nB):
    """4 * D * sum over selected (row, col) of |B_row| * |B_col| (exact, int64)."""
    sizes = torch.full((nB,), block, dtype=torch.int64, device=row_ptr.device)
    sizes[-1] = N - (nB - 1) * block
    rp = row_ptr.long()
    nnz = int(rp[-1])
    counts = rp[1:] - rp[:-1]
    rows = torch.arange(counts.numel(), device=rp.device)
    qs = sizes[rows % nB]
    ks = sizes[col_idx[:nnz].long()]
    per_row = torch.zeros(counts.numel(), dtype=torch.int64, device=rp.device)
    per_row.index_add_(0, torch.repeat_interleave(rows, counts), ks)
    return int(4 * D * (qs * per_row).sum().item()), nnz


class ClockSampler:
    """nvidia-smi samples every 200 ms while the timed region runs."""

    FIELDS = ("index,uuid,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.proc = None
        self.uuid = None
        try:
            self.uuid = "GPU-" + str(torch.cuda.get_device_properties(device_index).uuid)
        except Exception:
            pass

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=10)
        except Exception:
            self.proc.kill()
            out, _ = self.proc.communicate()
        rows = [[c.strip() for c in line.split(",")] for line in out.splitlines() if line.strip()]
        if self.uuid:
            mine = [r for r in rows if len(r) > 1 and r[1] == self.uuid]
            rows = mine or rows
        if not rows:
            return None
        try:
            sm = [float(r[2]) for r in rows]
            mx = max(float(r[3]) for r in rows)
            pw = [float(r[4]) for r in rows]
        except (ValueError, IndexError):
            return None
        thr = 0.5 * max(pw)
        load = [r for r, p in zip(rows, pw) if p >= thr] or rows
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in load for n, v in zip(names, r[6:10]) if v.lower().startswith("active")})
        return {"sm_mhz": statistics.median(float(r[2]) for r in load), "sm_max_mhz": mx,
                "reasons": reasons, "samples": len(rows), "samples_under_load": len(load),
                "power_w_max": max(pw)}


def dist_setup(backend: str = "nccl"):
    """Process group from the torchrun environment (one rank per GPU)."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import torch.distributed as dist
        kw = {}
        if backend == "nccl":
            torch.cuda.set_device(local)
            kw["device_id"] = torch.device("cuda", local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300), **kw)
    return world, rank, local


def _reduce(x: float, world: int, op: str) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX if op == "max" else dist.ReduceOp.SUM)
    return float(t.item())


def reduce_max(x: float, world: int) -> float:
    """Max over ranks (the job's time is its slowest rank's)."""
    return _reduce(x, world, "max")


def reduce_sum(x: float, world: int) -> float:
    """Sum over ranks (each rank runs its own batch)."""
    return _reduce(x, world, "sum")


def job_throughput(local_ms: float, local_flops: float, world: int) -> Tuple[float, float, float]:
    """(TFLOP/s of the whole job, max step ms over ranks, total FLOPs)."""
    ms = reduce_max(local_ms, world)
    flops = reduce_sum(local_flops, world)
    return flops / (ms * 1e-3) / 1e12, ms, flops


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ------------------------------------------------------------- oracle sample --

def oracle_sample(w, q, k, v, p, seconds, head=0):
    """Time the CPU oracle on one head: its own pooled scores, softmax and
    Top-p for every row, then attention + block mass for query-block rows
    spread over the head until about `seconds` of CPU time is spent.
    Returns (tflops, description, threads)."""
    import numpy as np
    from oracle import dsa_oracle as O
    try:
        from threadpoolctl import threadpool_info
        threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        threads = os.cpu_count() or 1
    f64 = lambda t: t.float().numpy().astype(np.float64)
    qh, kh, vh = f64(q[0, head]), f64(k[0, head]), f64(v[0, head])
    scale = 1.0 / math.sqrt(w.head_dim)
    nB = w.n_blocks
    t0 = time.perf_counter()
    P = O.block_probs(O.pool_blocks(qh, w.block), O.pool_blocks(kh, w.block), scale)
    rp, col = O.topp_select(P.astype(np.float32), p)
    t_search = time.perf_counter() - t0
    order = list(range(0, nB, max(1, nB // 64))) + [nB - 1]
    seen, rows, flops = set(), [], 0
    t_attn = 0.0
    for i in order:
        if i in seen:
            continue
        seen.add(i)
        t1 = time.perf_counter()
        Oo, lo, blk = O.sparse_attention_head(qh, kh, vh, w.block, scale, rp, col, rows=[i])
        O.block_mass(lo, blk, rp, w.N, w.block)
        t_attn += time.perf_counter() - t1
        a, b = i * w.block, min(w.N, (i + 1) * w.block)
        flops += sum(4 * w.head_dim * (b - a) * (min(w.N, (j + 1) * w.block) - j * w.block)
                     for j in col[rp[i]:rp[i + 1]])
        rows.append(i)
        if t_attn + t_search >= seconds:
            break
    t_total = t_attn + t_search * len(rows) / nB
    desc = (f"oracle (NumPy fp64) on head {head} of {w.name}: pooled scores, softmax and "
            f"exact Top-p for all {nB} rows ({t_search:.2f} s, pro-rated), then attention on "
            f"{len(rows)} of {nB} query-block rows ({t_attn:.2f} s); "
            f"{flops / 1e9:.1f} GFLOP executed")
    return flops / t_total / 1e12, desc, threads, t_total


def run_reference(args, world, rank):
    if rank != 0:
        return
    w = synth.WORKLOADS[args.workload]
    q, k, v = synth.make_qkv(w, args.seed, heads=[0])
    per_step = max(1.0, args.cpu_seconds / 4)
    for _ in range(args.warmup):
        oracle_sample(w, q, k, v, args.p, per_step / 4)
    vals, times = [], []
    desc, threads = "", 1
    for _ in range(args.steps):
        val, desc, threads, t = oracle_sample(w, q, k, v, args.p, per_step)
        vals.append(val)
        times.append(t)
    value = sum(vals) / len(vals)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * sum(times) / len(times), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_of(w, args),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads,
                         "kind": "oracle", "sample": desc},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def config_of(w, args):
    return {"workload": w.describe(), "p": args.p, "seed": args.seed,
            "batch": w.batch, "heads": w.heads, "tokens": w.N, "head_dim": w.head_dim,
            "block": w.block, "grid": [w.T, w.Hg, w.W], "parallelism": f"replicas{args.gpus}",
            "l2": "inputs larger than L2 (Q,K,V %.2f GB)" % (3 * w.BH * w.N * w.head_dim * 2 / 1e9)}



# --------------------------------------------------------------------- sweep --

def sweep(args):
    """Timing of the measurement plan's points, one JSON line each."""
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)

    def timed(fn, reps):
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(reps)]
        for a, b in ev:
            a.record(stream); fn(); b.record(stream)
        torch.cuda.synchronize(dev)
        return sum(a.elapsed_time(b) for a, b in ev) / reps

    def steady(fn, est_ms, seconds=0.6):
        reps = max(3, int(seconds * 1e3 / max(est_ms, 1e-2)))
        return timed(lambda: [fn() for _ in range(reps)], 1) / reps

    def point(w, q, k, v, p, cand=None, dense=None, label=None, extra=None, hier_sub=None):
        B, H, N, D, blk = w.batch, w.heads, w.N, w.head_dim, w.block
        nB, rows = w.n_blocks, w.BH * w.n_blocks
        scale = 1.0 / math.sqrt(D)
        P = torch.empty(B * H, nB, nB, device=dev)
        wp = torch.empty(ops.workspace_size(0, B, H, N, D, blk), device=dev, dtype=torch.uint8)
        wsel = torch.empty(ops.workspace_size(1, B, H, N, D, blk), device=dev, dtype=torch.uint8)
        rp = torch.empty(rows + 1, device=dev, dtype=torch.int32)
        ci = torch.empty(rows * nB, device=dev, dtype=torch.int32)
        order = torch.empty(rows, device=dev, dtype=torch.int32)
        out = torch.empty_like(q)
        lse = torch.empty(B, H, N, device=dev)
        cap = rows * nB if cand is None else int(cand[0][-1])
        bl = torch.empty(max(cap, 1), blk, device=dev)
        ms_ = torch.empty(max(cap, 1), device=dev)
        if hier_sub is not None:
            wh = torch.empty(ops.workspace_size(2 if hier_sub <= 2 else 3, B, H, N, D, blk),
                             device=dev, dtype=torch.uint8)
            score = lambda: ops.pool_score_hier(q, k, blk, hier_sub, scale, out=P, workspace=wh)
        else:
            score = lambda: ops.pool_score(q, k, blk, scale, cand=cand, out=P, workspace=wp)
        search = lambda: (score(),
                          ops.select_topp(P, p, cand=cand, row_ptr=rp, col_idx=ci, workspace=wsel),
                          ops.row_order(rp, B, H, nB, out=order))
        attend = lambda: ops.attn_fwd(q, k, v, rp, ci, blk, scale, out=out, lse=lse, blk_lse=bl,
                                      order=order)
        mass = lambda: ops.block_mass(lse, bl, rp, blk, mass=ms_)
        search(); attend(); mass(); ops.device_status(dev)
        flops, nnz = executed_flops(rp, ci, N, blk, D, nB)
        reps = 5
        t_s = timed(search, reps)
        t_a = timed(attend, reps)
        t_m = timed(mass, reps)
        step = t_s + t_a + t_m
        if dense is not None:
            # The whole step and the dense p = 1 reference (the same kernel
            # over an all-blocks CSR, with the same outputs), each timed in
            # steady state -- about 0.6 s of back-to-back work, queued ahead
            # -- in two alternating rounds; the second round is kept.  The
            # part is power-capped, so a short burst after a long kernel (or
            # the other way round) would see different clocks.
            step_fn = lambda: (search(), attend(), mass())
            d_est = timed(dense, 1)
            for _ in range(2):
                step_alt = steady(step_fn, step)
                dense_ms = steady(dense, d_est)
        line = {"sweep": label or w.name, "p": p, "reduced_search": cand is not None,
                "density": nnz / (rows * nB), "executed_tflop": flops / 1e12,
                "search_ms": t_s, "attn_ms": t_a, "mass_ms": t_m, "step_ms": step,
                "attn_tflops": flops / (t_a * 1e-3) / 1e12,
                "step_tflops": flops / (step * 1e-3) / 1e12}
        if dense is not None:
            red = (4 * D * B * H * N * N) / flops
            line.update({"dense_attn_ms": dense_ms, "step_ms_steady": step_alt,
                         "flop_reduction": red, "speedup_attn": dense_ms / t_a,
                         "speedup_pipeline": dense_ms / step_alt,
                         "pipeline_over_reduction": dense_ms / step_alt / red})
        if extra:
            line.update(extra)
        print(json.dumps(line), flush=True)
        return rp[: rows + 1].clone(), ci[:nnz].clone(), line

    def dense_of(w, q, k, v):
        B, H, N, D, blk = w.batch, w.heads, w.N, w.head_dim, w.block
        nB, rows = w.n_blocks, w.BH * w.n_blocks
        rpa = (torch.arange(rows + 1, device=dev, dtype=torch.int64) * nB).to(torch.int32)
        cia = torch.arange(nB, device=dev, dtype=torch.int32).repeat(rows)
        out = torch.empty_like(q)
        lse = torch.empty(B, H, N, device=dev)
        bl = torch.empty(rows * nB, blk, device=dev)
        f = lambda: ops.attn_fwd(q, k, v, rpa, cia, blk, 1.0 / math.sqrt(D), out=out,
                                 lse=lse, blk_lse=bl)
        f(); torch.cuda.synchronize(dev)
        return f

    # Wan2.1-like: p sweep, then reduced search
    w = synth.WAN21
    q, k, v = synth.make_qkv(w, 0, device="cuda")
    dms = dense_of(w, q, k, v)
    masks = {}
    for p in w.p:
        masks[p] = point(w, q, k, v, p, dense=dms)[:2]
    # the same point with the two-level (sub-block) estimate
    point(w, q, k, v, 0.9, dense=dms, label=w.name + " two-level estimate (sub 2)", hier_sub=2)
    # the same point on tokens in curve order (dense attention is
    # order-free), plus the cost of gathering Q, K, V and scattering O: the
    # enclosing cube's Hilbert curve, then the generalised curve of the grid
    for curve in ("hilbert", "gilbert"):
        order = ops.HilbertOrder(w.T, w.Hg, w.W, w.n_prefix, device=dev, curve=curve)
        qh, kh, vh = (order.gather(t) for t in (q, k, v))
        oh = torch.empty_like(q)
        perm_ms = timed(lambda: (order.gather(q, out=qh), order.gather(k, out=kh),
                                 order.gather(v, out=vh), order.scatter(qh, out=oh)), 3)
        point(w, qh, kh, vh, 0.9, dense=dms, label=w.name + " " + curve + " order",
              extra={"reorder_ms": perm_ms,
                     "reorder_bytes": 8 * q.numel() * q.element_size()})
        del qh, kh, vh, oh
    q1, k1, v1 = synth.make_qkv(w, 1, device="cuda")
    dms1 = dense_of(w, q1, k1, v1)
    point(w, q1, k1, v1, 0.7, dense=dms1, label=w.name + " seed1 full search")
    point(w, q1, k1, v1, 0.7, cand=masks[0.95], dense=dms1,
          label=w.name + " seed1 reduced search (candidates: seed0 p=0.95 mask)")
    del q, k, v, q1, k1, v1
    torch.cuda.empty_cache()
    # HunyuanVideo-like growing-sparsity schedule
    w = synth.HUNYUAN
    for step, p, bw, seed in synth.hunyuan_schedule(10):
        q, k, v = synth.make_qkv(w, seed, bandwidth=bw, device="cuda")
        dms = dense_of(w, q, k, v) if step in (0, 9) else None
        point(w, q, k, v, round(p, 4), dense=dms, label=f"{w.name} step {step}",
              extra={"bandwidth": bw, "seed": seed})
        del q, k, v
    # CogVideoX-like
    w = synth.COGVIDEOX
    q, k, v = synth.make_qkv(w, 0, device="cuda")
    point(w, q, k, v, 0.9, dense=dense_of(w, q, k, v))
    del q, k, v
    torch.cuda.empty_cache()
    gsrs_run(timed)
    backward_point(timed)


def backward_point(timed):
    """Backward of the attention on the Wan2.1-like grid with 8 heads at
    p = 0.9 (bf16, blocks of 128: the tcgen05 kernels).  Algorithmic FLOPs:
    the five contractions (Q K^T, dO V^T, dS K, dS^T Q, P^T dO) = 2.5 x the
    forward's executed FLOPs.  Executed on the tensor cores: 5 x the
    forward's -- Q K^T and dO V^T are computed on both sides (dq and dkdv
    kernels), and each gradient product runs twice (bf16 hi and lo terms of
    P and dS)."""
    import dataclasses
    dev = torch.device("cuda", 0)
    w = dataclasses.replace(synth.WAN21, heads=8)
    B, H, N, D, blk = w.batch, w.heads, w.N, w.head_dim, w.block
    q, k, v = synth.make_qkv(w, 0, device="cuda")
    scale = 1.0 / math.sqrt(D)
    sa = ops.sparse_attention(q, k, v, 0.9, block=blk, scale=scale)
    dO = torch.randn(q.shape, device=dev, generator=torch.Generator(device=dev).manual_seed(1)).to(q.dtype)
    ws = torch.empty(ops.workspace_size(4, B, H, N, D, blk), device=dev, dtype=torch.uint8)
    f = lambda: ops.attn_bwd(q, k, v, sa.out, dO, sa.lse, sa.row_ptr, sa.col_idx, blk, scale,
                             workspace=ws)
    f()
    ops.device_status(dev)
    t = timed(f, 3)
    fwd, nnz = executed_flops(sa.row_ptr, sa.col_idx, N, blk, D, w.n_blocks)
    peak = measured_peaks()["bf16_burst"]
    line = {"sweep": "backward (tcgen05, P and dS as bf16 hi + lo), wan2.1-like 8 heads", "p": 0.9,
            "nnz_blocks": nnz, "bwd_ms": t, "algorithmic_tflop": 2.5 * fwd / 1e12,
            "bwd_tflops": 2.5 * fwd / (t * 1e-3) / 1e12,
            "executed_tensor_tflops": 5 * fwd / (t * 1e-3) / 1e12,
            "frac_of_bf16_burst_peak_algorithmic": 2.5 * fwd / (t * 1e-3) / 1e12 / peak,
            "frac_of_bf16_burst_peak_executed": 5 * fwd / (t * 1e-3) / 1e12 / peak,
            "bound": "tensor (element-wise P, dS between the products)"}
    print(json.dumps(line), flush=True)


def gsrs_run(timed):
    """The step policy (warm-up, searches on exact block masses, mask reuse)
    over the HunyuanVideo-like 10-step inputs, against full attention at
    every step; each whole run timed twice, alternating, the second kept."""
    from dynamic_block_sparse_pool_b200.schedule import GsrsPolicy, GsrsRunner
    dev = torch.device("cuda", 0)
    w = synth.HUNYUAN
    B, H, N, D, blk = w.batch, w.heads, w.N, w.head_dim, w.block
    nB, rows = w.n_blocks, w.BH * w.n_blocks
    pol = GsrsPolicy(10, 1, (0.95, 0.9, 0.85, 0.8))
    inputs = [synth.make_qkv(w, seed, bandwidth=bw, device="cuda")
              for _, _, bw, seed in synth.hunyuan_schedule(10)]
    run = GsrsRunner(pol, B, H, N, D, blk, w.dtype, device=dev)
    all_rp, all_col = run.all_rp, run.all_col
    out = torch.empty_like(inputs[0][0])
    scale = 1.0 / math.sqrt(D)

    def sparse_run():
        run.have_base, run.cur = False, None
        for s, (q, k, v) in enumerate(inputs):
            run.step(s, q, k, v)

    def dense_run():
        for q, k, v in inputs:
            ops.attn_fwd(q, k, v, all_rp, all_col, blk, scale, out=out, want_lse=False,
                         want_blk_lse=False)

    # executed FLOPs: each step over the mask it attends to
    run.have_base, run.cur = False, None
    flops = 0
    for s, (q, k, v) in enumerate(inputs):
        res = run.step(s, q, k, v)
        flops += executed_flops(res.mask[0], res.mask[1], N, blk, D, nB)[0]
    ops.device_status(dev)
    dense_flops = 10 * 4 * D * B * H * N * N
    for _ in range(2):
        t_sparse = timed(sparse_run, 1)
        t_dense = timed(dense_run, 1)
    red = dense_flops / flops
    line = {"sweep": "step policy on hunyuanvideo-like 10-step inputs", "warmup": pol.warmup,
            "p": list(pol.p), "search_steps": pol.searches(),
            "kinds": [k for k, _ in pol.kinds()], "run_ms": t_sparse, "dense_run_ms": t_dense,
            "executed_tflop": flops / 1e12, "dense_tflop": dense_flops / 1e12,
            "speedup": t_dense / t_sparse, "flop_reduction": red,
            "speedup_over_reduction": t_dense / t_sparse / red,
            "run_tflops": flops / (t_sparse * 1e-3) / 1e12}
    print(json.dumps(line), flush=True)

def profile_rows():
    """One pass of each widening row's calls, sized for an ncu capture: the
    Wan2.1-like grid with 8 heads (Q, K, V 155 MB each, above L2) for the
    token reordering, the two-level estimate and a search step on exact
    block masses; one head for the backward."""
    import dataclasses
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    w = dataclasses.replace(synth.WAN21, heads=8)
    B, H, N, D, blk = w.batch, w.heads, w.N, w.head_dim, w.block
    scale = 1.0 / math.sqrt(D)
    q, k, v = synth.make_qkv(w, 0, device="cuda")
    # token reordering: gather Q into curve order, scatter it back
    order = ops.HilbertOrder(w.T, w.Hg, w.W, w.n_prefix, device=dev)
    qh = order.gather(q)
    back = order.scatter(qh)
    # two-level estimate (sub 2)
    ops.pool_score_hier(q, k, blk, 2, scale)
    # a search step on exact block masses: attention over a p = 0.95 mask,
    # its masses as dense rows, Top-p 0.9 within it
    sa = ops.sparse_attention(q, k, v, 0.95, block=blk, scale=scale)
    nnz = int(sa.row_ptr[-1])
    P = ops.mass_to_probs(sa.row_ptr, sa.col_idx, sa.mass, w.n_blocks)
    rp2, _ = ops.select_topp(P, 0.9, cand=(sa.row_ptr, sa.col_idx))
    ops.device_status(dev)
    ok_perm = bool(torch.equal(back, q))
    del q, k, v, qh, back, sa, P
    # backward on one head at p = 0.9
    w1 = dataclasses.replace(synth.WAN21, heads=1)
    q, k, v = synth.make_qkv(w1, 0, device="cuda")
    s1 = ops.sparse_attention(q, k, v, 0.9, block=blk, scale=scale)
    dO = torch.randn(q.shape, device=dev, generator=torch.Generator(device=dev).manual_seed(1)).to(q.dtype)
    ops.attn_bwd(q, k, v, s1.out, dO, s1.lse, s1.row_ptr, s1.col_idx, blk, scale)
    ops.device_status(dev)
    torch.cuda.synchronize(dev)
    print(json.dumps({"profile_rows": "wan2.1-like", "heads": H, "scatter_inverts_gather": ok_perm,
                      "search_step_mask_nnz": nnz, "reselected_nnz": int(rp2[-1]),
                      "bwd_heads": 1, "bwd_nnz": int(s1.row_ptr[-1])}), flush=True)


# ---------------------------------------------------------------- GPU bench --

def main():
    args = parse_args()
    if args.impl == "reference":
        # CPU-only: rank 0 times the oracle, the other ranks leave at once
        run_reference(args, int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")))
        return
    if args.sweep:
        sweep(args)
        return
    if args.profile_rows:
        profile_rows()
        return
    world, rank, local = dist_setup()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    w = synth.WORKLOADS[args.workload]
    if args.heads:
        import dataclasses
        w = dataclasses.replace(w, heads=args.heads)
    B, H, N, D, blk = w.batch, w.heads, w.N, w.head_dim, w.block
    nB = w.n_blocks
    rows = B * H * nB
    scale = 1.0 / math.sqrt(D)
    q_c, k_c, v_c = synth.make_qkv(w, args.seed + rank)
    q, k, v = q_c.to(dev), k_c.to(dev), v_c.to(dev)

    P = torch.empty(B * H, nB, nB, device=dev, dtype=torch.float32)
    ws_pool = torch.empty(ops.workspace_size(0, B, H, N, D, blk), device=dev, dtype=torch.uint8)
    ws_sel = torch.empty(ops.workspace_size(1, B, H, N, D, blk), device=dev, dtype=torch.uint8)
    row_ptr = torch.empty(rows + 1, device=dev, dtype=torch.int32)
    col_idx = torch.empty(rows * nB, device=dev, dtype=torch.int32)
    out = torch.empty_like(q)
    lse = torch.empty(B, H, N, device=dev, dtype=torch.float32)
    blk_lse = torch.empty(rows * nB, blk, device=dev, dtype=torch.float32)
    mass = torch.empty(rows * nB, device=dev, dtype=torch.float32)
    order = torch.empty(rows, device=dev, dtype=torch.int32)
    stream = torch.cuda.current_stream(dev)

    def search():
        ops.pool_score(q, k, blk, scale, out=P, workspace=ws_pool)
        ops.select_topp(P, args.p, row_ptr=row_ptr, col_idx=col_idx, workspace=ws_sel)
        ops.row_order(row_ptr, B, H, nB, out=order)

    def attend(rp=row_ptr, ci=col_idx, ro=order):
        ops.attn_fwd(q, k, v, rp, ci, blk, scale, out=out, lse=lse, blk_lse=blk_lse, order=ro)

    def finish(rp=row_ptr):
        ops.block_mass(lse, blk_lse, rp, blk, mass=mass)

    # one untimed pass for the mask statistics
    search(); attend(); finish()
    ops.device_status(dev)
    flops, nnz = executed_flops(row_ptr, col_idx, N, blk, D, nB)
    dense_flops = 4 * D * B * H * N * N
    for _ in range(args.warmup):
        search(); attend(); finish()
    torch.cuda.synchronize(dev)

    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    clocks = ClockSampler(local)
    barrier(world)
    torch.cuda.synchronize(dev)
    clocks.start()
    for s in range(args.steps):
        e = ev[s]
        e[0].record(stream); search()
        e[1].record(stream); attend()
        e[2].record(stream); finish()
        e[3].record(stream)
    torch.cuda.synchronize(dev)
    clk = clocks.stop()
    barrier(world)
    ops.device_status(dev)
    t_step = [e[0].elapsed_time(e[3]) for e in ev]
    t_search = [e[0].elapsed_time(e[1]) for e in ev]
    t_attn = [e[1].elapsed_time(e[2]) for e in ev]
    t_mass = [e[2].elapsed_time(e[3]) for e in ev]
    value, ms_step, total_flops = job_throughput(sum(t_step) / len(t_step), float(flops), world)
    ms_attn = sum(t_attn) / len(t_attn)
    attn_tflops = flops / (ms_attn * 1e-3) / 1e12
    peaks = measured_peaks()

    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16" if w.dtype == torch.bfloat16 else "f32", "data": "synthetic",
        "config": config_of(w, args),
        "gpu_launches": LAUNCHES_PER_STEP * args.steps,
    }
    traffic = None
    entry = ATTN_TRAFFIC.get(attn_source_hash())
    if entry is not None:
        name, p_cap, seed_cap, heads_cap, nbytes = entry
        if w.name == name and args.p == p_cap and args.seed == seed_cap and w.batch == 1:
            traffic = int(nbytes * w.heads / heads_cap)
    # The denominator is the measured burst cuBLAS bf16 rate: the sustained
    # figure was taken at a lower median SM clock than this loop runs at, so
    # it would flatter the fraction; it is reported beside it for context.
    line["roofline"] = {
        "bound": "tensor", "kernel": "attn_fwd_sm100_kernel", "achieved": attn_tflops,
        "peak": peaks["bf16_burst"], "unit": "TFLOP/s",
        "frac": attn_tflops / peaks["bf16_burst"],
        "peak_kind": f"{peaks['source']} bf16 burst (cuBLAS 8192^3)",
        "frac_of_sustained_peak": attn_tflops / peaks["bf16_sustained"],
        "sustained_peak_sm_mhz": peaks.get("sustained_sm_mhz"),
        "traffic": traffic,
        "algorithmic_flop_per_launch": flops,
    }
    line["breakdown_ms"] = {"search": sum(t_search) / len(t_search), "attn": ms_attn,
                            "mass": sum(t_mass) / len(t_mass)}
    line["mask"] = {"nnz_blocks": nnz, "density": nnz / (rows * nB),
                    "executed_tflop": flops / 1e12, "dense_tflop": dense_flops / 1e12}
    line["clocks"] = clk

    out_ref = out.clone()  # the p-run's O, before the dense run reuses `out`

    # dense p = 1 reference: the same kernel over an all-blocks CSR.  The part
    # runs at its power cap, so the sparse step and the dense run are timed
    # alternately (three rounds, each about 0.5 s of back-to-back work per
    # arm, the last round kept) so that both see the same clocks.
    if not args.no_dense:
        rp_all = (torch.arange(rows + 1, device=dev, dtype=torch.int64) * nB).to(torch.int32)
        col_all = torch.arange(nB, device=dev, dtype=torch.int32).repeat(rows)
        attend(rp_all, col_all, None)  # equal rows: index order is the longest-first one
        torch.cuda.synchronize(dev)

        def back_to_back(fn, reps):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            for _ in range(reps):
                fn()
            b.record(stream)
            torch.cuda.synchronize(dev)
            return a.elapsed_time(b) / reps

        ms_step_mean = sum(t_step) / len(t_step)
        k_sparse = max(3, int(500.0 / max(ms_step_mean, 1e-3)))
        k_dense = 4
        for _ in range(3):
            ms_sparse_alt = back_to_back(lambda: (search(), attend(), finish()), k_sparse)
            ms_dense = back_to_back(lambda: attend(rp_all, col_all, None), k_dense)
        red = dense_flops / flops
        line["speedup_vs_p1"] = {
            "dense_attn_ms": ms_dense,
            "dense_attn_tflops": dense_flops / (ms_dense * 1e-3) / 1e12,
            "sparse_step_ms_alternated": ms_sparse_alt,
            "attn_only": ms_dense / ms_attn,
            "pipeline": ms_dense / ms_sparse_alt,
            "executed_flop_reduction": red,
            "pipeline_over_reduction": ms_dense / ms_sparse_alt / red,
            "timing": f"alternated: {k_sparse} sparse steps then {k_dense} dense runs, "
                      "3 rounds, last kept",
        }
        del rp_all, col_all

    # end to end through the library's host-buffer call (dsa_sparse_attention_host):
    # pinned Q, K, V in, O out, with the PCIe copies of one chunk of heads
    # overlapping another's compute
    if not args.no_e2e:
        from dynamic_block_sparse_pool_b200.pipeline import HostPipeline
        qh, kh, vh = q_c.pin_memory(), k_c.pin_memory(), v_c.pin_memory()
        oh = torch.empty(q_c.shape, dtype=q_c.dtype).pin_memory()
        del P, ws_pool, ws_sel, col_idx, blk_lse, mass  # make room for the pipeline's slots
        torch.cuda.empty_cache()
        pipe = HostPipeline(B, H, N, D, w.dtype, blk)
        ke = max(2, args.steps // 3)
        ee = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(ke + 1)]
        for s_ in range(ke + 1):  # first iteration is a warm-up
            ee[s_][0].record(stream)
            pipe.run(qh, kh, vh, oh, args.p, scale)
            ee[s_][1].record(stream)
        torch.cuda.synchronize(dev)
        ms_e2e = reduce_max(sum(e[0].elapsed_time(e[1]) for e in ee[1:]) / ke, world)
        line["e2e"] = {"value": total_flops / (ms_e2e * 1e-3) / 1e12, "unit": "TFLOP/s",
                       "ms_per_step": ms_e2e,
                       "api": "dsa_sparse_attention_host (C ABI, host buffers)",
                       "chunk_heads": pipe.chunk,
                       "h2d_bytes_per_step": pipe.h2d_bytes(),
                       "d2h_bytes_per_step": pipe.d2h_bytes()}
        # the chunked host run must reproduce the device-resident run bit for bit
        line["e2e"]["matches_device_run"] = bool(torch.equal(oh.to(dev), out_ref))

    if rank == 0 and world == 1 and not args.no_cpu:
        val, desc, threads, _ = oracle_sample(w, q_c, k_c, v_c, args.p, args.cpu_seconds)
        line["cpu_baseline"] = {"value": val, "unit": "TFLOP/s", "cores": threads,
                                "kind": "oracle", "sample": desc}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
