#!/usr/bin/env python
"""Benchmark: EAGLE-3 mixed joint-softmax attention, forward + backward, on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step = one forward (block-0 causal attention, diagonal fold, normalise,
lse) and one backward (D_t, block-0 dK/dV/dQ against the merged lse, closed
form diagonal grads) over the whole synthetic workload, inputs resident in
HBM.  Prints ONE JSON line on rank 0.

For N > 1 (torchrun, one process per GPU) every rank runs its own replica of
the workload (the path shards over batch and heads with no exchange), so the
scaling is weak and value = all ranks' FLOPs / the max over ranks of the time.

--impl reference times the fp64 CPU oracle on the host cores on a bounded
sample of the same workload (the only reference implementation there is).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

METRIC = "joint-attention fwd+bwd TFLOP/s and tokens/s on 1 B200; % of BF16 tensor peak"
ROOT = os.path.dirname(os.path.abspath(__file__))


def peaks() -> dict:
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d["bf16_tflops_sustained"], "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


# ------------------------------------------------------------- accounting --
def visible_pairs(w) -> int:
    """Allowed (query, key) pairs of block 0 summed over all rows, batches and
    heads (causal triangle incl. the diagonal, per document, global offsets)."""
    t = np.arange(w.Tq, dtype=np.int64)
    qp = w.q_pos_offset + t
    if w.doc_lengths is not None:
        cu = np.concatenate([[0], np.cumsum(w.doc_lengths)]).astype(np.int64)
        d = np.clip(np.searchsorted(cu, qp, side="right") - 1, 0, len(cu) - 2)
        inside = (qp >= 0) & (qp < cu[-1])  # rows outside every document see nothing
        glo = np.where(inside, cu[d], 1 << 60)
        ghi = np.where(inside, cu[d + 1] - 1, -(1 << 60))
    else:
        glo = np.full_like(qp, -(1 << 60))
        ghi = np.full_like(qp, 1 << 60)
    ghi = np.minimum(ghi, qp)
    lo = np.maximum(glo - w.k_pos_offset, 0)
    hi = np.minimum(ghi - w.k_pos_offset, w.tk - 1)
    per_row = np.maximum(hi - lo + 1, 0)
    return int(per_row.sum()) * w.B * w.H


def flops(w) -> dict:
    pairs = visible_pairs(w)
    rows = w.B * w.Tq * w.H
    f = {"pairs": pairs,
         "fwd": 4 * w.D * pairs + 4 * w.D * (w.num_blocks - 1) * rows,
         "bwd": 10 * w.D * pairs + 8 * w.D * (w.num_blocks - 1) * rows if w.backward else 0}
    f["total"] = f["fwd"] + f["bwd"]
    return f


# ---------------------------------------------------------------- clocks --
class Clocks:
    """nvidia-smi sampler started before the warm-up; stop(t0, t1) keeps the
    samples whose timestamps fall inside the timed region [t0, t1] (wall clock)."""
    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.path = tempfile.mktemp(suffix=".csv")
        self.proc = None
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(gpu_index), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "50"], stdout=self.f,
                stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    @staticmethod
    def _when(stamp: str):
        import datetime
        for fmt in ("%Y/%m/%d %H:%M:%S.%f", "%Y/%m/%d %H:%M:%S"):
            try:
                return datetime.datetime.strptime(stamp, fmt).timestamp()
            except ValueError:
                pass
        return None

    def stop(self, t0: float | None = None, t1: float | None = None) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.12)  # let the sampler write the samples that close the window
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.f.close()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 10:
                    continue
                try:
                    rows.append((self._when(parts[0]), float(parts[2]), float(parts[3]),
                                 float(parts[4]), parts[6:10]))
                except ValueError:
                    continue
        os.unlink(self.path)
        inside = [r for r in rows if r[0] is not None and t0 is not None
                  and t0 - 0.05 <= r[0] <= t1 + 0.05]
        window = bool(inside)
        use = inside or [r for r in rows if r[3] > 200] or rows
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = set()
        for r in use:
            for n, v in zip(names, r[4]):
                if v.lower() == "active":
                    reasons.add(n)
        sm = [r[1] for r in use]
        power = [r[3] for r in use]
        smax = rows[-1][2] if rows else None
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "in_timed_region": window,
                "reasons": sorted(reasons), "samples": len(sm),
                "power_w_max": max(power) if power else None}


# ----------------------------------------------------------- DRAM traffic --
# dram__bytes_read.sum + dram__bytes_write.sum per launch of a kernel, from an
# ncu capture (the file names the command); dropped (null) as soon as the
# kernel sources differ from the ones the capture ran.
TRAFFIC_FILE = "profiles/dram_traffic_dense_bf16.json"


def csrc_digest() -> str:
    import hashlib
    root = os.path.dirname(os.path.abspath(__file__))
    src = os.path.join(root, "online_softmax_merge_eagle_b200", "csrc")
    h = hashlib.sha256()
    for name in sorted(os.listdir(src)):
        if name.endswith((".cu", ".cuh")):
            with open(os.path.join(src, name), "rb") as f:
                h.update(name.encode() + b"\0" + f.read())
    with open(os.path.join(root, "include", "eagleattn.h"), "rb") as f:
        h.update(f.read())
    return h.hexdigest()


def dram_traffic(workload: str, kernel: str):
    root = os.path.dirname(os.path.abspath(__file__))
    try:
        with open(os.path.join(root, TRAFFIC_FILE)) as f:
            data = json.load(f)
    except (OSError, ValueError):
        return None
    if data.get("csrc_sha256") != csrc_digest():
        return None
    ent = data.get("workloads", {}).get(workload, {}).get(kernel)
    return None if ent is None else ent.get("bytes_per_launch")


# --------------------------------------------------------------- helpers --
def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def max_over_ranks(x: float, world: int, device) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tflops(world: int, flop_per_rank: float, ms_max: float) -> float:
    """Whole-job throughput: every rank's FLOPs over the slowest rank's time."""
    return world * flop_per_rank / (ms_max * 1e-3) / 1e12


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def cpu_sample_inputs(w, sample_T: int, t=None):
    """The (b=0, h=0) slice of the workload's seeded inputs, first sample_T
    positions (a causal prefix: its rows see only its keys)."""
    from online_softmax_merge_eagle_b200.inputs import make_tensors
    if t is None:
        t = make_tensors(w.B, w.Tq, w.H, w.D, w.num_blocks, w.dtype, Tk=w.tk, seed=w.seed,
                         grad=w.backward)
    n = sample_T
    s = {"q": t["q"][:1, :n, :1].double().numpy(),
         "cache_k": t["cache_k"][:1, :, :(n if w.tk == w.Tq else w.tk), :1].double().numpy(),
         "cache_v": t["cache_v"][:1, :, :(n if w.tk == w.Tq else w.tk), :1].double().numpy()}
    if w.backward:
        s["grad_out"] = t["grad_out"][:1, :n, :1].double().numpy()
    return s


def sample_workload(w, sample_T):
    from dataclasses import replace
    docs = None
    if w.doc_lengths is not None:
        acc, docs = 0, []
        for L in w.doc_lengths:
            if acc >= sample_T:
                break
            docs.append(min(L, sample_T - acc))
            acc += docs[-1]
        docs = tuple(docs)
    Tk = None if w.Tk is None else w.Tk
    return replace(w, B=1, H=1, Tq=sample_T, Tk=Tk, doc_lengths=docs)


def run_oracle_sample(w, s, sample_T):
    import oracle
    sw = sample_workload(w, sample_T)
    cu = None if sw.doc_lengths is None else np.concatenate([[0], np.cumsum(sw.doc_lengths)])
    kw = dict(cu_seqlens=cu, q_pos_offset=w.q_pos_offset, k_pos_offset=w.k_pos_offset)
    t0 = time.perf_counter()
    oracle.fwd(s["q"], s["cache_k"], s["cache_v"], w.scale, **kw)
    if w.backward:
        oracle.bwd(s["q"], s["cache_k"], s["cache_v"], s["grad_out"], w.scale, **kw)
    dt = time.perf_counter() - t0
    return dt, flops(sw)["total"], oracle.get_threads()


CPU_SAMPLE_FLOP = 2.5e11   # ~5 s of the fp64 oracle on 16 host cores
REF_RUN_FLOP = 1.5e12      # whole --impl reference run (warm-up + timed steps)


def default_sample_T(w, budget: float = CPU_SAMPLE_FLOP) -> int:
    """Longest causal prefix of the (b=0, h=0) slice whose oracle work stays
    within `budget` FLOP (multiples of 128 positions, at least 128)."""
    n = w.Tq
    while n > 128 and flops(sample_workload(w, n))["total"] > budget:
        n = max(128, (int(n * 0.8) // 128) * 128)
    return n


# ------------------------------------------------------------- reference --
def reference_arm(args, w, world, rank):
    if rank != 0:
        return 0
    import oracle
    oracle.build()
    # every step is one bounded sample, so that the whole run stays within minutes
    n = default_sample_T(w, REF_RUN_FLOP / max(1, args.steps + args.warmup))
    s = cpu_sample_inputs(w, n)
    for _ in range(args.warmup):
        run_oracle_sample(w, s, n)
    times, fl, cores = [], 0, 1
    for _ in range(args.steps):
        dt, fl, cores = run_oracle_sample(w, s, n)
        times.append(dt)
    tot = sum(times)
    value = fl * args.steps / tot / 1e12
    sample = (f"(b=0,h=0) slice, first {n} positions of workload {w.name}: fwd"
              + ("+bwd" if w.backward else "") + f", {fl:.3e} FLOP per step")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": tot / args.steps * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(w),
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def workload_config(w) -> dict:
    c = {"workload": w.name, "B": w.B, "T": w.Tq, "Tk": w.tk, "H": w.H, "D": w.D,
         "num_blocks": w.num_blocks, "q_pos_offset": w.q_pos_offset,
         "docs": None if w.doc_lengths is None else len(w.doc_lengths),
         "chunks": w.chunks or None, "single_launch": w.single_launch or None,
         "backward": w.backward, "seed": w.seed}
    return c


# ------------------------------------------------------------------ ours --
def make_step(args, w, ea, inp, inp_cpu, dev):
    """Device buffers for workload w and a step(prof) closure that runs one
    forward + backward through the library.  prof = dict of (start, stop)
    torch.cuda.Event pairs: "fwd" and "bwd" bracket the main attention
    kernels (the library records them on its launch stream), "bwd_all" the
    whole backward call."""
    from online_softmax_merge_eagle_b200.schedules import (varlen_zigzag_backward,
                                                           varlen_zigzag_forward, zigzag_backward,
                                                           zigzag_forward)
    cu = None if inp["cu_seqlens"] is None else torch.as_tensor(inp["cu_seqlens"], device=dev)
    kw = dict(cu_seqlens=cu, max_seqlen=inp["max_seqlen"], q_pos_offset=w.q_pos_offset,
              k_pos_offset=w.k_pos_offset, impl=args.kernel_impl)
    q, k, v = inp["q"], inp["cache_k"], inp["cache_v"]
    g = inp.get("grad_out")
    out = torch.empty_like(q)
    lse = torch.empty(w.B, w.H, w.Tq, dtype=torch.float32, device=dev)
    dq = torch.empty_like(q) if w.backward else None
    dk = torch.empty_like(k) if w.backward else None
    dv = torch.empty_like(v) if w.backward else None
    ws = None
    if w.backward:
        ws = torch.empty(ea.bwd_workspace_size(q, k, v, **kw), dtype=torch.uint8, device=dev)
    det = bool(args.deterministic)

    def rec(prof, key, i):
        if prof is not None and key in prof:
            prof[key][i].record()

    def body(prof):
        if w.chunks and w.doc_lengths:
            # packed documents, each through the zig-zag chunk schedule
            cu_h = inp_cpu["cu_seqlens"]
            rec(prof, "fwd", 0)
            varlen_zigzag_forward(q, k, v, w.scale, cu_h, cp=w.chunks // 2,
                                  impl=args.kernel_impl, out=out, lse=lse,
                                  single_launch=w.single_launch)
            rec(prof, "fwd", 1)
            if w.backward:
                rec(prof, "bwd", 0)
                varlen_zigzag_backward(g, q, k, v, out, lse, w.scale, cu_h, cp=w.chunks // 2,
                                       impl=args.kernel_impl, dq=dq, dk=dk, dv=dv,
                                       deterministic=det,
                                       single_launch=w.single_launch and not det)
                rec(prof, "bwd", 1)
            return
        if w.chunks:
            # block 0 through the zig-zag chunk schedule (emulated cp = chunks / 2)
            rec(prof, "fwd", 0)
            zigzag_forward(q, k, v, w.scale, cp=w.chunks // 2, impl=args.kernel_impl, out=out,
                           lse=lse, single_launch=w.single_launch)
            rec(prof, "fwd", 1)
            if w.backward:
                rec(prof, "bwd", 0)
                zigzag_backward(g, q, k, v, out, lse, w.scale, cp=w.chunks // 2,
                                impl=args.kernel_impl, dq=dq, dk=dk, dv=dv, deterministic=det,
                                single_launch=w.single_launch and not det)
                rec(prof, "bwd", 1)
            return
        ea.fwd(q, k, v, w.scale, out=out, lse=lse, prof=None if prof is None else prof["fwd"],
               **kw)
        if w.backward:
            rec(prof, "bwd_all", 0)
            ea.bwd(g, q, k, v, out, lse, w.scale, workspace=ws, dq=dq, dk=dk, dv=dv,
                   prof=None if prof is None else prof["bwd"], deterministic=det, **kw)
            rec(prof, "bwd_all", 1)

    def step(prof=None):
        # NVTX range per step, visible to nsys / ncu --nvtx
        torch.cuda.nvtx.range_push("eagle_step")
        try:
            body(prof)
        finally:
            torch.cuda.nvtx.range_pop()

    return step, kw, (q, k, v)


def time_steps(step, steps, warmup, world, ea):
    """W untimed steps, then exactly `steps` steps between a barrier and a
    synchronize on both sides, timed with CUDA events on the launching stream.
    Returns (ms per step, per-kernel mean ms, launches, wall window)."""
    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    ev = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
    profs = [{key: (ev(), ev()) for key in ("fwd", "bwd", "bwd_all")} for _ in range(steps)]
    barrier(world)
    torch.cuda.synchronize()
    n0 = ea.launch_count()
    t0, t1 = ev(), ev()
    wall0 = time.time()
    t0.record()
    for i in range(steps):
        step(profs[i])
    t1.record()
    torch.cuda.synchronize()
    wall1 = time.time()
    n1 = ea.launch_count()
    barrier(world)

    def mean_ms(key):
        vals = []
        for pr in profs:
            a, b = pr[key]
            try:
                vals.append(a.elapsed_time(b))
            except (RuntimeError, ValueError):  # never recorded (e.g. no backward)
                return 0.0
        return statistics.mean(vals)
    kern = {"fwd_ms": mean_ms("fwd"), "bwd_block0_ms": mean_ms("bwd"),
            "bwd_all_ms": mean_ms("bwd_all")}
    return t0.elapsed_time(t1) / steps, kern, n1 - n0, (wall0, wall1)


def roofline_entry(achieved, peak, unit, bound, per_unit, units, peak_kind):
    return {"bound": bound, "achieved": achieved, "peak": peak, "unit": unit,
            "frac": (achieved / peak) if achieved else None, "peak_kind": peak_kind,
            "per_unit": per_unit, "units_per_launch": units}


def kernel_rooflines(w, fl, kern, pk, det=False):
    """Per-kernel entries: algorithmic work per launch / its mean CUDA-event
    duration, against the measured burst bf16 peak (tensor kernels, timed in
    a sub-second region) or the measured copy bandwidth (row pass)."""
    burst = pk["bf16_tflops"]
    src = " (" + pk["source"] + ")"
    out = {}
    if kern["fwd_ms"] > 0:
        a = fl["fwd"] / (kern["fwd_ms"] * 1e-3) / 1e12
        out["fwd"] = roofline_entry(a, burst, "TFLOP/s", "tensor",
                                    "4*D FLOP per pair + 4*D per row and diagonal block",
                                    fl["pairs"], "bf16_tflops burst" + src)
    if w.backward and kern["bwd_block0_ms"] > 0:
        a = 10 * w.D * fl["pairs"] / (kern["bwd_block0_ms"] * 1e-3) / 1e12
        out["bwd_block0"] = roofline_entry(a, burst, "TFLOP/s", "tensor", "10*D FLOP per pair",
                                           fl["pairs"], "bf16_tflops burst" + src)
    if w.backward and kern["bwd_all_ms"] > kern["bwd_block0_ms"] > 0 and not w.chunks:
        rows = w.B * w.Tq * w.H
        es = 2  # bf16
        per_row = (3 * w.D * es + (w.num_blocks - 1) * 4 * w.D * es + 8
                   + (4 * w.D if w.num_blocks > 1 or not det else 0))
        ms = kern["bwd_all_ms"] - kern["bwd_block0_ms"]
        gbs = rows * per_row / (ms * 1e-3) / 1e9
        e = roofline_entry(gbs, pk["hbm_gbs"], "GB/s", "hbm",
                           "bytes per row: dO, O, q + (NB-1) x (k, v read, dk, dv write) "
                           "+ the fp32 dQ accumulator row written + lse, D_t", rows,
                           "hbm_gbs" + src)
        e["kernel"] = "bwd_rows_kernel (bwd call minus its block-0 kernels)"
        out["bwd_rows"] = e
    return out


def ours_arm(args, w, world, rank, local):
    import online_softmax_merge_eagle_b200 as ea
    from online_softmax_merge_eagle_b200.inputs import WORKLOADS, make_workload

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    pk = peaks()
    inp_cpu = make_workload(w)
    inp = {n: (x.to(dev) if isinstance(x, torch.Tensor) else x) for n, x in inp_cpu.items()}
    step, kw, (q, k, v) = make_step(args, w, ea, inp, inp_cpu, dev)
    fl = flops(w)

    clocks = Clocks(local) if rank == 0 else None  # sampling starts before the warm-up
    ms, kern, launches, (wall0, wall1) = time_steps(step, args.steps, args.warmup, world, ea)
    clk = clocks.stop(wall0, wall1) if clocks else None
    ms_step = max_over_ranks(ms, world, dev)
    fwd_ms, bwd_ms = kern["fwd_ms"], kern["bwd_block0_ms"]

    tflops = job_tflops(world, fl["total"], ms_step)
    tokens = world * w.B * w.Tq / (ms_step * 1e-3)
    fwd_main_tf = fl["fwd"] / (fwd_ms * 1e-3) / 1e12 if fwd_ms > 0 else None
    bwd_main_tf = (10 * w.D * fl["pairs"]) / (bwd_ms * 1e-3) / 1e12 if bwd_ms > 0 else None
    # dominant kernel = the larger share of the step
    if w.backward and bwd_ms >= fwd_ms:
        dom, achieved = "bwd_block0", bwd_main_tf
    else:
        dom, achieved = "fwd", fwd_main_tf
    # the timed region is well under a second: the burst cuBLAS figure applies
    peak = pk["bf16_tflops"]
    per_kernel = kernel_rooflines(w, fl, kern, pk, bool(args.deterministic))

    e2e = e2e_measure(args, w, inp_cpu, kw, ea, dev, fl, world) if not args.no_e2e else None
    merge = merge_measure(ea, dev, pk) if not args.no_merge else None
    if merge:
        per_kernel["merge"] = roofline_entry(merge["GBps"], pk["hbm_gbs"], "GB/s", "hbm",
                                             "D*(4+4+2)+12 bytes per row (bf16 block)",
                                             merge["bytes_per_launch"] // (128 * 10 + 12),
                                             "hbm_gbs (" + pk["source"] + ")")
    del inp, step
    extra = {}
    for name in ([] if args.no_extra else [x for x in args.extra.split(",") if x]):
        if name == w.name:
            continue
        xw = WORKLOADS[name]
        xcpu = make_workload(xw)
        xin = {n: (x.to(dev) if isinstance(x, torch.Tensor) else x) for n, x in xcpu.items()}
        xstep, _, _ = make_step(args, xw, ea, xin, xcpu, dev)
        xfl = flops(xw)
        xms, xkern, _, _ = time_steps(xstep, max(3, args.steps // 2), args.warmup, world, ea)
        xms = max_over_ranks(xms, world, dev)
        extra[name] = {"value": job_tflops(world, xfl["total"], xms), "unit": "TFLOP/s",
                       "ms_per_step": xms, "flop_per_step": xfl,
                       "kernels": {**xkern,
                                   "fwd_tflops": xfl["fwd"] / (xkern["fwd_ms"] * 1e-3) / 1e12
                                   if xkern["fwd_ms"] > 0 else None,
                                   "bwd_block0_tflops": 10 * xw.D * xfl["pairs"] /
                                   (xkern["bwd_block0_ms"] * 1e-3) / 1e12
                                   if xkern["bwd_block0_ms"] > 0 else None},
                       "roofline": kernel_rooflines(xw, xfl, xkern, pk, bool(args.deterministic)),
                       "steps": max(3, args.steps // 2), "warmup": args.warmup}
        del xin, xstep

    if rank != 0:
        return 0
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        import oracle
        oracle.build()
        n = default_sample_T(w)
        s = cpu_sample_inputs(w, n, inp_cpu)
        dt, sfl, cores = run_oracle_sample(w, s, n)
        cpu = {"value": sfl / dt / 1e12, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
               "sample": f"(b=0,h=0) slice, first {n} positions, fwd"
                         + ("+bwd" if w.backward else "") + f"; {sfl:.3e} FLOP in {dt:.2f} s"}
    cfg = workload_config(w)
    cfg["l2"] = "inputs larger than L2 (%.2f GB read per step)" % (
        sum(t.numel() * t.element_size() for t in (q, k, v)) / 1e9)
    cfg["parallelism"] = f"replica x{world}"
    cfg["deterministic_bwd"] = bool(args.deterministic)
    line = {
        "metric": METRIC, "value": tflops, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16" if w.dtype == torch.bfloat16 else "f32", "data": "synthetic",
        "config": cfg,
        "tokens_per_s": tokens,
        "pct_bf16_peak": {"of_measured_burst": tflops / world / pk["bf16_tflops"],
                          "of_measured_sustained": tflops / world / pk["bf16_tflops_sustained"],
                          "of_nominal_2250": tflops / world / 2250.0},
        "flop_per_step": fl,
        "kernels": {"fwd_ms": fwd_ms, "fwd_tflops": fwd_main_tf, "bwd_block0_ms": bwd_ms,
                    "bwd_block0_tflops": bwd_main_tf, "bwd_all_ms": kern["bwd_all_ms"],
                    "impl": args.kernel_impl,
                    "bwd_mode": "deterministic pair" if args.deterministic else
                    "five products per tile pair (dQ by TMA reduce-add)"},
        "roofline": {"bound": "tensor", "kernel": dom, "achieved": achieved, "peak": peak,
                     "unit": "TFLOP/s", "frac": (achieved / peak) if achieved else None,
                     "peak_kind": "bf16_tflops burst (" + pk["source"] + ")",
                     "frac_of_sustained": (achieved / pk["bf16_tflops_sustained"])
                     if achieved else None,
                     "traffic": dram_traffic(w.name, dom),
                     "traffic_source": TRAFFIC_FILE},
        "roofline_per_kernel": per_kernel,
        "cpu_baseline": cpu,
        "e2e": e2e,
        "merge": merge,
        "extra_workloads": extra or None,
        "gpu_launches": launches,
        "clocks": clk,
    }
    print(json.dumps(line), flush=True)
    return 0


def e2e_measure(args, w, inp, kw, ea, dev, fl, world):
    """Same metric through the public API with HOST buffers: every step copies
    that step's inputs from pinned host memory, runs fwd + bwd, and copies
    every result back to pinned host memory.  Device buffers are doubled so
    that step i+1's host->device copy and step i-1's device->host copy run on
    their own streams (PCIe is full duplex) while step i computes."""
    names_in = [n for n in ("q", "cache_k", "cache_v", "grad_out") if n in inp and inp[n] is not None]
    host_in = {n: inp[n].pin_memory() for n in names_in}
    dev_in = [{n: torch.empty_like(inp[n], device=dev) for n in names_in} for _ in range(2)]

    def make_outs(q, k):
        o = {"out": torch.empty_like(q),
             "lse": torch.empty(w.B, w.H, w.Tq, dtype=torch.float32, device=dev)}
        if w.backward:
            o.update(dq=torch.empty_like(q), dk=torch.empty_like(k), dv=torch.empty_like(k))
        return o
    outs = [make_outs(d["q"], d["cache_k"]) for d in dev_in]
    ws = None
    if w.backward:
        d0 = dev_in[0]
        ws = torch.empty(ea.bwd_workspace_size(d0["q"], d0["cache_k"], d0["cache_v"], **kw),
                         dtype=torch.uint8, device=dev)
    host_out = {n: torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for n, t in outs[0].items()}
    h2d = sum(t.numel() * t.element_size() for t in host_in.values())
    d2h = sum(t.numel() * t.element_size() for t in host_out.values())
    compute = torch.cuda.current_stream()
    s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)

    def upload(i):
        with torch.cuda.stream(s_in):
            for n in names_in:
                dev_in[i % 2][n].copy_(host_in[n], non_blocking=True)
            ev = torch.cuda.Event()
            ev.record(s_in)
        return ev

    def run(i):
        d, o = dev_in[i % 2], outs[i % 2]
        if w.chunks and w.doc_lengths:
            from online_softmax_merge_eagle_b200.schedules import (varlen_zigzag_backward,
                                                                   varlen_zigzag_forward)
            varlen_zigzag_forward(d["q"], d["cache_k"], d["cache_v"], w.scale, inp["cu_seqlens"],
                                  cp=w.chunks // 2, out=o["out"], lse=o["lse"],
                                  single_launch=w.single_launch)
            if w.backward:
                varlen_zigzag_backward(d["grad_out"], d["q"], d["cache_k"], d["cache_v"],
                                       o["out"], o["lse"], w.scale, inp["cu_seqlens"],
                                       cp=w.chunks // 2, dq=o["dq"], dk=o["dk"], dv=o["dv"],
                                       single_launch=w.single_launch)
        elif w.chunks:
            from online_softmax_merge_eagle_b200.schedules import zigzag_backward, zigzag_forward
            zigzag_forward(d["q"], d["cache_k"], d["cache_v"], w.scale, cp=w.chunks // 2,
                           out=o["out"], lse=o["lse"], single_launch=w.single_launch)
            if w.backward:
                zigzag_backward(d["grad_out"], d["q"], d["cache_k"], d["cache_v"], o["out"],
                                o["lse"], w.scale, cp=w.chunks // 2, dq=o["dq"], dk=o["dk"],
                                dv=o["dv"], single_launch=w.single_launch)
        else:
            ea.fwd(d["q"], d["cache_k"], d["cache_v"], w.scale, out=o["out"], lse=o["lse"], **kw)
            if w.backward:
                ea.bwd(d["grad_out"], d["q"], d["cache_k"], d["cache_v"], o["out"], o["lse"],
                       w.scale, workspace=ws, dq=o["dq"], dk=o["dk"], dv=o["dv"],
                       deterministic=bool(args.deterministic), **kw)
        ev = torch.cuda.Event()
        ev.record(compute)
        return ev

    def download(i, done):
        with torch.cuda.stream(s_out):
            s_out.wait_event(done)
            for n in host_out:
                host_out[n].copy_(outs[i % 2][n], non_blocking=True)
            ev = torch.cuda.Event()
            ev.record(s_out)
        return ev

    def steps(n):
        # step i: upload(i) -> compute(i) -> download(i); buffers i % 2 are
        # reused by step i + 2 only after step i's compute and download
        s_in.wait_stream(compute)  # nothing starts before the timing event
        up = upload(0)
        comp, down = [None] * n, [None] * n
        for i in range(n):
            compute.wait_event(up)
            if i >= 2:
                compute.wait_event(down[i - 2])  # outputs of slot i % 2 read back
            comp[i] = run(i)
            if i + 1 < n:
                if i >= 1:
                    s_in.wait_event(comp[i - 1])  # inputs of slot (i + 1) % 2 consumed
                up = upload(i + 1)
            down[i] = download(i, comp[i])
        compute.wait_event(down[-1])

    steps(2)
    torch.cuda.synchronize()
    n = max(2, args.e2e_steps)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    a.record(compute)
    steps(n)
    b.record(compute)
    torch.cuda.synchronize()
    ms = max_over_ranks(a.elapsed_time(b) / n, world, dev)
    return {"value": world * fl["total"] / (ms * 1e-3) / 1e12, "unit": "TFLOP/s",
            "ms_per_step": ms, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "steps": n, "overlap": "double-buffered; copies on their own streams"}


def merge_measure(ea, dev, pk):
    """attn_merge_out_lse on one full-tensor merge of the chunked workload
    (1 x 131072 x 8 rows x 128, bf16 block): algorithmic bytes = read out,
    lse, block_out, block_lse + write out, lse."""
    B, T, H, D = 1, 131072, 8, 128
    g = torch.Generator(device=dev).manual_seed(1)
    out = torch.randn(B, T, H, D, device=dev, generator=g)
    lse = torch.randn(B, H, T, device=dev, generator=g)
    bo = torch.randn(B, T, H, D, device=dev, generator=g).to(torch.bfloat16)
    bl = torch.randn(B, H, T, device=dev, generator=g)
    rows = B * T * H
    nbytes = rows * (D * 4 * 2 + D * 2 + 4 * 3)
    for _ in range(3):
        ea.merge_out_lse(out, lse, bo, bl)
    torch.cuda.synchronize()
    n = 20
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(n)]
    for a, b in evs:
        a.record()
        ea.merge_out_lse(out, lse, bo, bl)
        b.record()
    torch.cuda.synchronize()
    ms = statistics.median(a.elapsed_time(b) for a, b in evs)
    gbs = nbytes / (ms * 1e-3) / 1e9
    return {"kernel": "attn_merge_out_lse", "bytes_per_launch": nbytes, "ms": ms, "GBps": gbs,
            "peak_hbm_gbs": pk["hbm_gbs"], "frac": gbs / pk["hbm_gbs"], "frac_of_nominal_8000":
            gbs / 8000.0, "l2": "working set 1.35 GB > L2"}


def main():
    from online_softmax_merge_eagle_b200.inputs import WORKLOADS
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="dense_bf16")
    ap.add_argument("--kernel-impl", choices=["auto", "tensor_core", "generic"], default="auto")
    ap.add_argument("--e2e-steps", type=int, default=6)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-merge", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--deterministic", type=int, default=0,
                    help="1: the reproducible backward pair instead of the five-product kernel")
    ap.add_argument("--extra", default="varlen_bf16",
                    help="comma-separated workloads also timed (device only) in the same run")
    ap.add_argument("--no-extra", action="store_true")
    args = ap.parse_args()
    world, rank, local = dist_setup()
    w = WORKLOADS[args.workload]
    if args.impl == "reference":
        return reference_arm(args, w, world, rank)
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    try:
        return ours_arm(args, w, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
