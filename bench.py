#!/usr/bin/env python
"""Throughput of SageSLA attention on B200: effective (dense-equivalent) TOPS
and ms per call at the 480P video-DiT shape (B=1, H=12, N=32768, d=128,
block=128, top-10%), one call of the whole operator per step.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload 480p|720p|dense|sweep0.05|sweep0.10|sweep0.20|sweep0.40|tiny|480p_classes]

--workload picks another of the seeded synthetic workloads (default: the
480P headline); the JSON line's metric string names the workload's shape.
480p_classes runs the three-class operator (per-head fractions, the lowest
half of every ranking left out of the linear branch) on the 480P shape.

One process per GPU (torchrun for N > 1).  Every (batch, head) problem is
independent, so each rank runs its own full-size problem with no collective
on the data path ("scaling": "weak"); ranks only meet at the timing barriers
and the max-over-ranks of the elapsed time.  Rank 0 prints one JSON line.

--impl reference times the CPU oracle (the plain C++ statement of the method
under oracle/, run as it stands on the host cores) on a bounded sample of the
same workload: one whole head per step.
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
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

WORKLOAD = "480p"
METRIC = "effective sparse-attn TOPS & ms/call, N=32768 H=12 d=128 top-10%, 1 B200"
UNIT = "TOPS"
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_BF16_TFLOPS = 1590.0
FALLBACK_HBM_GBS = 6650.0
PROFILE_SUMMARY = os.path.join(ROOT, "profiles", "k_attn_480p.md")
ATTN_SOURCE = os.path.join(ROOT, "int8_block_sparse_b200", "csrc", "k_attn.cuh")


# ---------------------------------------------------------------- work accounting

def metric_for(w) -> str:
    """The headline metric string, or the same wording for another workload's shape."""
    if w.name == WORKLOAD:
        return METRIC
    pct = f"{w.topk_frac * 100:g}%"
    if w.classes:
        fr = sorted(set(w.head_fracs)) if w.head_fracs else [w.topk_frac]
        pct = f"{fr[0] * 100:g}..{fr[-1] * 100:g}% per head, skip {(w.skip_frac or 0) * 100:g}%"
    if w.gran is not None:
        pct += f", scale per {w.gran} tokens"
    return (f"effective sparse-attn TOPS & ms/call, B={w.B} N={w.N} H={w.H} d={w.d} top-{pct}, 1 B200 "
            f"({w.name} workload)")


def dense_equivalent_ops(B, H, N, d):
    """4 * B * H * N^2 * d: QK^T and PV of dense attention, 2 ops per MAC each."""
    return 4.0 * B * H * N * N * d


def critical_ops(idx, N, d, block):
    """Ops of the critical-block work counted from the block lists idx
    [B, H, nblk, kc]: int8 QK^T and bf16 PV, 2 * rows_i * keys_j * d each for
    every kept (query block i, key block j), with the valid rows and keys of
    a partial last block.  Entries -1 (lists shorter than the pitch) count
    nothing."""
    import numpy as np

    nblk = idx.shape[-2]
    sizes = np.minimum(block, N - np.arange(nblk) * block).astype(np.float64)
    ix = idx.astype(np.int64)
    keys = np.where(ix >= 0, sizes[np.maximum(ix, 0)], 0.0).sum(axis=-1)   # [B, H, nblk]
    ops = float((2.0 * d * sizes[None, None, :] * keys).sum())
    return ops, ops


def algorithmic_bytes(B, H, N, d, nblk, kc, linear=None):
    """Bytes a call must move at least: q, k, v in (bf16), out (bf16), the
    INT8 codes written and read once, and the float32 linear states written
    and read once (none when every block is kept, or `linear` is False)."""
    b = B * H * N * d * (3 * 2 + 2 + 2 * 1 * 2)
    if (kc < nblk) if linear is None else linear:
        b += 2 * B * H * nblk * (d * d + d) * 4
    return float(b)


def call_roofline(qk_ops, pv_flops, bytes_alg, ms, peaks):
    """Roofline of the whole call: the slower of the critical-block work at the
    tensor peaks and the algorithmic bytes at the HBM peak, over the measured
    time per call."""
    bf16 = float(peaks["bf16_tflops"]) if peaks else FALLBACK_BF16_TFLOPS
    hbm = float(peaks["hbm_gbs"]) if peaks else FALLBACK_HBM_GBS
    t_tensor = qk_ops / (2.0 * bf16 * 1e12) + pv_flops / (bf16 * 1e12)
    t_hbm = bytes_alg / (hbm * 1e9)
    t_roof = max(t_tensor, t_hbm)
    return {"bound": "tensor" if t_tensor >= t_hbm else "hbm", "t_roof_ms": round(t_roof * 1e3, 4),
            "t_tensor_ms": round(t_tensor * 1e3, 4), "t_hbm_ms": round(t_hbm * 1e3, 4),
            "bytes_alg": bytes_alg, "frac": round(t_roof * 1e3 / ms, 4),
            "peaks": "measured (MEASURED_PEAKS.json)" if peaks else "fallback"}


def attn_roofline(qk_ops, pv_flops, peaks):
    """Peak for the mixed kernel: ops / (QK at the int8 peak + PV at the bf16 peak)."""
    if peaks is not None:
        bf16 = float(peaks["bf16_tflops"])
        src = "measured (MEASURED_PEAKS.json bf16_tflops burst; int8 = 2 x bf16, nominal ratio)"
    else:
        bf16 = FALLBACK_BF16_TFLOPS
        src = "fallback 1.59 PFLOP/s bf16 (int8 = 2 x bf16, nominal ratio)"
    i8 = 2.0 * bf16
    t_roof = qk_ops / (i8 * 1e12) + pv_flops / (bf16 * 1e12)
    return (qk_ops + pv_flops) / t_roof / 1e12, src


def load_peaks():
    try:
        with open(PEAKS_FILE) as f:
            return json.load(f)
    except (OSError, ValueError):
        return None


def profiled_traffic():
    """DRAM bytes per k_attn launch from the committed ncu summary, if it was
    taken on the kernel source as it is now (else None)."""
    try:
        with open(PROFILE_SUMMARY) as f:
            text = f.read()
        with open(ATTN_SOURCE, "rb") as f:
            sha = hashlib.sha256(f.read()).hexdigest()
    except OSError:
        return None
    vals = {}
    for line in text.splitlines():
        if ":" in line and line.strip().startswith("- "):
            k, v = line.strip()[2:].split(":", 1)
            vals[k.strip()] = v.strip().strip("`")
    if vals.get("k_attn.cuh sha256") != sha:
        return None
    try:
        return float(vals["dram bytes per launch (480p)"])
    except (KeyError, ValueError):
        return None


# ---------------------------------------------------------------- distributed plumbing

class Dist:
    def __init__(self, n_gpus):
        import torch

        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        if self.world != n_gpus:
            raise SystemExit(f"--gpus {n_gpus} but WORLD_SIZE {self.world}")
        self.pg = None
        if self.world > 1:
            import datetime

            import torch.distributed as dist

            backend = "nccl" if torch.cuda.is_available() else "gloo"
            if backend == "nccl":
                torch.cuda.set_device(self.local)
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
            self.pg = dist

    def barrier(self):
        if self.pg is not None:
            self.pg.barrier()

    def max(self, x: float) -> float:
        return reduce_max(x, self.pg)

    def close(self):
        if self.pg is not None:
            self.pg.destroy_process_group()


def reduce_max(x: float, dist_mod=None) -> float:
    """Max of a per-rank float over all ranks (identity without a process group)."""
    if dist_mod is None:
        return float(x)
    import torch

    dev = "cuda" if dist_mod.get_backend() == "nccl" else "cpu"
    t = torch.tensor([float(x)], dtype=torch.float64, device=dev)
    dist_mod.all_reduce(t, op=dist_mod.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_value(ops_per_rank: float, world: int, max_seconds: float) -> float:
    """Whole-job throughput in TOPS: all ranks' work over the slowest rank's time."""
    return ops_per_rank * world / max_seconds / 1e12


# ---------------------------------------------------------------- clocks

CLOCK_QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
               "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
               "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")


class ClockSampler:
    """nvidia-smi sampling of this rank's GPU during the timed region."""

    def __init__(self, device_index: int):
        self.proc = None
        self.path = None
        try:
            import torch

            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            sel = uuid if uuid.startswith("GPU-") else f"GPU-{uuid}"
        except Exception:
            sel = str(device_index)
        self.sel = sel

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.sel, f"--query-gpu={CLOCK_QUERY}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.15)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v == "Active"})
        loaded = [s for s in sm if mx and s > 0.5 * max(mx)] or sm
        return {"sm_mhz": statistics.median(loaded) if loaded else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons, "samples": len(rows)}


# ---------------------------------------------------------------- one operator, two mask kinds

def op_attn(S, t, w, out):
    """The device operator on the workload (three-class entry point where the workload asks for it)."""
    if w.classes:
        S.sla_attn_classes(t["q"], t["k"], t["v"], t["proj"], block=w.block, topk_frac=w.fracs,
                           skip_frac=w.skip_frac, out=out)
    else:
        S.sla_attn(t["q"], t["k"], t["v"], t["proj"], block=w.block, topk_frac=w.topk_frac, out=out, gran=w.gran)


def op_host(S, host, hout, w):
    if w.gran is not None:   # no host-buffer entry: the copies around the device call
        import torch

        dev = {k: v.to("cuda", non_blocking=True) for k, v in host.items()}
        out = S.sla_attn(dev["q"], dev["k"], dev["v"], dev["proj"], block=w.block, topk_frac=w.topk_frac,
                         gran=w.gran)
        hout.copy_(out, non_blocking=True)
        torch.cuda.synchronize()
    elif w.classes:
        S.sla_attn_classes_host(host["q"], host["k"], host["v"], host["proj"], hout, block=w.block,
                                topk_frac=w.fracs, skip_frac=w.skip_frac)
    else:
        S.sla_attn_host(host["q"], host["k"], host["v"], host["proj"], hout, block=w.block, topk_frac=w.topk_frac)


def op_mask(S, t, w):
    """(block lists [B, H, nblk, pitch], class map or None, kc per head, linear branch used)."""
    if w.classes:
        idx, cls = S.sla_mask_classes(t["q"], t["k"], w.block, w.fracs, w.skip_frac, classes=True)
        kc, kn, _ = S.head_counts(w.N, w.block, w.H, w.fracs, w.skip_frac)
        return idx.cpu().numpy(), cls.cpu().numpy(), kc, any(c + n < w.nblk for c, n in zip(kc, kn))
    kc = S.topk_count(w.N, w.block, w.topk_frac)
    return S.sla_mask(t["q"], t["k"], w.block, w.topk_frac).cpu().numpy(), None, [kc] * w.H, kc < w.nblk


def oracle_head(O, w, xs, h):
    """The CPU oracle on head h of the workload (xs: that head's inputs)."""
    if w.classes:
        fr = w.fracs[h] if isinstance(w.fracs, list) else w.fracs
        return O.sla_attention(xs["q"], xs["k"], xs["v"], xs["proj"], w.block, [fr], skip_frac=w.skip_frac)
    return O.sla_attention(xs["q"], xs["k"], xs["v"], xs["proj"], w.block, w.topk_frac, gran=w.gran)


# ---------------------------------------------------------------- CPU oracle sample

def oracle_sample(w, x, max_heads: int, budget_s: float):
    """Time the CPU oracle on every query block of whole heads of the workload
    (their quantisation, mask, linear states and outputs), head 0 first, until
    max_heads heads or about budget_s seconds.  Returns (seconds, ops, sample)."""
    from oracle import cpp_oracle as O

    dt, nh = 0.0, 0
    for h in range(min(max_heads, w.H)):
        xs = {k: (v[:1, h:h + 1] if v.ndim == 4 else v) for k, v in x.items()}
        t0 = time.perf_counter()
        oracle_head(O, w, xs, h)
        dt += time.perf_counter() - t0
        nh += 1
        if dt >= budget_s:
            break
    ops = nh * 4.0 * w.N * w.N * w.d   # dense-equivalent ops of those heads
    return dt, ops, (f"CPU oracle on heads 0..{nh - 1} of batch 0 of {w.name} (all {w.nblk} query blocks "
                     f"of {w.block} rows each, with their quantisation, mask and linear states); "
                     f"value = dense-equivalent ops of those heads / wall time")


def mask_parity(w, x, gidx, gcls=None):
    """The GPU's block lists (class maps, for the three-class mask) against
    the oracle's over the whole workload: rows, rows the oracle marks as near
    ties, rows that differ, and rows that differ without being near ties
    (must be 0)."""
    import numpy as np

    from oracle import cpp_oracle as O

    if w.classes:
        ref = O.block_mask_classes(x["q"], x["k"], w.block, w.fracs, w.skip_frac)
        diff = np.any(gcls != ref["cls"], axis=-1)
    else:
        ref = O.block_mask(x["q"], x["k"], w.block, w.topk_frac)
        diff = np.any(gidx != ref["idx"], axis=-1)
    return {"rows": int(diff.size), "near_tie_rows": int(ref["near_tie"].sum()),
            "differing_rows": int(diff.sum()), "differing_off_near_tie": int((diff & ~ref["near_tie"]).sum())}


def oracle_threads() -> int:
    """Worker threads of the C++ CPU oracle (every core this process may use)."""
    from oracle import cpp_oracle

    return cpp_oracle.threads()


# ---------------------------------------------------------------- arms

def run_ours(args, dist):
    import numpy as np
    import torch

    import int8_block_sparse_b200 as S
    from int8_block_sparse_b200.build import build
    from synth import CONFIGS, make_workload

    build()
    S.lib()
    dev = torch.device("cuda", dist.local)
    torch.cuda.set_device(dev)
    w = CONFIGS[args.workload]
    if args.heads:
        import dataclasses

        w = dataclasses.replace(w, H=args.heads, name=f"{w.name}-first{args.heads}heads",
                                head_fracs=w.head_fracs[:args.heads] if w.head_fracs else None)
        x = make_workload(CONFIGS[args.workload], heads=list(range(args.heads)))
    else:
        x = make_workload(w)
    t = {k: torch.from_numpy(x[k].view(np.int16)).view(torch.bfloat16).to(dev) for k in ("q", "k", "v", "proj")}
    out = torch.empty((w.B, w.H, w.N, w.d), dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        op_attn(S, t, w, out)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    rc = S.get_error()
    if rc != 0:
        raise SystemExit(f"device error after warm-up: {S.status_string(rc)}")

    sampler = ClockSampler(dist.local)
    sampler.start()
    S.profile_read()
    S.profile_enable(True)
    dist.barrier()
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    dist.barrier()
    S.profile_enable(False)
    clocks = sampler.stop()
    prof = S.profile_read()
    rc = S.get_error()
    if rc != 0:
        raise SystemExit(f"device error in the timed region: {S.status_string(rc)}")
    ms_local = e0.elapsed_time(e1) / args.steps
    ms = dist.max(ms_local)

    ops = dense_equivalent_ops(w.B, w.H, w.N, w.d)
    value = weak_scaling_value(ops, dist.world, ms / 1e3)
    gidx, gcls, kcs, linear = op_mask(S, t, w)
    kc = kcs[0] if len(set(kcs)) == 1 else kcs
    qk, pv = critical_ops(gidx, w.N, w.d, w.block)
    peaks = load_peaks()
    peak, peak_src = attn_roofline(qk, pv, peaks)
    attn_ms, attn_n = prof["attn"]
    attn_avg = attn_ms / max(attn_n, 1)
    achieved = (qk + pv) / (attn_avg / 1e3) / 1e12
    roof = {"bound": "tensor", "kernel": "k_attn<128,128> (critical-block attention)",
            "achieved": round(achieved, 1), "peak": round(peak, 1), "unit": "TFLOP/s",
            "frac": round(achieved / peak, 4), "traffic": profiled_traffic() if w.name == WORKLOAD else None,
            "peak_source": peak_src, "ops_per_launch": qk + pv,
            "kernel_ms": round(attn_avg, 4)}
    launches = int(sum(n for _, n in prof.values()))
    # per kind: summed event time per call (kernels on the two streams overlap)
    kernels = {k: {"ms_per_call": round(v[0] / args.steps, 4), "launches": int(v[1])} for k, v in prof.items()
               if v[1] > 0}

    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(S, t, w, args, dist)

    line = {
        "metric": metric_for(w), "value": round(value, 2), "unit": UNIT, "n_gpus": dist.world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "i8,bf16 (f32 accumulate; bf16 out)",
        "data": "synthetic (seeded field-plus-noise, see synth/workloads.py)",
        "config": {"workload": w.describe(), "kc": kc,
                   "parallelism": f"replicas x{dist.world} (independent problems per rank)",
                   "l2": (f"inputs larger than L2 (q, k, v: {3 * w.B * w.H * w.N * w.d * 2 / 1e6:.0f} MB), "
                          "no flush") if 3 * w.B * w.H * w.N * w.d * 2 > 126e6 else
                         "inputs smaller than L2 (launch-bound case), no flush"},
        "roofline": roof,
        "roofline_call": call_roofline(qk, pv, algorithmic_bytes(w.B, w.H, w.N, w.d, w.nblk, max(kcs), linear),
                                       ms, peaks),
        "kernels": kernels, "gpu_launches": launches, "clocks": clocks, "e2e": e2e,
    }
    if dist.rank == 0 and dist.world == 1 and not args.no_cpu:
        dt, cops, sample = oracle_sample(w, x, args.cpu_heads, args.cpu_budget)
        line["cpu_baseline"] = {"value": round(cops / dt / 1e12, 6), "unit": UNIT, "cores": oracle_threads(),
                                "kind": "oracle", "sample": sample, "seconds": round(dt, 2)}
        # near ties of the block mask (CPU oracle leg): every differing row must be one
        line["mask_parity"] = mask_parity(w, x, gidx, gcls)
        line["near_tie_rows"] = line["mask_parity"]["near_tie_rows"]
    return line


def run_linear(args, dist):
    """One W8A8 linear layer per step: X quantised in the call (k_quant2d) and
    the block-scaled INT8 GEMM (k_w8a8_gemm); the weights are quantised once
    before timing, as a deployed layer holds them."""
    import numpy as np
    import torch

    import int8_block_sparse_b200 as S
    from int8_block_sparse_b200.build import build
    from synth.linear import LINEAR_CONFIGS, make_linear_workload

    build()
    S.lib()
    dev = torch.device("cuda", dist.local)
    torch.cuda.set_device(dev)
    w = LINEAR_CONFIGS[args.workload]
    d = make_linear_workload(w)

    def to_dev(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(dev)

    x, wt = to_dev(d["x"]), to_dev(d["w"])
    b = to_dev(d["bias"]) if d["bias"] is not None else None
    wq, sw = S.w8a8_quant(wt)
    y = torch.empty((w.M, w.N), dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        S.w8a8_linear(x, wq, sw, b, out=y)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    rc = S.get_error()
    if rc != 0:
        raise SystemExit(f"device error after warm-up: {S.status_string(rc)}")
    sampler = ClockSampler(dist.local)
    sampler.start()
    S.profile_read()
    S.profile_enable(True)
    dist.barrier()
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    dist.barrier()
    S.profile_enable(False)
    clocks = sampler.stop()
    prof = S.profile_read()
    rc = S.get_error()
    if rc != 0:
        raise SystemExit(f"device error in the timed region: {S.status_string(rc)}")
    ms = dist.max(e0.elapsed_time(e1) / args.steps)
    ops = 2.0 * w.M * w.N * w.K
    value = weak_scaling_value(ops, dist.world, ms / 1e3)
    peaks = load_peaks()
    bf16 = float(peaks["bf16_tflops"]) if peaks else FALLBACK_BF16_TFLOPS
    hbm = float(peaks["hbm_gbs"]) if peaks else FALLBACK_HBM_GBS
    i8 = 2.0 * bf16
    g_ms, g_n = prof["w8a8"]
    g_avg = g_ms / max(g_n, 1)
    achieved = ops / (g_avg / 1e3) / 1e12
    roof = {"bound": "tensor", "kernel": "k_w8a8_gemm (block-scaled INT8 GEMM)", "achieved": round(achieved, 1),
            "peak": round(i8, 1), "unit": "TOPS", "frac": round(achieved / i8, 4), "traffic": None,
            "peak_source": ("measured (MEASURED_PEAKS.json bf16_tflops burst; int8 = 2 x bf16, nominal ratio)"
                            if peaks else "fallback 1.59 PFLOP/s bf16 (int8 = 2 x bf16, nominal ratio)"),
            "ops_per_launch": ops, "kernel_ms": round(g_avg, 4)}
    # bytes a call must move: X in (bf16), X codes out and in, W codes in, Y out (bf16), bias
    bytes_alg = float(w.M * w.K * 2 + 2 * w.M * w.K + w.N * w.K + w.M * w.N * 2 + (w.N * 2 if b is not None else 0))
    t_tensor, t_hbm = ops / (i8 * 1e12), bytes_alg / (hbm * 1e9)
    t_roof = max(t_tensor, t_hbm)
    call = {"bound": "tensor" if t_tensor >= t_hbm else "hbm", "t_roof_ms": round(t_roof * 1e3, 4),
            "t_tensor_ms": round(t_tensor * 1e3, 4), "t_hbm_ms": round(t_hbm * 1e3, 4), "bytes_alg": bytes_alg,
            "frac": round(t_roof * 1e3 / ms, 4), "peaks": "measured (MEASURED_PEAKS.json)" if peaks else "fallback"}
    kernels = {k: {"ms_per_call": round(v[0] / max(v[1], 1), 4), "launches": int(v[1])} for k, v in prof.items()
               if v[1] > 0}
    line = {
        "metric": (f"W8A8 linear TOPS & ms/call, M={w.M} N={w.N} K={w.K} (128x128 blocks), 1 B200 "
                   f"({w.name} workload)"),
        "value": round(value, 2), "unit": UNIT, "n_gpus": dist.world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(ms, 4), "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "i8 (int32 block sums, f32 promotion; bf16 out)",
        "data": "synthetic (seeded, see synth/linear.py)",
        "config": {"workload": w.describe(), "parallelism": f"replicas x{dist.world} (independent problems per rank)",
                   "l2": f"inputs larger than L2 (X: {w.M * w.K * 2 / 1e6:.0f} MB), no flush"},
        "roofline": roof, "roofline_call": call, "kernels": kernels,
        "gpu_launches": int(sum(v["launches"] for v in kernels.values())), "clocks": clocks,
    }
    if not args.no_e2e:
        hx = x.cpu().pin_memory()
        hy = torch.empty((w.M, w.N), dtype=torch.bfloat16).pin_memory()
        n = max(1, min(args.steps, args.e2e_steps))

        def e2e_step():
            dx = hx.to(dev, non_blocking=True)
            S.w8a8_linear(dx, wq, sw, b, out=y)
            hy.copy_(y, non_blocking=True)
            torch.cuda.synchronize(dev)

        e2e_step()
        dist.barrier()
        t0 = time.perf_counter()
        for _ in range(n):
            e2e_step()
        dt = dist.max((time.perf_counter() - t0) / n)
        line["e2e"] = {"value": round(weak_scaling_value(ops, dist.world, dt), 2), "unit": UNIT,
                       "h2d_bytes_per_step": hx.numel() * 2, "d2h_bytes_per_step": hy.numel() * 2,
                       "ms_per_step": round(dt * 1e3, 3), "steps": n,
                       "timer": "host wall clock: pinned X to the device, w8a8_linear, Y back, synchronised"}
    if dist.rank == 0 and dist.world == 1 and not args.no_cpu:
        dt, rows = linear_oracle_sample(w, d, args.cpu_budget)
        line["cpu_baseline"] = {"value": round(2.0 * rows * w.N * w.K / dt / 1e12, 6), "unit": UNIT,
                                "cores": oracle_threads(), "kind": "oracle",
                                "sample": (f"W8A8 oracle (plain C++, exact int32 block sums, one thread per core) "
                                           f"on the first {rows} rows of X of {w.name}: their quantisation and the "
                                           f"block-scaled product with all N columns; value = 2 * rows * N * K / "
                                           f"wall time"), "seconds": round(dt, 2)}
    return line


def linear_oracle_sample(w, d, budget_s):
    """Time the plain C++ W8A8 oracle on 128-row blocks of X (quantisation +
    product with the pre-quantised weights), block 0 first, until about
    budget_s seconds."""
    from oracle import w8a8_cpp as W

    wq, sw = W.quantize_2d(d["w"])
    dt, rows = 0.0, 0
    for rb in range((w.M + 127) // 128):
        xb = d["x"][rb * 128:(rb + 1) * 128]
        t0 = time.perf_counter()
        xq, sx = W.quantize_2d(xb)
        W.gemm(xq, sx, wq, sw, d["bias"])
        dt += time.perf_counter() - t0
        rows += xb.shape[0]
        if dt >= budget_s:
            break
    return dt, rows


def run_e2e(S, t, w, args, dist):
    """Same metric through the host-buffer entry point: H2D of q, k, v, proj,
    the operator, D2H of out, every step (host wall clock around the
    synchronous call)."""
    import torch

    host = {k: v.cpu().pin_memory() for k, v in t.items()}
    hout = torch.empty((w.B, w.H, w.N, w.d), dtype=torch.bfloat16).pin_memory()
    op_host(S, host, hout, w)
    n = max(1, min(args.steps, args.e2e_steps))
    dist.barrier()
    t0 = time.perf_counter()
    for _ in range(n):
        op_host(S, host, hout, w)
    dt = dist.max((time.perf_counter() - t0) / n)
    ops = dense_equivalent_ops(w.B, w.H, w.N, w.d)
    h2d = sum(v.numel() * v.element_size() for v in host.values())
    d2h = hout.numel() * hout.element_size()
    return {"value": round(weak_scaling_value(ops, dist.world, dt), 2), "unit": UNIT,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": round(dt * 1e3, 3),
            "steps": n, "timer": "host wall clock around the synchronous host-buffer call "
                                 f"({'sla_attn_classes_host' if w.classes else 'sla_attn_host'})"}


def run_reference_linear(args, dist):
    """The plain C++ W8A8 oracle as the reference arm: each step quantises one
    128-row block of X and multiplies it with the pre-quantised weights (all N
    columns), the blocks taken in turn."""
    from oracle import w8a8_cpp as W
    from synth.linear import LINEAR_CONFIGS, make_linear_workload

    w = LINEAR_CONFIGS[args.workload]
    n = args.warmup + args.steps
    nrb = (w.M + 127) // 128
    rows = sorted({r for s_ in range(n) for r in range((s_ % nrb) * 128, min(w.M, (s_ % nrb) * 128 + 128))})
    d = make_linear_workload(w, rows=rows)
    pos = {r: t for t, r in enumerate(rows)}
    wq, sw = W.quantize_2d(d["w"])

    def step(s_):
        rb = s_ % nrb
        lo, hi = rb * 128, min(w.M, rb * 128 + 128)
        xq, sx = W.quantize_2d(d["x"][pos[lo]:pos[lo] + (hi - lo)])
        W.gemm(xq, sx, wq, sw, d["bias"])
        return hi - lo

    for s_ in range(args.warmup):
        step(s_)
    t0 = time.perf_counter()
    done = sum(step(s_) for s_ in range(args.warmup, n))
    dt = time.perf_counter() - t0
    value = 2.0 * done * w.N * w.K / dt / 1e12
    ms_call = dt / max(done, 1) * w.M * 1e3
    metric = f"W8A8 linear TOPS & ms/call, M={w.M} N={w.N} K={w.K} (128x128 blocks), 1 B200 ({w.name} workload)"
    sample = (f"W8A8 oracle (plain C++), {args.steps} steps of one 128-row block of X of {w.name} "
              f"(quantisation + product with all N columns)")
    return {"impl": "reference", "metric": metric, "value": round(value, 6), "unit": UNIT, "n_gpus": dist.world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_call, 1),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64 (int8 codes)",
            "data": "synthetic (seeded, see synth/linear.py)",
            "config": {"workload": w.describe(), "note": "ms_per_step = projected time of one full call"},
            "cpu_baseline": {"value": round(value, 6), "unit": UNIT, "cores": oracle_threads(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": round(value, 6), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def run_reference(args, dist):
    """The CPU oracle as the reference arm: the plain C++ oracle, as it stands,
    on the host cores; each step is the whole operator on one head of the
    workload (every query block of it, with its quantisation, mask and linear
    states), the heads taken in turn."""
    from oracle import cpp_oracle as O
    from synth import CONFIGS, make_workload

    w = CONFIGS[args.workload]
    if dist.rank != 0:
        return None
    n = args.warmup + args.steps
    heads = sorted({s % w.H for s in range(n)})
    x = make_workload(w, heads=heads)
    pos = {h: t for t, h in enumerate(heads)}

    def step(s):
        h = pos[s % w.H]
        xs = {k: (v[:1, h:h + 1] if v.ndim == 4 else v) for k, v in x.items()}
        oracle_head(O, w, xs, s % w.H)

    for s_ in range(args.warmup):
        step(s_)
    t0 = time.perf_counter()
    for s_ in range(args.warmup, n):
        step(s_)
    per_head = (time.perf_counter() - t0) / max(args.steps, 1)
    value = 4.0 * w.N * w.N * w.d / per_head / 1e12
    ms_call = per_head * w.B * w.H * 1e3
    sample = (f"C++ CPU oracle, {args.steps} steps of one whole head of batch 0 of {w.name} (all {w.nblk} "
              f"query blocks with the head's quantisation, mask and linear states), heads in turn")
    return {"impl": "reference", "metric": metric_for(w), "value": round(value, 6), "unit": UNIT, "n_gpus": dist.world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_call, 1),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64 (int8 codes)",
            "data": "synthetic (seeded field-plus-noise, see synth/workloads.py)",
            "config": {"workload": w.describe(), "note": "ms_per_step = projected time of one full call"},
            "cpu_baseline": {"value": round(value, 6), "unit": UNIT, "cores": oracle_threads(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": round(value, 6), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--workload", default=WORKLOAD,
                    choices=["tiny", "480p", "720p", "dense", "sweep0.05", "sweep0.10", "sweep0.20", "sweep0.40",
                             "480p_classes", "480p_gran32", "w8a8_14b_ffn", "w8a8_14b_proj", "w8a8_1b3_ffn", "w8a8_small",
                             "w8a8_prof"])
    ap.add_argument("--cpu-heads", type=int, default=6,
                    help="most heads of the workload the CPU oracle baseline runs in full")
    ap.add_argument("--cpu-budget", type=float, default=15.0,
                    help="seconds after which the CPU oracle baseline stops adding heads")
    ap.add_argument("--heads", type=int, default=0,
                    help="keep only the first H heads (a smaller case for profiling; not the headline)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        raise SystemExit("--warmup must be at least 3")
    if args.impl == "reference":
        world = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        if rank != 0:
            return 0

        class _D:
            pass

        d = _D()
        d.rank, d.world = 0, world
        line = run_reference_linear(args, d) if args.workload.startswith("w8a8") else run_reference(args, d)
        print(json.dumps(line), flush=True)
        return 0
    dist = Dist(args.gpus)
    try:
        line = run_linear(args, dist) if args.workload.startswith("w8a8") else run_ours(args, dist)
        if dist.rank == 0:
            print(json.dumps(line), flush=True)
    finally:
        dist.close()
    return 0


if __name__ == "__main__":
    sys.exit(main())
