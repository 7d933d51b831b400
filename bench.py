#!/usr/bin/env python
"""Benchmark of the per-matrix optimizer step on B200.

Default workload: one Muon step over every 2-D matrix of a 32-layer dense GPT
(hidden 4096, 32 query / 8 KV heads of dim 128, FFN 14336): 224 fp32
matrices, 6.98 G parameters, synthetic gradients (Gaussian N(0, 1e-3^2) plus
a rank-16 spike with 10x its norm), random-init weights N(0, 0.02^2).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints ONE JSON line (rank 0).  ``value`` is whole-job TFLOP/s with the
pages' Newton-Schulz count 5 (4 m'^2 n' + 2 m'^3) per matrix (m' <= n'),
timed on the device with CUDA events over exactly K steps between a barrier
and a synchronize, max over ranks.  Inputs are far larger than L2, so no
flush is needed.  Multi-GPU runs are independent replicas (the step has no
exchange on one matrix); ``scaling`` is weak.
"""

import argparse
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

METRIC = "Muon/SOAP step TFLOP/s and matrices/s on 1 B200; % of BF16 tensor peak & HBM BW"
UNIT = "TFLOP/s"
WORKLOAD = "muon_step dense GPT 32 layers (hidden 4096, kv 1024, ffn 14336): 224 fp32 matrices, 6.98 G params"


# ----------------------------------------------------------------------------- helpers

def page_flops(m, n, steps=5):
    """The pages' Newton-Schulz count per matrix: steps * (4 m'^2 n' + 2 m'^3)."""
    mp, np_ = min(m, n), max(m, n)
    return steps * (4.0 * mp * mp * np_ + 2.0 * mp ** 3)


def gemm_alg_flops(m, n, steps=5):
    """Necessary tensor-core flops of our NS products per matrix: the two
    symmetric products only need their upper triangle (m'(m'+1)/2 entries)."""
    mp, np_ = min(m, n), max(m, n)
    gram = mp * (mp + 1) * np_
    poly = mp * (mp + 1) * mp
    update = 2.0 * mp * mp * np_
    return steps * (gram + poly + update)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    except (OSError, ValueError):
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 200 ms."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, mx, pw, reasons = [], [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    mx.append(float(parts[2]))
                except ValueError:
                    continue
                try:
                    pw.append(float(parts[3]))
                except ValueError:
                    pass
                for nm, v in zip(names, parts[5:9]):
                    if v.lower().startswith("active"):
                        reasons.add(nm)
        os.unlink(self.path)
        if not sm:
            return None
        out = {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
               "samples": len(sm)}
        if pw:
            out["power_w"] = statistics.median(pw)
        return out


def max_over_ranks(x, world, device="cpu"):
    """The largest of each rank's x (every rank gets it): a multi-GPU step
    takes as long as its slowest replica."""
    if world == 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


# ----------------------------------------------------------------------------- workloads on the GPU

def gpt_workload(device, layers=32, hidden=4096, kv=1024, ffn=14336, rank=16, noise=1e-3, ratio=10.0):
    """Synthetic dense-GPT matrices generated on the device (seeded torch
    generator; same recipe as workloads.gauss_spike)."""
    import torch
    import workloads as wl
    Ws, Gs, Bs, shapes = [], [], [], []
    for layer in range(layers):
        for name, m, n in wl.gpt_shapes(hidden, kv, ffn):
            g = torch.Generator(device=device)
            g.manual_seed(wl.seed_of("bench-cfg2", layer, name))
            W = torch.randn(m, n, generator=g, device=device) * 0.02
            G = torch.randn(m, n, generator=g, device=device) * noise
            P = torch.randn(m, rank, generator=g, device=device)
            Q = torch.randn(n, rank, generator=g, device=device)
            S = P @ Q.T
            S *= ratio * G.norm() / S.norm()
            G += S
            del S, P, Q
            Ws.append(W)
            Gs.append(G)
            Bs.append(torch.zeros_like(W))
            shapes.append((m, n))
    return Ws, Gs, Bs, shapes


def moe_workload(device, layers=4, experts=128, hidden=2048, ffn=768, noise=1e-3):
    import torch
    import workloads as wl
    Ws, Gs, Bs, shapes = [], [], [], []
    for layer in range(layers):
        for e in range(experts):
            g = torch.Generator(device=device)
            g.manual_seed(wl.seed_of("bench-cfg3", layer, e))
            scale = float(torch.randn(1, generator=g, device=device).exp())
            for m, n in ((ffn, hidden), (ffn, hidden), (hidden, ffn)):
                Ws.append(torch.randn(m, n, generator=g, device=device) * 0.02)
                Gs.append(torch.randn(m, n, generator=g, device=device) * (noise * scale))
                Bs.append(torch.zeros(m, n, device=device))
                shapes.append((m, n))
    return Ws, Gs, Bs, shapes


def capture_graph(fn):
    """Capture one call of ``fn`` (library launches on the current stream)
    into a CUDA graph, after one eager warm-up call on the capture stream."""
    import torch
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        fn()
    torch.cuda.current_stream().wait_stream(side)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    torch.cuda.synchronize()
    return g


def time_steps(fn, steps, warmup, sync_all=None):
    import torch
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    if sync_all:
        sync_all()
    s = torch.cuda.Event(enable_timing=True)
    e = torch.cuda.Event(enable_timing=True)
    s.record()
    for _ in range(steps):
        fn()
    e.record()
    torch.cuda.synchronize()
    return s.elapsed_time(e) / steps


# ----------------------------------------------------------------------------- our arm

def run_ours(args, world, rank, local):
    import torch
    import torch.distributed as dist
    from matrix_aware_optimizers_muon_b200 import OP_MUON, Context

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        # ranks that wait for a failed peer end with an error after 5 minutes
        dist.init_process_group("nccl", device_id=dev, timeout=datetime.timedelta(minutes=5))

    def barrier():
        if world > 1:
            dist.barrier()

    peaks, peak_kind = load_peaks()
    ctx = Context(local)
    Ws, Gs, Bs, shapes = gpt_workload(dev, layers=args.layers)
    ctx.reserve(OP_MUON, shapes)
    torch.cuda.synchronize()
    flops_page = sum(page_flops(m, n) for m, n in shapes)
    flops_gemm = sum(gemm_alg_flops(m, n) for m, n in shapes)
    params = sum(m * n for m, n in shapes)

    def step():
        ctx.muon_step(Ws, Gs, Bs, lr=0.02, weight_decay=0.01, momentum=0.95, reserve=False)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    ctx.profile(True)
    ctx.profile_read()
    clocks = ClockSampler(local)
    clocks.start()
    barrier()
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record()
    for _ in range(args.steps):
        step()
    t1.record()
    torch.cuda.synchronize()
    barrier()
    ms = t0.elapsed_time(t1) / args.steps
    clk = clocks.stop()
    prof = ctx.profile_read()
    ctx.profile(False)
    status = ctx.device_status()
    ms = max_over_ranks(ms, world, dev)

    gemm_ms = sum(prof[k][0] for k in ("gram", "poly", "update"))
    gemm_exec = sum(prof[k][1] for k in ("gram", "poly", "update"))
    gemm_launches = sum(prof[k][2] for k in ("gram", "poly", "update"))
    ew_ms = prof["prep"][0] + prof["apply"][0]
    launches = int(sum(v[2] for v in prof.values()))
    gemm_tf = flops_gemm * args.steps / (gemm_ms / 1e3) / 1e12 if gemm_ms > 0 else None
    peak_tf = peaks.get("bf16_tflops_sustained", peaks.get("bf16_tflops"))
    # prep moves 14 B/param (G 4, B read + write 8, bf16 N 2); the Muon apply
    # (W read + write 8, bf16 O 2) runs in the last update's epilogue, or as
    # apply_kernel when no update product ran
    ew_bytes = (14.0 + (10.0 if prof["apply"][2] > 0 else 0.0)) * params
    ew_gbs = ew_bytes * args.steps / (ew_ms / 1e3) / 1e9 if ew_ms > 0 else None

    value = flops_page * world / (ms / 1e3) / 1e12
    out = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": UNIT,
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms, 3),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded gradients: N(0,1e-3^2) + rank-16 spike at 10x norm; W ~ N(0,0.02^2))",
        "config": {"workload": WORKLOAD if args.layers == 32 else WORKLOAD.replace("32 layers", f"{args.layers} layers"),
                   "matrices": len(shapes), "params": params,
                   "ns_steps": 5, "coeffs": [3.4445, -4.775, 2.0315],
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                   "l2": "inputs (84 GB) far larger than L2; no flush"},
        "matrices_per_s": round(len(shapes) * world / (ms / 1e3), 2),
        "roofline": {
            "bound": "tensor",
            "kernel": "gemm_bf16_kernel (tcgen05; Gram + polynomial + update, all NS products)",
            "achieved": round(gemm_tf, 2) if gemm_tf else None,
            "peak": peak_tf,
            "unit": "TFLOP/s",
            "frac": round(gemm_tf / peak_tf, 4) if gemm_tf else None,
            "peak_source": f"{peak_kind} bf16_tflops_sustained",
            # DRAM bytes of one update launch (an iteration before the last)
            # on the 4096 x 14336 bucket (96 matrices): ncu captured 864.1 MB
            # on the one-layer batch of 3; traffic grows with the matrices
            "traffic": 864.1e6 * args.layers,
            "traffic_kernel": "update GEMM, 4096x14336 bucket, one launch (ncu, scaled by matrices)",
            "alg_flops_per_step": flops_gemm,
            "exec_flops_per_step": gemm_exec / args.steps,
            "launches_per_step": gemm_launches / args.steps,
            "ms_per_step": round(gemm_ms / args.steps, 3),
        },
        "roofline_elementwise": {
            "bound": "hbm",
            "kernel": ("prep_kernel (14 B/param; the apply runs in the last update's epilogue)"
                       if prof["apply"][2] == 0 else "prep_kernel + apply_kernel (24 B/param)"),
            "achieved": round(ew_gbs, 1) if ew_gbs else None,
            "peak": peaks.get("hbm_gbs"),
            "unit": "GB/s",
            "frac": round(ew_gbs / peaks["hbm_gbs"], 4) if ew_gbs else None,
            "ms_per_step": round(ew_ms / args.steps, 3),
        },
        "kernels_ms_per_step": {k: round(v[0] / args.steps, 3) for k, v in prof.items() if v[2]},
        "gpu_launches": launches,
        "device_status": status,
        "clocks": clk,
    }

    # end to end through the public API with host buffers
    if args.e2e:
        out["e2e"] = e2e_measure(ctx, Ws, Gs, Bs, flops_page, world, barrier, args)
    del Ws, Gs, Bs
    ctx.workspace = None
    torch.cuda.empty_cache()

    if args.extras and world == 1:
        out["extra"] = extras(ctx, dev, args)
    if rank == 0 and world == 1 and args.cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(args.cpu_seconds)
    if world > 1:
        dist.destroy_process_group()
    return out


def e2e_measure(ctx, Ws, Gs, Bs, flops_page, world, barrier, args):
    """The Muon step end to end through the public API, with every gradient
    copied from pinned host memory and the per-matrix status flags read back
    inside the timed region, over five steps.  The updated weights and
    momenta stay in device memory, where a training loop keeps them (the
    library's contract: parameters and state are updated in place on the
    device), so the flags are the step's only device-to-host result.  The step is taken as a training loop whose
    gradients arrive on the host would take it: the matrices are split into
    groups of whole layers; group k + 1's gradients copy on a side stream
    while muon_step runs on group k (each matrix's step is independent, so
    the result equals one call over all matrices).  The serial form (all
    copies, then one call) is timed beside it."""
    import torch
    steps = 5
    need = sum(g.numel() * g.element_size() for g in Gs)
    local_world = int(os.environ.get("LOCAL_WORLD_SIZE", str(world)))
    reason, host = None, None
    try:
        import psutil
        avail = psutil.virtual_memory().available
    except ImportError:
        avail = None
    if local_world > 1 and avail is not None and need * local_world > 0.8 * avail:
        reason = (f"{local_world} ranks x {need / 1e9:.1f} GB of pinned host inputs exceed 80 % of the "
                  f"host's available {avail / 1e9:.0f} GB")
    else:
        try:
            host = [torch.empty(g.shape, dtype=g.dtype, pin_memory=True) for g in Gs]
            for h, g in zip(host, Gs):
                h.copy_(g)
            flags = torch.zeros(len(Gs), dtype=torch.int32, device=Gs[0].device)
            flags_h = torch.empty(len(Gs), dtype=torch.int32, pin_memory=True)
        except RuntimeError as exc:
            reason, host = f"pinned host allocation failed: {exc}"[:200], None
    # every rank takes the same path: the timing below is collective
    ok = 0.0 if reason else 1.0
    if world > 1:
        ok = -max_over_ranks(-ok, world, Gs[0].device)
    if ok < 1.0:
        del host
        return {"value": None, "unit": UNIT, "reason": reason or "another rank could not pin its host inputs"}
    h2d = sum(h.numel() * 4 for h in host)
    hp = dict(lr=0.02, weight_decay=0.01, momentum=0.95, reserve=False)
    n = len(Gs)
    per_layer = 7
    layers = max(1, n // per_layer)
    groups = max(1, min(args.e2e_groups, layers))
    lpg = -(-layers // groups)
    bounds = sorted({min(n, k * lpg * per_layer) for k in range(groups)} | {n})
    comp = torch.cuda.current_stream()
    side = torch.cuda.Stream()
    copied = [torch.cuda.Event() for _ in bounds[:-1]]

    def pipelined():
        # a step's copies start after everything before it on the compute
        # stream (the previous step included), as the gradients of a training
        # step exist only after the previous optimizer step
        side.wait_stream(comp)
        for k in range(len(bounds) - 1):
            i0, i1 = bounds[k], bounds[k + 1]
            with torch.cuda.stream(side):
                for h, g in zip(host[i0:i1], Gs[i0:i1]):
                    g.copy_(h, non_blocking=True)
                copied[k].record(side)
            comp.wait_event(copied[k])
            ctx.muon_step(Ws[i0:i1], Gs[i0:i1], Bs[i0:i1], nonfinite=flags[i0:i1], stream=comp, **hp)
        flags_h.copy_(flags, non_blocking=True)

    def serial():
        for h, g in zip(host, Gs):
            g.copy_(h, non_blocking=True)
        ctx.muon_step(Ws, Gs, Bs, nonfinite=flags, **hp)
        flags_h.copy_(flags, non_blocking=True)

    def timed(fn):
        fn()
        torch.cuda.synchronize()
        barrier()
        s = torch.cuda.Event(enable_timing=True)
        e = torch.cuda.Event(enable_timing=True)
        s.record()
        for _ in range(steps):
            fn()
        e.record()
        torch.cuda.synchronize()
        return s.elapsed_time(e) / steps

    ms = max_over_ranks(timed(pipelined), world, Gs[0].device)
    ms_serial = max_over_ranks(timed(serial), world, Gs[0].device)
    del host
    return {"value": round(flops_page * world / (ms / 1e3) / 1e12, 2), "unit": UNIT,
            "ms_per_step": round(ms, 3), "steps": steps, "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": len(Gs) * 4, "nonfinite": int(flags_h.sum()),
            "layer_groups": len(bounds) - 1,
            "serial_ms_per_step": round(ms_serial, 3),
            "serial_value": round(flops_page * world / (ms_serial / 1e3) / 1e12, 2)}


def dyadic_gpu(n, dev, cond=1e4):
    """The sweep's known-SVD square input (workloads.dyadic recipe), built on
    the device: G[i, j] = g[i xor j]."""
    import torch
    import workloads as wl
    d = wl.dyadic_spectrum(wl.rng_of("cfg5", n), n, cond)
    g = torch.from_numpy(wl.fwht(d) / n).to(dev, torch.float32)
    idx = torch.arange(n, device=dev)
    return g[idx[:, None] ^ idx[None, :]].contiguous()


def heads_gpu(count, dim, dev, cond=1e4):
    """Batched per-head inputs U diag(s) V^T with Haar-random U, V."""
    import torch
    import workloads as wl
    g = torch.Generator(device=dev)
    g.manual_seed(wl.seed_of("bench-heads", count, dim))
    s = torch.from_numpy(wl.geometric_spectrum(dim, cond)).to(dev, torch.float32)
    s = s * (dim / s.norm())
    U, _ = torch.linalg.qr(torch.randn(count, dim, dim, generator=g, device=dev))
    V, _ = torch.linalg.qr(torch.randn(count, dim, dim, generator=g, device=dev))
    return ((U * s) @ V.transpose(1, 2)).contiguous()


def soap_flops(m, n, left, right):
    """The SOAP step's count per matrix: factor EMAs 2m^2n / 2n^2m, power
    steps 2k^3, QR counted as Householder (8/3)k^3 whatever algorithm runs,
    and the rotations: rotating M and G in and the update back out."""
    f = 0.0
    rot = 0.0
    if left:
        f += 2.0 * m * m * n + 2.0 * m ** 3 + (8.0 / 3.0) * m ** 3
        rot += 2.0 * m * m * n
    if right:
        f += 2.0 * n * n * m + 2.0 * n ** 3 + (8.0 / 3.0) * n ** 3
        rot += 2.0 * m * n * n
    return f + 3.0 * rot, 3.0 * rot


def soap_workload(dev, sq=4096, wide=14336, n_sq=4, n_wide=4, rank=32, noise=1e-3, ratio=10.0):
    """SOAP matrices: n_sq two-sided sq x sq, n_wide sq x wide with the wide
    side on the identity basis.  Gradients: fixed rank-32 spike at 10x the
    noise norm plus fresh Gaussian noise every step."""
    import torch
    import workloads as wl
    mats, spikes = [], []
    for kind, count, n in (("sq", n_sq, sq), ("wide", n_wide, wide)):
        for i in range(count):
            g = torch.Generator(device=dev)
            g.manual_seed(wl.seed_of("bench-cfg4", kind, i))
            m = sq
            d = dict(W=torch.randn(m, n, generator=g, device=dev) * 0.02,
                     G=torch.empty(m, n, device=dev),
                     M=torch.zeros(m, n, device=dev), V=torch.zeros(m, n, device=dev),
                     L=torch.zeros(m, m, device=dev), QL=torch.eye(m, device=dev))
            if kind == "sq":
                d["R"] = torch.zeros(n, n, device=dev)
                d["QR"] = torch.eye(n, device=dev)
            P = torch.randn(m, rank, generator=g, device=dev)
            Q = torch.randn(n, rank, generator=g, device=dev)
            mats.append(d)
            spikes.append((P @ Q.T, g))
    def fill():
        for d, (S, g) in zip(mats, spikes):
            E = torch.randn(d["G"].shape, generator=g, device=dev) * noise
            d["G"].copy_(E + S * (ratio * E.norm() / S.norm()))
    return mats, fill


def soap_bench(ctx, dev, steps=3, warm=10, side=4096):
    import torch
    mats, fill = soap_workload(dev, sq=side, wide=side * 14336 // 4096)
    fl, rot = 0.0, 0.0
    for d in mats:
        f, r = soap_flops(d["W"].shape[0], d["W"].shape[1], "L" in d, "R" in d)
        fl += f
        rot += r
    hp = dict(lr=3e-3, beta1=0.95, beta2=0.95, eps=1e-8, weight_decay=0.0, damping=0.0)
    for t in range(1, warm + 1):
        fill()
        ctx.soap_step(mats, t, **hp)
    torch.cuda.synchronize()
    # steps warm + 1 .. warm + steps timed as they run; the per-kernel
    # breakdown comes from as many further steps with the launch events on
    total = 0.0
    for t in range(warm + 1, warm + 1 + steps):
        fill()
        s = torch.cuda.Event(enable_timing=True)
        e = torch.cuda.Event(enable_timing=True)
        s.record()
        ctx.soap_step(mats, t, reserve=False, **hp)
        e.record()
        torch.cuda.synchronize()
        total += s.elapsed_time(e)
    ctx.profile(True)
    ctx.profile_read()
    for t in range(warm + 1 + steps, warm + 1 + 2 * steps):
        fill()
        ctx.soap_step(mats, t, reserve=False, **hp)
    torch.cuda.synchronize()
    prof = ctx.profile_read()
    ctx.profile(False)
    ms = total / steps
    k = {kk: round(v[0] / steps, 3) for kk, v in prof.items() if v[2]}
    rot_ms = prof["soap_rot"][0] / steps
    rot_exec = prof["soap_rot"][1] / steps
    return {"workload": f"soap_step 4 x {side}^2 (two-sided) + 4 x {side}x{side * 14336 // 4096} (left side only), steps "
                        f"{warm + 1}-{warm + steps} after {warm} warm steps; refresh qr(L Q), damping 0",
            "ms": round(ms, 3), "TFLOP/s": round(fl / (ms / 1e3) / 1e12, 1),
            "flops_per_step": fl, "matrices_per_s": round(len(mats) / (ms / 1e3), 1),
            "kernels_ms_per_step": k,
            "rotation_gemm": {"ms": round(rot_ms, 3),
                              "useful_TFLOP/s": round(rot / (rot_ms / 1e3) / 1e12, 1) if rot_ms else None,
                              "executed_TFLOP/s": round(rot_exec / (rot_ms / 1e3) / 1e12, 1) if rot_ms else None,
                              "note": "two-plane operands: 3 bf16 MMAs per useful product"},
            "kernels_note": ("kernels_ms_per_step: further steps with per-launch events (their overhead included); "
                             "with the events on, the refresh launches all 16 passes, the unneeded ones gated off "
                             "on the device (qr_chol, qr_rowblock, qr_trail include those launches)"),
            "gpu_launches": int(sum(v[2] for v in prof.values()) / steps)}


def soap_muon_bench(ctx, dev, steps=3, warm=10):
    """SOAP-Muon on the SOAP workload (the same matrices, sides and gradient
    stream): SOAP's refresh and rotations plus Newton-Schulz on every matrix."""
    import torch
    mats, fill = soap_workload(dev)
    for d in mats:
        d["B"] = d.pop("M")
    fl = 0.0
    for d in mats:
        m, n = d["W"].shape
        f, _ = soap_flops(m, n, "L" in d, "R" in d)
        fl += f + page_flops(m, n)
    hp = dict(lr=0.02, weight_decay=0.01, momentum=0.95, beta2=0.95, shampoo_beta=0.9, eps=1e-8, damping=0.0)
    for t in range(1, warm + 1):
        fill()
        ctx.soap_muon_step(mats, t, **hp)
    torch.cuda.synchronize()
    total = 0.0
    for t in range(warm + 1, warm + 1 + steps):
        fill()
        s = torch.cuda.Event(enable_timing=True)
        e = torch.cuda.Event(enable_timing=True)
        s.record()
        ctx.soap_muon_step(mats, t, reserve=False, **hp)
        e.record()
        torch.cuda.synchronize()
        total += s.elapsed_time(e)
    ctx.profile(True)
    ctx.profile_read()
    for t in range(warm + 1 + steps, warm + 1 + 2 * steps):
        fill()
        ctx.soap_muon_step(mats, t, reserve=False, **hp)
    torch.cuda.synchronize()
    prof = ctx.profile_read()
    ctx.profile(False)
    ms = total / steps
    return {"workload": f"soap_muon_step on the SOAP matrices (4 x 4096^2 two-sided, 4 x 4096x14336 left side), "
                        f"steps {warm + 1}-{warm + steps}; refresh qr(L Q), damping 0",
            "ms": round(ms, 3), "TFLOP/s": round(fl / (ms / 1e3) / 1e12, 1), "flops_per_step": fl,
            "matrices_per_s": round(len(mats) / (ms / 1e3), 1),
            "kernels_ms_per_step": {kk: round(v[0] / steps, 3) for kk, v in prof.items() if v[2]},
            "gpu_launches": int(sum(v[2] for v in prof.values()) / steps),
            "note": "flops: the SOAP count plus the Newton-Schulz page count of each matrix"}


def fwht_last(x):
    """Unnormalised Walsh-Hadamard transform along the last axis (power of 2)."""
    import torch
    n = x.shape[-1]
    y = x.reshape(-1, n)
    h = 1
    while h < n:
        y = y.view(y.shape[0], n // (2 * h), 2, h)
        y = torch.stack((y[:, :, 0, :] + y[:, :, 1, :], y[:, :, 0, :] - y[:, :, 1, :]), dim=2)
        h *= 2
    return y.reshape(x.shape)


def quintic_map(t, steps=5, coeffs=(3.4445, -4.7750, 2.0315)):
    a, b, c = coeffs
    for _ in range(steps):
        t = a * t + b * t ** 3 + c * t ** 5
    return t


def sv_spread(O, d):
    """Singular-value spread of the NS output of a dyadic known-SVD input
    G = H diag(d) H / n: H O H / n is diagonal in exact arithmetic with
    entries sign(d) phi^5(|d| / ||d||); its diagonal gives the output's
    singular values on the input's own singular vectors."""
    import numpy as np
    import torch
    n = O.shape[0]
    D = fwht_last(fwht_last(O.double()).T.contiguous()) / n
    diag = torch.diagonal(D).abs().cpu().numpy()
    off = float((torch.linalg.matrix_norm(D) ** 2 - (torch.diagonal(D) ** 2).sum()).clamp(min=0).sqrt())
    exact = quintic_map(np.abs(d) / (np.linalg.norm(d) + 1e-7))
    q = [0, 5, 50, 95, 100]
    return {"gpu_percentiles_0_5_50_95_100": [round(float(v), 4) for v in np.percentile(diag, q)],
            "exact_percentiles_0_5_50_95_100": [round(float(v), 4) for v in np.percentile(exact, q)],
            "max_abs_dev_from_exact": round(float(np.abs(diag - exact).max()), 5),
            "offdiag_rel": round(off / float(np.linalg.norm(diag)), 6)}


def extras(ctx, dev, args):
    """The other workloads, measured the same way (short runs)."""
    import torch
    import workloads as wl
    res = {}
    # single 256 x 512 Muon step (latency)
    W, G, B = (torch.from_numpy(x).to(dev) for x in wl.cfg1())
    ctx.reserve(0, [(256, 512)])
    call = lambda: ctx.muon_step([W], [G], [B], reserve=False)
    ms_eager = time_steps(call, 50, 5)
    graph = capture_graph(call)
    ms = time_steps(graph.replay, 50, 5)
    del graph
    res["muon_256x512_us"] = round(ms * 1e3, 1)
    res["muon_256x512_eager_call_us"] = round(ms_eager * 1e3, 1)
    ctx.workspace = None
    # MoE experts, grouped
    Ws, Gs, Bs, shapes = moe_workload(dev)
    ctx.reserve(0, shapes)
    call = lambda: ctx.muon_step(Ws, Gs, Bs, reserve=False)
    ms_eager = time_steps(call, 5, 2)
    graph = capture_graph(call)
    ms = time_steps(graph.replay, 5, 2)
    del graph
    ctx.profile(True)
    ctx.profile_read()
    call()
    torch.cuda.synchronize()
    prof = ctx.profile_read()
    ctx.profile(False)
    fl = sum(page_flops(m, n) for m, n in shapes)
    gemm = [k for k in ("gram", "poly", "update")]
    g_ms = sum(prof[k][0] for k in gemm)
    g_fl = sum(prof[k][1] for k in gemm)
    res["muon_moe_1536x768x2048"] = {
        "ms": round(ms, 3), "TFLOP/s": round(fl / (ms / 1e3) / 1e12, 1),
        "matrices_per_s": round(len(shapes) / (ms / 1e3), 1), "eager_call_ms": round(ms_eager, 3),
        "kernels_ms": {k: round(v[0], 3) for k, v in prof.items() if v[2]},
        "gemm_executed_TFLOP/s": round(g_fl / (g_ms / 1e3) / 1e12, 1) if g_ms else None,
        "note": "ms: CUDA-graph replay of the whole step; kernels_ms from one eager step"}
    del Ws, Gs, Bs
    ctx.workspace = None
    torch.cuda.empty_cache()
    # Newton-Schulz sweep on known-SVD inputs (condition number 1e4)
    sweep = {}
    for n in (512, 1024, 2048, 4096, 8192, 16384):
        Gt = dyadic_gpu(n, dev)
        out = torch.empty_like(Gt)
        ctx.reserve(2, [(n, n)])
        reps = 10 if n <= 4096 else 3
        ms = time_steps(lambda: ctx.ns_orthogonalize([Gt], [out], reserve=False), reps, 2)
        sweep[str(n)] = {"ms": round(ms, 3), "TFLOP/s": round(page_flops(n, n) / (ms / 1e3) / 1e12, 1)}
        ctx.workspace = None
        d = wl.dyadic_spectrum(wl.rng_of("cfg5", n), n, 1e4)
        sweep[str(n)]["sv_spread"] = sv_spread(out, d)
        del Gt, out
        ctx.workspace = None
        torch.cuda.empty_cache()
    Ht = heads_gpu(4096, 128, dev)                    # one [4096, 128, 128] tensor
    Ho = torch.empty_like(Ht)
    ctx.reserve(2, [(128, 128)] * 4096)
    call = lambda: ctx.ns_orthogonalize_batch(Ht, Ho, reserve=False)
    ms_eager = time_steps(call, 20, 3)
    # the per-matrix list form of the same call (4096 tensors marshalled)
    Hl, Hol = list(Ht.unbind(0)), list(Ho.unbind(0))
    ms_list = time_steps(lambda: ctx.ns_orthogonalize(Hl, Hol, reserve=False), 5, 2)
    del Hl, Hol
    # the same call replayed from a CUDA graph: the device time alone
    graph = capture_graph(call)
    ms = time_steps(graph.replay, 20, 3)
    del graph
    ctx.profile(True)
    ctx.profile_read()
    call()
    torch.cuda.synchronize()
    kern = ctx.profile_read()["ns_small"]
    ctx.profile(False)
    fl = 4096 * page_flops(128, 128)
    sweep["heads_4096x128x128"] = {"ms": round(ms, 3), "TFLOP/s": round(fl / (ms / 1e3) / 1e12, 2),
                                   "eager_call_ms": round(ms_eager, 3), "list_call_ms": round(ms_list, 3),
                                   "ns_small_kernel_ms": round(kern[0], 3), "ns_small_launches": kern[2],
                                   "note": "ms: CUDA-graph replay; eager_call_ms: the strided batch call "
                                           "(ns_orthogonalize_strided) eagerly; list_call_ms: the same "
                                           "matrices as a list of 4096 tensors"}
    res["ns_sweep"] = sweep
    del Ht, Ho
    ctx.workspace = None
    torch.cuda.empty_cache()
    res["soap"] = soap_bench(ctx, dev)
    ctx.workspace = None
    torch.cuda.empty_cache()
    res["soap_muon"] = soap_muon_bench(ctx, dev)
    ctx.workspace = None
    torch.cuda.empty_cache()
    return res


# ----------------------------------------------------------------------------- CPU oracle

def cpu_baseline(seconds):
    """The fp64 oracle as it stands, on this host's cores, on a bounded
    sample of the same workload: Muon steps on layer-0 matrices of the dense
    GPT (Wk, Wv: 1024 x 4096; then Wq if time allows)."""
    import numpy as np
    import workloads as wl
    from oracle import muon as omuon
    cores = len(os.sched_getaffinity(0))
    done_flops, t_total, names = 0.0, 0.0, []
    for name, m, n in [("wk", 1024, 4096), ("wv", 1024, 4096), ("wq", 4096, 4096)]:
        W, G = wl.cfg2_matrix(0, name, m, n)
        B = np.zeros_like(W)
        t = time.perf_counter()
        omuon.muon_step(W, G, B)
        t_total += time.perf_counter() - t
        done_flops += page_flops(m, n)
        names.append(f"{name} {m}x{n}")
        if t_total > seconds:
            break
    return {"value": round(done_flops / t_total / 1e12, 5), "unit": UNIT, "cores": cores,
            "kind": "oracle", "seconds": round(t_total, 2),
            "sample": "fp64 NumPy Muon steps on layer-0 matrices of the dense GPT: " + ", ".join(names)}


def run_reference(args, world, rank):
    """Reference arm: the oracle, timed on the host cores."""
    if rank != 0:
        return None
    cores = len(os.sched_getaffinity(0))
    import numpy as np
    import workloads as wl
    from oracle import muon as omuon
    W, G = wl.cfg2_matrix(0, "wk", 1024, 4096)
    B = np.zeros_like(W)
    fl = page_flops(1024, 4096)
    for _ in range(args.warmup):
        omuon.muon_step(W, G, B)
    t = time.perf_counter()
    for _ in range(args.steps):
        omuon.muon_step(W, G, B)
    dt = (time.perf_counter() - t) / args.steps
    value = round(fl / dt / 1e12, 5)
    sample = "one fp64 NumPy Muon step on the layer-0 Wk matrix (1024 x 4096) per step"
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt * 1e3, 2),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": WORKLOAD, "sample": sample},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def run_soap_only(args, world, rank, local):
    """The SOAP step alone (profiling and ncu runs)."""
    import torch
    from matrix_aware_optimizers_muon_b200 import Context
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    ctx = Context(local)
    res = soap_bench(ctx, dev, steps=args.steps, warm=max(args.warmup, 1), side=args.soap_side)
    return {"metric": METRIC, "value": res["TFLOP/s"], "unit": UNIT, "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": res["ms"], "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": {"workload": res["workload"]},
            "soap": res}


def run_moe_only(args, world, rank, local):
    """The MoE Muon step alone (profiling and ncu runs): --moe-layers x
    --moe-experts experts, three matrices each, steps timed with CUDA events
    after the warm-up, then one step with the per-launch events on."""
    import torch
    from matrix_aware_optimizers_muon_b200 import Context
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    ctx = Context(local)
    Ws, Gs, Bs, shapes = moe_workload(dev, layers=args.moe_layers, experts=args.moe_experts)
    ctx.reserve(0, shapes)
    call = lambda: ctx.muon_step(Ws, Gs, Bs, reserve=False)
    ms = time_steps(call, args.steps, max(args.warmup, 3))
    ctx.profile(True)
    ctx.profile_read()
    call()
    torch.cuda.synchronize()
    prof = ctx.profile_read()
    ctx.profile(False)
    fl = sum(page_flops(m, n) for m, n in shapes)
    gemm = ("gram", "poly", "update")
    g_ms = sum(prof[k][0] for k in gemm)
    g_fl = sum(prof[k][1] for k in gemm)
    return {"metric": METRIC, "value": round(fl / (ms / 1e3) / 1e12, 1), "unit": UNIT, "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": f"muon_step MoE experts: {args.moe_layers} layers x {args.moe_experts} experts x "
                                   f"(gate, up 768x2048; down 2048x768), {len(shapes)} matrices"},
            "matrices_per_s": round(len(shapes) / (ms / 1e3), 1),
            "kernels_ms": {k: round(v[0], 3) for k, v in prof.items() if v[2]},
            "gemm_executed_TFLOP/s": {k: round(prof[k][1] / (prof[k][0] / 1e3) / 1e12, 1) for k in gemm if prof[k][0]},
            "gemm_executed_TFLOP/s_all": round(g_fl / (g_ms / 1e3) / 1e12, 1) if g_ms else None}


def run_heads_only(args, world, rank, local):
    """Newton-Schulz on --heads matrices of 128 x 128 in one strided call
    (profiling and ncu runs)."""
    import torch
    from matrix_aware_optimizers_muon_b200 import Context
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    ctx = Context(local)
    Ht = heads_gpu(args.heads, 128, dev)
    Ho = torch.empty_like(Ht)
    ctx.reserve(2, [(128, 128)] * args.heads)
    call = lambda: ctx.ns_orthogonalize_batch(Ht, Ho, reserve=False)
    ms = time_steps(call, args.steps, max(args.warmup, 3))
    fl = args.heads * page_flops(128, 128)
    return {"metric": METRIC, "value": round(fl / (ms / 1e3) / 1e12, 1), "unit": UNIT, "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 4), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": f"ns_orthogonalize_strided on {args.heads} matrices of 128 x 128"}}


def gemm_vs_cublas(args, local):
    """The Newton-Schulz products of the dense-GPT 4096 x 14336 bucket (and a
    square 8192^3 product) through this library's GEMM and through cuBLAS
    (torch.bmm / torch.matmul) on the same bf16 operands.  Each phase runs
    back to back for --seconds after a 1 s warm-up, so both sides are timed
    at the clock the 1 kW power cap settles them at; the SM clock and board
    power are sampled per phase.  --once runs each product once on a batch
    of 3 (a small case for counter captures)."""
    import torch
    from matrix_aware_optimizers_muon_b200 import Context
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    ctx = Context(local)
    gen = torch.Generator(device=dev).manual_seed(5)
    bt = 3 if args.once else 96
    m, n = 4096, 14336
    X = (torch.randn(bt, m, n, device=dev, generator=gen) * 0.02).to(torch.bfloat16)
    P = (torch.randn(bt, m, m, device=dev, generator=gen) * 0.02).to(torch.bfloat16)
    P = ((P + P.mT) * 0.5).contiguous()
    Y = torch.empty_like(X)
    A = torch.empty(bt, m, m, device=dev, dtype=torch.bfloat16)
    s8 = 8192
    A8 = (torch.randn(s8, s8, device=dev, generator=gen) * 0.02).to(torch.bfloat16)
    B8 = (torch.randn(s8, s8, device=dev, generator=gen) * 0.02).to(torch.bfloat16)
    D8 = torch.empty(s8, s8, device=dev, dtype=torch.bfloat16)
    f_prod = 2.0 * m * m * n * bt                   # Gram or update, full product
    ops = [
        ("update P X", "ours", f_prod,
         lambda: ctx.gemm_bf16(P, X, Y, M=m, N=n, K=m, batch=bt, b_mn=True)),
        ("update P X", "cublas", f_prod, lambda: torch.bmm(P, X, out=Y)),
        ("Gram X X^T", "ours (symmetric)", f_prod,
         lambda: ctx.gemm_bf16(X, X, A, M=m, N=m, K=n, batch=bt, sym=True)),
        ("Gram X X^T", "ours (full)", f_prod, lambda: ctx.gemm_bf16(X, X, A, M=m, N=m, K=n, batch=bt)),
        ("Gram X X^T", "cublas", f_prod, lambda: torch.bmm(X, X.mT, out=A)),
        ("8192^3", "ours", 2.0 * s8 ** 3, lambda: ctx.gemm_bf16(A8, B8, D8, M=s8, N=s8, K=s8, b_mn=True)),
        ("8192^3", "cublas", 2.0 * s8 ** 3, lambda: torch.matmul(A8, B8, out=D8)),
    ]
    torch.cuda.synchronize()
    if args.once:
        for _, _, _, fn in ops:
            fn()
        torch.cuda.synchronize()
        return {"workload": "gemm-vs-cublas once (batch 3)", "device_status": ctx.device_status()}
    rows = []
    for _rep in range(2):
        for prod, impl, flops, fn in ops:
            t0 = time.time()
            while time.time() - t0 < 1.0:
                for _ in range(4):
                    fn()
                torch.cuda.synchronize()
            clk = ClockSampler(local)
            clk.start()
            ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            reps = 0
            t0 = time.time()
            ev0.record()
            while time.time() - t0 < args.seconds:
                for _ in range(4):
                    fn()
                reps += 4
                torch.cuda.synchronize()
            ev1.record()
            torch.cuda.synchronize()
            c = clk.stop() or {}
            ms = ev0.elapsed_time(ev1) / reps
            tf = flops / (ms * 1e-3) / 1e12
            rows.append({"product": prod, "impl": impl, "ms": round(ms, 4), "TFLOP/s": round(tf, 1),
                         "sm_mhz": c.get("sm_mhz"), "power_w": c.get("power_w"),
                         "TFLOP/s per GHz": round(tf / c["sm_mhz"] * 1e3, 1) if c.get("sm_mhz") else None,
                         "reasons": c.get("reasons")})
    return {"workload": f"gemm-vs-cublas sustained, batch {bt} of 4096 x 14336 (flops: full products)",
            "phases": rows, "device_status": ctx.device_status()}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-e2e", dest="e2e", action="store_false")
    ap.add_argument("--e2e-groups", type=int, default=32,
                    help="e2e: layer groups whose gradient copies overlap the previous group's step")
    ap.add_argument("--no-extras", dest="extras", action="store_false")
    ap.add_argument("--no-cpu-baseline", dest="cpu_baseline", action="store_false")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--workload", choices=["muon", "soap", "moe", "heads", "gemm-vs-cublas"], default="muon",
                    help="muon: the dense-GPT Muon step (the benchmark line); soap: the SOAP step alone; "
                         "moe: the MoE Muon step alone; "
                         "gemm-vs-cublas: the NS products against cuBLAS at the sustained clock")
    ap.add_argument("--heads", type=int, default=4096, help="heads: matrices of 128 x 128")
    ap.add_argument("--moe-layers", type=int, default=4, help="moe: layers (4 = the benchmark workload)")
    ap.add_argument("--moe-experts", type=int, default=128, help="moe: experts per layer (128 = the benchmark)")
    ap.add_argument("--seconds", type=float, default=3.0, help="gemm-vs-cublas: timed seconds per phase")
    ap.add_argument("--once", action="store_true", help="gemm-vs-cublas: each product once, batch 3")
    ap.add_argument("--soap-side", type=int, default=4096,
                    help="soap: side of the square matrices and factors (4096 = the benchmark workload; "
                         "1024 for small profiling cases)")
    ap.add_argument("--layers", type=int, default=32,
                    help="dense-GPT layers (32 = the benchmark workload; fewer for small profiling cases)")
    args = ap.parse_args()
    world, rank, local = dist_setup()
    if args.impl == "reference":
        out = run_reference(args, world, rank)
    elif args.workload == "soap":
        out = run_soap_only(args, world, rank, local)
    elif args.workload == "moe":
        out = run_moe_only(args, world, rank, local)
    elif args.workload == "heads":
        out = run_heads_only(args, world, rank, local)
    elif args.workload == "gemm-vs-cublas":
        out = gemm_vs_cublas(args, local)
    else:
        out = run_ours(args, world, rank, local)
    if rank == 0 and out is not None:
        print(json.dumps(out), flush=True)


if __name__ == "__main__":
    main()
