"""Benchmark of the H3-style DiT attention core on B200.

One step = the whole hot path over one batch of the 5 s 1344x768 clip latent
(31x48x84 = 124,992 tokens, 56 heads x 96, bf16, structured synthetic data):
    fused QK-RMSNorm + 3D RoPE, with the router's block pooling folded in
    ->  router scores and top-k (sparsity 0.75)  ->  block-sparse attention
    ->  dense attention
The headline value is attention TFLOP/s over the whole step (algorithmic
FLOPs of both attention passes / step time).  Per-kernel times come from CUDA
events on the launching stream inside the timed region.  Beside the headline,
outside the timed step, the same four launches run on the 10 s clip
(61x48x84 = 245,952 tokens, sparsity 0.80) and are reported under
kernels.video10s_untimed_step (--no-video10s skips them).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

Under torchrun (N > 1) every rank runs its own clip (weak scaling, no data-path
collective); rank 0 prints the max-over-ranks line.  --impl reference times the
fp64 CPU oracle on a bounded sample of the same workload instead.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

WORKLOAD = "video5s_sparse"
FFN_WIDTH = 14336  # DiT FFN width of the model table (52hbtv.com H3-Image page, section 二)
SPARSITY = 0.75
L2_GB = 0.126  # B200 L2: 126 MB
METRIC = "attention TFLOP/s and % of B200 bf16 peak at ~125k tokens; prologue GB/s vs HBM"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
PROFILE_TRAFFIC = os.path.join(ROOT, "profiles", "traffic.json")


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def attention_flops(N: int, heads: int, B: int, d: int = 96, blocks: np.ndarray | None = None, block: int = 128):
    """4*d FLOPs per (query, key) pair attended: QK^T and PV, 2 FLOPs per MAC each."""
    if blocks is None:
        return 4.0 * d * heads * B * float(N) * float(N)
    nblk = (N + block - 1) // block
    lens = np.full(nblk, block, dtype=np.float64)
    lens[-1] = N - (nblk - 1) * block
    # sum over (b, h, i, j in list_i) of |blk_i| * |blk_j|
    pairs = lens[blocks].sum(axis=-1)                  # [B, H, nblk]
    return 4.0 * d * float((pairs * lens[None, None, :]).sum())


def prologue_bytes(N: int, heads: int, B: int, d: int = 96) -> float:
    """Read + write of Q and K in bf16: 4 bytes per element per tensor pair."""
    return 2.0 * 2 * 2 * B * N * heads * d


def router_bytes(N: int, heads: int, B: int, d: int = 96) -> float:
    """The separate pooling pass reads Q and K once."""
    return 2.0 * 2 * B * N * heads * d


def pooled_bytes(N: int, heads: int, B: int, d: int = 96, block: int = 128) -> float:
    """fp32 block means of Q and K written by the fused prologue."""
    return 2.0 * 4 * B * heads * ((N + block - 1) // block) * d


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples during the timed region."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.QUERY}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [ln for ln in out.splitlines() if ln.strip()]

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in getattr(self, "lines", []):
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


def dist_setup(n_gpus: int):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch.distributed as dist

        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return rank, world, local


def allreduce_max(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch.distributed as dist

    dev = "cuda" if torch.cuda.is_available() else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


def load_traffic():
    """ncu DRAM bytes per launch, kept only while the kernel sources are unchanged."""
    if not os.path.exists(PROFILE_TRAFFIC):
        return {}
    import hashlib

    with open(PROFILE_TRAFFIC) as f:
        rec = json.load(f)
    out = {}
    for kernel, ent in rec.items():
        # every file the kernel is compiled from, hashed in the listed order
        paths = [os.path.join(ROOT, p) for p in ent["sources"]]
        if not all(os.path.exists(p) for p in paths):
            continue
        h = hashlib.sha256()
        for p in paths:
            with open(p, "rb") as f:
                h.update(f.read())
        if h.hexdigest() == ent["sha256"]:
            out[kernel] = ent
    return out


def config_of(w, world: int, kk: int) -> dict:
    """The workload description both arms print (kk: KV blocks kept per query block)."""
    B, N, heads, D, grid = w.B, w.N, w.heads, w.head_dim, w.grid
    nblk = (N + 127) // 128
    wide = D != 96
    gb = B * N * heads * D * 2 / 1e9
    return {
        "workload": f"{w.name}: B={B}, {heads} heads x {D}, grid {grid[0]}x{grid[1]}x{grid[2]} = {N:,} tokens "
                    f"per GPU; " + (f"router with its own pooling (sparsity {SPARSITY}, k={kk}/{nblk}) + sparse + "
                                    "dense attention (no prologue: its 3D RoPE is defined for 96 channels)" if wide
                                    else f"prologue with block pooling + router scores/top-k (sparsity {SPARSITY}, "
                                    f"k={kk}/{nblk}) + sparse + dense attention"),
        "tokens": N, "heads": heads, "head_dim": D, "batch_per_gpu": B, "sparsity": SPARSITY,
        "parallelism": f"dp{world} (independent clips per GPU)",
        "l2": (f"inputs larger than L2 (Q, K, V {gb:.2f} GB each); no explicit flush" if 3 * gb > L2_GB
               else f"inputs fit in L2 (Q, K, V {gb * 1e3:.2f} MB each): a correctness-size case, not a timing one"),
    }


# ----------------------------------------------------------------- GPU arm

def run_gpu(args, rank, world, local):
    import rope_block_sparse_b200 as h3a
    from rope_block_sparse_b200 import synth

    w = synth.WORKLOADS[args.workload]
    grid, heads, B, N = w.grid, w.heads, w.B, w.N
    d = synth.draw_workload(args.workload, seed=rank)
    dev = torch.device("cuda", local)
    q, k, v = (d[n].to(dev) for n in "qkv")
    gq, gk = d["gamma_q"].to(dev), d["gamma_k"].to(dev)
    # the 3D RoPE prologue is defined for 96 channels; a 128-wide workload runs
    # the router (with its own pooling) and attention on the inputs directly
    wide = w.head_dim != 96
    qn, kn = (q, k) if wide else (torch.empty_like(q), torch.empty_like(k))
    o_dense, o_sparse = torch.empty_like(q), torch.empty_like(q)
    nblk = (N + 127) // 128
    kk = h3a.route_k(nblk, SPARSITY)
    blocks = torch.empty((B, heads, nblk, kk), dtype=torch.int32, device=dev)
    ws = torch.empty(h3a.route_workspace_size(q), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    # one step: the prologue with the router's pooling folded in, the router's
    # scores and top-k from those means, sparse attention, dense attention
    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        if not wide:
            h3a.qk_norm_rope_pool(q, k, gq, gk, grid, workspace=ws, out=(qn, kn))
        if ev is not None:
            ev[1].record(stream)
        if wide:
            h3a.route(qn, kn, SPARSITY, workspace=ws, out=blocks)
        else:
            h3a.route_pooled(qn, SPARSITY, ws, out=blocks)
        if ev is not None:
            ev[2].record(stream)
        h3a.attention(qn, kn, v, blocks, out=o_sparse)
        if ev is not None:
            ev[3].record(stream)
        h3a.attention(qn, kn, v, None, out=o_dense)
        if ev is not None:
            ev[4].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if h3a.last_device_error() != 0:
        raise RuntimeError("device-side timeout during warm-up")
    flops_dense = attention_flops(N, heads, B, d=w.head_dim)
    flops_sparse = attention_flops(N, heads, B, d=w.head_dim, blocks=blocks.cpu().numpy())

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        for i in range(args.steps):
            step(evs[i])
        torch.cuda.synchronize()
    barrier(world)
    if h3a.last_device_error() != 0:
        raise RuntimeError("device-side timeout in the timed region")
    per = np.array([[evs[i][j].elapsed_time(evs[i][j + 1]) for j in range(4)] for i in range(args.steps)])
    step_ms_local = float(sum(evs[i][0].elapsed_time(evs[i][4]) for i in range(args.steps)) / args.steps)
    step_ms = allreduce_max(step_ms_local, world)
    kern_ms = {name: allreduce_max(float(per[:, j].mean()), world)
               for j, name in enumerate(["prologue_pool", "router_scores", "attention_sparse", "attention_dense"])}

    # for comparison, outside the timed region: the separate prologue and the
    # router with its own pooling pass
    sep = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(5)]
    for i in range(0 if wide else 6):
        e = sep[i - 1] if i > 0 else None
        if e is not None:
            e[0].record(stream)
        h3a.qk_norm_rope(q, k, gq, gk, grid, out=(qn, kn))
        if e is not None:
            e[1].record(stream)
        h3a.route(qn, kn, SPARSITY, workspace=ws, out=blocks)
        if e is not None:
            e[2].record(stream)
    torch.cuda.synchronize()
    if not wide:
        # the variant whose RMSNorm spans the whole hidden state, outside the timed step
        gfq = synth.draw_gamma("gamma_q", rank, heads * 96).to(dev)
        gfk = synth.draw_gamma("gamma_k", rank, heads * 96).to(dev)
        fe = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
        for i in range(4):
            if i == 3:
                fe[0].record(stream)
            h3a.qk_fullnorm_rope(q, k, gfq, gfk, grid, out=(qn, kn))
        fe[1].record(stream)
        torch.cuda.synchronize()
        kern_ms["prologue_fullnorm"] = allreduce_max(fe[0].elapsed_time(fe[1]), world)
    dit = time_dit_ops(h3a, synth, q, k, B, N, heads * w.head_dim, stream, world, rank)
    pk, pk_src = peaks()
    video10s = None
    if args.video10s and not wide:
        video10s = time_video10s(h3a, synth, stream, world, rank, pk)
    if wide:
        kern_ms["prologue"] = kern_ms["prologue_pool"] = 0.0
        kern_ms["router"] = kern_ms["router_scores"]
    else:
        kern_ms["prologue"] = allreduce_max(float(np.mean([e[0].elapsed_time(e[1]) for e in sep])), world)
        kern_ms["router"] = allreduce_max(float(np.mean([e[1].elapsed_time(e[2]) for e in sep])), world)

    # end to end through the public API with host buffers: every step copies its
    # Q, K, V in from pinned host memory and both outputs back out.  The copies
    # run on their own streams, double-buffered: step i+1's inputs go up and
    # step i-1's outputs come down while step i computes; within a step the
    # prologue and router start once Q and K are in (V is still uploading) and
    # the sparse output goes down while dense attention runs.  The timed span
    # runs from the first upload's start to the last download's end.
    e2e = None
    if args.e2e_steps > 0:
        hq, hk, hv = (d[n].pin_memory() for n in "qkv")
        hod = torch.empty(q.shape, dtype=torch.bfloat16).pin_memory()
        hos = torch.empty(q.shape, dtype=torch.bfloat16).pin_memory()
        h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv))
        d2h = hod.numel() * 2 + hos.numel() * 2
        ins = [(q, k, v), tuple(torch.empty_like(t) for t in (q, k, v))]
        outs = [(o_sparse, o_dense), (torch.empty_like(o_sparse), torch.empty_like(o_dense))]
        up, down = torch.cuda.Stream(), torch.cuda.Stream()
        ev = lambda: torch.cuda.Event()
        qk_ready, v_ready, in_free = [ev(), ev()], [ev(), ev()], [ev(), ev()]
        sparse_ready, out_ready, out_free = [ev(), ev()], [ev(), ev()], [ev(), ev()]

        def compute(slot):
            qb, kb, vb = ins[slot]
            osb, odb = outs[slot]
            stream.wait_event(qk_ready[slot])
            if wide:
                h3a.route(qb, kb, SPARSITY, workspace=ws, out=blocks)
                qa, ka = qb, kb
            else:
                h3a.qk_norm_rope_pool(qb, kb, gq, gk, grid, workspace=ws, out=(qn, kn))
                h3a.route_pooled(qn, SPARSITY, ws, out=blocks)
                qa, ka = qn, kn
            stream.wait_event(v_ready[slot])
            h3a.attention(qa, ka, vb, blocks, out=osb)
            sparse_ready[slot].record(stream)
            h3a.attention(qa, ka, vb, None, out=odb)

        def upload(slot):
            with torch.cuda.stream(up):
                up.wait_event(in_free[slot])
                ins[slot][0].copy_(hq, non_blocking=True)
                ins[slot][1].copy_(hk, non_blocking=True)
                qk_ready[slot].record(up)
                ins[slot][2].copy_(hv, non_blocking=True)
                v_ready[slot].record(up)

        def run(nsteps, t0=None, t1=None):
            for e in in_free + out_free:
                e.record(stream)  # every slot starts free
            if t0 is not None:
                t0.record(up)
            upload(0)
            for i in range(nsteps):
                slot = i % 2
                if i + 1 < nsteps:
                    upload(1 - slot)
                stream.wait_event(out_free[slot])
                compute(slot)
                in_free[slot].record(stream)
                out_ready[slot].record(stream)
                with torch.cuda.stream(down):
                    down.wait_event(sparse_ready[slot])
                    hos.copy_(outs[slot][0], non_blocking=True)
                    down.wait_event(out_ready[slot])
                    hod.copy_(outs[slot][1], non_blocking=True)
                    out_free[slot].record(down)
            if t1 is not None:
                t1.record(down)

        run(2)
        torch.cuda.synchronize()
        barrier(world)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        run(args.e2e_steps, e0, e1)
        torch.cuda.synchronize()
        barrier(world)
        e2e_ms = allreduce_max(e0.elapsed_time(e1) / args.e2e_steps, world)
        e2e = {"value": round(world * (flops_dense + flops_sparse) / (e2e_ms * 1e-3) / 1e12, 3), "unit": "TFLOP/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": round(e2e_ms, 3),
               "steps": args.e2e_steps,
               "overlap": "uploads and downloads on their own streams, double-buffered; the prologue and router "
                          "start once Q and K are in, the sparse output goes down during dense attention"}
        del ins[1], outs[1]
    clocks = clk.summary()
    if rank != 0:
        return None

    dense_tflops = flops_dense / (kern_ms["attention_dense"] * 1e-3) / 1e12
    sparse_tflops = flops_sparse / (kern_ms["attention_sparse"] * 1e-3) / 1e12
    D = w.head_dim
    router_gbs = router_bytes(N, heads, B, D) / (kern_ms["router"] * 1e-3) / 1e9
    if not wide:
        pro_gbs = prologue_bytes(N, heads, B) / (kern_ms["prologue"] * 1e-3) / 1e9
        fused_gbs = (prologue_bytes(N, heads, B) + pooled_bytes(N, heads, B)) / (kern_ms["prologue_pool"] * 1e-3) / 1e9
    # the sparse path's routing cost: scores + top-k, plus what pooling adds to the prologue
    route_cost = kern_ms["router_scores"] + max(0.0, kern_ms["prologue_pool"] - kern_ms["prologue"])
    traffic = load_traffic()
    peak_t = pk["bf16_tflops_sustained"]
    line = {
        "metric": METRIC,
        "value": round(world * (flops_dense + flops_sparse) / (step_ms * 1e-3) / 1e12, 3),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(step_ms, 3),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic",
        "config": config_of(w, world, kk),
        "roofline": {
            "kernel": "attention_kernel (dense)",
            "bound": "tensor",
            "achieved": round(dense_tflops, 2),
            "peak": peak_t,
            "unit": "TFLOP/s",
            "frac": round(dense_tflops / peak_t, 4),
            "peak_source": f"{pk_src} bf16 sustained (kernel timed inside a long step)",
            "frac_of_burst": round(dense_tflops / pk["bf16_tflops"], 4),
            "frac_of_spec_2250": round(dense_tflops / 2250.0, 4),
            "traffic": None if wide else traffic.get("attention_dense", {}).get("bytes_per_launch"),
            "algorithmic_flops_per_launch": flops_dense,
        },
        "kernels": ({
            "router": {"ms": round(kern_ms["router"], 4), "pool_read_GB/s": round(router_gbs, 1)},
        } if wide else {
            "prologue_pool": {"ms": round(kern_ms["prologue_pool"], 4), "GB/s": round(fused_gbs, 1),
                              "frac_hbm": round(fused_gbs / pk["hbm_gbs"], 4),
                              "frac_8TBs": round(fused_gbs / 8000.0, 4),
                              "traffic": traffic.get("prologue_pool", {}).get("bytes_per_launch")},
            "router_scores": {"ms": round(kern_ms["router_scores"], 4)},
            "separate_prologue_untimed_step": {"ms": round(kern_ms["prologue"], 4), "GB/s": round(pro_gbs, 1),
                                               "frac_hbm": round(pro_gbs / pk["hbm_gbs"], 4),
                                               "frac_8TBs": round(pro_gbs / 8000.0, 4),
                                               "traffic": traffic.get("prologue", {}).get("bytes_per_launch")},
            "separate_router_untimed_step": {"ms": round(kern_ms["router"], 4),
                                             "pool_read_GB/s": round(router_gbs, 1)},
            "prologue_fullwidth_rmsnorm_untimed_step": {
                "traffic": traffic.get("prologue_fullnorm", {}).get("bytes_per_launch"),
                "ms": round(kern_ms["prologue_fullnorm"], 4),
                "GB/s": round(prologue_bytes(N, heads, B) / (kern_ms["prologue_fullnorm"] * 1e-3) / 1e9, 1),
                "frac_hbm": round(prologue_bytes(N, heads, B) / (kern_ms["prologue_fullnorm"] * 1e-3) / 1e9
                                  / pk["hbm_gbs"], 4)},
        }) | {
            "attention_sparse": {"ms": round(kern_ms["attention_sparse"], 3), "TFLOP/s": round(sparse_tflops, 2),
                                 "effective_dense_equiv_TFLOP/s":
                                     round(flops_dense / (kern_ms["attention_sparse"] * 1e-3) / 1e12, 2),
                                 "algorithmic_flops": flops_sparse},
            "attention_dense": {"ms": round(kern_ms["attention_dense"], 3), "TFLOP/s": round(dense_tflops, 2)},
            "sparse_speedup_incl_router": round(kern_ms["attention_dense"] /
                                                (kern_ms["attention_sparse"] + route_cost), 3),
        } | {name: dict(ent, frac_hbm=round(ent["GB/s"] / pk["hbm_gbs"], 4),
                        traffic=traffic.get(ent.pop("traffic_key"), {}).get("bytes_per_launch"))
             for name, ent in dit.items()} | ({"video10s_untimed_step": video10s} if video10s else {}),
        "gpu_launches": args.steps * 4,
        "clocks": clocks,
        "e2e": e2e,
    }
    if args.cpu_baseline and world == 1:
        line["cpu_baseline"] = cpu_baseline(d, w, args.cpu_rows)
    return line


def time_video10s(h3a, synth, stream, world, rank, pk, reps=2):
    """The 10 s clip (61x48x84 = 245,952 tokens, 56 heads x 96), outside the
    timed step: the same four launches as a step -- prologue with pooling,
    router scores/top-k at sparsity 0.80, sparse attention, dense attention --
    one untimed pass, then `reps` timed with CUDA events on the launching
    stream.  Returns the per-kernel times, dense and sparse TFLOP/s, their
    fractions of the measured bf16 peaks and the sparse/dense wall-clock ratio
    with routing charged to the sparse path."""
    name, sparsity = "video10s", 0.80
    w = synth.WORKLOADS[name]
    d = synth.draw_workload(name, seed=rank)
    dev = torch.device("cuda", torch.cuda.current_device())
    q, k, v = (d[n].to(dev) for n in "qkv")
    gq, gk = d["gamma_q"].to(dev), d["gamma_k"].to(dev)
    del d
    qn, kn = torch.empty_like(q), torch.empty_like(k)
    o_dense, o_sparse = torch.empty_like(q), torch.empty_like(q)
    nblk = (w.N + 127) // 128
    kk = h3a.route_k(nblk, sparsity)
    blocks = torch.empty((w.B, w.heads, nblk, kk), dtype=torch.int32, device=dev)
    ws = torch.empty(h3a.route_workspace_size(q), dtype=torch.uint8, device=dev)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(reps + 1)]
    for i in range(reps + 1):
        ev = evs[i]
        ev[0].record(stream)
        h3a.qk_norm_rope_pool(q, k, gq, gk, w.grid, workspace=ws, out=(qn, kn))
        ev[1].record(stream)
        h3a.route_pooled(qn, sparsity, ws, out=blocks)
        ev[2].record(stream)
        h3a.attention(qn, kn, v, blocks, out=o_sparse)
        ev[3].record(stream)
        h3a.attention(qn, kn, v, None, out=o_dense)
        ev[4].record(stream)
    torch.cuda.synchronize()
    if h3a.last_device_error() != 0:
        raise RuntimeError("device-side timeout in the 245,952-token pass")
    ms = [allreduce_max(float(np.mean([evs[i][j].elapsed_time(evs[i][j + 1]) for i in range(1, reps + 1)])), world)
          for j in range(4)]
    flops_dense = attention_flops(w.N, w.heads, w.B)
    flops_sparse = attention_flops(w.N, w.heads, w.B, blocks=blocks.cpu().numpy())
    pro_bytes = prologue_bytes(w.N, w.heads, w.B) + pooled_bytes(w.N, w.heads, w.B)
    dense_t = flops_dense / (ms[3] * 1e-3) / 1e12
    sparse_t = flops_sparse / (ms[2] * 1e-3) / 1e12
    del q, k, v, qn, kn, o_dense, o_sparse, blocks, ws
    torch.cuda.empty_cache()
    return {
        "workload": f"{name}: B=1, 56 heads x 96, grid 61x48x84 = {w.N:,} tokens; prologue with block pooling + "
                    f"router scores/top-k (sparsity {sparsity}, k={kk}/{nblk}) + sparse + dense attention; "
                    f"{reps} timed passes after one untimed",
        "prologue_pool_ms": round(ms[0], 4),
        "prologue_pool_GB/s": round(pro_bytes / (ms[0] * 1e-3) / 1e9, 1),
        "router_scores_ms": round(ms[1], 4),
        "attention_sparse_ms": round(ms[2], 3),
        "attention_dense_ms": round(ms[3], 3),
        "dense_TFLOP/s": round(dense_t, 2),
        "dense_frac_sustained": round(dense_t / pk["bf16_tflops_sustained"], 4),
        "dense_frac_burst": round(dense_t / pk["bf16_tflops"], 4),
        "sparse_TFLOP/s": round(sparse_t, 2),
        "sparse_frac_sustained": round(sparse_t / pk["bf16_tflops_sustained"], 4),
        "sparse_effective_dense_equiv_TFLOP/s": round(flops_dense / (ms[2] * 1e-3) / 1e12, 2),
        "algorithmic_flops_dense": flops_dense,
        "algorithmic_flops_sparse": flops_sparse,
        "sparse_speedup_incl_router": round(ms[3] / (ms[2] + ms[1]), 3),
    }


def time_dit_ops(h3a, synth, q, k, B, N, width, stream, world, rank, reps=10):
    """The other fused DiT operators at the clip's shape, outside the timed step:
    the gated residual + AdaLN update over B*N rows of the `width`-wide hidden
    state (x and f are the resident Q and K buffers viewed as [B, N, width]) and
    SwiGLU at the model's FFN width of 14,336 (52hbtv.com H3-Image page,
    section 二, model table; the [a | b] input drawn on the device from a seeded
    generator), and the Cache-DiT residual difference of x
    against f.  Algorithmic bytes: 8 per element (x, f read; h, y written), 6
    per SwiGLU output (a, b read; out written), 4 per compared value."""
    x = q.view(B, N, width)
    f = k.view(B, N, width)
    cond = synth.draw_dit(B, 1, width, seed=rank)
    gate, shift, scale = (cond[n].to(q.device) for n in ("gate", "shift", "scale"))
    h, y = torch.empty_like(x), torch.empty_like(x)
    ffn = FFN_WIDTH
    g = torch.Generator(device=q.device).manual_seed(1000 + rank)
    a_b = torch.randn((B * N, 2 * ffn), generator=g, device=q.device, dtype=torch.float32).to(torch.bfloat16)
    out = torch.empty((B * N, ffn), dtype=torch.bfloat16, device=q.device)

    def t(fn):
        for _ in range(3):
            fn()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            fn()
        e1.record(stream)
        torch.cuda.synchronize()
        return allreduce_max(e0.elapsed_time(e1) / reps, world)

    ms_ad = t(lambda: h3a.residual_adaln(x, f, gate, shift, scale, out=(h, y)))
    ms_sw = t(lambda: h3a.swiglu(a_b, out=out))
    ws = torch.empty(h3a.h3a.RESIDUAL_DIFF_WORKSPACE_BYTES, dtype=torch.uint8, device=q.device)
    rel = (torch.empty(1, dtype=torch.float64, device=q.device), torch.empty(1, dtype=torch.int32, device=q.device))
    ms_rd = t(lambda: h3a.residual_diff(x, f, 0.04, workspace=ws, out=rel))
    del a_b, out, h, y
    torch.cuda.empty_cache()
    rows = B * N
    return {
        "dit_residual_adaln_untimed_step": {"ms": round(ms_ad, 4), "rows": rows, "width": width,
                                            "GB/s": round(8.0 * rows * width / (ms_ad * 1e-3) / 1e9, 1),
                                            "traffic_key": "residual_adaln"},
        "dit_swiglu_untimed_step": {"ms": round(ms_sw, 4), "rows": rows, "ffn_width": ffn,
                                    "GB/s": round(6.0 * rows * ffn / (ms_sw * 1e-3) / 1e9, 1),
                                    "traffic_key": "swiglu"},
        "cache_dit_residual_diff_untimed_step": {"ms": round(ms_rd, 4), "values": rows * width,
                                                 "GB/s": round(4.0 * rows * width / (ms_rd * 1e-3) / 1e9, 1),
                                                 "traffic_key": "residual_diff"},
    }


# ----------------------------------------------------------------- oracle (CPU)

def _oracle_inputs(d, w, sparsity, times=None):
    """The oracle's prologue and router outputs for the whole workload; their
    wall-clock seconds go into `times` (prologue_s, router_s) when given."""
    import oracle

    oracle.build()
    t0 = time.perf_counter()
    if w.head_dim != 96:  # no prologue at this width: attention sees the inputs as drawn
        qb, kb = d["q"], d["k"]
    else:
        qb = oracle.qk_norm_rope_bf16(d["q"], d["gamma_q"].numpy(), w.grid)
        kb = oracle.qk_norm_rope_bf16(d["k"], d["gamma_k"].numpy(), w.grid)
    t1 = time.perf_counter()
    idx, _ = oracle.route(qb, kb, sparsity)
    t2 = time.perf_counter()
    if times is not None:
        times["prologue_s"] = t1 - t0 if w.head_dim == 96 else None
        times["router_s"] = t2 - t1
    return qb, kb, idx


def _oracle_sample(d, w, qb, kb, idx, rows):
    """Dense and sparse oracle attention on `rows`; returns (seconds, algorithmic FLOPs)."""
    import oracle

    N = w.N
    t0 = time.perf_counter()
    oracle.attention_rows(qb, kb, d["v"], rows)
    oracle.attention_rows(qb, kb, d["v"], rows, idx)
    dt = time.perf_counter() - t0
    nblk = (N + 127) // 128
    lens = np.full(nblk, 128.0)
    lens[-1] = N - (nblk - 1) * 128
    bh, n = rows // N, rows % N
    sparse_keys = lens[idx.reshape(-1, nblk, idx.shape[-1])[bh, n // 128]].sum(axis=-1).sum()
    flops = 4.0 * w.head_dim * (len(rows) * N + sparse_keys)
    return dt, flops


def cpu_baseline(d, w, nrows):
    import oracle
    from rope_block_sparse_b200 import synth

    times = {}
    qb, kb, idx = _oracle_inputs(d, w, SPARSITY, times)
    rows = synth.sample_rows(w.B, w.heads, w.N, nrows, seed=4321).numpy()
    dt, flops = _oracle_sample(d, w, qb, kb, idx, rows)
    full = {"router_s": round(times["router_s"], 3)}
    if times["prologue_s"] is not None:
        full["prologue_s"] = round(times["prologue_s"], 3)
        full["prologue_GB/s"] = round(prologue_bytes(w.N, w.heads, w.B) / times["prologue_s"] / 1e9, 3)
    return {"value": round(flops / dt / 1e12, 6), "unit": "TFLOP/s", "cores": oracle.threads(), "kind": "oracle",
            "sample": f"fp64 oracle dense + sparse (0.75) attention for {len(rows)} sampled query rows of "
                      f"{WORKLOAD} (prologue and router outputs computed by the oracle beforehand); "
                      f"{dt:.1f} s",
            "full_size": full | {"note": "the oracle's prologue (Q and K) and router (pooling, scores, top-k) "
                                         "over the whole workload, wall-clock seconds on the same cores"}}


def run_router_only(args, local):
    """Scores + top-k alone (h3a_route_pooled) on seeded random block means of
    the workload's shape -- a small case for profilers: about 42 MB on the
    device at 124,992 tokens instead of the full step's tensors.  Prints one
    JSON line with the mean time of --steps calls after --warmup calls."""
    import rope_block_sparse_b200 as h3a
    from rope_block_sparse_b200 import synth

    w = synth.WORKLOADS[args.workload]
    if w.head_dim != 96:
        raise SystemExit("--kernel-only router takes a head_dim-96 workload (the pooled router's width)")
    dev = torch.device("cuda", local)
    D, nblk = w.head_dim, (w.N + 127) // 128
    # q only supplies the shape: the router reads the block means in the workspace
    q = torch.empty((w.N + w.heads) * D, dtype=torch.bfloat16, device=dev).as_strided(
        (w.B, w.N, w.heads, D), (0, D, D, 1))
    ws = torch.empty(h3a.route_workspace_size(q), dtype=torch.uint8, device=dev)
    g = torch.Generator(device=dev).manual_seed(0)
    ws.view(torch.float32).copy_(0.3 * torch.randn(ws.numel() // 4, generator=g, device=dev))
    sparsity = w.sparsity if w.sparsity else SPARSITY
    blocks = torch.empty((w.B, w.heads, nblk, h3a.route_k(nblk, sparsity)), dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream()
    for _ in range(args.warmup):
        h3a.route_pooled(q, sparsity, ws, out=blocks)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(args.steps):
        h3a.route_pooled(q, sparsity, ws, out=blocks)
    e1.record(stream)
    torch.cuda.synchronize()
    return {"kernel": "score_topk_kernel (h3a_route_pooled)",
            "workload": f"{w.name}: seeded N(0, 0.3^2) block means of {w.B} x {w.heads} heads x {nblk} blocks x {D}, "
                        f"sparsity {sparsity} (k = {blocks.shape[-1]})",
            "ms": round(e0.elapsed_time(e1) / args.steps, 4), "steps": args.steps, "warmup": args.warmup}


def run_reference(args, rank, world):
    """Reference arm: the fp64 oracle on the host cores, each step a bounded sample."""
    if rank != 0:
        return None
    import oracle
    from rope_block_sparse_b200 import synth

    w = synth.WORKLOADS[args.workload]
    d = synth.draw_workload(args.workload, seed=0)
    qb, kb, idx = _oracle_inputs(d, w, SPARSITY)
    rows_per_step = min(args.ref_rows, w.B * w.heads * w.N)
    times, flops = [], []
    for i in range(args.warmup + args.steps):
        rows = synth.sample_rows(w.B, w.heads, w.N, rows_per_step, seed=1000 + i).numpy()
        dt, fl = _oracle_sample(d, w, qb, kb, idx, rows)
        if i >= args.warmup:
            times.append(dt)
            flops.append(fl)
    value = sum(flops) / sum(times) / 1e12
    sample = (f"fp64 oracle dense + sparse ({SPARSITY}) attention for {rows_per_step} sampled query rows per step "
              f"of {w.name}; prologue and router outputs precomputed by the oracle")
    return {
        "impl": "reference",
        "metric": METRIC,
        "value": round(value, 6),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(1e3 * sum(times) / len(times), 3),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic",
        "config": config_of(w, world, idx.shape[-1]),
        "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": oracle.threads(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["native", "reference"], default="native")
    ap.add_argument("--workload", default=WORKLOAD, help="synthetic workload (clip32k: small profiler case)")
    ap.add_argument("--e2e-steps", type=int, default=None,
                    help="steps of the end-to-end pass (default: --steps; 0 skips it)")
    ap.add_argument("--no-cpu-baseline", dest="cpu_baseline", action="store_false")
    ap.add_argument("--cpu-rows", type=int, default=4096, help="query rows of the CPU-baseline sample")
    ap.add_argument("--ref-rows", type=int, default=128, help="query rows per reference-arm step")
    ap.add_argument("--no-video10s", dest="video10s", action="store_false",
                    help="skip the 245,952-token pass reported beside the headline")
    ap.add_argument("--kernel-only", choices=["router"], default=None,
                    help="time one kernel alone on a small case for profilers (one GPU): router = scores + top-k")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.e2e_steps is None:
        args.e2e_steps = args.steps
    return args


def main():
    args = parse_args()
    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        world = int(os.environ.get("WORLD_SIZE", "1"))
        line = run_reference(args, rank, world)
        if line is not None:
            print(json.dumps(line), flush=True)
        return
    if args.kernel_only == "router":
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
        print(json.dumps(run_router_only(args, int(os.environ.get("LOCAL_RANK", "0")))), flush=True)
        return
    rank, world, local = dist_setup(args.gpus)
    try:
        line = run_gpu(args, rank, world, local)
        if line is not None:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist

            dist.destroy_process_group()


if __name__ == "__main__":
    main()
