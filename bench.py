"""Benchmark of one decoupled sparse attention step on B200: Reassign Cache + fused attention.

    python bench.py [--gpus N --steps K --warmup W] [--workload wan14b] [--impl reference]

A step is one pass of the whole hot path over one batch of synthetic input: da_reassign
(reassign every key to its cached centroid, refresh the per-(block, cluster) statistics and
the per-head totals) followed by da_attention, timed as its two public halves (the per-q-block
compensation values, then the fused kernel: exact attention on the fixed blocks and the cluster
columns in one online softmax).  The metric is effective TFLOP/s, where effective
FLOPs = sum over heads and q-blocks of 4 * |q-block| * (kept keys + C) * d; the reassignment
is inside the timed step but its FLOPs are not counted.

Under torchrun every rank runs its own copy of the workload with its own seed (heads are
independent: weak scaling, no collective on the data path); the step time is the maximum
over ranks of CUDA-event time.  Rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

import workloads as W

ROOT = os.path.dirname(os.path.abspath(__file__))
METRIC = "effective TFLOP/s & ms/call of reassign+fused sparse attn; % of bf16 TC peak"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
ATT_SRC = os.path.join(ROOT, "block_sparse_cluster_b200", "csrc", "attention_tc.cu")
ATT_PROFILE = os.path.join(ROOT, "profiles", "attention_tc_kernel_wan14b.md")


def source_code_sha1(path: str) -> str:
    """sha1 of a CUDA source with its comments and blank space removed: an edit of the comments
    alone leaves it unchanged, any change of the code changes it."""
    import hashlib
    import re
    text = open(path, encoding="utf-8").read()
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    text = re.sub(r"\s+", " ", text).strip()
    return hashlib.sha1(text.encode()).hexdigest()


def attention_traffic(w) -> "float | None":
    """DRAM bytes (read + write) per launch of attention_tc_kernel from the committed ncu summary,
    whose record line names the workload and the code hash (comments aside) of the kernel source
    it was captured from: null for another workload or once the code has changed since the
    capture."""
    import re
    try:
        text = open(ATT_PROFILE).read()
        sha = source_code_sha1(ATT_SRC)
    except OSError:
        return None
    m = re.search(r"traffic record: workload=(\w+) heads=(\d+) bytes_per_launch=([0-9.e+]+) "
                  r"attention_tc\.cu code-sha1=([0-9a-f]{40})", text)
    if not m or m.group(1) != w.name or int(m.group(2)) != w.H or m.group(4) != sha:
        return None
    return float(m.group(3))


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while the timed region runs."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.proc = None
        self.dev = device_index

    def __enter__(self):
        try:
            uuid = str(torch.cuda.get_device_properties(self.dev).uuid)
            sel = ["-i", uuid if uuid.startswith("GPU-") else "GPU-" + uuid]
        except Exception:
            sel = []
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                                          "-lms", "200", *sel], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                                         text=True)
        except Exception:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()
                out = ""
            self.lines = [l for l in out.splitlines() if l.strip()]

    def summary(self):
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for l in self.lines:
            f = [x.strip() for x in l.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


def _dist():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    if ws > 1 and not torch.distributed.is_initialized():
        import datetime
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        torch.distributed.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def head_slice(H: int, rank: int, world: int) -> range:
    """The heads rank `rank` of `world` takes when the ranks split one workload's heads: contiguous
    slices, the first H % world ranks one head more."""
    base, extra = divmod(H, world)
    lo = rank * base + min(rank, extra)
    return range(lo, lo + base + (1 if rank < extra else 0))


def _sum_over_ranks(x: float, ws: int, device) -> float:
    if ws == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.SUM)
    return float(t.item())


def _max_over_ranks(x: float, ws: int, device) -> float:
    if ws == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def _barrier(ws: int):
    if ws > 1:
        torch.distributed.barrier()


# ---------------------------------------------------------------------------
# the fp64 oracle timed on host cores (cpu_baseline and the reference arm)

def oracle_item_sampler(w: W.Workload, seed: int):
    """Per work item (head h, q-block i): the oracle's reassignment of key block i of that head and
    its decoupled attention for q-block i.  The complement statistics need an assignment of every
    key of the head; the generator's own cluster labels stand in for it (the timing does not depend
    on which valid assignment is used)."""
    import oracle
    b, h = 0, 0
    q, k, v, mu = W.head_qkv(w, seed, b, h)
    plan = W.head_plan(w, seed, b, h)
    labels = W.head_labels(w, seed, b, h).numpy()
    Qf, Kf, Vf, Cf = (x.float().numpy().astype(np.float64) for x in (q, k, v, mu))
    blk_len = [min(w.block, w.N - i * w.block) for i in range(w.nB)]
    rng = np.random.default_rng(seed)

    def run(n_items: int):
        flops = 0.0
        t0 = time.perf_counter()
        for _ in range(n_items):
            i = int(rng.integers(0, w.nB))
            s0, s1 = i * w.block, min(w.N, (i + 1) * w.block)
            oracle.reassign(Kf[s0:s1], Cf)
            oracle.attention_qblock(Qf, Kf, Vf, Cf, plan[i], labels, i, w.block)
            kept = sum(blk_len[j] for j in plan[i])
            flops += 4.0 * blk_len[i] * (kept + w.C) * w.d
        return flops, time.perf_counter() - t0

    return run


def _single_thread():
    """Run the oracle on one host core (BLAS pools limited to one thread), so `cores` is exact."""
    from threadpoolctl import threadpool_limits
    return threadpool_limits(limits=1)


def cpu_baseline(w: W.Workload, seed: int, budget_s: float = 12.0):
    run = oracle_item_sampler(w, seed)
    flops, t, items = 0.0, 0.0, 0
    with _single_thread():
        run(1)  # warm caches
        while t < budget_s and items < 400:
            f, dt = run(4)
            flops += f
            t += dt
            items += 4
    return {"value": flops / t / 1e12, "unit": "TFLOP/s", "cores": 1, "kind": "oracle",
            "sample": f"{items} work items of head 0 (reassign of one key block + decoupled attention of one "
                      f"q-block each, random q-blocks), fp64 numpy, {t:.1f} s"}


def run_reference(args, w: W.Workload, ws: int, rank: int):
    if rank != 0:
        return
    run = oracle_item_sampler(w, args.seed)
    per_step = max(1, args.ref_items)
    flops, t = 0.0, 0.0
    with _single_thread():
        for _ in range(args.warmup):
            run(per_step)
        for _ in range(args.steps):
            f, dt = run(per_step)
            flops += f
            t += dt
    value = flops / t / 1e12
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": ws,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * t / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": _config(w, args),
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": 1, "kind": "oracle",
                             "sample": f"{per_step} random work items of head 0 per step (reassign of one key "
                                       f"block + decoupled attention of one q-block each), fp64 numpy"},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def _config(w: W.Workload, args):
    return {"workload": f"{w.name}: B={w.B} H={w.H} N={w.N} ({w.T}x{w.Hs}x{w.Ws} latent) d={w.d} block={w.block} "
                        f"C={w.C} density={w.density}",
            "B": w.B, "H": w.H, "N": w.N, "d": w.d, "block": w.block, "C": w.C, "density": w.density,
            "seed": args.seed,
            "parallelism": ("heads split over the ranks (strong)" if getattr(args, "split_heads", False)
                            else "independent heads per rank (weak)"),
            "l2": _l2_note(w)}


def _l2_note(w: W.Workload) -> str:
    qkv = 3 * w.B * w.H * w.N * w.d * (2 if w.dtype == "bf16" else 4)
    if qkv > 126e6:
        return f"inputs (Q, K, V: {qkv / 1e9:.2f} GB) exceed the 126 MB L2; no flush between steps"
    return f"inputs (Q, K, V: {qkv / 1e6:.1f} MB) fit in the 126 MB L2; steady state, no flush between steps"


# ---------------------------------------------------------------------------
# Reassign-cache loop: the plan is prepared once and the keys drift from step to step; each step
# reassigns them to the cached centroids.  Reported per step: the device time of reassign +
# attention, and the error against dense attention with the cached centroids and with fresh ones
# (20 GPU Lloyd iterations on that step's keys, untimed), with both k-means objectives.

def run_loop(args):
    import block_sparse_cluster_b200 as da
    import torch.nn.functional as F

    w = W.WORKLOADS["loop"]
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    dims = da.Dims(w.B, w.H, w.N, w.d, w.C, w.block, w.torch_dtype)
    eng = da.DecoupledAttention(dims, dev)
    fresh = da.DecoupledAttention(dims, dev)
    rows = []
    for step in range(w.steps):
        inp = W.make_inputs(w, seed=args.seed, step=step)
        Q, K, V, cent = (x.to(dev) for x in (inp.Q, inp.K, inp.V, inp.centroids))
        if step == 0:
            eng.prepare(inp.kv_idx.to(dev), inp.kv_cnt.to(dev))     # the plan is fixed across steps
            fresh.mask = eng.mask
        O = torch.empty_like(Q)
        for _ in range(max(3, args.warmup)):
            eng.step(Q, K, V, cent, O)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        eng.step(Q, K, V, cent, O)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        ms = e0.elapsed_time(e1)
        a_cached = eng.stats.assign.long()
        # fresh clusters for comparison: Lloyd from the cached centroids on this step's keys
        cent_f = cent.clone()
        da.kmeans(dims, K, cent_f, 20, fresh.stats, fresh.ws)
        O_f = torch.empty_like(Q)
        fresh.step(Q, K, V, cent_f, O_f)
        from torch.nn.attention import SDPBackend, sdpa_kernel
        with sdpa_kernel(SDPBackend.EFFICIENT_ATTENTION):           # fp32, no score matrix in memory
            dense = F.scaled_dot_product_attention(Q.float(), K.float(), V.float())
        nrm = dense.norm()

        def obj(c, a):
            return float(((K.float() - torch.gather(c.float(), 2, a[..., None].expand(-1, -1, -1, w.d))) ** 2).sum())

        rows.append({"step": step, "ms": ms, "err_cached": float((O.float() - dense).norm() / nrm),
                     "err_fresh": float((O_f.float() - dense).norm() / nrm),
                     "sse_cached": obj(cent, a_cached), "sse_fresh": obj(cent_f, fresh.stats.assign.long())})
    if eng.status() != 0 or fresh.status() != 0:
        raise RuntimeError("device status after the loop")
    print(json.dumps({"metric": "reassign-cache loop: ms per step (reassign + attention) and drift error",
                      "workload": f"{w.name}: B={w.B} H={w.H} N={w.N} d={w.d} C={w.C} steps={w.steps} "
                                  f"drift={w.drift} per-head density in {list(w.density_range)}",
                      "data": "synthetic", "steps": rows}), flush=True)


def run_spread(args):
    """The variance-corrected cluster logits (ESTRA abstract's correction, read as a diagonal
    Gaussian about each representative): da_reassign + da_cluster_spread + da_attention_spread,
    which runs on the tensor cores for bf16 with d = block = 128 (the CUDA cores otherwise).  One
    JSON line with the step time and its split."""
    import block_sparse_cluster_b200 as da
    w = W.WORKLOADS[args.workload]
    if args.heads > 0:
        w = W.scaled(w, H=args.heads)
    dev = torch.device("cuda", 0)
    inp = W.make_inputs(w, seed=args.seed)
    dims = da.Dims(w.B, w.H, w.N, w.d, w.C, w.block, w.torch_dtype)
    eff = W.effective_flops(w, inp.kv_cnt, inp.kv_idx)
    eng = da.DecoupledAttention(dims, dev)
    Q, K, V, cent = (x.to(dev) for x in (inp.Q, inp.K, inp.V, inp.centroids))
    eng.prepare(inp.kv_idx.to(dev), inp.kv_cnt.to(dev))
    O = torch.empty_like(Q)
    spread = torch.empty(w.B, w.H, w.C, w.d, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(evs=None):
        if evs is not None:
            evs[0].record(stream)
        da.da_reassign(dims, K, V, cent, eng.stats, eng.ws)
        if evs is not None:
            evs[1].record(stream)
        da.da_cluster_spread(dims, K, cent, eng.stats, spread)
        if evs is not None:
            evs[2].record(stream)
        da.da_attention_spread(dims, Q, K, V, eng.mask, cent, eng.stats, spread, 0.0, O, None, eng.ws)
        if evs is not None:
            evs[3].record(stream)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize(dev)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    for k in range(args.steps):
        step(evs[k])
    torch.cuda.synchronize(dev)
    if eng.status() != 0:
        raise RuntimeError("device status: " + da.da_status_string(eng.status()))
    ms = sum(e[0].elapsed_time(e[3]) for e in evs) / args.steps
    split = {name: sum(e[i].elapsed_time(e[i + 1]) for e in evs) / args.steps
             for i, name in enumerate(("reassign", "cluster_spread", "attention_spread"))}
    print(json.dumps({
        "metric": "effective TFLOP/s & ms/call of reassign + cluster spread + variance-corrected attention",
        "value": eff / (ms * 1e-3) / 1e12, "unit": "TFLOP/s", "ms_per_step": ms, "steps": args.steps,
        "warmup": args.warmup, "higher_is_better": True, "dtype": {"bf16": "bf16", "f32": "f32"}[w.dtype],
        "data": "synthetic", "breakdown_ms": split, "effective_flop_per_step": eff,
        "config": _config(w, args)}))


def run_sip(args):
    """Inclusion-probability reweighting (AB-Attention abstract's estimator): one call of
    da_attention_sip per step on the plan's blocks with seeded inclusion probabilities; the fused
    tensor-core kernel with the weights as bias rows.  Effective FLOPs count the kept keys only."""
    import block_sparse_cluster_b200 as da
    w = W.WORKLOADS[args.workload]
    if args.heads > 0:
        w = W.scaled(w, H=args.heads)
    dev = torch.device("cuda", 0)
    inp = W.make_inputs(w, seed=args.seed)
    dims = da.Dims(w.B, w.H, w.N, w.d, w.C, w.block, w.torch_dtype)
    flops_all = W.effective_flops(w, inp.kv_cnt, inp.kv_idx)
    eff = flops_all - float(w.B * w.H * 4 * w.N * w.C * w.d)       # drop the cluster columns
    incl = W.inclusion_probabilities(w, args.seed, inp.kv_idx.shape[-1]).to(dev)
    ws = da.workspace(dims, dev)
    Q, K, V = (x.to(dev) for x in (inp.Q, inp.K, inp.V))
    sched = torch.empty(w.B * w.H * w.nB, dtype=torch.int32, device=dev)
    mask = da.da_mask_prepare(dims, da.BlockMask(inp.kv_idx.to(dev), inp.kv_cnt.to(dev)), sched, ws)
    O = torch.empty_like(Q)
    for _ in range(max(3, args.warmup)):
        da.da_attention_sip(dims, Q, K, V, mask, incl, 0.0, O, None, ws)
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        da.da_attention_sip(dims, Q, K, V, mask, incl, 0.0, O, None, ws)
    e1.record()
    torch.cuda.synchronize(dev)
    if da.da_device_status(ws) != 0:
        raise RuntimeError("device status after the timed calls")
    ms = e0.elapsed_time(e1) / args.steps
    print(json.dumps({
        "metric": "effective TFLOP/s & ms/call of inclusion-probability reweighted block-sparse attention",
        "value": eff / (ms * 1e-3) / 1e12, "unit": "TFLOP/s", "ms_per_step": ms, "steps": args.steps,
        "warmup": args.warmup, "higher_is_better": True, "dtype": "bf16", "data": "synthetic",
        "pct_of_bf16_peak": 100.0 * eff / (ms * 1e-3) / 1e12 / _peaks()[0]["bf16_tflops"],
        "effective_flop_per_step": eff, "config": _config(w, args)}))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="wan14b", choices=list(W.WORKLOADS))
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--e2e-groups", type=int, default=8, help="head groups pipelined in the end-to-end leg")
    ap.add_argument("--cpu-budget", type=float, default=12.0)
    ap.add_argument("--ref-items", type=int, default=8)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--heads", type=int, default=0, help="override the head count (profiling runs)")
    ap.add_argument("--split-heads", action="store_true",
                    help="under torchrun, the ranks share one workload's heads (strong scaling) instead of each "
                         "running its own copy")
    ap.add_argument("--loop", action="store_true", help="run the reassign-cache loop workload instead")
    ap.add_argument("--spread", action="store_true",
                    help="time the variance-corrected path (reassign + cluster spread + corrected attention)")
    ap.add_argument("--sip", action="store_true",
                    help="time the inclusion-probability reweighted attention (no compensation)")
    args = ap.parse_args()
    if args.loop:
        run_loop(args)
        return
    if args.spread:
        run_spread(args)
        return
    if args.sip:
        run_sip(args)
        return
    ws, rank, local = _dist()
    w = W.WORKLOADS[args.workload]
    if args.heads > 0:
        w = W.scaled(w, H=args.heads)
    if args.impl == "reference":
        run_reference(args, w, ws, rank)
        if ws > 1:
            torch.distributed.destroy_process_group()
        return

    import block_sparse_cluster_b200 as da

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if args.split_heads:
        # the ranks share one workload's heads (strong scaling): same seed, a slice of heads each
        seed = args.seed
        inp = W.make_inputs(w, seed=seed, heads=head_slice(w.H, rank, ws))
    else:
        # every rank its own copy of the workload (weak scaling)
        seed = args.seed + 1000 * rank
        inp = W.make_inputs(w, seed=seed)
    full_w = w
    w = inp.w
    dims = da.Dims(w.B, w.H, w.N, w.d, w.C, w.block, w.torch_dtype)
    eff = W.effective_flops(w, inp.kv_cnt, inp.kv_idx)
    eff_job = _sum_over_ranks(eff, ws, dev)

    stream = torch.cuda.current_stream(dev)
    eng = da.DecoupledAttention(dims, dev)
    Q, K, V, cent = (x.to(dev) for x in (inp.Q, inp.K, inp.V, inp.centroids))
    eng.prepare(inp.kv_idx.to(dev), inp.kv_cnt.to(dev))
    O = torch.empty_like(Q)
    torch.cuda.synchronize(dev)

    def step(evs=None):
        # da_reassign, then da_attention as its two public halves (the per-q-block compensation
        # values, then the fused attention kernel); events between the calls time each
        if evs is not None:
            evs[0].record(stream)
        da.da_reassign(dims, K, V, cent, eng.stats, eng.ws)
        if evs is not None:
            evs[1].record(stream)
        da.da_compensation(dims, eng.mask, eng.stats, eng.ws)
        if evs is not None:
            evs[2].record(stream)
        da.da_attention_prebuilt(dims, Q, K, V, eng.mask, cent, eng.stats, 0.0, O, None, eng.ws)
        if evs is not None:
            evs[3].record(stream)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize(dev)
    if eng.status() != 0:
        raise RuntimeError("device status after warm-up: " + da.da_status_string(eng.status()))

    K_steps = args.steps
    att_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(K_steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    _barrier(ws)
    torch.cuda.synchronize(dev)
    with ClockSampler(local) as clk:
        start.record(stream)
        for k in range(K_steps):
            step(att_ev[k])
        end.record(stream)
        torch.cuda.synchronize(dev)
    _barrier(ws)
    st = eng.status()
    if st != 0:
        raise RuntimeError("device status after timing: " + da.da_status_string(st))
    ms_local = start.elapsed_time(end) / K_steps
    step_ms = sorted(e[0].elapsed_time(e[3]) for e in att_ev)
    median_ms_local = step_ms[len(step_ms) // 2]
    reas_ms_local = sum(e[0].elapsed_time(e[1]) for e in att_ev) / K_steps
    comp_ms_local = sum(e[1].elapsed_time(e[2]) for e in att_ev) / K_steps
    att_ms_local = sum(e[2].elapsed_time(e[3]) for e in att_ev) / K_steps
    ms = _max_over_ranks(ms_local, ws, dev)
    att_ms = _max_over_ranks(att_ms_local, ws, dev)
    comp_ms = _max_over_ranks(comp_ms_local, ws, dev)
    value = eff_job / (ms * 1e-3) / 1e12

    # one cold step: L2 flushed by writing a 256 MB buffer first (the timed steps above run warm)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    flush.fill_(1)
    cold = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
    step(cold)
    torch.cuda.synchronize(dev)
    cold_ms = _max_over_ranks(cold[0].elapsed_time(cold[3]), ws, dev)
    del flush
    median_ms = _max_over_ranks(median_ms_local, ws, dev)

    # End to end through the same public calls: pinned host inputs in, O back to the host.  The
    # heads go in groups on three streams, so that group g+1's inputs cross PCIe while group g
    # computes and group g-1's output returns (each group is a head slice with its own buffers).
    e2e = None
    if not args.no_e2e:
        groups = max(d for d in range(1, min(args.e2e_groups, w.H) + 1) if w.H % d == 0) if w.B == 1 else 1
        hg = w.H // groups
        gdims = da.Dims(w.B, hg, w.N, w.d, w.C, w.block, w.torch_dtype)
        sl = lambda t, g: t[:, g * hg:(g + 1) * hg]
        engs = []
        for g in range(groups):
            e = da.DecoupledAttention(gdims, dev)
            e.prepare(sl(inp.kv_idx, g).contiguous().to(dev), sl(inp.kv_cnt, g).contiguous().to(dev))
            engs.append(e)
        pinned = [x.pin_memory() for x in (inp.Q, inp.K, inp.V, inp.centroids)]
        O_host = torch.empty(O.shape, dtype=O.dtype, pin_memory=True)
        h2d = sum(x.numel() * x.element_size() for x in pinned)
        d2h = O_host.numel() * O_host.element_size()
        s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        ev_in = [torch.cuda.Event() for _ in range(groups)]
        ev_done = [torch.cuda.Event() for _ in range(groups)]
        ev_out = [torch.cuda.Event() for _ in range(groups)]
        dev_bufs = (Q, K, V, cent)

        def e2e_step(first):
            for g in range(groups):
                if not first:
                    s_in.wait_event(ev_done[g])            # the group's inputs are free again
                with torch.cuda.stream(s_in):
                    for dst, src in zip(dev_bufs, pinned):
                        sl(dst, g).copy_(sl(src, g), non_blocking=True)
                ev_in[g].record(s_in)
                stream.wait_event(ev_in[g])
                if not first:
                    stream.wait_event(ev_out[g])            # the group's output has left the GPU
                engs[g].step(sl(Q, g), sl(K, g), sl(V, g), sl(cent, g), sl(O, g), stream=stream)
                ev_done[g].record(stream)
                s_out.wait_event(ev_done[g])
                with torch.cuda.stream(s_out):
                    sl(O_host, g).copy_(sl(O, g), non_blocking=True)
                ev_out[g].record(s_out)

        e2e_step(True)                                  # untimed warm-up of the three streams
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        _barrier(ws)
        torch.cuda.synchronize(dev)
        e0.record(stream)
        s_in.wait_stream(stream)
        for k in range(args.e2e_steps):
            e2e_step(False)
        stream.wait_stream(s_out)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        for e in engs:
            if e.status() != 0:
                raise RuntimeError("device status after the end-to-end steps")
        e2e_ms = _max_over_ranks(e0.elapsed_time(e1) / args.e2e_steps, ws, dev)
        e2e = {"value": eff_job / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s", "ms_per_step": e2e_ms,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "head_groups": groups}

    if rank == 0:
        peaks, kind = _peaks()
        peak = float(peaks["bf16_tflops"])
        att_tflops = eff / (att_ms * 1e-3) / 1e12
        sustained = float(peaks.get("bf16_tflops_sustained", peak))
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": ws, "steps": K_steps,
            "warmup": max(3, args.warmup), "ms_per_step": ms, "higher_is_better": True,
            "scaling": "strong" if args.split_heads else "weak",
            "vs_baseline": None, "dtype": "bf16" if w.dtype == "bf16" else "f32", "data": "synthetic",
            "config": _config(full_w, args),
            "pct_of_bf16_peak": 100.0 * (value / ws) / peak,
            "breakdown_ms": {"reassign": reas_ms_local, "compensation": comp_ms_local, "attention": att_ms_local},
            "ms_per_step_median": median_ms, "cold_ms_per_step": cold_ms,
            "effective_flop_per_step_per_gpu": eff_job / ws,
            # the dominant kernel: attention_tc_kernel alone (exact blocks and cluster columns in one
            # online softmax, on compensation values built by the pre-pass); frac_incl_compensation
            # counts the pre-pass kernel's time too, frac_step the whole step (reassign included)
            "roofline": {"bound": "tensor", "kernel": "attention_tc_kernel",
                         "achieved": att_tflops, "peak": peak, "unit": "TFLOP/s", "frac": att_tflops / peak,
                         "peak_source": f"{kind} bf16 dense (burst)",
                         "frac_of_sustained": att_tflops / sustained,
                         "frac_incl_compensation": eff / ((att_ms + comp_ms) * 1e-3) / 1e12 / peak,
                         "frac_step": (value / ws) / peak,
                         "traffic": attention_traffic(w)},
            "e2e": e2e,
            "gpu_launches": K_steps * LAUNCHES_PER_STEP,
            "clocks": clk.summary(),
        }
        if ws == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(w, args.seed, args.cpu_budget)
        print(json.dumps(line), flush=True)
    if ws > 1:
        _barrier(ws)
        torch.distributed.destroy_process_group()


# kernels of ours per timed step: reassign (centroid norms, assignment with block statistics,
# totals) + attention (compensation chunks, fused attention)
LAUNCHES_PER_STEP = 5

if __name__ == "__main__":
    main()
