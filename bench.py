#!/usr/bin/env python
"""Benchmark of the SCOPE per-layer sparse-attention hot path on B200.

One step = one SCOPE layer through the C ABI (scope_forward): query clustering, key
subspace clustering, LUT / Top-p / k_head / top-up selection and the gathered sparse
attention, on the HunyuanVideo-shaped 720p layer (B=1, 24 heads, 33x45x80 = 118800
tokens, d=128 split 16/56/56, bf16, Cq=300, Cm=333, rho=0.9, alpha=0.1, 5 Lloyd
iterations), synthetic inputs from the seeded generator.

Metric: effective TFLOP/s of the layer = 4 * sum_c n_c * r_c * d / layer time (the
attention FLOPs over the selected pairs only), plus the layer time in ms.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl scope|reference]

Multi-GPU (torchrun, one rank per GPU): every rank runs its own layer (weak scaling,
no collective on the data path); the time is the max over ranks.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from free_sparse_attention_b200 import synth  # noqa: E402
from free_sparse_attention_b200.workloads import ALL, HUNYUAN720  # noqa: E402

METRIC = "SCOPE layer effective TFLOP/s (4*sum n_c*r_c*d / layer time) at 118800 tokens"


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": p["hbm_gbs"], "bf16": p["bf16_tflops"],
                "bf16_sustained": p.get("bf16_tflops_sustained", p["bf16_tflops"]),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16": 1590.0, "bf16_sustained": 1400.0, "source": "fallback"}


def per_clock_frac(achieved, clk, pk):
    """Achieved TFLOP/s per SM MHz (median clock sampled during the timed region) against
    the sustained bf16 matmul's TFLOP/s per MHz at the median clock it ran at."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if not clk or not os.path.exists(path):
        return None
    with open(path) as f:
        peak_mhz = json.load(f).get("clocks_under_load", {}).get("sm_mhz_median")
    if not peak_mhz or not clk.get("sm_mhz"):
        return None
    return (achieved / clk["sm_mhz"]) / (pk["bf16_sustained"] / peak_mhz)


def kernels_per_forward(iters: int) -> int:
    # clustering: init + iters x (pack, tensor-core assign, exact assign, hist, scan,
    # scatter, update); selection: check, top-p, k_head, mask; attention: items, zero-fill,
    # attention
    return 1 + 7 * iters + 4 + 3


def workload_desc(w):
    return (f"{w.name}: B={w.B} H={w.H} grid {w.T}x{w.Hg}x{w.Wg} (N={w.N}) d={w.d} "
            f"({w.d_t}/{w.d_h}/{w.d_w}) {w.dtype} Cq={w.Cq} Cm={w.Cm} rho={w.rho} "
            f"alpha={w.alpha} iters={w.iters}")


class ClockSampler:
    """nvidia-smi clock / throttle sampling during the timed region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.path = f"/tmp/scope_clocks_{os.getpid()}.csv"

    def start(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=self.f, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.f.close()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        os.unlink(self.path)
        if not sm:
            return None
        load = [s for s in sm if mx is None or s > 0.3 * mx] or sm
        return {"sm_mhz": statistics.median(load), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def max_over_ranks(value: float, device="cpu") -> float:
    """Maximum of a per-rank time over all ranks (no-op in a single process).  Every rank
    must call it at the same point."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


# ----------------------------------------------------------------------------- CPU oracle
ORACLE_SAMPLE_FRAMES = 4   # both CPU legs (cpu_baseline and --impl reference) use this sample


def oracle_sample(w, T_sample=ORACLE_SAMPLE_FRAMES, khead_off=False):
    """The oracle on a bounded sub-layer: head (0, 0) of the same workload with the
    grid cut to the first T_sample frames (N_s = T_sample*Hg*Wg tokens); every stage
    runs in full on it.  Each stage's cost is EXTRAPOLATED to the whole layer by its
    complexity (clustering and selection linear in N per head, attention by its
    effective FLOPs); the sample's own realised density estimates the layer's."""
    import oracle
    ws = w.with_(T=T_sample, H=1, B=1)
    x = synth.layer_inputs(ws)
    q, k, v = x["q"][0], x["k"][0], x["v"][0]
    t0 = time.perf_counter()
    rq = oracle.kmeans(q, 0, ws.d, ws.Cq, ws.iters, init_idx=x["q_init"][0])
    rk = oracle.cluster_keys(k, (ws.d_t, ws.d_h, ws.d_w), ws.Cm, ws.iters, init_idx3=x["k_init"][0])
    t1 = time.perf_counter()
    sel = oracle.select(rq["centroids"], rq["sizes"], rk["centroids"], rk["codes"],
                        (ws.d_t, ws.d_h, ws.d_w), ws.rho, ws.alpha, khead_off=khead_off)
    t2 = time.perf_counter()
    oracle.attention(q, k, v, rq["assign"], sel["mask"])
    t3 = time.perf_counter()
    nr = float(np.dot(rq["sizes"].astype(np.float64), sel["r"].astype(np.float64)))
    eff = 4.0 * nr * ws.d
    density = nr / (ws.N * ws.N)
    scale = (w.N / ws.N) * w.H * w.B
    desc = (f"EXTRAPOLATED from the oracle on head (0,0) cut to the first {T_sample} frames "
            f"(N_s={ws.N}): clustering {t1 - t0:.2f}s, selection {t2 - t1:.2f}s, attention {t3 - t2:.2f}s "
            f"({eff / (t3 - t2) / 1e9:.2f} GFLOP/s, sample density {density:.4f}); clustering and "
            f"selection scaled by N/N_s x heads, attention by the layer's effective FLOPs")
    return {"clust_s": (t1 - t0) * scale, "sel_s": (t2 - t1) * scale, "attn_rate": eff / (t3 - t2),
            "desc": desc, "threads": oracle.num_threads(), "density": density,
            "sample_s": t3 - t0}


def layer_seconds_from_sample(s, flops):
    return s["clust_s"] + s["sel_s"] + flops / s["attn_rate"]


def sample_layer_flops(w, s):
    """Effective FLOPs of the whole layer estimated by the oracle alone: dense FLOPs times
    the realised density of its own sample (no GPU value enters the CPU legs)."""
    return 4.0 * w.B * w.H * w.N * w.N * w.d * s["density"]


def oracle_baseline(w, khead_off=False):
    """The CPU leg both arms report: the extrapolated oracle layer time and its metric."""
    s = oracle_sample(w, khead_off=khead_off)
    flops = sample_layer_flops(w, s)
    sec = layer_seconds_from_sample(s, flops)
    return {"value": flops / sec / 1e12, "unit": "TFLOP/s", "cores": s["threads"], "kind": "oracle",
            "extrapolated": True, "sample": s["desc"], "layer_s": sec}


def run_reference(args, w):
    world, rank, _ = dist_setup()
    if rank != 0:
        return 0
    for _ in range(args.warmup):
        oracle_sample(w, khead_off=args.khead_off)
    times, desc, threads, flops = [], "", 1, 0.0
    for _ in range(args.steps):
        s = oracle_sample(w, khead_off=args.khead_off)
        flops = sample_layer_flops(w, s)
        times.append(layer_seconds_from_sample(s, flops))
        desc, threads = s["desc"], s["threads"]
    sec = statistics.median(times)
    value = flops / sec / 1e12
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": sec * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded generator G)",
            "config": {"workload": workload_desc(w), "parallelism": "oracle, OpenMP threads"},
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                             "extrapolated": True, "sample": desc},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------- GPU arm
def traffic_from_profile(kernel_file):
    """DRAM bytes per attention launch from the committed ncu summary, if the kernel
    source is unchanged since it was captured (else None)."""
    prof = os.path.join(ROOT, "profiles", "attn_tc_hunyuan720p.json")
    if not os.path.exists(prof):
        return None
    with open(prof) as f:
        p = json.load(f)
    with open(kernel_file, "rb") as f:
        h = hashlib.sha256(f.read()).hexdigest()
    if p.get("kernel_sha256") != h:
        return None
    return p.get("dram_bytes_per_launch")


def ablation_inputs(args, w, x):
    """With --random-partition, the channels of q and k permuted alike (logits unchanged;
    the key subspaces become random channel subsets)."""
    if args.random_partition is not None:
        perm = np.random.default_rng(args.random_partition).permutation(w.d)
        x["q"] = np.ascontiguousarray(x["q"][..., perm])
        x["k"] = np.ascontiguousarray(x["k"][..., perm])
    return x


def ablation_params(args):
    """scope_params switches of the ablations (the method when none is asked for)."""
    from free_sparse_attention_b200 import capi
    return {"khead_mode": capi.SCOPE_KHEAD_OFF if args.khead_off else capi.SCOPE_KHEAD_ONLINE,
            "key_clustering": capi.SCOPE_KEYS_FULL if args.full_keys else capi.SCOPE_KEYS_SUBSPACES}


def ablation_desc(args):
    s = ""
    if args.full_keys:
        s += " ablation: full-d key clustering (one k-means over all d channels)"
    if args.khead_off:
        s += " ablation: online k_head off (r_c = b_c)"
    if args.random_partition is not None:
        s += f" ablation: random channel partition (seed {args.random_partition})"
    return s


def run_scope(args, w):
    import torch
    import torch.distributed as dist
    from free_sparse_attention_b200 import capi

    world, rank, local = dist_setup()
    torch.cuda.set_device(local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    capi.lib()
    p = capi.Params.from_workload(w, **ablation_params(args))
    x = ablation_inputs(args, w, synth.layer_inputs(w))
    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    host = {n: torch.from_numpy(x[n]).reshape(w.B, w.H, w.N, w.d).to(dt).pin_memory() for n in "qkv"}
    host["qi"] = torch.from_numpy(x["q_init"]).reshape(w.B, w.H, w.Cq).pin_memory()
    host["ki"] = torch.from_numpy(x["k_init"]).reshape(w.B, w.H, 3, w.Cm).pin_memory()
    del x
    dev = {n: t.cuda() for n, t in host.items()}
    ws = capi.alloc_workspace(p)
    O = torch.empty_like(dev["q"])
    _, it = capi.forward(p, dev["q"], dev["k"], dev["v"], dev["qi"], dev["ki"], ws=ws, out=O,
                         intermediates=True)
    torch.cuda.synchronize()
    status = capi.get_device_status(ws)
    n_c = it["q_sizes"].double()
    r_c = it["final_counts"].double()
    flops = float(4.0 * (n_c * r_c).sum().item() * w.d)
    density = float((n_c * r_c).sum().item() / (w.B * w.H * w.N * w.N))
    kh = it["k_head"].double()
    khead_stats = {"min": int(kh.min().item()), "mean": float(kh.mean().item()), "max": int(kh.max().item()),
                   "clusters_topped_up": int((it["final_counts"] > it["base_counts"]).sum().item()),
                   "clusters": int(it["final_counts"].numel())}
    # Top-p decisions within 1e-6 of a tie (the band in which the binary64 reference logs a
    # near tie) and within 3e-7 (where the selection's fixed-point masses could reorder the
    # decision), counted by the selection kernel
    near_ties = capi.get_selection_stats(p, ws)
    del it

    def mk_events():
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(5)]
        for e in evs:
            e.record()
        return evs

    for _ in range(args.warmup):
        capi.forward(p, dev["q"], dev["k"], dev["v"], dev["qi"], dev["ki"], ws=ws, out=O)
    stage_evs = [mk_events() for _ in range(args.steps)]
    torch.cuda.synchronize()
    clocks = ClockSampler(local)
    clocks.start()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for s in range(args.steps):
        capi.forward(p, dev["q"], dev["k"], dev["v"], dev["qi"], dev["ki"], ws=ws, out=O,
                     stage_events=stage_evs[s])
    e1.record()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clk = clocks.stop()
    ms_mean = e0.elapsed_time(e1) / args.steps
    # per-step layer times from each step's first stage event to the next step's (the last
    # to the closing event); the step time reported is their median
    starts = [ev[0] for ev in stage_evs] + [e1]
    step_ms = [starts[i].elapsed_time(starts[i + 1]) for i in range(args.steps)]
    st = np.array([[ev[i].elapsed_time(ev[i + 1]) for i in range(4)] for ev in stage_evs])
    stage_ms = np.median(st, axis=0)
    ms = max_over_ranks(statistics.median(step_ms), device="cuda")
    ms_mean = max_over_ranks(ms_mean, device="cuda")
    status |= capi.get_device_status(ws)

    # end to end through the C ABI with host buffers: every step copies its inputs H2D from
    # pinned host memory and reads its output back D2H, all inside the timed region.
    O_dev = O.clone()
    Oh = [torch.empty(O.shape, dtype=O.dtype, pin_memory=True) for _ in range(2)]
    h2d = sum(host[n].numel() * host[n].element_size() for n in host)
    d2h = Oh[0].numel() * Oh[0].element_size()
    comp = torch.cuda.current_stream()

    # serial form: copies, layer and read-back one after another on one stream
    def e2e_serial_step():
        for n in host:
            dev[n].copy_(host[n], non_blocking=True)
        capi.forward(p, dev["q"], dev["k"], dev["v"], dev["qi"], dev["ki"], ws=ws, out=O)
        Oh[0].copy_(O, non_blocking=True)

    for _ in range(max(1, min(args.warmup, 2))):
        e2e_serial_step()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e0.record()
    for _ in range(args.steps):
        e2e_serial_step()
    e1.record()
    torch.cuda.synchronize()
    e2e_serial_ms = max_over_ranks(e0.elapsed_time(e1) / args.steps, device="cuda")

    # pipelined form: two device input/output sets; step i+1's H2D (copy stream s_in) and step
    # i-1's D2H (copy stream s_out) run under step i's layer, events guard every buffer reuse
    dev2 = [dev, {n: torch.empty_like(t) for n, t in dev.items()}]
    O2 = [O, torch.empty_like(O)]
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()

    def e2e_pipelined(n_steps, start_ev):
        in_ready = [torch.cuda.Event() for _ in range(n_steps)]
        done = [torch.cuda.Event() for _ in range(n_steps)]
        read = [torch.cuda.Event() for _ in range(n_steps)]
        s_in.wait_event(start_ev)
        for i in range(n_steps):
            b = i % 2
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(done[i - 2])     # layer i-2 has consumed input set b
                for n in host:
                    dev2[b][n].copy_(host[n], non_blocking=True)
                in_ready[i].record(s_in)
            comp.wait_event(in_ready[i])
            if i >= 2:
                comp.wait_event(read[i - 2])          # output set b has been read back
            capi.forward(p, dev2[b]["q"], dev2[b]["k"], dev2[b]["v"], dev2[b]["qi"], dev2[b]["ki"],
                         ws=ws, out=O2[b], stream=comp)
            done[i].record(comp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(done[i])
                Oh[b].copy_(O2[b], non_blocking=True)
                read[i].record(s_out)
        comp.wait_event(read[n_steps - 1])

    warm = torch.cuda.Event()
    warm.record(comp)
    e2e_pipelined(2, warm)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e0.record(comp)
    e2e_pipelined(args.steps, e0)
    e1.record(comp)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / args.steps, device="cuda")
    # every step computes the same layer: its read-back output equals the device-resident run
    e2e_match = bool(torch.equal(Oh[0], Oh[1]) and torch.equal(Oh[0].cuda(), O_dev))
    del dev2, O2

    # the same layer captured once into a CUDA graph and replayed (device-resident inputs):
    # what the per-launch host overhead of the ~60 launches and memsets of a layer costs
    graph = None
    if world == 1:
        try:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                capi.forward(p, dev["q"], dev["k"], dev["v"], dev["qi"], dev["ki"], ws=ws, out=O)
            for _ in range(args.warmup):
                g.replay()
            torch.cuda.synchronize()
            e0.record()
            for _ in range(args.steps):
                g.replay()
            e1.record()
            torch.cuda.synchronize()
            graph = {"ms_per_step": e0.elapsed_time(e1) / args.steps,
                     "output_matches_device_run": bool(torch.equal(O, O_dev)),
                     "device_status": capi.get_device_status(ws)}
            del g
        except Exception as ex:   # report, do not fail the bench line
            graph = {"error": f"{type(ex).__name__}: {ex}"[:300]}
    del O_dev

    # dense attention on the same shape (library comparator, not part of the path)
    dense_ms = None
    if not args.no_dense:
        import torch.nn.functional as F
        for _ in range(2):
            F.scaled_dot_product_attention(dev["q"], dev["k"], dev["v"])
        torch.cuda.synchronize()
        e0.record()
        for _ in range(3):
            F.scaled_dot_product_attention(dev["q"], dev["k"], dev["v"])
        e1.record()
        torch.cuda.synchronize()
        dense_ms = e0.elapsed_time(e1) / 3

    pk = peaks()
    attn_ms = float(stage_ms[3])
    achieved = flops / (attn_ms * 1e-3) / 1e12
    traffic = traffic_from_profile(os.path.join(ROOT, "free_sparse_attention_b200", "csrc",
                                                "attention_tc.cu"))
    clust_bytes = w.iters * 2 * w.B * w.H * w.N * w.d * 2
    clust_flops = 2.0 * w.iters * w.B * w.H * w.N * (w.Cq * w.d + w.Cm * w.d)
    nw = (w.N + 31) // 32
    sel_bytes = w.B * w.H * (6 * w.N + w.Cq * nw * 4)
    value = world * flops / (ms * 1e-3) / 1e12
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded generator G: smooth field + noise, 3D RoPE)",
        "config": {"workload": workload_desc(w) + ablation_desc(args),
                   "global_batch": world * w.B, "seq_len": w.N,
                   "parallelism": f"{world} independent layers, one per GPU (no collective)",
                   "l2": "inputs larger than L2 (Q, K, V = 2.19 GB resident in HBM)"},
        "roofline": {"bound": "tensor", "kernel": "attn_tc_kernel (tcgen05 sparse attention)",
                     "achieved": achieved, "peak": pk["bf16"], "unit": "TFLOP/s",
                     "frac": achieved / pk["bf16"], "traffic": traffic,
                     "peak_source": f"{pk['source']} bf16 burst",
                     "frac_of_sustained": achieved / pk["bf16_sustained"],
                     "frac_per_clock": per_clock_frac(achieved, clk, pk)},
        "stages_ms": {"clustering": float(stage_ms[0]), "selection": float(stage_ms[1]),
                      "worklist": float(stage_ms[2]), "attention": attn_ms},
        "stage_fractions": {
            "clustering_hbm": clust_bytes / (stage_ms[0] * 1e-3) / 1e9 / pk["hbm_gbs"],
            # distance contractions 2 N C d_m per iteration (the tensor cores issue twice that
            # for the bf16 hi/lo centroid split), against the measured bf16 peak
            "clustering_tensor": clust_flops / (stage_ms[0] * 1e-3) / 1e12 / pk["bf16_sustained"],
            "selection_hbm": sel_bytes / (stage_ms[1] * 1e-3) / 1e9 / pk["hbm_gbs"]},
        "density": density, "effective_tflop_per_layer": flops / 1e12,
        "ms_per_step_mean": ms_mean, "k_head": khead_stats, "near_ties": near_ties,
        "dense_sdpa_ms": dense_ms,
        "e2e": {"value": world * flops / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s", "ms_per_step": e2e_ms,
                "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
                "pipelining": "two device buffer sets; step i+1's H2D and step i-1's D2H on their own "
                              "copy streams under step i's layer",
                "output_matches_device_run": e2e_match,
                "serial": {"value": world * flops / (e2e_serial_ms * 1e-3) / 1e12, "ms_per_step": e2e_serial_ms}},
        "graph": graph,
        "gpu_launches": kernels_per_forward(w.iters) * args.steps,
        "device_status": status,
        "clocks": clk,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline and not args.full_keys:
        line["cpu_baseline"] = oracle_baseline(w, khead_off=args.khead_off)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


def profile_once(w):
    """One warm-up layer and one layer, nothing else (the command ncu captures)."""
    import torch
    from free_sparse_attention_b200 import capi
    p = capi.Params.from_workload(w)
    x = synth.layer_inputs(w)
    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    Q, K, V = (torch.from_numpy(x[n]).reshape(w.B, w.H, w.N, w.d).to("cuda", dt) for n in "qkv")
    qi = torch.from_numpy(x["q_init"]).reshape(w.B, w.H, w.Cq).cuda()
    ki = torch.from_numpy(x["k_init"]).reshape(w.B, w.H, 3, w.Cm).cuda()
    ws = capi.alloc_workspace(p)
    for _ in range(2):
        O = capi.forward(p, Q, K, V, qi, ki, ws=ws)
    torch.cuda.synchronize()
    st = capi.get_device_status(ws)
    print(json.dumps({"workload": workload_desc(w), "device_status": st,
                      "out_finite": bool(torch.isfinite(O.float()).all().item())}))
    return 0 if st == 0 else 1


def run_warm_start(args, w):
    """Warm-started clustering across denoising steps (review page, pith_inferences: the
    clusters of consecutive steps are close): step A is the layer as usual; step B, the
    next denoising step (the same inputs plus seeded noise of 5 % of their RMS), clusters
    with A's centroids as the initial centroids and `args.warm_start` Lloyd iterations,
    then selects and attends through the stage entry points.  Times B (CUDA events, inputs
    resident) against the cold layer on B's inputs and reports the attention output's
    relative RMS difference between the two."""
    import torch
    from free_sparse_attention_b200 import capi

    capi.lib()
    p = capi.Params.from_workload(w)
    pw = capi.Params.from_workload(w, iters=args.warm_start)
    x = synth.layer_inputs(w)
    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    rng = np.random.default_rng(4321)

    def dev(a):
        return torch.from_numpy(np.ascontiguousarray(a, np.float32)).reshape(w.B, w.H, w.N, w.d).to("cuda", dt)

    A = {n: dev(x[n]) for n in "qkv"}
    B = {}
    for n in "qkv":
        a = x[n]
        B[n] = dev(a + 0.05 * float(np.sqrt(np.mean(a.astype(np.float64) ** 2))) * rng.standard_normal(a.shape))
    qi = torch.from_numpy(x["q_init"]).reshape(w.B, w.H, w.Cq).cuda()
    ki = torch.from_numpy(x["k_init"]).reshape(w.B, w.H, 3, w.Cm).cuda()
    del x
    ws = capi.alloc_workspace(p)
    _, itA = capi.forward(p, A["q"], A["k"], A["v"], qi, ki, ws=ws, intermediates=True)
    qc0, kc0 = itA["q_centroids"].clone(), itA["k_centroids"].clone()
    del itA
    O_cold, itB = capi.forward(p, B["q"], B["k"], B["v"], qi, ki, ws=ws, intermediates=True)
    Ow = torch.empty_like(O_cold)

    def warm_step():
        qc, qa, qs = capi.cluster_queries(pw, B["q"], init_cent=qc0, ws=ws)
        kc, kk = capi.cluster_keys(pw, B["k"], init_cent=kc0, ws=ws)
        sel = capi.build_lut_and_select(p, qc, qs, kc, kk, ws=ws)
        capi.sparse_attention(p, B["q"], B["k"], B["v"], qa, sel["sel_mask"], sel["final_counts"], ws=ws, out=Ow)
        return qs, sel["final_counts"]

    def cold_step():
        capi.forward(p, B["q"], B["k"], B["v"], qi, ki, ws=ws, out=O_cold)

    def timed(fn):
        for _ in range(args.warmup):
            fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(args.steps):
            fn()
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / args.steps

    warm_ms = timed(warm_step)
    cold_ms = timed(cold_step)
    qs, fc = warm_step()
    torch.cuda.synchronize()
    flops = float(4.0 * (qs.double() * fc.double()).sum().item() * w.d)
    diff = (Ow.float() - O_cold.float())
    rel = float(torch.sqrt((diff ** 2).mean() / (O_cold.float() ** 2).mean()).item())
    status = capi.get_device_status(ws)
    print(json.dumps({
        "metric": METRIC + ", warm-started clustering", "value": flops / (warm_ms * 1e-3) / 1e12,
        "unit": "TFLOP/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": warm_ms, "higher_is_better": True, "dtype": w.dtype,
        "config": {"workload": workload_desc(w), "warm_start_iters": args.warm_start,
                   "next_step_inputs": "same layer + seeded N(0, (0.05 rms)^2) noise"},
        "cold_ms_same_inputs": cold_ms, "speedup": cold_ms / warm_ms,
        "attention_rel_rms_vs_cold": rel, "device_status": status}))
    return 0


def run_fidelity(args, w):
    """Proxy-ranking fidelity (review page, falsifier / skeptic's concrete test) of the layer
    the bench times: `args.fidelity` seeded queries per head, the fraction of each query's
    true top 10 % keys (exact logits) kept by its cluster's selection and by the proxy
    ranking's own top 10 %, and Spearman's rho of the proxy with the exact logits for the
    first 4 of them per head."""
    import torch
    from free_sparse_attention_b200 import capi

    capi.lib()
    p = capi.Params.from_workload(w, **ablation_params(args))
    x = ablation_inputs(args, w, synth.layer_inputs(w))
    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    Q, K, V = (torch.from_numpy(x[n]).reshape(w.B, w.H, w.N, w.d).to("cuda", dt) for n in "qkv")
    qi = torch.from_numpy(x["q_init"]).reshape(w.B, w.H, w.Cq).cuda()
    ki = torch.from_numpy(x["k_init"]).reshape(w.B, w.H, 3, w.Cm).cuda()
    del x
    ws = capi.alloc_workspace(p)
    _, it = capi.forward(p, Q, K, V, qi, ki, ws=ws, intermediates=True)
    rng = np.random.default_rng(77)
    samples = np.concatenate([bh * w.N + np.sort(rng.choice(w.N, args.fidelity, replace=False))
                              for bh in range(w.B * w.H)]).astype(np.int64)
    smp = torch.from_numpy(samples).cuda()
    frac = 0.1
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record()
    rs, rp = capi.selection_recall(p, Q, K, it["q_assign"], it["q_centroids"], it["k_centroids"],
                                   it["k_codes"], it["sel_mask"], smp, frac)
    e1.record()
    torch.cuda.synchronize()
    recall_ms = e0.elapsed_time(e1)
    rs, rp = rs.cpu().numpy(), rp.cpu().numpy()
    # Spearman's rho of the proxy with the exact logits, the first 4 sampled queries per head
    sub = torch.from_numpy(samples.reshape(w.B * w.H, -1)[:, :4].reshape(-1).copy()).cuda()
    e0.record()
    rho = capi.rank_correlation(p, Q, K, it["q_assign"], it["q_centroids"], it["k_centroids"], it["k_codes"], sub)
    e1.record()
    torch.cuda.synchronize()
    rank_ms = e0.elapsed_time(e1)
    rho = rho.cpu().numpy()
    n_c = it["q_sizes"].double()
    density = float((n_c * it["final_counts"].double()).sum().item() / (w.B * w.H * w.N * w.N))
    print(json.dumps({
        "metric": "recall of each sampled query's true top 10 % keys (exact logits)",
        "workload": workload_desc(w) + ablation_desc(args),
        "samples": int(samples.size), "density": density,
        "recall_selection": {"mean": float(rs.mean()), "min": float(rs.min()), "p10": float(np.percentile(rs, 10))},
        "recall_proxy_top10": {"mean": float(rp.mean()), "min": float(rp.min()), "p10": float(np.percentile(rp, 10))},
        "spearman_proxy_vs_logits": {"samples": int(rho.size), "mean": float(rho.mean()), "min": float(rho.min()),
                                     "max": float(rho.max()), "kernel_ms": rank_ms},
        "kernel_ms": recall_ms, "device_status": capi.get_device_status(ws)}))
    return 0


def dense_prefix_schedule(name, n_steps=50):
    """(dense_layers, dense_steps) of the dense-prefix schedule the pages print (review page,
    major_comments: "§4, Implementation details"): the first attention layer dense at every
    denoising step, and every layer dense for the first 10 % of the steps on HunyuanVideo and
    20 % on Wan2.1 / Wan2.2 (the other shapes take the Wan share)."""
    frac = 0.10 if "hunyuan" in name else 0.20
    return 1, round(frac * n_steps)


def run_schedule(args, w):
    """The step before the path and the dense-prefix schedule (review page, major_comments:
    "§4, Implementation details"), on pre-RoPE inputs resident in HBM:
      rope      scope_rope3d of Q and K (HBM-bound: 2 reads + 2 writes of B*H*N*d elements);
      dense     scope_dense_attention, the schedule's dense branch (4 N^2 d flops per head),
                beside torch's scaled_dot_product_attention on the same tensors (library);
      sparse    scope_attention_layer on a sparse (layer, step): RoPE + the SCOPE layer;
      dense_l   scope_attention_layer on a dense (layer, step): RoPE + dense attention.
    The schedule-weighted mean is the time of a layer >= 1 averaged over `n_steps` steps
    of which the first `dense_steps` are dense."""
    import torch
    from free_sparse_attention_b200 import capi

    capi.lib()
    p = capi.Params.from_workload(w)
    x = synth.layer_inputs(w, rope=False)
    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    Q, K, V = (torch.from_numpy(x[n]).reshape(w.B, w.H, w.N, w.d).to("cuda", dt) for n in "qkv")
    qi = torch.from_numpy(x["q_init"]).reshape(w.B, w.H, w.Cq).cuda()
    ki = torch.from_numpy(x["k_init"]).reshape(w.B, w.H, 3, w.Cm).cuda()
    del x
    ws = capi.alloc_workspace(p)
    Qr, Kr, O = torch.empty_like(Q), torch.empty_like(K), torch.empty_like(Q)
    n_steps = 50
    dense_layers, dense_steps = dense_prefix_schedule(w.name, n_steps)
    sparse_s = capi.Schedule(layer=dense_layers, step=dense_steps, dense_layers=dense_layers,
                             dense_steps=dense_steps, rope=1, rope_base=10000.0)
    dense_s = capi.Schedule(layer=0, step=dense_steps, dense_layers=dense_layers,
                            dense_steps=dense_steps, rope=1, rope_base=10000.0)

    def timed(fn, reps):
        for _ in range(args.warmup):
            fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            fn()
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / reps

    rope_ms = timed(lambda: capi.rope3d(p, Q, K, out_q=Qr, out_k=Kr), max(args.steps, 20))
    capi.rope3d(p, Q, K, out_q=Qr, out_k=Kr)
    dense_ms = timed(lambda: capi.dense_attention(p, Qr, Kr, V, ws=ws, out=O), args.steps)
    sdpa_ms = timed(lambda: torch.nn.functional.scaled_dot_product_attention(Qr, Kr, V), args.steps)
    sparse_ms = timed(lambda: capi.attention_layer(p, sparse_s, Q, K, V, qi, ki, ws=ws, out=O, out_q=Qr,
                                                   out_k=Kr), args.steps)
    dense_layer_ms = timed(lambda: capi.attention_layer(p, dense_s, Q, K, V, qi, ki, ws=ws, out=O, out_q=Qr,
                                                        out_k=Kr), args.steps)
    status = capi.get_device_status(ws)
    pk = peaks()
    elt = 2 if w.dtype == "bf16" else 4
    rope_bytes = 4 * w.B * w.H * w.N * w.d * elt
    rope_gbs = rope_bytes / (rope_ms * 1e-3) / 1e9
    dense_flops = 4.0 * w.B * w.H * w.N * w.N * w.d
    mean_ms = (dense_steps * dense_layer_ms + (n_steps - dense_steps) * sparse_ms) / n_steps
    print(json.dumps({
        "metric": "SCOPE layer under the dense-prefix schedule (ms, pre-RoPE inputs)",
        "value": mean_ms, "unit": "ms", "higher_is_better": False, "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "dtype": w.dtype,
        "config": {"workload": workload_desc(w), "n_steps": n_steps, "dense_steps": dense_steps,
                   "dense_layers": dense_layers, "rope_base": 10000.0,
                   "l2": "inputs larger than L2 (Q, K, V resident in HBM)"},
        "rope": {"ms": rope_ms, "bytes": rope_bytes, "achieved_gbs": rope_gbs, "peak_gbs": pk["hbm_gbs"],
                 "frac": rope_gbs / pk["hbm_gbs"], "kernel": "rope3d_kernel (Q and K in one launch)"},
        "dense_attention": {"ms": dense_ms, "tflops": dense_flops / (dense_ms * 1e-3) / 1e12,
                            "frac": dense_flops / (dense_ms * 1e-3) / 1e12 / pk["bf16_sustained"],
                            "torch_sdpa_ms": sdpa_ms},
        "layer_sparse_ms": sparse_ms, "layer_dense_ms": dense_layer_ms,
        "device_status": status}))
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["scope", "reference"], default="scope")
    ap.add_argument("--workload", default=HUNYUAN720.name, choices=sorted(ALL))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-dense", action="store_true")
    ap.add_argument("--heads", type=int, default=0,
                    help="override the head count (small cases for profiling)")
    ap.add_argument("--profile-once", action="store_true",
                    help="run the layer once (after one warm-up) and exit; for ncu captures")
    ap.add_argument("--rho", type=float, default=None,
                    help="override the workload's Top-p threshold (rho sweeps)")
    ap.add_argument("--khead-off", action="store_true",
                    help="ablation: the online k_head disabled (r_c = b_c)")
    ap.add_argument("--random-partition", type=int, default=None, metavar="SEED",
                    help="ablation: permute the channels of Q and K alike (seeded), so the key "
                         "subspaces are random channel subsets")
    ap.add_argument("--fidelity", type=int, default=0, metavar="S",
                    help="proxy-ranking fidelity of S sampled queries per head (no timing run)")
    ap.add_argument("--warm-start", type=int, default=0, metavar="ITERS",
                    help="time a next-step layer whose clustering starts from the previous "
                         "step's centroids with ITERS Lloyd iterations")
    ap.add_argument("--full-keys", action="store_true",
                    help="ablation: one k-means of the keys over all d channels (cluster-level proxy)")
    ap.add_argument("--cm", type=int, default=0,
                    help="override the key centroid count Cm (e.g. 3 Cm with --full-keys)")
    ap.add_argument("--schedule", action="store_true",
                    help="pre-RoPE inputs: time 3D RoPE, the dense branch and the layer wrapper "
                         "under the dense-prefix schedule (no main timing run)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    w = ALL[args.workload]
    if args.heads:
        w = w.with_(H=args.heads)
    if args.rho is not None:
        w = w.with_(rho=args.rho)
    if args.cm:
        w = w.with_(Cm=args.cm)
    if args.profile_once:
        return profile_once(w)
    if args.warm_start:
        return run_warm_start(args, w)
    if args.fidelity:
        return run_fidelity(args, w)
    if args.schedule:
        return run_schedule(args, w)
    if args.impl == "reference":
        return run_reference(args, w)
    return run_scope(args, w)


if __name__ == "__main__":
    sys.exit(main())
