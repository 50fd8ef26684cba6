#!/usr/bin/env python
"""Benchmark of the SharQ hot path on B200.

One step (default) = the three linears of a Qwen2.5-7B-shaped decoder
layer (qkv 3584 -> 4608, gate+up 3584 -> 37888, down 18944 -> 3584) at
prefill M = 4096 tokens, each run as the fused prepare (RMSNorm on qkv and
gate+up + 2:4 mask + NVFP4 backbone + NVFP4 residual with its own tensor
scale) followed by the two-path tcgen05 FP4 linear.  Weights are quantised
once, outside the timed region.  Inputs are seeded synthetic tensors
(Student-t(3) activations with a LogNormal(0, 0.5) per-token scale,
N(0, 0.02) weights).  ``--workload`` selects the other shapes (Llama-3.1-8B
linears at M in {1, 16, 128, 2048}, the Qwen3-30B-A3B expert layer, the
format/mask sweep at M = 16384, a LayerNorm DiT block).

Metric: effective TFLOP/s = sum over linears of 2*M*N*K / step time; the
JSON line also carries tokens/s, the roofline of the dominant kernel (the
FP4 linear) and of the prepare kernel, the CPU oracle baseline, the SM
clocks seen during the timed region and an end-to-end figure with host
buffers.  ``--impl reference`` times the CPU oracle instead.

``--fuse-mlp`` runs the MLP producer-fused: the gate+up linear writes
H = silu(gate) * up and max |H| in its epilogue, and the down projection
prepares that H from the producer's amax instead of a synthetic input.

Multi-GPU: the path has no exchange step at this scale; each rank runs an
independent replica (weak scaling) and the slowest rank's time counts.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

from activation_sparsity_prep_b200 import workloads as wl  # noqa: E402

METRIC = "SharQ linear eff. TFLOPS & tokens/s, % of FP4 roofline; prep kernel HBM GB/s"
L2_FLUSH_BYTES = 512 << 20          # > 126 MB L2
# (fmt, zero-filled backbone): read X 2 + backbone codes + scales + residual
# codes + scales; the compressed pair backbone stores K/4 code bytes and K/16
# metadata bytes per row instead of K/2 codes
PREP_BYTES_PER_ELEM = {(0, 1): 3.125, (1, 1): 3.0625, (1, 0): 2.875}


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["sharq", "reference"], default="sharq")
    ap.add_argument("--workload", default="qwen7b")
    ap.add_argument("--M", type=int, default=None,
                    help="rows per linear (default: 2048 for llama8b, the workload's own M otherwise)")
    ap.add_argument("--fmt", default="nvfp4")
    ap.add_argument("--nm", default="2:4",
                    help="n:m of the backbone mask; 4:8p = the pair-granular 4:8 backbone, stored "
                         "compressed for the sparse tensor-core MMA (MXFP4, RMSNorm workloads)")
    ap.add_argument("--residual", choices=["own", "shared"], default="own",
                    help="tensor scale of the NVFP4 residual: its own (default) or the backbone's")
    ap.add_argument("--fuse-mlp", action="store_true",
                    help="SwiGLU MLP with the producer-fused prepare: gate+up writes silu(gate)*up "
                         "and its amax, down prepares that H without its own amax pass")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    return ap.parse_args()


def rank_info():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), "measured"
    except Exception:
        return 6650.0, 1590.0, "fallback"


# --------------------------------------------------------- multi-rank ----

def max_over_ranks(value: float, device=None) -> float:
    """The slowest rank's figure (every rank returns it); identity on one
    rank.  The tensor lives on `device` (cuda for NCCL, cpu for gloo)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(work_per_step: float, world: int, steps: int, total_ms: float) -> float:
    """Weak scaling: every rank does `work_per_step` per step, the job takes
    the slowest rank's time."""
    return work_per_step * world * steps / (total_ms * 1e-3)


# ------------------------------------------------------------- clocks ----

class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons while running."""
    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None
        self.path = None
        self.window = None       # (start, end) of the timed region, host epoch seconds

    def mark(self, t0: float, t1: float):
        self.window = (t0, t1)

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "10"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        if not self.path or not os.path.exists(self.path):
            return None
        rows = []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 10:
                continue
            try:
                ts = parts[0]
                t = time.mktime(time.strptime(ts.split(".")[0], "%Y/%m/%d %H:%M:%S"))
                t += float("0." + ts.split(".")[1]) if "." in ts else 0.0
                rows.append((t, float(parts[2]), float(parts[3]),
                             {n for n, v in zip(names, parts[6:10]) if v.lower() == "active"}))
            except (ValueError, IndexError):
                continue
        os.unlink(self.path)
        if not rows:
            return None
        inside = rows
        where = "all samples (none fell inside the timed region)"
        if self.window:
            w = [r for r in rows if self.window[0] - 0.005 <= r[0] <= self.window[1] + 0.005]
            if w:
                inside, where = w, "samples inside the timed region"
        sm = [r[1] for r in inside]
        reasons = set().union(*[r[3] for r in inside])
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(r[2] for r in rows),
                "reasons": sorted(reasons), "samples": len(inside), "window": where,
                "interval_ms": 10}


# ------------------------------------------------------------- inputs ----

def make_inputs(W: wl.Workload, M: int):
    out = []
    for L in W.linears:
        d = wl.linear_inputs(W, L, M)
        out.append((L, d))
    return out


def flops_of(linears, M):
    return sum(2.0 * M * L.N * L.K for L, _ in linears)


def source_sha(*names):
    h = hashlib.sha256()
    for n in names:
        with open(os.path.join(ROOT, "activation_sparsity_prep_b200", "csrc", n), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic(launch_key: str, sha: str):
    """DRAM bytes (read + write) of this exact launch from the committed ncu
    summary, or None when the kernel source changed since the capture."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            t = json.load(f)[launch_key]
    except Exception:
        return None
    if t.get("source_sha") != sha:
        return None
    return t["dram_bytes"]


# ------------------------------------------------------------ CPU arm ----

def oracle_sample_step(linears, rows: int, quantized, fmt="nvfp4", n=2, m=4, residual="own",
                       fuse_mlp=False, pairs=False):
    """One bounded oracle step: prepare and linear of the first `rows` rows
    of every linear.  fuse_mlp: the down projection's input is the SwiGLU of
    the gate+up output (rounded to bf16) instead of its synthetic tensor.
    pairs: the pair-granular 4:8 prepare (its compressed form is only a
    storage layout; the linear reads the same operands).
    Returns (seconds, effective flops of the sample)."""
    import oracle
    t0 = time.perf_counter()
    fl = 0.0
    H = None
    for (L, d), Wq in zip(linears, quantized):
        X = d["X"][:rows] if not (fuse_mlp and L.name == "down") else H
        if pairs:
            P = oracle.prepare_pairs(X, d["gamma"], wl.EPS)[0]
        else:
            P = oracle.prepare(X, d["gamma"], wl.EPS, n, m, fmt, residual_scale=residual,
                               norm=d["norm"], beta=d["beta"])
        if fuse_mlp and L.name == "gate_up":
            H = oracle.bf16_rne_from_f64(oracle.swiglu_linear(P, Wq))
        else:
            oracle.linear(P, Wq)
        fl += 2.0 * rows * L.N * L.K
    return time.perf_counter() - t0, fl


def mlp_fusable(W) -> bool:
    names = [L.name for L in W.linears]
    return "gate_up" in names and "down" in names


def gate_up_interleaved(W_bits):
    """The synthetic gate+up weight [2I, K] read as gate rows then up rows,
    in the fused linear's interleaved layout."""
    import oracle
    I = W_bits.shape[0] // 2
    return oracle.interleave_gate_up(W_bits[:I], W_bits[I:])


def oracle_moe_sample_step(W, sample, fmt="nvfp4", n=2, m=4, residual="own", fuse_mlp=False):
    """Bounded oracle step of the grouped layer: every sampled dispatched row
    through its own expert's two-path linear.  fuse_mlp: gate+up gives the
    SwiGLU of each sampled (token, expert) row, which (rounded to bf16) is the
    down projection's input for the same rows."""
    import oracle
    t0 = time.perf_counter()
    fl = 0.0
    H = None
    for li, (L, X, g, rows, experts, wq) in enumerate(sample):
        P = oracle.prepare(X if X is not None else H, g, wl.EPS, n, m, fmt, residual_scale=residual)
        Hs = np.zeros((len(rows), L.N // 2)) if fuse_mlp and li == 0 else None
        for e in sorted(set(experts.tolist())):
            sel = np.nonzero(experts == e)[0].astype(np.int32)
            if Hs is not None:
                Hs[sel] = oracle.swiglu_linear(oracle.gather_rows(P, rows[sel]), wq[e])
            else:
                oracle.linear(oracle.gather_rows(P, rows[sel]), wq[e])
            fl += 2.0 * len(sel) * L.N * L.K
        if Hs is not None:
            H = oracle.bf16_rne_from_f64(Hs)
    return time.perf_counter() - t0, fl


def moe_reference_sample(W, fmt, tokens: int = 4, fuse_mlp=False):
    """Sampled operands of the grouped layer: the first `tokens` tokens for
    gate+up (each with its top-k experts) and the first tokens*top-k
    dispatched rows for down, with only the experts they reach quantised.
    fuse_mlp: down takes the same (token, expert) rows, its input the
    gate+up SwiGLU (X None), and gate+up weights in the interleaved layout."""
    import oracle
    T, E, topk = W.moe["T"], W.moe["E"], W.moe["topk"]
    ex = wl.routing(W.cfg, T, E, topk)
    ri, off = wl.group_by_expert(ex.astype(np.int32), E)
    sample = []
    for li, L in enumerate(W.linears):
        if li == 0:
            X = wl.activation(W.dist, W.cfg, L.index, tokens, L.K)
            rows = np.repeat(np.arange(tokens, dtype=np.int32), topk)
            experts = ex[:tokens].reshape(-1)
        elif fuse_mlp:
            X = None
            rows = np.arange(tokens * topk, dtype=np.int32)
            experts = ex[:tokens].reshape(-1)
        else:
            nrow = tokens * topk
            X = wl.activation(W.dist, W.cfg, L.index, T * topk, L.K)[:nrow]
            rows = np.arange(nrow, dtype=np.int32)
            experts = (np.searchsorted(off, rows, side="right") - 1).astype(np.int64)
        g = wl.gamma_ones(L.K) if L.norm else None

        def wbits(e, li=li, L=L):
            Wb = wl.weight(W.cfg * 1000 + li, 100 + int(e), L.N, L.K)
            return gate_up_interleaved(Wb) if fuse_mlp and li == 0 else Wb

        wq = {int(e): oracle.quantize_weight(wbits(e), fmt) for e in set(experts.tolist())}
        sample.append((L, X, g, rows, experts, wq))
    return sample


def host_cores():
    """CPU cores this process may run on (its affinity set)."""
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def blas_threads():
    try:
        import threadpoolctl
        info = threadpoolctl.threadpool_info()
        return max([i.get("num_threads", 1) for i in info if i.get("user_api") == "blas"] or [1])
    except Exception:
        return 1


def cpu_baseline(linears, args, budget_s: float = 10.0, rows: int = 16):
    """The oracle timed on the host over a bounded sample (the first `rows`
    rows of every linear): once with the BLAS pool at its default size and
    once with one thread, about `budget_s` seconds each."""
    import oracle
    n_, m_ = nm_of(args)
    quantized = [oracle.quantize_weight(gate_up_interleaved(d["W"]) if args.fuse_mlp and L.name == "gate_up"
                                        else d["W"], args.fmt) for L, d in linears]

    def timed():
        total_t, total_f, n = 0.0, 0.0, 0
        while total_t < budget_s and n < 50:
            t, f = oracle_sample_step(linears, rows, quantized, args.fmt, n_, m_, args.residual,
                                      args.fuse_mlp, pairs_of(args))
            total_t += t
            total_f += f
            n += 1
        return total_f / total_t / 1e12, n

    threads = blas_threads()
    value, n = timed()
    one = None
    try:
        import threadpoolctl
        with threadpoolctl.threadpool_limits(limits=1, user_api="blas"):
            one, _ = timed()
    except Exception:
        pass
    return {"value": value, "unit": "TFLOP/s", "cores": host_cores(), "kind": "oracle",
            "threads": {"gemm_blas": threads, "prepare": 1},
            "single_thread_value": one,
            "sample": f"{n} passes of: oracle prepare + fp64 two-path linear on the first {rows} "
                      f"rows of each of the {len(linears)} linears (all N"
                      f"{'; SwiGLU of gate+up feeds down' if args.fuse_mlp else ''}"
                      f"{'; pair-granular 4:8 prepare' if pairs_of(args) else ''}); prepare "
                      f"single-threaded C, GEMM numpy/OpenBLAS fp64 on {threads} threads "
                      f"(single_thread_value: the same sample with one BLAS thread)"}


def workload_desc(W, M):
    """The workload description both arms put in config["workload"]."""
    if W.moe is None:
        return (f"{W.name}: " + ", ".join(f"{L.name} {L.K}x{L.N}" for L in W.linears)
                + f"; M={M}, prepare+linear each")
    T, E, topk = W.moe["T"], W.moe["E"], W.moe["topk"]
    return (f"{W.name}: Qwen3-30B-A3B-shaped expert layer, {T} tokens, {E} experts, top-{topk}; "
            f"gate_up {W.linears[0].K}x{W.linears[0].N} (rows gathered by index), "
            f"down {W.linears[1].K}x{W.linears[1].N} (rows in dispatch order); grouped prepare+linear")


def bench_config(args, W, M):
    return {"workload": workload_desc(W, M), "M": M, "fmt": args.fmt, "nm": args.nm,
            "backbone": ("pair-granular 4:8, compressed [M, K/4] + pair metadata, sparse tensor-core MMA"
                         if pairs_of(args) else "element n:m, zero-filled [M, K/2], dense MMA"),
            "residual_scale": args.residual,
            "mlp": ("producer-fused: gate_up writes H = silu(gate)*up and max|H| (SwiGLU epilogue), "
                    "down prepares that H from the producer's amax" if args.fuse_mlp else
                    "separate: every linear reads its own synthetic input"),
            "l2": "flushed between timed steps (512 MiB write)",
            "timing": "CUDA graph per step, per-kernel external events"}


def run_reference(args):
    rank, world, _ = rank_info()
    if rank != 0:
        return 0
    W = wl.WORKLOADS[args.workload]
    n, m = nm_of(args)
    cores = host_cores()
    threads = blas_threads()
    if W.moe is None:
        linears = make_inputs(W, args.M)
        import oracle
        quantized = [oracle.quantize_weight(gate_up_interleaved(d["W"]) if args.fuse_mlp and L.name == "gate_up"
                                            else d["W"], args.fmt) for L, d in linears]
        rows = 16
        step = lambda: oracle_sample_step(linears, rows, quantized, args.fmt, n, m, args.residual,
                                          args.fuse_mlp, pairs_of(args))
        what = (f"first {rows} rows of each linear per step (all N), of M={args.M}"
                + ("; the SwiGLU of gate+up (bf16) feeds down" if args.fuse_mlp else "")
                + ("; pair-granular 4:8 prepare" if pairs_of(args) else ""))
        M = args.M
    else:
        sample = moe_reference_sample(W, args.fmt, fuse_mlp=args.fuse_mlp)
        step = lambda: oracle_moe_sample_step(W, sample, args.fmt, n, m, args.residual, args.fuse_mlp)
        what = ("4 tokens through gate+up (each with its top-8 experts) and "
                + ("the SwiGLU of those 32 (token, expert) rows through down" if args.fuse_mlp else
                   "the first 32 dispatched rows through down") + ", per step")
        M = W.moe["T"]
    for _ in range(args.warmup):
        step()
    times, fl = [], 0.0
    for _ in range(args.steps):
        t, f = step()
        times.append(t)
        fl = f
    tot = sum(times)
    value = fl * args.steps / tot / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": tot / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64 GEMM over FP4-decoded operands; f32 prepare",
        "data": "synthetic",
        "config": bench_config(args, W, M),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                         "threads": {"gemm_blas": threads, "prepare": 1},
                         "sample": what + f"; prepare single-threaded C, GEMM numpy/OpenBLAS fp64 "
                                          f"on {threads} threads"},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------ GPU arm ----

def nm_of(args):
    n, m = (int(v) for v in args.nm.rstrip("p").split(":"))
    return n, m


def pairs_of(args) -> bool:
    """--nm 4:8p: the pair-granular backbone on the sparse MMA."""
    return args.nm.endswith("p")


def traffic_tag(args) -> str:
    """Part of a profiles/traffic.json key that names the kernel form."""
    return (("_pairs" if pairs_of(args) else "") + ("_shared" if args.residual == "shared" else "")
            + ("_fused" if args.fuse_mlp else ""))


def build_units(args, dev):
    """Device buffers and closures for one step of the chosen workload.
    A unit is one prepare followed by one (plain or grouped) linear."""
    import torch

    import activation_sparsity_prep_b200 as sq

    W = wl.WORKLOADS[args.workload]
    fmt = sq._FMT[args.fmt]
    n, m = nm_of(args)
    pairs = pairs_of(args)
    bf = torch.bfloat16
    up = lambda a: torch.from_numpy(a).view(bf).to(dev)
    units = []
    if W.moe is None:
        M = args.M
        fused = None          # (H, amax) of the SwiGLU gate+up, when the MLP is fused
        for L in W.linears:
            d = wl.linear_inputs(W, L, M)
            g = None if d["gamma"] is None else up(d["gamma"])
            b = None if d["beta"] is None else up(d["beta"])
            swiglu = args.fuse_mlp and L.name == "gate_up"
            Wt = up(d["W"])
            if swiglu:
                Wt = sq.interleave_gate_up(Wt[:L.N // 2], Wt[L.N // 2:])
            w = sq.quantize_weight(Wt, fmt)
            del Wt
            P = sq.Prepared.empty(M, L.K, n, m, fmt, device=dev, residual_scale=args.residual,
                                  pairs=pairs)
            ws = torch.empty(max(256, sq.prepare_workspace_bytes(M, L.K, fmt)), dtype=torch.uint8, device=dev)
            if swiglu:
                Y = torch.empty((M, L.N // 2), dtype=bf, device=dev)
                amax = torch.empty((1,), dtype=torch.float32, device=dev)
                fused = (Y, amax)
            else:
                Y = torch.empty((M, L.N), dtype=bf, device=dev)
            if args.fuse_mlp and L.name == "down":
                X, amax = fused
                u = dict(name=L.name, rows=M, prep_rows=M, N=L.N, K=L.K, X=X, Y=Y, host_input=False)
                u["prep"] = (lambda X=X, amax=amax, P=P, ws=ws:
                             sq.prepare_amax(X, amax, n, m, fmt, out=P, ws=ws))
                u["gemm"] = (lambda P=P, w=w, Y=Y: sq.linear(P, w, out=Y))
                units.append(u)
                continue
            X = up(d["X"])
            u = dict(name=L.name, rows=M, prep_rows=M, N=L.N, K=L.K, X=X, Y=Y, swiglu=swiglu)
            if swiglu:
                u["gemm"] = (lambda P=P, w=w, Y=Y, amax=amax: sq.linear_swiglu(P, w, out=Y, amax=amax))
            if L.layernorm:
                u["prep"] = (lambda X=X, g=g, b=b, P=P, ws=ws:
                             sq.prepare_layernorm(X, g, b, wl.EPS, n, m, fmt, out=P, ws=ws))
            else:
                u["prep"] = (lambda X=X, g=g, P=P, ws=ws: sq.prepare(X, g, wl.EPS, n, m, fmt, out=P, ws=ws))
            if "gemm" not in u:
                u["gemm"] = (lambda P=P, w=w, Y=Y: sq.linear(P, w, out=Y))
            units.append(u)
        return units, M
    T, E, topk = W.moe["T"], W.moe["E"], W.moe["topk"]
    ri, off = wl.group_by_expert(wl.routing(W.cfg, T, E, topk), E)
    ri_d = torch.from_numpy(ri).to(dev)
    off_d = torch.from_numpy(off).to(dev)
    fused = None
    for li, L in enumerate(W.linears):
        rows_in = T if li == 0 else T * topk             # gate_up reads tokens, down dispatched rows
        swiglu = args.fuse_mlp and li == 0
        g = up(wl.gamma_ones(L.K)) if L.norm else None
        w = sq.Weight.empty(L.N, L.K, fmt, device=dev, E=E)
        sb = sq.scale_bytes(L.N, L.K, fmt)
        for e in range(E):
            we = sq.Weight(w.codes[e], w.scales[e * sb:(e + 1) * sb], w.tensor_scale[e:e + 1],
                           L.N, L.K, w.fmt)
            Wt = up(wl.weight(W.cfg * 1000 + li, 100 + e, L.N, L.K))
            if swiglu:
                Wt = sq.interleave_gate_up(Wt[:L.N // 2], Wt[L.N // 2:])
            sq.quantize_weight(Wt, fmt, out=we)
        P = sq.Prepared.empty(rows_in, L.K, n, m, fmt, device=dev, residual_scale=args.residual)
        ws = torch.empty(max(256, sq.prepare_workspace_bytes(rows_in, L.K, fmt)), dtype=torch.uint8, device=dev)
        mws = torch.empty(sq.moe_workspace_bytes(T * topk, E, L.K, fmt), dtype=torch.uint8, device=dev)
        Y = torch.empty((T * topk, L.N // 2 if swiglu else L.N), dtype=bf, device=dev)
        rix = ri_d if li == 0 else None
        if args.fuse_mlp and li == 1:
            X, amax = fused
            u = dict(name=L.name, rows=T * topk, prep_rows=rows_in, N=L.N, K=L.K, X=X, Y=Y,
                     host_input=False)
            u["prep"] = (lambda X=X, amax=amax, P=P, ws=ws: sq.prepare_amax(X, amax, n, m, fmt, out=P, ws=ws))
        else:
            X = up(wl.activation(W.dist, W.cfg, L.index, rows_in, L.K))
            u = dict(name=L.name, rows=T * topk, prep_rows=rows_in, N=L.N, K=L.K, X=X, Y=Y, swiglu=swiglu)
            u["prep"] = (lambda X=X, g=g, P=P, ws=ws: sq.prepare(X, g, wl.EPS, n, m, fmt, out=P, ws=ws))
        if swiglu:
            amax = torch.empty((1,), dtype=torch.float32, device=dev)
            fused = (Y, amax)
            u["gemm"] = (lambda P=P, w=w, Y=Y, rix=rix, mws=mws, amax=amax:
                         sq.moe_linear_swiglu(P, rix, off_d, w, out=Y, amax=amax, ws=mws, T=T * topk))
        else:
            u["gemm"] = (lambda P=P, w=w, Y=Y, rix=rix, mws=mws:
                         sq.moe_linear(P, rix, off_d, w, out=Y, ws=mws, T=T * topk))
        units.append(u)
    return units, T


def run_sharq(args):
    import torch
    import torch.distributed as dist

    import activation_sparsity_prep_b200 as sq

    rank, world, local = rank_info()
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    dev = torch.device("cuda", local)
    fmt = sq._FMT[args.fmt]
    n, m = nm_of(args)
    units, tokens_per_step = build_units(args, dev)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)

    def step():
        for u in units:
            u["prep"]()
            u["gemm"]()

    # eager warm-up (lazy init), then capture one step with per-kernel events
    step()
    torch.cuda.synchronize()
    assert sq.last_device_status() == 0
    evs = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(2 * len(units) + 1)]
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            evs[0].record()
            for i, u in enumerate(units):
                u["prep"]()
                evs[2 * i + 1].record()
                u["gemm"]()
                evs[2 * i + 2].record()
    torch.cuda.synchronize()

    for _ in range(args.warmup):
        flush.zero_()
        g.replay()
    torch.cuda.synchronize()

    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    step_ms, prep_ms, lin_ms = [], [[] for _ in units], [[] for _ in units]
    with ClockSampler(local) as clk:
        t_start = time.time()
        for _ in range(args.steps):
            flush.zero_()                    # L2 flushed between timed steps
            g.replay()
            torch.cuda.synchronize()
            step_ms.append(evs[0].elapsed_time(evs[-1]))
            for i in range(len(units)):
                prep_ms[i].append(evs[2 * i].elapsed_time(evs[2 * i + 1]))
                lin_ms[i].append(evs[2 * i + 1].elapsed_time(evs[2 * i + 2]))
        clk.mark(t_start, time.time())
    torch.cuda.synchronize()
    status = sq.last_device_status()
    total_ms = max_over_ranks(sum(step_ms), dev)
    if world > 1:
        dist.barrier()
    clocks = clk.summary()

    fl_step = sum(2.0 * u["rows"] * u["N"] * u["K"] for u in units)
    ms_step = total_ms / args.steps
    value = whole_job_rate(fl_step, world, args.steps, total_ms) / 1e12
    tokens = whole_job_rate(tokens_per_step, world, args.steps, total_ms)

    hbm, bf16, src = peaks()
    fp4_peak = 4.0 * bf16           # dense FP4 = 4x dense bf16 (nominal 9 vs 2.25 PFLOP/s)
    lin_t = [statistics.mean(x) * 1e-3 for x in lin_ms]
    prep_t = [statistics.mean(x) * 1e-3 for x in prep_ms]
    # Dominant kernel: the largest linear launch.  Algorithmic dense-equivalent
    # flops of the two-path linear: 2MNK on the dense residual plus 2MNK*(n/m)
    # on the n:m-sparse backbone at twice the dense rate.
    alg_factor = 2.0 * (1.0 + 0.5 * n / m)
    dom = max(range(len(units)), key=lambda i: lin_t[i])
    ud = units[dom]
    # roofline time = max(flops / FP4 peak, algorithmic bytes / HBM): weight codes
    # + scales once, activation codes + scales of both paths, bf16 output
    sfb = 1.0 / (16 if fmt == 0 else 32)
    pairs = pairs_of(args)
    bb_bytes = (0.25 + 1.0 / 16 + sfb) if pairs else (0.5 + sfb)     # compressed codes + metadata
    lin_bytes = (ud["N"] * ud["K"] * (0.5 + sfb) + ud["rows"] * ud["K"] * (bb_bytes + 0.5 + sfb)
                 + 2.0 * ud["Y"].numel())
    lin_flops = alg_factor * ud["rows"] * ud["N"] * ud["K"]
    hbm_bound = lin_bytes / (hbm * 1e9) > lin_flops / (fp4_peak * 1e12)
    if hbm_bound:
        achieved, lin_peak, lin_unit = lin_bytes / lin_t[dom] / 1e9, hbm, "GB/s"
    else:
        achieved, lin_peak, lin_unit = lin_flops / lin_t[dom] / 1e12, fp4_peak, "TFLOP/s"
    # the key names the kernel form: the pair backbone and the shared residual
    # scale run other instances (and the shared scale the 256-wide tile)
    tag = traffic_tag(args)
    lin_key = (f"linear_{args.fmt}{tag}_{args.workload}_{ud['name']}{'_swiglu' if ud.get('swiglu') else ''}"
               f"_M{args.M}")
    traffic = profiled_traffic(lin_key, source_sha("linear.cu", "common.cuh"))
    # Prepare roofline on its largest launch (algorithmic bytes per element:
    # read X 2, backbone codes 0.5 (zero-filled) + scales, residual codes 0.5 + scales)
    bpe = PREP_BYTES_PER_ELEM[(fmt, 0 if pairs else 1)]
    pdom = max(range(len(units)), key=lambda i: prep_t[i])
    up_ = units[pdom]
    prep_ach = bpe * up_["prep_rows"] * up_["K"] / prep_t[pdom] / 1e9
    prep_key = f"prepare_{args.fmt}{tag}_{args.workload}_{up_['name']}_M{args.M}"
    prep_traffic = profiled_traffic(prep_key, source_sha("prepare.cu", "common.cuh"))

    # end-to-end: host inputs (pinned) in, host outputs out, every step
    e2e = None
    if not args.no_e2e:
        fed = [u for u in units if u.get("host_input", True)]      # inputs that come from the host
        hx = [u["X"].cpu().pin_memory() for u in fed]
        hy = [torch.empty(u["Y"].shape, dtype=u["Y"].dtype, pin_memory=True) for u in units]
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ts = []
        cur = torch.cuda.current_stream()
        for it in range(args.warmup + args.steps):
            flush.zero_()
            e0.record(cur)
            for u, h in zip(fed, hx):
                u["X"].copy_(h, non_blocking=True)
            g.replay()
            for u, h in zip(units, hy):
                h.copy_(u["Y"], non_blocking=True)
            e1.record(cur)
            torch.cuda.synchronize()
            if it >= args.warmup:
                ts.append(e0.elapsed_time(e1))
        tot = max_over_ranks(sum(ts), dev)
        e2e = {"value": whole_job_rate(fl_step, world, args.steps, tot) / 1e12, "unit": "TFLOP/s",
               "h2d_bytes_per_step": int(sum(h.numel() * h.element_size() for h in hx)),
               "d2h_bytes_per_step": int(sum(h.numel() * h.element_size() for h in hy)),
               "ms_per_step": tot / args.steps}

    base = None
    if (rank == 0 and world == 1 and not args.no_cpu_baseline
            and wl.WORKLOADS[args.workload].moe is None):
        linears = make_inputs(wl.WORKLOADS[args.workload], args.M)
        base = cpu_baseline(linears, args)

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "nvfp4" if fmt == 0 else "mxfp4", "data": "synthetic",
            "config": bench_config(args, wl.WORKLOADS[args.workload], tokens_per_step),
            "tokens_per_s": tokens,
            "roofline": {"bound": "hbm" if hbm_bound else "tensor", "achieved": achieved,
                         "peak": lin_peak, "unit": lin_unit, "frac": achieved / lin_peak,
                         "traffic": traffic, "algorithmic_bytes": lin_bytes,
                         "algorithmic_flops": lin_flops,
                         "kernel": f"{'moe_' if wl.WORKLOADS[args.workload].moe else ''}linear_kernel "
                                   f"(two-path FP4 GEMM{', SwiGLU epilogue' if ud.get('swiglu') else ''}), "
                                   f"{ud['name']} launch rows={ud['rows']} N={ud['N']} K={ud['K']}",
                         "peak_note": (f"{src} copy bandwidth" if hbm_bound else
                                       f"dense FP4 = 4 x {src} bf16 burst ({bf16:.0f} TFLOP/s)"),
                         "achieved_note": f"{alg_factor:g}*M*N*K per launch ({n}:{m} backbone at 2x "
                                          f"rate + dense residual)"
                                          + ("; backbone on tcgen05.mma.sp" if pairs else
                                             "; backbone zero-filled on the dense MMA")},
            "prepare_roofline": {"bound": "hbm", "achieved": prep_ach, "peak": hbm, "unit": "GB/s",
                                 "frac": prep_ach / hbm, "traffic": prep_traffic,
                                 "kernel": f"prepare_kernel, {up_['name']} launch rows={up_['prep_rows']} "
                                           f"K={up_['K']}",
                                 "bytes_per_elem": bpe, "peak_note": f"{src} copy bandwidth"},
            "kernel_ms": {u["name"]: {"prepare": statistics.mean(p), "linear": statistics.mean(l)}
                          for u, p, l in zip(units, prep_ms, lin_ms)},
            # dense-rate equivalent of what the tensor cores execute: both paths as
            # dense MMAs (zero-filled backbone), or the residual dense plus the
            # compressed backbone on the sparse MMA at twice the rate
            "executed_fp4_tflops": sum((3.0 if pairs else 4.0) * u["rows"] * u["N"] * u["K"]
                                       for u in units) / sum(lin_t) / 1e12,
            "prepare_gbs_all": sum(bpe * u["prep_rows"] * u["K"] for u in units) / sum(prep_t) / 1e9,
            "gpu_launches": (2 * len(units) + (len(units) if wl.WORKLOADS[args.workload].moe else 0))
                            * args.steps,
            "device_status": status,
            "clocks": clocks,
            "e2e": e2e,
            "cpu_baseline": base,
        }
        print(json.dumps(line), flush=True)
    del g
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main():
    args = parse_args()
    if args.M is None:
        Ms = wl.WORKLOADS[args.workload].Ms
        args.M = 2048 if args.workload == "llama8b" else (Ms[0] if Ms else 0)
    if args.fuse_mlp and not mlp_fusable(wl.WORKLOADS[args.workload]):
        raise SystemExit("--fuse-mlp needs a workload with gate_up and down linears")
    if pairs_of(args):
        W = wl.WORKLOADS[args.workload]
        if (args.nm != "4:8p" or args.fmt != "mxfp4" or args.fuse_mlp or W.moe is not None
                or any(L.layernorm for L in W.linears)):
            raise SystemExit("--nm 4:8p: MXFP4, RMSNorm (or no norm) plain linears, no --fuse-mlp")
    if args.impl == "reference":
        return run_reference(args)
    return run_sharq(args)


if __name__ == "__main__":
    sys.exit(main())
