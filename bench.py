"""Benchmark of the routed sparse-MoE block on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W]
                    [--workload decode|prefill|stack|mix] [--impl ours|reference]

Default (the configuration the headline metric is quoted on): one routed-MoE
layer, d=2048, 512 experts (SwiGLU ffn 512) + shared expert, top-10, 2-bit
group-32 weights with fp16 scales, Zipf(1.1) popularity, frequency-ordered
slots, verify windows of T = 1, 2, 3 and 4 tokens.  A step is one pass of the
block (router, top-k, expert FFNs, shared expert, combine) over a batch of
2048 rounds of the four windows (8192 windows, 20480 tokens), each window on
the next of 32 independent layer copies (16 GB of weights, far above the
126 MB L2) with fresh tokens.  The step is captured as one CUDA graph and
replayed; the timed region holds exactly K steps, bracketed by a barrier and
device syncs, timed with CUDA events, max over ranks.  The same line carries
the metric's other half, the 8192-token prefill chunk (config of its own,
timed the same way), as a `prefill` object.  One process per GPU; ranks run
independent replicas (no collective on the data path).

Prints one JSON line (rank 0).
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
sys.path.insert(0, ROOT)

METRIC = ("routed-MoE tokens/s (decode 1–4 tok, 8192 prefill); HBM GB/s & TC util vs peak")


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=None)
    p.add_argument("--warmup", type=int, default=None)
    p.add_argument("--workload", default="decode", choices=["decode", "prefill", "stack", "mix"])
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--layers", type=int, default=32, help="independent layer copies rotated")
    p.add_argument("--topk", type=int, default=None,
                   help="decode: experts per token (the pages' 'Faster' mode is top_k - 1)")
    p.add_argument("--prefer-hot", type=int, default=0,
                   help="decode: a selection bonus on each layer's N most popular experts")
    p.add_argument("--prefer-bonus", type=float, default=0.5)
    p.add_argument("--adapt-every", type=int, default=0,
                   help="mix: re-order every layer's slots by its decayed routing counts every N "
                        "decode steps (0: frozen layout)")
    p.add_argument("--adapt-swaps", type=int, default=96)
    p.add_argument("--adapt-decay", type=float, default=0.5)
    p.add_argument("--rounds", type=int, default=2048,
                   help="rounds of the T=1..4 windows in one decode step (smaller for profiling)")
    p.add_argument("--l2-next", action="store_true",
                   help="each decode step prefetches the next layer's router and shared expert "
                        "into L2 (its bytes then count in that step's DRAM traffic)")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-prefill", action="store_true",
                   help="decode workload only (no prefill object in the line)")
    p.add_argument("--prefill-steps", type=int, default=500)
    p.add_argument("--cpu-seconds", type=float, default=12.0)
    return p.parse_args()


# ----------------------------------------------------------------- plumbing
def dist_init():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                    device_id=torch.device("cuda", local))
        else:   # host-only ranks (the oracle arm, tests)
            dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=120))
    return rank, world, local


def _reduce_device():
    import torch.distributed as dist
    return "cuda" if dist.get_backend() == "nccl" else "cpu"


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(v: float, world: int) -> float:
    if world == 1:
        return v
    import torch
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device=_reduce_device())
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(v: float, world: int) -> float:
    if world == 1:
        return v
    import torch
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device=_reduce_device())
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 200 ms."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        self.p = None

    def __enter__(self):
        try:
            self.p = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.Q}",
                                       "--format=csv,noheader,nounits", "-lms", "200",
                                       "-i", str(self.dev)], stdout=self.f,
                                      stderr=subprocess.DEVNULL)
        except OSError:
            self.p = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        if self.p is not None:
            self.p.terminate()
            try:
                self.p.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.p.kill()

    def summary(self):
        self.f.flush()
        rows = []
        with open(self.f.name) as f:
            for line in f:
                parts = [s.strip() for s in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(rows)}


def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d["bf16_tflops_sustained"]), "src": "measured"}
    except (OSError, KeyError, ValueError):
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                "src": "fallback"}


def sources_sha256() -> str:
    """Hash of the kernel sources (csrc + the C header)."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "routed_expert_ffn_06_b200", "csrc")
    for f in sorted(os.listdir(csrc)):
        h.update(f.encode())
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(fh.read())
    with open(os.path.join(ROOT, "include", "moe.h"), "rb") as fh:
        h.update(fh.read())
    return h.hexdigest()


def measured_traffic(name: str):
    """DRAM bytes (read + write) per launch of the named kernel group from an
    ncu capture recorded in profiles/traffic.json; None when the file is missing
    or the kernel sources changed after the counters were taken."""
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            d = json.load(f)[name]
        if d.get("sources_sha256") != sources_sha256():
            return None
        return int(d["dram_bytes_per_launch"])
    except (OSError, KeyError, ValueError, TypeError):
        return None


# ------------------------------------------------------------------ decode
DECODE_WINDOWS = (1, 2, 3, 4)
PREFILL_LAUNCHES = 10       # router GEMM, top-k, prep, hist, scan, scatter, gather, GEMM1,
                            # GEMM2, combine per 8192-token chunk (router split at load)
WORKLOAD_DECODE = ("decode single layer: d=2048, 512 experts ffn=512 + shared ffn=512, top-10, "
                   "2-bit g32 fp16 scales, Zipf(1.1) popularity, frequency-ordered slots; "
                   "verify windows T=1,2,3,4")
WORKLOAD_PREFILL = ("prefill chunk single layer: 8192 tokens, d=2048, 512 experts ffn=512 + "
                    "shared ffn=512, top-10, 2-bit g32, router bias N(0,0.5)")


def expert_bytes(shape) -> int:
    from routed_expert_ffn_06_b200 import synth
    return shape.codes_bytes + shape.n_scales * 2


def oracle_cpu_baseline(layer_cpu, windows, seconds, seed=777):
    """The oracle, as it stands, on this host's cores: whole windows until
    `seconds` of CPU work have run.  Returns (tokens/s, cores, sample)."""
    import oracle
    from routed_expert_ffn_06_b200 import synth
    OL = oracle.OracleLayer(layer_cpu)
    toks, t0, n_win = 0, time.perf_counter(), 0
    while time.perf_counter() - t0 < seconds:
        for T in windows:
            x = synth.make_tokens(T, layer_cpu.shape.d, seed=seed, step=n_win)
            OL.block_forward(x)
            toks += T
            n_win += 1
    dt = time.perf_counter() - t0
    return toks / dt, oracle.num_threads(), f"{n_win} windows ({toks} tokens, T cycling {windows})"


def bench_decode(args, rank, world, local):
    """The headline line: the decode layer (windows of 1..4 tokens) as `value`,
    with the 8192-token prefill chunk of the same metric in a `prefill` object."""
    import numpy as np
    import torch

    from routed_expert_ffn_06_b200 import moe, synth
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    moe.load()
    wl = synth.WORKLOADS["decode"]
    sh = wl["shape"]
    if args.topk:
        import dataclasses
        sh = dataclasses.replace(sh, k=args.topk)
    NL = args.layers
    K = args.steps if args.steps is not None else 20
    W = args.warmup if args.warmup is not None else 5
    R = args.rounds                        # rounds of the four windows per step
    nwin = len(DECODE_WINDOWS)
    ntok_step = R * sum(DECODE_WINDOWS)
    t_gen = time.time()
    layers = [synth.make_layer(sh, seed=rank * 1000 + i, layer=i, device=dev, bias=wl["bias"],
                               slot=wl["slot"]) for i in range(NL)]
    t_gen = time.time() - t_gen
    prefs = [None] * NL
    if args.prefer_hot:   # selection bonus on each layer's hottest experts (rank 1..N)
        prefs = [torch.where(l.rank.to(dev) <= args.prefer_hot, args.prefer_bonus, 0.0).float()
                 for l in layers]
    structs = [moe.make_layer_struct(l, p) for l, p in zip(layers, prefs)]
    if args.l2_next:   # window w runs on copy w % NL: its successor is the next copy
        moe.link_l2_next(structs)
    ws = moe.alloc_workspace(structs[0], max(DECODE_WINDOWS))
    # fresh tokens for every window of a step
    xs = [[synth.make_tokens(T, sh.d, seed=rank * 1000 + 7, step=r * nwin + i, device=dev)
           for i, T in enumerate(DECODE_WINDOWS)] for r in range(R)]
    ys = [torch.empty(T, sh.d, dtype=torch.bfloat16, device=dev) for T in DECODE_WINDOWS]
    stream = torch.cuda.Stream(device=dev)

    def layer_of(r, i):
        return structs[(r * nwin + i) % NL]

    def enqueue_step():
        for r in range(R):
            for i, T in enumerate(DECODE_WINDOWS):
                moe.moe_block_forward(layer_of(r, i), xs[r][i], T, ys[i], 0, ws, stream)

    # eager pass: kernel attributes and tensor maps set up; routing of every
    # window for the byte counts (the block forward records it in the workspace)
    ids_all = [[None] * nwin for _ in range(R)]
    wts_all = [[None] * nwin for _ in range(R)]
    eb = expert_bytes(sh)
    with torch.cuda.stream(stream):
        for r in range(R):
            for i, T in enumerate(DECODE_WINDOWS):
                ids = torch.empty(T, sh.k, dtype=torch.int32, device=dev)
                wts = torch.empty(T, sh.k, dtype=torch.float32, device=dev)
                moe.moe_route_topk(layer_of(r, i), xs[r][i], T, 0, None, ids, wts, ws, stream)
                ids_all[r][i], wts_all[r][i] = ids, wts
        enqueue_step()
    stream.synchronize()
    st, code = moe.moe_workspace_error(ws, stream)
    if st != 0:
        raise RuntimeError(f"device error word {code:#x}")
    uniq = [[int(torch.unique(ids_all[r][i]).numel()) for i in range(nwin)] for r in range(R)]
    U_mean = {str(T): round(float(np.mean([uniq[r][i] for r in range(R)])), 2)
              for i, T in enumerate(DECODE_WINDOWS)}
    # fitted Zipf exponent of the realised selection counts (all windows, all
    # layer copies, experts ranked by their own layer's popularity profile)
    counts = np.zeros(sh.E)
    for r in range(R):
        for i in range(nwin):
            rank_of = layers[(r * nwin + i) % NL].rank.numpy() - 1
            np.add.at(counts, rank_of[ids_all[r][i].cpu().numpy().ravel()], 1)
    top = np.sort(counts)[::-1][:200]
    top = top[top > 0]
    zipf_s = float(-np.polyfit(np.log(np.arange(1, len(top) + 1)), np.log(top), 1)[0])
    # algorithmic bytes of one step: per window the router (E x d fp32), the
    # window's unique experts and the shared expert, the tokens in and out
    step_bytes = sum(sh.E * sh.d * 4 + (uniq[r][i] + 1) * eb + 2 * T * sh.d * 2
                     for r in range(R) for i, T in enumerate(DECODE_WINDOWS))

    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        enqueue_step()
    with torch.cuda.stream(stream):
        for _ in range(W):
            g.replay()
    stream.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        with torch.cuda.stream(stream):
            e0.record(stream)
            for _ in range(K):
                g.replay()
            e1.record(stream)
        stream.synchronize()
    torch.cuda.synchronize()
    barrier(world)
    ms = max_over_ranks(e0.elapsed_time(e1), world)
    clocks = clk.summary()
    value = K * ntok_step * world / (ms / 1e3)
    peaks = measured_peaks()
    layer_gbs = step_bytes / (ms / K / 1e3) / 1e9
    del g

    # the expert step alone (moe_expert_ffn_decode on the eager pass's routing:
    # expert kernel + combine), one graph per window size, events around the
    # replays on the launching stream (events inside a graph would break the
    # programmatic overlap of its kernels)
    per_T, exp_ms_total, exp_bytes, n_exp = {}, 0.0, 0, 0
    Rc = min(R, 256)
    for i, T in enumerate(DECODE_WINDOWS):
        gt = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gt, stream=stream):
            for r in range(Rc):
                moe.moe_expert_ffn_decode(layer_of(r, i), xs[r][i], T, ids_all[r][i],
                                          wts_all[r][i], ys[i], 0, ws, stream)
        c0 = torch.cuda.Event(enable_timing=True)
        c1 = torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            gt.replay()
            c0.record(stream)
            for _ in range(4):
                gt.replay()
            c1.record(stream)
        stream.synchronize()
        t_ms = c0.elapsed_time(c1) / 4
        per_T[str(T)] = round(1e3 * t_ms / Rc, 2)
        exp_ms_total += t_ms
        exp_bytes += sum((uniq[r][i] + 1) * eb + 2 * T * sh.d * 2 for r in range(Rc))
        n_exp += Rc
        del gt
    achieved = exp_bytes / (exp_ms_total / 1e3) / 1e9

    # end to end through the public call: every window's tokens copied from
    # pinned host memory, the block forward, the output copied back; captured
    # as one CUDA graph per step (the copies are nodes of the graph)
    xh = [[x.cpu().pin_memory() for x in xs[r]] for r in range(R)]
    yh = [[torch.empty(T, sh.d, dtype=torch.bfloat16).pin_memory() for T in DECODE_WINDOWS]
          for _ in range(R)]
    xd = [torch.empty(T, sh.d, dtype=torch.bfloat16, device=dev) for T in DECODE_WINDOWS]
    Ke = min(K, 4)
    ge = torch.cuda.CUDAGraph()
    with torch.cuda.graph(ge, stream=stream):
        for r in range(R):
            for i, T in enumerate(DECODE_WINDOWS):
                xd[i].copy_(xh[r][i], non_blocking=True)
                moe.moe_block_forward(layer_of(r, i), xd[i], T, ys[i], 0, ws, stream)
                yh[r][i].copy_(ys[i], non_blocking=True)
    with torch.cuda.stream(stream):
        ge.replay()
    stream.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    f0 = torch.cuda.Event(enable_timing=True)
    f1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        f0.record(stream)
        for _ in range(Ke):
            ge.replay()
        f1.record(stream)
    stream.synchronize()
    e2e_ms = max_over_ranks(f0.elapsed_time(f1), world)
    e2e_value = Ke * ntok_step * world / (e2e_ms / 1e3)
    del ge

    res = {
        "metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": world,
        "steps": K, "warmup": W, "ms_per_step": round(ms / K, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f16",
        "data": "synthetic (seeded; random-init weights of the stated architecture)",
        "config": {"workload": WORKLOAD_DECODE,
                   "step": f"{R} rounds of the T=1,2,3,4 windows ({R * nwin} windows), each window "
                           f"on the next of {NL} layer copies with fresh tokens",
                   "tokens_per_step": ntok_step, "layer_copies": NL,
                   "l2": "inputs larger than L2 (32 layer copies rotated, "
                         f"{NL * (sh.E * eb + sh.E * sh.d * 4) / 1e9:.1f} GB)",
                   "parallelism": f"replicas x{world}",
                   "mma": "f16 x f16 -> f32 (weights dequantised in registers)",
                   "unique_experts_per_window": U_mean, "zipf_s_fitted": round(zipf_s, 3),
                   "l2_prefetch_next": bool(args.l2_next),
                   "top_k": sh.k, "prefer_hot": args.prefer_hot,
                   "prefer_bonus": args.prefer_bonus if args.prefer_hot else None,
                   "weights_gen_s": round(t_gen, 1)},
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"],
                     "unit": "GB/s", "frac": round(achieved / peaks["hbm_gbs"], 4),
                     "traffic": measured_traffic("decode_expert_step"), "peak_src": peaks["src"],
                     "kernel": "expert step (decode_gu_kernel + decode_dn_kernel per "
                               "moe_expert_ffn_decode call)",
                     "bytes_per_launch": round(exp_bytes / n_exp),
                     "us_per_launch_by_T": per_T,
                     "timing": "graphs of expert steps only, events around the replays"},
        "layer_roofline": {"bound": "hbm", "achieved": round(layer_gbs, 1),
                           "peak": peaks["hbm_gbs"], "unit": "GB/s",
                           "frac": round(layer_gbs / peaks["hbm_gbs"], 4),
                           "bytes_per_step": step_bytes,
                           "us_per_window": round(1e3 * ms / K / (R * nwin), 3),
                           "what": "whole block (router, experts, combine) over the timed steps"},
        "clocks": clocks,
        "e2e": {"value": round(e2e_value, 1), "unit": "tokens/s",
                "h2d_bytes_per_step": ntok_step * sh.d * 2, "d2h_bytes_per_step": ntok_step * sh.d * 2,
                "steps": Ke,
                "path": "moe_block_forward via the ctypes binding with each window's pinned-host "
                        "copies in and out, captured as one CUDA graph per step"},
        "gpu_launches": K * R * nwin * 3,   # router, expert, combine per window
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, cores, sample = oracle_cpu_baseline(layers[0].to("cpu"), DECODE_WINDOWS,
                                               args.cpu_seconds)
        res["cpu_baseline"] = {"value": round(v, 3), "unit": "tokens/s", "cores": cores,
                               "kind": "oracle", "sample": sample}
    del layers, structs, xs
    torch.cuda.empty_cache()
    if not args.no_prefill:
        res["prefill"] = measure_prefill(args, rank, world, local, K=args.prefill_steps, W=3)
        res["gpu_launches"] += res["prefill"]["gpu_launches"]
    return res


def measure_prefill(args, rank, world, local, K, W):
    """One layer, 8192-token chunk, 2-bit, router bias ~ N(0, 0.5).  A step is
    one block forward over the chunk (router, top-k, bucketing, grouped GEMMs,
    shared expert, combine); two layer copies alternate."""
    import torch

    from routed_expert_ffn_06_b200 import moe, synth
    dev = torch.device("cuda", local)
    wl = synth.WORKLOADS["prefill"]
    sh, T = wl["shape"], wl["T"]
    NL = 2
    layers = [synth.make_layer(sh, seed=rank * 1000 + i, layer=i, device=dev, bias=wl["bias"],
                               bias_std=wl["bias_std"], slot=wl["slot"]) for i in range(NL)]
    structs = [moe.make_layer_struct(l) for l in layers]
    # router weights split into bf16 hi/lo once per layer, as at model load
    splits = [moe.moe_router_split(L) for L in structs]
    for L, sp in zip(structs, splits):
        L.router_w_split = sp.data_ptr()
    ws = moe.alloc_workspace(structs[0], T)
    xs = [synth.make_tokens(T, sh.d, seed=rank * 1000 + 3, step=i, device=dev) for i in range(4)]
    y = torch.empty(T, sh.d, dtype=torch.bfloat16, device=dev)
    ids = torch.empty(T, sh.k, dtype=torch.int32, device=dev)
    wts = torch.empty(T, sh.k, dtype=torch.float32, device=dev)
    stream = torch.cuda.Stream(device=dev)

    def step(s, ev=None):
        L = structs[s % NL]
        x = xs[s % len(xs)]
        moe.moe_route_topk(L, x, T, 0, None, ids, wts, ws, stream)
        if ev is not None:
            ev[0].record(stream)
        moe.moe_expert_ffn_prefill(L, x, T, ids, wts, y, None, None, 0, ws, stream)
        if ev is not None:
            ev[1].record(stream)

    with torch.cuda.stream(stream):
        for s in range(W):
            step(s)
    stream.synchronize()
    st, code = moe.moe_workspace_error(ws, stream)
    if st != 0:
        raise RuntimeError(f"device error word {code:#x}")
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
    barrier(world)
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        with torch.cuda.stream(stream):
            e0.record(stream)
            for s in range(K):
                step(W + s, evs[s])
            e1.record(stream)
        stream.synchronize()
    barrier(world)
    ms = max_over_ranks(e0.elapsed_time(e1), world)
    exp_ms = max_over_ranks(sum(ev[0].elapsed_time(ev[1]) for ev in evs) / K, world)
    peaks = measured_peaks()
    flops = 2.0 * T * (sh.k + 1) * 3 * sh.F * sh.d          # gate/up + down, routed + shared
    achieved = flops / (exp_ms / 1e3) / 1e12
    # e2e: the chunk from pinned host memory, the public block call, back to the host
    xh = xs[0].cpu().pin_memory()
    yh = torch.empty(T, sh.d, dtype=torch.bfloat16).pin_memory()
    xd = torch.empty_like(xs[0])
    Ke = min(K, 10)
    barrier(world)
    torch.cuda.synchronize()
    f0 = torch.cuda.Event(enable_timing=True)
    f1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        f0.record(stream)
        for s in range(Ke):
            xd.copy_(xh, non_blocking=True)
            moe.moe_block_forward(structs[s % NL], xd, T, y, 0, ws, stream)
            yh.copy_(y, non_blocking=True)
        f1.record(stream)
    stream.synchronize()
    e2e_ms = max_over_ranks(f0.elapsed_time(f1), world)
    res = {
        "workload": WORKLOAD_PREFILL, "value": round(K * T * world / (ms / 1e3), 1),
        "unit": "tokens/s", "steps": K, "warmup": W, "ms_per_step": round(ms / K, 4),
        "tokens_per_step": T,
        "roofline": {"bound": "tensor", "achieved": round(achieved, 1),
                     "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                     "frac": round(achieved / peaks["bf16_tflops"], 4),
                     "traffic": measured_traffic("prefill_expert_step"),
                     "peak_src": peaks["src"] + " (bf16 burst; fp16 has the same nominal rate)",
                     "kernel": "expert step (prep, bucketing, gather, GEMM1, GEMM2, combine per "
                               "moe_expert_ffn_prefill call)",
                     "flops_per_launch": flops, "us_per_launch": round(exp_ms * 1e3, 1)},
        "clocks": clk.summary(),
        "e2e": {"value": round(Ke * T * world / (e2e_ms / 1e3), 1), "unit": "tokens/s",
                "h2d_bytes_per_step": T * sh.d * 2, "d2h_bytes_per_step": T * sh.d * 2,
                "steps": Ke, "path": "moe_block_forward via the ctypes binding, pinned host x/y"},
        "gpu_launches": K * PREFILL_LAUNCHES,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        OL = oracle.OracleLayer(layers[0].to("cpu"))
        n_tok, t0 = 0, time.perf_counter()
        xc = xs[0].cpu()
        while time.perf_counter() - t0 < args.cpu_seconds:
            OL.block_forward(xc, rows=list(range(n_tok, n_tok + 32)))
            n_tok += 32
        dt = time.perf_counter() - t0
        res["cpu_baseline"] = {"value": round(n_tok / dt, 3), "unit": "tokens/s",
                               "cores": oracle.num_threads(), "kind": "oracle",
                               "sample": f"{n_tok} of the chunk's 8192 tokens"}
    return res


def bench_prefill(args, rank, world, local):
    """--workload prefill: the prefill chunk as the line's value."""
    import torch
    torch.cuda.set_device(local)
    from routed_expert_ffn_06_b200 import moe
    moe.load()
    K = args.steps if args.steps is not None else 40
    W = args.warmup if args.warmup is not None else 5
    p = measure_prefill(args, rank, world, local, K, W)
    res = {"metric": METRIC, "value": p["value"], "unit": "tokens/s", "n_gpus": world,
           "steps": K, "warmup": W, "ms_per_step": p["ms_per_step"], "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": "f16",
           "data": "synthetic (seeded; random-init weights of the stated architecture)",
           "config": {"workload": WORKLOAD_PREFILL, "tokens_per_step": p["tokens_per_step"],
                      "layer_copies": 2,
                      "l2": "inputs larger than L2 (504 MB packed weights per layer)",
                      "parallelism": f"replicas x{world}",
                      "mma": "tcgen05 kind::f16, fp16 operands (weights dequantised to smem), "
                             "fp32 TMEM"},
           "roofline": p["roofline"], "clocks": p["clocks"], "e2e": p["e2e"],
           "gpu_launches": p["gpu_launches"]}
    if "cpu_baseline" in p:
        res["cpu_baseline"] = p["cpu_baseline"]
    return res


# ------------------------------------------------------------------- stack
def _stack_layers(wl, rank, dev):
    from routed_expert_ffn_06_b200 import synth
    return [synth.make_layer(wl["shape"], seed=rank * 1000, layer=l, device=dev, bias=wl["bias"],
                             slot=wl["slot"]) for l in range(wl["layers"])]


def _stack_bytes_per_step(structs, x, T, ws, stream):
    """Algorithmic HBM bytes of one decode step through the stack: every
    layer's router (E x d fp32), its unique selected experts and the shared
    expert, and the window in and out; the routing is taken from an eager pass
    over the same input."""
    import torch

    from routed_expert_ffn_06_b200 import moe
    L0 = structs[0]
    eb = _expert_bytes_struct(L0)
    ids = torch.empty(T, L0.top_k, dtype=torch.int32, device=x.device)
    wts = torch.empty(T, L0.top_k, dtype=torch.float32, device=x.device)
    y = [torch.empty_like(x), torch.empty_like(x)]
    tot, src = 0, x
    flags = moe.F_PRENORM | moe.F_RESIDUAL
    for l, L in enumerate(structs):
        moe.moe_route_topk(L, src, T, flags, None, ids, wts, ws, stream)
        stream.synchronize()
        U = int(torch.unique(ids).numel())
        tot += L.n_experts * L.d_model * 4 + (U + 1) * eb + 2 * T * L.d_model * 2
        moe.moe_block_forward(L, src, T, y[l % 2], flags, ws, stream)
        src = y[l % 2]
    stream.synchronize()
    return tot


def _expert_bytes_struct(L) -> int:
    gb = 8 if L.bits == 2 else 12
    return 3 * L.ffn * L.d_model // 32 * (gb + 2)


def bench_stack(args, rank, world, local):
    """48 routed-MoE layers, 3-bit (~34 GB), Zipf profile, frequency-ordered
    slots, 4 tokens per step, x <- x + MoE(RMSNorm(x)); a step is one pass of
    the 48 layers, captured as one CUDA graph."""
    import torch

    from routed_expert_ffn_06_b200 import moe, synth
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    moe.load()
    wl = synth.WORKLOADS["decode_stack"]
    sh, T, NLy = wl["shape"], wl["T"], wl["layers"]
    K = args.steps if args.steps is not None else wl["steps"]
    W = args.warmup if args.warmup is not None else 5
    t_gen = time.time()
    layers = _stack_layers(wl, rank, dev)
    t_gen = time.time() - t_gen
    structs = [moe.make_layer_struct(l) for l in layers]
    if args.l2_next:   # layer l is followed by l + 1, the last by the next step's first
        moe.link_l2_next(structs)
    ws = moe.alloc_workspace(structs[0], T)
    G = 16
    x0 = [synth.make_tokens(T, sh.d, seed=rank * 1000 + 9, step=s, device=dev) for s in range(G)]
    bufs = [torch.empty(T, sh.d, dtype=torch.bfloat16, device=dev) for _ in range(2)]
    flags = moe.F_PRENORM | moe.F_RESIDUAL
    stream = torch.cuda.Stream(device=dev)

    def enqueue(s, src=None):
        src = x0[s % G] if src is None else src
        for l in range(NLy):
            dst = bufs[l % 2]
            moe.moe_block_forward(structs[l], src, T, dst, flags, ws, stream)
            src = dst

    with torch.cuda.stream(stream):
        for s in range(2):
            enqueue(s)
    stream.synchronize()
    step_bytes = _stack_bytes_per_step(structs, x0[0], T, ws, stream)
    graphs = []
    for s in range(G):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            enqueue(s)
        graphs.append(g)
    with torch.cuda.stream(stream):
        for s in range(W):
            graphs[s % G].replay()
    stream.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        with torch.cuda.stream(stream):
            e0.record(stream)
            for s in range(K):
                graphs[s % G].replay()
            e1.record(stream)
        stream.synchronize()
    barrier(world)
    ms = max_over_ranks(e0.elapsed_time(e1), world)
    st, code = moe.moe_workspace_error(ws, stream)
    if st != 0:
        raise RuntimeError(f"device error word {code:#x}")
    # end to end: the window from pinned host memory, 48 layers, back to the host
    xh = x0[0].cpu().pin_memory()
    yh = torch.empty(T, sh.d, dtype=torch.bfloat16).pin_memory()
    xd = torch.empty_like(x0[0])
    Ke = min(K, 64)
    barrier(world)
    torch.cuda.synchronize()
    f0 = torch.cuda.Event(enable_timing=True)
    f1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        f0.record(stream)
        for s in range(Ke):
            xd.copy_(xh, non_blocking=True)
            enqueue(s, xd)
            yh.copy_(bufs[(NLy - 1) % 2], non_blocking=True)
        f1.record(stream)
    stream.synchronize()
    e2e_ms = max_over_ranks(f0.elapsed_time(f1), world)
    peaks = measured_peaks()
    achieved = step_bytes / (ms / K / 1e3) / 1e9
    eb = _expert_bytes_struct(structs[0])
    res = {
        "metric": METRIC, "value": round(K * T * world / (ms / 1e3), 1), "unit": "tokens/s",
        "n_gpus": world, "steps": K, "warmup": W, "ms_per_step": round(ms / K, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f16",
        "data": "synthetic (seeded; random-init weights of the stated architecture)",
        "config": {"workload": "decode 48-layer stack of routed-MoE blocks: d=2048, 512 experts "
                               "ffn=512 + shared, top-10, 3-bit g32, Zipf profile, "
                               "frequency-ordered slots, 4 tokens/step, pre-norm + residual",
                   "tokens_per_step": T,
                   "weights_gb": round(NLy * (sh.E * eb + eb + sh.E * sh.d * 4) / 1e9, 2),
                   "l2": "inputs larger than L2 (34 GB of weights per step)",
                   "l2_prefetch_next": bool(args.l2_next),
                   "weights_gen_s": round(t_gen, 1), "parallelism": f"replicas x{world}"},
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"],
                     "unit": "GB/s", "frac": round(achieved / peaks["hbm_gbs"], 4),
                     "traffic": None, "peak_src": peaks["src"],
                     "kernel": "one step: 48 x (router, gate/up, down)",
                     "bytes_per_launch": step_bytes},
        "clocks": clk.summary(),
        "e2e": {"value": round(Ke * T * world / (e2e_ms / 1e3), 1), "unit": "tokens/s",
                "h2d_bytes_per_step": T * sh.d * 2, "d2h_bytes_per_step": T * sh.d * 2,
                "steps": Ke, "path": "48 x moe_block_forward via the ctypes binding, pinned host x/y"},
        "gpu_launches": K * NLy * 3,
    }
    return res


def bench_mix(args, rank, world, local):
    """48 routed-MoE layers, 3-bit: a 32,768-token prompt read as 4 chunks of
    8192 tokens (each chunk through all 48 layers), then 512 decode steps of 4
    tokens; every 64 decode steps each layer's expert ranking is re-drawn (the
    router bias permuted), the packed slot layout staying as it was."""
    import torch

    from routed_expert_ffn_06_b200 import moe, synth
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    moe.load()
    wl = synth.WORKLOADS["mix"]
    sh, T, NLy = wl["shape"], wl["T"], wl["layers"]
    C, NC = wl["chunk"], wl["chunks"]
    DS = args.steps if args.steps is not None else wl["decode_steps"]
    drift = wl["drift_every"]
    W = args.warmup if args.warmup is not None else 3
    t_gen = time.time()
    layers = _stack_layers(wl, rank, dev)
    t_gen = time.time() - t_gen
    AE = args.adapt_every
    counts = [torch.zeros(sh.E, dtype=torch.float32, device=dev) if AE else None for _ in layers]
    structs = [moe.make_layer_struct(l, route_counts=c) for l, c in zip(layers, counts)]
    splits = [moe.moe_router_split(L) for L in structs]   # once per layer, as at model load
    for L, sp in zip(structs, splits):
        L.router_w_split = sp.data_ptr()
    if args.l2_next:
        moe.link_l2_next(structs)
    ws = moe.alloc_workspace(structs[0], C)
    if AE:
        n = moe.moe_adapt_workspace_bytes(structs[0], args.adapt_swaps)
        aws = torch.zeros(n + 256, dtype=torch.uint8, device=dev)
        aws = aws[(-aws.data_ptr()) % 256:]
    flags = moe.F_PRENORM | moe.F_RESIDUAL
    stream = torch.cuda.Stream(device=dev)
    biases = [[l.router_bias.clone()] + [synth.permute_profile(l, seed=rank * 1000, epoch=e + 1)
                                          for e in range(DS // drift + 1)] for l in layers]
    chunks = [synth.make_tokens(C, sh.d, seed=rank * 1000 + 21, step=c, device=dev) for c in range(NC)]
    cb = [torch.empty(C, sh.d, dtype=torch.bfloat16, device=dev) for _ in range(2)]
    G = 16
    wins = [synth.make_tokens(T, sh.d, seed=rank * 1000 + 22, step=s, device=dev) for s in range(G)]
    wb = [torch.empty(T, sh.d, dtype=torch.bfloat16, device=dev) for _ in range(2)]

    def run_stack(src, bufs, n):
        for l in range(NLy):
            moe.moe_block_forward(structs[l], src, n, bufs[l % 2], flags, ws, stream)
            src = bufs[l % 2]

    def set_epoch(e):
        for l in range(NLy):
            layers[l].router_bias.copy_(biases[l][e], non_blocking=True)

    with torch.cuda.stream(stream):
        for _ in range(W):
            run_stack(chunks[0], cb, C)
            run_stack(wins[0], wb, T)
    stream.synchronize()
    graphs = []
    for s in range(G):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            run_stack(wins[s], wb, T)
        graphs.append(g)
    barrier(world)
    torch.cuda.synchronize()
    p0, p1, d1 = (torch.cuda.Event(enable_timing=True) for _ in range(3))
    with ClockSampler(local) as clk:
        with torch.cuda.stream(stream):
            set_epoch(0)
            p0.record(stream)
            for c in range(NC):
                run_stack(chunks[c], cb, C)
            p1.record(stream)
            for s in range(DS):
                if s % drift == 0:
                    set_epoch(s // drift)
                if AE and s > 0 and s % AE == 0:
                    for L in structs:
                        moe.moe_adapt_layout(L, args.adapt_decay, args.adapt_swaps, None, aws,
                                             stream)
                graphs[s % G].replay()
            d1.record(stream)
        stream.synchronize()
    barrier(world)
    ms_pf = max_over_ranks(p0.elapsed_time(p1), world)
    ms_dec = max_over_ranks(p1.elapsed_time(d1), world)
    st, code = moe.moe_workspace_error(ws, stream)
    if st != 0:
        raise RuntimeError(f"device error word {code:#x}")
    ntok = NC * C + DS * T
    ms = ms_pf + ms_dec
    peaks = measured_peaks()
    flops = 2.0 * NC * C * (sh.k + 1) * 3 * sh.F * sh.d * NLy
    eb = _expert_bytes_struct(structs[0])
    return {
        "metric": METRIC, "value": round(ntok * world / (ms / 1e3), 1), "unit": "tokens/s",
        "n_gpus": world, "steps": DS, "warmup": W, "ms_per_step": round(ms_dec / DS, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f16",
        "data": "synthetic (seeded; random-init weights of the stated architecture)",
        "config": {"workload": "48-layer 3-bit stack: 32,768-token prompt as 4 x 8192 chunks, then "
                               "512 decode steps of 4 tokens, expert ranking re-drawn every 64 steps",
                   "tokens": ntok, "weights_gb": round(NLy * (sh.E * eb + eb + sh.E * sh.d * 4) / 1e9, 2),
                   "l2": "inputs larger than L2 (34 GB of weights)",
                   "l2_prefetch_next": bool(args.l2_next),
                   "weights_gen_s": round(t_gen, 1), "parallelism": f"replicas x{world}"},
        "adaptive_layout": ({"every_steps": AE, "max_swaps": args.adapt_swaps,
                             "decay": args.adapt_decay} if AE else None),
        "prefill_tokens_per_s": round(NC * C * world / (ms_pf / 1e3), 1),
        "decode_tokens_per_s": round(DS * T * world / (ms_dec / 1e3), 1),
        "roofline": {"bound": "tensor", "achieved": round(flops / (ms_pf / 1e3) / 1e12, 1),
                     "peak": peaks["bf16_tflops_sustained"], "unit": "TFLOP/s",
                     "frac": round(flops / (ms_pf / 1e3) / 1e12 / peaks["bf16_tflops_sustained"], 4),
                     "traffic": None, "peak_src": peaks["src"] + " (bf16 sustained)",
                     "kernel": "prefill phase: 4 chunks x 48 layers (expert GEMM FLOPs)"},
        "clocks": clk.summary(),
        "gpu_launches": NC * NLy * 11 + DS * NLy * 3,
    }


# --------------------------------------------------------------- reference
def run_reference(args, rank, world):
    """The fp64 oracle on the host cores, on the same workload, metric and unit
    as our arm (a bounded sample of it per step)."""
    if rank != 0:
        return None
    import oracle
    from routed_expert_ffn_06_b200 import synth
    K = args.steps if args.steps is not None else 20
    W = args.warmup if args.warmup is not None else 5
    if args.workload == "prefill":
        wl = synth.WORKLOADS["prefill"]
        layer = synth.make_layer(wl["shape"], seed=0, device="cpu", bias=wl["bias"],
                                 bias_std=wl["bias_std"], slot=wl["slot"])
        OL = oracle.OracleLayer(layer)
        x = synth.make_tokens(wl["T"], wl["shape"].d, seed=3, step=0)
        per = 8    # tokens of the 8192 chunk per step

        def step(s):
            OL.block_forward(x, rows=list(range((s * per) % wl["T"], (s * per) % wl["T"] + per)))
        workload = WORKLOAD_PREFILL
        sample = f"{per} of the chunk's tokens per step"
        tok = per
    elif args.workload in ("stack", "mix"):
        wl = synth.WORKLOADS["decode_stack"]
        nl = 2   # layers of the stack per step (the oracle is far too slow for 48)
        layers = [oracle.OracleLayer(synth.make_layer(wl["shape"], seed=0, layer=l, device="cpu",
                                                      bias=wl["bias"], slot=wl["slot"]))
                  for l in range(nl)]

        import torch

        def step(s):
            x = synth.make_tokens(wl["T"], wl["shape"].d, seed=9, step=s)
            for OL in layers:
                r = OL.block_forward(x, flags=oracle.PRENORM | oracle.RESIDUAL)
                x = torch.from_numpy(r["y"]).to(torch.bfloat16)
        workload = ("decode 48-layer stack of routed-MoE blocks, 3-bit, 4 tokens/step, pre-norm + "
                    "residual")
        sample = f"{nl} of the 48 layers per step, scaled to 48"
        tok = wl["T"] * nl / 48.0
    else:
        wl = synth.WORKLOADS["decode"]
        layer = synth.make_layer(wl["shape"], seed=0, device="cpu", bias=wl["bias"], slot=wl["slot"])
        OL = oracle.OracleLayer(layer)

        def step(s):
            for i, T in enumerate(DECODE_WINDOWS):
                OL.block_forward(synth.make_tokens(T, wl["shape"].d, seed=7, step=s * 4 + i))
        workload = WORKLOAD_DECODE
        sample = "one round of the T=1,2,3,4 windows (10 tokens) per step"
        tok = sum(DECODE_WINDOWS)
    for s in range(W):
        step(s)
    t0 = time.perf_counter()
    for s in range(K):
        step(W + s)
    dt = time.perf_counter() - t0
    v = K * tok / dt
    return {"metric": METRIC, "value": round(v, 3), "unit": "tokens/s", "n_gpus": world,
            "steps": K, "warmup": W, "ms_per_step": round(1e3 * dt / K, 2),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "impl": "reference", "config": {"workload": workload},
            "cpu_baseline": {"value": round(v, 3), "unit": "tokens/s", "cores": oracle.num_threads(),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": round(v, 3), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def main():
    args = parse()
    rank, world, local = dist_init()
    try:
        if args.impl == "reference":
            res = run_reference(args, rank, world)
        elif args.workload == "decode":
            res = bench_decode(args, rank, world, local)
        elif args.workload == "prefill":
            res = bench_prefill(args, rank, world, local)
        elif args.workload == "mix":
            res = bench_mix(args, rank, world, local)
        else:
            res = bench_stack(args, rank, world, local)
        if rank == 0 and res is not None:
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
