#!/usr/bin/env python
"""Benchmark of the ISPA warmup hot path on B200.

One step = the whole hot path over one batch of synthetic input: dual-stream
attention of every chunk, Gram accumulation of its rows, the closed-form
Delta W solve, the reconstruction error of every layer and the layer ranking.
Default workload: the 1.3B-class full warmup (30 layers of 12 heads x 128,
4 chunks of 4680 queries over 1560 sink + 4680 local + 0..14040 history
keys). The same invocation also measures the 14B-class warmup (40 layers,
40 heads) and the 1.3B single chunk (the last warmup chunk of one layer) and
reports them as the sub-objects ``14B-warmup`` and ``1.3B-chunk``.
``--config c1|c3`` makes one of those the main line (no sub-objects);
``--config c4`` runs the post-transition streaming benchmark.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints one JSON line (rank 0). ``value`` is the step's algorithmic TFLOP
(attention 4*Nq*Nk*d counted once, Gram 4*N*d^2, solve (1/3+4)*d^3; the
error pass is an HBM-bound reduction credited with no flops) divided by the
device time of the step, summed over all ranks' work; the attention TFLOP/s
and the absorb ms per layer, each against its roofline, are the per-stage
figures.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "dual-stream attention TFLOP/s and absorb ms/layer at 1.3B/14B shapes, % roofline"
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
TF32_FILE = os.path.join(ROOT, "profiles", "tf32_peak_cublas_gemm_8192.txt")
L2_FLUSH_BYTES = 512 << 20


# ---------------------------------------------------------------- work model

def step_work(cfg):
    """Algorithmic FLOPs of one step, split by stage."""
    d = cfg.d
    attn = 0.0
    for c in range(cfg.n_chunks):
        nk = cfg.sink_tokens + cfg.chunk_tokens + len(cfg.history_frames_of(c)) * cfg.tokens_per_frame
        attn += 4.0 * cfg.chunk_tokens * nk * d
    gram = 4.0 * cfg.warmup_rows * d * d
    solve = (1.0 / 3.0 + 4.0) * d ** 3
    L = cfg.layers
    # the error stage reads G, R, S, W W^T, Delta W and B once (W W^T is
    # formed when the weights load, outside the step): no flops credited
    return {"attention": attn * L, "gram": gram * L, "solve": solve * L, "error": 0.0}


def peaks():
    try:
        with open(PEAKS_FILE) as f:
            p = json.load(f)
        return p["bf16_tflops"], p["hbm_gbs"], "measured"
    except Exception:
        return 1590.0, 6650.0, "fallback"


def tf32_peak(bf16_peak):
    """Dense tf32 tensor rate: cuBLAS tf32 GEMM measured on this GPU model
    (``--measure-tf32-peak``, summary committed under profiles/), else half
    the bf16 peak (the nominal ratio)."""
    try:
        with open(TF32_FILE) as f:
            kv = dict(line.strip().split("=", 1) for line in f if "=" in line and not line.startswith("#"))
        return float(kv["tf32_tflops"]), "measured cuBLAS tf32 GEMM (burst)"
    except Exception:
        return bf16_peak / 2.0, "bf16 peak x 1/2 (nominal tf32:bf16 ratio)"


def measure_tf32_peak():
    """cuBLAS fp32 GEMM with tf32 tensor cores allowed, 8192^3, burst timing."""
    import torch
    torch.backends.cuda.matmul.allow_tf32 = True
    n = 8192
    a = torch.randn(n, n, device="cuda")
    b = torch.randn(n, n, device="cuda")
    c = torch.empty(n, n, device="cuda")
    for _ in range(5):
        torch.matmul(a, b, out=c)
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    reps = 20
    s.record()
    for _ in range(reps):
        torch.matmul(a, b, out=c)
    e.record()
    torch.cuda.synchronize()
    ms = s.elapsed_time(e) / reps
    print(json.dumps({"tf32_tflops": round(2.0 * n ** 3 / (ms * 1e-3) / 1e12, 1), "n": n,
                      "ms_per_gemm": round(ms, 4), "reps": reps,
                      "device": torch.cuda.get_device_name()}), flush=True)


def error_bytes(cfg):
    """Bytes the batched error pass reads per layer (fp32, W W^T resident):
    the 128 x 128 tiles of G and S on and above the diagonal, R, W W^T,
    Delta W and B in full."""
    t = cfg.d // 128
    upper = t * (t + 1) // 2
    return int((2 * upper * 128 * 128 + 4 * cfg.d * cfg.d) * 4)


def absorb_roofline(cfg, gram_ms, solve_ms, bf16_peak, hbm_peak):
    """Precision-constrained roofline of the absorb per layer: Gram 4 N d^2 at
    the tf32 rate, solve (1/3 + 4) d^3 at a third of it (three tf32 products
    per fp32-accurate product), error 6 d^2 fp32 reads at the HBM rate. For
    context, also the time if every flop ran at the bf16 rate (a bound that
    ignores the precision the solve needs)."""
    d, L = cfg.d, cfg.layers
    tf32, src = tf32_peak(bf16_peak)
    t_gram = 4.0 * cfg.warmup_rows * d * d / (tf32 * 1e12)
    t_solve = (1.0 / 3.0 + 4.0) * d ** 3 / (tf32 / 3.0 * 1e12)
    t_err = 6.0 * d * d * 4 / (hbm_peak * 1e9)
    t_star = (t_gram + t_solve + t_err) * 1e3
    t_bf16 = ((4.0 * cfg.warmup_rows * d * d + (1.0 / 3.0 + 4.0) * d ** 3) / (bf16_peak * 1e12)
              + t_err) * 1e3
    got = (gram_ms + solve_ms) / L
    return {"bound": "tensor (tf32 Gram, 3xTF32 solve) + hbm (error)",
            "t_star_ms_per_layer": round(t_star, 4), "achieved_ms_per_layer": round(got, 4),
            "frac": round(t_star / got, 4), "tf32_peak": tf32, "tf32_peak_source": src,
            "hbm_peak": hbm_peak,
            "bf16_only": {"t_ms_per_layer": round(t_bf16, 4), "frac": round(t_bf16 / got, 4),
                          "note": "every flop at the bf16 rate: context, not the target"},
            "parts_ms_per_layer": {"gram": round(gram_ms / L, 4), "solve_error": round(solve_ms / L, 4),
                                   "t_star_gram": round(t_gram * 1e3, 4),
                                   "t_star_solve": round(t_solve * 1e3, 4),
                                   "t_star_error": round(t_err * 1e3, 4)}}


def source_hash():
    """Hash of the attention kernel's sources with comments and blank lines
    removed: a change of the code invalidates the committed traffic figures,
    a change of the comments does not."""
    h = hashlib.sha256()
    for f in ("attention.cu", "sm100.cuh", "attention.h"):
        with open(os.path.join(ROOT, "kv_cache_absorption_b200", "csrc", f)) as fh:
            for line in fh:
                code = re.sub(r"//.*$", "", line).strip()
                if code:
                    h.update(code.encode() + b"\n")
    return h.hexdigest()[:16]


def traffic_file(workload_name):
    return os.path.join(ROOT, "profiles", f"dual_attention_{workload_name}_traffic.txt")


def traffic_per_launch(workload_name, layers_per_launch=1):
    """DRAM bytes per attention launch of this workload from the committed ncu
    summary, or None when there is none, the kernel source changed since the
    counters were taken, or they were taken on launches of another number of
    layers."""
    try:
        with open(traffic_file(workload_name)) as f:
            kv = dict(line.strip().split("=", 1) for line in f if "=" in line and not line.startswith("#"))
        if kv.get("source_hash") != source_hash():
            return None
        if int(kv.get("layers_per_launch", "1")) != layers_per_launch:
            return None
        return float(kv["dram_bytes_per_launch"])
    except Exception:
        return None


# ---------------------------------------------------------------- clocks

class ClockSampler:
    FIELDS = ("pci.bus_id,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, bus_id: str, period_ms: int = 50):
        self.bus_id = bus_id.lower()
        self.proc = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", str(period_ms)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                text=True)
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
            out = ""
        rows = []
        for line in out.splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            if not parts[0].lower().endswith(self.bus_id[-12:]):
                continue
            try:
                rows.append(parts)
            except ValueError:
                pass
        if not rows:   # bus id not reported: use the only GPU in the list, if there is one
            ids = {line.split(",")[0].strip() for line in out.splitlines() if line.count(",") >= 8}
            if len(ids) == 1:
                rows = [[p.strip() for p in line.split(",")] for line in out.splitlines()
                        if line.count(",") >= 8]
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v.strip() == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": float(rows[0][2]) if rows[0][2].replace(".", "").isdigit() else None,
                "reasons": reasons, "samples": len(rows)}


# ---------------------------------------------------------------- oracle timing (host)

_ORACLE_INPUTS = {}


def oracle_timing(cfg, att_rows: int = 256, gram_rows: int = 1024, seed: int = 0):
    """Times the float64 oracle on a bounded sample of one layer of ``cfg``,
    each stage at a size where its cost grows with the work: dual attention
    of ``att_rows`` query rows of the last chunk for one head (heads are
    independent; one head keeps the per-call work on the keys small next to
    the rows'), all keys; the Gram and the direct error of ``gram_rows`` rows
    (the attention rows repeated: their cost does not depend on the values);
    the full-size closed-form solve. Returns per-stage (flops, seconds)."""
    import numpy as np
    import oracle
    from ispa_synth import layer_streams
    key = (cfg.name, seed)
    if key not in _ORACLE_INPUTS:      # inputs widened to float64 once, outside the timing
        st = layer_streams(cfg, 0, seed=seed)
        ch = {k: oracle.as_f64(v) for k, v in st.chunk(cfg.n_chunks - 1).items()}
        _ORACLE_INPUTS[key] = (ch, oracle.as_f64(st.w))
    ch, w = _ORACLE_INPUTS[key]
    h = {k: v[:, :1] for k, v in ch.items()}          # head 0
    rows = min(att_rows, ch["q"].shape[0])
    nk = ch["k_sink"].shape[0] + ch["k_loc"].shape[0] + ch["k_hist"].shape[0]
    d, hd = cfg.d, cfg.head_dim
    t0 = time.perf_counter()
    o = oracle.dual_attention(h["q"][:rows], h["k_sink"], h["v_sink"], h["k_loc"], h["v_loc"],
                              h["k_hist"], h["v_hist"])
    t1 = time.perf_counter()
    reps = -(-gram_rows // rows)
    a_loc = np.tile(o["a_loc"], (reps, cfg.heads))[:gram_rows]     # [gram_rows, d]
    a_full = np.tile(o["a_full"], (reps, cfg.heads))[:gram_rows]
    d_rows = a_full - a_loc
    t2 = time.perf_counter()
    G, R, S = oracle.gram(a_loc, d_rows)
    t3 = time.perf_counter()
    dW, B = oracle.absorb(G, R, w, oracle.default_lambda(G))   # full d x d solve
    t4 = time.perf_counter()
    oracle.reconstruction_error(a_loc, a_full, w, dW)
    t5 = time.perf_counter()
    return {
        "attention": (4.0 * rows * nk * hd, t1 - t0),
        "gram": (4.0 * gram_rows * d * d, t3 - t2),
        "solve": ((1.0 / 3.0 + 4.0) * d ** 3, t4 - t3),
        "error": (4.0 * gram_rows * d * d, t5 - t4),
    }


def cpu_cores():
    try:
        n = len(os.sched_getaffinity(0))
    except Exception:
        n = os.cpu_count() or 1
    blas = None
    try:
        from threadpoolctl import threadpool_info
        blas = max((i.get("num_threads", 0) for i in threadpool_info()), default=None)
    except Exception:
        pass
    return n, blas


def oracle_throughput(cfg, budget_s: float):
    """Oracle throughput on this workload mix, extrapolated stage by stage
    from bounded samples: t_full = sum_s F_s * (t_s / f_s); samples repeat
    until about half the budget is spent."""
    work = step_work(cfg)
    acc = {s: [0.0, 0.0] for s in work}
    spent, n = 0.0, 0
    while n < 2 or (spent < budget_s * 0.5 and n < 20):
        timing = oracle_timing(cfg)
        for s in acc:
            acc[s][0] += timing[s][0]
            acc[s][1] += timing[s][1]
        spent += sum(t for _, t in timing.values())
        n += 1
    stages = {s: work[s] * acc[s][1] / max(acc[s][0], 1.0) for s in work if work[s] > 0}
    t_full = sum(stages.values())
    total = sum(work.values())
    cores, blas = cpu_cores()
    return {"value": round(total / t_full / 1e12, 6), "unit": "TFLOP/s", "cores": blas or cores,
            "host_cores": cores, "blas_threads": blas,
            "stage_seconds_per_full_step": {s: round(t, 3) for s, t in stages.items()},
            "kind": "oracle",
            "sample": (f"{n} x: float64 oracle on 256 query rows of the last chunk for one head "
                       f"(all keys), the Gram and direct error of 1024 rows, one full "
                       f"{cfg.d}x{cfg.d} solve; per-stage rates extrapolated to the full step"),
            "seconds_per_full_step": round(t_full, 3)}


def dist_setup():
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def clocks_rejected(clocks) -> bool:
    """A timed region whose clock record shows hw_slowdown, hw_thermal_slowdown or
    sw_thermal_slowdown, or SM clocks under 75% of their maximum with no reason
    active. sw_power_cap alone is kept (normal under load on a 1 kW part)."""
    if not clocks:
        return False
    bad = {"hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"}
    if bad & set(clocks.get("reasons") or []):
        return True
    sm, mx = clocks.get("sm_mhz"), clocks.get("sm_max_mhz")
    return bool(sm and mx and sm < 0.75 * mx and not clocks.get("reasons"))


def any_over_ranks(flag: bool, world: int) -> bool:
    if world == 1:
        return bool(flag)
    import torch
    import torch.distributed as dist
    t = torch.tensor([1.0 if flag else 0.0], device="cuda")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return bool(t.item() > 0)


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device="cuda")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ---------------------------------------------------------------- our arm

def workload(args):
    from ispa_synth import CONFIGS, scaled
    cfg = CONFIGS[args.config]
    if args.layers is not None and args.layers != cfg.layers:
        # keep the workload's fraction of L-Layers
        k = cfg.select_k if cfg.select_k is not None else cfg.layers // 2
        k = max(0, min(args.layers, round(k * args.layers / cfg.layers)))
        cfg = scaled(cfg, name=f"{cfg.name}-{args.layers}layers", layers=args.layers, select_k=k)
    return cfg


def make_inputs(cfg, rank, device, layers=None, replica=True):
    """Per layer: its Q/K/V frame streams and the chunk dicts (views into
    them); the projections stacked as one [L, d, d] tensor; the streams'
    storage, one [L, frames, tokens, heads, head_dim] tensor per Q, K, V (a
    chunk of every layer is one strided view of it). ``layers`` lists the
    global layer ids to build (default: all); replicas (one full copy of the
    workload per rank) draw rank-specific seeds, layer shards the global
    ones."""
    import torch
    from ispa_synth import stacked_layer_streams
    layers = list(range(cfg.layers)) if layers is None else layers
    ids = [l + (1000 * rank if replica else 0) for l in layers]
    streams, qkv = stacked_layer_streams(cfg, ids, seed=0, device=device)
    chunks = [[st.chunk(c) for c in range(cfg.n_chunks)] for st in streams]
    W_all = torch.stack([st.w for st in streams])
    for st in streams:
        st.w = None
    return streams, chunks, W_all, qkv


def config_of(cfg, world, sharded, K):
    """The ``config`` object of a bench line (both arms print the same one)."""
    return {"workload": cfg.name, "layers": cfg.layers, "heads": cfg.heads,
            "head_dim": cfg.head_dim, "d": cfg.d, "chunks": cfg.n_chunks,
            "chunk_rows": cfg.chunk_tokens, "sink": cfg.sink_tokens,
            "history": [len(cfg.history_frames_of(c)) * cfg.tokens_per_frame
                        for c in range(cfg.n_chunks)],
            "select_k": K, "l2": "flushed (512 MB write) before every timed step",
            "weights": "W and W W^T per layer resident (W W^T formed once at load)",
            "parallelism": (f"layer-sharded x{world} (errors all-gathered)" if sharded else
                            f"replicas x{world}" if world > 1 else "single GPU")}


def bus_id_of(dev):
    import torch
    pr = torch.cuda.get_device_properties(dev)
    return f"{getattr(pr, 'pci_domain_id', 0):08x}:{getattr(pr, 'pci_bus_id', 0):02x}:" \
           f"{getattr(pr, 'pci_device_id', 0):02x}.0"


def measure_warmup(args, cfg, world, rank, steps, warmup, with_e2e, with_cpu):
    """Times the whole warmup step of ``cfg`` and returns its bench fields."""
    import torch
    from kv_cache_absorption_b200 import ispa
    from kv_cache_absorption_b200.warmup import LayerWarmup, rank as rank_layers
    from kv_cache_absorption_b200.sharding import gather_errors, owned_layers
    from ispa_synth import stacked_chunk
    dev = torch.device("cuda", torch.cuda.current_device())
    # several GPUs: multi-layer warmups shard their layers (l on rank l mod N,
    # errors all-gathered for the ranking); a one-layer step runs as replicas
    sharded = world > 1 and cfg.layers >= world
    my_layers = owned_layers(cfg.layers, world, rank) if sharded else list(range(cfg.layers))
    layer_streams_, chunks_per_layer, W_all, qkv = make_inputs(cfg, rank, dev, my_layers,
                                                               replica=not sharded)
    max_hist = max(len(cfg.history_frames_of(c)) for c in range(cfg.n_chunks)) * cfg.tokens_per_frame
    L = cfg.layers
    L_mine = len(my_layers)
    # the same chunk of `group` layers in one attention launch (one grid over
    # all their units: whole waves of the SMs), groups in flight on as many
    # streams as slots (their launches fill each other's tails); 10 layers a
    # launch and two streams by default
    group = max(1, min(args.group, L_mine))
    stacked_chunks = ([stacked_chunk(cfg, qkv, c) for c in range(cfg.n_chunks)]
                      if group > 1 else None)
    runner = LayerWarmup(cfg.heads, cfg.head_dim, cfg.chunk_tokens, cfg.sink_tokens,
                         cfg.chunk_tokens, max_hist, n_layers=L_mine, device=dev,
                         n_slots=max(1, min(args.slots, L_mine)), group=group)
    groups = runner.layer_groups() if group > 1 else [(l, 1) for l in range(L_mine)]
    K = cfg.select_k if cfg.select_k is not None else L // 2
    err_mine = torch.empty(L_mine, 2, dtype=torch.float64, device=dev)
    err = torch.empty(L, 2, dtype=torch.float64, device=dev)
    perm = torch.empty(L, dtype=torch.int32, device=dev)
    sel = torch.empty(L, dtype=torch.uint8, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    E = lambda: torch.cuda.Event(enable_timing=True)
    runner.weight_gram(W_all)     # W W^T per layer: model weights only, formed once at load
    streams = [torch.cuda.current_stream()] + [torch.cuda.Stream() for _ in range(runner.n_slots - 1)]

    def chunks_in(sets_stacked, sets_per_layer, strms):
        if sets_stacked is not None:
            runner.layers_chunks_stacked(sets_stacked, strms)
        else:
            runner.layers_chunks(sets_per_layer, strms)

    def step():
        chunks_in(stacked_chunks, chunks_per_layer, streams)
        runner.absorb_all(W_all, err_mine)    # every layer's solve + error, batched
        err.copy_(gather_errors(err_mine, L, world) if sharded else err_mine)
        rank_layers(err, K, perm, sel)

    def step_instrumented(ev):
        """The same work on one stream with events around every stage (the
        per-stage breakdown; not the timed steps)."""
        for l0, n in groups:
            for c in range(cfg.n_chunks):
                ev["a0"].append(E()); ev["a0"][-1].record()
                if stacked_chunks is not None:
                    runner.attention_layers(stacked_chunks[c], l0, n)
                else:
                    runner.attention(chunks_per_layer[l0][c])
                ev["a1"].append(E()); ev["a1"][-1].record()
                for j in range(n):
                    if stacked_chunks is not None:
                        runner.gram_group(c == 0, j, l0 + j)
                    else:
                        runner.gram(first=(c == 0), layer=l0 + j)
                ev["g1"].append(E()); ev["g1"][-1].record()
        runner.solve_all(W_all)
        ev["e0"].append(E()); ev["e0"][-1].record()
        runner.error_all(W_all, err_mine)
        ev["s1"].append(E()); ev["s1"][-1].record()
        err.copy_(gather_errors(err_mine, L, world) if sharded else err_mine)
        rank_layers(err, K, perm, sel)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    if ispa.read_status(runner.status) != 0:
        raise RuntimeError(f"device status {ispa.read_status(runner.status)} after warmup")

    def timed():
        starts, ends = [], []
        barrier(world)
        torch.cuda.synchronize()
        sampler = ClockSampler(bus_id_of(dev))
        time.sleep(0.15)
        launches0 = ispa.ispa_kernel_launches()
        for _ in range(steps):
            flush.zero_()                   # L2 flush between timed steps, outside the events
            s0, e0 = E(), E()
            s0.record()
            step()
            e0.record()
            starts.append(s0), ends.append(e0)
        torch.cuda.synchronize()
        launches_ = ispa.ispa_kernel_launches() - launches0
        clocks_ = sampler.stop()
        barrier(world)
        return sum(a.elapsed_time(b) for a, b in zip(starts, ends)) / steps, launches_, clocks_

    step_ms, launches, clocks = timed()
    # a slowdown other than the power cap, or clocks stuck low with no reason
    # (a clock lock left by someone else): measured once more, on every rank
    if any_over_ranks(clocks_rejected(clocks), world):
        first = clocks
        step_ms, launches, clocks = timed()
        if clocks is not None:
            clocks = dict(clocks, remeasured_after=(first or {}).get("reasons") or ["clocks low"])

    # per-stage breakdown: a few more steps on one stream, events around every stage
    n_inst = max(1, min(steps, 5))
    ev = {"a0": [], "a1": [], "g1": [], "e0": [], "s1": []}
    for _ in range(n_inst):
        flush.zero_()
        step_instrumented(ev)
    torch.cuda.synchronize()
    attn_ms = sum(a.elapsed_time(b) for a, b in zip(ev["a0"], ev["a1"])) / n_inst
    gram_ms = sum(a.elapsed_time(b) for a, b in zip(ev["a1"], ev["g1"])) / n_inst
    # batched solve + error of all layers: from the end of the last Gram to s1
    per_step = len(groups) * cfg.n_chunks
    solve_ms = sum(ev["g1"][(i + 1) * per_step - 1].elapsed_time(ev["s1"][i])
                   for i in range(n_inst)) / n_inst
    # of which the batched error pass (one read of every layer's matrices)
    error_ms = sum(a.elapsed_time(b) for a, b in zip(ev["e0"], ev["s1"])) / n_inst
    # the attention calls alone, with the layers in flight on the step's streams
    # (the concurrency the timed step runs them at; no Gram, solve or error)
    def attention_pass():
        n_s = len(streams)
        fork = torch.cuda.Event()
        fork.record(streams[0])
        for s_ in streams[1:]:
            s_.wait_event(fork)
        for g, (l0, n) in enumerate(groups):
            for c in range(cfg.n_chunks):
                if stacked_chunks is not None:
                    runner.attention_layers(stacked_chunks[c], l0, n, stream=streams[g % n_s],
                                            slot=g % n_s)
                else:
                    runner.attention(chunks_per_layer[l0][c], stream=streams[g % n_s],
                                     slot=g % n_s)
        for s_ in streams[1:]:
            join = torch.cuda.Event()
            join.record(s_)
            streams[0].wait_event(join)

    attention_pass()
    torch.cuda.synchronize()
    a0, a1 = E(), E()
    flush.zero_()
    a0.record(streams[0])
    for _ in range(n_inst):
        attention_pass()
    a1.record(streams[0])
    torch.cuda.synchronize()
    attn_streams_ms = a0.elapsed_time(a1) / n_inst
    status = ispa.read_status(runner.status)
    step_ms_max = max_over_ranks(step_ms, world)

    work = step_work(cfg)
    total = sum(work.values())
    share = L_mine / L                 # this rank's part of the workload
    value = total * (1 if sharded else world) / (step_ms_max * 1e-3) / 1e12
    attn_tflops = work["attention"] * share / (attn_ms * 1e-3) / 1e12
    absorb_ms_layer = (gram_ms + solve_ms) / L_mine
    bf16_peak, hbm_peak, peak_src = peaks()
    attn_launches = len(groups) * cfg.n_chunks
    sm_mhz = clocks.get("sm_mhz") if clocks else None
    roofline = {
        "bound": "tensor", "kernel": "dual-stream attention (branch_attention_kernel, merge fused)",
        "achieved": round(attn_tflops, 2), "peak": bf16_peak, "unit": "TFLOP/s",
        "frac": round(attn_tflops / bf16_peak, 4), "peak_source": f"{peak_src} bf16 dense (burst)",
        "traffic": traffic_per_launch(cfg.name, group),
        "algorithmic_flops_per_launch": work["attention"] * share / attn_launches,
        "algorithmic_bytes_per_launch": attention_bytes(cfg) * L_mine / attn_launches,
        "ms_per_launch": attn_ms / attn_launches,
        "launches_per_step": attn_launches,
        # box-to-box comparable: the attention time in SM clock cycles
        "sm_mcycles_per_step": round(attn_ms * sm_mhz * 1e-3, 3) if sm_mhz else None,
    }
    absorb_flops = (work["gram"] + work["solve"]) * share
    out = {
        "metric": METRIC, "value": round(value, 3), "unit": "TFLOP/s", "n_gpus": world,
        "steps": steps, "warmup": warmup, "ms_per_step": round(step_ms_max, 4),
        "higher_is_better": True, "scaling": "strong" if sharded else "weak", "vs_baseline": None,
        "dtype": "bf16 QK^T, fp16 PV, tf32 Gram, fp32 solve",
        "data": "synthetic AR(1) rho=0.9 bf16 Q/K/V, W ~ N(0,1/d), seeded",
        "config": config_of(cfg, world, sharded, K),
        "attention_tflops": round(attn_tflops, 2),
        "attention_frac_of_bf16_peak": round(attn_tflops / bf16_peak, 4),
        "attention_ms_per_step": round(attn_ms, 4),
        # as the step runs them: layers in flight on the step's streams
        "attention_tflops_layers_in_flight": round(work["attention"] * share
                                                   / (attn_streams_ms * 1e-3) / 1e12, 2),
        "attention_frac_layers_in_flight": round(work["attention"] * share
                                                 / (attn_streams_ms * 1e-3) / 1e12 / bf16_peak, 4),
        "attention_streams": len(streams),
        "attention_layers_per_launch": group,
        "absorb_ms_per_layer": round(absorb_ms_layer, 4),
        "gram_ms_per_step": round(gram_ms, 4), "solve_error_ms_per_step": round(solve_ms, 4),
        "absorb_tflops": round(absorb_flops / ((gram_ms + solve_ms) * 1e-3) / 1e12, 2),
        "roofline": roofline,
        "absorb_roofline": absorb_roofline(cfg, gram_ms * L / L_mine, solve_ms * L / L_mine,
                                           bf16_peak, hbm_peak),
        "error_hbm": {
            "kernel": "batched layer error from W W^T (dot5_kernel + finalize)",
            "ms_per_step": round(error_ms, 4),
            "algorithmic_bytes_per_layer": error_bytes(cfg),
            "achieved": round(error_bytes(cfg) * L_mine / (error_ms * 1e-3) / 1e9, 1),
            "peak": hbm_peak, "unit": "GB/s",
            "frac": round(error_bytes(cfg) * L_mine / (error_ms * 1e-3) / 1e9 / hbm_peak, 4)},
        "gpu_launches": int(launches),
        "device_status": status,
        "clocks": clocks,
    }
    if with_e2e:
        out["e2e"] = run_e2e(args, cfg, layer_streams_, chunks_per_layer, qkv, W_all, runner,
                             err, perm, sel, K, world, err_mine if sharded else None, streams,
                             grouped=stacked_chunks is not None)
    if with_cpu and rank == 0 and world == 1:
        out["cpu_baseline"] = oracle_throughput(cfg, args.cpu_budget)
    return out


def attention_bytes(cfg):
    """Algorithmic DRAM bytes of one layer's attention over all its chunks:
    Q, K and V read once (bf16), A_loc and D written (fp32), A_full written
    (bf16), three LSE rows per head written (fp32)."""
    d = cfg.d
    total = 0.0
    for c in range(cfg.n_chunks):
        keys = cfg.sink_tokens + cfg.chunk_tokens + len(cfg.history_frames_of(c)) * cfg.tokens_per_frame
        total += (cfg.chunk_tokens + 2 * keys) * d * 2 + cfg.chunk_tokens * d * (4 + 4 + 2) \
            + 3 * cfg.heads * cfg.chunk_tokens * 4
    return total


SUB_WORKLOADS = (("14B-warmup", "c3"), ("1.3B-chunk", "c1"))
SUB_KEYS = ("value", "unit", "ms_per_step", "steps", "warmup", "config", "attention_tflops",
            "attention_frac_of_bf16_peak", "attention_ms_per_step",
            "attention_tflops_layers_in_flight", "attention_frac_layers_in_flight", "absorb_ms_per_layer",
            "gram_ms_per_step", "solve_error_ms_per_step", "absorb_tflops", "roofline",
            "absorb_roofline", "gpu_launches", "device_status", "clocks", "cpu_baseline")


def run_ours(args):
    import torch
    from kv_cache_absorption_b200 import build
    build.build()
    from ispa_synth import CONFIGS
    world, rank, local = dist_setup()
    cfg = workload(args)
    out = measure_warmup(args, cfg, world, rank, args.steps, args.warmup,
                         with_e2e=not args.no_e2e, with_cpu=not args.no_cpu_baseline)
    # the other shapes the metric is quoted on, in the same invocation
    if args.config == "c2" and args.layers is None and not args.no_sub:
        for key, name in SUB_WORKLOADS:
            torch.cuda.empty_cache()
            sub_steps = max(3, min(args.steps, 5 if name == "c3" else 50))
            sub = measure_warmup(args, CONFIGS[name], world, rank, sub_steps, args.warmup,
                                 with_e2e=False, with_cpu=not args.no_cpu_baseline)
            out[key] = {k: sub[k] for k in SUB_KEYS if k in sub}
    if rank == 0:
        print(json.dumps(out), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def run_e2e(args, cfg, streams, chunks_per_layer, qkv, W_all, runner, err, perm, sel, K, world,
            err_mine=None, cuda_streams=None, grouped=False):
    """Same step through the public API with the instance's inputs in pinned
    host memory: every step copies each layer's Q/K/V frame streams
    host->device, runs the warmup, and copies every Delta W, the errors and
    the ranking device->host. The model weights (W and W W^T) stay resident,
    as they would in a serving process. As a serving loop would, the copy of
    step i + 1's inputs (on a copy stream, into the other of two device input
    sets) overlaps step i's compute; the timed region runs from the first
    copy to the last result read back."""
    import dataclasses
    import torch
    from ispa_synth import stacked_chunk
    from kv_cache_absorption_b200.warmup import rank as rank_layers
    from kv_cache_absorption_b200.sharding import gather_errors
    # two device input sets, each the three [L, frames, ...] stream tensors;
    # the per-layer and stacked chunks are views into them
    qkv2 = tuple(torch.empty_like(x) for x in qkv)
    clones = [dataclasses.replace(st, q=qkv2[0][i], k=qkv2[1][i], v=qkv2[2][i])
              for i, st in enumerate(streams)]
    sets = []
    for ss, store in ((streams, qkv), (clones, qkv2)):
        per_layer = [[st.chunk(c) for c in range(cfg.n_chunks)] for st in ss]
        stacked = [stacked_chunk(cfg, store, c) for c in range(cfg.n_chunks)] if grouped else None
        sets.append((per_layer, stacked, store))
    dev_sets = [list(store) for _, _, store in sets]
    for per_layer, stacked, store in sets:   # every chunk input is a view into an uploaded set
        owners = {t.untyped_storage().data_ptr() for t in store}
        views = [x for layer_chunks in per_layer for ch in layer_chunks for x in ch.values()]
        views += [x for sch in (stacked or []) for x in sch.values()]
        assert all(x.numel() == 0 or x.untyped_storage().data_ptr() in owners for x in views)
    host_tensors = [t.cpu().pin_memory() for t in dev_sets[0]]
    L, d = cfg.layers, cfg.d
    dW_host = torch.empty(runner.n_layers, d, d, dtype=torch.float32).pin_memory()
    err_host = torch.empty(L, 2, dtype=torch.float64).pin_memory()
    perm_host = torch.empty(L, dtype=torch.int32).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in host_tensors)
    d2h = dW_host.numel() * 4 + err_host.numel() * 8 + perm_host.numel() * 4
    compute = torch.cuda.current_stream()
    copy = torch.cuda.Stream()
    copied = [torch.cuda.Event(), torch.cuda.Event()]
    consumed = [torch.cuda.Event(), torch.cuda.Event()]

    def upload(i):
        b = i % 2
        with torch.cuda.stream(copy):
            if i >= 2:
                copy.wait_event(consumed[b])      # step i - 2 is done with this set
            for h, dv in zip(host_tensors, dev_sets[b]):
                dv.copy_(h, non_blocking=True)
            copied[b].record(copy)

    def compute_step(i):
        b = i % 2
        compute.wait_event(copied[b])
        if grouped:
            runner.layers_chunks_stacked(sets[b][1], cuda_streams)
        else:
            runner.layers_chunks(sets[b][0], cuda_streams)
        if err_mine is not None:
            runner.absorb_all(W_all, err_mine)
            err.copy_(gather_errors(err_mine, L, world))
        else:
            runner.absorb_all(W_all, err)
        rank_layers(err, K, perm, sel)
        consumed[b].record(compute)
        dW_host.copy_(runner.dW, non_blocking=True)
        err_host.copy_(err, non_blocking=True)
        perm_host.copy_(perm, non_blocking=True)

    def run(n, t0=None, t1=None):
        if t0 is not None:
            t0.record(copy)
        upload(0)
        for i in range(n):
            if i + 1 < n:
                upload(i + 1)
            compute_step(i)
        if t1 is not None:
            t1.record(compute)

    n = max(3, min(args.steps, 30))
    run(2)
    torch.cuda.synchronize()
    barrier(world)
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    run(n, s, e)
    torch.cuda.synchronize()
    ms = max_over_ranks(s.elapsed_time(e) / n, world)
    total = sum(step_work(cfg).values())
    reps = 1 if err_mine is not None else world
    return {"value": round(total * reps / (ms * 1e-3) / 1e12, 3), "unit": "TFLOP/s",
            "ms_per_step": round(ms, 4), "steps": n, "h2d_bytes_per_step": int(h2d),
            "d2h_bytes_per_step": int(d2h),
            "pipelining": "step i+1's host->device copy overlaps step i's compute"}


# ---------------------------------------------------------------- streaming (after the transition)

STREAM_METRIC = "post-transition streaming tokens/s (all layers) and KV bytes, ISPA vs all-F-Layer"


def run_streaming(args):
    """One step = one post-transition stream: every streaming chunk through
    every layer (F-Layers: full attention over the growing history, then W;
    L-Layers: sink + chunk attention, then W + Delta W). The warmup, the
    batched absorb, the ranking and the transition run once, untimed. The
    same stream with every layer kept full is timed alongside."""
    import torch
    from kv_cache_absorption_b200 import build
    build.build()
    from kv_cache_absorption_b200 import ispa
    from kv_cache_absorption_b200.warmup import LayerWarmup, rank as rank_layers
    from kv_cache_absorption_b200.streaming import KVCache, StreamingLayers, kv_cache_bytes

    world, rank, local = dist_setup()
    dev = torch.device("cuda", torch.cuda.current_device())
    cfg = workload(args)
    if cfg.stream_chunks < 1:
        raise SystemExit("the streaming benchmark needs a workload with streaming chunks (c4)")
    streams, warm_chunks, W_all, _ = make_inputs(cfg, rank, dev)
    L = cfg.layers
    K = cfg.select_k if cfg.select_k is not None else L // 2
    # warmup and transition
    warm_hist = max(len(cfg.history_frames_of(c)) for c in range(cfg.n_chunks)) * cfg.tokens_per_frame
    runner = LayerWarmup(cfg.heads, cfg.head_dim, cfg.chunk_tokens, cfg.sink_tokens,
                         cfg.chunk_tokens, warm_hist, n_layers=L, device=dev)
    runner.weight_gram(W_all)
    for li, chunks in enumerate(warm_chunks):
        for c, ch in enumerate(chunks):
            runner.chunk(ch, first=(c == 0), layer=li)
    err = torch.empty(L, 2, dtype=torch.float64, device=dev)
    perm = torch.empty(L, dtype=torch.int32, device=dev)
    sel = torch.empty(L, dtype=torch.uint8, device=dev)
    runner.absorb_all(W_all, err)
    rank_layers(err, K, perm, sel)
    c_first, c_last = cfg.n_chunks, cfg.n_chunks + cfg.stream_chunks - 1
    hist_last = len(cfg.history_frames_of(c_last)) * cfg.tokens_per_frame
    sl = StreamingLayers(cfg.heads, cfg.head_dim, cfg.chunk_tokens, cfg.sink_tokens,
                         cfg.chunk_tokens, hist_last, n_layers=L, device=dev)
    sl.transition(W_all, runner.dW, sel.cpu().bool())
    sl.quantize_weights(W_all, runner.dW)
    torch.cuda.synchronize()
    status = ispa.read_status(runner.status)
    del runner, warm_chunks
    torch.cuda.empty_cache()
    # per layer and streaming chunk: the new query rows and the chunk's keys
    # and values, which each step appends to the layer's KV cache
    new_rows = []
    for st in streams:
        rows = []
        for c in range(c_first, c_last + 1):
            ch = st.chunk(c)
            rows.append((ch["q"], ch["k_loc"], ch["v_loc"]))
        new_rows.append(rows)
    local_sel = sel.cpu().bool()

    def caches(all_full):
        """The layers' KV caches at the transition: an F-Layer's holds the
        sink and the history so far, with room for the rest of the stream; an
        L-Layer's only the sink and one chunk."""
        out = []
        for l, st in enumerate(streams):
            full = all_full or not bool(local_sel[l])
            kc = KVCache(cfg.heads, cfg.head_dim, cfg.sink_tokens, cfg.chunk_tokens,
                         hist_last, full, device=dev)
            ch = st.chunk(c_first)
            kc.set_sink(ch["k_sink"], ch["v_sink"])
            if full:
                kc.set_history(ch["k_hist"], ch["v_hist"])
            out.append(kc)
        return out

    kv_ispa_c, kv_full_c = caches(False), caches(True)
    torch.cuda.synchronize()
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)

    def one_pass(kv, all_full, w8a8=False):
        for kc in kv:
            kc.rewind()
        for j in range(cfg.stream_chunks):
            for l in range(L):
                q, k, v = new_rows[l][j]
                kv[l].append(k, v)
                sl.layer(l, kv[l].chunk_inputs(q), local=False if all_full else None, w8a8=w8a8)

    def timed(all_full, w8a8=False):
        kv = kv_full_c if all_full else kv_ispa_c
        for _ in range(args.warmup):
            one_pass(kv, all_full, w8a8)
        torch.cuda.synchronize()
        barrier(world)
        ms = []
        for _ in range(args.steps):
            flush.zero_()
            s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            s0.record()
            one_pass(kv, all_full, w8a8)
            s1.record()
            torch.cuda.synchronize()
            ms.append(s0.elapsed_time(s1))
        return max_over_ranks(sum(ms) / len(ms), world)

    bus = torch.cuda.get_device_properties(dev)
    bus_id = f"{getattr(bus, 'pci_domain_id', 0):08x}:{getattr(bus, 'pci_bus_id', 0):02x}:" \
             f"{getattr(bus, 'pci_device_id', 0):02x}.0"
    sampler = ClockSampler(bus_id)
    time.sleep(0.15)
    launches0 = ispa.ispa_kernel_launches()
    ms_ispa = timed(False)
    launches = (ispa.ispa_kernel_launches() - launches0) // (args.warmup + args.steps)
    ms_full = timed(True)
    ms_w8a8 = timed(False, True)
    clocks = sampler.stop()
    status |= ispa.read_status(sl.status)
    n_local = int(sel.sum().item())
    tokens = cfg.stream_chunks * cfg.chunk_tokens
    d = cfg.d
    f_flops = 0.0
    for c in range(c_first, c_last + 1):
        nk = cfg.sink_tokens + cfg.chunk_tokens + len(cfg.history_frames_of(c)) * cfg.tokens_per_frame
        f_flops += 4.0 * cfg.chunk_tokens * nk * d
    kv_all = kv_cache_bytes(L, 0, cfg.sink_tokens, hist_last, cfg.chunk_tokens, d)
    kv_ispa = kv_cache_bytes(L - n_local, n_local, cfg.sink_tokens, hist_last, cfg.chunk_tokens, d)
    kv_alloc = {"ispa": sum(kc.nbytes for kc in kv_ispa_c), "all_f": sum(kc.nbytes for kc in kv_full_c)}
    bf16_peak, _, peak_src = peaks()
    out = {
        "metric": STREAM_METRIC, "value": round(tokens * world / (ms_ispa * 1e-3), 1),
        "unit": "tokens/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(ms_ispa, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16 QK^T, fp16 PV, bf16 projection",
        "data": "synthetic AR(1) rho=0.9 bf16 Q/K/V, W ~ N(0,1/d), seeded",
        "config": {"workload": cfg.name, "layers": L, "local_layers": n_local, "heads": cfg.heads,
                   "head_dim": cfg.head_dim, "d": d, "stream_chunks": cfg.stream_chunks,
                   "chunk_rows": cfg.chunk_tokens, "sink": cfg.sink_tokens,
                   "history": [len(cfg.history_frames_of(c_first)) * cfg.tokens_per_frame,
                               hist_last],
                   "l2": "flushed (512 MB write) before every timed step",
                   "selection": "K lowest-error layers of this instance's warmup"},
        "all_f_tokens_per_s": round(tokens * world / (ms_full * 1e-3), 1),
        "all_f_ms_per_step": round(ms_full, 3),
        "speedup_vs_all_f": round(ms_full / ms_ispa, 3),
        "ispa_w8a8_tokens_per_s": round(tokens * world / (ms_w8a8 * 1e-3), 1),
        "ispa_w8a8_speedup_vs_all_f": round(ms_full / ms_w8a8, 3),
        "kv_bytes_last_chunk": {"ispa": kv_ispa, "all_f": kv_all,
                                "saved_frac": round(1 - kv_ispa / kv_all, 4)},
        "kv_cache_bytes_allocated": kv_alloc,
        "f_layer_attention_tflops_all_f": round(f_flops * L / (ms_full * 1e-3) / 1e12, 2),
        "attention_frac_of_bf16_peak_all_f": round(f_flops * L / (ms_full * 1e-3) / 1e12 / bf16_peak, 4),
        "peak_source": f"{peak_src} bf16 dense (burst)",
        "gpu_launches": int(launches), "device_status": status, "clocks": clocks,
    }
    if rank == 0:
        print(json.dumps(out), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


# ---------------------------------------------------------------- reference arm

def oracle_streaming_timing(cfg, rows: int = 64, seed: int = 0):
    """The float64 oracle on a bounded sample of the streaming step: one
    F-Layer and one L-Layer on ``rows`` query rows of the first and the last
    streaming chunk for one head (all keys, the projection of that head's
    columns). Returns {kind: [seconds, flops]}."""
    import oracle
    from ispa_synth import layer_streams
    key = ("stream", cfg.name, seed)
    if key not in _ORACLE_INPUTS:      # inputs widened to float64 once, outside the timing
        st = layer_streams(cfg, 0, seed=seed)
        c0, c1 = cfg.n_chunks, cfg.n_chunks + cfg.stream_chunks - 1
        chunks = [{k: oracle.as_f64(v)[:, :1] for k, v in st.chunk(c).items()} for c in (c0, c1)]
        _ORACLE_INPUTS[key] = (chunks, oracle.as_f64(st.w)[:cfg.head_dim])
    chunks, w = _ORACLE_INPUTS[key]
    hd, d = cfg.head_dim, cfg.d
    t = {"F": [0.0, 0.0], "L": [0.0, 0.0]}
    for ch in chunks:
        nk = ch["k_sink"].shape[0] + ch["k_loc"].shape[0] + ch["k_hist"].shape[0]
        nl = ch["k_sink"].shape[0] + ch["k_loc"].shape[0]
        for kind, local, n in (("F", False, nk), ("L", True, nl)):
            t0 = time.perf_counter()
            oracle.streaming_layer(ch["q"][:rows], ch["k_sink"], ch["v_sink"], ch["k_loc"],
                                   ch["v_loc"], ch["k_hist"], ch["v_hist"], w, None, local=local)
            t[kind][0] += time.perf_counter() - t0
            t[kind][1] += rows * (4.0 * n * hd + 2.0 * hd * d)
    return t


def run_reference_streaming(args, cfg, world):
    """Oracle throughput of the streaming step, tokens/s, extrapolated from
    the sampled rows by each layer kind's work (attention over its keys and
    the projection) over every streaming chunk."""
    d = cfg.d
    K = cfg.select_k if cfg.select_k is not None else cfg.layers // 2
    work = {"F": 0.0, "L": 0.0}
    for c in range(cfg.n_chunks, cfg.n_chunks + cfg.stream_chunks):
        nk = cfg.sink_tokens + cfg.chunk_tokens + len(cfg.history_frames_of(c)) * cfg.tokens_per_frame
        nl = cfg.sink_tokens + cfg.chunk_tokens
        work["F"] += (cfg.layers - K) * cfg.chunk_tokens * (4.0 * nk * d + 2.0 * d * d)
        work["L"] += K * cfg.chunk_tokens * (4.0 * nl * d + 2.0 * d * d)
    rows = 64
    acc = {"F": [0.0, 0.0], "L": [0.0, 0.0]}
    for i in range(args.warmup + args.steps):
        t = oracle_streaming_timing(cfg, rows)
        if i >= args.warmup:
            for k in acc:
                acc[k][0] += t[k][0]
                acc[k][1] += t[k][1]
    secs = sum(work[k] * acc[k][0] / acc[k][1] for k in work)
    tokens = cfg.stream_chunks * cfg.chunk_tokens
    value = tokens / secs
    cores, blas = cpu_cores()
    sample = (f"per step: float64 oracle on {rows} query rows of the first and the last "
              f"streaming chunk for one head through one F-Layer and one L-Layer (all keys, "
              f"projection); extrapolated by each layer kind's work to the whole stream")
    print(json.dumps({
        "impl": "reference", "metric": STREAM_METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": secs * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": {"workload": cfg.name, "d": d, "layers": cfg.layers,
                                        "local_layers": K},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": blas or cores,
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0}}), flush=True)


def run_reference(args):
    """The float64 oracle on the host cores. Each step times one bounded
    sample of the workload (``ms_per_step`` is that sample's wall time); the
    reported rate is the stage-weighted extrapolation of the sampled rates to
    the full step (its duration in ``full_step_s_extrapolated``)."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    cfg = workload(args)
    if cfg.stream_chunks > 0:
        run_reference_streaming(args, cfg, world)
        return
    work = step_work(cfg)
    total = sum(work.values())
    acc = {s: [0.0, 0.0] for s in work}
    wall = []
    for i in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        timing = oracle_timing(cfg)
        if i >= args.warmup:
            wall.append(time.perf_counter() - t0)
            for s in acc:
                acc[s][0] += timing[s][0]
                acc[s][1] += timing[s][1]
    stages = {s: work[s] * acc[s][1] / acc[s][0] for s in work if acc[s][0] > 0 and work[s] > 0}
    t_full = sum(stages.values())
    value = total / t_full / 1e12
    cores, blas = cpu_cores()
    sample = (f"per step: float64 oracle on 256 query rows of the last chunk for one head (all "
              f"keys), the Gram and direct error of 1024 rows, one full {cfg.d}x{cfg.d} solve; "
              f"rates extrapolated stage by stage to the full step")
    K = cfg.select_k if cfg.select_k is not None else cfg.layers // 2
    out = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
           "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
           "ms_per_step": sum(wall) / len(wall) * 1e3, "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
           "config": config_of(cfg, 1, False, K),
           "step_is": "a bounded sample of the workload (see cpu_baseline.sample)",
           "full_step_s_extrapolated": round(t_full, 3),
           "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": blas or cores,
                            "host_cores": cores, "blas_threads": blas,
                            "stage_seconds_per_full_step": {k: round(t, 3)
                                                            for k, t in stages.items()},
                            "kind": "oracle", "sample": sample},
           "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                   "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--config", choices=("c1", "c2", "c3", "c4"), default="c2")
    ap.add_argument("--layers", type=int, default=None,
                    help="override the workload's layer count (smaller captures for ncu)")
    ap.add_argument("--slots", type=int, default=2,
                    help="layers in flight on separate streams in a multi-layer warmup")
    ap.add_argument("--group", type=int, default=10,
                    help="layers per attention launch in the warmups (1: one launch per layer)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-sub", action="store_true",
                    help="measure only the main workload (no 14B / single-chunk sub-objects)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=20.0)
    ap.add_argument("--measure-tf32-peak", action="store_true",
                    help="time a cuBLAS tf32 GEMM (the absorb roofline's tf32 rate) and exit")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.measure_tf32_peak:
        measure_tf32_peak()
        return
    if args.impl == "reference":
        run_reference(args)
    elif args.config == "c4":
        run_streaming(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
