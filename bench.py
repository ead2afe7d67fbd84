"""Benchmark of the routed block-sparse attention path on B200.

One step = one pass of the whole hot path over one layer of the chunk-48
workload (40 heads, 48 query blocks, 2256 history blocks of 128 tokens,
head_dim 128, bf16): Gilbert order + neighbour table, block importance, soft
fusion and route build, routed attention.  Inputs are resident in HBM and
larger than L2 (K + V = 5.9 GB), so no L2 flush is needed between steps.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl velox|reference]

Prints one JSON line.  value = routed-attention FLOPs of the step (4 b^2 d per
routed tile, from the actual route lengths) over the step time, summed over
ranks (weak scaling: every rank runs its own layer; there is no data-path
collective).  Per-call times, the roofline of the attention kernel, an
end-to-end number through host buffers and the CPU oracle baseline are added.
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "routed attn µs/call & TFLOP/s at chunk-48 shape; % of B200 bf16 peak"
UNIT = "TFLOP/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
LAUNCHES_PER_STEP = 7  # neighbours, pool, logits, softmax, route, schedule, attention


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled while the timed region runs."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self._t = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self._t = threading.Thread(target=self._read, daemon=True)
            self._t.start()
        except Exception:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            if self._t:
                self._t.join(timeout=2)

    def summary(self):
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
            except ValueError:
                continue
            for nm, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


def _dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def _barrier(world):
    if world > 1:
        torch.distributed.barrier()


def _max_over_ranks(x: float, world: int, device="cuda") -> float:
    if world == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def _sum_over_ranks(x: float, world: int, device="cuda") -> float:
    if world == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.SUM)
    return float(t.item())


def rank_workload(rank: int, heads: int = 0):
    """Weak scaling: rank r runs layer r of the chunk-48 workload (its own
    seeds); the path has no exchange between ranks."""
    from synth import config
    wl = config(3, layer=rank)
    if heads:
        # reduced head count: only for small profiler captures, never a bench value
        from dataclasses import replace
        wl = replace(wl, heads=heads)
    return wl


def aggregate(flops_step: float, ms_step: float, world: int, device="cuda"):
    """Whole-job throughput: FLOPs of all ranks over the slowest rank's step."""
    ms = _max_over_ranks(ms_step, world, device)
    flops = _sum_over_ranks(flops_step, world, device)
    return flops / (ms * 1e-3) / 1e12, ms


# ---------------------------------------------------------------- oracle ---
def cpu_oracle_sample(inp, attn_rows: int = 48, heads=tuple(range(12)), step_heads=None,
                      cache=None):
    """Time the oracle on a bounded sample of one step and scale to a step.

    Sample: the neighbour table, then for each head of `heads` its importance
    (all N x M blocks), the routes of its N rows and attention of the first
    `attn_rows` of them.  The step estimate multiplies each part by its share
    of the full step (`step_heads` heads, default the workload's, and their
    rows).  The default (12 whole heads of the chunk-48 layer) is 10-20 s of
    CPU work.  Only the oracle calls are timed, after one untimed warm-up
    call of the attention oracle: each head's fp64 host copy
    is made before its timed spans, kept in `cache` when one is given and
    dropped after use otherwise, so host memory holds one head at a time.
    """
    from oracle import attention as oatt
    from oracle import gilbert as ogil
    from oracle import importance as oimp
    from oracle import route as ort
    from threadpoolctl import threadpool_info

    wl = inp.wl
    H, N, M, b = wl.heads, wl.n_q_blocks, wl.n_kv_blocks, wl.b
    if step_heads is not None:
        H = step_heads
    prm = ort.Params(lam=wl.params.lam, tau=wl.params.tau, g_ref=wl.params.g_ref,
                     theta_cov=wl.params.theta_cov, theta_unc=wl.params.theta_unc,
                     k_cov=wl.params.k_cov, k_unc=wl.params.k_unc)

    def host(h):
        if cache is not None and h in cache:
            return cache[h]
        qkv = tuple(x[h].to(torch.float64).cpu().numpy() for x in (inp.Q, inp.K, inp.V))
        if cache is not None:
            cache[h] = qkv
        return qkv

    g = inp.g.cpu().numpy()
    cov = inp.covered.cpu().numpy()
    T, Hl, Wl = wl.lattice
    t0 = time.perf_counter()
    nbr = ogil.neighbour_blocks(T, Hl, Wl, wl.n_chunks, b, wl.q_chunk, wl.cache_first_block, M)
    t_nbr = time.perf_counter() - t0
    t_imp = t_route = t_attn = 0.0
    lens = []
    rows = min(attn_rows, N)
    for k, h in enumerate(heads):
        Qh, Kh, Vh = host(h)
        if k == 0:  # untimed: the BLAS thread pool and first allocations start up here
            oatt.routed_attention_block(Qh[:b], Kh, Vh, list(range(0, M, max(1, M // 150))), b)
        t0 = time.perf_counter()
        p = oimp.importance(Qh, Kh, b, 1.0).astype(np.float32)
        t1 = time.perf_counter()
        routes = [ort.route_row(p[i], g[i], bool(cov[i]), prm, wl.prev_begin, wl.prev_count,
                                nbr[i]) for i in range(N)]
        t2 = time.perf_counter()
        for i in range(rows):
            oatt.routed_attention_block(Qh[i * b:(i + 1) * b], Kh, Vh,
                                        routes[i][0] + routes[i][1], b)
        t3 = time.perf_counter()
        t_imp += t1 - t0
        t_route += t2 - t1
        t_attn += t3 - t2
        lens += [len(r[0]) + len(r[1]) for r in routes]
        del Qh, Kh, Vh
    nh = len(heads)
    step_s = t_nbr + (H / nh) * (t_imp + t_route) + (H * N / (nh * rows)) * t_attn
    threads = [x.get("num_threads", 1) for x in threadpool_info()
               if x.get("user_api") == "blas"]
    return {"step_s": step_s, "sample_s": t_nbr + t_imp + t_route + t_attn,
            "threads": max(threads) if threads else 1, "mean_len": float(np.mean(lens)),
            "sample": (f"Gilbert neighbour table; for each of {nh} heads: importance "
                       f"({N}x{M} blocks), routes of its {N} rows, attention of {rows} rows; "
                       f"scaled to a step of {H} heads and {H * N} rows")}


def run_reference(args, world, rank):
    """--impl reference: the CPU oracle, on the host cores, rank 0 only."""
    if rank != 0:
        return
    import dataclasses
    from synth import config, make_inputs
    wl = config(3)
    # the sample works on one head: draw a one-head layer of the same shape
    # and distributions (drawing all 40 heads on the CPU would take minutes)
    inp = make_inputs(dataclasses.replace(wl, heads=1), "cpu")
    # FLOPs of the step: mean route length of the sampled head's oracle routes
    times, flops_step = [], None
    cache = {}
    for s in range(args.warmup + args.steps):
        r = cpu_oracle_sample(inp, attn_rows=8, heads=(0,), step_heads=wl.heads, cache=cache)
        if s >= args.warmup:
            times.append(r["step_s"])
        if flops_step is None:
            flops_step = 4.0 * 128 ** 3 * wl.heads * wl.n_q_blocks * r["mean_len"]
    mean_s = sum(times) / len(times)
    value = flops_step / mean_s / 1e12
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": mean_s * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": {"workload": "chunk48 (H=40, N=48, M=2256, d=128, b_tok=128)"},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": r["threads"],
                             "kind": "oracle", "sample": r["sample"]},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- velox ---
def run_velox(args, world, rank, local):
    import routed_block_sparse_b200 as rbs
    from routed_block_sparse_b200.pipeline import layer_for
    from synth import make_inputs

    dev = torch.device("cuda", local if world > 1 else 0)
    wl = rank_workload(rank, args.heads)
    inp = make_inputs(wl, dev)
    layer = layer_for(wl, device=dev)
    H, N, M, b, d = wl.heads, wl.n_q_blocks, wl.n_kv_blocks, wl.b, wl.d
    T, Hl, Wl = wl.lattice
    stream = torch.cuda.current_stream(dev)

    def step(ev=None, st=None):
        st = stream if st is None else st
        if ev is not None:
            ev[0].record(st)
        rbs.velox_gilbert_order(T, Hl, Wl, wl.n_chunks, b, wl.q_chunk, wl.cache_first_block, M,
                                nbr_ids=layer.nbr_ids, nbr_cnt=layer.nbr_cnt,
                                S_max=layer.S_max, dev_status=layer.dev_status, stream=st)
        if ev is not None:
            ev[1].record(st)
        layer.importance(inp.Q, inp.K, st)
        if ev is not None:
            ev[2].record(st)
        layer.route(inp.g, inp.covered, stream=st)
        if ev is not None:
            ev[3].record(st)
        layer.attend(inp.Q, inp.K, inp.V, stream=st)
        if ev is not None:
            ev[4].record(st)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    status = layer.status()
    route_len = layer.route_len.to(torch.float64)
    tiles = float(route_len.sum().item())
    flops_step = 4.0 * b * b * d * tiles
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    _barrier(world)
    torch.cuda.synchronize(dev)
    with ClockSampler(dev.index or 0) as clocks:
        t_start.record(stream)
        for k in range(args.steps):
            step(evs[k])
        t_end.record(stream)
        torch.cuda.synchronize(dev)
    _barrier(world)
    torch.cuda.synchronize(dev)
    total_ms = t_start.elapsed_time(t_end)
    parts = np.array([[e[j].elapsed_time(e[j + 1]) for j in range(4)] for e in evs])
    gil_ms, imp_ms, route_ms, attn_ms = parts.mean(axis=0)
    value, ms_step = aggregate(flops_step, total_ms / args.steps, world)

    peaks, peak_kind = _peaks()
    attn_tflops = flops_step / (attn_ms * 1e-3) / 1e12
    imp_bytes = H * N * b * d * 2 + H * M * b * d * 2 + H * N * M * 4
    route_bytes = (H * N * M * 4 + N * M * 4 + N + N * layer.S_max * 4 + N * 4
                   + H * N * layer.R_max * 4 + 2 * H * N * 4)
    imp_gbs = imp_bytes / (imp_ms * 1e-3) / 1e9
    ir_gbs = (imp_bytes + route_bytes) / ((imp_ms + route_ms) * 1e-3) / 1e9
    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    bf16 = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    bf16_sus = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
    traffic = None
    tpath = os.path.join(ROOT, "profiles", "attn_traffic.json")
    if os.path.exists(tpath):
        try:
            with open(tpath) as f:
                tj = json.load(f)
            if tj.get("kernel_source_hash") == _attn_source_hash():
                # recorded for a launch of tj["heads"] heads; every head has
                # the same route statistics and its own K/V
                traffic = tj["bytes_per_launch"] * wl.heads / tj.get("heads", wl.heads)
        except Exception:
            traffic = None

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) bf16 Q/K/V; g U[0,1] half zeroed; coverage Bernoulli 0.5)",
        "config": {"workload": "chunk48" if H == 40 else f"chunk48 reduced to {H} heads",
                   "heads": H, "n_q_blocks": N, "n_kv_blocks": M,
                   "head_dim": d, "b_tok": b, "k_cov": wl.params.k_cov, "k_unc": wl.params.k_unc,
                   "theta": wl.params.theta_unc, "lattice": [T, Hl, Wl],
                   "l2": "inputs larger than L2 (K+V 5.9 GB per layer), no flush"},
        "attn_us": attn_ms * 1e3, "attn_tflops": attn_tflops,
        "importance_us": imp_ms * 1e3, "importance_gbs": imp_gbs,
        "route_us": route_ms * 1e3, "gilbert_us": gil_ms * 1e3,
        "importance_route_gbs": ir_gbs, "importance_route_hbm_frac": ir_gbs / hbm,
        "routed_tiles": tiles, "mean_route_len": tiles / (H * N), "dev_status": status,
        # the attention kernel is timed inside a ~1 s loop of back-to-back steps
        # that runs under the 1 kW power cap (see "clocks"), so its denominator
        # is the measured sustained bf16 figure; the burst fraction is reported too
        "roofline": {"bound": "tensor", "achieved": attn_tflops, "peak": bf16_sus,
                     "unit": "TFLOP/s", "frac": attn_tflops / bf16_sus, "traffic": traffic,
                     "peak_source": f"{peak_kind} bf16 dense, sustained under the power cap",
                     "frac_of_burst_peak": attn_tflops / bf16, "burst_peak": bf16},
        "gpu_launches": LAUNCHES_PER_STEP * args.steps,
        "clocks": clocks.summary(),
    }

    # the same step captured once as a CUDA graph and replayed (the seven
    # launches go out as one graph launch); reported beside the eager timing
    line["graph"] = _graph_replay(step, args.steps, dev)

    # end to end through the public API with host buffers
    if args.e2e_steps > 0:
        line["e2e"] = _e2e(args, wl, inp, layer, dev, stream, flops_step, world)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        r = cpu_oracle_sample(inp)
        line["cpu_baseline"] = {"value": flops_step / r["step_s"] / 1e12, "unit": UNIT,
                                "cores": r["threads"], "kind": "oracle", "sample": r["sample"],
                                "sample_seconds": r["sample_s"]}
    if rank == 0:
        print(json.dumps(line), flush=True)


def _graph_replay(step, steps, dev):
    try:
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            step(st=torch.cuda.current_stream(dev))
        for _ in range(3):
            graph.replay()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize(dev)
        a.record()
        for _ in range(steps):
            graph.replay()
        b.record()
        torch.cuda.synchronize(dev)
        ms = a.elapsed_time(b) / steps
        del graph
        return {"ms_per_step": ms, "steps": steps}
    except Exception as e:  # reported, not fatal: the eager numbers stand alone
        return {"error": str(e)[:200]}


def _e2e(args, wl, inp, layer, dev, stream, flops_step, world):
    """Per step: pinned host -> device copy of Q, K, V, g, covered; the four
    calls; device -> host copy of O and lse.  Timed with CUDA events."""
    host = {k: getattr(inp, k).cpu().pin_memory() for k in ("Q", "K", "V", "g", "covered")}
    out_O = torch.empty_like(layer.O, device="cpu").pin_memory()
    out_lse = torch.empty_like(layer.lse, device="cpu").pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = out_O.numel() * out_O.element_size() + out_lse.numel() * out_lse.element_size()
    T, Hl, Wl = wl.lattice
    import routed_block_sparse_b200 as rbs

    def one():
        for k, t in host.items():
            getattr(inp, k).copy_(t, non_blocking=True)
        rbs.velox_gilbert_order(T, Hl, Wl, wl.n_chunks, wl.b, wl.q_chunk, wl.cache_first_block,
                                wl.n_kv_blocks, nbr_ids=layer.nbr_ids, nbr_cnt=layer.nbr_cnt,
                                S_max=layer.S_max, dev_status=layer.dev_status, stream=stream)
        layer.forward(inp.Q, inp.K, inp.V, inp.g, inp.covered, stream)
        out_O.copy_(layer.O, non_blocking=True)
        out_lse.copy_(layer.lse, non_blocking=True)

    one()
    torch.cuda.synchronize(dev)
    a = torch.cuda.Event(enable_timing=True)
    z = torch.cuda.Event(enable_timing=True)
    _barrier(world)
    a.record(stream)
    for _ in range(args.e2e_steps):
        one()
    z.record(stream)
    torch.cuda.synchronize(dev)
    ms = _max_over_ranks(a.elapsed_time(z) / args.e2e_steps, world)
    val = _sum_over_ranks(flops_step, world) / (ms * 1e-3) / 1e12
    return {"value": val, "unit": UNIT, "ms_per_step": ms, "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h}


def run_sweep(args):
    """History-length sweep (chunk-48 per-chunk shape, M cache blocks): the
    routed path and the library's own dense kernel over the same cache, one
    JSON line per M.  Not the bench line; for the scaling table."""
    from routed_block_sparse_b200.pipeline import layer_for
    from synth import make_inputs, sweep_workload
    from synth.configs import SWEEP_M

    for M in SWEEP_M:
        wl = sweep_workload(M)
        inp = make_inputs(wl, "cuda")
        layer = layer_for(wl)
        layer.forward(inp.Q, inp.K, inp.V, inp.g, inp.covered)
        torch.cuda.synchronize()
        tiles = float(layer.route_len.sum().item())
        out = {"sweep_M": M, "mean_route_len": tiles / (wl.heads * wl.n_q_blocks)}
        for mode in ("routed", "dense"):
            n_t = tiles if mode == "routed" else float(wl.heads * wl.n_q_blocks * M)
            for _ in range(3):
                layer.attend(inp.Q, inp.K, inp.V, dense=(mode == "dense"))
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            reps = 20
            a.record()
            for _ in range(reps):
                layer.attend(inp.Q, inp.K, inp.V, dense=(mode == "dense"))
            b.record()
            torch.cuda.synchronize()
            ms = a.elapsed_time(b) / reps
            out[f"{mode}_us"] = ms * 1e3
            out[f"{mode}_tflops"] = 4.0 * 128 ** 3 * n_t / (ms * 1e-3) / 1e12
        out["speedup_routed_vs_dense"] = out["dense_us"] / out["routed_us"]
        print(json.dumps(out), flush=True)
        del inp, layer
        torch.cuda.empty_cache()


def _time_us(fn, reps=50, warm=3):
    for _ in range(warm):
        fn()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(reps):
        fn()
    b.record()
    torch.cuda.synchronize()
    return a.elapsed_time(b) / reps * 1e3


def run_geometry(args):
    """The geometry chain at the chunk-48 shape, one JSON line of per-call
    times (not the bench line): slab table of the 2256 history blocks (188
    frames of 32 x 48 tokens, 2 x 2 depth samples per token), multiwarp depth
    of the 4 current frames from the first and last frames of the 30 most
    recent chunks, the current chunk's 48 query slabs and tokens, slab
    overlap g (8^3 samples per pair) and coverage rho."""
    import numpy as np
    import routed_block_sparse_b200 as rbs
    from synth.depth import make_rollout

    T, H, W, b, nc, s = 4, 32, 48, 128, 48, 2
    q_chunk = nc - 1
    per_chunk = T * H * W // b
    M, N = q_chunk * per_chunk, per_chunk
    hist_frames = q_chunk * T
    roll = make_rollout(20261203, nc * T, H, W, s)
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    cams = dev(roll.cams)
    n_cam = cams.shape[0]
    depth, conf, mask = dev(roll.depth[:hist_frames]), dev(roll.conf[:hist_frames]), \
        dev(roll.mask[:hist_frames])
    cell = torch.empty(nc * T * H * W, dtype=torch.int32, device="cuda")
    rbs.velox_gilbert_order(T, H, W, nc, b, cell_of_rank=cell)
    src = []
    for c in range(q_chunk - 1, q_chunk - 31, -1):          # 30 most recent chunks
        src += [c * T + T - 1, c * T]                        # last, first frame
    src_depth = dev(roll.depth[src])
    src_cam = torch.tensor(src, dtype=torch.int32, device="cuda")
    tgt_cam = torch.arange(hist_frames, hist_frames + T, dtype=torch.int32, device="cuda")
    hs = torch.empty(M, 8, dtype=torch.int32, device="cuda")
    qs = torch.empty(N, 8, dtype=torch.int32, device="cuda")
    zq = torch.empty(T, H, W, device="cuda")
    uvz = torch.empty(N, b, 3, device="cuda")
    g = torch.empty(N, M, device="cuda")
    rho = torch.empty(N, device="cuda")
    cov = torch.empty(N, dtype=torch.uint8, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    mw_ws = torch.empty(rbs.velox_multiwarp_workspace_size(len(src), T, H, W), dtype=torch.uint8,
                        device="cuda")

    def table():
        rbs.velox_slab_table(depth, conf, mask, hist_frames, 0, H, W, s, cell, cell.numel(), b, 0,
                             M, 0.5, 16, 0.1, 0.9, hs, st)

    def warp():
        rbs.velox_multiwarp(cams, n_cam, src_depth, src_cam, len(src), tgt_cam, T, H, W, s, 2, zq,
                            mw_ws, st)

    def qtable():
        rbs.velox_slab_table(zq, None, None, T, hist_frames, H, W, 1, cell, cell.numel(), b,
                             q_chunk * per_chunk, N, 0.5, 8, 0.1, 0.9, qs, st, token_uvz=uvz)

    def overlap():
        rbs.velox_slab_overlap(cams, n_cam, qs, N, hs, M, 8, g, st)

    def coverage():
        rbs.velox_coverage(cams, n_cam, qs, uvz, N, b, hs, M, 0.9, rho, cov, st)

    out = {"geometry": "chunk48", "N": N, "M": M, "grid": 8, "b": b, "depth_samples": s,
           "multiwarp_sources": len(src)}
    for name, fn in (("slab_table", table), ("multiwarp", warp), ("query_slabs", qtable),
                     ("slab_overlap", overlap), ("coverage", coverage)):
        out[name + "_us"] = _time_us(fn)

    def chain():
        table(); warp(); qtable(); overlap(); coverage()
    out["chain_us"] = _time_us(chain, reps=20)
    torch.cuda.synchronize()
    out.update({"valid_history_slabs": int(hs[:, 7].sum().item()),
                "query_holes": float((zq == 0).float().mean().item()),
                "nonzero_pairs": int((g > 0).sum().item()),
                "covered_blocks": int(cov.sum().item()), "dev_status": int(st.item())})
    print(json.dumps(out), flush=True)


def run_two_phase(args):
    """Routed history tiles plus the 48 blocks of the current chunk (chunk-48
    shape): the one-pass two-phase kernel against the history-only routed
    call.  One JSON line.  Not the bench line."""
    import routed_block_sparse_b200 as rbs
    from routed_block_sparse_b200.pipeline import layer_for
    from synth import config, make_current, make_inputs

    wl = config(3, 0)
    inp = make_inputs(wl, "cuda")
    Kc, Vc = make_current(wl, "cuda")
    layer = layer_for(wl)
    layer.forward(inp.Q, inp.K, inp.V, inp.g, inp.covered)
    torch.cuda.synchronize()
    H, N, M = wl.heads, wl.n_q_blocks, wl.n_kv_blocks
    hist = float(layer.route_len.sum().item())
    t_r = _time_us(lambda: layer.attend(inp.Q, inp.K, inp.V), reps=20)

    def two():
        rbs.velox_two_phase_attn(inp.Q, inp.K, inp.V, layer.route_ids, layer.route_len,
                                 layer.R_max, Kc, Vc, N, H, N, M, 128, 128, layer.softmax_scale,
                                 layer.O, layer.lse, layer.dev_status, row_order=layer.row_order)
    t_2 = _time_us(two, reps=20)
    tiles = hist + H * N * N
    print(json.dumps({"two_phase": "chunk48", "mean_route_len": hist / (H * N),
                      "current_blocks": N, "routed_us": t_r, "two_phase_us": t_2,
                      "two_phase_tflops": 4.0 * 128 ** 3 * tiles / (t_2 * 1e-6) / 1e12,
                      "routed_tflops": 4.0 * 128 ** 3 * hist / (t_r * 1e-6) / 1e12,
                      "dev_status": layer.status()}), flush=True)


def run_variants(args):
    """The comparison rows, one JSON line each (not the bench line): the
    geometry-model audit at the audit scale (40 heads, 12 query blocks, 143
    history blocks), the model-only route (lambda = 0) against the fused
    route at the chunk-48 shape, and the THW-linear order's neighbour table
    against the Gilbert order's."""
    import routed_block_sparse_b200 as rbs
    from routed_block_sparse_b200.pipeline import audit_metrics, layer_for
    from synth import config, make_inputs

    # 1. audit workload (H 40, N 12, M 143; tau 0.1, lambda 2, g_ref 0.2)
    wl = config(2)
    inp = make_inputs(wl, "cuda")
    layer = layer_for(wl)
    p = layer.importance(inp.Q, inp.K)
    H, N, M = wl.heads, wl.n_q_blocks, wl.n_kv_blocks
    counts = torch.empty(H, N, 6, dtype=torch.int32, device="cuda")
    prm = rbs.route_params(2.0, 0.1, 0.2, 0.9, 0.9, 80, 150)
    t_a = _time_us(lambda: rbs.velox_route_audit(p, inp.g, H, N, M, prm, 50, 80, counts))
    print(json.dumps({"variant": "audit", "config": "audit H40 N12 M143", "audit_us": t_a,
                      **audit_metrics(counts, M), "random_expectation": 50 / M}), flush=True)
    del inp, layer

    # 2. model-only (lambda = 0) vs fused routing at chunk-48
    wl = config(3)
    inp = make_inputs(wl, "cuda")
    out = {"variant": "model_only_vs_fused", "config": "chunk48 H40 N48 M2256"}
    for name, lam in (("fused", wl.params.lam), ("model_only", 0.0)):
        layer = layer_for(wl)
        layer.prm = rbs.route_params(lam, wl.params.tau, wl.params.g_ref, wl.params.theta_cov,
                                     wl.params.theta_unc, wl.params.k_cov, wl.params.k_unc)
        layer.importance(inp.Q, inp.K)
        t_r = _time_us(lambda: layer.route(inp.g, inp.covered), reps=20)
        t_att = _time_us(lambda: layer.attend(inp.Q, inp.K, inp.V), reps=10)
        out[name + "_route_us"] = t_r
        out[name + "_attn_us"] = t_att
        out[name + "_mean_route_len"] = float(layer.route_len.float().mean().item())
        del layer
    print(json.dumps(out), flush=True)
    del inp

    # 3. THW-linear vs Gilbert: neighbour table at the chunk-48 lattice
    T, Hl, Wl, b, nc = 4, 32, 48, 128, 48
    Nq = T * Hl * Wl // b
    ids = torch.empty(Nq, 64, dtype=torch.int32, device="cuda")
    cnt = torch.empty(Nq, dtype=torch.int32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = {"variant": "thw_linear_vs_gilbert", "lattice": "T4 32x48 b128, 48 chunks"}
    for name, fn in (("gilbert", rbs.velox_gilbert_order), ("thw", rbs.velox_thw_linear_order)):
        call = lambda: fn(T, Hl, Wl, nc, b, nc - 1, 0, (nc - 1) * Nq, nbr_ids=ids, nbr_cnt=cnt,
                          S_max=64, dev_status=st)
        out[name + "_nbr_us"] = _time_us(call)
        # safeguards within the whole lattice (the cache holding every chunk)
        fn(T, Hl, Wl, nc, b, nc - 2, 0, nc * Nq, nbr_ids=ids, nbr_cnt=cnt, S_max=64,
           dev_status=st)
        torch.cuda.synchronize()
        out[name + "_mean_safeguards"] = float(cnt.float().mean().item())
    out["dev_status"] = int(st.item())
    print(json.dumps(out), flush=True)


def run_layers(args):
    """Full denoising step at chunk 48: `args.layers` layers with independent
    per-layer inputs (seeded per layer), regenerated into reused buffers
    between layers outside the timed spans (40 layers of K+V would be 236 GB).
    Per layer the importance, route build + schedule and attention run back to
    back on one stream; the summed times are reported."""
    from routed_block_sparse_b200.pipeline import layer_for
    from synth import config, make_inputs

    wl0 = config(5, 0)
    layer = layer_for(wl0)
    inp = make_inputs(wl0, "cuda")
    stream = torch.cuda.current_stream()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
    t_route = t_attn = 0.0
    tiles = 0.0
    status = 0
    for li in range(args.layers):
        inp = make_inputs(config(5, li), "cuda", out=inp)
        torch.cuda.synchronize()
        ev[0].record(stream)
        layer.importance(inp.Q, inp.K, stream)
        layer.route(inp.g, inp.covered, stream=stream)
        ev[1].record(stream)
        layer.attend(inp.Q, inp.K, inp.V, stream=stream)
        ev[2].record(stream)
        torch.cuda.synchronize()
        t_route += ev[0].elapsed_time(ev[1])
        t_attn += ev[1].elapsed_time(ev[2])
        tiles += float(layer.route_len.sum().item())
        status |= layer.status()
    flops = 4.0 * 128 ** 3 * tiles
    print(json.dumps({"mode": "layers", "layers": args.layers,
                      "route_build_ms_total": t_route, "attention_ms_total": t_attn,
                      "attention_tflops": flops / (t_attn * 1e-3) / 1e12,
                      "route_share": t_route / (t_route + t_attn), "dev_status": status,
                      "note": "importance + route build + schedule per layer counted as route build"}),
          flush=True)


def _attn_source_hash() -> str:
    import hashlib
    p = os.path.join(ROOT, "routed_block_sparse_b200", "csrc", "attn.cu")
    with open(p, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="velox", choices=["velox", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--sweep", action="store_true",
                    help="history-length sweep: routed vs dense attention per M (extra lines)")
    ap.add_argument("--variants", action="store_true",
                    help="audit, model-only routing and THW-linear comparisons")
    ap.add_argument("--geometry", action="store_true",
                    help="time slab overlap and coverage at the chunk-48 shape")
    ap.add_argument("--two-phase", action="store_true",
                    help="time two-phase attention (history routes + current chunk)")
    ap.add_argument("--layers", type=int, default=0,
                    help="full-step mode: this many chunk-48 layers with per-layer inputs "
                         "(extra line with the summed route-build and attention times)")
    ap.add_argument("--heads", type=int, default=0,
                    help="run a reduced head count (profiler captures only)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        world = int(os.environ.get("WORLD_SIZE", "1"))
        run_reference(args, world, rank)
        return
    world, rank, local = _dist_setup()
    try:
        if args.sweep:
            run_sweep(args)
            return
        if args.geometry:
            run_geometry(args)
            return
        if args.variants:
            run_variants(args)
            return
        if args.two_phase:
            run_two_phase(args)
            return
        if args.layers:
            run_layers(args)
            return
        run_velox(args, world, rank, local)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
