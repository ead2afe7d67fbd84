"""Benchmark of the routed block-sparse attention path on B200.

One step = one pass of the whole hot path over one layer of the chunk-48
workload (40 heads, 48 query blocks, 2256 history blocks of 128 tokens,
head_dim 128, bf16): Gilbert order + neighbour table, block importance, soft
fusion and route build, routed attention.  Inputs are resident in HBM and
larger than L2 (K + V = 5.9 GB), so no L2 flush is needed between steps.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl velox|reference]

Prints one JSON line.  value = routed-attention FLOPs of the step (4 b^2 d per
routed tile, from the actual route lengths), summed over ranks, over the
slowest rank's step time.  With N ranks the heads of the one layer are split
across them (strong scaling; `--shard layers` gives every rank its own layer
instead); there is no data-path collective.  Per-call times, the roofline of
the attention kernel (with the SM clock measured from the GPU beside the
attention calls: the driver's sampled clock does not show the power
limiter), two end-to-end numbers through host buffers (`e2e`: every input
of the step copied in each step; `e2e_rollout`: the KV cache kept in HBM and
only what a rollout's step brings in copied) and the CPU oracle baseline are
added.
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
    """SM clock and clock-event reasons sampled while the timed region runs.

    Reads only (NVML queries of the launching device, every `period_s`; the
    nvidia-smi command line at 20 ms when NVML cannot be used).  __enter__
    returns once the first sample has arrived, so a short timed region still
    gets samples from its start.
    """

    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device, period_s: float = 0.005):
        self.device = torch.device(device)
        self.period = period_s
        self.samples = []      # (sm_mhz, set of reason names)
        self.sm_max = None
        self.source = None
        self._stop = threading.Event()
        self._t = None
        self.proc = None

    def __enter__(self):
        try:
            self._start_nvml()
        except Exception:
            self._start_smi()
        t0 = time.time()
        while not self.samples and time.time() - t0 < 3.0 and (self._t and self._t.is_alive()):
            time.sleep(0.002)
        return self

    def _start_nvml(self):
        import pynvml
        pynvml.nvmlInit()
        idx = torch.cuda._get_nvml_device_index(self.device)
        h = pynvml.nvmlDeviceGetHandleByIndex(idx)
        self.sm_max = float(pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM))
        bits = {"hw_slowdown": pynvml.nvmlClocksEventReasonHwSlowdown,
                "hw_thermal_slowdown": pynvml.nvmlClocksEventReasonHwThermalSlowdown,
                "sw_thermal_slowdown": pynvml.nvmlClocksEventReasonSwThermalSlowdown,
                "sw_power_cap": pynvml.nvmlClocksEventReasonSwPowerCap}
        reasons_fn = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            pynvml.nvmlDeviceGetCurrentClocksThrottleReasons
        self.source = f"nvml (device {idx}, every {self.period * 1e3:.0f} ms)"

        def run():
            while not self._stop.is_set():
                try:
                    mhz = float(pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM))
                    r = int(reasons_fn(h))
                    self.samples.append((mhz, {n for n, b in bits.items() if r & b}))
                except Exception:
                    pass
                self._stop.wait(self.period)

        self._t = threading.Thread(target=run, daemon=True)
        self._t.start()

    def _start_smi(self):
        gpu = self.device.index or 0
        try:
            gpu = torch.cuda._get_nvml_device_index(self.device)
        except Exception:
            pass
        self.proc = subprocess.Popen(
            ["nvidia-smi", f"--id={gpu}", f"--query-gpu={self.QUERY}",
             "--format=csv,noheader,nounits", "-lms", "20"],
            stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        self.source = "nvidia-smi (every 20 ms)"

        def run():
            for line in self.proc.stdout:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    mhz = float(parts[1])
                    self.sm_max = float(parts[2])
                except ValueError:
                    continue
                self.samples.append((mhz, {n for n, v in zip(self.NAMES, parts[5:9])
                                           if v.lower() == "active"}))

        self._t = threading.Thread(target=run, daemon=True)
        self._t.start()

    def __exit__(self, *exc):
        self._stop.set()
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
        if self._t:
            self._t.join(timeout=2)

    def summary(self):
        sm = [m for m, _ in self.samples]
        reasons = set()
        for _, r in self.samples:
            reasons |= r
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": self.sm_max,
                "sm_mhz_min": min(sm) if sm else None, "reasons": sorted(reasons),
                "samples": len(sm), "source": self.source}


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


def head_range(rank: int, world: int, H: int):
    """Heads [h0, h1) that rank `rank` of `world` owns when the H heads of one
    layer are split across ranks: contiguous, sizes differing by at most one,
    every head owned by exactly one rank."""
    return rank * H // world, (rank + 1) * H // world


def rank_workload(rank: int, world: int = 1, heads: int = 0, shard: str = "heads"):
    """The chunk-48 layer share of one rank, and its heads within the layer.

    shard="heads" (default): rank r runs heads head_range(r, world, 40) of
    layer 0 -- one layer split across the ranks (strong scaling).  Heads are
    independent in every step of the path and g, the coverage flags and the
    neighbour table are shared inputs, so no data crosses between ranks.
    shard="layers": rank r runs all heads of its own layer r (weak scaling).
    `heads` > 0 reduces the head count (profiler captures only, never a
    bench value).
    """
    from dataclasses import replace
    from synth import config
    wl = config(3, layer=rank if shard == "layers" else 0)
    if heads:
        wl = replace(wl, heads=heads)
    if shard == "layers" or world == 1:
        return wl, (0, wl.heads)
    return wl, head_range(rank, world, wl.heads)


def bench_config(wl, heads=None) -> dict:
    """The `config` object of the bench line (both arms)."""
    T, Hl, Wl = wl.lattice
    H = wl.heads
    return {"workload": "chunk48" if H == 40 else f"chunk48 reduced to {H} heads",
            "heads": H, "n_q_blocks": wl.n_q_blocks, "n_kv_blocks": wl.n_kv_blocks,
            "head_dim": wl.d, "b_tok": wl.b, "k_cov": wl.params.k_cov,
            "k_unc": wl.params.k_unc, "theta": wl.params.theta_unc, "lattice": [T, Hl, Wl],
            "l2": "inputs larger than L2 (K+V 5.9 GB per layer), no flush"}


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
    """--impl reference: the CPU oracle, as it stands, on the host cores.

    Rank 0 only.  Each step is a bounded sample of the chunk-48 layer: one
    whole head (1/40 of the layer's work) -- its importance over all 48 x
    2256 blocks, the routes of its 48 query blocks and attention of those 48
    rows -- timed as it runs; value = that head's routed-attention FLOPs over
    the measured time, the same metric and unit as the GPU arm.  The Gilbert
    neighbour table, built once per layer (about 0.2 % of the oracle's layer
    time), is built once before the steps and reported on its own.
    """
    if rank != 0:
        return
    import dataclasses
    from oracle import attention as oatt
    from oracle import gilbert as ogil
    from oracle import importance as oimp
    from oracle import route as ort
    from synth import config, make_inputs
    from threadpoolctl import threadpool_info

    wl = config(3)
    # one head of the chunk-48 shape and distributions (drawing all 40 heads
    # on the CPU would take minutes)
    inp = make_inputs(dataclasses.replace(wl, heads=1), "cpu")
    H, N, M, b = wl.heads, wl.n_q_blocks, wl.n_kv_blocks, wl.b
    prm = ort.Params(lam=wl.params.lam, tau=wl.params.tau, g_ref=wl.params.g_ref,
                     theta_cov=wl.params.theta_cov, theta_unc=wl.params.theta_unc,
                     k_cov=wl.params.k_cov, k_unc=wl.params.k_unc)
    Qh, Kh, Vh = (x[0].to(torch.float64).numpy() for x in (inp.Q, inp.K, inp.V))
    g, cov = inp.g.numpy(), inp.covered.numpy()
    T, Hl, Wl = wl.lattice
    t0 = time.perf_counter()
    nbr = ogil.neighbour_blocks(T, Hl, Wl, wl.n_chunks, b, wl.q_chunk, wl.cache_first_block, M)
    t_nbr = time.perf_counter() - t0

    def one_head():
        p = oimp.importance(Qh, Kh, b, 1.0).astype(np.float32)
        routes = [ort.route_row(p[i], g[i], bool(cov[i]), prm, wl.prev_begin, wl.prev_count,
                                nbr[i]) for i in range(N)]
        tiles = 0
        for i in range(N):
            ids = routes[i][0] + routes[i][1]
            oatt.routed_attention_block(Qh[i * b:(i + 1) * b], Kh, Vh, ids, b)
            tiles += len(ids)
        return tiles

    times, flops = [], []
    for st in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        tiles = one_head()
        dt = time.perf_counter() - t0
        if st >= args.warmup:
            times.append(dt)
            flops.append(4.0 * b * b * wl.d * tiles)
    value = sum(flops) / sum(times) / 1e12
    threads = [x.get("num_threads", 1) for x in threadpool_info() if x.get("user_api") == "blas"]
    cores = max(threads) if threads else 1
    sample = (f"one whole head per step (1/{H} of the chunk-48 layer): importance ({N}x{M} "
              f"blocks), routes of its {N} query blocks, attention of those {N} rows; "
              f"fp64 numpy oracle, {cores} BLAS threads")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
            "n_gpus": max(world, args.gpus), "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": statistics.mean(times) * 1e3, "higher_is_better": True,
            "scaling": "strong" if args.shard == "heads" else "weak", "vs_baseline": None,
            "dtype": "f64", "data": "synthetic (the GPU arm's recipe, one head)",
            "config": bench_config(wl), "sample_per_step": sample,
            "neighbour_table_ms": t_nbr * 1e3,
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- velox ---
def run_velox(args, world, rank, local):
    import routed_block_sparse_b200 as rbs
    from routed_block_sparse_b200.pipeline import layer_for
    from synth import make_inputs

    dev = torch.device("cuda", local if world > 1 else 0)
    wl_layer, (h0, h1) = rank_workload(rank, world, args.heads, args.shard)
    inp = make_inputs(wl_layer, dev, heads=(h0, h1))
    wl = inp.wl  # this rank's heads
    layer = layer_for(wl, device=dev)
    H, N, M, b, d = wl.heads, wl.n_q_blocks, wl.n_kv_blocks, wl.b, wl.d
    T, Hl, Wl = wl.lattice
    stream = torch.cuda.current_stream(dev)

    side = torch.cuda.Stream(dev)

    # One step.  The neighbour table (a1) does not depend on the importance
    # (a2, a3): it runs on a side stream forked at the start of the step and
    # joined before the route build, which needs both.  Events: 0 step start,
    # 1 / 2 importance start / end (main stream), 3 route end, 4 attention end,
    # 5 / 6 neighbour table start / end (side stream).
    def step(ev=None, st=None):
        st = stream if st is None else st
        if ev is not None:
            ev[0].record(st)
        side.wait_stream(st)
        if ev is not None:
            ev[5].record(side)
        rbs.velox_gilbert_order(T, Hl, Wl, wl.n_chunks, b, wl.q_chunk, wl.cache_first_block, M,
                                nbr_ids=layer.nbr_ids, nbr_cnt=layer.nbr_cnt,
                                S_max=layer.S_max, dev_status=layer.dev_status, stream=side)
        if ev is not None:
            ev[6].record(side)
            ev[1].record(st)
        layer.importance(inp.Q, inp.K, st)
        if ev is not None:
            ev[2].record(st)
        st.wait_stream(side)
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
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(7)] for _ in range(args.steps)]
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    _barrier(world)
    torch.cuda.synchronize(dev)
    with ClockSampler(dev) as clocks:
        t_start.record(stream)
        for k in range(args.steps):
            step(evs[k])
        t_end.record(stream)
        torch.cuda.synchronize(dev)
    _barrier(world)
    torch.cuda.synchronize(dev)
    total_ms = t_start.elapsed_time(t_end)
    parts = np.array([[e[5].elapsed_time(e[6]), e[1].elapsed_time(e[2]),
                       e[2].elapsed_time(e[3]), e[3].elapsed_time(e[4])] for e in evs])
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

    clk = clocks.summary()
    strong = args.shard == "heads"
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "strong" if strong else "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) bf16 Q/K/V; g U[0,1] half zeroed; coverage Bernoulli 0.5)",
        "config": bench_config(wl_layer),
        "shard": ({"by": "heads", "heads_of_rank0": [h0, h1], "layer": 0} if strong and world > 1
                  else {"by": args.shard if world > 1 else "none"}),
        "attn_us": attn_ms * 1e3, "attn_tflops": attn_tflops,
        "importance_us": imp_ms * 1e3, "importance_gbs": imp_gbs,
        "route_us": route_ms * 1e3, "gilbert_us": gil_ms * 1e3,
        "importance_route_gbs": ir_gbs, "importance_route_hbm_frac": ir_gbs / hbm,
        "routed_tiles": tiles, "mean_route_len": tiles / (H * N), "dev_status": status,
        # the timed loop is short (tens to hundreds of ms), so the denominator
        # is the measured burst bf16 figure; the sustained (power-capped)
        # figure and the fraction against it are reported beside it, and the
        # clock-normalised time (us x median SM MHz) lets runs on boxes that
        # settle at different clocks be compared
        "roofline": {"bound": "tensor", "achieved": attn_tflops, "peak": bf16,
                     "unit": "TFLOP/s", "frac": attn_tflops / bf16, "traffic": traffic,
                     "peak_source": f"{peak_kind} bf16 dense burst (cuBLAS 8192^3, best of 10)",
                     "sustained_peak": bf16_sus, "frac_of_sustained_peak": attn_tflops / bf16_sus,
                     "attn_mcycles_per_call": (attn_ms * 1e3 * clk["sm_mhz"] / 1e6
                                               if clk["sm_mhz"] else None)},
        "gpu_launches": LAUNCHES_PER_STEP * args.steps,
        "clocks": clk,
    }

    # the same step captured once as a CUDA graph and replayed (the seven
    # launches go out as one graph launch); reported beside the eager timing
    line["graph"] = _graph_replay(step, args.steps, dev)
    # the SM clock inside the attention kernel, measured from the GPU (after
    # the timed region): NVML's sampled clock does not show the power limiter
    eff = _attn_effective_clock(layer, inp, dev, stream)
    if eff is not None:
        sms = torch.cuda.get_device_properties(dev).multi_processor_count
        line["roofline"]["effective_sm_mhz"] = eff
        line["roofline"]["attn_cycles_per_tile_per_sm"] = attn_ms * 1e3 * eff * sms / tiles
        line["roofline"]["effective_clock_source"] = (
            "velox_clock_probe (one CTA, clock64 against %globaltimer every 2 us) on a side "
            "stream beside 5 attention calls after the timed region; middle half of their span")

    # end to end through the public API with host buffers
    if args.e2e_steps > 0:
        line["e2e"] = _e2e(args, wl, inp, layer, dev, stream, flops_step, world)
        line["e2e_rollout"] = _e2e_rollout(args, wl, inp, layer, dev, stream, flops_step, world)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        r = cpu_oracle_sample(inp)
        line["cpu_baseline"] = {"value": flops_step / r["step_s"] / 1e12, "unit": UNIT,
                                "cores": r["threads"], "kind": "oracle", "sample": r["sample"],
                                "sample_seconds": r["sample_s"]}
    if rank == 0:
        print(json.dumps(line), flush=True)


def _attn_effective_clock(layer, inp, dev, stream, calls=5, n=6000, pause_ns=2000):
    """Median SM clock (MHz) while `calls` attention calls run back to back,
    from the clock probe on a side stream; None if it cannot be read."""
    import routed_block_sparse_b200 as rbs
    try:
        samples = torch.zeros(n, 2, dtype=torch.int64, device=dev)
        side = torch.cuda.Stream(dev)
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize(dev)
        rbs.velox_clock_probe(samples, n, pause_ns, stream=side)
        a.record(stream)
        for _ in range(calls):
            layer.attend(inp.Q, inp.K, inp.V, stream=stream)
        b.record(stream)
        torch.cuda.synchronize(dev)
        span_ns = a.elapsed_time(b) * 1e6
        x = samples.cpu().numpy().astype(np.float64)
        c, t = x[:, 0], x[:, 1]
        rate = np.diff(c) / np.maximum(np.diff(t), 1.0)
        mid = (t[1:] >= t[0] + 0.25 * span_ns) & (t[1:] <= t[0] + 0.75 * span_ns)
        if not mid.any():
            return None
        return float(np.median(rate[mid]) * 1e3)
    except Exception:
        return None


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
        # timed after the eager loop, when the clock may have started to drop
        # under the power cap: the median SM clock of this loop is reported
        with ClockSampler(dev) as clocks:
            a.record()
            for _ in range(steps):
                graph.replay()
            b.record()
            torch.cuda.synchronize(dev)
        ms = a.elapsed_time(b) / steps
        del graph
        return {"ms_per_step": ms, "steps": steps, "sm_mhz": clocks.summary()["sm_mhz"]}
    except Exception as e:  # reported, not fatal: the eager numbers stand alone
        return {"error": str(e)[:200]}


def _e2e_grouped(args, wl, inp, layer, dev, stream, flops_step, world, group_copies):
    """One end-to-end step through the public API, timed with CUDA events on
    the launching stream: g and the coverage flags, then each head group's
    inputs (group_copies(h0, h1): (device view, pinned host tensor) pairs)
    cross on a copy stream; the launching stream runs the neighbour table,
    then a group's importance, route build and attention as soon as its
    inputs have landed, and a third stream sends the group's O and lse back
    while later groups are still crossing or computing.  The heads are independent through the whole path, so
    this is the same step as one call over all heads."""
    from dataclasses import replace
    from routed_block_sparse_b200.pipeline import layer_for
    import routed_block_sparse_b200 as rbs

    g_h = inp.g.cpu().pin_memory()
    c_h = inp.covered.cpu().pin_memory()
    out_O = torch.empty_like(layer.O, device="cpu").pin_memory()
    out_lse = torch.empty_like(layer.lse, device="cpu").pin_memory()
    T, Hl, Wl = wl.lattice
    H = wl.heads
    n_groups = max(1, min(args.e2e_groups, H))
    bounds = [head_range(k, n_groups, H) for k in range(n_groups)]  # as a head split
    plans = [group_copies(h0, h1) for h0, h1 in bounds]
    h2d = g_h.numel() * g_h.element_size() + c_h.numel() * c_h.element_size() + sum(
        src.numel() * src.element_size() for plan in plans for _, src in plan)
    d2h = out_O.numel() * out_O.element_size() + out_lse.numel() * out_lse.element_size()
    layers = [layer_for(replace(wl, heads=h1 - h0), device=dev) for h0, h1 in bounds]
    for lg in layers[1:]:  # one neighbour table per step, read by every group
        lg.nbr_ids, lg.nbr_cnt = layers[0].nbr_ids, layers[0].nbr_cnt
    copy = torch.cuda.Stream(dev)   # host -> device
    back = torch.cuda.Stream(dev)   # device -> host
    ev_in = [torch.cuda.Event() for _ in bounds]
    ev_out = [torch.cuda.Event() for _ in bounds]
    ev_gc = torch.cuda.Event()

    def one():
        copy.wait_stream(stream)  # the last step is done with every input
        with torch.cuda.stream(copy):
            inp.g.copy_(g_h, non_blocking=True)
            inp.covered.copy_(c_h, non_blocking=True)
            ev_gc.record(copy)
            for plan, ev in zip(plans, ev_in):
                for dst, src in plan:
                    dst.copy_(src, non_blocking=True)
                ev.record(copy)
        l0 = layers[0]
        rbs.velox_gilbert_order(T, Hl, Wl, wl.n_chunks, wl.b, wl.q_chunk, wl.cache_first_block,
                                wl.n_kv_blocks, nbr_ids=l0.nbr_ids, nbr_cnt=l0.nbr_cnt,
                                S_max=l0.S_max, dev_status=l0.dev_status, stream=stream)
        stream.wait_event(ev_gc)
        for (h0, h1), ev, done, lg in zip(bounds, ev_in, ev_out, layers):
            stream.wait_event(ev)
            lg.forward(inp.Q[h0:h1], inp.K[h0:h1], inp.V[h0:h1], inp.g, inp.covered, stream)
            done.record(stream)
            back.wait_event(done)
            with torch.cuda.stream(back):
                out_O[h0:h1].copy_(lg.O, non_blocking=True)
                out_lse[h0:h1].copy_(lg.lse, non_blocking=True)
        stream.wait_stream(back)  # the step ends when O and lse are on the host

    one()
    torch.cuda.synchronize(dev)
    status = max(int(lg.status()) for lg in layers)
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
            "d2h_bytes_per_step": d2h, "head_groups": n_groups, "dev_status": status}


def _e2e(args, wl, inp, layer, dev, stream, flops_step, world):
    """Every input of the step (Q, K, V, g, the coverage flags) copied from
    pinned host memory each step; O and lse copied back."""
    host = {k: getattr(inp, k).cpu().pin_memory() for k in ("Q", "K", "V")}

    def copies(h0, h1):
        return [(getattr(inp, k)[h0:h1], host[k][h0:h1]) for k in ("Q", "K", "V")]

    return _e2e_grouped(args, wl, inp, layer, dev, stream, flops_step, world, copies)


def _e2e_rollout(args, wl, inp, layer, dev, stream, flops_step, world):
    """The step as a rollout runs it, with the KV cache kept in HBM: each step
    copies in the current chunk's Q, the previous chunk's K and V (into the
    cache slots that chunk occupies), g and the coverage flags, and copies O
    and lse out.  Each history chunk crosses the
    host link once, when it joins the cache; the synthetic steps re-send the
    same previous chunk into the same slots, so the cache does not change
    between them."""
    # token rows of the previous chunk's blocks (K and V are [H][M*b][d])
    t0, t1 = wl.prev_begin * wl.b, (wl.prev_begin + wl.prev_count) * wl.b
    q_h = inp.Q.cpu().pin_memory()
    k_new = inp.K[:, t0:t1].cpu().pin_memory()
    v_new = inp.V[:, t0:t1].cpu().pin_memory()

    def copies(h0, h1):
        # one copy per tensor and group: the slots of the group's heads are a
        # strided view (torch stages it through a contiguous device buffer)
        return [(inp.Q[h0:h1], q_h[h0:h1]), (inp.K[h0:h1, t0:t1], k_new[h0:h1]),
                (inp.V[h0:h1, t0:t1], v_new[h0:h1])]

    out = _e2e_grouped(args, wl, inp, layer, dev, stream, flops_step, world, copies)
    out["inputs"] = ("current chunk's Q, previous chunk's K/V into its cache slots, g, "
                     "coverage flags; the rest of the KV cache stays in HBM")
    return out


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


def run_dense_vs_cudnn(args):
    """Dense attention over the whole chunk-48 history (H=40, 6,144 query
    tokens, 288,768 cache tokens, d=128): this library's dense mode
    (route_ids = NULL) against torch's scaled_dot_product_attention on its
    cuDNN backend (NVIDIA's fused attention for this GPU) and on its
    FlashAttention-2 backend, the same bf16 tensors, each trial after a
    cool-down, the kinds interleaved.  Context for the attention kernel's
    roofline fraction; not the bench line."""
    import time
    import torch.nn.functional as F
    from torch.nn.attention import SDPBackend, sdpa_kernel
    from routed_block_sparse_b200.pipeline import layer_for
    from synth import config, make_inputs

    wl = config(3)
    inp = make_inputs(wl, "cuda")
    layer = layer_for(wl)
    H, N, M, b, d = wl.heads, wl.n_q_blocks, wl.n_kv_blocks, 128, 128
    q = inp.Q.view(1, H, N * b, d)
    k = inp.K.view(1, H, M * b, d)
    v = inp.V.view(1, H, M * b, d)
    flops = 4.0 * H * (N * b) * (M * b) * d
    kinds = {"velox_dense": lambda: layer.attend(inp.Q, inp.K, inp.V, dense=True)}
    for name, be in (("cudnn", SDPBackend.CUDNN_ATTENTION),
                     ("flash2", SDPBackend.FLASH_ATTENTION)):
        def call(be=be):
            with sdpa_kernel([be]):
                return F.scaled_dot_product_attention(q, k, v)
        kinds[name] = call
    out = {"workload": "dense attention, chunk-48 layer over its whole history",
           "heads": H, "q_tokens": N * b, "kv_tokens": M * b, "head_dim": d,
           "tflop_per_call": flops / 1e12}
    layer.attend(inp.Q, inp.K, inp.V, dense=True)
    mine = layer.O.view(1, H, N * b, d).float()
    for name in list(kinds):
        if name == "velox_dense":
            continue
        try:
            o = kinds[name]()
            torch.cuda.synchronize()
            out[f"{name}_max_abs_vs_velox"] = float((o.float() - mine).abs().max())
            del o
        except RuntimeError as e:  # backend not built for this GPU or shape
            out[f"{name}_error"] = str(e)[:160]
            del kinds[name]
    del mine
    best = {n: float("inf") for n in kinds}
    for _ in range(3):
        for name, fn in kinds.items():
            torch.cuda.synchronize()
            time.sleep(1.0)
            best[name] = min(best[name], _time_us(fn, reps=5, warm=2))
    for name, us in best.items():
        out[f"{name}_ms"] = us / 1e3
        out[f"{name}_tflops"] = flops / (us * 1e-6) / 1e12
    if "cudnn" in best:
        out["velox_dense_vs_cudnn"] = best["cudnn"] / best["velox_dense"]
    print(json.dumps(out), flush=True)


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


def _geometry_chain(layout: str = "gilbert", seed: int = 20261203):
    """The geometry chain at the chunk-48 shape for one token order: slab
    table of the 2256 history blocks (188 frames of 32 x 48 tokens, 2 x 2
    depth samples per token), multiwarp depth of the 4 current frames from the
    first and last frames of the 30 most recent chunks, the current chunk's 48
    query slabs and tokens, slab overlap g (8^3 samples per pair) and coverage
    rho.  Returns the buffers and the five calls (not yet run)."""
    import numpy as np
    import routed_block_sparse_b200 as rbs
    from synth.depth import make_rollout

    T, H, W, b, nc, s = 4, 32, 48, 128, 48, 2
    q_chunk = nc - 1
    per_chunk = T * H * W // b
    M, N = q_chunk * per_chunk, per_chunk
    hist_frames = q_chunk * T
    roll = make_rollout(seed, nc * T, H, W, s)
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    cams = dev(roll.cams)
    n_cam = cams.shape[0]
    depth, conf, mask = dev(roll.depth[:hist_frames]), dev(roll.conf[:hist_frames]), \
        dev(roll.mask[:hist_frames])
    cell = torch.empty(nc * T * H * W, dtype=torch.int32, device="cuda")
    order = rbs.velox_gilbert_order if layout == "gilbert" else rbs.velox_thw_linear_order
    order(T, H, W, nc, b, cell_of_rank=cell)
    src = []
    for c in range(q_chunk - 1, q_chunk - 31, -1):          # 30 most recent chunks
        src += [c * T + T - 1, c * T]                        # last, first frame
    src_depth = dev(roll.depth[src])
    src_cam = torch.tensor(src, dtype=torch.int32, device="cuda")
    tgt_cam = torch.arange(hist_frames, hist_frames + T, dtype=torch.int32, device="cuda")
    buf = {"hs": torch.empty(M, 8, dtype=torch.int32, device="cuda"),
           "qs": torch.empty(N, 8, dtype=torch.int32, device="cuda"),
           "zq": torch.empty(T, H, W, device="cuda"),
           "uvz": torch.empty(N, b, 3, device="cuda"),
           "g": torch.empty(N, M, device="cuda"),
           "rho": torch.empty(N, device="cuda"),
           "cov": torch.empty(N, dtype=torch.uint8, device="cuda"),
           "st": torch.zeros(1, dtype=torch.int32, device="cuda"),
           "mw_ws": torch.empty(rbs.velox_multiwarp_workspace_size(len(src), T, H, W),
                                dtype=torch.uint8, device="cuda"),
           "cell": cell}
    B = buf

    def table():
        rbs.velox_slab_table(depth, conf, mask, hist_frames, 0, H, W, s, cell, cell.numel(), b, 0,
                             M, 0.5, 16, 0.1, 0.9, B["hs"], B["st"])

    def warp():
        rbs.velox_multiwarp(cams, n_cam, src_depth, src_cam, len(src), tgt_cam, T, H, W, s, 2,
                            B["zq"], B["mw_ws"], B["st"])

    def qtable():
        rbs.velox_slab_table(B["zq"], None, None, T, hist_frames, H, W, 1, cell, cell.numel(), b,
                             q_chunk * per_chunk, N, 0.5, 8, 0.1, 0.9, B["qs"], B["st"],
                             token_uvz=B["uvz"])

    def overlap():
        rbs.velox_slab_overlap(cams, n_cam, B["qs"], N, B["hs"], M, 8, B["g"], B["st"])

    def coverage():
        rbs.velox_coverage(cams, n_cam, B["qs"], B["uvz"], N, b, B["hs"], M, 0.9, B["rho"],
                           B["cov"], B["st"])

    calls = (("slab_table", table), ("multiwarp", warp), ("query_slabs", qtable),
             ("slab_overlap", overlap), ("coverage", coverage))
    meta = {"N": N, "M": M, "grid": 8, "b": b, "depth_samples": s,
            "multiwarp_sources": len(src)}
    return buf, calls, meta


def run_geometry(args):
    """The geometry chain at the chunk-48 shape (Gilbert order), one JSON
    line of per-call times (not the bench line)."""
    buf, calls, meta = _geometry_chain("gilbert")
    out = {"geometry": "chunk48", **meta}
    for name, fn in calls:
        out[name + "_us"] = _time_us(fn)

    def chain():
        for _, fn in calls:
            fn()
    out["chain_us"] = _time_us(chain, reps=20)
    torch.cuda.synchronize()
    out.update({"valid_history_slabs": int(buf["hs"][:, 7].sum().item()),
                "query_holes": float((buf["zq"] == 0).float().mean().item()),
                "nonzero_pairs": int((buf["g"] > 0).sum().item()),
                "covered_blocks": int(buf["cov"].sum().item()),
                "dev_status": int(buf["st"].item())})
    print(json.dumps(out), flush=True)


def _route_union(route_ids: torch.Tensor, route_len: torch.Tensor) -> float:
    """Mean over heads of the number of distinct tiles the head's routes
    touch (the K/V tiles a launch must read at least once)."""
    ids = route_ids.cpu().numpy()
    lens = route_len.cpu().numpy()
    total = 0
    for h in range(ids.shape[0]):
        seen = set()
        for i in range(ids.shape[1]):
            seen.update(ids[h, i, :lens[h, i]].tolist())
        total += len(seen)
    return total / max(1, ids.shape[0])


def _route_runs(route_ids: torch.Tensor, route_len: torch.Tensor):
    """Mean route length and mean length of the runs of consecutive block
    ids in the routes (each route taken as a sorted set)."""
    ids = route_ids.cpu().numpy().reshape(-1, route_ids.shape[-1])
    lens = route_len.cpu().numpy().reshape(-1)
    total = runs = 0
    for r in range(ids.shape[0]):
        v = np.sort(ids[r, :lens[r]])
        if len(v):
            total += len(v)
            runs += 1 + int(np.count_nonzero(np.diff(v) != 1))
    return total / max(1, ids.shape[0]), total / max(1, runs)


def run_layouts(args):
    """Gilbert against THW-linear token order through the whole routed path
    at the chunk-48 shape: the geometry chain of each order (slab tables from
    the same depth maps, multiwarp, g, coverage), then importance, route
    build and attention.  Two input recipes: `random` (the N(0, 1) Q/K/V of
    the bench, the same rows under both orders) and `positional` (Q/K from
    synth.positional, whose q . k follows the distance between the tokens'
    lattice positions, each token keeping its values under both orders; V
    N(0, 1)).  One JSON line per order and recipe: mean route length, mean
    run of consecutive block ids in a route, distinct tiles per head (the
    K/V a launch must read), attention time.  `--layout` and `--qk` restrict
    it (for an ncu capture)."""
    from routed_block_sparse_b200.pipeline import layer_for
    from synth import config, make_inputs
    from synth.positional import positional_qk

    wl = config(3)
    if args.heads:
        from dataclasses import replace
        wl = replace(wl, heads=args.heads)
    inp = make_inputs(wl, "cuda")
    T, Hl, Wl = wl.lattice
    q0 = wl.q_chunk * T * Hl * Wl  # rank of the current chunk's first token
    for layout in (("gilbert", "thw") if args.layout == "both" else (args.layout,)):
        buf, calls, _ = _geometry_chain(layout)
        for _, fn in calls:
            fn()
        for qk in (("random", "positional") if args.qk == "both" else (args.qk,)):
            if qk == "positional":
                cell = buf["cell"]
                Q, K = positional_qk(cell[q0:q0 + wl.n_q_blocks * wl.b],
                                     cell[:wl.n_kv_blocks * wl.b], wl.heads, Hl, Wl,
                                     cell.numel(), wl.d)
            else:
                Q, K = inp.Q, inp.K
            layer = layer_for(wl, order=layout)
            layer.importance(Q, K)
            layer.route(buf["g"], buf["cov"])
            torch.cuda.synchronize()
            mean_len, mean_run = _route_runs(layer.route_ids, layer.route_len)
            union = _route_union(layer.route_ids, layer.route_len)
            t_att = _time_us(lambda: layer.attend(Q, K, inp.V), reps=20)
            tiles = float(layer.route_len.sum().item())
            print(json.dumps({"layout": layout, "qk": qk, "config": bench_config(wl),
                              "g_nonzero_pairs": int((buf["g"] > 0).sum().item()),
                              "covered_blocks": int(buf["cov"].sum().item()),
                              "mean_route_len": mean_len, "mean_run_len": mean_run,
                              "distinct_tiles_per_head": union,
                              "attn_us": t_att,
                              "attn_tflops": 4.0 * 128 ** 3 * tiles / (t_att * 1e-6) / 1e12,
                              "dev_status": layer.status() | int(buf["st"].item())}),
                  flush=True)
            del layer
            if qk == "positional":
                del Q, K
            torch.cuda.empty_cache()
        del buf
        torch.cuda.empty_cache()


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

    def two():
        rbs.velox_two_phase_attn(inp.Q, inp.K, inp.V, layer.route_ids, layer.route_len,
                                 layer.R_max, Kc, Vc, N, H, N, M, 128, 128, layer.softmax_scale,
                                 layer.O, layer.lse, layer.dev_status, row_order=layer.row_order)
    # three alternating rounds of 10 calls each, so that both forms see the
    # same clock (it drops as the power cap is reached); the fastest round of
    # each is reported
    t_rs, t_2s = [], []
    for _ in range(3):
        t_rs.append(_time_us(lambda: layer.attend(inp.Q, inp.K, inp.V), reps=10))
        t_2s.append(_time_us(two, reps=10))
    t_r, t_2 = min(t_rs), min(t_2s)
    tiles = hist + H * N * N
    print(json.dumps({"two_phase": "chunk48", "mean_route_len": hist / (H * N),
                      "current_blocks": N, "routed_us": t_r, "two_phase_us": t_2,
                      "routed_us_rounds": t_rs, "two_phase_us_rounds": t_2s,
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


def _spawn_ranks(n: int) -> int:
    import socket
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n}",
           "--master-addr", "127.0.0.1", f"--master-port={port}", os.path.abspath(__file__),
           *sys.argv[1:]]
    return subprocess.call(cmd)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--shard", default="heads", choices=["heads", "layers"],
                    help="N > 1: split one layer's heads over the ranks (strong scaling) or "
                         "give every rank its own layer (weak scaling)")
    ap.add_argument("--impl", default="velox", choices=["velox", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--e2e-groups", type=int, default=8,
                    help="head groups the end-to-end step pipelines its host copies over")
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
    ap.add_argument("--layouts", action="store_true",
                    help="Gilbert vs THW-linear order through geometry, routes and attention")
    ap.add_argument("--layout", default="both", choices=["both", "gilbert", "thw"])
    ap.add_argument("--qk", default="both", choices=["both", "random", "positional"],
                    help="--layouts input recipe: random N(0,1) Q/K or positional Q/K")
    ap.add_argument("--dense-vs-cudnn", action="store_true",
                    help="dense attention: this library against torch SDPA (cuDNN, FA2)")
    ap.add_argument("--heads", type=int, default=0,
                    help="run a reduced head count (profiler captures only)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ and args.impl == "velox":
        # start one rank per GPU (the same command under torch.distributed.run)
        sys.exit(_spawn_ranks(args.gpus))
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
        if args.dense_vs_cudnn:
            run_dense_vs_cudnn(args)
            return
        if args.geometry:
            run_geometry(args)
            return
        if args.layouts:
            run_layouts(args)
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
