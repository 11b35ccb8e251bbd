"""Benchmark of route-layer chunk-routing sparse attention on B200.

One step = one route layer over one synthetic sequence: rdl_summary_pool +
rdl_route_score_topk + rdl_route_attn on the 16K Dream-7B-shaped prefill (28 query heads,
4 KV heads, head dim 128, K = 32 chunks, window radius 256, rank-64 residual), inputs
resident in HBM.  The metric is route-layer query tokens per second (content rows; the
mask-slot rows are produced by the summary pool inside the same step).  The JSON line
also carries the 128K decode block (score + attention with cached summaries, ms per step)
and the 28-layer 128K attention stack (ms per denoising step).

    python bench.py [--gpus N --steps K --warmup W] [--impl reference]

Under torchrun every rank processes its own sequence (no exchange between ranks), the
timed region is bracketed by barriers and the reported time is the max over ranks.
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

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "route-layer sparse-attn query-tokens/s at 16K-128K; decode-step ms at 128K"
# DRAM bytes of one rdl_route_attn call on the 16K prefill (window + chunk kernels), from one
# ncu capture of the current kernels; set to None when either kernel changes.
ATTN_PREFILL_TRAFFIC = 941.8e6
# DRAM bytes of one 128K decode step (the six decode kernels, one launch each, caches cold
# between kernels under ncu, so intermediates re-read from DRAM here stay in L2 live); set to
# None when a decode kernel changes.
DECODE_STEP_TRAFFIC = 108.34e6
UNIT = "query-tokens/s"
PEAK_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(PEAK_FALLBACK), "fallback"


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-i", str(self.gpu)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
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
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


# ----------------------------------------------------------------------------- algorithmic work

def attn_flops(dims, q_pos, idx) -> float:
    """2 (QK) + 2 (PV) flops x d per attended key per (row, head): window keys |W(p)| and
    the 63 content keys of each selected chunk, content rows only."""
    L, w, d, Hq, Hkv = dims.L, dims.w, dims.d, dims.Hq, dims.Hkv
    G = Hq // Hkv
    pos = np.arange(L) if q_pos is None else np.asarray(q_pos[0], dtype=np.int64)
    content = (pos % 64) != 63
    win = np.minimum(L, pos + w + 1) - np.maximum(0, pos - w) if w >= 0 else np.zeros_like(pos)
    nsel = (idx[0] >= 0).sum(axis=-1)                       # [Hkv, Lq]
    keys = (win[None, :] + 63 * nsel) * content[None, :]    # per (group, row)
    return float(4 * d * G * keys.sum())


def score_flops(dims) -> float:
    Lq, C = dims.Lq, dims.L // 64
    return float(2 * Lq * dims.D * dims.r + 2 * Lq * dims.r * dims.Hq * dims.d
                 + 2 * Lq * dims.Hq * C * dims.d)


def decode_bytes(dims, idx) -> dict:
    """Bytes a decode step must move: summaries + entropies, every distinct selected
    (group, chunk) K/V slab, the window K/V, the queries, residual inputs and outputs."""
    C = dims.L // 64
    s_bytes = 4 * dims.B * dims.Hq * C * (dims.d + 1)
    uniq = sum(len(set(idx[b, g][idx[b, g] >= 0].tolist())) for b in range(idx.shape[0])
               for g in range(idx.shape[1]))
    chunk_bytes = uniq * 2 * 64 * dims.d * 2
    win_keys = min(dims.L, 64 + 2 * dims.w)                 # union of the block's windows
    win_bytes = dims.B * dims.Hkv * win_keys * 2 * dims.d * 2
    io = 2 * dims.B * dims.Lq * (2 * dims.Hq * dims.d + dims.D) + 2 * (dims.D * dims.r
                                                                       + dims.r * dims.Hq * dims.d)
    return {"total": s_bytes + chunk_bytes + win_bytes + io, "unique_pairs": uniq,
            "summary": s_bytes, "chunks": chunk_bytes}


# ----------------------------------------------------------------------------- ranks

def rank_seed(base: int, rank: int) -> int:
    """Each rank draws its own independent sequence (no data exchange between ranks)."""
    return base + 1000 * rank


def max_over_ranks(x: float, world: int, device=None) -> float:
    """Max of a per-rank time over all ranks (every rank calls it the same number of times)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(rows_per_rank: int, world: int, ms_max: float) -> float:
    """Whole-job rows per second: all ranks' rows over the slowest rank's time."""
    return world * rows_per_rank / (ms_max / 1e3)


# ----------------------------------------------------------------------------- oracle arm

def oracle_sample(wl, n_rows: int, seed: int = 0):
    """Time the fp64 oracle on a bounded sample of the workload: all summaries + n rows."""
    from threadpoolctl import threadpool_limits
    from oracle import rdl_oracle as O
    from diffusion_lms_b200.workloads import as_f64
    f = {n: as_f64(getattr(wl, n)) for n in ("q", "q_mask", "k", "v", "x", "w_down", "w_up")}
    dm = wl.dims
    rng = np.random.default_rng(seed)
    pos = np.arange(dm.L) if wl.q_pos is None else wl.q_pos[0]
    cand = np.array([i for i in range(dm.Lq) if pos[i] % 64 != 63])
    rows = np.sort(rng.choice(cand, size=min(n_rows, cand.size), replace=False))
    with threadpool_limits(limits=1):
        t0 = time.perf_counter()
        s, H, _ = O.summary_pool(f["q_mask"], f["k"], f["v"])
        idx, z = O.route_score_topk(f["q"], wl.q_pos, f["x"], f["w_down"], f["w_up"], s, H,
                                    Hkv=dm.Hkv, K=dm.K, w=dm.w, lam=dm.lam, L=dm.L, rows=rows)
        O.route_attn(f["q"], wl.q_pos, f["k"], f["v"], idx, z, w=dm.w, rows=rows)
        dt = time.perf_counter() - t0
    return dt, rows.size


def run_reference(args, rank):
    from diffusion_lms_b200 import workloads as W
    if rank != 0:
        return
    wl = W.prefill_16k()
    n = args.ref_rows
    for _ in range(args.warmup):
        oracle_sample(wl, max(1, n // 8))
    times = [oracle_sample(wl, n, seed=s)[0] for s in range(args.steps)]
    ms = 1e3 * statistics.mean(times)
    val = n / (ms / 1e3)
    sample = (f"all 256x28 summaries + {n} random content rows of the 16K prefill per step "
              f"(fp64 NumPy, 1 BLAS thread)")
    line = {"metric": METRIC, "value": val, "unit": UNIT, "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "impl": "reference",
            "config": {"workload": wl.name, "L": 16384, "Hq": 28, "Hkv": 4, "d": 128, "K": 32,
                       "w": 256, "r": 64, "D": 3584, "rows_per_step": n},
            "cpu_baseline": {"value": val, "unit": UNIT, "cores": 1, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": val, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def decode_bench(args, dev, stream, flush, rank, world, max_ranks, pk, pk_kind):
    """128K decode block: rdl_route_score_topk + rdl_route_attn with cached summaries,
    captured once in a CUDA graph and replayed; L2 flushed between replays (untimed)."""
    import torch
    from diffusion_lms_b200 import api, rdl
    from diffusion_lms_b200 import workloads as W
    wd = W.decode_128k(seed=rank_seed(3, rank))
    dinp = api.to_device(wd, dev)
    dinp.dims.flags = rdl.FLAG_SPLIT_SUMMARY      # summaries pooled once per block, pre-split
    dout = api.alloc_outputs(dinp.dims, dinp.dtype, dev)
    api.summary_pool(dinp, dout, stream=stream)

    def dstep():
        api.score_topk(dinp, dout, stream=stream)
        api.route_attn(dinp, dout, stream=stream)

    for _ in range(args.warmup):
        dstep()
    torch.cuda.synchronize()
    # per-call split (eager launches)
    eag = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    for s_ in range(args.steps):
        flush.zero_()
        e = eag[s_]
        e[0].record(stream)
        api.score_topk(dinp, dout, stream=stream)
        e[1].record(stream)
        api.route_attn(dinp, dout, stream=stream)
        e[2].record(stream)
    torch.cuda.synchronize()
    dper = np.array([[e[0].elapsed_time(e[1]), e[1].elapsed_time(e[2])] for e in eag])
    # graph replay of the whole step
    g = torch.cuda.CUDAGraph()
    cs = torch.cuda.Stream(device=dev)
    cs.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(cs):
        with torch.cuda.graph(g, stream=cs):
            api.score_topk(dinp, dout, stream=cs)
            api.route_attn(dinp, dout, stream=cs)
    torch.cuda.synchronize()
    for _ in range(args.warmup):
        g.replay()
    torch.cuda.synchronize()
    gev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    for s_ in range(args.steps):
        flush.zero_()
        gev[s_][0].record(stream)
        g.replay()
        gev[s_][1].record(stream)
    torch.cuda.synchronize()
    gms = np.array([e[0].elapsed_time(e[1]) for e in gev])
    d_ms = max_over_ranks(float(np.median(gms)), world, dev) if world > 1 else float(np.median(gms))
    assert rdl.rdl_last_device_status() == rdl.OK
    db = decode_bytes(dinp.dims, dout.idx.cpu().numpy())
    d_ach = db["total"] / (d_ms / 1e3) / 1e9
    del g
    return {"workload": wd.name, "ms_per_step": d_ms, "timing": "CUDA-graph replay, median",
            "eager_ms_per_step": float(np.median(dper.sum(axis=1))),
            "score_ms": float(np.median(dper[:, 0])), "attn_ms": float(np.median(dper[:, 1])),
            "query_tokens_per_s": world * 32 / (d_ms / 1e3),
            "roofline": {"bound": "hbm", "achieved": d_ach, "peak": pk["hbm_gbs"], "unit": "GB/s",
                         "frac": d_ach / pk["hbm_gbs"], "algorithmic_bytes": db["total"],
                         "traffic": DECODE_STEP_TRAFFIC,
                         "traffic_source": "ncu dram__bytes_read.sum + dram__bytes_write.sum of the six "
                                           "decode kernels, one launch each "
                                           "(profiles/launches_route_decode_128k.md)",
                         "unique_group_chunk_pairs": db["unique_pairs"],
                         "peak_source": f"hbm_gbs ({pk_kind})"}}


def stack_bench(args, dev, stream, flush, rank, world, pk, pk_kind):
    """28-layer attention stack at 128K for one 32-query decode block (every 4th layer a
    route layer: score + two-level attention over cached pre-split summaries; the other 21
    the bidirectional sliding window), all 28 layers captured in one CUDA graph and replayed;
    L2 flushed between replays (untimed).  Inputs are drawn on the device (N(0,1) K/V/Q/x,
    N(0, 0.02^2) residual weights), the shapes of the 28-layer stack workload."""
    import torch
    from diffusion_lms_b200 import api, rdl
    from diffusion_lms_b200.workloads import STACK_LAYERS, is_route_layer
    L, Lq, Hq, Hkv, d, D, r, K, w = 131072, 32, 28, 4, 128, 3584, 64, 32, 256
    C = L // 64
    gen = torch.Generator(device=dev)
    gen.manual_seed(rank_seed(5, rank))

    def rn(*shape, scale=1.0):
        return (torch.randn(*shape, generator=gen, device=dev) * scale).to(torch.bfloat16)

    q_pos = torch.arange(L - 64, L - 32, dtype=torch.int32, device=dev)[None]
    layers = []
    for layer in range(STACK_LAYERS):
        route = is_route_layer(layer)
        dm = rdl.Dims(B=1, L=L, Lq=Lq, Hq=Hq, Hkv=Hkv, d=d, D=D, r=r, K=K, w=w, lam=0.1,
                      flags=rdl.FLAG_SPLIT_SUMMARY if route else 0)
        inp = api.DeviceInputs(dm, "bf16", rn(1, Lq, Hq, d), rn(1, Hkv, L, d), rn(1, Hkv, L, d),
                               rn(1, Lq, D), rn(D, r, scale=0.02), rn(r, Hq * d, scale=0.02),
                               q_pos, rn(1, C, Hq, d) if route else None)
        out = api.alloc_outputs(dm, "bf16", dev)
        if route:
            api.summary_pool(inp, out, stream=stream)     # once per block, untimed
        layers.append((route, inp, out))
    torch.cuda.synchronize()

    def run(st):
        for route, inp, out in layers:
            if route:
                api.score_topk(inp, out, stream=st)
                api.route_attn(inp, out, stream=st)
            else:
                api.swa_attn(inp, out, stream=st)

    cs = torch.cuda.Stream(device=dev)
    cs.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(cs):
        run(cs)
    torch.cuda.synchronize()
    launches0 = rdl.launch_count()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(cs):
        with torch.cuda.graph(g, stream=cs):
            run(cs)
    launches = rdl.launch_count() - launches0
    torch.cuda.synchronize()
    for _ in range(args.warmup):
        g.replay()
    torch.cuda.synchronize()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    for s_ in range(args.steps):
        flush.zero_()
        ev[s_][0].record(stream)
        g.replay()
        ev[s_][1].record(stream)
    torch.cuda.synchronize()
    ms = float(np.median([e[0].elapsed_time(e[1]) for e in ev]))
    assert rdl.rdl_last_device_status() == rdl.OK
    del g

    def time_graph(fn, reps):
        gg = torch.cuda.CUDAGraph()
        with torch.cuda.stream(cs):
            fn(cs)
        torch.cuda.synchronize()
        with torch.cuda.stream(cs):
            with torch.cuda.graph(gg, stream=cs):
                fn(cs)
        torch.cuda.synchronize()
        for _ in range(args.warmup):
            gg.replay()
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(reps)]
        for e in evs:
            flush.zero_()
            e[0].record(stream)
            gg.replay()
            e[1].record(stream)
        torch.cuda.synchronize()
        return float(np.median([e[0].elapsed_time(e[1]) for e in evs]))

    # the same stack with the window radius of the pages' Table 3 layout (1280) on the 21
    # sliding-window layers
    for route, inp, out in layers:
        if not route:
            inp.dims.w = 1280
    ms_w1280 = time_graph(run, args.steps)
    for route, inp, out in layers:
        if not route:
            inp.dims.w = w
    # dense bidirectional attention of the same 32-query block over the whole 128K cache (one
    # layer), against the routed layer (score + two-level attention)
    route0 = next(x for x in layers if x[0])
    dense_in = api.DeviceInputs(rdl.Dims(B=1, L=L, Lq=Lq, Hq=Hq, Hkv=Hkv, d=d, D=D, r=r, K=K, w=L,
                                         lam=0.1), "bf16", route0[1].q, route0[1].k, route0[1].v,
                                route0[1].x, route0[1].w_down, route0[1].w_up, q_pos, None)
    dense_out = api.alloc_outputs(dense_in.dims, "bf16", dev)
    ms_dense = time_graph(lambda st: api.swa_attn(dense_in, dense_out, stream=st), args.steps)
    ms_route = time_graph(lambda st: (api.score_topk(route0[1], route0[2], stream=st),
                                      api.route_attn(route0[1], route0[2], stream=st)), args.steps)
    assert rdl.rdl_last_device_status() == rdl.OK
    # bytes the step must move: per route layer as decode_bytes, per window layer its K/V
    # window plus queries and outputs
    by = 0
    for route, inp, out in layers:
        if route:
            by += decode_bytes(inp.dims, out.idx.cpu().numpy())["total"]
        else:
            by += min(L, 64 + 2 * w) * Hkv * 2 * d * 2 + 2 * Lq * 2 * Hq * d
    ach = by / (ms / 1e3) / 1e9
    return {"workload": "stack_128k (28 layers: 7 route, 21 sliding window)", "ms_per_step": ms,
            "timing": "one CUDA graph of all 28 layers, median of replays, L2 flushed between",
            "kernels_per_step": launches,
            "ms_per_step_window_1280": ms_w1280,
            "dense_vs_route_one_layer": {"dense_bidirectional_ms": ms_dense, "route_ms": ms_route,
                                         "ratio": ms_dense / ms_route,
                                         "note": "attention of one layer for the 32-query block "
                                                 "over the 128K cache; the pages' 172x is the "
                                                 "whole-model per-token time"},
            "roofline": {"bound": "hbm", "achieved": ach, "peak": pk["hbm_gbs"], "unit": "GB/s",
                         "frac": ach / pk["hbm_gbs"], "algorithmic_bytes": by,
                         "peak_source": f"hbm_gbs ({pk_kind})"}}


# ----------------------------------------------------------------------------- our arm

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--ref-rows", type=int, default=96)
    ap.add_argument("--cpu-rows", type=int, default=96)
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-stack", action="store_true")
    ap.add_argument("--stack-only", action="store_true",
                    help="time only the 28-layer 128K stack (profiling aid)")
    ap.add_argument("--decode-only", action="store_true",
                    help="time only the 128K decode block (profiling aid)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))

    if args.impl == "reference":
        run_reference(args, rank)
        return

    import torch
    import torch.distributed as dist
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=300),
                                device_id=dev)

    from diffusion_lms_b200 import api, rdl
    from diffusion_lms_b200 import workloads as W

    def barrier():
        if world > 1:
            dist.barrier()

    def max_ranks(x: float) -> float:
        return max_over_ranks(x, world, dev)

    stream = torch.cuda.current_stream()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)   # > 126 MB L2

    pk, pk_kind = peaks()
    if args.stack_only:
        st_ = stack_bench(args, dev, stream, flush, rank, world, pk, pk_kind)
        if rank == 0:
            print(json.dumps({"stack_128k": st_}), flush=True)
        return
    if args.decode_only:
        dec = decode_bench(args, dev, stream, flush, rank, world, max_ranks, pk, pk_kind)
        if rank == 0:
            print(json.dumps({"decode_128k": dec}), flush=True)
        return

    # ---------------- 16K prefill route layer (the headline workload)
    wl = W.prefill_16k(seed=rank_seed(2, rank))
    inp = api.to_device(wl, dev)
    out = api.alloc_outputs(inp.dims, inp.dtype, dev)

    def step():
        api.route_layer(inp, out, stream=stream)

    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    assert rdl.rdl_last_device_status() == rdl.OK

    n_evt = 4
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(n_evt)] for _ in range(args.steps)]
    clocks = ClockSampler(torch.cuda.current_device())
    clocks.start()
    barrier()
    torch.cuda.synchronize()
    launches0 = rdl.launch_count()
    for s_ in range(args.steps):
        flush.zero_()                       # L2 flushed between timed steps (not timed)
        e = ev[s_]
        e[0].record(stream)
        api.summary_pool(inp, out, stream=stream)
        e[1].record(stream)
        api.score_topk(inp, out, stream=stream)
        e[2].record(stream)
        api.route_attn(inp, out, stream=stream)
        e[3].record(stream)
    torch.cuda.synchronize()
    launches = rdl.launch_count() - launches0
    barrier()
    clk = clocks.stop()
    per = np.array([[e[i].elapsed_time(e[i + 1]) for i in range(n_evt - 1)] for e in ev])
    ms_step_local = float(per.sum(axis=1).mean())
    ms_step = max_ranks(ms_step_local)
    content_rows = int(((np.arange(wl.dims.L) % 64) != 63).sum())
    value = job_throughput(content_rows, world, ms_step)
    call_ms = per.mean(axis=0)
    assert rdl.rdl_last_device_status() == rdl.OK

    idx_np = out.idx.cpu().numpy()
    fl_attn = attn_flops(wl.dims, None, idx_np)
    fl_score = score_flops(wl.dims)
    calls = {"rdl_summary_pool": float(call_ms[0]), "rdl_route_score_topk": float(call_ms[1]),
             "rdl_route_attn": float(call_ms[2])}
    dominant = max(calls, key=calls.get)
    if dominant == "rdl_route_attn":
        achieved = fl_attn / (call_ms[2] / 1e3) / 1e12
        roof = {"kernel": "rdl_route_attn (window + chunk launches)", "bound": "tensor",
                "achieved": achieved, "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
                "frac": achieved / pk["bf16_tflops"], "traffic": ATTN_PREFILL_TRAFFIC,
                "traffic_source": "ncu dram__bytes_read.sum + dram__bytes_write.sum of "
                                  "window_tc_kernel<1> + chunk_tc_kernel, one launch each "
                                  "(profiles/attn_traffic_route_prefill_16k.md)",
                "algorithmic_flops": fl_attn, "peak_source": f"bf16_tflops ({pk_kind}, burst)"}
    elif dominant == "rdl_route_score_topk":
        achieved = fl_score / (call_ms[1] / 1e3) / 1e12
        roof = {"kernel": "rdl_route_score_topk", "bound": "tensor", "achieved": achieved,
                "peak": pk["bf16_tflops"], "unit": "TFLOP/s", "frac": achieved / pk["bf16_tflops"],
                "traffic": None, "algorithmic_flops": fl_score,
                "peak_source": f"bf16_tflops ({pk_kind}, burst)"}
    else:
        by = 2 * 2 * wl.dims.Hkv * wl.dims.L * wl.dims.d + 4 * wl.dims.Hq * (wl.dims.L // 64) * (wl.dims.d + 1)
        achieved = by / (call_ms[0] / 1e3) / 1e9
        roof = {"kernel": "rdl_summary_pool", "bound": "hbm", "achieved": achieved,
                "peak": pk["hbm_gbs"], "unit": "GB/s", "frac": achieved / pk["hbm_gbs"],
                "traffic": None, "peak_source": f"hbm_gbs ({pk_kind})"}

    # ---------------- end to end through the public API with host buffers
    pin = {n: getattr(inp, n).cpu().pin_memory() for n in ("q", "k", "v", "x", "w_down", "w_up")}
    h_o = torch.empty_like(out.o, device="cpu").pin_memory()
    h_idx = torch.empty_like(out.idx, device="cpu").pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in pin.values())
    d2h = h_o.numel() * h_o.element_size() + h_idx.numel() * h_idx.element_size()

    def e2e_step():
        for n, t in pin.items():
            getattr(inp, n).copy_(t, non_blocking=True)
        api.route_layer(inp, out, stream=stream)
        h_o.copy_(out.o, non_blocking=True)
        h_idx.copy_(out.idx, non_blocking=True)

    for _ in range(2):
        e2e_step()
    torch.cuda.synchronize()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n_e2e = max(3, args.steps // 2)
    e0.record(stream)
    for _ in range(n_e2e):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_ranks(e0.elapsed_time(e1) / n_e2e)
    e2e = {"value": job_throughput(content_rows, world, e2e_ms), "unit": UNIT,
           "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms}
    del pin, h_o, h_idx

    # ---------------- 128K decode block (summaries cached; score + attention)
    decode = None
    if not args.no_decode:
        del inp, out
        torch.cuda.empty_cache()
        decode = decode_bench(args, dev, stream, flush, rank, world, max_ranks, pk, pk_kind)
    stack = None
    if not args.no_stack:
        torch.cuda.empty_cache()
        stack = stack_bench(args, dev, stream, flush, rank, world, pk, pk_kind)

    # ---------------- CPU baseline (rank 0, oracle on a bounded sample)
    cpu = None
    if rank == 0 and not args.no_cpu_baseline:
        dt, n = oracle_sample(wl, args.cpu_rows)
        cpu = {"value": n / dt, "unit": UNIT, "cores": 1, "kind": "oracle",
               "sample": f"all 256x28 summaries + {n} random content rows of the 16K prefill "
                         f"(fp64 NumPy, 1 BLAS thread), {dt:.1f} s"}

    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": "bf16", "data": "synthetic",
                "config": {"workload": wl.name, "L": 16384, "Hq": 28, "Hkv": 4, "d": 128, "K": 32,
                           "w": 256, "r": 64, "D": 3584, "content_rows": content_rows,
                           "l2": "flushed between timed steps (256 MB write, untimed)",
                           "parallelism": f"independent sequence per GPU x{world}"},
                "breakdown_ms": calls, "roofline": roof, "cpu_baseline": cpu, "e2e": e2e,
                "gpu_launches": launches, "clocks": clk, "decode_128k": decode, "stack_128k": stack}
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
