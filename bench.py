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
# DRAM traffic of the dominant kernels from ncu captures, each entry keyed by the hash of the
# library sources it was taken on; an entry whose hash differs from the current sources is
# stale and reported as null.
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic.json")
UNIT = "query-tokens/s"
PEAK_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def kernel_sources_sha() -> str:
    """sha256 (16 hex digits) of the CUDA library sources and the C header."""
    import glob
    import hashlib
    h = hashlib.sha256()
    files = sorted(glob.glob(os.path.join(ROOT, "diffusion_lms_b200", "csrc", "*.cu*")))
    for f in files + [os.path.join(ROOT, "include", "rdl.h")]:
        with open(f, "rb") as fh:
            h.update(os.path.basename(f).encode() + b"\0" + fh.read())
    return h.hexdigest()[:16]


def recorded_traffic(key: str):
    """(bytes per launch or None, note) for `key`, if captured on the current sources."""
    if not os.path.exists(TRAFFIC_FILE):
        return None, "no ncu capture recorded"
    with open(TRAFFIC_FILE) as f:
        rec = json.load(f).get(key)
    if rec is None:
        return None, "no ncu capture recorded for this kernel"
    if rec.get("sources_sha") != kernel_sources_sha():
        return None, "kernel sources changed since the last ncu capture"
    return float(rec["bytes"]), rec.get("what", "")


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
#
# The fp64 oracle as it stands, run on the host's cores: spawn-started worker processes (one
# BLAS thread each) pool the summaries of a share of the heads, then score, select and attend
# a share of the sampled rows.  Each worker receives the stored (bf16 bit) inputs it needs and
# calls only oracle functions; the parent measures the wall time of both phases.

MAX_ORACLE_WORKERS = 32
_ORACLE_WL = {}


def oracle_workers() -> int:
    return max(1, min(os.cpu_count() or 1, MAX_ORACLE_WORKERS))


def _oracle_init(maker, seed):
    """Worker start-up: draw the workload's stored inputs from its seed (the same bits the
    parent holds; the generator is deterministic)."""
    from diffusion_lms_b200 import workloads as W
    wl = getattr(W, maker)(seed=seed)
    _ORACLE_WL.clear()
    _ORACLE_WL.update({n: getattr(wl, n) for n in ("q", "q_mask", "k", "v", "x", "w_down", "w_up")})


def _oracle_pool_heads(task):
    from threadpoolctl import threadpool_limits
    from oracle import rdl_oracle as O
    from diffusion_lms_b200.workloads import as_f64
    heads, G = task
    with threadpool_limits(limits=1):
        qm = as_f64(_ORACLE_WL["q_mask"][:, :, heads])
        out = []
        for j, h in enumerate(heads):
            kf = as_f64(_ORACLE_WL["k"][:, h // G:h // G + 1])
            s, H, _ = O.summary_pool(qm[:, :, j:j + 1], kf)
            out.append((h, s[:, 0], H[:, 0]))
    return out


def _oracle_rows(task):
    from threadpoolctl import threadpool_limits
    from oracle import rdl_oracle as O
    from diffusion_lms_b200.workloads import as_f64
    rows, pos, s, H, kw = task
    wl = _ORACLE_WL
    with threadpool_limits(limits=1):
        qf = as_f64(wl["q"][:, rows])
        idx, z = O.route_score_topk(qf, pos, as_f64(wl["x"][:, rows]), as_f64(wl["w_down"]),
                                    as_f64(wl["w_up"]), s, H, Hkv=kw["Hkv"], K=kw["K"],
                                    w=kw["w"], lam=kw["lam"], L=kw["L"])
        O.route_attn(qf, pos, as_f64(wl["k"]), as_f64(wl["v"]), idx, z, w=kw["w"])
    return int(rows.size)


class OracleRunner:
    """Spawn-started worker pool timing the oracle on bounded samples of one workload."""

    def __init__(self, wl, maker: str, seed: int, workers: int):
        import multiprocessing as mp
        self.wl = wl
        self.workers = workers
        self.pool = mp.get_context("spawn").Pool(workers, initializer=_oracle_init,
                                                 initargs=(maker, seed))

    def close(self):
        self.pool.close()
        self.pool.join()

    def sample(self, n_rows: int, seed: int = 0):
        """(seconds, rows): all summaries of the sequence + n random content rows."""
        wl = self.wl
        dm = wl.dims
        G = dm.Hq // dm.Hkv
        rng = np.random.default_rng(seed)
        pos_all = np.arange(dm.L) if wl.q_pos is None else wl.q_pos[0]
        cand = np.flatnonzero(pos_all[:dm.Lq] % 64 != 63)
        rows = np.sort(rng.choice(cand, size=min(n_rows, cand.size), replace=False))
        nw = self.workers
        kw = dict(Hkv=dm.Hkv, K=dm.K, w=dm.w, lam=dm.lam, L=dm.L)
        t0 = time.perf_counter()
        head_sets = [list(range(dm.Hq))[i::nw] for i in range(nw)]
        s = np.zeros((dm.B, dm.Hq, dm.C, dm.d))
        H = np.zeros((dm.B, dm.Hq, dm.C))
        for part in self.pool.map(_oracle_pool_heads, [(hs, G) for hs in head_sets if hs]):
            for h, sh, Hh in part:
                s[:, h], H[:, h] = sh, Hh
        tasks = [(r, pos_all[r][None, :].astype(np.int64), s, H, kw)
                 for r in np.array_split(rows, nw) if r.size]
        done = sum(self.pool.map(_oracle_rows, tasks))
        return time.perf_counter() - t0, done


def run_reference(args, rank):
    """The oracle arm: the fp64 oracle on the host's cores, each step a bounded sample of the
    16K prefill route layer (all summaries + ref_rows content rows)."""
    from diffusion_lms_b200 import workloads as W
    if rank != 0:
        return
    wl = W.prefill_16k(seed=2)
    runner = OracleRunner(wl, "prefill_16k", 2, oracle_workers())
    n = args.ref_rows if args.ref_rows > 0 else 16 * runner.workers
    for _ in range(args.warmup):
        runner.sample(max(runner.workers, n // 8))
    times = [runner.sample(n, seed=s_)[0] for s_ in range(args.steps)]
    runner.close()
    ms = 1e3 * statistics.median(times)
    val = n / (ms / 1e3)
    sample = (f"all 256x28 summaries + {n} random content rows of the 16K prefill per step "
              f"(fp64 NumPy oracle, {runner.workers} spawn-started processes x 1 BLAS thread; "
              f"host has {os.cpu_count()} cores)")
    line = {"metric": METRIC, "value": val, "unit": UNIT, "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "impl": "reference",
            "config": {"workload": wl.name, "L": 16384, "Hq": 28, "Hkv": 4, "d": 128, "K": 32,
                       "w": 256, "r": 64, "D": 3584, "rows_per_step": n},
            "cpu_baseline": {"value": val, "unit": UNIT, "cores": runner.workers, "kind": "oracle",
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
    d_traffic, d_traffic_note = recorded_traffic("route_decode_128k.step")
    d_ach = db["total"] / (d_ms / 1e3) / 1e9
    del g
    return {"workload": wd.name, "ms_per_step": d_ms, "timing": "CUDA-graph replay, median",
            "eager_ms_per_step": float(np.median(dper.sum(axis=1))),
            "score_ms": float(np.median(dper[:, 0])), "attn_ms": float(np.median(dper[:, 1])),
            "query_tokens_per_s": world * 32 / (d_ms / 1e3),
            "roofline": {"bound": "hbm", "achieved": d_ach, "peak": pk["hbm_gbs"], "unit": "GB/s",
                         "frac": d_ach / pk["hbm_gbs"], "algorithmic_bytes": db["total"],
                         "traffic": d_traffic, "traffic_source": d_traffic_note,
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


# ----------------------------------------------------------------------------- prefill

def time_prefill(api, inp, out, stream, flush, steps, warmup, events=True):
    """Per-step CUDA-event times [steps, 3] (summary pool, score + top-K, attention) of a
    route-layer prefill step, L2 flushed before every step (untimed)."""
    import torch
    for _ in range(warmup):
        flush.zero_()
        api.route_layer(inp, out, stream=stream)
    torch.cuda.synchronize()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(steps)]
    for s_ in range(steps):
        flush.zero_()
        e = ev[s_]
        e[0].record(stream)
        api.summary_pool(inp, out, stream=stream)
        e[1].record(stream)
        api.score_topk(inp, out, stream=stream)
        e[2].record(stream)
        api.route_attn(inp, out, stream=stream)
        e[3].record(stream)
    torch.cuda.synchronize()
    return np.array([[e[i].elapsed_time(e[i + 1]) for i in range(3)] for e in ev])


def prefill_roofline(dims, idx, call_ms, step_ms, pk, pk_kind, traffic_key):
    """Roofline of the dominant call (the attention call, window + chunk launches) and of the
    whole step, both against the measured bf16 burst peak."""
    fl_attn = attn_flops(dims, None, idx)
    fl_score = score_flops(dims)
    ach = fl_attn / (call_ms[2] / 1e3) / 1e12
    traffic, note = recorded_traffic(traffic_key)
    roof = {"kernel": "rdl_route_attn (window + chunk launches)", "bound": "tensor",
            "achieved": ach, "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
            "frac": ach / pk["bf16_tflops"], "traffic": traffic,
            "traffic_source": note, "algorithmic_flops": fl_attn,
            "peak_source": f"bf16_tflops ({pk_kind}, burst)"}
    step_fl = fl_attn + fl_score
    step_ach = step_fl / (step_ms / 1e3) / 1e12
    step = {"bound": "tensor", "algorithmic_flops": step_fl, "achieved": step_ach,
            "peak": pk["bf16_tflops"], "unit": "TFLOP/s", "frac": step_ach / pk["bf16_tflops"]}
    return roof, step


def prefill_variants(args, api, rdl, wl, dev, stream, flush, world, max_ranks):
    """The 16K prefill step with the ablations of the pages' Table 6 (mean summary, no
    entropy, no residual) beside the default, each timed like the headline step."""
    import torch
    res = {}
    for name, mod in (("mean_summary", dict(flags=rdl.FLAG_MEAN_SUMMARY)),
                      ("no_entropy", dict(lam=0.0)), ("no_residual", dict(r=0))):
        inp = api.to_device(wl, dev)
        for k_, v_ in mod.items():
            setattr(inp.dims, k_, v_)
        if mod.get("r") == 0:
            inp.x = None
        out = api.alloc_outputs(inp.dims, inp.dtype, dev)
        per = time_prefill(api, inp, out, stream, flush, max(3, args.steps // 2), args.warmup)
        ms = max_ranks(float(np.median(per.sum(axis=1))))
        assert rdl.rdl_last_device_status() == rdl.OK
        res[name] = {"ms_per_step": ms, "query_tokens_per_s": world * 16128 / (ms / 1e3),
                     "breakdown_ms": {"rdl_summary_pool": float(np.median(per[:, 0])),
                                      "rdl_route_score_topk": float(np.median(per[:, 1])),
                                      "rdl_route_attn": float(np.median(per[:, 2]))}}
        del inp, out
        torch.cuda.empty_cache()
    return res


def prefill_long_bench(make_wl, args, api, rdl, dev, stream, flush, world, max_ranks, pk, pk_kind):
    """A longer route-layer prefill (64K mixture keys, 128K), timed like the 16K step."""
    import torch
    wl = make_wl()
    inp = api.to_device(wl, dev)
    out = api.alloc_outputs(inp.dims, inp.dtype, dev)
    per = time_prefill(api, inp, out, stream, flush, max(3, args.steps // 2), args.warmup)
    ms = max_ranks(float(np.median(per.sum(axis=1))))
    assert rdl.rdl_last_device_status() == rdl.OK
    call_ms = np.median(per, axis=0)
    rows = int(((np.arange(wl.dims.L) % 64) != 63).sum())
    roof, step = prefill_roofline(wl.dims, out.idx.cpu().numpy(), call_ms, ms, pk, pk_kind,
                                  f"{wl.name}.rdl_route_attn")
    res = {"workload": wl.name, "ms_per_step": ms, "query_tokens_per_s": world * rows / (ms / 1e3),
           "content_rows": rows, "timing": "median of per-step CUDA events, L2 flushed between",
           "breakdown_ms": {"rdl_summary_pool": float(call_ms[0]),
                            "rdl_route_score_topk": float(call_ms[1]),
                            "rdl_route_attn": float(call_ms[2])},
           "roofline": roof, "step_roofline": step}
    del inp, out
    torch.cuda.empty_cache()
    return res


# ----------------------------------------------------------------------------- our arm

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--ref-rows", type=int, default=0,
                    help="oracle rows per reference step (0: 16 per worker process)")
    ap.add_argument("--cpu-rows", type=int, default=0,
                    help="oracle rows of the CPU baseline (0: 48 per worker process)")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-stack", action="store_true")
    ap.add_argument("--no-64k", action="store_true")
    ap.add_argument("--no-128k", action="store_true")
    ap.add_argument("--no-variants", action="store_true")
    ap.add_argument("--stack-only", action="store_true",
                    help="time only the 28-layer 128K stack (profiling aid)")
    ap.add_argument("--decode-only", action="store_true",
                    help="time only the 128K decode block (profiling aid)")
    ap.add_argument("--prefill-only", choices=["64k", "128k", "16k_k8"], default=None,
                    help="time only this prefill workload (profiling aid)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))

    if args.impl == "reference":
        run_reference(args, rank)
        return

    # the oracle's worker processes start (spawn) before any GPU work of this process
    from diffusion_lms_b200 import workloads as W
    wl = W.prefill_16k(seed=rank_seed(2, rank))
    runner = None
    if rank == 0 and not args.no_cpu_baseline:
        runner = OracleRunner(wl, "prefill_16k", rank_seed(2, rank), oracle_workers())

    import torch
    import torch.distributed as dist
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=300),
                                device_id=dev)

    from diffusion_lms_b200 import api, rdl

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
    if args.prefill_only:
        make = {"64k": lambda: W.prefill_64k(seed=rank_seed(4, rank)),
                "128k": lambda: W.prefill_128k(seed=rank_seed(6, rank)),
                "16k_k8": lambda: W.prefill_16k_k8(seed=rank_seed(7, rank))}[args.prefill_only]
        rec = prefill_long_bench(make, args, api, rdl, dev, stream, flush, world, max_ranks, pk, pk_kind)
        if rank == 0:
            print(json.dumps({"prefill_" + args.prefill_only: rec}), flush=True)
        return

    # ---------------- 16K prefill route layer (the headline workload)
    inp = api.to_device(wl, dev)
    out = api.alloc_outputs(inp.dims, inp.dtype, dev)
    for _ in range(args.warmup):
        flush.zero_()
        api.route_layer(inp, out, stream=stream)
    torch.cuda.synchronize()
    assert rdl.rdl_last_device_status() == rdl.OK

    clocks = ClockSampler(torch.cuda.current_device())
    clocks.start()
    barrier()
    torch.cuda.synchronize()
    launches0 = rdl.launch_count()
    per = time_prefill(api, inp, out, stream, flush, args.steps, 0)
    launches = rdl.launch_count() - launches0
    barrier()
    clk = clocks.stop()
    ms_step = max_ranks(float(np.median(per.sum(axis=1))))
    content_rows = int(((np.arange(wl.dims.L) % 64) != 63).sum())
    value = job_throughput(content_rows, world, ms_step)
    call_ms = np.median(per, axis=0)
    assert rdl.rdl_last_device_status() == rdl.OK
    calls = {"rdl_summary_pool": float(call_ms[0]), "rdl_route_score_topk": float(call_ms[1]),
             "rdl_route_attn": float(call_ms[2])}
    roof, step_roof = prefill_roofline(wl.dims, out.idx.cpu().numpy(), call_ms, ms_step, pk,
                                       pk_kind, "route_prefill_16k.rdl_route_attn")

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
    del pin, h_o, h_idx, inp, out
    torch.cuda.empty_cache()

    variants = None
    if not args.no_variants:
        variants = prefill_variants(args, api, rdl, wl, dev, stream, flush, world, max_ranks)
    p64 = p128 = None
    if not args.no_64k:
        p64 = prefill_long_bench(lambda: W.prefill_64k(seed=rank_seed(4, rank)), args, api, rdl,
                                 dev, stream, flush, world, max_ranks, pk, pk_kind)
    if not args.no_128k:
        p128 = prefill_long_bench(lambda: W.prefill_128k(seed=rank_seed(6, rank)), args, api, rdl,
                                  dev, stream, flush, world, max_ranks, pk, pk_kind)
    # ---------------- 128K decode block (summaries cached; score + attention)
    decode = None
    if not args.no_decode:
        decode = decode_bench(args, dev, stream, flush, rank, world, max_ranks, pk, pk_kind)
    stack = None
    if not args.no_stack:
        torch.cuda.empty_cache()
        stack = stack_bench(args, dev, stream, flush, rank, world, pk, pk_kind)

    # ---------------- CPU baseline (rank 0, the oracle on a bounded sample, all worker cores)
    cpu = None
    if runner is not None:
        n = args.cpu_rows if args.cpu_rows > 0 else 48 * runner.workers
        dt, n = runner.sample(n)
        runner.close()
        cpu = {"value": n / dt, "unit": UNIT, "cores": runner.workers, "kind": "oracle",
               "sample": f"all 256x28 summaries + {n} random content rows of the 16K prefill "
                         f"(fp64 NumPy oracle, {runner.workers} spawn-started processes x 1 BLAS "
                         f"thread; host has {os.cpu_count()} cores), {dt:.1f} s"}

    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": "bf16", "data": "synthetic",
                "config": {"workload": wl.name, "L": 16384, "Hq": 28, "Hkv": 4, "d": 128, "K": 32,
                           "w": 256, "r": 64, "D": 3584, "content_rows": content_rows,
                           "l2": "flushed between timed steps (256 MB write, untimed)",
                           "timing": "median of per-step CUDA events",
                           "parallelism": f"independent sequence per GPU x{world}"},
                "breakdown_ms": calls, "roofline": roof, "step_roofline": step_roof,
                "cpu_baseline": cpu, "e2e": e2e,
                "gpu_launches": launches, "clocks": clk, "prefill_64k": p64, "prefill_128k": p128,
                "prefill_16k_variants": variants, "decode_128k": decode, "stack_128k": stack}
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
