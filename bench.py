#!/usr/bin/env python
"""Loki decode-attention benchmark on B200.

One step = one Loki decode layer-step (project q, low-dim score scan, top-k,
sparse attention over the selected tokens, combine) over the Llama2-13B-shaped
batched decode workload (B = 16, H = 40, D = 128, S = 4096, d = 32, k = 512,
bf16), with the KV-cache resident in HBM. Inputs are seeded synthetic
low-rank keys; the PCA basis is calibrated and the cache is filled through the
library itself (loki_calibrate_pca, loki_append_keys) before timing.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints ONE JSON line on rank 0. `value` is microseconds per layer-step for the
whole job (max-over-ranks device time / (K * N)); lower is better. The K
steps cycle through enough distinct layer caches that no step finds its
inputs in L2; a workload too small for that flushes L2 before every step and
the flushes are timed alone and taken out. Multi-GPU runs (torchrun) are
weak-scaled replicas: the path has no exchange step, so ranks share nothing
but the final max-reduction of their timings.

    python bench.py --sweep        # every sweep point: Loki and dense device times
    python bench.py --ncu-case     # a few untimed full-size calls, for ncu

--impl reference times the fp64 CPU oracle on the host cores on a bounded
sample of the same workload (this tier has no runnable upstream code).
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import re
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "Loki decode-attn µs/layer-step, HBM GB/s (% roofline), speedup vs dense"
UNIT = "us/layer-step"
FALLBACK_HBM_GBS = 6650.0
L2_FLUSH_BYTES = 256 << 20  # > 126 MB of L2


def parse_args():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="llama2-13b")
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="CPU time budget of the oracle baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--sweep", action="store_true",
                    help="time every sweep point at the Llama2-13B head shape (device-generated "
                         "inputs, Loki decode and dense decode), one JSON line per point")
    ap.add_argument("--ncu-case", action="store_true",
                    help="run a few untimed decode, dense and append steps on seeded random "
                         "full-size buffers (a small, allocation-light program for ncu)")
    return ap.parse_args()


# ---------------------------------------------------------------------------
# environment helpers
# ---------------------------------------------------------------------------

def dist_env():
    return int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)), \
        int(os.environ.get("LOCAL_RANK", 0))


def max_over_ranks(x: float, world: int, device=None) -> float:
    """Max of a per-rank number over all ranks (the job's timing is its slowest rank)."""
    if world <= 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_us_per_step(max_rank_total_ms: float, steps: int, world: int) -> float:
    """Each rank runs `steps` full layer-steps of its own replica in the timed region,
    so the job completes steps * world layer-steps in the slowest rank's time."""
    return max_rank_total_ms * 1e3 / (steps * world)


def replica_seed(base_seed: int, rank: int) -> int:
    """Replicas draw independent inputs: rank r offsets the workload seed."""
    return base_seed + 1_000_000 * rank


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def host_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML every 2 ms (from the
    start of warm-up to the end of the timed region)."""

    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown",
               0x4: "sw_power_cap", 0x80: "hw_power_brake_slowdown", 0x2: "applications_clocks_setting"}

    def __init__(self, torch_device_index: int):
        self.samples, self.reasons = [], set()
        self.ok = False
        self._stop = threading.Event()
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            uuid = str(torch.cuda.get_device_properties(torch_device_index).uuid)
            h = None
            for i in range(pynvml.nvmlDeviceGetCount()):
                hh = pynvml.nvmlDeviceGetHandleByIndex(i)
                u = pynvml.nvmlDeviceGetUUID(hh)
                u = u.decode() if isinstance(u, bytes) else u
                if u.replace("GPU-", "") == uuid.replace("GPU-", ""):
                    h = hh
            if h is None:
                h = pynvml.nvmlDeviceGetHandleByIndex(torch_device_index)
            self.nvml, self.h = pynvml, h
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # pragma: no cover - no NVML
            self.err = str(e)

    def _run(self):
        n = self.nvml
        while not self._stop.is_set():
            try:
                self.samples.append(n.nvmlDeviceGetClockInfo(self.h, n.NVML_CLOCK_SM))
                mask = n.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for bit, name in self.REASONS.items():
                    if mask & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(0.002)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0,
                    "note": getattr(self, "err", "no samples")}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


def traffic_from_profiles(kernel: str, workload: str):
    """DRAM bytes per launch from a committed ncu summary, if its source hash is current."""
    path = os.path.join(ROOT, "profiles", f"{kernel}_{workload}.md")
    if not os.path.exists(path):
        return None
    txt = open(path).read()
    m_t = re.search(r"traffic_bytes_per_launch:\s*([0-9.e+]+)", txt)
    m_h = re.search(r"source_sha256:\s*([0-9a-f]{64})", txt)
    m_f = re.search(r"source_file:\s*(\S+)", txt)
    if not (m_t and m_h and m_f):
        return None
    src = os.path.join(ROOT, m_f.group(1))
    if not os.path.exists(src):
        return None
    if hashlib.sha256(open(src, "rb").read()).hexdigest() != m_h.group(1):
        return None
    return float(m_t.group(1))


# ---------------------------------------------------------------------------
# CPU oracle baseline (rank 0 only)
# ---------------------------------------------------------------------------

def oracle_sample_rows(wl, n_rows, seed=11):
    """Host inputs of a seeded sample of (b, h_q) rows: q, K~ (oracle-rotated), V, P."""
    import numpy as np

    import oracle
    import workloads
    rows = workloads.sample_rows(wl, n_rows, seed)
    cache = {}
    out = []
    for b, h in rows:
        hk = h // wl.G
        if ("P", hk) not in cache:
            R = workloads.rotation(wl, hk)
            P, _ = oracle.calibrate_pca(workloads.calibration_keys(wl, hk, R))
            cache[("P", hk)] = (R, P.astype(np.float32).astype(np.float64))
        R, P = cache[("P", hk)]
        if (b, hk) not in cache:
            K = workloads.keys_block(wl, b, hk, R)
            cache[(b, hk)] = (oracle.rotate_keys(K, P, wl.dtype),
                              workloads.values_block(wl, b, hk).astype(np.float64))
        Kt, V = cache[(b, hk)]
        out.append((workloads.query_vec(wl, b, h, R).astype(np.float64), Kt, V, P))
    return out


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return 1


def cpu_oracle_time(wl, seconds: float, threads: int = 0):
    """Time oracle.loki_decode_row over sampled rows; returns (us per layer-step, info).
    threads > 0 limits the BLAS threads for the measurement."""
    import contextlib

    import oracle
    sample = oracle_sample_rows(wl, 8)
    limit = contextlib.nullcontext()
    if threads:
        try:
            from threadpoolctl import threadpool_limits
            limit = threadpool_limits(limits=threads, user_api="blas")
        except Exception:
            pass
    per_row = []
    with limit:
        used = blas_threads()
        t_end = time.perf_counter() + seconds
        i = 0
        while (time.perf_counter() < t_end or len(per_row) < 4) and len(per_row) < 100000:
            q, Kt, V, P = sample[i % len(sample)]
            t0 = time.perf_counter()
            oracle.loki_decode_row(q, Kt, V, P, wl.d, wl.k, wl.scale)
            per_row.append(time.perf_counter() - t0)
            i += 1
    mean_row = sum(per_row) / len(per_row)
    rows = wl.B * wl.H_q
    return mean_row * rows * 1e6, {
        "rows_timed": len(per_row), "distinct_rows": len(sample),
        "cores": used, "host_cores": host_cores()}


# ---------------------------------------------------------------------------
# GPU benchmark
# ---------------------------------------------------------------------------

def build_gpu_inputs(wl, dev, rank):
    """Seeded inputs on the device; P and the rotated cache come from the library."""
    import torch

    import sparse_attention_decode_loki_b200 as loki
    import workloads
    wl_r = wl.with_(seed=replica_seed(wl.seed, rank))
    g = workloads.generate(wl_r)
    dt = torch.bfloat16 if wl.dtype == "bf16" else torch.float32
    K_cal = torch.from_numpy(g["K_cal"]).to(dev).to(dt)
    P, eig = loki.loki_calibrate_pca(K_cal)
    S_max = wl.S
    Kt = torch.empty((wl.B, wl.H_kv, S_max, wl.D), dtype=dt, device=dev)
    V = torch.empty_like(Kt)
    # low-dimensional key plane: a contiguous copy of the first d rotated columns
    Kt_lo = torch.empty((wl.B, wl.H_kv, S_max, wl.d), dtype=dt, device=dev)
    K_raw = torch.from_numpy(g.pop("K")).to(dev).to(dt)
    V_raw = torch.from_numpy(g.pop("V")).to(dev).to(dt)
    loki.loki_append_keys(K_raw, V_raw, P, Kt, V, 0, Kt_lo=Kt_lo)
    # the new token of the timed append (one per sequence and KV head)
    K_new = K_raw[:, :, -1:].contiguous()
    V_new = V_raw[:, :, -1:].contiguous()
    del K_raw, V_raw
    q = torch.from_numpy(g["q"]).to(dev).to(dt)
    torch.cuda.synchronize()
    return {"q": q, "Kt": Kt, "V": V, "Kt_lo": Kt_lo, "P": P, "eig": eig, "K_new": K_new,
            "V_new": V_new, "q_host": g["q"]}


L2_BYTES = 126 << 20


def layer_count(hot_bytes: int, layer_bytes: int, free_bytes: int, max_layers: int = 64) -> int:
    """Distinct layer caches to cycle through so that consecutive steps never
    find their inputs in L2: enough layers that the others' hot bytes between
    two visits of a layer are at least twice the L2 size, within half the
    free device memory. 1 means the steps must flush L2 instead."""
    if hot_bytes <= 0:
        return 1
    need = 1 + -(-2 * L2_BYTES // hot_bytes)
    if hot_bytes >= L2_BYTES:
        need = max(2, min(need, 4))
    fit = int(0.5 * free_bytes // max(layer_bytes, 1))
    n = min(need, fit, max_layers)
    return n if n >= need else 1


NOMINAL_HBM_BYTES = 180e9


def workload_config(wl, n_layers: int, world: int) -> dict:
    """The `config` object of the JSON line (both arms)."""
    return {"workload": wl.name, "B": wl.B, "H_q": wl.H_q, "H_kv": wl.H_kv, "D": wl.D, "S": wl.S,
            "d": wl.d, "k": wl.k, "cache_dtype": wl.dtype,
            "cache_layout": "rotated K rows + contiguous d-column key plane",
            "layers": n_layers,
            "l2": ("inputs larger than L2: consecutive steps cycle through "
                   f"{n_layers} distinct layer caches ({wl.loki_bytes() / 1e6:.1f} MB of "
                   "hot bytes each), no flush" if n_layers > 1 else
                   "flushed before every step (256 MiB write, then a 256 MiB read so "
                   "no dirty lines remain), flush excluded"),
            "timing": "K consecutive layer-steps (one loki_decode_attention_plane call "
                      "each) captured in CUDA graphs and replayed back to back, CUDA "
                      "events on the launching stream around all K",
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU"}


def layer_bytes_of(wl) -> int:
    return wl.elem_bytes * wl.B * wl.H_kv * wl.S * (2 * wl.D + wl.d)


def actual_bytes_per_step(workload: str):
    """DRAM bytes of one decode step as ncu counted them (sum over the step's
    kernels), from the committed profile summaries whose sources still match."""
    names = ["score_plane", "topk", "sparse_attn", "project_query"]
    vals = [traffic_from_profiles(n, workload) for n in names]
    if any(v is None for v in vals):
        return None
    return sum(vals)


def count_launches(fn) -> int:
    """Kernels of this library that one call of fn launches (CUPTI activity
    records through the torch profiler, taken once before any timing)."""
    import torch
    from torch.profiler import ProfilerActivity, profile
    torch.cuda.synchronize()
    with profile(activities=[ProfilerActivity.CUDA]) as prof:
        fn()
        torch.cuda.synchronize()
    return sum(1 for e in prof.events()
               if e.device_type.name == "CUDA" and "loki::" in e.name)


def run_ours(args):
    import torch

    import sparse_attention_decode_loki_b200 as loki
    import workloads

    rank, world, local = dist_env()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=dev)
    wl = workloads.get(args.workload)
    inp = build_gpu_inputs(wl, dev, rank)
    q, Kt, V, P, Kt_lo = inp["q"], inp["Kt"], inp["V"], inp["P"], inp["Kt_lo"]
    B, H_q, H_kv, S, D, d, k = wl.B, wl.H_q, wl.H_kv, wl.S, wl.D, wl.d, wl.k
    e = wl.elem_bytes
    stream = torch.cuda.current_stream(dev)
    cap = torch.cuda.Stream(dev)

    # ---- layers: distinct copies of the cache, so consecutive steps never hit L2 --
    free, _ = torch.cuda.mem_get_info(dev)
    n_layers = layer_count(wl.loki_bytes(), layer_bytes_of(wl), free)
    layers = [(Kt, V, Kt_lo)] + [(Kt.clone(), V.clone(), Kt_lo.clone())
                                 for _ in range(n_layers - 1)]
    outs = [torch.empty_like(q) for _ in range(n_layers)]
    idxs = [torch.empty((B, H_q, k), dtype=torch.int32, device=dev) for _ in range(n_layers)]
    ws = torch.empty(loki.loki_decode_workspace_size(B, H_q, H_kv, S, D, d, k),
                     dtype=torch.uint8, device=dev)
    out, idx = outs[0], idxs[0]

    flush_w = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    flush_r = torch.zeros(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    flush_sink = torch.empty((), dtype=torch.float32, device=dev)

    def flush():
        """Evict L2: write 256 MiB, then read another 256 MiB so the dirty lines
        are written back here and the next call starts with a cold, clean L2."""
        flush_w.zero_()
        torch.sum(flush_r, dim=0, out=flush_sink)

    def decode_layer(j):
        Ktj, Vj, Kloj = layers[j]
        loki.loki_decode_attention(q, Ktj, Vj, P, S, d, k, wl.scale, out=outs[j],
                                   selected_idx=idxs[j], workspace=ws, Kt_lo=Kloj)

    def capture(body):
        g_ = torch.cuda.CUDAGraph()
        cap.wait_stream(stream)
        with torch.cuda.stream(cap):
            with torch.cuda.graph(g_, stream=cap):
                body()
        stream.wait_stream(cap)
        torch.cuda.synchronize()
        return g_

    def step_graphs(fn_layer, steps):
        """Graphs that together run exactly `steps` consecutive layer-steps
        (layers cycling; an L2 flush before each step when there is one layer)."""
        def body(n):
            def run():
                for i in range(n):
                    if n_layers == 1:
                        flush()
                    fn_layer(i % n_layers)
            return run
        per = max(n_layers, 1)
        plan = [per] * (steps // per) + ([steps % per] if steps % per else [])
        graphs = {n_: capture(body(n_)) for n_ in set(plan)}
        return plan, graphs

    def diff_us(fn, R=8, reps=5):
        """Device time of one call with a cold L2, without per-replay launch
        overhead: a graph of R x (L2 flush, call) minus one of R x (L2 flush)."""
        fn()
        torch.cuda.synchronize()

        def with_call():
            for _ in range(R):
                flush()
                fn()

        def flush_only():
            for _ in range(R):
                flush()

        gw, gf = capture(with_call), capture(flush_only)
        tw, tf = [], []
        for i in range(reps + 1):
            for g_, t_ in ((gw, tw), (gf, tf)):
                e0 = torch.cuda.Event(enable_timing=True)
                e1 = torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                g_.replay()
                e1.record(stream)
                torch.cuda.synchronize()
                if i:
                    t_.append(e0.elapsed_time(e1))
        del gw, gf
        return (statistics.median(tw) - statistics.median(tf)) * 1e3 / R

    # ---- the timed region: exactly K layer-steps ------------------------------------
    decode_layer(0)
    torch.cuda.synchronize()
    launches_per_step = count_launches(lambda: decode_layer(0))
    plan, graphs = step_graphs(decode_layer, args.steps)
    wplan, wgraphs = step_graphs(decode_layer, max(args.warmup, 1))
    with ClockSampler(local) as clk:
        for n_ in wplan:
            wgraphs[n_].replay()
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for n_ in plan:
            graphs[n_].replay()
        e1.record(stream)
        torch.cuda.synchronize()
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize()
    timed_ms = e0.elapsed_time(e1)
    del graphs, wgraphs
    if n_layers == 1:
        # one layer: every step began with an L2 flush; time the same number of
        # flushes alone and take them out (they are not part of the step)
        fplan, fgraphs = step_graphs(lambda j: None, args.steps)
        g0 = torch.cuda.Event(enable_timing=True)
        g1_ = torch.cuda.Event(enable_timing=True)
        g0.record(stream)
        for n_ in fplan:
            fgraphs[n_].replay()
        g1_.record(stream)
        torch.cuda.synchronize()
        timed_ms -= g0.elapsed_time(g1_)
        del fgraphs
    total_ms = max_over_ranks(timed_ms, world, dev)
    us_per_step_rank = total_ms * 1e3 / args.steps
    value = whole_job_us_per_step(total_ms, args.steps, world)

    # ---- the same step, one layer, as a single graph replay after an L2 flush -------
    g1 = capture(lambda: decode_layer(0))
    single = []
    for i in range(min(200, max(20, args.steps)) + 3):
        flush()
        a0 = torch.cuda.Event(enable_timing=True)
        a1 = torch.cuda.Event(enable_timing=True)
        a0.record(stream)
        g1.replay()
        a1.record(stream)
        torch.cuda.synchronize()
        if i >= 3:
            single.append(a0.elapsed_time(a1) * 1e3)
    del g1
    decode_device_us = diff_us(lambda: decode_layer(0))

    # ---- per-kernel device times: each step entry point alone, after an L2 flush ----
    q_rot = torch.empty((B, H_q, D), dtype=torch.float32, device=dev)
    scores = torch.empty((B, H_q, S), dtype=torch.float32, device=dev)
    sp_ws = torch.empty(loki.loki_sparse_attention_workspace_size(B, H_q, k, D), dtype=torch.uint8,
                        device=dev)
    loki.loki_project_query(q, P, q_rot)
    loki.loki_score_lowdim(q_rot, Kt_lo, S, d, scores)
    loki.loki_topk(scores, k, idx)
    comps = {
        "project_query": lambda: loki.loki_project_query(q, P, q_rot),
        "score_lowdim": lambda: loki.loki_score_lowdim(q_rot, Kt_lo, S, d, scores),
        "topk": lambda: loki.loki_topk(scores, k, idx),
        "sparse_attention+combine": lambda: loki.loki_sparse_attention(q_rot, Kt, V, idx, S,
                                                                       wl.scale, out, sp_ws),
    }
    kern_us = {n_: diff_us(f_) for n_, f_ in comps.items()}

    # ---- the single-kernel variant, where the shape fits it -----------------------
    fused_us = None
    try:
        loki.loki_decode_attention_fused(q, Kt, V, Kt_lo, P, S, d, k, wl.scale, out=out,
                                         selected_idx=idx)
        torch.cuda.synchronize()
        fused_us = diff_us(lambda: loki.loki_decode_attention_fused(
            q, Kt, V, Kt_lo, P, S, d, k, wl.scale, out=out, selected_idx=idx))
    except loki.LokiError:
        pass

    # ---- dense baseline on the same caches, timed like the headline ---------------
    q_rot_dt = loki.loki_project_query(q, P).to(q.dtype)
    dws = torch.empty(loki.dense_decode_workspace_size(B, H_q, H_kv, S, D), dtype=torch.uint8,
                      device=dev)
    dout = torch.empty_like(q)

    def dense_layer(j):
        loki.dense_decode_attention(q_rot_dt, layers[j][0], layers[j][1], S, wl.scale, dout, dws)

    dense_layer(0)
    dsteps = max(n_layers, min(args.steps, 200))
    dplan, dgraphs = step_graphs(dense_layer, dsteps)
    for n_ in dplan[:1]:
        dgraphs[n_].replay()
    torch.cuda.synchronize()
    d0 = torch.cuda.Event(enable_timing=True)
    d1 = torch.cuda.Event(enable_timing=True)
    d0.record(stream)
    for n_ in dplan:
        dgraphs[n_].replay()
    d1.record(stream)
    torch.cuda.synchronize()
    dense_ms = d0.elapsed_time(d1)
    del dgraphs
    if n_layers == 1:  # take the flushes out, as for the headline
        fplan, fgraphs = step_graphs(lambda j: None, dsteps)
        d0.record(stream)
        for n_ in fplan:
            fgraphs[n_].replay()
        d1.record(stream)
        torch.cuda.synchronize()
        dense_ms -= d0.elapsed_time(d1)
        del fgraphs
    dense_us = dense_ms * 1e3 / dsteps
    dense_device_us = diff_us(lambda: dense_layer(0))

    # ---- append of one new token per (sequence, KV head), device time ---------------
    Kt_app = torch.empty((B, H_kv, 8, D), dtype=q.dtype, device=dev)
    V_app = torch.empty_like(Kt_app)
    append_us = diff_us(lambda: loki.loki_append_keys(inp["K_new"], inp["V_new"], P, Kt_app,
                                                      V_app, 0))

    # ---- the step with its append folded in: the last token re-appended -----------
    pos = S - 1

    def decode_step():
        loki.loki_decode_step(q, inp["K_new"], inp["V_new"], P, Kt, V, pos, d, k, wl.scale,
                              out=out, selected_idx=idx, workspace=ws, Kt_lo=Kt_lo)

    def append_then_decode():
        loki.loki_append_keys(inp["K_new"], inp["V_new"], P, Kt, V, pos, Kt_lo=Kt_lo)
        loki.loki_decode_attention(q, Kt, V, P, S, d, k, wl.scale, out=out, selected_idx=idx,
                                   workspace=ws, Kt_lo=Kt_lo)

    step_us = diff_us(decode_step)
    append_decode_us = diff_us(append_then_decode)

    # ---- offline PCA calibration of one layer (all KV heads), device time --------
    K_cal = torch.from_numpy(workloads.generate(wl, with_keys=False)["K_cal"]).to(dev).to(q.dtype)
    Pc = torch.empty_like(P)
    eigc = torch.empty((H_kv, D), dtype=torch.float32, device=dev)
    cws = torch.empty(loki.loki_calibrate_workspace_size(K_cal.shape[0], H_kv, D),
                      dtype=torch.uint8, device=dev)
    loki.loki_calibrate_pca(K_cal, Pc, eigc, cws)
    torch.cuda.synchronize()
    c0 = torch.cuda.Event(enable_timing=True)
    c1 = torch.cuda.Event(enable_timing=True)
    c0.record(stream)
    for _ in range(3):
        loki.loki_calibrate_pca(K_cal, Pc, eigc, cws)
    c1.record(stream)
    torch.cuda.synchronize()
    calibrate_ms = c0.elapsed_time(c1) / 3

    # ---- end to end through the public API with host buffers ---------------------
    q_pin = torch.from_numpy(inp["q_host"]).to(q.dtype).pin_memory()
    out_pin = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    idx_pin = torch.empty(idx.shape, dtype=idx.dtype).pin_memory()

    def e2e_step(j):
        if n_layers == 1:
            flush()
        q.copy_(q_pin, non_blocking=True)
        decode_layer(j)
        out_pin.copy_(outs[j], non_blocking=True)
        idx_pin.copy_(idxs[j], non_blocking=True)

    n_e2e = max(20, min(args.steps, 1000))
    for j in range(3):
        e2e_step(j % n_layers)
    torch.cuda.synchronize()
    f0 = torch.cuda.Event(enable_timing=True)
    f1 = torch.cuda.Event(enable_timing=True)
    f0.record(stream)
    for i in range(n_e2e):
        e2e_step(i % n_layers)
    f1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = f0.elapsed_time(f1) / n_e2e
    if n_layers == 1:  # the flushes are not part of the step
        fl = capture(lambda: flush())
        c0 = torch.cuda.Event(enable_timing=True)
        c1 = torch.cuda.Event(enable_timing=True)
        c0.record(stream)
        for _ in range(50):
            fl.replay()
        c1.record(stream)
        torch.cuda.synchronize()
        e2e_ms -= c0.elapsed_time(c1) / 50
        del fl
    e2e_us = max_over_ranks(e2e_ms * 1e3, world, dev)
    h2d = q_pin.numel() * q_pin.element_size()
    d2h = out_pin.numel() * out_pin.element_size() + idx_pin.numel() * idx_pin.element_size()

    # ---- roofline of the dominant kernel and of the whole step -------------------
    peak, peak_kind = load_peaks()
    alg = {
        "score_lowdim": e * B * H_kv * S * d,
        "sparse_attention+combine": e * B * H_q * 2 * k * D,
    }
    dom = max(alg, key=lambda n: kern_us[n])
    achieved = alg[dom] / (kern_us[dom] * 1e-6) / 1e9
    step_bytes = wl.loki_bytes()
    prof_name = {"score_lowdim": "score_plane", "sparse_attention+combine": "sparse_attn"}[dom]
    traffic = traffic_from_profiles(prof_name, wl.name)
    actual = actual_bytes_per_step(wl.name)

    res = {
        "metric": METRIC,
        "value": round(value, 3),
        "unit": UNIT,
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(us_per_step_rank / 1e3, 6),
        "higher_is_better": False,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16" if wl.dtype == "bf16" else "f32",
        "data": "synthetic (seeded low-rank keys, N(0,1) values; PCA and cache built by the library)",
        "config": workload_config(wl, n_layers, world),
        "timing_detail": "single_layer_*: one call per graph replay after an L2 flush; "
                         "*_device_us and kernels_us: graph of 8 x (L2 flush, call) minus "
                         "graph of 8 x (L2 flush), over 8",
        "tokens_per_s": round(B * world * 1e6 / us_per_step_rank, 1),
        "hbm_gbs": round(step_bytes / (us_per_step_rank * 1e-6) / 1e9, 1),
        "hbm_frac_of_" + peak_kind: round(step_bytes / (us_per_step_rank * 1e-6) / 1e9 / peak, 4),
        "hbm_frac_actual_of_" + peak_kind: (None if actual is None else round(
            actual / (us_per_step_rank * 1e-6) / 1e9 / peak, 4)),
        "actual_bytes_per_step": actual,
        "ideal_bytes_per_step": step_bytes,
        "moved_bytes_per_step": wl.moved_bytes(),
        "single_layer_graph_us": round(statistics.mean(single), 3),
        "decode_device_us": round(decode_device_us, 3),
        "fused_kernel_device_us": None if fused_us is None else round(fused_us, 3),
        "dense_us": round(dense_us, 3),
        "dense_device_us": round(dense_device_us, 3),
        "speedup_vs_dense": round(dense_us / us_per_step_rank, 3),
        "append_device_us": round(append_us, 3),
        "decode_step_with_append_device_us": round(step_us, 3),
        "append_then_decode_device_us": round(append_decode_us, 3),
        "calibrate_layer_ms": {"value": round(calibrate_ms, 3), "kv_heads": H_kv,
                               "keys_per_head": int(K_cal.shape[0])},
        "kernels_us": {n_: round(v_, 3) for n_, v_ in kern_us.items()},
        "roofline": {"bound": "hbm", "kernel": dom, "achieved": round(achieved, 1),
                     "peak": peak, "peak_kind": peak_kind, "unit": "GB/s",
                     "frac": round(achieved / peak, 4), "traffic": traffic,
                     "algorithmic_bytes": alg[dom]},
        "e2e": {"value": round(e2e_us / world, 3), "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h},
        "gpu_launches": launches_per_step * args.steps,
        "gpu_launches_per_step": launches_per_step,
        "clocks": clk.summary(),
    }
    if rank == 0 and not args.no_cpu_baseline:
        cpu_us, info = cpu_oracle_time(wl, args.cpu_seconds)
        cpu1_us, info1 = cpu_oracle_time(wl, min(4.0, args.cpu_seconds), threads=1)
        res["cpu_baseline"] = {"value": round(cpu_us, 1), "unit": UNIT, "cores": info["cores"],
                               "kind": "oracle",
                               "sample": f"extrapolated: {info['rows_timed']} timed (batch, head) "
                                         f"rows drawn from {info['distinct_rows']} seeded rows "
                                         f"of {wl.name}, mean row time x B*H_q = {B * H_q}",
                               "host_cores": info["host_cores"],
                               "one_thread_value": round(cpu1_us, 1)}
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    if rank == 0:
        print(json.dumps(res), flush=True)


def run_reference(args):
    """The fp64 oracle on the host cores as the reference arm: each step runs
    B * H_q row decodes (cycling through seeded sampled rows of the workload)
    when the whole run fits in about two minutes, else a bounded sample of
    rows per step, scaled to B * H_q and labelled as extrapolated."""
    rank, world, _ = dist_env()
    if rank != 0:
        return
    import workloads
    wl = workloads.get(args.workload)
    import oracle
    sample = oracle_sample_rows(wl, 8)
    rows_full = wl.B * wl.H_q
    t0 = time.perf_counter()
    for q, Kt, V, P in sample:
        oracle.loki_decode_row(q, Kt, V, P, wl.d, wl.k, wl.scale)
    t_row = (time.perf_counter() - t0) / len(sample)
    budget_s = 120.0
    steps_all = args.steps + args.warmup
    if steps_all * rows_full * t_row <= budget_s:
        rows_per_step = rows_full
    else:
        rows_per_step = max(1, int(budget_s / (steps_all * t_row)))

    def step(i):
        for j in range(rows_per_step):
            q, Kt, V, P = sample[(i * rows_per_step + j) % len(sample)]
            oracle.loki_decode_row(q, Kt, V, P, wl.d, wl.k, wl.scale)

    for i in range(args.warmup):
        step(i)
    t0 = time.perf_counter()
    for i in range(args.steps):
        step(i)
    dt = time.perf_counter() - t0
    us = dt / args.steps * (rows_full / rows_per_step) * 1e6
    if rows_per_step == rows_full:
        sample_txt = (f"full steps: {rows_full} (batch, head) row decodes per step, cycling "
                      f"through {len(sample)} seeded rows of {wl.name}")
    else:
        sample_txt = (f"extrapolated: {rows_per_step} (batch, head) rows per step from "
                      f"{len(sample)} seeded rows of {wl.name}, scaled by B*H_q / "
                      f"{rows_per_step} = {rows_full / rows_per_step:.1f}")
    n_layers = layer_count(wl.loki_bytes(), layer_bytes_of(wl), int(NOMINAL_HBM_BYTES))
    res = {
        "metric": METRIC, "value": round(us, 1), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(us / 1e3, 3),
        "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded low-rank keys)", "impl": "reference",
        "config": workload_config(wl, n_layers, world),
        "cpu_baseline": {"value": round(us, 1), "unit": UNIT, "cores": blas_threads(),
                         "kind": "oracle", "sample": sample_txt},
        "e2e": {"value": round(us, 1), "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(res), flush=True)


def run_ncu_case(args):
    """Each hot-path kernel a few times on the workload's full-size buffers, nothing timed."""
    import torch

    import sparse_attention_decode_loki_b200 as loki
    import workloads
    wl = workloads.get(args.workload)
    dev = torch.device("cuda", 0)
    dt = torch.bfloat16 if wl.dtype == "bf16" else torch.float32
    g = torch.Generator(device=dev)
    g.manual_seed(wl.seed)
    Kt = torch.randn((wl.B, wl.H_kv, wl.S, wl.D), generator=g, device=dev, dtype=dt)
    V = torch.randn((wl.B, wl.H_kv, wl.S, wl.D), generator=g, device=dev, dtype=dt)
    q = torch.randn((wl.B, wl.H_q, wl.D), generator=g, device=dev, dtype=dt)
    Kt_lo = Kt[..., : wl.d].contiguous()
    # an orthonormal basis from the host (seeded), so the launch list holds only this library
    import numpy as np
    Pn = np.linalg.qr(np.random.default_rng(wl.seed).standard_normal((wl.H_kv, wl.D, wl.D)))[0]
    P = torch.from_numpy(np.ascontiguousarray(Pn, dtype=np.float32)).to(dev)
    for _ in range(max(1, args.steps)):
        loki.loki_decode_attention(q, Kt, V, P, wl.S, wl.d, wl.k, wl.scale, Kt_lo=Kt_lo)
    for _ in range(2):
        loki.dense_decode_attention(q, Kt, V, wl.S, wl.scale)
    Kc = torch.empty((wl.B, wl.H_kv, 8, wl.D), dtype=dt, device=dev)
    loki.loki_append_keys(Kt[:, :, :1].contiguous(), V[:, :, :1].contiguous(), P, Kc,
                          torch.empty_like(Kc), 0)
    torch.cuda.synchronize()


def device_inputs(wl, dev, seed: int, S_cap: int):
    """Sweep-point inputs drawn on the device with the workload's recipe
    (low-rank keys K = Z diag(sigma) R^T + N(0, 0.01^2) per KV head, queries
    alike, V ~ N(0, 1)); the PCA basis and the rotated cache with its key
    plane come from the library. Timing inputs only: parity is checked by the
    tests on the host generator's streams."""
    import torch

    import sparse_attention_decode_loki_b200 as loki
    import workloads
    gen = torch.Generator(device=dev)
    gen.manual_seed(seed)
    dt = torch.bfloat16
    D, H_kv, S = wl.D, wl.H_kv, S_cap
    sigma = torch.exp(-torch.arange(D, dtype=torch.float32, device=dev) / wl.tau)
    Rt = [torch.from_numpy(workloads.rotation(wl, h).T.copy()).float().to(dev) for h in range(H_kv)]

    def lowrank(n, h):
        z = torch.randn((n, D), generator=gen, device=dev) * sigma
        return z @ Rt[h] + wl.noise_std * torch.randn((n, D), generator=gen, device=dev)

    K_cal = torch.stack([lowrank(wl.n_cal, h) for h in range(H_kv)], dim=1).to(dt)
    P, _ = loki.loki_calibrate_pca(K_cal)
    Kt = torch.empty((wl.B, H_kv, S, D), dtype=dt, device=dev)
    V = torch.empty_like(Kt)
    Kt_lo = torch.empty((wl.B, H_kv, S, wl.d), dtype=dt, device=dev)
    for b in range(wl.B):
        Kb = torch.stack([lowrank(S, h) for h in range(H_kv)]).to(dt)[None]
        Vb = torch.randn((1, H_kv, S, D), generator=gen, device=dev).to(dt)
        loki.loki_append_keys(Kb, Vb, P, Kt[b:b + 1], V[b:b + 1], 0, Kt_lo=Kt_lo[b:b + 1])
        del Kb, Vb
    q = torch.stack([torch.stack([lowrank(1, h // wl.G)[0] for h in range(wl.H_q)])
                     for _ in range(wl.B)]).to(dt)
    torch.cuda.synchronize()
    return q, Kt, V, Kt_lo, P


def run_sweep(args):
    """Every sweep point: Loki decode and dense decode device times (graph of
    8 x (L2 flush, call) minus 8 x (L2 flush)), ideal-bytes HBM fraction,
    tokens/s and the speedup over dense. S is capped where a point's cache and
    key plane do not fit in 85 % of free device memory."""
    import torch

    import sparse_attention_decode_loki_b200 as loki
    import workloads
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    cap = torch.cuda.Stream(dev)
    peak, peak_kind = load_peaks()
    flush_w = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    flush_r = torch.zeros(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    sink = torch.empty((), dtype=torch.float32, device=dev)

    def flush():
        flush_w.zero_()
        torch.sum(flush_r, dim=0, out=sink)

    def diff_us(fn, R=8, reps=3):
        fn()
        torch.cuda.synchronize()

        def graph(body):
            g_ = torch.cuda.CUDAGraph()
            cap.wait_stream(stream)
            with torch.cuda.stream(cap):
                with torch.cuda.graph(g_, stream=cap):
                    body()
            stream.wait_stream(cap)
            torch.cuda.synchronize()
            return g_

        def with_call():
            for _ in range(R):
                flush()
                fn()

        def flush_only():
            for _ in range(R):
                flush()

        gw, gf = graph(with_call), graph(flush_only)
        tw, tf = [], []
        for i in range(reps + 1):
            for g_, t_ in ((gw, tw), (gf, tf)):
                e0 = torch.cuda.Event(enable_timing=True)
                e1 = torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                g_.replay()
                e1.record(stream)
                torch.cuda.synchronize()
                if i:
                    t_.append(e0.elapsed_time(e1))
        del gw, gf
        return (statistics.median(tw) - statistics.median(tf)) * 1e3 / R

    pts = [p for p in workloads.sweep_points()
           if args.workload in ("llama2-13b", "sweep") or p.name.startswith(args.workload)]
    for wl in pts:
        free, _ = torch.cuda.mem_get_info(dev)
        per_token = wl.elem_bytes * wl.B * wl.H_kv * (2 * wl.D + wl.d) + 4 * wl.B * wl.H_q
        S = wl.S
        if S * per_token > 0.85 * free:
            S = int(0.85 * free // per_token) // 4096 * 4096
        k = S * wl.k // wl.S
        w2 = wl.with_(S=S, k=k)
        q, Kt, V, Kt_lo, P = device_inputs(w2, dev, w2.seed, S)
        B, H_q, H_kv, D, d = w2.B, w2.H_q, w2.H_kv, w2.D, w2.d
        out = torch.empty_like(q)
        idx = torch.empty((B, H_q, k), dtype=torch.int32, device=dev)
        ws = torch.empty(loki.loki_decode_workspace_size(B, H_q, H_kv, S, D, d, k),
                         dtype=torch.uint8, device=dev)

        def decode():
            loki.loki_decode_attention(q, Kt, V, P, S, d, k, w2.scale, out=out, selected_idx=idx,
                                       workspace=ws, Kt_lo=Kt_lo)

        loki_us = diff_us(decode)
        q_rot = loki.loki_project_query(q, P).to(q.dtype)
        dws = torch.empty(loki.dense_decode_workspace_size(B, H_q, H_kv, S, D), dtype=torch.uint8,
                          device=dev)
        dout = torch.empty_like(q)
        dense_us = diff_us(lambda: loki.dense_decode_attention(q_rot, Kt, V, S, w2.scale, dout, dws))
        ideal = w2.loki_bytes()
        dense_bytes = w2.elem_bytes * B * H_kv * 2 * S * D
        print(json.dumps({
            "point": wl.name, "B": B, "S": S, "S_capped": S != wl.S, "d": d, "k": k,
            "loki_device_us": round(loki_us, 3), "dense_device_us": round(dense_us, 3),
            "speedup_vs_dense": round(dense_us / loki_us, 3),
            "tokens_per_s": round(B * 1e6 / loki_us, 1),
            "ideal_bytes": ideal, "hbm_frac_ideal_of_" + peak_kind:
                round(ideal / (loki_us * 1e-6) / 1e9 / peak, 4),
            "moved_bytes": w2.moved_bytes(), "hbm_frac_moved_of_" + peak_kind:
                round(w2.moved_bytes() / (loki_us * 1e-6) / 1e9 / peak, 4),
            "dense_hbm_frac_of_" + peak_kind:
                round(dense_bytes / (dense_us * 1e-6) / 1e9 / peak, 4),
            "data": "synthetic, drawn on the device"}), flush=True)
        del q, Kt, V, Kt_lo, P, out, idx, ws, dws, dout, q_rot
        torch.cuda.empty_cache()


def relaunch_ranks(n: int) -> int:
    """Run this command as n ranks (one process per GPU) under torch.distributed.run."""
    import subprocess
    import socket
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n}",
           "--master-addr", "127.0.0.1", "--master-port", str(port),
           os.path.abspath(__file__)] + sys.argv[1:]
    return subprocess.call(cmd)


def main():
    args = parse_args()
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        # one process per GPU: start the ranks and let them print
        sys.exit(relaunch_ranks(args.gpus))
    _, world, _ = dist_env()
    if world != args.gpus:
        print(f"bench.py: --gpus {args.gpus} but WORLD_SIZE={world}; using {world} ranks",
              file=sys.stderr)
    if args.ncu_case:
        run_ncu_case(args)
        return
    if args.sweep:
        run_sweep(args)
        return
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
