#!/usr/bin/env python
"""Benchmark of the QSA decode step on B200: queries/s and HBM roofline.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload long|quarter|...]
    python bench.py --impl reference ...   # the CPU oracle, timed on the host

One step = one pass of the whole hot path over one batch: qsa_append_kv of the
batch's new tokens (the current token of every sequence), the indexer scores
and top-K selection (qsa_index_scores + qsa_topk_blocks, or the fused
qsa_index_topk, as the Decoder chooses or --select forces), qsa_sparse_decode
and qsa_combine (or the merged qsa_sparse_attention with --merge kernel), all
enqueued on one stream with the cache resident in HBM.  Between timed steps the open micro-block sums
are restored (the step appends the same token again) and L2 is flushed by
writing a 512 MiB buffer; neither is inside the timed events.

Multi-GPU (torchrun, one rank per GPU): every rank decodes its own copy of the
workload (independent queries; weak scaling, no data-path collective); the
step time is the max over ranks.
"""
from __future__ import annotations

import argparse
import glob
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from workloads import configs as C  # noqa: E402

METRIC = "QSA decode queries/s and HBM GB/s (% of ~8 TB/s) at 128K-256K ctx, top-512"
FALLBACK_HBM_GBS = 6650.0


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["native", "reference"], default="native")
    ap.add_argument("--workload", default="long", choices=list(C.ALL) + list(C.FP8))
    ap.add_argument("--batch", type=int, default=0, help="use only the first N sequences (profiling a small case)")
    ap.add_argument("--context", type=int, default=0, help="override every context length (profiling a small case)")
    ap.add_argument("--select", choices=["auto", "fused", "split"], default="auto",
                    help="indexer + top-K as one fused kernel, as two kernels, or as the library chooses")
    ap.add_argument("--merge", choices=["kernel", "separate"], default="separate",
                    help="split-KV merge inside the attention kernel, or as the separate combine kernel")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="oracle time budget for the CPU baseline")
    ap.add_argument("--dcp", type=int, default=0,
                    help="decode context parallelism over this many ranks: time rank 0's share of a step on one GPU")
    ap.add_argument("--dcp-interleave", type=int, default=1, help="DCP shard interleave, in 64-token pages")
    return ap.parse_args()


# ---------------------------------------------------------------- distributed plumbing


def dist_init():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return rank, ws, local


def barrier(ws):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, ws: int) -> float:
    if ws == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def dist_close(ws):
    if ws > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


# ---------------------------------------------------------------- clocks


class ClockSampler:
    """Samples the SM clock and the clock-event (throttle) reasons of one GPU
    through NVML (the counters nvidia-smi prints) every ~2 ms in a background
    thread while the timed region runs."""

    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, device_index: int):
        self.dev = device_index
        self.samples = []
        self.max_mhz = None
        self.ok = False

    def _handle(self, nv):
        try:
            pci = torch.cuda.get_device_properties(self.dev)
            bus = f"{pci.pci_domain_id:08X}:{pci.pci_bus_id:02X}:{pci.pci_device_id:02X}.0"
            return nv.nvmlDeviceGetHandleByPciBusId(bus)
        except Exception:  # noqa: BLE001
            return nv.nvmlDeviceGetHandleByIndex(self.dev)

    def __enter__(self):
        import threading
        try:
            import pynvml as nv
            nv.nvmlInit()
            self.nv = nv
            self.h = self._handle(nv)
            self.max_mhz = nv.nvmlDeviceGetMaxClockInfo(self.h, nv.NVML_CLOCK_SM)
            self.ok = True
        except Exception:  # noqa: BLE001
            return self
        self.stop = threading.Event()

        def loop():
            nv, h = self.nv, self.h
            while not self.stop.is_set():
                try:
                    mhz = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                    reasons = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                    self.samples.append((mhz, reasons))
                except Exception:  # noqa: BLE001
                    pass
                time.sleep(0.002)
        self.thread = threading.Thread(target=loop, daemon=True)
        self.thread.start()
        return self

    def __exit__(self, *exc):
        if self.ok:
            self.stop.set()
            self.thread.join(timeout=5)

    def summary(self):
        if not self.ok or not self.samples:
            return None
        reasons = set()
        for _, r in self.samples:
            for bit, name in self.REASONS.items():
                if r & bit:
                    reasons.add(name)
        return {"sm_mhz": statistics.median(m for m, _ in self.samples), "sm_max_mhz": self.max_mhz,
                "samples": len(self.samples), "reasons": sorted(reasons), "source": "NVML, 2 ms period"}


# ---------------------------------------------------------------- algorithmic bytes


def algorithmic_bytes(wl: C.Workload, count: np.ndarray, q_pos: np.ndarray, splits_used: int) -> dict:
    """Bytes each kernel must move at minimum, per launch (one step)."""
    nb = (q_pos.astype(np.int64) + 1) // 4
    t = (q_pos.astype(np.int64) + 1) % 4
    n_new = wl.batch * wl.new_tokens
    tok_in = wl.hkv * 256 * 2 * 2                       # K + V bytes of one new token (BF16 inputs)
    tok_kv = wl.hkv * 256 * 2 * (1 if wl.kv_fp8 else 2)  # K + V bytes of one cached token
    append = n_new * (tok_in + tok_kv + 128 * 2)       # read new K/V/kidx, write K/V (+kc, small)
    side = int(nb.sum()) * 128 * 2                      # kc rows read
    scores_w = int(nb.sum()) * 4
    index = side + scores_w
    topk = int(nb.sum()) * 4 + wl.nq * wl.k_top * 4
    sel_tokens = int((4 * count.astype(np.int64) + t).sum())
    kv = sel_tokens * tok_kv
    q_bytes = wl.nq * wl.hq * 256 * 2
    partials = splits_used * 256 * 4
    decode = kv + q_bytes + partials
    out = wl.nq * wl.hq * 256 * 2
    combine = partials + out
    index_topk = index + wl.nq * wl.k_top * 4  # the fused kernel never reads the scores back
    attention = decode + out                   # split kernel + its in-kernel merge
    return {"append_kv": append, "index_scores": index, "topk": topk, "index_topk": index_topk,
            "sparse_decode": decode, "combine": combine, "sparse_attention": attention,
            "pipeline_spec": side + kv + out, "side_cache": side, "selected_kv": kv, "output": out}


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


def kernel_source_sha(kernel: str) -> str:
    """Hash of the kernel's source file and of every shared device header."""
    csrc = os.path.join(ROOT, "sparse_attention_decode_03_b200", "csrc")
    src = {"sparse_attention": "sparse_decode", "topk": "topk", "append_kv": "append_kv"}.get(kernel, kernel)
    h = hashlib.sha256()
    for f in [os.path.join(csrc, f"{src}.cu")] + sorted(glob.glob(os.path.join(csrc, "*.cuh"))):
        if os.path.exists(f):
            h.update(open(f, "rb").read())
    return h.hexdigest()[:16]


def profiled_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from the committed ncu summary of that kernel on
    that workload, if it was taken on the kernel's current source."""
    p = os.path.join(ROOT, "profiles", f"{kernel}_{workload}.md")
    if not os.path.exists(p):
        return None
    txt = open(p).read()
    m_sha = re.search(r"kernel_source_sha:\s*([0-9a-f]+)", txt)
    m_t = re.search(r"dram_bytes_per_launch:\s*([0-9.eE+]+)", txt)
    if not m_sha or not m_t or m_sha.group(1) != kernel_source_sha(kernel):
        return None
    return float(m_t.group(1))


# ---------------------------------------------------------------- CPU oracle (baseline / reference arm)


def oracle_sample(wl: C.Workload, budget_s: float, max_queries: int | None = None, start_row: int = 0):
    """Time the CPU oracle on a bounded sample of the workload's queries.
    Inputs (regenerated rows) are prepared first and held in host memory, like
    the GPU's resident cache; only the oracle's own work is timed."""
    from oracle import qsa_oracle as O
    from tests import oracle_ref as R
    try:
        from threadpoolctl import threadpool_info
        cores = max([int(i.get("num_threads", 1)) for i in threadpool_info()] or [1])
    except Exception:  # noqa: BLE001
        cores = 1
    done, t_oracle = 0, 0.0
    row = start_row
    while t_oracle < budget_s and (max_queries is None or done < max_queries) and done < wl.nq:
        d = R.query_inputs(wl, row % wl.nq)
        kid = R.kidx_seq(wl, d["seq"], d["p"] + 1)
        reader = R.kv_reader(wl, d["seq"])
        cache = {}

        def rows(pos, _r=reader, _c=cache):
            key = np.asarray(pos).tobytes()
            if key not in _c:
                _c[key] = _r(pos)
            return _c[key]
        O.decode_query(d["q"], d["q_idx"], d["w"], d["p"], kid, rows, wl.k_top, wl.scale)   # untimed: fetch rows
        t0 = time.perf_counter()
        O.decode_query(d["q"], d["q_idx"], d["w"], d["p"], kid, rows, wl.k_top, wl.scale)
        t_oracle += time.perf_counter() - t0
        done += 1
        row += max(1, wl.nq // 7)
    return done, t_oracle, cores


def run_reference(args, rank, ws):
    if rank != 0:
        return
    wl = C.get(args.workload)
    per_query, sampled = [], []
    total_q = 0
    budget = max(2.0, 60.0 / max(1, args.steps + args.warmup))
    for i in range(args.warmup + args.steps):
        n, t, cores = oracle_sample(wl, budget, max_queries=2, start_row=i)
        if i >= args.warmup:
            per_query.append(t / n)
            sampled.append(t)
            total_q += n
    qps = 1.0 / statistics.mean(per_query)
    line = {"impl": "reference", "metric": METRIC, "value": qps, "unit": "queries/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000.0 * statistics.mean(per_query) * wl.nq,
            "ms_per_step_kind": (f"projection: the mean oracle time of the {total_q} sampled queries x the "
                                 f"workload's {wl.nq} queries per step (each timed step runs at most 2 queries)"),
            "sampled_ms_per_step": 1000.0 * statistics.mean(sampled),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {**wl.describe(), "parallelism": "host cores"},
            "cpu_baseline": {"value": qps, "unit": "queries/s", "cores": cores, "kind": "oracle",
                             "sample": f"{total_q} queries of the workload, fp64 numpy oracle, inputs regenerated "
                                       f"and resident in host memory"},
            "e2e": {"value": qps, "unit": "queries/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- native arm


def run_native(args, rank, ws, local):
    import sparse_attention_decode_03_b200 as qsa
    from workloads import harness as H

    wl = C.get(args.workload)
    if args.batch:
        wl = C.shrink(wl, list(wl.lengths[:args.batch]), name=f"{wl.name}-first{args.batch}")
    if args.context:
        wl = C.shrink(wl, [args.context - wl.new_tokens] * wl.batch, name=f"{wl.name}-ctx{args.context}")
    dev = torch.device("cuda", local)
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    cache = H.build_cache(wl, dev_status=st)
    # the step's inputs live in one staged buffer (one host-to-device copy per step in the e2e leg)
    io = qsa.StepIO(wl.batch * wl.new_tokens, wl.nq, wl.hq, wl.hkv, dev)
    for k, t in H.step_inputs(wl, device="cpu").items():
        io.host[k].copy_(t)
    io.upload()
    torch.cuda.synchronize()
    inp = io.dev
    dec = qsa.Decoder(cache, wl.hq, wl.nq, k=wl.k_top, scale=wl.scale, target_ctas=sms,
                      chunk_units=H.chunk_units_for(wl), fused={"auto": None, "fused": True, "split": False}[args.select],
                      merged=args.merge == "kernel")
    dec.dev_status = st
    saved_partial = cache.kc_partial.clone()
    flush = torch.empty(512 << 20, dtype=torch.uint8, device=dev)
    flush_read = torch.ones(64 << 20, dtype=torch.int32, device=dev)
    flush_sink = torch.zeros((), dtype=torch.int64, device=dev)
    stream = torch.cuda.Stream(device=dev)   # the step's stream (captured into a CUDA graph below)
    names = (["append_kv"] + (["index_topk"] if dec.fused else ["index_scores", "topk"])
             + (["sparse_attention"] if dec.merged else ["sparse_decode", "combine"]))

    calls = [qsa.bind_append_kv(cache, inp["k_new"], inp["v_new"], inp["kidx_new"], inp["seq_id"], inp["pos"], st,
                                stream=stream)]
    calls += dec.bind(inp["q"], inp["q_idx"], inp["w"], inp["q_seq"], inp["q_pos"], stream=stream)

    def flush_l2():
        # write 512 MiB, then read 256 MiB, so L2 is left holding clean lines
        # (dirty flush lines would otherwise be written back inside the next
        # timed step)
        flush.zero_()
        flush_sink.copy_(flush_read.sum())

    def between():
        with torch.cuda.stream(stream):
            cache.kc_partial.copy_(saved_partial)
            flush_l2()

    def graph_of(fns, reps=1):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for _ in range(reps):
                for f in fns:
                    f()
        return g

    def replay_ms(g):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            e0.record(stream)
            g.replay()
            e1.record(stream)
        e1.synchronize()
        return e0.elapsed_time(e1)

    # eager warm-up through the bound calls, then the step as one CUDA graph
    # (no timing events inside it: an event between two kernels costs the GPU
    # several microseconds)
    for _ in range(max(3, args.warmup)):
        for call in calls:
            call()
        between()
    torch.cuda.synchronize()
    status = int(st.item())
    if status:
        raise RuntimeError(f"device status {qsa.dev_status_names(status)}")
    graph = qsa.StepGraph(calls, stream)
    for _ in range(max(3, args.warmup)):
        graph.replay()
        between()
    torch.cuda.synchronize()

    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    barrier(ws)
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        wall0 = time.perf_counter()
        for i in range(args.steps):
            torch.cuda.nvtx.range_push("qsa_step")   # lets a profiler select the timed launches
            evs[i][0].record(stream)
            graph.replay()
            evs[i][1].record(stream)
            torch.cuda.nvtx.range_pop()
            between()
        torch.cuda.synchronize()
        wall = time.perf_counter() - wall0
    barrier(ws)
    status = int(st.item())
    if status:
        raise RuntimeError(f"device status after the timed steps: {qsa.dev_status_names(status)}")
    step_ms = [a.elapsed_time(b) for a, b in evs]
    mean_ms = statistics.mean(step_ms)
    total_ms = max_over_ranks(sum(step_ms), ws)
    value = ws * wl.nq * args.steps / (total_ms / 1000.0)

    # ---- per-kernel device time, cold L2: a graph of R x (flush, kernel) minus
    # a graph of R x flush, divided by R
    reps = 8
    g_flush = graph_of([flush_l2], reps)
    kern_ms = {}
    for n, call in zip(names, calls):
        g_k = graph_of([flush_l2, call], reps)
        for _ in range(2):
            replay_ms(g_k)
            replay_ms(g_flush)
        t_k = min(replay_ms(g_k) for _ in range(5))
        t_f = min(replay_ms(g_flush) for _ in range(5))
        kern_ms[n] = max(t_k - t_f, 1e-6) / reps
        between()
    torch.cuda.synchronize()
    status = int(st.item())
    if status:
        raise RuntimeError(f"device status after the kernel timing: {qsa.dev_status_names(status)}")

    # ---- e2e: the step's inputs from pinned host memory (one copy of the staged
    # buffer) + the step (graph) + out/lse back to pinned host memory
    out_host = dec.host_outputs()
    h2d = io.nbytes
    d2h = 0
    e2e_ms = []
    for i in range(args.steps + 2):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            e0.record(stream)
            io.upload(stream)
            graph.replay()
            d2h = dec.download(out_host, wl.nq, stream)
            e1.record(stream)
        e1.synchronize()
        if i >= 2:
            e2e_ms.append(e0.elapsed_time(e1))
        between()
    torch.cuda.synchronize()
    status = int(st.item())
    if status:
        raise RuntimeError(f"device status after the e2e steps: {qsa.dev_status_names(status)}")
    e2e_total = max_over_ranks(sum(e2e_ms), ws)
    e2e_seq_value = ws * wl.nq * len(e2e_ms) / (e2e_total / 1000.0)

    # ---- e2e, pipelined (the serving form, qsa.StepPipeline): two slots; the
    # inputs of step i + 1 go up and the outputs of step i - 1 come back while
    # step i computes.  K steps back to back, every one with its own H2D and
    # D2H copies; no L2 flush (the K/V cache is larger than L2), the open
    # micro-block sums restored on the compute stream before every step.
    ios2, decs2, calls2 = [], [], []
    for _ in range(2):
        io_s = qsa.StepIO(wl.batch * wl.new_tokens, wl.nq, wl.hq, wl.hkv, dev)
        io_s.host_buf.copy_(io.host_buf)
        d_s = qsa.Decoder(cache, wl.hq, wl.nq, k=wl.k_top, scale=wl.scale, target_ctas=sms,
                          chunk_units=H.chunk_units_for(wl), fused=dec.fused, merged=dec.merged)
        d_s.dev_status = st
        v = io_s.dev
        calls2.append([qsa.bind_append_kv(cache, v["k_new"], v["v_new"], v["kidx_new"], v["seq_id"], v["pos"], st,
                                          stream=stream)]
                      + d_s.bind(v["q"], v["q_idx"], v["w"], v["q_seq"], v["q_pos"], stream=stream))
        ios2.append(io_s)
        decs2.append(d_s)

    def restore(cs):
        with torch.cuda.stream(cs):
            cache.kc_partial.copy_(saved_partial)

    pipe = qsa.StepPipeline(ios2, decs2, calls2, stream, before=restore, nq=wl.nq)
    n_warm = max(3, args.warmup)
    for i in range(n_warm):
        pipe.step(i)
    torch.cuda.synchronize()
    p0, p1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(ws)
    torch.cuda.synchronize()
    p0.record(pipe.up_stream)
    for i in range(args.steps):
        pipe.step(n_warm + i)
    p1.record(pipe.down_stream)
    p1.synchronize()
    torch.cuda.synchronize()
    barrier(ws)
    status = int(st.item())
    if status:
        raise RuntimeError(f"device status after the pipelined e2e steps: {qsa.dev_status_names(status)}")
    pipe_ms = max_over_ranks(p0.elapsed_time(p1), ws)
    e2e_value = ws * wl.nq * args.steps / (pipe_ms / 1000.0)
    # the last step's outputs as read back equal the device's
    out_h, lse_h = pipe.outputs(n_warm + args.steps - 1)
    last = decs2[(n_warm + args.steps - 1) % 2]
    if not (torch.equal(out_h.view(torch.int16), last.out.cpu().view(torch.int16))
            and torch.equal(lse_h.view(torch.int32), last.lse.cpu().view(torch.int32))):
        raise RuntimeError("pipelined e2e: host outputs differ from the device's")
    # append + (scores + top-K, or the fused kernel) + (attention + combine, or merged)
    launches_per_step = 1 + (1 if dec.fused else 2) + (1 if dec.merged else 2)

    # ---- roofline of the dominant kernel
    count = dec.count[:wl.nq].cpu().numpy()
    q_pos = inp["q_pos"].cpu().numpy()
    n_slots = wl.nq * wl.hkv * (wl.k_top + 1)
    chunks = math.ceil(n_slots / dec.chunk_units)
    splits_used = (chunks + wl.nq * wl.hkv) * (wl.hq // wl.hkv)
    ab = algorithmic_bytes(wl, count, q_pos, splits_used)
    peak, peak_kind = measured_peaks()
    dom = max(names, key=lambda n: kern_ms[n])
    dom_key = {"topk": "topk"}.get(dom, dom)
    achieved = ab[dom_key] / (kern_ms[dom] / 1000.0) / 1e9
    traffic = profiled_traffic(dom, wl.name)
    kernels = {n: {"ms": round(kern_ms[n], 5), "alg_bytes": ab[n],
                   "gbs": round(ab[n] / (kern_ms[n] / 1000.0) / 1e9, 1)} for n in names}
    pipeline_gbs = ab["pipeline_spec"] / (mean_ms / 1000.0) / 1e9

    line = {
        "metric": METRIC, "value": value, "unit": "queries/s", "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": mean_ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "e4m3 kv + bf16" if wl.kv_fp8 else "bf16", "data": "synthetic",
        "config": {**wl.describe(), "l2": "flushed between timed steps (512 MiB write, then 256 MiB read); inputs also larger than L2",
                   "step": " + ".join(["append_kv"] + (["index_topk (fused)"] if dec.fused else ["index_scores", "topk_blocks"])
                                      + (["sparse_attention (split kernel with in-kernel merge)"] if dec.merged
                                         else ["sparse_decode", "combine"])) + ", one CUDA graph",
                   "kernel_timing": "per kernel: CUDA events around a graph of 8 x (L2 flush, kernel) minus one of 8 x (L2 flush), / 8",
                   "parallelism": f"dp{ws} (independent replicas)" if ws > 1 else "single GPU",
                   "chunk_units": dec.chunk_units, "max_splits": dec.max_splits},
        "hbm": {"pipeline_alg_bytes": ab["pipeline_spec"], "achieved_gbs": round(pipeline_gbs, 1), "peak_gbs": peak,
                "frac": round(pipeline_gbs / peak, 4), "peak_kind": f"{peak_kind} STREAM copy"},
        "roofline": {"kernel": dom, "bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(achieved / peak, 4), "traffic": traffic,
                     "alg_bytes_per_launch": ab[dom_key], "peak_kind": f"{peak_kind} (hbm_gbs)"},
        "kernels": kernels,
        "e2e": {"value": e2e_value, "unit": "queries/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": pipe_ms / args.steps,
                "mode": "pipelined (qsa.StepPipeline, two slots): every step's pinned-host inputs copied up and "
                        "its out/lse copied back, overlapped with the neighbouring steps' compute; steps back to back",
                "sequential": {"value": e2e_seq_value, "ms_per_step": statistics.mean(e2e_ms),
                               "mode": "upload, step, download, synchronise; one step at a time"}},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clk.summary(),
        "wall_s_timed_region": round(wall, 3),
    }
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        n, t, cores = oracle_sample(wl, args.cpu_seconds)
        line["cpu_baseline"] = {"value": n / t, "unit": "queries/s", "cores": cores, "kind": "oracle",
                                "sample": f"{n} of the workload's {wl.nq} queries (rows spread over the batch), "
                                          f"fp64 numpy oracle, inputs regenerated and resident in host memory"}
    if rank == 0:
        print(json.dumps(line), flush=True)


def run_dcp(args, rank, ws, local):
    """Rank 0 of a DCP group of args.dcp ranks, on one GPU: its replicated
    selector and its K/V shard, and its share of every step (append, scores,
    top-K, localisation, attention over its blocks, merge of its splits, and
    the merge over the ranks).  The all-gather of the ranks' (o, lse) between
    the attention and the final merge is not timed (one GPU: no peer)."""
    import sparse_attention_decode_03_b200 as qsa
    from workloads import harness as H

    if ws != 1:
        raise SystemExit("--dcp times one rank's share on one GPU; run it without torchrun")
    R, I = args.dcp, args.dcp_interleave
    wl = C.get(args.workload)
    if args.batch:
        wl = C.shrink(wl, list(wl.lengths[:args.batch]), name=f"{wl.name}-first{args.batch}")
    dev = torch.device("cuda", local)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    sh = qsa.DCPShard(R, 0, I)
    pages = [-(-L // 64) for L in wl.total_lengths]
    selector = qsa.PagedCache(wl.num_pages(), wl.batch, wl.pages_per_seq(), wl.hkv, block_table=C.block_table(wl),
                              device=dev, with_kv=False)
    bt, used = sh.shard_block_table(pages)
    shard = qsa.PagedCache(max(1, used), wl.batch, bt.shape[1], wl.hkv, block_table=bt, device=dev, with_kc=False,
                           kv_dtype=qsa.KV_FP8_E4M3 if wl.kv_fp8 else qsa.KV_BF16)
    rk = qsa.DCPRank(selector, shard, wl.hq, wl.nq, R, 0, I, k=wl.k_top, scale=wl.scale)
    rk.dev_status = st
    for b, L in enumerate(wl.lengths):
        for a0 in range(0, L, 32768):
            a1 = min(L, a0 + 32768)
            pos = torch.arange(a0, a1, device=dev)
            rk.append(C.k_rows(wl, b, pos, dev), C.v_rows(wl, b, pos, dev), C.kidx_rows(wl, b, pos, dev),
                      torch.full((a1 - a0,), b, dtype=torch.int32, device=dev), pos.to(torch.int32))
    inp = H.step_inputs(wl, device=dev)
    saved = selector.kc_partial.clone()
    stream = torch.cuda.Stream(device=dev)
    flush = torch.empty(512 << 20, dtype=torch.uint8, device=dev)
    flush_read = torch.ones(64 << 20, dtype=torch.int32, device=dev)
    flush_sink = torch.zeros((), dtype=torch.int64, device=dev)

    def flush_l2():
        flush.zero_()
        flush_sink.copy_(flush_read.sum())

    def between():
        with torch.cuda.stream(stream):
            selector.kc_partial.copy_(saved)
            flush_l2()

    def step():
        rk.append(inp["k_new"], inp["v_new"], inp["kidx_new"], inp["seq_id"], inp["pos"], stream)
        rk.attend(inp["q"], inp["q_idx"], inp["w"], inp["q_seq"], inp["q_pos"], stream)
        rk.merge(wl.nq, stream)

    with torch.cuda.stream(stream):
        for _ in range(max(3, args.warmup)):
            step()
            for j in range(R):               # the exchange, emulated once outside the timed steps
                rk.o_all[j].copy_(rk.o_rank)
                rk.lse_all[j].copy_(rk.lse_rank)
            between()
    torch.cuda.synchronize()
    if int(st.item()):
        raise RuntimeError(f"device status {qsa.dev_status_names(int(st.item()))}")
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        step()
    for _ in range(3):
        with torch.cuda.stream(stream):
            g.replay()
        between()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        for i in range(args.steps):
            with torch.cuda.stream(stream):
                evs[i][0].record(stream)
                g.replay()
                evs[i][1].record(stream)
            between()
        torch.cuda.synchronize()
    if int(st.item()):
        raise RuntimeError(f"device status after the timed steps: {qsa.dev_status_names(int(st.item()))}")
    step_ms = [a.elapsed_time(b) for a, b in evs]
    mean_ms = statistics.mean(step_ms)
    # the shard attention kernel alone, cold L2 (graph of 8 x (flush, kernel) minus 8 x flush)
    nq = wl.nq
    decode_call = lambda: qsa.qsa_sparse_decode(
        shard, inp["q"], inp["q_seq"], rk.q_pos_local[:nq], rk.sel_local[:nq], rk.count_local[:nq], rk.k, rk.scale,
        rk.chunk_units, rk.max_splits, rk.part_o[:nq], rk.part_lse[:nq], st, stream)

    def gtime(fns):
        gg = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gg, stream=stream):
            for _ in range(8):
                for f in fns:
                    f()
        best = 1e9
        for _ in range(6):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            with torch.cuda.stream(stream):
                e0.record(stream)
                gg.replay()
                e1.record(stream)
            e1.synchronize()
            best = min(best, e0.elapsed_time(e1))
        return best
    dec_ms = max(gtime([flush_l2, decode_call]) - gtime([flush_l2]), 1e-6) / 8
    torch.cuda.synchronize()
    tok_kv = wl.hkv * 256 * 2 * (1 if wl.kv_fp8 else 2)
    cl = rk.count_local[:nq].cpu().numpy().astype(np.int64)
    ql = rk.q_pos_local[:nq].cpu().numpy().astype(np.int64)
    qp = inp["q_pos"].cpu().numpy().astype(np.int64)
    tail_here = ((ql + 1) % 4 == (qp + 1) % 4) & ((qp + 1) % 4 > 0)
    sel_tokens = int((4 * cl).sum() + ((qp + 1) % 4)[tail_here].sum())
    dec_bytes = sel_tokens * tok_kv + nq * wl.hq * 256 * 2
    peak, peak_kind = measured_peaks()
    achieved = dec_bytes / (dec_ms / 1000.0) / 1e9
    line = {
        "metric": METRIC, "value": nq / (mean_ms / 1000.0), "unit": "queries/s", "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": mean_ms, "higher_is_better": True, "scaling": "strong",
        "vs_baseline": None, "dtype": "e4m3 kv + bf16" if wl.kv_fp8 else "bf16", "data": "synthetic",
        "config": {**wl.describe(), "parallelism": f"dcp{R} (interleave {I} pages): rank 0 of {R} on one GPU, "
                   "its own K/V shard and a replicated selector; the all-gather of the ranks' (o, lse) is not timed",
                   "step": "append (side cache + shard) + index_scores + topk + localize + sparse_decode (shard) + "
                           "merge of the rank's splits + merge over the ranks, one CUDA graph",
                   "l2": "flushed between timed steps"},
        "roofline": {"kernel": "sparse_decode (rank 0 shard)", "bound": "hbm", "achieved": round(achieved, 1),
                     "peak": peak, "unit": "GB/s", "frac": round(achieved / peak, 4), "traffic": None,
                     "alg_bytes_per_launch": dec_bytes, "peak_kind": f"{peak_kind} (hbm_gbs)",
                     "ms": round(dec_ms, 5)},
        "rank0_selected_blocks": int(cl.sum()), "all_selected_blocks": int(rk.count[:nq].sum()),
        "gpu_launches": 9 * args.steps,  # 2 appends, 2 localisations, scores, top-K, attention, 2 merges
        "clocks": clk.summary(),
    }
    print(json.dumps(line), flush=True)


def main():
    args = parse_args()
    rank, ws, local = dist_init()
    try:
        if args.impl == "reference":
            run_reference(args, rank, ws)
        elif args.dcp > 1:
            run_dcp(args, rank, ws, local)
        else:
            run_native(args, rank, ws, local)
    finally:
        dist_close(ws)


if __name__ == "__main__":
    main()
