#!/usr/bin/env python
"""Benchmark of the TurboQuant KV-cache hot path on B200.

One step is one decode step of a Llama-3.3-70B-shaped model over a packed
cache: for each of 80 layers, append the new token's K/V (tq_quantize, 16
sequences x 8 kv heads) and attend (tq_attend, 64 query heads, context
32768 + 1, K at 3-bit + QJL, V at 4 bits). Value = packed-KV bytes read per
step / step time (GB/s). The cache is 45 GB, far larger than L2, so no flush
is needed between steps.

Also reported on the same line: the attention kernels' roofline (measured
copy-kernel and MEASURED_PEAKS.json HBM peaks), tq_quantize throughput on a
bulk prefill, an end-to-end figure through host buffers, GPU clocks during
the timed region, and the fp64 CPU oracle timed on a bounded sample.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl tq|reference]
Multi-GPU runs (torchrun, one rank per GPU) are weak scaling: every rank runs
its own copy of the workload; no collective touches the data path.
"""
from __future__ import annotations

import argparse
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

METRIC = "tq_attend packed-KV GB/s and % of HBM peak; tq_quantize Mtokens/s"
DEFAULT_WORKLOAD = "llama3.3-70b_decode_32k"


def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["tq", "reference"], default="tq")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--layers", type=int, default=None, help="override layer count (development)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-graph", action="store_true",
                    help="time the eager launch loop only (no CUDA graph of the step)")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-secondary", action="store_true",
                    help="skip the other long-context workloads reported beside the bench line")
    ap.add_argument("--report", choices=["all", "single", "qwen3b", "qwen32b", "sweep", "formats",
                                         "cudacore"],
                    default=None,
                    help="measure the other workloads instead of the bench line: one JSON line each")
    return ap.parse_args(argv)


# ---------------------------------------------------------------- plumbing

class Dist:
    """One process per GPU (torchrun env); the ranks run independent replicas of
    the workload (weak scaling) and meet only to take the max of their step
    times and the sum of their bytes. backend "nccl" on GPUs, "gloo" on CPU."""

    def __init__(self):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local_rank = int(os.environ.get("LOCAL_RANK", "0"))
        self.pg = None
        self.device = None

    def init(self, backend="nccl"):
        import torch
        import torch.distributed as dist
        if backend == "nccl":
            torch.cuda.set_device(self.local_rank)
            self.device = torch.device("cuda", self.local_rank)
        else:
            self.device = torch.device("cpu")
        if self.world > 1:
            from datetime import timedelta
            kw = {"timeout": timedelta(seconds=600)}
            if backend == "nccl":
                kw["device_id"] = self.device
            dist.init_process_group(backend, **kw)
            self.pg = dist

    def barrier(self):
        if self.pg:
            self.pg.barrier()

    def _reduce(self, x: float, op) -> float:
        if not self.pg:
            return x
        import torch
        t = torch.tensor([x], dtype=torch.float64, device=self.device)
        self.pg.all_reduce(t, op=op)
        return float(t.item())

    def max(self, x: float) -> float:
        return self._reduce(x, self.pg.ReduceOp.MAX if self.pg else None)

    def sum(self, x: float) -> float:
        return self._reduce(x, self.pg.ReduceOp.SUM if self.pg else None)

    def close(self):
        if self.pg:
            self.pg.destroy_process_group()


def whole_job_gbs(total_bytes: float, ms_max: float) -> float:
    """Whole-job throughput: the bytes every rank processed in one step, over
    the slowest rank's step time (ms)."""
    return total_bytes / (ms_max / 1e3) / 1e9


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples during the timed region."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.idx), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, smax, reasons, power = [], [], set(), []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
                power.append(float(parts[3]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        os.unlink(self.path)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "power_w_max": max(power) if power else None,
                "samples": len(sm), "reasons": sorted(reasons)}


TRAFFIC_FILE = os.path.join(ROOT, "profiles", "attend_split_llama70b_32k.json")


def profiled_traffic(workload: str):
    """DRAM bytes (read + write) per split-kernel launch, from the data file
    written beside the ncu summary of this workload's capture, if it was taken
    on the attention source as it is now (else None)."""
    import hashlib
    src = os.path.join(ROOT, "kv_cache_vector_04_b200", "csrc", "attend_impl.cuh")
    if workload != DEFAULT_WORKLOAD or not os.path.exists(TRAFFIC_FILE):
        return None
    with open(TRAFFIC_FILE) as f:
        rec = json.load(f)
    with open(src, "rb") as f:
        sha = hashlib.sha1(f.read()).hexdigest()
    if rec.get("kernel_source_sha1") != sha or rec.get("workload") != workload:
        return None
    return int(rec["dram_bytes_per_launch"])


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            j = json.load(f)
        return j.get("hbm_gbs"), "measured"
    return 6650.0, "fallback"


# ---------------------------------------------------------------- inputs

def load_inputs():
    """The seeded input generators (kv_cache_vector_04_b200/inputs.py). Once the
    package is imported (the GPU arm), its own module; otherwise the file is
    loaded on its own, so that the reference arm never maps the CUDA library
    (the package's __init__ loads it)."""
    name = "kv_cache_vector_04_b200.inputs"
    if name in sys.modules:
        return sys.modules[name]
    if "kv_cache_vector_04_b200" in sys.modules:
        from kv_cache_vector_04_b200 import inputs
        return inputs
    import importlib.util
    if "_tq_inputs_file" not in sys.modules:
        spec = importlib.util.spec_from_file_location(
            "_tq_inputs_file", os.path.join(ROOT, "kv_cache_vector_04_b200", "inputs.py"))
        mod = importlib.util.module_from_spec(spec)
        sys.modules["_tq_inputs_file"] = mod
        spec.loader.exec_module(mod)
    return sys.modules["_tq_inputs_file"]


# ---------------------------------------------------------------- CPU oracle sample

class OracleSample:
    """The fp64 oracle's decode attention over `streams` (batch, kv-head)
    streams of the workload (all their query heads, N tokens each): the codes
    are computed once, then timed repeatedly."""

    def __init__(self, w, streams: int = 4, N: int | None = None):
        import numpy as np
        import torch
        inputs = load_inputs()
        from oracle import oracle as O
        self.O, self.np = O, np
        self.N = w.N if N is None else N
        self.streams = streams
        self.tab = O.Tables(w.d, w.bits, 1, fmt=w.fmt) if w.fmt is not None else O.Tables(w.d, w.bits, 1)
        g = w.Hq // w.Hkv
        k, v = inputs.kv_pair(w, self.N, layer=0, device="cpu", B=1, Hkv=streams)
        codes = [O.quantize(self.tab, k[0, h].numpy(), v[0, h].numpy()) for h in range(streams)]
        self.st = {key: np.stack([c[key] for c in codes])[None]
                   for key in ("kidx", "ksign", "knorm", "rnorm", "vidx", "vnorm")}
        q = inputs.queries(w, B=1, Hq=streams * g)
        self.qb = q.contiguous().view(torch.int16).numpy().view(np.uint16)
        self.q_bf16 = w.q_dtype == torch.bfloat16
        self.seq = np.array([self.N], np.int32)
        self.bytes_per_rep = streams * self.N * bytes_per_head_token(w)
        self.g = g

    def run(self, seconds: float):
        """Repeat the attention until about `seconds` of work; (GB/s, seconds per rep)."""
        reps, t_total = 0, 0.0
        while t_total < seconds or reps == 0:
            t0 = time.perf_counter()
            self.O.attend_batch(self.tab, self.qb, self.q_bf16, self.st, self.seq, self.streams)
            t_total += time.perf_counter() - t0
            reps += 1
        self.last = (reps, t_total)
        return self.bytes_per_rep * reps / t_total / 1e9, t_total / reps

    def describe(self) -> str:
        reps, t_total = self.last
        return ("fp64 C oracle decode attention over %d (batch, kv-head) streams x %d query heads x "
                "%d tokens of layer 0, %d repetitions in %.1f s (append of one token excluded: "
                "<0.01%% of the step)" % (self.streams, self.g, self.N, reps, t_total))


def cpu_oracle_sample(w, seconds: float, streams: int = 4, N: int | None = None):
    """Time the oracle on a bounded sample: (GB/s, description, threads, seconds per rep)."""
    smp = OracleSample(w, streams, N)
    gbs, per = smp.run(seconds)
    threads = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
    return gbs, smp.describe(), threads, per


# ---------------------------------------------------------------- workload description

def fmt_of(w):
    """(B_K, B_V, qjl) of a workload: its named format, else TurboQuant at w.bits."""
    return tuple(w.fmt) if w.fmt is not None else (w.bits - 1, w.bits, 1)


def bytes_per_head_token(w) -> int:
    """Packed K + V bytes of one (token, kv head): codes, signs and fp16 norms
    (the tile layout of include/tq.h, per token)."""
    kb, vb, qjl = fmt_of(w)
    return ((kb + qjl) * w.d // 8 + 2 + 2 * qjl) + (vb * w.d // 8 + 2)


def workload_config(w, layers: int, world: int) -> dict:
    """The `config` of a bench line: the workload as both arms run it (the
    context includes the decode step's appended token)."""
    N = w.N
    per_tok = bytes_per_head_token(w)
    layer_bytes = w.B * w.Hkv * (N + 1) * per_tok
    return {"workload": w.name, "layers": layers, "batch": w.B, "q_heads": w.Hq,
            "kv_heads": w.Hkv, "head_dim": w.d, "bits": w.bits, "context": N + 1,
            "format": list(fmt_of(w)),
            "packed_cache_gb": round(layers * w.B * w.Hkv * (N + 16) * per_tok / 1e9, 2),
            "step": "per layer: tq_append_attend (append 1 token, then attend)",
            "l2": l2_note(layers * layer_bytes, layer_bytes),
            "parallelism": "replicas x%d (weak)" % world}


# ---------------------------------------------------------------- GPU arm

def workload_by_name(name: str):
    inputs = load_inputs()
    if name in inputs.WORKLOADS:
        return inputs.WORKLOADS[name]
    extra = {x.name: x for x in inputs.sweep_workloads() + inputs.format_workloads()}
    if name in extra:
        return extra[name]
    raise SystemExit("unknown workload %r" % name)


def run_tq(args, dist: Dist):
    import torch
    import kv_cache_vector_04_b200 as tq
    from kv_cache_vector_04_b200 import inputs

    w = workload_by_name(args.workload)
    layers = args.layers or w.layers
    dev = torch.device("cuda", dist.local_rank)
    ctx = tq.tq_init(w.d, w.bits, 1) if w.fmt is None else tq.tq_init_ex(w.d, *w.fmt, 1)
    lay = tq.tq_cache_layout(ctx)
    per_tok = lay["tile_bytes"] // 16                     # K + V bytes per head-token
    assert per_tok == bytes_per_head_token(w), (per_tok, bytes_per_head_token(w))
    N = w.N
    cap = N + 16
    zeros = torch.zeros(w.B, dtype=torch.int32, device=dev)

    # ---- prefill: quantize every layer's cache (inputs drawn on the device)
    caches = []
    q_tput = None
    for L in range(layers):
        k, v = inputs.kv_pair(w, N, layer=L, device=dev)
        cache = tq.new_cache(ctx, w.B, w.Hkv, cap, device=dev)
        if L == 0:
            # bulk tq_quantize throughput, timed on this layer's prefill
            s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            for _ in range(2):
                tq.tq_quantize(ctx, k, v, zeros, cache)
            torch.cuda.synchronize()
            reps = 5
            s.record()
            for _ in range(reps):
                tq.tq_quantize(ctx, k, v, zeros, cache)
            e.record()
            torch.cuda.synchronize()
            t = s.elapsed_time(e) / 1e3 / reps
            toks = w.B * w.Hkv * N
            q_bytes = toks * (2 * w.d * 2 + per_tok)
            q_tput = {"metric": "tq_quantize Mtokens/s (bulk prefill; token = one K+V head-vector pair)",
                      "value": round(toks / t / 1e6, 2), "unit": "Mtokens/s",
                      "workload": "one layer: %d seq x %d kv heads x %d tokens" % (w.B, w.Hkv, N),
                      "ms_per_launch": round(t * 1e3, 4),
                      "Mkeys_per_s": round(toks / t / 1e6, 2),
                      "hbm_gbs": round(q_bytes / t / 1e9, 1)}
        else:
            tq.tq_quantize(ctx, k, v, zeros, cache)
        caches.append(cache)
        del k, v
    torch.cuda.synchronize()
    torch.cuda.empty_cache()      # release the prefill's generator temporaries
    assert tq.tq_status(ctx) == 0

    # ---- decode-step inputs (one new token per sequence and layer)
    qs = [inputs.queries(w, layer=L, device=dev) for L in range(layers)]
    news = [inputs.kv_pair(w, 1, layer=10_000 + L, device=dev) for L in range(layers)]
    start = torch.full((w.B,), N, dtype=torch.int32, device=dev)
    seq = torch.full((w.B,), N + 1, dtype=torch.int32, device=dev)
    ws = tq.new_workspace(ctx, w.B, w.Hq, w.Hkv, N + 1)
    outs = [torch.empty((w.B, w.Hq, w.d), dtype=torch.float32, device=dev) for _ in range(layers)]
    launches_per_step = layers * 3   # per layer: prologue with the append, split, reduce

    def step(events=None):
        for L in range(layers):
            nk, nv = news[L]
            if events is not None:
                events[L][0].record()
            tq.tq_append_attend(ctx, qs[L], nk, nv, start, caches[L], seq, N + 1, out=outs[L],
                                workspace=ws)
            if events is not None:
                events[L][1].record()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()

    # ---- the whole step (all layers) as one CUDA graph
    graph = None
    if not args.no_graph:
        side = torch.cuda.Stream(device=dev)
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            step()
        torch.cuda.current_stream().wait_stream(side)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            step()
        for _ in range(args.warmup):
            graph.replay()
        torch.cuda.synchronize()

    # ---- copy-kernel HBM peak in the same process (1 GiB -> 1 GiB)
    src = torch.empty(1 << 30, dtype=torch.uint8, device=dev)
    dst = torch.empty_like(src)
    for _ in range(3):
        tq.tq_copy(src, dst)
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    for _ in range(10):
        tq.tq_copy(src, dst)
    e.record()
    torch.cuda.synchronize()
    copy_gbs = 2 * (1 << 30) * 10 / (s.elapsed_time(e) / 1e3) / 1e9
    del src, dst

    # ---- timed region
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    clocks = ClockSampler(vis.split(",")[dist.local_rank] if vis else dist.local_rank)
    clocks.start()
    ev = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(layers)] for _ in range(args.steps)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    dist.barrier()
    torch.cuda.synchronize()
    t_start.record()
    for k_ in range(args.steps):
        step(ev[k_])
    t_end.record()
    torch.cuda.synchronize()
    dist.barrier()
    ms_eager = dist.max(t_start.elapsed_time(t_end) / args.steps)
    attend_ms = statistics.mean(a.elapsed_time(b) for row in ev for (a, b) in row)
    ms_graph = None
    if graph is not None:
        dist.barrier()
        torch.cuda.synchronize()
        t_start.record()
        for _ in range(args.steps):
            graph.replay()
        t_end.record()
        torch.cuda.synchronize()
        dist.barrier()
        ms_graph = dist.max(t_start.elapsed_time(t_end) / args.steps)
    clk = clocks.stop()
    ms = ms_graph if ms_graph is not None else ms_eager
    assert tq.tq_status(ctx) == 0

    bytes_step = layers * w.B * w.Hkv * (N + 1) * per_tok
    bytes_attend = w.B * w.Hkv * (N + 1) * per_tok
    total_bytes = dist.sum(bytes_step)
    value = whole_job_gbs(total_bytes, ms)
    peak, peak_kind = measured_peaks()
    # The attention call's rate: one layer's algorithmic bytes over the layer's
    # share of the timed step (CUDA events around the graph replays; launches of
    # consecutive layers overlap there as in a real decode step). The per-call
    # eager figure (events around each call, which also cut the overlap between
    # layers) is reported beside it.
    achieved = bytes_attend / (ms / layers / 1e3) / 1e9
    achieved_call = bytes_attend / (attend_ms / 1e3) / 1e9

    # ---- end to end through host buffers: q, new K/V from pinned host memory
    e2e = None
    if not args.no_e2e:
        q_host = [q.cpu().pin_memory() for q in qs]
        k_host = [(a.cpu().pin_memory(), b.cpu().pin_memory()) for a, b in news]
        out_host = [torch.empty(o.shape, dtype=o.dtype).pin_memory() for o in outs]
        # Double-buffered device inputs. Layer L + 1's inputs upload on one copy
        # stream while layer L computes; layer L's output downloads on another
        # (PCIe is full duplex). The step ends when every output is on the host.
        comp = torch.cuda.current_stream()
        h2d_s, d2h_s = torch.cuda.Stream(), torch.cuda.Stream()
        bufs = [(torch.empty_like(qs[0]), torch.empty_like(news[0][0]), torch.empty_like(news[0][1]))
                for _ in range(2)]
        ev_in = [torch.cuda.Event() for _ in range(2)]
        ev_free = [torch.cuda.Event() for _ in range(2)]
        ev_out = [torch.cuda.Event() for _ in range(layers)]

        def upload(L):
            i = L % 2
            with torch.cuda.stream(h2d_s):
                h2d_s.wait_event(ev_free[i])          # layer L - 2 is done with this buffer
                bufs[i][0].copy_(q_host[L], non_blocking=True)
                bufs[i][1].copy_(k_host[L][0], non_blocking=True)
                bufs[i][2].copy_(k_host[L][1], non_blocking=True)
                ev_in[i].record(h2d_s)

        def host_step():
            for i in range(2):
                ev_free[i].record(comp)
            upload(0)
            for L in range(layers):
                i = L % 2
                if L + 1 < layers:
                    upload(L + 1)
                comp.wait_event(ev_in[i])
                tq.tq_append_attend(ctx, bufs[i][0], bufs[i][1], bufs[i][2], start, caches[L], seq,
                                    N + 1, out=outs[L], workspace=ws, stream=comp)
                ev_free[i].record(comp)
                ev_out[L].record(comp)
                with torch.cuda.stream(d2h_s):
                    d2h_s.wait_event(ev_out[L])
                    out_host[L].copy_(outs[L], non_blocking=True)
            comp.wait_stream(d2h_s)
            comp.wait_stream(h2d_s)

        for _ in range(max(args.warmup, 3)):
            host_step()
        torch.cuda.synchronize()
        dist.barrier()
        s.record()
        for _ in range(args.steps):
            host_step()
        e.record()
        torch.cuda.synchronize()
        dist.barrier()
        e2e_ms = dist.max(s.elapsed_time(e) / args.steps)
        h2d = layers * (qs[0].numel() * qs[0].element_size() +
                        2 * news[0][0].numel() * news[0][0].element_size())
        d2h = layers * outs[0].numel() * outs[0].element_size()
        e2e = {"value": round(total_bytes / (e2e_ms / 1e3) / 1e9, 1), "unit": "GB/s",
               "ms_per_step": round(e2e_ms, 4), "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h,
               "copies": "pinned host buffers; per layer, inputs upload and the output "
                         "downloads on two copy streams, overlapping the neighbouring "
                         "layers' compute; the step ends when all outputs are on the host"}

    line = {
        "metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": dist.world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f16 tensor-core operands, f32 accumulate (codes u2-u4)",
        "data": "synthetic",
        "config": dict(workload_config(w, layers, dist.world),
                       step_launch="one CUDA graph per step" if ms_graph is not None else "eager"),
        "pct_of_hbm_peak": round(100.0 * value / dist.world / peak, 1),
        "ms_per_step_eager": round(ms_eager, 4),
        "ms_per_step_graph": round(ms_graph, 4) if ms_graph is not None else None,
        "ms_per_layer": round(ms / layers, 4),
        "roofline": {"bound": "hbm",
                     "kernel": "tq_append_attend per layer (prologue with the append + split + reduce)",
                     "timing": ("step time / layers, CUDA events around %s" %
                                ("graph replays" if ms_graph is not None else "eager steps")),
                     "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(achieved / peak, 3), "peak_kind": peak_kind,
                     "traffic": profiled_traffic(w.name),
                     "traffic_note": "dram read+write bytes of one split-kernel launch of this "
                                     "workload from an ncu capture; null when the attention "
                                     "source changed since",
                     "algorithmic_bytes_per_launch": bytes_attend,
                     "frac_of_same_run_copy_kernel": round(achieved / copy_gbs, 3),
                     "achieved_per_call_eager": round(achieved_call, 1),
                     "frac_per_call_eager": round(achieved_call / peak, 3)},
        "copy_kernel_gbs": round(copy_gbs, 1),
        "quantize": q_tput,
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clk,
        "e2e": e2e,
    }
    if dist.rank == 0 and dist.world == 1 and not args.no_cpu_baseline:
        gbs, desc, threads, _ = cpu_oracle_sample(w, args.cpu_seconds, N=N + 1)
        line["cpu_baseline"] = {"value": round(gbs, 4), "unit": "GB/s", "cores": threads,
                                "kind": "oracle", "sample": desc}
    for L in range(layers):
        caches[L] = None
    return line


def run_reference(args, dist: Dist):
    """The fp64 CPU oracle as the reference arm: each step is a bounded sample
    (about half a second: 4 (batch, kv head) streams of the workload over the
    same context as the GPU arm, N + 1 tokens) of oracle decode attention."""
    w = workload_by_name(args.workload)
    if dist.rank != 0:
        return None
    smp = OracleSample(w, streams=4, N=w.N + 1)
    times = []
    for i in range(args.warmup + args.steps):
        gbs, _ = smp.run(0.5)
        if i >= args.warmup:
            times.append(gbs)
    value = statistics.mean(times)
    desc = smp.describe() + "; %d timed steps of ~0.5 s, mean GB/s" % args.steps
    threads = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
    layers = getattr(args, "layers", None) or w.layers
    return {"impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s",
            "n_gpus": dist.world, "steps": args.steps, "warmup": args.warmup,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f64", "data": "synthetic",
            "config": dict(workload_config(w, layers, dist.world), step_launch="one CUDA graph per step"),
            "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": threads,
                             "kind": "oracle", "sample": desc},
            "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def _time_ms(fn, reps: int, warm: int = 3) -> float:
    import torch
    for _ in range(warm):
        fn()
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    for _ in range(reps):
        fn()
    e.record()
    torch.cuda.synchronize()
    return s.elapsed_time(e) / reps


L2_BYTES = 126e6   # B200 L2


def l2_note(step_bytes: float, layer_bytes: float) -> str:
    """How the timed steps meet L2: a step that reads more than L2 holds
    evicts its own data before the next step reads it again, so no flush is
    needed; a smaller one runs warm."""
    if step_bytes > L2_BYTES:
        return "inputs larger than L2: %.0f MB per step (%.1f MB per layer), no flush" % (
            step_bytes / 1e6, layer_bytes / 1e6)
    return "inputs fit in L2 (%.1f MB per step): warm-L2 figures, not HBM-bound" % (step_bytes / 1e6)


def report_single_head():
    """The pages' GB10 speed test shape (d = 128, 3 bits, 8192 keys, 64 fp16
    queries on one head): quantize the 8192 keys and values, the 64 x 8192
    estimated logits, and the attention step. 1.6 MB: it stays in L2, so these
    are latency figures."""
    import torch
    import kv_cache_vector_04_b200 as tq
    from kv_cache_vector_04_b200 import inputs
    w = inputs.WORKLOADS["single_head_d128_b3"]
    dev = torch.device("cuda", 0)
    ctx = tq.tq_init(w.d, w.bits, 1)
    k, v = inputs.kv_pair(w, w.N, device=dev)
    cache = tq.new_cache(ctx, 1, 1, w.N)
    zeros = torch.zeros(1, dtype=torch.int32, device=dev)
    q = inputs.queries(w, device=dev)
    seq = torch.full((1,), w.N, dtype=torch.int32, device=dev)
    ws = tq.new_workspace(ctx, 1, w.Hq, 1, w.N)
    sc = torch.empty((1, w.Hq, w.N), dtype=torch.float32, device=dev)
    out = torch.empty((1, w.Hq, w.d), dtype=torch.float32, device=dev)
    q_ms = _time_ms(lambda: tq.tq_quantize(ctx, k, v, zeros, cache), 50)
    s_ms = _time_ms(lambda: tq.tq_scores(ctx, q, cache, seq, w.N, out=sc, workspace=ws), 50)
    a_ms = _time_ms(lambda: tq.tq_attend(ctx, q, cache, seq, w.N, out=out, workspace=ws), 50)
    assert tq.tq_status(ctx) == 0
    return {"report": "single_head_d128_b3", "quantize_8192_ms": round(q_ms, 4),
            "scores_64x8192_ms": round(s_ms, 4), "attend_64x8192_ms": round(a_ms, 4),
            "context_pages_gb10_pytorch": {"quantize_8192_ms": 31.04, "inner_product_64x8192_ms": 11.16},
            "note": "1.6 MB of packed cache, resident in L2: launch-latency bound"}


def report_cudacore():
    """The tensor-core split kernel against the CUDA-core comparison kernel
    (lookup tables; QJL term by sign-nibble tables, then by bit-plane
    popcounts) on one Llama-3.3-70B-shaped layer: tq_attend calls over the
    same 562 MB cache (larger than L2), CUDA events around each arm's calls."""
    import torch
    import kv_cache_vector_04_b200 as tq
    inputs = load_inputs()
    w = inputs.WORKLOADS[DEFAULT_WORKLOAD]
    dev = torch.device("cuda", 0)
    ctx = tq.tq_init(w.d, w.bits, 1)
    N = w.N
    cache = tq.new_cache(ctx, w.B, w.Hkv, N + 16, device=dev)
    k, v = inputs.kv_pair(w, N, layer=0, device=dev)
    tq.tq_quantize(ctx, k, v, torch.zeros(w.B, dtype=torch.int32, device=dev), cache)
    del k, v
    q = inputs.queries(w, layer=0, device=dev)
    seq = torch.full((w.B,), N, dtype=torch.int32, device=dev)
    ws = tq.new_workspace(ctx, w.B, w.Hq, w.Hkv, N)
    out = torch.empty((w.B, w.Hq, w.d), dtype=torch.float32, device=dev)
    per_tok = tq.tq_cache_layout(ctx)["tile_bytes"] // 16
    nbytes = w.B * w.Hkv * N * per_tok
    peak, peak_kind = measured_peaks()
    arms = [("tensor_core", lambda: tq.tq_attend(ctx, q, cache, seq, N, out=out, workspace=ws), 20),
            ("cuda_core_nibble_qjl", lambda: tq.tq_attend_cudacore(ctx, q, cache, seq, N, 1, out=out,
                                                                   workspace=ws), 5),
            ("cuda_core_popcount_qjl", lambda: tq.tq_attend_cudacore(ctx, q, cache, seq, N, 2, out=out,
                                                                     workspace=ws), 2)]
    res = {"report": "cudacore_llama70b_32k", "workload": w.name, "bytes_per_call": nbytes,
           "peak_gbs": peak, "peak_kind": peak_kind}
    for name, fn, reps in arms:
        clocks = ClockSampler(0)
        clocks.start()
        ms = _time_ms(fn, reps, warm=2)
        clk = clocks.stop()
        gbs = nbytes / (ms / 1e3) / 1e9
        res[name] = {"ms_per_call": round(ms, 3), "gbs": round(gbs, 1), "frac": round(gbs / peak, 4),
                     "calls": reps, "sm_mhz": clk.get("sm_mhz"), "reasons": clk.get("reasons")}
    assert tq.tq_status(ctx) == 0
    return res


def _brief(line: dict) -> dict:
    keep = {"value": line["value"], "unit": line["unit"], "ms_per_step": line["ms_per_step"],
            "ms_per_step_eager": line.get("ms_per_step_eager"),
            "ms_per_layer": line.get("ms_per_layer"),
            "pct_of_hbm_peak": line.get("pct_of_hbm_peak"),
            "attend_gbs": line["roofline"]["achieved"], "attend_frac": line["roofline"]["frac"],
            "quantize_mtok_s": (line.get("quantize") or {}).get("value"),
            "quantize_hbm_gbs": (line.get("quantize") or {}).get("hbm_gbs"),
            "config": line["config"]}
    return keep


def run_report(args, dist: Dist):
    base = dict(vars(args))
    base.update(no_cpu_baseline=True, no_e2e=True)

    def run(**kw):
        a = argparse.Namespace(**dict(base, **kw))
        return _brief(run_tq(a, dist))

    which = args.report
    if which in ("all", "single"):
        print(json.dumps(report_single_head()), flush=True)
    if which in ("all", "qwen3b"):
        print(json.dumps(dict(report="qwen2.5-3b_decode_8k",
                              **run(workload="qwen2.5-3b_decode_8k", layers=None))), flush=True)
    if which in ("all", "qwen32b"):
        print(json.dumps(dict(report="qwen2.5-32b_prefill_decode_128k",
                              **run(workload="qwen2.5-32b_prefill_decode_128k", layers=None,
                                    steps=32, warmup=3))), flush=True)
    if which in ("all", "sweep"):
        from kv_cache_vector_04_b200 import inputs
        for w in inputs.sweep_workloads():
            print(json.dumps(dict(report=w.name, **run(workload=w.name, layers=1, steps=10,
                                                         warmup=3))), flush=True)
    if which in ("all", "cudacore"):
        print(json.dumps(report_cudacore()), flush=True)
    if which in ("all", "formats"):
        from kv_cache_vector_04_b200 import inputs
        for w in inputs.format_workloads():
            print(json.dumps(dict(report=w.name, **run(workload=w.name, layers=1, steps=10,
                                                         warmup=3))), flush=True)


def secondary_workloads(args, dist: Dist) -> dict:
    """The other long-context workloads, measured after the bench line's own
    timed region and reported beside it: one layer of the Qwen2.5-32B-shaped
    128K decode (32 timed steps) and the nine sweep points at 65536 tokens.
    Each entry carries its own clock sample."""
    from kv_cache_vector_04_b200 import inputs
    base = dict(vars(args))
    base.update(no_cpu_baseline=True, no_e2e=True, no_graph=False)

    def run(**kw):
        line = run_tq(argparse.Namespace(**dict(base, **kw)), dist)
        return {"format": line["config"]["format"], "context": line["config"]["context"],
                "ms_per_layer": line["ms_per_layer"], "packed_gbs": line["value"],
                "attend_gbs": line["roofline"]["achieved"], "attend_frac": line["roofline"]["frac"],
                "quantize_mtok_s": (line.get("quantize") or {}).get("value"),
                "clocks": {"sm_mhz": line["clocks"].get("sm_mhz"),
                           "reasons": line["clocks"].get("reasons")}}

    out = {"note": "one layer each, step as one CUDA graph; attend_* from the step time "
                   "(prologue with the append + split + reduce); frac of the measured HBM peak"}
    out["qwen2.5-32b_prefill_decode_128k"] = run(workload="qwen2.5-32b_prefill_decode_128k",
                                                 layers=1, steps=32, warmup=3)
    for w in inputs.sweep_workloads():
        if w.N == 65536:
            out[w.name] = run(workload=w.name, layers=1, steps=10, warmup=3)
    return out


def main(argv=None):
    args = parse_args(argv)
    dist = Dist()
    if args.report:
        dist.init()
        try:
            run_report(args, dist)
        finally:
            dist.close()
        return 0
    if args.impl == "reference":
        # the oracle runs on the host; only rank 0 works, the others exit cleanly
        line = run_reference(args, dist)
        if line is not None:
            print(json.dumps(line), flush=True)
        return 0
    dist.init()
    try:
        line = run_tq(args, dist)
        if (dist.world == 1 and args.workload == DEFAULT_WORKLOAD and args.layers is None
                and not args.no_secondary):
            import torch
            torch.cuda.empty_cache()
            line["secondary"] = secondary_workloads(args, dist)
        if dist.rank == 0:
            print(json.dumps(line), flush=True)
    finally:
        dist.close()
    return 0


if __name__ == "__main__":
    sys.exit(main())
