"""Benchmark of the ragged pack -> attend -> CLS pipeline on one or more B200s.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Workload: the serving regime of "Dispatch-Aware Ragged Attention for Pruned
Vision Transformers" (abstract: BS=1-4; radpulse sections on the dispatch
floor): DeiT-S shapes (197 tokens, 6 heads, head_dim 64, f16), batch sizes
B in {1, 2, 4} and pruning rates {0, 25, 50, 80}% with +-10 points of
per-image jitter.  One step is twelve calls, one per (B, rate); a call is the
whole pipeline (pack with cu_seqlens, ragged attention with the CLS rows
extracted in its epilogue) through the C ABI, followed by a stream
synchronisation, so the time per call is host dispatch + device time.

The reported value is microseconds per call (lower is better), over all
calls of all ranks (with N GPUs each rank runs an independent replica).
Inputs are rotated over enough copies to exceed twice the L2 size, so every
call reads its inputs from HBM.  Extra keys report the host/device split,
CUDA-graph replay, a padded-SDPA baseline timed the same way, the roofline
of the attention kernel (here and on the larger B=32 / B=64 / B=512
workloads), and the CPU oracle timed on the host cores.
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

import synthetic  # noqa: E402

L2_BYTES = 126 * 1024 * 1024
CASES = [(B, p) for B in synthetic.SERVING_BATCHES for p in synthetic.SERVING_RATES]


def max_over_ranks(value: float, dist, device=None) -> float:
    """The largest of every rank's value (the job's time is its slowest rank's)."""
    if not dist:
        return float(value)
    import torch
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def us_per_call(ms: float, steps: int, calls_per_step: int, world: int) -> float:
    """Microseconds per call over all calls of all ranks, from the max-over-ranks time."""
    return ms * 1000.0 / (steps * calls_per_step * world)


FUSED_SOURCES = ("attn_resident.cuh", "pack.cuh", "mma_common.cuh", "common.cuh")
TRAFFIC_RECORD = os.path.join(ROOT, "profiles", "fused_serving_traffic.txt")


def fused_source_hash() -> str:
    import hashlib
    h = hashlib.sha256()
    for name in FUSED_SOURCES:
        with open(os.path.join(ROOT, "ragged_variable_length_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def recorded_traffic():
    """DRAM bytes per fused launch from the committed ncu record, or None when the
    kernel sources changed since the counters were taken."""
    try:
        fields = {}
        with open(TRAFFIC_RECORD) as f:
            for line in f:
                if ":" in line and not line.startswith("#"):
                    k, v = line.split(":", 1)
                    fields[k.strip()] = v.strip()
        if fields.get("kernel_source_sha256") != fused_source_hash():
            return None
        return int(fields["dram_bytes_per_launch_mean"])
    except (OSError, KeyError, ValueError):
        return None


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), "measured"
    except Exception:
        return 6650.0, 1590.0, "fallback"


# --------------------------------------------------------------------------
# clocks during the timed region
# --------------------------------------------------------------------------

class ClockSampler:
    """nvidia-smi in a child process, sampling every 100 ms (reads only)."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu = gpu_id
        self.proc = None
        self.lines = []
        self.t0 = self.t1 = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()
        time.sleep(0.3)

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def mark(self, which):
        setattr(self, which, time.time())

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.15)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        for ts, line in self.lines:
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append((ts, float(parts[1]), float(parts[2]), parts[4:]))
            except ValueError:
                continue
        if not rows:
            return None
        inside = [r for r in rows if self.t0 is not None and self.t0 <= r[0] <= self.t1 + 0.1]
        if not inside:
            inside = [min(rows, key=lambda r: abs(r[0] - (self.t1 or r[0])))]
        reasons = set()
        names = ["active_mask", "hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in inside:
            for name, val in zip(names[1:], r[3][1:]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(r[1] for r in inside), "sm_max_mhz": max(r[2] for r in inside),
                "reasons": sorted(reasons), "samples": len(inside)}


# --------------------------------------------------------------------------
# our arm
# --------------------------------------------------------------------------

def attn_bytes(w) -> int:
    """Algorithmic bytes of one attention launch: Q, K, V read and O written
    once, cu_seqlens read, CLS rows written."""
    e = w.elem_bytes
    return 4 * w.T * w.H * w.d * e + 4 * (w.B + 1) + w.B * w.H * w.d * e


def fused_bytes(w, packed_written: bool = True) -> int:
    """Algorithmic bytes of one fused pipeline launch: the mask, the kept dense
    q/k/v rows read once, the packed rows written (when materialised), the
    attention output and CLS rows written, cu_seqlens written."""
    e = w.elem_bytes
    rows = w.T * w.row_bytes
    return (w.B * w.L_full + rows * (2 if packed_written else 1) + w.T * w.H * w.d * e
            + w.B * w.H * w.d * e + 4 * (w.B + 1))


def pack_bytes(w) -> int:
    """Algorithmic bytes of one pack launch: the mask, the kept rows read and
    written, cu_seqlens written."""
    return w.B * w.L_full + 2 * w.T * w.row_bytes + 4 * (w.B + 1)


def optional(fn):
    """Runs one of the extra measurements.  A Python-level failure there is
    reported in its key (and its traceback on stderr) instead of ending the
    run before the JSON line with the headline number is printed."""
    try:
        return fn()
    except Exception as e:  # noqa: BLE001 - any failure of an extra is reported, not raised
        import traceback
        traceback.print_exc()
        return {"error": f"{type(e).__name__}: {e}"[:300]}


def run_ours(args, rank, world, dist):
    import torch
    import ragged_variable_length_b200 as rv

    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    rv.load()  # fails loudly if the CUDA library is missing
    # A created stream (the library records its pipeline graphs on one; the
    # legacy default stream cannot be captured) is current for everything below.
    stream = torch.cuda.Stream(device=dev)
    torch.cuda.set_stream(stream)
    hbm_peak, bf16_peak, peak_kind = peaks()

    # ---- inputs: enough copies of the 12 serving batches to exceed 2x L2 ----
    per_copy = sum(synthetic.serving(B, p).qkv.nbytes for B, p in CASES)
    ncopies = max(2, int(np.ceil(2 * L2_BYTES / per_copy)))
    workloads = {c: [synthetic.serving(B, p, copy=c) for B, p in CASES] for c in range(ncopies)}
    pipes = {c: [] for c in range(ncopies)}
    for c in range(ncopies):
        for w in workloads[c]:
            pl = rv.Pipeline(w.B, w.L_full, w.H, torch.float16, device=dev, flags=rv.RAGGED_PIPELINE_FUSED)
            pl.dense_qkv.copy_(torch.from_numpy(w.qkv).to(dev))
            pl.keep.copy_(torch.from_numpy(w.keep).to(dev))
            pl.bind_inputs(pl.dense_qkv, pl.keep)
            pipes[c].append(pl)
    torch.cuda.synchronize()

    # Every pipeline is also recorded as a CUDA graph (one kernel node), twice:
    # by torch (Pipeline.capture) and by libragged (Pipeline.record).  A
    # headline call is one crossing into libragged that launches its graph and
    # waits for it (ragged_pipeline_graph_launch with RAGGED_PIPELINE_SYNC).
    for c in range(ncopies):
        for pl in pipes[c]:
            pl.capture()
            pl.record()
    torch.cuda.synchronize()

    def step(s):
        for pl in pipes[s % ncopies]:
            pl.launch(sync=True)

    def step_torch_graph(s):
        for pl in pipes[s % ncopies]:
            pl.replay()
            stream.synchronize()

    def step_direct(s):
        for pl in pipes[s % ncopies]:
            pl.run_sync()   # one C call: enqueue, then wait for completion

    for s in range(args.warmup):
        step(s)
        step_direct(s)
        step_torch_graph(s)
    try:
        sampler = ClockSampler("GPU-" + str(torch.cuda.get_device_properties(dev).uuid))
    except Exception:
        sampler = ClockSampler(str(dev.index))
    sampler.start()
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler.mark("t0")
    e0.record(stream)
    for s in range(args.steps):
        step(s)
    e1.record(stream)
    torch.cuda.synchronize()
    sampler.mark("t1")
    if dist:
        dist.barrier()
    clocks = sampler.stop()
    ms = max_over_ranks(e0.elapsed_time(e1), dist, dev)
    calls = args.steps * len(CASES) * world
    value_us = us_per_call(ms, args.steps, len(CASES), world)

    # The same calls without the graph: one C call per pipeline run.
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    d0, d1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    d0.record(stream)
    for s in range(args.steps):
        step_direct(s)
    d1.record(stream)
    torch.cuda.synchronize()
    direct_ms = max_over_ranks(d0.elapsed_time(d1), dist, dev)
    direct_us = us_per_call(direct_ms, args.steps, len(CASES), world)

    # The same calls through torch's graph of the pipeline: replay, then a
    # stream synchronisation (two crossings into torch per call).
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    g0.record(stream)
    for s in range(args.steps):
        step_torch_graph(s)
    g1.record(stream)
    torch.cuda.synchronize()
    torch_graph_us = us_per_call(max_over_ranks(g0.elapsed_time(g1), dist, dev), args.steps, len(CASES), world)

    # Warm, reported separately: the same graph calls on one input copy only,
    # whose 12 batches (about 12 MiB) stay in L2 from one step to the next.
    for _ in range(args.warmup):
        step(0)
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    warm_start, warm_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    warm_start.record(stream)
    for _ in range(args.steps):
        step(0)
    warm_end.record(stream)
    torch.cuda.synchronize()
    warm_ms = max_over_ranks(warm_start.elapsed_time(warm_end), dist, dev)
    warm_us = us_per_call(warm_ms, args.steps, len(CASES), world)

    # ---- per-call host / device / total split, per case ----
    detail = {}
    reps = args.per_case_calls
    for i, (B, p) in enumerate(CASES):
        host, dev_t, tot = [], [], []
        for r in range(reps):
            pl = pipes[r % ncopies][i]
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            torch.cuda.synchronize()
            t0 = time.perf_counter()
            a.record(stream)
            h0 = time.perf_counter()
            pl()
            h1 = time.perf_counter()
            b.record(stream)
            stream.synchronize()
            host.append((h1 - h0) * 1e6)
            dev_t.append(a.elapsed_time(b) * 1e3)
            t0 = time.perf_counter()
            pl.launch(sync=True)
            tot.append((time.perf_counter() - t0) * 1e6)
        entry = {"calls": reps}
        for name, xs in (("host", host), ("device", dev_t), ("total", tot)):
            entry[f"{name}_us"] = round(statistics.median(xs), 2)
            entry[f"{name}_p10_us"] = round(float(np.percentile(xs, 10)), 2)
            entry[f"{name}_p90_us"] = round(float(np.percentile(xs, 90)), 2)
        # sequences/s from the synchronous total; useful TFLOP/s and the
        # roofline fraction from the device time of the call
        w0 = workloads[0][i]
        dev_s = statistics.median(dev_t) * 1e-6
        t_roof_case = max(fused_bytes(w0) / (hbm_peak * 1e9), w0.useful_flops() / (bf16_peak * 1e12))
        entry["seq_per_s"] = round(B / (statistics.median(tot) * 1e-6), 1)
        entry["useful_tflops"] = round(w0.useful_flops() / dev_s / 1e12, 4)
        entry["roofline_frac"] = round(t_roof_case / dev_s, 4)
        detail[f"b{B}_p{int(p * 100)}"] = entry

    # ---- where the host side of a headline call goes ----
    # A headline call is graph launch + kernel + stream synchronisation.  The
    # same pattern around a graph holding one trivial kernel (a one-element
    # fill) gives its floor; enqueue-only and idle-synchronise times split it.
    def host_split(n=2000):
        tiny = torch.zeros(1, device=dev)
        side = torch.cuda.Stream()
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            tiny.fill_(1.0)
            g_empty = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g_empty, stream=side):
                tiny.fill_(1.0)
        stream.wait_stream(side)
        torch.cuda.synchronize()
        pl = pipes[0][len(CASES) - 1]
        enq, idle, empty_call, call, lib_call = [], [], [], [], []
        for r in range(n):
            torch.cuda.synchronize()
            t0 = time.perf_counter()
            pl.replay()
            t1 = time.perf_counter()
            stream.synchronize()
            enq.append((t1 - t0) * 1e6)
            t0 = time.perf_counter()
            stream.synchronize()
            idle.append((time.perf_counter() - t0) * 1e6)
            t0 = time.perf_counter()
            g_empty.replay()
            stream.synchronize()
            empty_call.append((time.perf_counter() - t0) * 1e6)
            t0 = time.perf_counter()
            pl.replay()
            stream.synchronize()
            call.append((time.perf_counter() - t0) * 1e6)
            t0 = time.perf_counter()
            pl.launch(sync=True)
            lib_call.append((time.perf_counter() - t0) * 1e6)
        med = lambda xs: round(statistics.median(xs), 2)
        return {"case": f"b{CASES[-1][0]}_p{int(CASES[-1][1] * 100)}", "calls": n,
                "graph_replay_enqueue_us": med(enq), "stream_sync_idle_us": med(idle),
                "empty_kernel_graph_call_us": med(empty_call), "fused_graph_call_us": med(call),
                "fused_library_graph_call_us": med(lib_call),
                "note": "median over calls; empty_kernel_graph_call_us is the floor of graph launch + "
                        "one-kernel execution + synchronisation on this host through torch, the rest of a "
                        "call is the fused kernel beyond a trivial one; fused_graph_call_us goes through "
                        "torch (replay + synchronize), fused_library_graph_call_us is the headline call "
                        "(one crossing: ragged_pipeline_graph_launch with RAGGED_PIPELINE_SYNC)"}

    hsplit = optional(host_split)

    # ---- end to end from pinned host buffers ----
    host_in = {}
    for c in range(ncopies):
        for i, w in enumerate(workloads[c]):
            host_in[(c, i)] = (torch.from_numpy(w.qkv).pin_memory(), torch.from_numpy(w.keep).pin_memory(),
                               torch.empty((w.B, w.H, w.d), dtype=torch.float16).pin_memory())
    h2d = sum(host_in[(0, i)][0].nbytes + host_in[(0, i)][1].nbytes for i in range(len(CASES)))
    d2h = sum(host_in[(0, i)][2].nbytes for i in range(len(CASES)))

    def e2e_step(s):
        c = s % ncopies
        for i, pl in enumerate(pipes[c]):
            qkv_h, keep_h, cls_h = host_in[(c, i)]
            pl.dense_qkv.copy_(qkv_h, non_blocking=True)
            pl.keep.copy_(keep_h, non_blocking=True)
            pl.launch(sync=False)
            cls_h.copy_(pl.cls_out, non_blocking=True)
            stream.synchronize()

    for s in range(args.warmup):
        e2e_step(s)
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    x0, x1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    x0.record(stream)
    for s in range(args.steps):
        e2e_step(s)
    x1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(x0.elapsed_time(x1), dist, dev)
    e2e_us = us_per_call(e2e_ms, args.steps, len(CASES), world)
    # the last step's CLS rows must match the device result
    ok_e2e = all(torch.equal(host_in[((args.steps - 1) % ncopies, i)][2], pl.cls_out.cpu())
                 for i, pl in enumerate(pipes[(args.steps - 1) % ncopies]))

    # ---- kernel durations: CUDA graphs of back-to-back launches, CUDA events ----
    lib = rv.load()

    def attn_launcher(pl, w):
        D = w.H * w.d
        base = pl.packed_qkv.data_ptr()
        e = w.elem_bytes

        def launch(strm):
            st = lib.ragged_attn_fwd(base, base + D * e, base + 2 * D * e, 3 * D, w.d, pl.cu_seqlens.data_ptr(),
                                     w.B, w.L_full, w.H, w.d, w.scale, 0 if w.dtype == "f16" else 1,
                                     pl.out.data_ptr(), D, pl.cls_out.data_ptr(), strm)
            assert st == 0, rv.ragged_last_error()
        return launch

    def pack_launcher(pl, w):
        def launch(strm):
            st = lib.ragged_pack(pl.dense_qkv.data_ptr(), w.B, w.L_full, w.row_bytes, pl.keep.data_ptr(),
                                 pl.packed_qkv.data_ptr(), pl.cu_seqlens.data_ptr(), None, strm)
            assert st == 0, rv.ragged_last_error()
        return launch

    def graph_time(launchers, replays=3):
        """Average device time per launch of `launchers`, recorded back to back in
        one CUDA graph and replayed between two events on the launching stream."""
        side = torch.cuda.Stream()
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            for f in launchers:
                f(side.cuda_stream)
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=side):
                for f in launchers:
                    f(side.cuda_stream)
        stream.wait_stream(side)
        torch.cuda.synchronize()
        g.replay()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(replays):
            g.replay()
        b.record(stream)
        torch.cuda.synchronize()
        return a.elapsed_time(b) / 1000.0 / (replays * len(launchers))

    def pipeline_launcher(pl):
        def launch(strm):
            pl.bind_inputs(pl.dense_qkv, pl.keep, stream=strm)
            pl()
            pl.bind_inputs(pl.dense_qkv, pl.keep)
        return launch

    all_pw = [(pipes[c][i], workloads[c][i]) for c in range(ncopies) for i in range(len(CASES))]
    t_fused = graph_time([pipeline_launcher(p_) for p_, _ in all_pw])
    b_fused = float(np.mean([fused_bytes(w_) for _, w_ in all_pw]))
    t_attn = graph_time([attn_launcher(p_, w_) for p_, w_ in all_pw])
    t_pack = graph_time([pack_launcher(p_, w_) for p_, w_ in all_pw])
    b_attn = float(np.mean([attn_bytes(w_) for _, w_ in all_pw]))
    b_pack = float(np.mean([pack_bytes(w_) for _, w_ in all_pw]))
    flops = float(np.mean([w_.useful_flops() for _, w_ in all_pw]))
    roofline = {"bound": "hbm", "achieved": round(b_fused / t_fused / 1e9, 2), "peak": hbm_peak,
                "unit": "GB/s", "frac": round(b_fused / t_fused / 1e9 / hbm_peak, 4), "traffic": recorded_traffic(),
                "kernel": "attn_resident_kernel<__half, DenseRows> (fused pack + attention + CLS)",
                "avg_launch_us": round(t_fused * 1e6, 3), "bytes_per_launch": int(b_fused),
                "launches_timed": 3 * len(all_pw), "peak_kind": peak_kind,
                "timing": "CUDA graph of back-to-back launches over all input copies, CUDA events",
                "useful_tflops": round(flops / t_fused / 1e12, 4),
                "split_path": {"attention_us": round(t_attn * 1e6, 3), "attention_bytes": int(b_attn),
                               "attention_GBps": round(b_attn / t_attn / 1e9, 2),
                               "pack_us": round(t_pack * 1e6, 3), "pack_bytes": int(b_pack),
                               "pack_GBps": round(b_pack / t_pack / 1e9, 2)}}

    # ---- larger workloads: attention roofline (single GPU, same kernel family) ----
    def measure_larger():
        larger = {}
        for name, make, copies in (("deit_b_p80_b32", lambda c: synthetic.make_workload(
                                        "deit_b_p80_b32", 32, 197, 12,
                                        synthetic.deit_b_pruned80().lengths, "bf16", 1002, 1 + c), 36),
                                   ("hires384_b64", lambda c: synthetic.hires_384(seed=1004 + 100 * c), 3),
                                   ("sweep_b512_p0", lambda c: synthetic.sweep(0.0, seed=1005 + 100 * c), 1),
                                   ("sweep_b512_p50", lambda c: synthetic.sweep(0.5, seed=1005 + 100 * c), 2)):
            ws = [make(c) for c in range(copies)]
            pls = []
            for w in ws:
                pl = rv.Pipeline(w.B, w.L_full, w.H, torch.float16 if w.dtype == "f16" else torch.bfloat16, device=dev,
                                 flags=rv.RAGGED_PIPELINE_SPLIT)
                pl.dense_qkv.view(torch.int16).copy_(torch.from_numpy(w.qkv.view(np.int16)).to(dev))
                pl.keep.copy_(torch.from_numpy(w.keep).to(dev))
                pl()
                pls.append(pl)
            torch.cuda.synchronize()
            bts = float(np.mean([attn_bytes(w_) for w_ in ws]))
            fl = float(np.mean([w_.useful_flops() for w_ in ws]))
            t_roof = max(bts / (hbm_peak * 1e9), fl / (bf16_peak * 1e12))
            per_kernel = {}
            for kname, kcode in (("streaming", rv.RAGGED_ATTN_STREAMING), ("resident", rv.RAGGED_ATTN_RESIDENT),
                                 ("tcgen05", rv.RAGGED_ATTN_TCGEN05), ("persistent", rv.RAGGED_ATTN_PERSISTENT)):
                prev = rv.ragged_set_attn_kernel(kcode)
                try:
                    t = graph_time([attn_launcher(p_, w_) for p_, w_ in zip(pls, ws)], replays=max(3, 30 // copies))
                finally:
                    rv.ragged_set_attn_kernel(prev)
                per_kernel[kname] = {"avg_launch_us": round(t * 1e6, 2), "GBps": round(bts / t / 1e9, 1),
                                     "useful_tflops": round(fl / t / 1e12, 2), "roofline_frac": round(t_roof / t, 4)}
            t = graph_time([attn_launcher(p_, w_) for p_, w_ in zip(pls, ws)], replays=max(3, 30 // copies))
            larger[name] = {"auto": {"avg_launch_us": round(t * 1e6, 2), "roofline_frac": round(t_roof / t, 4)},
                            "kernels": per_kernel, "t_roof_us": round(t_roof * 1e6, 2),
                            "bytes_per_launch": int(bts), "useful_flops": int(fl),
                            "l2": f"inputs rotated over {copies} copies" if copies > 1 else "packed q/k/v exceed L2"}
            del pls
            torch.cuda.empty_cache()
        return larger

    # ---- per-launch floor of the attention kernels: one sequence of one token ----
    def launch_floor():
        w = synthetic.make_workload("one_token", 1, 1, 12, [1], "bf16", 1002, 9)
        pl = rv.Pipeline(1, 1, 12, torch.bfloat16, device=dev, flags=rv.RAGGED_PIPELINE_SPLIT)
        pl.dense_qkv.view(torch.int16).copy_(torch.from_numpy(w.qkv.view(np.int16)).to(dev))
        pl.keep.copy_(torch.from_numpy(w.keep).to(dev))
        pl()
        torch.cuda.synchronize()
        tiny = torch.zeros(1, device=dev)
        res = {"empty_torch_kernel_us": round(graph_time([lambda strm: tiny.fill_(1.0)] * 32, replays=10) * 1e6, 2)}
        for kname, kcode in (("streaming", rv.RAGGED_ATTN_STREAMING), ("resident", rv.RAGGED_ATTN_RESIDENT),
                             ("tcgen05", rv.RAGGED_ATTN_TCGEN05), ("persistent", rv.RAGGED_ATTN_PERSISTENT)):
            prev = rv.ragged_set_attn_kernel(kcode)
            try:
                res[kname + "_us"] = round(graph_time([attn_launcher(pl, w)] * 32, replays=10) * 1e6, 2)
            finally:
                rv.ragged_set_attn_kernel(prev)
        res["note"] = ("average per launch of 32 back-to-back launches in a CUDA graph: attention on one "
                       "1-token sequence with 12 heads (bf16), the fixed cost a launch pays whatever its work")
        return res

    single = world == 1 and not args.quick
    larger = optional(measure_larger) if single else {}
    if single and isinstance(larger, dict) and "error" not in larger:
        larger["launch_floor"] = optional(launch_floor)

    # ---- padded PyTorch SDPA baseline, same calls, same synchronisation ----
    padded = optional(lambda: padded_baseline(args, pipes, workloads, ncopies, stream))

    # ---- other attention paths on the same calls, and the mask producers ----
    comps = optional(lambda: comparators(args, pipes, workloads, stream)) if single else None
    masks = optional(mask_producers) if single else None
    block = optional(deit_block) if single else None

    # ---- CPU oracle on a bounded sample (rank 0, one GPU only) ----
    cpu = optional(lambda: cpu_baseline(min_seconds=10.0)) if rank == 0 and single else None

    gpu_launches = 1 * args.steps * len(CASES)   # one fused launch per call
    hw = {"metric": "ragged attn µs/call (host+device) at BS1-4; useful TFLOP/s & % roofline",
          "value": round(value_us, 3), "unit": "µs/call", "n_gpus": world, "steps": args.steps,
          "warmup": args.warmup, "ms_per_step": round(ms / args.steps, 4), "higher_is_better": False,
          "scaling": "weak", "vs_baseline": None, "dtype": "f16", "data": "synthetic",
          "config": {"workload": "serving_deit_s_b1-4_p0-80", "B": list(synthetic.SERVING_BATCHES),
                     "prune_rates": list(synthetic.SERVING_RATES), "jitter": 0.10, "L_full": 197,
                     "heads": 6, "head_dim": 64, "calls_per_step": len(CASES),
                     "call": "Pipeline.launch(sync=True): one call into libragged that launches its CUDA graph "
                             "of ragged_pipeline in fused mode (one kernel: pack, attention, CLS) and waits "
                             "for it; torch_graph_us_per_call = torch's graph of the same call, replay + stream "
                             "synchronize; direct_call_us_per_call = the pipeline as one C call that enqueues "
                             "and waits (RAGGED_PIPELINE_SYNC)",
                     "l2": f"inputs rotated over {ncopies} copies ({ncopies * per_copy / 2**20:.0f} MiB > 2x L2)",
                     "parallelism": "replicas" if world > 1 else "single"},
          "e2e": {"value": round(e2e_us, 3), "unit": "µs/call", "h2d_bytes_per_step": int(h2d),
                  "d2h_bytes_per_step": int(d2h), "cls_matches_device": bool(ok_e2e)},
          "gpu_launches": gpu_launches,
          "roofline": roofline,
          "direct_call_us_per_call": round(direct_us, 3),
          "torch_graph_us_per_call": round(torch_graph_us, 3),
          "warm_us_per_call": round(warm_us, 3),
          "per_case": detail,
          "host_split": hsplit,
          "padded_sdpa": padded,
          "comparators": comps,
          "mask_producers": masks,
          "deit_block": block,
          "larger_workloads_attention": larger,
          "clocks": clocks,
          "cpu_baseline": cpu}
    if rank == 0:
        print(json.dumps(hw), flush=True)


def sdpa_backend(q, k, v, mask) -> str:
    """Name of the SDPA backend torch's dispatcher picks for these arguments
    (torch._fused_sdp_choice, mapped through the public SDPBackend enum)."""
    try:
        import torch
        from torch.nn.attention import SDPBackend
        names = {int(b): n for n, b in SDPBackend.__members__.items()}
        return names.get(int(torch._fused_sdp_choice(q, k, v, mask, 0.0, False)), "unknown")
    except Exception as e:  # noqa: BLE001 - a private query; its failure is only reported
        return f"unknown ({type(e).__name__})"


def padded_baseline(args, pipes, workloads, ncopies, stream):
    """Pad every survivor set to the batch's longest (Lmax known on the host),
    mask padded keys, run torch SDPA, take the CLS rows.  Each case records
    the SDPA backend that runs."""
    import torch
    import torch.nn.functional as F
    backends = {}

    def call(pl, Lmax, probe=False):
        keep = pl.keep.bool()
        keep[:, 0] = True
        L = keep.sum(1)
        idx = torch.argsort((~keep).to(torch.int8), dim=1, stable=True)[:, :Lmax]
        B, _, three, H, d = pl.dense_qkv.shape
        g = torch.gather(pl.dense_qkv, 1, idx[:, :, None, None, None].expand(B, Lmax, three, H, d))
        q, k, v = g.permute(2, 0, 3, 1, 4).unbind(0)             # [B, H, Lmax, d]
        valid = torch.arange(Lmax, device=keep.device)[None, :] < L[:, None]
        if probe:   # outside the timed calls
            backends[(B, Lmax)] = sdpa_backend(q, k, v, valid[:, None, None, :])
        o = F.scaled_dot_product_attention(q, k, v, attn_mask=valid[:, None, None, :])
        return o[:, :, 0]

    res = {}
    reps = max(20, min(200, args.steps))
    for i, (B, p) in enumerate(CASES):
        # Every copy's shape once, untimed: each new Lmax makes the SDPA
        # backend (cuDNN) build a plan, which belongs to no steady-state call.
        for c in range(ncopies):
            call(pipes[c][i], int(workloads[c][i].Lmax))
        tot = []
        for r in range(reps):
            c = r % ncopies
            Lmax = int(workloads[c][i].Lmax)
            torch.cuda.synchronize()
            t0 = time.perf_counter()
            cls = call(pipes[c][i], Lmax)
            stream.synchronize()
            tot.append((time.perf_counter() - t0) * 1e6)
        ref = pipes[0][i].cls_out.float()
        err = float((call(pipes[0][i], int(workloads[0][i].Lmax), probe=True).float() - ref).abs().max())
        res[f"b{B}_p{int(p * 100)}"] = {"total_us": round(statistics.median(tot), 2), "max_abs_vs_ragged": err,
                                         "sdpa_backend": backends.get((B, int(workloads[0][i].Lmax)), "unknown")}
    return res


def comparators(args, pipes, workloads, stream):
    """Other ways to run the same per-sequence attention on the serving calls,
    each call synchronised like ours (median µs):
      varlen_attn         torch.nn.attention.varlen.varlen_attn (FlashAttention
                          varlen, the pages' FA2 comparator) on the packed q/k/v
                          of the same call, plus the CLS gather;
      nested_sdpa         scaled_dot_product_attention on jagged NestedTensors
                          built from the same packed q/k/v and cu_seqlens;
      torch_varlen_path   the whole call in PyTorch: keep mask -> nonzero (a
                          host sync) -> row gather -> cumsum cu_seqlens ->
                          varlen_attn -> CLS.
    max_abs_vs_ragged compares each CLS result with ours."""
    import torch
    import torch.nn.functional as F
    import ragged_variable_length_b200 as rv
    try:
        from torch.nn.attention.varlen import varlen_attn
    except ImportError:
        varlen_attn = None
    reps = max(20, min(200, args.steps))

    def timed(fn):
        tot = []
        for r in range(reps + 3):
            torch.cuda.synchronize()
            t0 = time.perf_counter()
            fn()
            stream.synchronize()
            if r >= 3:
                tot.append((time.perf_counter() - t0) * 1e6)
        return round(statistics.median(tot), 2)

    res = {}
    for i, (B, p) in enumerate(CASES):
        w, pl = workloads[0][i], pipes[0][i]
        H, d = w.H, w.d
        packed, cu = rv.ragged_pack(pl.dense_qkv, pl.keep)
        T, Lmax = int(w.lengths.sum()), int(w.Lmax)
        q, k, v = (packed[:T, j].contiguous() for j in range(3))
        first = cu[:-1].long()
        ref = pl.cls_out.float()
        entry = {}
        cases = {}
        if varlen_attn is not None:
            cases["varlen_attn"] = lambda: varlen_attn(q, k, v, cu, cu, Lmax, Lmax, scale=0.125)[first]

            def native():
                keep = pl.keep.bool()
                keep[:, 0] = True
                idx = keep.flatten().nonzero().squeeze(1)
                rows = pl.dense_qkv.view(-1, 3, H, d).index_select(0, idx)
                cuv = torch.zeros(B + 1, dtype=torch.int32, device=rows.device)
                cuv[1:] = torch.cumsum(keep.sum(1, dtype=torch.int32), 0)
                o = varlen_attn(rows[:, 0].contiguous(), rows[:, 1].contiguous(), rows[:, 2].contiguous(), cuv, cuv,
                                Lmax, Lmax, scale=0.125)
                return o[cuv[:-1].long()]
            cases["torch_varlen_path"] = native

        def nested():
            offs = cu.long()
            qn, kn, vn = (torch.nested.nested_tensor_from_jagged(x, offs).transpose(1, 2) for x in (q, k, v))
            o = F.scaled_dot_product_attention(qn, kn, vn, scale=0.125)
            return o.transpose(1, 2).values()[first]
        cases["nested_sdpa"] = nested
        for name, fn in cases.items():
            try:
                err = float((fn().float() - ref).abs().max())
                entry[name] = {"total_us": timed(fn), "max_abs_vs_ragged": err}
            except Exception as e:   # an unsupported path on this torch build is reported, not fatal
                entry[name] = {"unavailable": f"{type(e).__name__}: {str(e)[:120]}"}
        res[f"b{B}_p{int(p * 100)}"] = entry
        del packed, q, k, v
    return res


def mask_producers():
    """Device time per launch of the keep-mask producers, from a CUDA graph of
    50 back-to-back launches between two events: ragged_pack_topk (top-k
    selection fused into pack), ragged_mask_l2 (Threshold-l2 over the q
    features of each token) and, for reference, ragged_pack with a given
    mask, on a serving batch and on the B=512 sweep shape."""
    import torch
    import ragged_variable_length_b200 as rv
    res = {}
    for name, w in (("serving_b4", synthetic.serving(4, 0.5)), ("sweep_b512", synthetic.sweep(0.5))):
        rng = synthetic.rng_for(4001)
        dense = torch.from_numpy(w.qkv.view(np.int16)).cuda().view(torch.float16)
        scores = torch.from_numpy(rng.standard_normal((w.B, w.L_full)).astype(np.float32)).cuda()
        kc = torch.from_numpy(w.lengths.astype(np.int32)).cuda()
        packed = torch.empty((w.B * w.L_full, 3, w.H, 64), dtype=torch.float16, device="cuda")
        cu = torch.empty(w.B + 1, dtype=torch.int32, device="cuda")
        keep = torch.empty((w.B, w.L_full), dtype=torch.uint8, device="cuda")
        qfeat = dense.view(w.B, w.L_full, 3 * w.H * 64)[:, :, :w.H * 64]
        keep_given = torch.from_numpy(w.keep).cuda()
        out = {}
        for kname, fn in (("pack_topk", lambda: rv.ragged_pack_topk(dense, scores, kc, packed=packed, cu_seqlens=cu)),
                          ("mask_l2", lambda: rv.ragged_mask_l2(qfeat, 8.0, keep=keep)),
                          ("pack_given_mask", lambda: rv.ragged_pack(dense, keep_given, packed=packed,
                                                                     cu_seqlens=cu))):
            for _ in range(3):
                fn()
            torch.cuda.synchronize()
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph):
                for _ in range(50):
                    fn()
            graph.replay()
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            graph.replay()
            e1.record()
            torch.cuda.synchronize()
            out[kname] = round(e0.elapsed_time(e1) * 1000 / 50, 2)
            del graph
        res[name] = {"us_per_launch": out, "B": w.B, "L_full": w.L_full, "row_bytes": w.row_bytes}
    return res


def deit_block():
    """One random-weight DeiT-S encoder block (D = 384, 6 heads, MLP 1536, f16)
    on pruned tokens, two ways, each captured as a CUDA graph and timed by
    replay between events:
      packed  ragged_pack of the dense tokens -> LayerNorm -> QKV GEMM on the T
              survivors -> ragged_attn_fwd -> projection -> residual ->
              LayerNorm -> MLP (GELU) -> residual -> CLS rows (cu_seqlens);
      padded  survivors gathered to [B, Lmax] (Lmax from the generator) -> the
              same layers on B * Lmax rows with SDPA under a key-padding mask
              -> CLS rows.
    The GEMMs are cuBLAS (torch); T and Lmax come from the host-side
    generator, so neither path synchronises.  cls_max_abs compares the two."""
    import torch
    import torch.nn.functional as F
    import ragged_variable_length_b200 as rv
    D, H, d, M, L_full = 384, 6, 64, 1536, 197
    g = torch.Generator(device="cuda").manual_seed(5001)
    wt = lambda *shape: (torch.randn(*shape, device="cuda", generator=g) * 0.02).half()
    Wqkv, Wo, W1, W2 = wt(3 * D, D), wt(D, D), wt(M, D), wt(D, M)
    res = {}
    for B, rate in ((32, 0.5), (64, 0.5), (64, 0.0)):
        rng = synthetic.rng_for(5002, B * 10 + int(rate * 10))
        lengths = synthetic.serving_lengths(rng, B, rate)
        keep_np = synthetic.topk_keep_mask(rng, L_full, lengths)
        x = torch.from_numpy(rng.standard_normal((B, L_full, D)).astype(np.float16)).cuda()
        keep = torch.from_numpy(keep_np).cuda()
        T, Lmax = int(lengths.sum()), int(lengths.max())
        idx = torch.from_numpy(np.stack([np.concatenate([np.flatnonzero(r), np.zeros(Lmax - r.sum(), np.int64)])
                                         for r in keep_np])).cuda()
        valid = torch.arange(Lmax, device="cuda")[None, :] < torch.from_numpy(lengths).cuda()[:, None]

        def packed_block():
            xp, cu = rv.ragged_pack(x, keep)
            h = xp[:T]
            qkv = F.linear(F.layer_norm(h, (D,)), Wqkv).view(T, 3, H, d)
            a = rv.ragged_attn_fwd(qkv[:, 0], qkv[:, 1], qkv[:, 2], cu, L_full, 0.125).view(T, D)
            h = h + F.linear(a, Wo)
            h = h + F.linear(F.gelu(F.linear(F.layer_norm(h, (D,)), W1)), W2)
            return h[cu[:-1].long()]

        def padded_block():
            h = torch.gather(x, 1, idx[:, :, None].expand(B, Lmax, D))
            qkv = F.linear(F.layer_norm(h, (D,)), Wqkv).view(B, Lmax, 3, H, d).permute(2, 0, 3, 1, 4)
            a = F.scaled_dot_product_attention(qkv[0], qkv[1], qkv[2], attn_mask=valid[:, None, None, :])
            h = h + F.linear(a.transpose(1, 2).reshape(B, Lmax, D), Wo)
            h = h + F.linear(F.gelu(F.linear(F.layer_norm(h, (D,)), W1)), W2)
            return h[:, 0]

        entry = {"B": B, "prune_rate": rate, "T": T, "Lmax": Lmax}
        outs = {}
        for name, fn in (("packed_us", packed_block), ("padded_us", padded_block)):
            for _ in range(3):
                fn()
            torch.cuda.synchronize()
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph):
                out = fn()
            graph.replay()
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            for _ in range(20):
                graph.replay()
            e1.record()
            torch.cuda.synchronize()
            entry[name] = round(e0.elapsed_time(e1) * 1000 / 20, 2)
            outs[name] = out.float().clone()
            del graph
        entry["speedup"] = round(entry["padded_us"] / entry["packed_us"], 3)
        entry["cls_max_abs"] = float((outs["packed_us"] - outs["padded_us"]).abs().max())
        res[f"b{B}_p{int(rate * 100)}"] = entry
    return res


def cpu_baseline(min_seconds=10.0, single_thread_seconds=5.0):
    """The CPU oracle, as it stands, on the bench's calls (whole pipeline per
    call), on all host cores and, beside it, on one thread."""
    import oracle
    ws = [synthetic.serving(B, p) for B, p in CASES]

    def timed(seconds, threads):
        oracle.pipeline(ws[0], threads=threads)
        n, t0 = 0, time.perf_counter()
        while True:
            for w in ws:
                oracle.pipeline(w, threads=threads)
                n += 1
            if time.perf_counter() - t0 >= seconds:
                break
        return time.perf_counter() - t0, n

    cores = oracle.num_cores()
    dt, n = timed(min_seconds, 0)
    dt1, n1 = timed(single_thread_seconds, 1)
    return {"value": round(dt * 1e6 / n, 1), "unit": "µs/call", "cores": cores, "kind": "oracle",
            "sample": f"{n} calls ({n // len(ws)} passes over the 12 serving batches), fp64 C oracle, "
                      f"{cores} threads",
            "single_thread": {"value": round(dt1 * 1e6 / n1, 1), "unit": "µs/call", "cores": 1,
                              "sample": f"{n1} calls ({n1 // len(ws)} passes), fp64 C oracle, 1 thread"}}


# --------------------------------------------------------------------------
# reference arm: the CPU oracle on the same workload
# --------------------------------------------------------------------------

def run_reference(args, rank, world):
    if rank != 0:
        return
    import oracle
    ws = [synthetic.serving(B, p) for B, p in CASES]
    for s in range(args.warmup):
        oracle.pipeline(ws[s % len(ws)])
    n, t0 = 0, time.perf_counter()
    for s in range(args.steps):
        for w in ws:
            oracle.pipeline(w)
            n += 1
    dt = time.perf_counter() - t0
    v = dt * 1e6 / n
    cores = oracle.num_cores()
    print(json.dumps({
        "impl": "reference", "metric": "ragged attn µs/call (host+device) at BS1-4; useful TFLOP/s & % roofline",
        "value": round(v, 1), "unit": "µs/call", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(dt * 1000 / args.steps, 3), "higher_is_better": False, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": "serving_deit_s_b1-4_p0-80", "B": list(synthetic.SERVING_BATCHES),
                   "prune_rates": list(synthetic.SERVING_RATES), "L_full": 197, "heads": 6, "head_dim": 64,
                   "calls_per_step": len(CASES), "call": "CPU oracle pipeline (pack, attention, CLS)"},
        "cpu_baseline": {"value": round(v, 1), "unit": "µs/call", "cores": cores, "kind": "oracle",
                         "sample": f"{args.steps} steps x {len(ws)} calls, fp64 C oracle, {cores} threads"},
        "e2e": {"value": round(v, 1), "unit": "µs/call", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


PROFILE_CASES = ("serving", "hires", "sweep", "masks")


def run_profile_case(case: str) -> None:
    """One untimed pass of a workload, for an ncu capture of its kernels.

    serving: the fused pipeline once on each of the 12 serving batches.
    hires:   the 384x384 B=64 workload packed, then attention twice with each
             of the streaming mma.sync, tcgen05 and persistent tcgen05 kernels.
    sweep:   the B=512, 0% pruning sweep workload packed, then attention twice
             with each of the same three kernels.
    masks:   on the B=512, 50% pruning sweep workload: ragged_pack_topk,
             ragged_mask_l2 over the q features, ragged_pack with the given
             mask, each launched once.
    """
    import torch
    import ragged_variable_length_b200 as rv
    torch.cuda.set_device(0)
    if case == "serving":
        pls = []
        for B, p in CASES:
            w = synthetic.serving(B, p)
            pl = rv.Pipeline(w.B, w.L_full, w.H, torch.float16, flags=rv.RAGGED_PIPELINE_FUSED)
            pl.dense_qkv.copy_(torch.from_numpy(w.qkv))
            pl.keep.copy_(torch.from_numpy(w.keep))
            pls.append(pl)
        torch.cuda.synchronize()
        for pl in pls:
            pl()
    elif case in ("hires", "sweep"):
        w = synthetic.hires_384() if case == "hires" else synthetic.sweep(0.0)
        dt = torch.bfloat16 if w.dtype == "bf16" else torch.float16
        pl = rv.Pipeline(w.B, w.L_full, w.H, dt, flags=rv.RAGGED_PIPELINE_SPLIT)
        pl.dense_qkv.view(torch.int16).copy_(torch.from_numpy(w.qkv.view(np.int16)))
        pl.keep.copy_(torch.from_numpy(w.keep))
        for kern in (rv.RAGGED_ATTN_STREAMING, rv.RAGGED_ATTN_TCGEN05, rv.RAGGED_ATTN_PERSISTENT):
            rv.ragged_set_attn_kernel(kern)
            pl()
            pl()
        rv.ragged_set_attn_kernel(rv.RAGGED_ATTN_AUTO)
    elif case == "masks":
        w = synthetic.sweep(0.5)
        rng = synthetic.rng_for(4001)
        dense = torch.from_numpy(w.qkv.view(np.int16)).cuda().view(torch.float16)
        scores = torch.from_numpy(rng.standard_normal((w.B, w.L_full)).astype(np.float32)).cuda()
        kc = torch.from_numpy(w.lengths.astype(np.int32)).cuda()
        packed = torch.empty((w.B * w.L_full, 3, w.H, 64), dtype=torch.float16, device="cuda")
        cu = torch.empty(w.B + 1, dtype=torch.int32, device="cuda")
        qfeat = dense.view(w.B, w.L_full, 3 * w.H * 64)[:, :, :w.H * 64]
        keep_given = torch.from_numpy(w.keep).cuda()
        torch.cuda.synchronize()
        rv.ragged_pack_topk(dense, scores, kc, packed=packed, cu_seqlens=cu)
        rv.ragged_mask_l2(qfeat, 8.0)
        rv.ragged_pack(dense, keep_given, packed=packed, cu_seqlens=cu)
    torch.cuda.synchronize()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--quick", action="store_true", help="skip the larger workloads and the CPU baseline")
    ap.add_argument("--profile", choices=PROFILE_CASES, help="one untimed pass of a workload (for ncu), no JSON")
    ap.add_argument("--per-case-calls", type=int, default=None,
                    help="synchronised calls per (B, rate) for the host/device/total split "
                         "(default 1000; with --quick, the step count clamped to [20, 200])")
    args = ap.parse_args()
    if args.per_case_calls is None:
        args.per_case_calls = max(20, min(200, args.steps)) if args.quick else 1000
    if args.per_case_calls < 1:
        ap.error("--per-case-calls must be positive")
    if args.profile:
        run_profile_case(args.profile)
        return
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    dist = None
    if world > 1:
        import datetime
        import torch
        import torch.distributed as tdist
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", 0)))
        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
        dist = tdist
    try:
        run_ours(args, rank, world, dist)
    finally:
        if dist:
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
