"""Benchmark of the KV-cache format conversions on B200.

Headline workload (one JSON line on rank 0): the contiguous FP8 partial-window
workload -- K and V FP16 caches [4, 4096, 8, 128] (N(0,1) with 1% +-U(20,60000)
outliers and 0.1% subnormals), window offset 1024, width 2048.  One step is
fp16_to_fp8 of K and V, then fp8_to_fp16 of K and V, through the C ABI's fused
K+V calls (one launch per direction) on resident device buffers; the same step
through the single-tensor calls (4 launches) is reported in per_op.  The metric
is algorithmic GB/s (bytes read + bytes written: 3 bytes per element per
conversion).

Timing.  `--steps` consecutive steps run back to back (replayed from CUDA
graphs) between one pair of CUDA events.  The inputs are larger than L2: the
step keeps 8 independent copies of the workload (about 1.3 GB) and step i
converts copy i % 8, so every copy has been evicted by the other copies'
traffic before it comes round again; L2 is flushed once before the timed
steps.  The latency of one step on its own (L2 flushed before it, events
around it) is reported beside it under `isolated`.

Extra keys:
  roofline      the dominant kernel's achieved GB/s (algorithmic bytes per
                launch / mean CUDA-event duration) against the measured HBM
                copy peak in MEASURED_PEAKS.json;
  cpu_baseline  the CPU oracle (single-threaded C++) timed on this host on the
                same step;
  e2e           the same metric through the public Python API with pinned host
                buffers: host->device copy of the windows, the two conversions,
                device->host copy of the decoded windows every step, all inside
                the events; steps pipelined over three streams (upload,
                convert, download) and two buffer sets;
  per_op        every other conversion on its own workload (contiguous Q4/Q6,
                paged Q4 decode / prefill, the model-sized paged Q6 layers), each
                as GB/s and fraction of the HBM peak (--per-op, on by default).

Multi-GPU (torchrun, one rank per GPU): every rank converts its own shard of
sequences (weak scaling, no collective on the data path); the step time is the
max over ranks.  ``--impl reference`` times the CPU oracle instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch  # noqa: E402

import workloads  # noqa: E402

HEADLINE = dict(workload="fp8_window_contiguous", shape=(4, 4096, 8, 128), offset=1024, width=2048)
FLUSH_BYTES = 256 << 20
L2_BYTES = 126 << 20  # B200 L2 size
PEAKS_PATH = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_HBM_GBS = 6650.0

BYTES_PER_ELEM = {"fp8": 3.0, 4: 2.0 + 0.5 + 2.0 / 32, 6: 2.0 + 0.75 + 2.0 / 32, 8: 2.0 + 1.0 + 2.0 / 32}


# ------------------------------------------------------------- host logic ----

def shard_range(total: int, rank: int, world: int):
    """Contiguous share [lo, hi) of `total` units for `rank` of `world` (sizes differ by <= 1)."""
    base, rem = divmod(total, world)
    lo = rank * base + min(rank, rem)
    return lo, lo + base + (1 if rank < rem else 0)


def max_over_ranks(value: float, device=None) -> float:
    """Max of a per-rank float over the process group (identity without one)."""
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def hbm_peak():
    try:
        with open(PEAKS_PATH) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic.txt")


# the sources the conversion kernels (and their launch code) are built from; the
# attention kernels and the bulk-copy engine do not affect the headline kernel
CONVERSION_SOURCES = ("codec.cuh", "tiles.cuh", "ops.cuh", "ldg_engine.cuh", "kvq.cu")


def kernel_source_digest() -> str:
    """sha256 over the conversion kernels' CUDA sources, to tell whether recorded ncu
    counters of the headline kernel are current."""
    import hashlib

    h = hashlib.sha256()
    for name in CONVERSION_SOURCES:
        with open(os.path.join(ROOT, "kv_cache_quantization_fp16_b200", "csrc", name), "rb") as fh:
            h.update(name.encode() + fh.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str):
    """DRAM bytes (read + write) per launch of `kernel` on the headline workload from the
    committed ncu summary, or None when the kernels changed since it was captured."""
    try:
        with open(TRAFFIC_FILE) as f:
            for line in f:
                parts = line.split()
                if len(parts) == 3 and not line.startswith("#") and parts[0] == kernel:
                    return int(parts[1]) if parts[2] == kernel_source_digest() else None
    except OSError:
        pass
    return None


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons while running."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self.marks = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            threading.Thread(target=self._read, daemon=True).start()
        except (OSError, ValueError):
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def mark(self):
        self.marks.append(time.time())

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        rows = []
        for t, line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append((t, float(parts[1]), float(parts[2]), parts[5:9]))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        lo, hi = (self.marks[0], self.marks[-1]) if len(self.marks) >= 2 else (rows[0][0], rows[-1][0])
        inside = [r for r in rows if lo <= r[0] <= hi] or rows
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in inside for n, v in zip(names, r[3]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(r[1] for r in inside), "sm_max_mhz": max(r[2] for r in inside),
                "reasons": reasons, "samples": len(inside)}


# ---------------------------------------------------------- GPU workloads ----

class L2Flush:
    """Evict L2 between timed steps without leaving dirty lines behind: write a buffer
    twice the size of L2, then read another one, so the lines the next step evicts
    are clean and no write-back of the flush lands inside its timing."""

    def __init__(self, dev, nbytes=FLUSH_BYTES):
        self.w = torch.empty(nbytes, dtype=torch.uint8, device=dev)
        self.r = torch.zeros(nbytes // 4, dtype=torch.int32, device=dev)

    def __call__(self):
        self.w.zero_()
        self.sink = torch.amax(self.r)


STREAM_SETS = 8  # input sets a stream of steps rotates through (8 x ~168 MB, well above the 126 MB L2)


class Fp8Step:
    """Headline step on one rank: FP8 encode then decode of the K and V windows, through
    the fused K+V calls (one launch per direction).  The step holds `sets` independent
    copies of the workload; step i converts copy i % sets, so a stream of steps never
    finds its inputs in L2 (every copy is evicted by the others' traffic before it
    comes round again)."""

    def __init__(self, kvq, dev, batch, seed_shift=0, sets=STREAM_SETS):
        B, S, H, D = HEADLINE["shape"]
        shape = (batch, S, H, D)
        self.kvq, self.batch = kvq, batch
        self.sets = []
        for r in range(sets):
            k, v = workloads.fp8_window(seed=workloads.SEED_BASE + 2 + seed_shift + 100003 * r, shape=shape,
                                        device=dev)
            self.sets.append(dict(k=k, v=v, k8=torch.zeros(shape, dtype=torch.uint8, device=dev),
                                  v8=torch.zeros(shape, dtype=torch.uint8, device=dev),
                                  ky=torch.zeros_like(k), vy=torch.zeros_like(v)))
        first = self.sets[0]
        self.set_bytes = sum(t.numel() * t.element_size() for t in first.values())
        self.k, self.v, self.k8, self.v8, self.ky, self.vy = (first[n] for n in ("k", "v", "k8", "v8", "ky", "vy"))
        self.off, self.w = HEADLINE["offset"], HEADLINE["width"]
        self.elems_per_tensor = batch * self.w * H * D
        self.launch_bytes = BYTES_PER_ELEM["fp8"] * 2 * self.elems_per_tensor  # K and V
        self.bytes_per_step = 2 * self.launch_bytes
        self.launches_per_step = 2
        self.names = ["fp16_to_fp8_kv", "fp8_to_fp16_kv"]

    def launch(self, j, i=0):
        """Launch j (0: encode, 1: decode) of step i alone."""
        t = self.sets[i % len(self.sets)]
        kvq, b, o, w = self.kvq, self.batch, self.off, self.w
        if j == 0:
            kvq.fp16_to_fp8_kv(t["k"], t["k8"], t["v"], t["v8"], b, o, w)
        else:
            kvq.fp8_to_fp16_kv(t["k8"], t["ky"], t["v8"], t["vy"], b, o, w)

    def run(self, i=0, ev=None):
        """Step i (input copy i % sets); `ev`, if given, is an event recorded between
        the two conversions."""
        t = self.sets[i % len(self.sets)]
        kvq, b, o, w = self.kvq, self.batch, self.off, self.w
        kvq.fp16_to_fp8_kv(t["k"], t["k8"], t["v"], t["v8"], b, o, w)
        if ev is not None:
            ev.record()
        kvq.fp8_to_fp16_kv(t["k8"], t["ky"], t["v8"], t["vy"], b, o, w)


def capture(fn, n_marks=0):
    """Capture fn(marks) in a CUDA graph (after one eager warm-up on a side stream), so
    a step replays its launches back to back without host launch gaps.  `marks` are
    external events recorded between the launches, readable after each replay."""
    marks = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(n_marks)]
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        fn(None)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn(marks if n_marks else None)
    torch.cuda.synchronize()
    return g, marks


def time_device(fn, steps, warmup, flush, sampler=None, n_marks=0, collective=True):
    """Per-step CUDA-event times (ms) of the captured fn, with an L2 flush (outside the
    events) before each step.  With marks, also the per-launch segments of every step.
    `collective`: bracket the timed region with a barrier over all ranks (every rank must
    then make the same call); False for rank-local measurements."""
    g, marks = capture(fn, n_marks)
    for _ in range(warmup):
        flush()
        g.replay()
    torch.cuda.synchronize()
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    segs = []
    if collective:
        _barrier()
    torch.cuda.synchronize()
    if sampler:
        sampler.mark()
    for i in range(steps):
        flush()
        starts[i].record()
        g.replay()
        ends[i].record()
        if n_marks:
            ends[i].synchronize()
            pts = [starts[i]] + marks + [ends[i]]
            segs.append([a.elapsed_time(b) for a, b in zip(pts[:-1], pts[1:])])
    torch.cuda.synchronize()
    if sampler:
        sampler.mark()
    if collective:
        _barrier()
    per_step = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    del g
    return per_step, segs


def _barrier():
    import torch.distributed as dist

    if dist.is_available() and dist.is_initialized():
        dist.barrier()


def _upload_graph(g):
    """Upload an instantiated CUDA graph to the device (driver cuGraphUpload) so that its
    first replay inside a timed region costs what later replays cost; a no-op where the
    driver call is unavailable."""
    import ctypes

    try:
        drv = ctypes.CDLL("libcuda.so.1")
        drv.cuGraphUpload(ctypes.c_void_p(g.raw_cuda_graph_exec()),
                          ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    except (OSError, AttributeError, RuntimeError):
        pass


def _stream_graph(launch, n):
    """CUDA graph of steps 0..n-1 of `launch(i)`, back to back, uploaded to the device."""
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for i in range(n):
            launch(i)
    _upload_graph(g)
    return g


def time_stream(launch, sets, steps, warmup, flush, sampler=None, collective=True, chunk=None):
    """Mean device time (ms) per step of `steps` consecutive steps, timed by one pair of
    CUDA events around all of them.  Step i is launch(i); it converts input copy i % sets,
    so no step finds its inputs in L2 (sets = 1 for workloads larger than L2).  The steps
    are replayed from CUDA graphs of `chunk` steps (a multiple of `sets`; about 256 by
    default, so that graph boundaries, which break the chaining of launches, are rare),
    plus one graph for the remainder.  L2 is flushed once before the timed region, and
    with `collective` a barrier over all ranks brackets it."""
    if chunk is None:
        chunk = sets * max(1, 256 // sets)
    cur = torch.cuda.current_stream()
    side = torch.cuda.Stream()
    side.wait_stream(cur)
    eager = min(warmup, sets)  # the first warm-up steps run eagerly, so first-call set-up precedes capture
    with torch.cuda.stream(side):
        for i in range(eager):
            launch(i)
    cur.wait_stream(side)
    torch.cuda.synchronize()
    graphs = {}

    def run(n):
        for m in [chunk] * (n // chunk) + ([n % chunk] if n % chunk else []):
            if m not in graphs:
                graphs[m] = _stream_graph(launch, m)
            graphs[m].replay()

    run(warmup - eager)
    for m in {chunk if steps >= chunk else 0, steps % chunk} - {0}:  # capture before timing
        if m not in graphs:
            graphs[m] = _stream_graph(launch, m)
    flush()
    torch.cuda.synchronize()
    if collective:
        _barrier()
    torch.cuda.synchronize()
    if sampler:
        sampler.mark()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    run(steps)
    e.record()
    torch.cuda.synchronize()
    if sampler:
        sampler.mark()
    if collective:
        _barrier()
    ms = s.elapsed_time(e) / steps
    graphs.clear()
    return ms


def stream_shares(step, sets, reps=20):
    """Fraction of a stream step taken by each of its two launches: the same stream with an
    event between every two launches (captured in the graph), averaged over `reps` replays.
    Event nodes serialize the launches, so only the proportions are used."""
    n = sets
    evs = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(2 * n + 1)]
    cur = torch.cuda.current_stream()
    side = torch.cuda.Stream()
    side.wait_stream(cur)
    with torch.cuda.stream(side):
        for i in range(n):
            step.run(i)
    cur.wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for i in range(n):
            evs[2 * i].record()
            step.run(i, evs[2 * i + 1])
        evs[2 * n].record()
    seg = [0.0, 0.0]
    for _ in range(reps):
        g.replay()
        torch.cuda.synchronize()
        for i in range(n):
            seg[0] += evs[2 * i].elapsed_time(evs[2 * i + 1])
            seg[1] += evs[2 * i + 1].elapsed_time(evs[2 * i + 2])
    del g
    tot = seg[0] + seg[1]
    return [x / tot for x in seg], [x / (reps * n) for x in seg]


def e2e_fp8(kvq, step: Fp8Step, steps, warmup, dev):
    """The headline step end to end through the public Python API, from pinned host
    buffers: every step copies its K/V windows host -> device, runs the two fused
    conversions and copies the decoded windows device -> host.  Steps are pipelined
    the way a serving loop would run them: uploads on one stream, conversions on a
    second, downloads on a third, two device buffer sets used alternately, so step
    i+1's upload overlaps step i's download (PCIe is full duplex).  The timed region
    runs from before the first upload to after the last download."""
    B, S, H, D = step.k.shape
    o, w = step.off, step.w
    sets = step.sets[:2]
    host_in = [(t["k"].cpu().pin_memory(), t["v"].cpu().pin_memory()) for t in sets]
    host_out = [(torch.empty_like(hk).pin_memory(), torch.empty_like(hv).pin_memory()) for hk, hv in host_in]
    s_in, s_cv, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in sets]
    ev_cv = [torch.cuda.Event() for _ in sets]
    ev_out = [torch.cuda.Event() for _ in sets]
    for e in ev_cv + ev_out:
        e.record()

    def once(i):
        r = i % 2
        t, (hk, hv), (yk, yv) = sets[r], host_in[r], host_out[r]
        with torch.cuda.stream(s_in):
            s_in.wait_event(ev_cv[r])  # the conversions of step i-2 are done with this set's inputs
            for b in range(B):
                t["k"][b, o:o + w].copy_(hk[b, o:o + w], non_blocking=True)
                t["v"][b, o:o + w].copy_(hv[b, o:o + w], non_blocking=True)
            ev_in[r].record(s_in)
        with torch.cuda.stream(s_cv):
            s_cv.wait_event(ev_in[r])
            s_cv.wait_event(ev_out[r])  # the download of step i-2 is done with this set's outputs
            kvq.fp16_to_fp8_kv(t["k"], t["k8"], t["v"], t["v8"], B, o, w)
            kvq.fp8_to_fp16_kv(t["k8"], t["ky"], t["v8"], t["vy"], B, o, w)
            ev_cv[r].record(s_cv)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_cv[r])
            for b in range(B):
                yk[b, o:o + w].copy_(t["ky"][b, o:o + w], non_blocking=True)
                yv[b, o:o + w].copy_(t["vy"][b, o:o + w], non_blocking=True)
            ev_out[r].record(s_out)

    for i in range(warmup):
        once(i)
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(s_in)
    for i in range(steps):
        once(i)
    s_out.wait_stream(s_in)
    s_out.wait_stream(s_cv)
    end.record(s_out)
    torch.cuda.synchronize()
    ms = start.elapsed_time(end) / steps
    win_bytes = B * w * H * D * 2
    return ms, 2 * win_bytes, 2 * win_bytes


def per_op_measurements(kvq, dev, peak, steps, flush, step, include_model=True):
    """Each remaining conversion on its own workload.  Throughput rows time `steps`
    consecutive launches (time_stream) on inputs larger than L2: workloads above the L2
    size as they are, smaller ones rotating through independent input copies.  Rows
    whose launch moves under a megabyte (paged decode, width 1) report the latency of one
    launch on its own instead (L2 flushed before it, CUDA events around it)."""
    out = []

    def record(name, config, nbytes, launch, sets=1, n=steps, stream=None):
        if stream is None:
            stream = nbytes >= 1 << 20
        if stream:
            ms, timing = time_stream(launch, sets, n, 3, flush, collective=False), "stream"
            if sets > 1:
                timing += f", {sets} rotating input copies"
            if nbytes < 1 << 20:
                timing += " (inputs stay in L2, as a just-written decode token's would)"
        else:
            per, _ = time_device(lambda ev: launch(0), n, 3, flush, collective=False)
            ms, timing = statistics.mean(per), "isolated launch, L2 flushed"
        out.append({"op": name, "config": config, "bytes": int(nbytes), "us": round(ms * 1e3, 2),
                    "gbs": round(nbytes / ms / 1e6, 1), "frac": round(nbytes / ms / 1e6 / peak, 3),
                    "timing": timing})

    # the headline step through the page's single-tensor calls (4 launches instead of 2)
    B, S, H, D = HEADLINE["shape"]
    o, w = HEADLINE["offset"], HEADLINE["width"]

    def per_tensor_step(i):
        t = step.sets[i % len(step.sets)]
        kvq.fp16_to_fp8(t["k"], t["k8"], B, o, w)
        kvq.fp16_to_fp8(t["v"], t["v8"], B, o, w)
        kvq.fp8_to_fp16(t["k8"], t["ky"], B, o, w)
        kvq.fp8_to_fp16(t["v8"], t["vy"], B, o, w)
    record("fp8_step_single_tensor_calls", "headline window, fp16_to_fp8(K), (V), fp8_to_fp16(K), (V): 4 launches",
           4 * BYTES_PER_ELEM["fp8"] * B * w * H * D, per_tensor_step, sets=len(step.sets))

    # contiguous Q4 / Q6 / Q8, channel outliers [16, 8192, 8, 128] (537 MB of FP16 K+V)
    k, v = workloads.channel_outliers(device=dev)
    B, S, H, D = k.shape
    n = 2 * k.numel()
    ky, vy = torch.empty_like(k), torch.empty_like(v)
    for wb in (4, 6, 8):
        cs, ss = kvq.q_shapes(tuple(k.shape), wb)
        kc = torch.empty(cs, dtype=torch.uint8, device=dev)
        vc = torch.empty_like(kc)
        ks = torch.empty(ss, dtype=torch.float16, device=dev)
        vs = torch.empty_like(ks)
        cfg = f"contiguous [16,8192,8,128] K+V wbits={wb}"
        record(f"fp16_to_q_kv/q{wb}", cfg, BYTES_PER_ELEM[wb] * n,
               lambda i: kvq.fp16_to_q_kv(k, kc, ks, v, vc, vs, B, 0, S, 0, None, None, wb))
        record(f"q_to_fp16_kv/q{wb}", cfg, BYTES_PER_ELEM[wb] * n,
               lambda i: kvq.q_to_fp16_kv(kc, ky, ks, vc, vy, vs, B, 0, S, 0, None, None, wb))
        del kc, vc, ks, vs
    # FP8 alone on the big tensor
    k8 = torch.empty(k.shape, dtype=torch.uint8, device=dev)
    record("fp16_to_fp8", "contiguous [16,8192,8,128] K", 3.0 * k.numel(),
           lambda i: kvq.fp16_to_fp8(k, k8, B, 0, S))
    record("fp8_to_fp16", "contiguous [16,8192,8,128] K", 3.0 * k.numel(),
           lambda i: kvq.fp8_to_fp16(k8, ky, B, 0, S))
    del k, v, ky, vy, k8
    torch.cuda.empty_cache()

    # paged Q4 / FP8 decode and prefill on the 2048-page pool.  Input copy r of the
    # prefill rows is the same pool read through a block table whose pages are shifted by
    # 256 r (mod 2048): the windows land on other physical pages.
    pool = workloads.paged_pool(device=dev)
    P, ps, H, D = pool.k.shape
    sets = STREAM_SETS
    bts = [torch.where(pool.block_table >= 0, (pool.block_table + (P // sets) * r) % P, pool.block_table)
           for r in range(sets)]
    cs, ss = kvq.q_shapes(tuple(pool.k.shape), 4)
    kc = torch.zeros(cs, dtype=torch.uint8, device=dev)
    vc = torch.zeros_like(kc)
    ks = torch.zeros(ss, dtype=torch.float16, device=dev)
    vs = torch.zeros_like(ks)
    lens = pool.cache_seqlens.cpu()
    k8p, v8p = torch.zeros(pool.k.shape, dtype=torch.uint8, device=dev), torch.zeros(pool.k.shape, dtype=torch.uint8,
                                                                                    device=dev)
    sl = pool.cache_seqlens
    for phase, off, w in (("decode", 0, 1), ("prefill", -512, 512)):
        npos = sum(max(0, int(L) + off + w) - max(0, int(L) + off) for L in lens)
        nb8 = BYTES_PER_ELEM["fp8"] * 2 * npos * H * D
        cfg8 = f"paged 2048x256x8x128 pool, 32 seqs, {phase} width={w}, K+V"
        record(f"fp16_to_fp8_kv/{phase}", cfg8, nb8,
               lambda i: kvq.fp16_to_fp8_kv(pool.k, k8p, pool.v, v8p, 32, off, w, ps, sl, bts[i % sets]), sets)
        record(f"fp8_to_fp16_kv/{phase}", cfg8, nb8,
               lambda i: kvq.fp8_to_fp16_kv(k8p, pool.k, v8p, pool.v, 32, off, w, ps, sl, bts[i % sets]), sets)
        nb = BYTES_PER_ELEM[4] * 2 * npos * H * D
        cfg = f"paged 2048x256x8x128 pool, 32 seqs, {phase} width={w}"
        record(f"fp16_to_q_kv/q4/{phase}", cfg, nb,
               lambda i: kvq.fp16_to_q_kv(pool.k, kc, ks, pool.v, vc, vs, 32, off, w, ps, sl, bts[i % sets], 4),
               sets)
        record(f"q_to_fp16_kv/q4/{phase}", cfg, nb,
               lambda i: kvq.q_to_fp16_kv(kc, pool.k, ks, vc, pool.v, vs, 32, off, w, ps, sl, bts[i % sets], 4),
               sets)
        if phase == "decode":  # the same single-token launches back to back
            record("fp16_to_q_kv/q4/decode/stream", cfg, nb,
                   lambda i: kvq.fp16_to_q_kv(pool.k, kc, ks, pool.v, vc, vs, 32, off, w, ps, sl, bts[i % sets], 4),
                   sets, stream=True)
            record("fp16_to_fp8_kv/decode/stream", cfg8, nb8,
                   lambda i: kvq.fp16_to_fp8_kv(pool.k, k8p, pool.v, v8p, 32, off, w, ps, sl, bts[i % sets]),
                   sets, stream=True)
    del kc, vc, ks, vs, k8p, v8p
    torch.cuda.empty_cache()

    # decode attention straight from the quantized pool: 32 sequences, 32 query heads
    # (4 per kv head), one new token each, every cached position attended (>= 280 MB of
    # codes and scales per launch)
    for wb in (4, 6, 8):
        fn, nb = attention_setup(kvq, dev, pool, wb)
        record(f"decode_attention_q/q{wb}/paged",
               f"paged 2048x256x8x128 pool, 32 seqs, 32 query heads, wbits={wb}", nb, lambda i: fn())
        del fn
        torch.cuda.empty_cache()
    fn, nb = attention_setup_fp8(kvq, dev, pool)
    record("decode_attention_fp8/paged", "paged 2048x256x8x128 pool, 32 seqs, 32 query heads, E5M2", nb,
           lambda i: fn())
    del fn
    torch.cuda.empty_cache()

    # the small-batch end of decode: one sequence of 16384 positions (contiguous Q4
    # [1, 16384, 8, 128], 32 query heads); 8 independent caches rotate, so that the 18.9 MB a
    # launch reads is not in L2
    fns, nb = attention_batch1_setup(kvq, dev)
    record("decode_attention_q/q4/batch1", "contiguous [1, 16384, 8, 128] Q4, 1 sequence, 32 query heads", nb,
           lambda i: fns[i % len(fns)](), sets=len(fns))
    del fns
    torch.cuda.empty_cache()
    del pool
    torch.cuda.empty_cache()

    if include_model:
        out.extend(model_layers(kvq, dev, peak, min(20, max(3, steps // 10)), flush))
    return out


ATTN_QUERY_HEADS = 32


def attention_bytes(lens, kv_heads, head_dim, wbits, n_heads=ATTN_QUERY_HEADS):
    """Algorithmic bytes of one decode_attention_q launch: the K and V codes and scales
    of every attended position, the queries read and the outputs written."""
    per_row = head_dim * wbits // 8 + 2 * (head_dim // 32)
    npos = sum(int(L) for L in lens)
    return 2 * npos * kv_heads * per_row + 2 * 2 * len(lens) * n_heads * head_dim


def attention_batch1_setup(kvq, dev, seq_len=16384, copies=8, n_heads=ATTN_QUERY_HEADS):
    """`copies` independent Q4 caches of one sequence ([1, seq_len, 8, 128], quantized untimed)
    and the decode-attention launch over each; returns (launches, algorithmic bytes per launch)."""
    H, D = 8, 128
    shape = (1, seq_len, H, D)
    cs, ss = kvq.q_shapes(shape, 4)
    lens = torch.full((1,), seq_len, dtype=torch.int32, device=dev)
    ws = torch.empty(max(16, kvq.attention_workspace_bytes(shape, 1, n_heads)), dtype=torch.uint8, device=dev)
    fns = []
    for i in range(copies):
        k, v = workloads.normal_kv(shape, workloads.SEED_BASE + 90 + i, device=dev)
        kc, vc = (torch.empty(cs, dtype=torch.uint8, device=dev) for _ in range(2))
        ks, vs = (torch.empty(ss, dtype=torch.float16, device=dev) for _ in range(2))
        kvq.fp16_to_q_kv(k, kc, ks, v, vc, vs, 1, 0, seq_len, 0, None, None, 4)
        del k, v
        g = torch.Generator(device="cpu").manual_seed(workloads.SEED_BASE + 78 + i)
        q = torch.randn(1, n_heads, D, generator=g).half().to(dev)
        out = torch.empty_like(q)

        def fn(q=q, kc=kc, ks=ks, vc=vc, vs=vs, out=out):
            kvq.decode_attention_q(q, kc, ks, vc, vs, out, 1, lens, 4, 1.0 / math.sqrt(D), workspace=ws)
        fn()
        fns.append(fn)
    return fns, attention_bytes([seq_len], H, D, 4, n_heads)


def attention_setup_fp8(kvq, dev, pool, n_heads=ATTN_QUERY_HEADS):
    """Encode the whole pool to E5M2 (untimed) and return (launch, algorithmic bytes) of decode
    attention over it: one byte per cached element, no scales."""
    P, ps, H, D = pool.k.shape
    batch = pool.cache_seqlens.numel()
    k8 = torch.zeros(pool.k.shape, dtype=torch.uint8, device=dev)
    v8 = torch.zeros_like(k8)
    full = pool.block_table.shape[1] * ps
    kvq.fp16_to_fp8_kv(pool.k, k8, pool.v, v8, batch, -full, full, ps, pool.cache_seqlens, pool.block_table)
    g = torch.Generator(device="cpu").manual_seed(workloads.SEED_BASE + 77)
    q = torch.randn(batch, n_heads, D, generator=g).half().to(dev)
    out = torch.empty_like(q)
    ws = torch.empty(max(16, kvq.attention_workspace_bytes(tuple(pool.k.shape), batch, n_heads, ps,
                                                           pool.block_table.shape[1])), dtype=torch.uint8, device=dev)
    scale = 1.0 / math.sqrt(D)

    def fn():
        kvq.decode_attention_fp8(q, k8, v8, out, batch, pool.cache_seqlens, scale, ps, pool.block_table, ws)
    fn()
    npos = sum(int(L) for L in pool.cache_seqlens.cpu().tolist())
    return fn, 2 * npos * H * D + 2 * 2 * batch * n_heads * D


def attention_setup(kvq, dev, pool, wbits, n_heads=ATTN_QUERY_HEADS):
    """Quantize the whole pool (untimed) and return (launch, algorithmic bytes)."""
    P, ps, H, D = pool.k.shape
    batch = pool.cache_seqlens.numel()
    cs, ss = kvq.q_shapes(tuple(pool.k.shape), wbits)
    kc, vc = (torch.zeros(cs, dtype=torch.uint8, device=dev) for _ in range(2))
    ks, vs = (torch.zeros(ss, dtype=torch.float16, device=dev) for _ in range(2))
    full = pool.block_table.shape[1] * ps
    kvq.fp16_to_q_kv(pool.k, kc, ks, pool.v, vc, vs, batch, -full, full, ps, pool.cache_seqlens, pool.block_table,
                     wbits)
    g = torch.Generator(device="cpu").manual_seed(workloads.SEED_BASE + 77)
    q = torch.randn(batch, n_heads, D, generator=g).half().to(dev)
    out = torch.empty_like(q)
    ws = torch.empty(max(16, kvq.attention_workspace_bytes(tuple(pool.k.shape), batch, n_heads, ps,
                                                           pool.block_table.shape[1])), dtype=torch.uint8, device=dev)
    scale = 1.0 / math.sqrt(D)

    def fn():
        kvq.decode_attention_q(q, kc, ks, vc, vs, out, batch, pool.cache_seqlens, wbits, scale, ps, pool.block_table,
                               ws)
    fn()
    return fn, attention_bytes(pool.cache_seqlens.cpu().tolist(), H, D, wbits, n_heads)


def model_layers(kvq, dev, peak, steps, flush, layers=32):
    """32 layers x K/V of 8 x 32768 x 8 x 128 FP16 in 256-position pages (~48 GB resident):
    full-window q_to_fp16_kv over all layers, then fp16_to_q_kv over all layers."""
    L = []
    for i in range(layers):
        pool = workloads.model_layer(i, device=dev)
        cs, ss = kvq.q_shapes(tuple(pool.k.shape), 6)
        kc = torch.empty(cs, dtype=torch.uint8, device=dev)
        vc = torch.empty_like(kc)
        ks = torch.empty(ss, dtype=torch.float16, device=dev)
        vs = torch.empty_like(ks)
        kvq.fp16_to_q_kv(pool.k, kc, ks, pool.v, vc, vs, 8, -32768, 32768, 256, pool.cache_seqlens,
                         pool.block_table, 6)  # setup, untimed
        L.append((pool, kc, vc, ks, vs))
    torch.cuda.synchronize()
    n = 2 * L[0][0].k.numel() * layers
    nb = BYTES_PER_ELEM[6] * n

    def deq():
        for pool, kc, vc, ks, vs in L:
            kvq.q_to_fp16_kv(kc, pool.k, ks, vc, pool.v, vs, 8, -32768, 32768, 256, pool.cache_seqlens,
                             pool.block_table, 6)

    def qnt():
        for pool, kc, vc, ks, vs in L:
            kvq.fp16_to_q_kv(pool.k, kc, ks, pool.v, vc, vs, 8, -32768, 32768, 256, pool.cache_seqlens,
                             pool.block_table, 6)

    res = []
    cfg = "paged Q6, 32 layers x K/V 8x32768x8x128, page 256, shuffled block_table"
    for name, fn in (("q_to_fp16_kv/q6/model32", deq), ("fp16_to_q_kv/q6/model32", qnt)):
        ms = time_stream(lambda i: fn(), 1, steps, 3, flush, collective=False, chunk=1)
        res.append({"op": name, "config": cfg, "bytes": int(nb), "us": round(ms * 1e3, 1),
                    "gbs": round(nb / ms / 1e6, 1), "frac": round(nb / ms / 1e6 / peak, 3), "timing": "stream"})
    del L
    torch.cuda.empty_cache()
    return res


# ------------------------------------------------------ single-op cases ----

CASES = ("headline_fp8enc_kv", "headline_fp8dec_kv", "headline_fp8enc", "headline_fp8dec", "fp8enc", "fp8dec", "q4enc",
         "q4dec", "q6enc", "q6dec", "q8enc", "q8dec", "paged_prefill_q4enc", "paged_prefill_q4dec",
         "paged_decode_q4enc", "model_layer_q6enc", "model_layer_q6dec", "attn_paged_q4", "attn_paged_q6",
         "attn_paged_q8", "attn_paged_fp8", "attn_batch1_q4")


def run_case(kvq, dev, name, batch, steps, warmup, peak, stream=False):
    """One conversion on one workload, `steps` timed launches (for quick sweeps and ncu).
    Contiguous cases use the channel-outlier recipe at [batch, 8192, 8, 128] (batch 4:
    268 MB of FP16 K+V, above the L2 size); paged cases the 2048-page pool; model cases
    one 1024-page layer."""
    flush = L2Flush(dev)
    if stream and name.startswith("headline") and name.endswith("_kv"):
        # the fused headline launch alone, rotating through the step's 8 input copies
        step = Fp8Step(kvq, dev, HEADLINE["shape"][0])
        j = 0 if "enc" in name else 1
        for i in range(len(step.sets)):
            step.run(i)  # valid E5M2 inputs for the decoder
        ms = time_stream(lambda i: step.launch(j, i), len(step.sets), steps, warmup, flush, collective=False)
        nb = step.launch_bytes
        return {"case": name, "batch": batch, "bytes": int(nb), "us": round(ms * 1e3, 2), "gbs": round(nb / ms / 1e6, 1),
                "frac": round(nb / ms / 1e6 / peak, 3), "timing": "stream, 8 rotating input copies"}
    if name.startswith("headline") and name.endswith("_kv"):
        B, S, H, D = HEADLINE["shape"]
        o, w = HEADLINE["offset"], HEADLINE["width"]
        k, v = workloads.fp8_window(shape=(B, S, H, D), device=dev)
        k8, v8 = torch.zeros(k.shape, dtype=torch.uint8, device=dev), torch.zeros(v.shape, dtype=torch.uint8, device=dev)
        ky, vy = torch.empty_like(k), torch.empty_like(v)
        kvq.fp16_to_fp8_kv(k, k8, v, v8, B, o, w)
        nb = 3.0 * 2 * B * w * H * D
        fn = (lambda: kvq.fp16_to_fp8_kv(k, k8, v, v8, B, o, w)) if "enc" in name else \
             (lambda: kvq.fp8_to_fp16_kv(k8, ky, v8, vy, B, o, w))
    elif name.startswith("headline"):
        B, S, H, D = HEADLINE["shape"]
        o, w = HEADLINE["offset"], HEADLINE["width"]
        k, _ = workloads.fp8_window(shape=(B, S, H, D), device=dev)
        k8 = torch.zeros(k.shape, dtype=torch.uint8, device=dev)
        y = torch.empty_like(k)
        kvq.fp16_to_fp8(k, k8, B, o, w)
        nb = 3.0 * B * w * H * D
        fn = (lambda: kvq.fp16_to_fp8(k, k8, B, o, w)) if name.endswith("enc") else \
             (lambda: kvq.fp8_to_fp16(k8, y, B, o, w))
    elif name.startswith("fp8") or name[:2] in ("q4", "q6", "q8"):
        k, v = workloads.channel_outliers(shape=(batch, 8192, 8, 128), device=dev)
        B, S = k.shape[:2]
        if name.startswith("fp8"):
            k8 = torch.zeros(k.shape, dtype=torch.uint8, device=dev)
            y = torch.empty_like(k)
            kvq.fp16_to_fp8(k, k8, B, 0, S)
            nb = 3.0 * k.numel()
            fn = (lambda: kvq.fp16_to_fp8(k, k8, B, 0, S)) if name == "fp8enc" else \
                 (lambda: kvq.fp8_to_fp16(k8, y, B, 0, S))
        else:
            wb = int(name[1])
            cs, ss = kvq.q_shapes(tuple(k.shape), wb)
            kc, vc = (torch.zeros(cs, dtype=torch.uint8, device=dev) for _ in range(2))
            ks, vs = (torch.zeros(ss, dtype=torch.float16, device=dev) for _ in range(2))
            ky, vy = torch.empty_like(k), torch.empty_like(v)
            kvq.fp16_to_q_kv(k, kc, ks, v, vc, vs, B, 0, S, 0, None, None, wb)
            nb = BYTES_PER_ELEM[wb] * 2 * k.numel()
            fn = (lambda: kvq.fp16_to_q_kv(k, kc, ks, v, vc, vs, B, 0, S, 0, None, None, wb)) \
                if name.endswith("enc") else (lambda: kvq.q_to_fp16_kv(kc, ky, ks, vc, vy, vs, B, 0, S, 0, None,
                                                                        None, wb))
    elif name == "attn_batch1_q4":
        fns, nb = attention_batch1_setup(kvq, dev, copies=1)
        fn = fns[0]
    elif name == "attn_paged_fp8":
        pool = workloads.paged_pool(device=dev)
        fn, nb = attention_setup_fp8(kvq, dev, pool)
    elif name.startswith("attn_paged"):
        pool = workloads.paged_pool(device=dev)
        fn, nb = attention_setup(kvq, dev, pool, int(name[-1]))
    elif name.startswith("paged"):
        pool = workloads.paged_pool(device=dev)
        P, ps, H, D = pool.k.shape
        off, w = (0, 1) if "decode" in name else (-512, 512)
        cs, ss = kvq.q_shapes(tuple(pool.k.shape), 4)
        kc, vc = (torch.zeros(cs, dtype=torch.uint8, device=dev) for _ in range(2))
        ks, vs = (torch.zeros(ss, dtype=torch.float16, device=dev) for _ in range(2))
        lens = pool.cache_seqlens.cpu()
        npos = sum(max(0, int(L) + off + w) - max(0, int(L) + off) for L in lens)
        nb = BYTES_PER_ELEM[4] * 2 * npos * H * D
        args = (32, off, w, ps, pool.cache_seqlens, pool.block_table, 4)
        kvq.fp16_to_q_kv(pool.k, kc, ks, pool.v, vc, vs, *args)
        fn = (lambda: kvq.fp16_to_q_kv(pool.k, kc, ks, pool.v, vc, vs, *args)) if name.endswith("enc") else \
             (lambda: kvq.q_to_fp16_kv(kc, pool.k, ks, vc, pool.v, vs, *args))
    else:
        pool = workloads.model_layer(0, device=dev)
        cs, ss = kvq.q_shapes(tuple(pool.k.shape), 6)
        kc, vc = (torch.zeros(cs, dtype=torch.uint8, device=dev) for _ in range(2))
        ks, vs = (torch.zeros(ss, dtype=torch.float16, device=dev) for _ in range(2))
        args = (8, -32768, 32768, 256, pool.cache_seqlens, pool.block_table, 6)
        kvq.fp16_to_q_kv(pool.k, kc, ks, pool.v, vc, vs, *args)
        nb = BYTES_PER_ELEM[6] * 2 * pool.k.numel()
        fn = (lambda: kvq.fp16_to_q_kv(pool.k, kc, ks, pool.v, vc, vs, *args)) if name.endswith("enc") else \
             (lambda: kvq.q_to_fp16_kv(kc, pool.k, ks, vc, pool.v, vs, *args))
    if stream:
        if nb < L2_BYTES:
            raise SystemExit(f"--stream needs inputs larger than L2; case {name} moves {nb / 1e6:.0f} MB")
        ms = time_stream(lambda i: fn(), 1, steps, warmup, flush, collective=False)
        return {"case": name, "batch": batch, "bytes": int(nb), "us": round(ms * 1e3, 2),
                "gbs": round(nb / ms / 1e6, 1), "frac": round(nb / ms / 1e6 / peak, 3), "timing": "stream"}
    per, _ = time_device(lambda ev: fn(), steps, warmup, flush, collective=False)
    ms = statistics.mean(per)
    return {"case": name, "batch": batch, "bytes": int(nb), "us": round(ms * 1e3, 2),
            "us_min": round(min(per) * 1e3, 2), "gbs": round(nb / ms / 1e6, 1),
            "frac": round(nb / ms / 1e6 / peak, 3), "timing": "isolated launches, L2 flushed before each"}


# -------------------------------------------------------------- CPU oracle ----

def oracle_step_sample(batch=4, max_seconds=12.0, min_reps=1):
    """Time the CPU oracle on the headline step (all four conversions of the full window),
    repeating until about max_seconds.  Returns (GB/s, seconds per step, reps, description)."""
    import numpy as np

    import oracle

    B, S, H, D = HEADLINE["shape"]
    k, v = workloads.fp8_window(shape=(batch, S, H, D))
    kn = k.view(torch.int16).numpy().view(np.uint16)
    vn = v.view(torch.int16).numpy().view(np.uint16)
    k8 = np.zeros(kn.shape, np.uint8)
    v8 = np.zeros(vn.shape, np.uint8)
    ky = np.zeros(kn.shape, np.uint16)
    vy = np.zeros(vn.shape, np.uint16)
    o, w = HEADLINE["offset"], HEADLINE["width"]
    reps, t0 = 0, time.perf_counter()
    while True:
        oracle.fp16_to_fp8_kv(kn, k8, vn, v8, batch, o, w)
        oracle.fp8_to_fp16_kv(k8, ky, v8, vy, batch, o, w)
        reps += 1
        if reps >= min_reps and time.perf_counter() - t0 >= max_seconds:
            break
    dt = (time.perf_counter() - t0) / reps
    nbytes = 4 * BYTES_PER_ELEM["fp8"] * batch * w * H * D
    desc = f"{reps} full step(s): FP8 encode+decode of K and V, batch {batch}, window {o}..{o + w}"
    return nbytes / dt / 1e9, dt, reps, desc


# ------------------------------------------------------------------- main ----

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-per-op", action="store_true", help="skip the per-op table")
    ap.add_argument("--no-model", action="store_true", help="skip the 32-layer model-sized rows")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--case", choices=CASES, action="append",
                    help="time only these single conversions (for sweeps and ncu); no headline line")
    ap.add_argument("--case-batch", type=int, default=4)
    ap.add_argument("--stream", action="store_true",
                    help="with --case: time the launches back to back (one event pair) instead of one at a "
                         "time with L2 flushed; the headline cases rotate through 8 input copies")
    ap.add_argument("--engine", choices=["auto", "ldg", "bulk"], default="auto",
                    help="load engine of the conversion kernels (plain loads or TMA bulk copies)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank != 0:
            return 0
        return run_reference(args)

    import datetime

    import torch.distributed as dist

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
    import kv_cache_quantization_fp16_b200 as kvq

    peak, peak_kind = hbm_peak()
    kvq.set_engine(args.engine)
    if args.case:
        for c in args.case:
            print(json.dumps(run_case(kvq, dev, c, args.case_batch, args.steps, args.warmup, peak, args.stream)),
                  flush=True)
        return 0
    flush = L2Flush(dev)
    sampler = ClockSampler(local_rank).start() if rank == 0 else None

    # weak scaling: a global batch of 4 sequences per rank; rank r converts its shard of
    # it (4 sequences), its inputs seeded by the shard's first global sequence index
    global_batch = HEADLINE["shape"][0] * world
    lo, hi = shard_range(global_batch, rank, world)
    batch = hi - lo
    step = Fp8Step(kvq, dev, batch, seed_shift=lo)
    # timed region: `steps` consecutive steps over rotating input copies (inputs larger
    # than L2), one pair of CUDA events around all of them, max over ranks
    ms_local = time_stream(step.run, len(step.sets), args.steps, args.warmup, flush, sampler)
    ms = max_over_ranks(ms_local, dev)
    # per-launch durations inside the step: the step time split in the proportions of an
    # event-marked pass; the dominant launch is then timed on its own, as a stream of
    # `steps` launches of it over the same rotating input copies
    share, seg_ms = stream_shares(step, len(step.sets))
    names = step.names
    launch_ms = [ms_local * f for f in share]
    dom_i = 0 if launch_ms[0] >= launch_ms[1] else 1
    dom_ms = time_stream(lambda i: step.launch(dom_i, i), len(step.sets), args.steps, args.warmup, flush,
                         collective=False)
    dom = (names[dom_i], dom_ms)
    achieved = step.launch_bytes / dom[1] / 1e6
    # one step on its own (L2 flushed before it, CUDA events around it): the latency of a
    # single isolated call, launch and event overhead included
    iso, iso_segs = time_device(lambda ev: step.run(0, ev[0] if ev else None), 200, 5, flush, None, n_marks=1,
                                collective=False)
    iso_ms = statistics.mean(iso)
    iso_seg_ms = [statistics.mean(x[i] for x in iso_segs) for i in range(2)]

    e2e_ms, h2d, d2h = e2e_fp8(kvq, step, max(10, args.steps // 10), 3, dev)
    e2e_ms = max_over_ranks(e2e_ms, dev)

    per_op = []
    if world == 1 and not args.no_per_op:
        per_op = per_op_measurements(kvq, dev, peak, min(200, max(20, args.steps // 5)), flush, step,
                                     include_model=not args.no_model)
    if sampler:
        sampler.stop()

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return 0

    cpu = None
    if not args.no_cpu_baseline:
        gbs, dt, reps, desc = oracle_step_sample()
        cpu = {"value": round(gbs, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
               "sample": desc, "seconds_per_step": round(dt, 3)}

    total_bytes = world * step.bytes_per_step
    value = total_bytes / ms / 1e6
    line = {
        "metric": "KV-cache convert GB/s (read+write), FP8 E5M2 encode+decode of K and V",
        "value": round(value, 1),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f16->u8->f16",
        "data": "synthetic (seeded N(0,1) with 1% outliers and 0.1% subnormals, drawn on device)",
        "config": {"workload": HEADLINE["workload"], "shape": list(HEADLINE["shape"]),
                   "global_batch": global_batch, "offset": HEADLINE["offset"], "width": HEADLINE["width"],
                   "ops": ["fp16_to_fp8 of K and V (one fused launch)", "fp8_to_fp16 of K and V (one fused launch)"],
                   "launch": f"{args.steps} consecutive steps (2 fused K+V launches each) replayed from CUDA graphs, "
                             "one pair of CUDA events around them",
                   "l2": f"inputs larger than L2: step i converts input copy i % {len(step.sets)} "
                         f"({len(step.sets)} x {step.set_bytes / 1e6:.0f} MB), L2 flushed once before the timed steps",
                   "parallelism": f"replicas x{world}, each rank its own 4 sequences"},
        "roofline": {"bound": "hbm", "kernel": dom[0], "achieved": round(achieved, 1), "peak": peak,
                     "unit": "GB/s", "frac": round(achieved / peak, 3), "peak_kind": peak_kind,
                     "bytes_per_launch": int(step.launch_bytes), "us_per_launch": round(dom[1] * 1e3, 2),
                     "duration": f"CUDA events around {args.steps} back-to-back launches of this kernel alone, "
                                 "rotating through the same input copies as the step",
                     "us_per_launch_in_step": round(launch_ms[dom_i] * 1e3, 2),
                     "in_step": "timed step time x this launch's share of an event-marked pass of the same stream",
                     "traffic": recorded_traffic(dom[0])},
        "per_kernel_us": {n: round(t * 1e3, 2) for n, t in zip(names, launch_ms)},
        "per_kernel_us_marked": {n: round(t * 1e3, 2) for n, t in zip(names, seg_ms)},
        "isolated": {"us_per_step": round(iso_ms * 1e3, 2),
                     "per_kernel_us": {n: round(t * 1e3, 2) for n, t in zip(names, iso_seg_ms)},
                     "gbs": round(step.bytes_per_step / iso_ms / 1e6, 1),
                     "how": "one step at a time: L2 flushed, CUDA events around the step's graph and "
                            "between its launches (includes ~6 us of event and launch overhead)"},
        "cpu_baseline": cpu,
        "e2e": {"value": round(world * step.bytes_per_step / e2e_ms / 1e6, 2), "unit": "GB/s",
                "ms_per_step": round(e2e_ms, 4), "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": step.launches_per_step * args.steps,  # in the timed region
        "clocks": sampler.summary() if sampler else None,
        "per_op": per_op,
    }
    print(json.dumps(line), flush=True)
    return 0


REF_SECONDS = 60.0  # the reference arm's timed steps take about this long in all


def run_reference(args):
    """The CPU oracle as the reference arm: each step is a bounded sample of the headline
    step, FP8 encode + decode of K and V over the first n positions of one sequence's
    window, single-threaded, on this host; n (a multiple of 16, at most the window) is
    chosen from a calibration step so that the `steps` timed steps take about
    REF_SECONDS."""
    import numpy as np

    import oracle

    B, S, H, D = HEADLINE["shape"]
    o, w = HEADLINE["offset"], HEADLINE["width"]
    k, v = workloads.fp8_window(shape=(1, S, H, D))
    kn = k.view(torch.int16).numpy().view(np.uint16)
    vn = v.view(torch.int16).numpy().view(np.uint16)
    k8, v8 = np.zeros(kn.shape, np.uint8), np.zeros(vn.shape, np.uint8)
    ky, vy = np.zeros(kn.shape, np.uint16), np.zeros(vn.shape, np.uint16)

    def once_n(n):
        oracle.fp16_to_fp8_kv(kn, k8, vn, v8, 1, o, n)
        oracle.fp8_to_fp16_kv(k8, ky, v8, vy, 1, o, n)

    t0 = time.perf_counter()
    once_n(16)
    per_pos = (time.perf_counter() - t0) / 16
    n = int(REF_SECONDS / max(1, args.steps) / per_pos) // 16 * 16
    n = max(16, min(w, n))

    def once():
        oracle.fp16_to_fp8_kv(kn, k8, vn, v8, 1, o, n)
        oracle.fp8_to_fp16_kv(k8, ky, v8, vy, 1, o, n)

    for _ in range(args.warmup):
        once()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        once()
    dt = (time.perf_counter() - t0) / args.steps
    nbytes = 4 * BYTES_PER_ELEM["fp8"] * n * H * D
    value = nbytes / dt / 1e9
    sample = f"per step: positions {o}..{o + n} of one of the 4 sequences (of the window {o}..{o + w}), K and V, encode + decode"
    line = {
        "impl": "reference",
        "metric": "KV-cache convert GB/s (read+write), FP8 E5M2 encode+decode of K and V",
        "value": round(value, 4), "unit": "GB/s", "n_gpus": args.gpus, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(dt * 1e3, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f16->u8->f16",
        "data": "synthetic (seeded, same recipe as the GPU arm)",
        # the GPU arm's workload (its global batch at this N); each step times the sample above
        "config": {"workload": HEADLINE["workload"], "shape": list(HEADLINE["shape"]),
                   "global_batch": HEADLINE["shape"][0] * max(1, args.gpus), "offset": o, "width": w},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
