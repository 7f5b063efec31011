"""Benchmark of the KV-cache format conversions on B200.

Headline workload (one JSON line on rank 0): the paged Q6 KV cache of a 32-layer
model -- per layer, K and V pools of 1024 pages x 256 positions x 8 kv heads x 128
(8 sequences x 32768 positions, shuffled block table; K N(0,1) times a per-channel
lognormal scale, V N(0,1)), about 48 GB resident.  One step is the full-window
q_to_fp16_kv of every layer, then fp16_to_q_kv of every layer, one fused K+V launch
per layer and direction (64 launches).  The metric is algorithmic GB/s (bytes read
+ bytes written: 2 + 0.75 + 2/32 bytes per element per conversion).

Timing.  `--repeats` regions of exactly `--steps` consecutive steps, each between
one pair of CUDA events with a barrier over the ranks and a device synchronize on
both sides, the step replayed from a CUDA graph; the value is the median region
(min and max beside it), the max over ranks of each.  The inputs (48 GB) are far
larger than L2, so no flush is needed between steps.

Extra keys:
  roofline      the dominant direction's layer launch: algorithmic bytes per launch
                / its CUDA-event duration (that direction's 32 launches alone,
                `--steps` times between one pair of events), against the measured
                HBM copy peak in MEASURED_PEAKS.json; `traffic` from the committed
                ncu record (profiles/traffic.txt) while the kernels are unchanged;
  cpu_baseline  the CPU oracle timed on this host on bounded samples of layer 0 of
                the same step, on every core (single-threaded functions over
                disjoint position ranges) and on one core, with the all-layer step
                time those rates imply;
  e2e           the same step through the public Python API from pinned host
                memory: per layer, Q6 codes and scales host->device, both
                conversions, codes and scales device->host, all inside the events;
                three streams, layers pipelined;
  per_op        every other conversion on its own workload (the FP8 partial-window
                step, contiguous Q4/Q6/Q8 and FP8, paged Q4 and FP8 decode /
                prefill, decode attention), each as GB/s and fraction of the HBM
                peak (on by default; --no-per-op skips it).

Multi-GPU (torchrun, one rank per GPU): every rank converts its own model's cache
(weak scaling, no collective on the data path); each region's time is the max over
ranks.  ``--impl reference`` times the CPU oracle instead (rank 0 only).
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

FP8_WINDOW = dict(workload="fp8_window_contiguous", shape=(4, 4096, 8, 128), offset=1024, width=2048)
# the headline workload: one model's paged Q6 KV cache, every layer dequantized then quantized
MODEL32 = dict(workload="paged_q6_model32", layers=32, seqs=8, seq_len=32768, kv_heads=8, head_dim=128,
               page_size=256, wbits=6)
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
        B, S, H, D = FP8_WINDOW["shape"]
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
        self.off, self.w = FP8_WINDOW["offset"], FP8_WINDOW["width"]
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


class ModelStep:
    """Headline step on one rank: the paged Q6 KV cache of a 32-layer model (per layer K and V
    pools of 1024 pages x 256 positions x 8 kv heads x 128, 8 sequences x 32768 positions,
    a shuffled block table), full-window q_to_fp16_kv of every layer, then fp16_to_q_kv of
    every layer: one fused K+V launch per layer and direction, 64 launches per step.  About
    48 GB stay resident on the device, far above the L2 size, so no step finds its inputs in
    L2.  Rank r of a multi-GPU run holds layers seeded 32 r .. 32 r + 31 (its own model
    replica's cache)."""

    def __init__(self, kvq, dev, layer0=0):
        m = MODEL32
        self.kvq, self.wb, self.n = kvq, m["wbits"], m["seq_len"]
        self.layers = []
        for i in range(m["layers"]):
            pool = workloads.model_layer(layer0 + i, seqs=m["seqs"], seq_len=m["seq_len"], page_size=m["page_size"],
                                         heads=m["kv_heads"], head_dim=m["head_dim"], device=dev)
            cs, ss = kvq.q_shapes(tuple(pool.k.shape), self.wb)
            t = dict(pool=pool, kc=torch.empty(cs, dtype=torch.uint8, device=dev),
                     vc=torch.empty(cs, dtype=torch.uint8, device=dev),
                     ks=torch.empty(ss, dtype=torch.float16, device=dev),
                     vs=torch.empty(ss, dtype=torch.float16, device=dev))
            self.quantize(t)  # set-up, untimed: the Q6 cache the step starts from
            self.layers.append(t)
        torch.cuda.synchronize()
        pool = self.layers[0]["pool"]
        self.elems_per_launch = 2 * pool.k.numel()  # K and V
        self.launch_bytes = BYTES_PER_ELEM[self.wb] * self.elems_per_launch
        self.launches_per_step = 2 * len(self.layers)
        self.bytes_per_step = self.launches_per_step * self.launch_bytes
        self.names = ["q_to_fp16_kv/q6/model_layer", "fp16_to_q_kv/q6/model_layer"]

    def _args(self, t):
        p = t["pool"]
        return (MODEL32["seqs"], -self.n, self.n, MODEL32["page_size"], p.cache_seqlens, p.block_table, self.wb)

    def dequantize(self, t):
        p = t["pool"]
        self.kvq.q_to_fp16_kv(t["kc"], p.k, t["ks"], t["vc"], p.v, t["vs"], *self._args(t))

    def quantize(self, t):
        p = t["pool"]
        self.kvq.fp16_to_q_kv(p.k, t["kc"], t["ks"], p.v, t["vc"], t["vs"], *self._args(t))

    def half(self, j):
        """Launches of direction j (0: dequantize every layer, 1: quantize every layer)."""
        for t in self.layers:
            (self.dequantize if j == 0 else self.quantize)(t)

    def run(self, ev=None):
        self.half(0)
        if ev is not None:
            ev.record()
        self.half(1)


def time_repeats(fn, steps, warmup, repeats, sampler=None, collective=True):
    """`repeats` timed regions, each of exactly `steps` consecutive steps between one pair of
    CUDA events (a barrier over the ranks and a device synchronize on both sides, the max
    over ranks taken); fn is captured once as a CUDA graph of one step and replayed.
    Returns the mean ms per step of every region."""
    cur = torch.cuda.current_stream()
    side = torch.cuda.Stream()
    side.wait_stream(cur)
    with torch.cuda.stream(side):
        fn()  # first-call set-up precedes capture
    cur.wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    _upload_graph(g)
    for _ in range(warmup):
        g.replay()
    torch.cuda.synchronize()
    out = []
    if sampler:
        sampler.mark()
    for _ in range(repeats):
        if collective:
            _barrier()
        torch.cuda.synchronize()
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record()
        for _ in range(steps):
            g.replay()
        e.record()
        torch.cuda.synchronize()
        ms = s.elapsed_time(e) / steps
        out.append(max_over_ranks(ms, torch.device("cuda", torch.cuda.current_device())) if collective else ms)
    if collective:
        _barrier()
    if sampler:
        sampler.mark()
    del g
    return out


def model_shares(step, reps=3):
    """ms of each direction inside a step: one event recorded between the two halves of a
    captured step, read over `reps` replays (one event between two 7 ms halves costs
    nothing measurable)."""
    marks = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(3)]
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        marks[0].record()
        step.run(marks[1])
        marks[2].record()
    seg = [0.0, 0.0]
    for _ in range(reps):
        g.replay()
        torch.cuda.synchronize()
        seg[0] += marks[0].elapsed_time(marks[1])
        seg[1] += marks[1].elapsed_time(marks[2])
    del g
    return [x / reps for x in seg]


def e2e_model(kvq, step: ModelStep, steps, warmup):
    """The headline step end to end through the public Python API from pinned host memory:
    per layer, the host -> device copy of its Q6 codes and scales (K and V), the
    dequantize and quantize launches, and the device -> host copy of the re-quantized
    codes and scales.  Layers are pipelined as a serving loop would: uploads on one
    stream, conversions on a second, downloads on a third, so layer i+1's upload and
    layer i-1's download overlap layer i's conversions (PCIe is full duplex).  Two pinned
    host buffer sets alternate (layer i reads set i % 2).  Returns (ms per step, host ->
    device bytes per step, device -> host bytes per step)."""
    names = ("kc", "ks", "vc", "vs")
    host_in = [{n: step.layers[r][n].cpu().pin_memory() for n in names} for r in range(2)]
    host_out = [{n: torch.empty_like(h[n]).pin_memory() for n in names} for h in host_in]
    s_in, s_cv, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    L = len(step.layers)
    ev_in = [torch.cuda.Event() for _ in range(L)]
    ev_cv = [torch.cuda.Event() for _ in range(L)]
    ev_out = [torch.cuda.Event() for _ in range(L)]
    for e in ev_out:
        e.record()

    def once():
        for i, t in enumerate(step.layers):
            hi, ho = host_in[i % 2], host_out[i % 2]
            with torch.cuda.stream(s_in):
                s_in.wait_event(ev_out[i])  # the previous download of this layer's codes is done
                for n in names:
                    t[n].copy_(hi[n], non_blocking=True)
                ev_in[i].record(s_in)
            with torch.cuda.stream(s_cv):
                s_cv.wait_event(ev_in[i])
                step.dequantize(t)
                step.quantize(t)
                ev_cv[i].record(s_cv)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_cv[i])
                for n in names:
                    ho[n].copy_(t[n], non_blocking=True)
                ev_out[i].record(s_out)

    for _ in range(warmup):
        once()
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(s_in)
    for _ in range(steps):
        once()
    s_out.wait_stream(s_in)
    s_out.wait_stream(s_cv)
    end.record(s_out)
    torch.cuda.synchronize()
    ms = start.elapsed_time(end) / steps
    per_layer = sum(host_in[0][n].numel() * host_in[0][n].element_size() for n in names)
    return ms, L * per_layer, L * per_layer


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


def per_op_measurements(kvq, dev, peak, steps, flush):
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

    # the FP8 partial-window step (K and V [4, 4096, 8, 128], window 1024..3072): encode then
    # decode through the fused K+V calls, 2 launches, rotating through 8 input copies
    step = Fp8Step(kvq, dev, FP8_WINDOW["shape"][0])
    record("fp8_window_step", "contiguous K+V [4,4096,8,128], window 1024..3072, fp16_to_fp8_kv then "
           "fp8_to_fp16_kv (2 fused launches)", step.bytes_per_step, step.run, sets=len(step.sets))
    record("fp8_window_step/fp16_to_fp8_kv", "the same window, the encode launch alone", step.launch_bytes,
           lambda i: step.launch(0, i), sets=len(step.sets))
    # the same step through the page's single-tensor calls (4 launches instead of 2)
    B, S, H, D = FP8_WINDOW["shape"]
    o, w = FP8_WINDOW["offset"], FP8_WINDOW["width"]

    def per_tensor_step(i):
        t = step.sets[i % len(step.sets)]
        kvq.fp16_to_fp8(t["k"], t["k8"], B, o, w)
        kvq.fp16_to_fp8(t["v"], t["v8"], B, o, w)
        kvq.fp8_to_fp16(t["k8"], t["ky"], B, o, w)
        kvq.fp8_to_fp16(t["v8"], t["vy"], B, o, w)
    record("fp8_step_single_tensor_calls", "FP8 window, fp16_to_fp8(K), (V), fp8_to_fp16(K), (V): 4 launches",
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
    del pool, step
    torch.cuda.empty_cache()
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


# ------------------------------------------------------ single-op cases ----

CASES = ("fp8_window_enc_kv", "fp8_window_dec_kv", "fp8_window_enc", "fp8_window_dec", "fp8enc", "fp8dec", "q4enc",
         "q4dec", "q6enc", "q6dec", "q8enc", "q8dec", "paged_prefill_q4enc", "paged_prefill_q4dec",
         "paged_decode_q4enc", "model_layer_q6enc", "model_layer_q6dec", "attn_paged_q4", "attn_paged_q6",
         "attn_paged_q8", "attn_paged_fp8", "attn_batch1_q4")


def run_case(kvq, dev, name, batch, steps, warmup, peak, stream=False):
    """One conversion on one workload, `steps` timed launches (for quick sweeps and ncu).
    Contiguous cases use the channel-outlier recipe at [batch, 8192, 8, 128] (batch 4:
    268 MB of FP16 K+V, above the L2 size); paged cases the 2048-page pool; model cases
    one 1024-page layer."""
    flush = L2Flush(dev)
    if stream and name.startswith("fp8_window") and name.endswith("_kv"):
        # the fused FP8 window launch alone, rotating through the step's 8 input copies
        step = Fp8Step(kvq, dev, FP8_WINDOW["shape"][0])
        j = 0 if "enc" in name else 1
        for i in range(len(step.sets)):
            step.run(i)  # valid E5M2 inputs for the decoder
        ms = time_stream(lambda i: step.launch(j, i), len(step.sets), steps, warmup, flush, collective=False)
        nb = step.launch_bytes
        return {"case": name, "batch": batch, "bytes": int(nb), "us": round(ms * 1e3, 2), "gbs": round(nb / ms / 1e6, 1),
                "frac": round(nb / ms / 1e6 / peak, 3), "timing": "stream, 8 rotating input copies"}
    if name.startswith("fp8_window") and name.endswith("_kv"):
        B, S, H, D = FP8_WINDOW["shape"]
        o, w = FP8_WINDOW["offset"], FP8_WINDOW["width"]
        k, v = workloads.fp8_window(shape=(B, S, H, D), device=dev)
        k8, v8 = torch.zeros(k.shape, dtype=torch.uint8, device=dev), torch.zeros(v.shape, dtype=torch.uint8, device=dev)
        ky, vy = torch.empty_like(k), torch.empty_like(v)
        kvq.fp16_to_fp8_kv(k, k8, v, v8, B, o, w)
        nb = 3.0 * 2 * B * w * H * D
        fn = (lambda: kvq.fp16_to_fp8_kv(k, k8, v, v8, B, o, w)) if "enc" in name else \
             (lambda: kvq.fp8_to_fp16_kv(k8, ky, v8, vy, B, o, w))
    elif name.startswith("fp8_window"):
        B, S, H, D = FP8_WINDOW["shape"]
        o, w = FP8_WINDOW["offset"], FP8_WINDOW["width"]
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
        if stream:
            # the per-op table's stream: input copy r is the pool read through a block table whose
            # pages are shifted by 256 r, so the windows of consecutive launches differ
            sets = STREAM_SETS
            bts = [torch.where(pool.block_table >= 0, (pool.block_table + (P // sets) * r) % P, pool.block_table)
                   for r in range(sets)]
            enc = name.endswith("enc")

            def launch(i):
                a = (32, off, w, ps, pool.cache_seqlens, bts[i % sets], 4)
                if enc:
                    kvq.fp16_to_q_kv(pool.k, kc, ks, pool.v, vc, vs, *a)
                else:
                    kvq.q_to_fp16_kv(kc, pool.k, ks, vc, pool.v, vs, *a)
            ms = time_stream(launch, sets, steps, warmup, flush, collective=False)
            return {"case": name, "batch": 32, "bytes": int(nb), "us": round(ms * 1e3, 2),
                    "gbs": round(nb / ms / 1e6, 1), "frac": round(nb / ms / 1e6 / peak, 3),
                    "timing": f"stream, {sets} rotating block tables", "engine": kvq.get_engine()}
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

def host_layer(layer_pool, kc, ks, vc, vs):
    """Host copies of one model layer's Q6 cache (codes, scales, paging tables) and FP16
    output pools for the oracle."""
    import numpy as np

    def u16(t):
        return t.cpu().contiguous().view(torch.int16).numpy().view(np.uint16)

    h = dict(kc=kc.cpu().numpy(), vc=vc.cpu().numpy(), ks=u16(ks), vs=u16(vs),
             lens=layer_pool.cache_seqlens.cpu().numpy().astype(np.int32),
             bt=layer_pool.block_table.cpu().numpy().astype(np.int32), ps=layer_pool.page_size)
    shape = tuple(layer_pool.k.shape)
    h["ky"], h["vy"] = np.zeros(shape, np.uint16), np.zeros(shape, np.uint16)
    return h


def oracle_model_tasks(h, tasks, threads, wbits=6):
    """The oracle's q_to_fp16_kv then fp16_to_q_kv (as written: single-threaded functions)
    over the position ranges `tasks` = [(sequence, first, end)] of a host layer, `threads`
    ranges at a time on disjoint positions (a harness split; ctypes releases the GIL).
    Returns (seconds, positions)."""
    from concurrent.futures import ThreadPoolExecutor

    import oracle

    def one(task):
        i, a, b = task
        L = int(h["lens"][i])
        sl, bt = h["lens"][i:i + 1], h["bt"][i:i + 1]
        assert oracle.q_to_fp16_kv(h["kc"], h["ky"], h["ks"], h["vc"], h["vy"], h["vs"], 1, a - L, b - a, h["ps"],
                                   sl, bt, wbits) == oracle.OK
        assert oracle.fp16_to_q_kv(h["ky"], h["kc"], h["ks"], h["vy"], h["vc"], h["vs"], 1, a - L, b - a, h["ps"],
                                   sl, bt, wbits) == oracle.OK

    t0 = time.perf_counter()
    if threads == 1:
        for task in tasks:
            one(task)
    else:
        with ThreadPoolExecutor(threads) as ex:
            list(ex.map(one, tasks))
    return time.perf_counter() - t0, sum(b - a for _, a, b in tasks)


def position_tasks(lens, npos, chunk):
    """Ranges of at most `chunk` positions covering the first `npos` positions of the
    layer, sequence by sequence."""
    tasks, left = [], npos
    for i, L in enumerate(lens):
        for a in range(0, int(L), chunk):
            if left <= 0:
                return tasks
            b = min(int(L), a + chunk, a + left)
            tasks.append((i, a, b))
            left -= b - a
    return tasks


def range_positions(npos, cores):
    """Positions per task of the all-core oracle runs: about four tasks per core, from 64 to
    512 positions, a multiple of 64."""
    return max(64, min(512, npos // (4 * cores) // 64 * 64))


def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def oracle_model_baseline(h, seconds=10.0):
    """The CPU oracle on bounded samples of layer 0 of the headline step (dequantize then
    quantize, K and V), on 1 core and on every core; GB/s in the headline's algorithmic
    bytes, and the all-layer step time these rates imply (extrapolated)."""
    bpp = 2 * 2 * MODEL32["kv_heads"] * MODEL32["head_dim"] * BYTES_PER_ELEM[MODEL32["wbits"]]  # bytes/position
    total = int(sum(int(L) for L in h["lens"]))
    dt, n = oracle_model_tasks(h, position_tasks(h["lens"], 64, 64), 1)  # calibration
    per_pos = dt / n
    n1 = max(64, min(total, int(seconds / per_pos) // 64 * 64))
    t1, p1 = oracle_model_tasks(h, position_tasks(h["lens"], n1, 256), 1)
    cores = host_cores()
    nall = max(64, min(total, int(seconds * cores / per_pos) // 64 * 64))
    tall, pall = oracle_model_tasks(h, position_tasks(h["lens"], nall, range_positions(nall, cores)), cores)
    step_bytes = 2 * MODEL32["layers"] * 2 * MODEL32["seqs"] * MODEL32["seq_len"] * MODEL32["kv_heads"] * \
        MODEL32["head_dim"] * BYTES_PER_ELEM[MODEL32["wbits"]]
    g1, gall = bpp * p1 / t1 / 1e9, bpp * pall / tall / 1e9
    return {"value": round(gall, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
            "sample": f"layer 0 of the headline workload, its first {pall} (of {total}) sequence positions "
                      f"in ranges of {range_positions(nall, cores)} over {cores} threads: q_to_fp16_kv then "
                      f"fp16_to_q_kv of K and V (Q6), the oracle's single-threaded functions as written",
            "seconds": round(tall, 2),
            "single_core": {"value": round(g1, 4), "unit": "GB/s", "cores": 1, "seconds": round(t1, 2),
                            "sample": f"layer 0, its first {p1} positions, one thread"},
            "step_seconds_extrapolated": {"all_cores": round(step_bytes / (gall * 1e9), 1),
                                          "single_core": round(step_bytes / (g1 * 1e9), 1),
                                          "how": "the whole 32-layer step at the sampled rates (extrapolated)"}}


# ------------------------------------------------------------------- main ----

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--repeats", type=int, default=25,
                    help="timed regions of --steps steps each; the value is their median")
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-per-op", action="store_true", help="skip the per-op table")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--case", choices=CASES, action="append",
                    help="time only these single conversions (for sweeps and ncu); no headline line")
    ap.add_argument("--case-batch", type=int, default=4)
    ap.add_argument("--stream", action="store_true",
                    help="with --case: time the launches back to back (one event pair) instead of one at a "
                         "time with L2 flushed; the FP8 window cases rotate through 8 input copies")
    ap.add_argument("--attention-path", choices=["auto", "mma", "tcgen05"], default="auto",
                    help="decode-attention kernel (warp-level mma.sync tiles or tcgen05 with tensor-memory "
                         "accumulators)")
    ap.add_argument("--engine", choices=["auto", "ldg", "bulk", "ldg_tiled"], default="auto",
                    help="load engine of the conversion kernels (plain loads, TMA bulk copies, or plain loads "
                         "with per-sequence paged tiles)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.steps < 1 or args.repeats < 1:
        ap.error("--steps and --repeats must be >= 1")

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
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    import kv_cache_quantization_fp16_b200 as kvq

    peak, peak_kind = hbm_peak()
    kvq.set_engine(args.engine)
    kvq.set_attention_path(args.attention_path)
    if args.case:
        for c in args.case:
            r = run_case(kvq, dev, c, args.case_batch, args.steps, args.warmup, peak, args.stream)
            r.setdefault("engine", kvq.get_engine())
            if c.startswith("attn"):
                r["attention_path"] = kvq.get_attention_path()
            print(json.dumps(r), flush=True)
        return 0
    sampler = ClockSampler(local_rank).start() if rank == 0 else None

    # weak scaling: every rank converts its own model replica's 32-layer cache (~48 GB)
    step = ModelStep(kvq, dev, layer0=MODEL32["layers"] * rank)
    # timed regions: `repeats` x (exactly `steps` consecutive steps between one pair of CUDA
    # events, barrier + synchronize on both sides, max over ranks); the value is the median
    reps = time_repeats(step.run, args.steps, args.warmup, args.repeats, sampler)
    ms = statistics.median(reps)
    # the two directions inside a step (one event between the halves), then the dominant one
    # timed alone: `steps` x its 32 layer launches between one pair of events, 3 regions
    seg_ms = model_shares(step)
    dom_i = 0 if seg_ms[0] >= seg_ms[1] else 1
    dom_reps = time_repeats(lambda: step.half(dom_i), args.steps, 3, 3, collective=False)
    dom_launch_ms = statistics.median(dom_reps) / len(step.layers)
    achieved = step.launch_bytes / dom_launch_ms / 1e6
    # end to end: Q6 codes and scales up from pinned host memory, both conversions, codes and
    # scales back down, every layer of every step
    e2e_steps = max(2, min(args.steps, 5))
    e2e_ms, h2d, d2h = e2e_model(kvq, step, e2e_steps, 1)
    e2e_ms = max_over_ranks(e2e_ms, dev)

    host = None
    if rank == 0 and not args.no_cpu_baseline:
        t = step.layers[0]
        host = host_layer(t["pool"], t["kc"], t["ks"], t["vc"], t["vs"])
    del step
    torch.cuda.empty_cache()

    per_op = []
    if world == 1 and not args.no_per_op:
        per_op = per_op_measurements(kvq, dev, peak, min(200, max(20, 10 * args.steps)), L2Flush(dev))
    if sampler:
        sampler.stop()

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return 0

    cpu = oracle_model_baseline(host) if host is not None else None
    bytes_per_step = 2 * MODEL32["layers"] * BYTES_PER_ELEM[MODEL32["wbits"]] * 2 * MODEL32["seqs"] * \
        MODEL32["seq_len"] * MODEL32["kv_heads"] * MODEL32["head_dim"]
    value = world * bytes_per_step / ms / 1e6
    launches = 2 * MODEL32["layers"]
    names = ["q_to_fp16_kv/q6/model_layer", "fp16_to_q_kv/q6/model_layer"]
    line = {
        "metric": "KV-cache convert GB/s (read+write), paged Q6 dequantize + quantize of every layer",
        "value": round(value, 1),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f16<->u6 codes + f16 scales",
        "data": "synthetic (seeded: K N(0,1) x per-channel lognormal scale, V N(0,1), shuffled block tables; "
                "drawn on the device)",
        "config": {"workload": MODEL32["workload"], "layers": MODEL32["layers"], "seqs": MODEL32["seqs"],
                   "seq_len": MODEL32["seq_len"], "kv_heads": MODEL32["kv_heads"], "head_dim": MODEL32["head_dim"],
                   "page_size": MODEL32["page_size"], "wbits": MODEL32["wbits"],
                   "ops": ["q_to_fp16_kv of every layer (one fused K+V launch each)",
                           "fp16_to_q_kv of every layer (one fused K+V launch each)"],
                   "bytes_per_step": int(bytes_per_step),
                   "launch": f"{args.steps} consecutive steps ({launches} launches each) replayed from a CUDA graph "
                             f"of one step between one pair of CUDA events; {args.repeats} such regions, value = "
                             "the median region",
                   "repeats_ms_per_step": {"median": round(ms, 4), "min": round(min(reps), 4),
                                           "max": round(max(reps), 4), "n": len(reps)},
                   "l2": "inputs larger than L2: ~48 GB resident per rank, no flush needed",
                   "parallelism": f"replicas x{world}, each rank its own model's 32-layer cache"},
        "roofline": {"bound": "hbm", "kernel": names[dom_i], "achieved": round(achieved, 1), "peak": peak,
                     "unit": "GB/s", "frac": round(achieved / peak, 3), "peak_kind": peak_kind,
                     "bytes_per_launch": int(step_launch_bytes()), "us_per_launch": round(dom_launch_ms * 1e3, 2),
                     "duration": f"CUDA events around {args.steps} x its {MODEL32['layers']} layer launches, "
                                 "the direction alone, median of 3 regions",
                     "us_per_launch_in_step": round(seg_ms[dom_i] / MODEL32["layers"] * 1e3, 2),
                     "in_step": "its half of a step, one event between the halves, / layers",
                     "traffic": recorded_traffic(names[dom_i])},
        "per_direction_ms_in_step": {n: round(t, 4) for n, t in zip(names, seg_ms)},
        "cpu_baseline": cpu,
        "e2e": {"value": round(world * bytes_per_step / e2e_ms / 1e6, 2), "unit": "GB/s",
                "ms_per_step": round(e2e_ms, 3), "steps": e2e_steps, "h2d_bytes_per_step": int(h2d),
                "d2h_bytes_per_step": int(d2h),
                "how": "per layer: Q6 codes + scales host->device, dequantize + quantize, codes + scales "
                       "device->host; three streams, layers pipelined"},
        "gpu_launches": launches * args.steps * args.repeats,  # in the timed regions
        "clocks": sampler.summary() if sampler else None,
        "per_op": per_op,
    }
    print(json.dumps(line), flush=True)
    return 0


def step_launch_bytes():
    """Algorithmic bytes of one layer launch of the headline step (K and V, Q6)."""
    return BYTES_PER_ELEM[MODEL32["wbits"]] * 2 * MODEL32["seqs"] * MODEL32["seq_len"] * MODEL32["kv_heads"] * \
        MODEL32["head_dim"]


REF_SECONDS = 60.0  # the reference arm's timed steps take about this long in all


def run_reference(args):
    """The CPU oracle as the reference arm, on the headline workload's metric: each step
    dequantizes then re-quantizes (Q6, K and V) a bounded sample of one layer -- the first
    n positions of a layer drawn by the headline recipe (one sequence, shuffled 256-position
    pages) -- with the oracle's single-threaded functions run over disjoint position
    ranges on every host core.  n (at most 16384) is chosen from a calibration step so that the
    `warmup` + `steps` steps take about REF_SECONDS."""
    import numpy as np

    import oracle

    n_max = 16384
    pool = workloads.model_layer(0, seqs=1, seq_len=n_max, page_size=MODEL32["page_size"],
                                 heads=MODEL32["kv_heads"], head_dim=MODEL32["head_dim"])
    kb = pool.k.view(torch.int16).numpy().view(np.uint16)
    vb = pool.v.view(torch.int16).numpy().view(np.uint16)
    P, ps, H, D = kb.shape
    wb = MODEL32["wbits"]
    kc = np.zeros((P, ps, H, D * wb // 8), np.uint8)
    vc = np.zeros_like(kc)
    ks = np.zeros((P, ps, H, D // 32), np.uint16)
    vs = np.zeros_like(ks)
    lens = pool.cache_seqlens.numpy().astype(np.int32)
    bt = pool.block_table.numpy().astype(np.int32)
    cores = host_cores()
    h = dict(kc=kc, vc=vc, ks=ks, vs=vs, lens=lens, bt=bt, ps=ps, ky=kb.copy(), vy=vb.copy())
    # the Q6 cache the steps start from (set-up, untimed): quantize with the oracle
    from concurrent.futures import ThreadPoolExecutor

    def setup(task):
        i, a, b = task
        assert oracle.fp16_to_q_kv(kb, kc, ks, vb, vc, vs, 1, a - n_max, b - a, ps, lens, bt, wb) == oracle.OK
    with ThreadPoolExecutor(cores) as ex:
        list(ex.map(setup, position_tasks(lens, n_max, 512)))
    dt, n = oracle_model_tasks(h, position_tasks(lens, 512, 512), 1)  # calibration, one core
    per_pos_all = dt / n / cores
    total_steps = args.steps + args.warmup
    npos = int(REF_SECONDS / total_steps / per_pos_all) // 512 * 512
    npos = max(512, min(n_max, npos))
    tasks = position_tasks(lens, npos, range_positions(npos, cores))
    for _ in range(args.warmup):
        oracle_model_tasks(h, tasks, cores)
    t = sum(oracle_model_tasks(h, tasks, cores)[0] for _ in range(args.steps))
    dt = t / args.steps
    nbytes = 2 * 2 * npos * H * D * BYTES_PER_ELEM[wb]
    value = nbytes / dt / 1e9
    sample = (f"per step: positions 0..{npos} of one sequence of a layer drawn by the headline recipe, Q6 "
              f"q_to_fp16_kv then fp16_to_q_kv of K and V, {range_positions(npos, cores)}-position ranges over "
              f"{cores} threads")
    line = {
        "impl": "reference",
        "metric": "KV-cache convert GB/s (read+write), paged Q6 dequantize + quantize of every layer",
        "value": round(value, 4), "unit": "GB/s", "n_gpus": args.gpus, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(dt * 1e3, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f16<->u6 codes + f16 scales",
        "data": "synthetic (seeded, the GPU arm's recipe)",
        # the GPU arm's workload (its replicas at this N); each step times the sample above
        "config": {"workload": MODEL32["workload"], "layers": MODEL32["layers"], "seqs": MODEL32["seqs"],
                   "seq_len": MODEL32["seq_len"], "kv_heads": H, "head_dim": D, "page_size": ps, "wbits": wb,
                   "replicas": max(1, args.gpus)},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
