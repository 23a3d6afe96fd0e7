#!/usr/bin/env python
"""Throughput of the NVFP4 routed-expert MoE block on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = one pass of the whole chain over one batch: nvfp4_moe_forward
with no global scale given (the batch's activation global scale, route,
quantise+permute, L1 gate_up GEMM with fused SiLU*up re-quantisation and L2
down GEMM in one persistent launch, combine).
Headline workload: the 384-expert prefill MoE (T=4096, top-6, H=7168,
I=3072, Zipf-skewed routing with empty experts) -> tokens/s, TFLOP/s and the
fraction of the FP4 peak; the 48-expert decode MoE (T=64) is measured in the
same run -> GB/s and the fraction of HBM bandwidth.  Inputs are seeded
synthetic data of those shapes (nvfp4_moe_expert_topk_b200.workloads).

With torchrun (N > 1) every rank runs its own replica of the workload (data
parallel over token batches, weights replicated, no collective on the data
path); timing is the max over ranks; value = all ranks' tokens / that time.

--impl reference times the CPU oracle (oracle/, plain C) on this host's
cores on a bounded sample of the same workload (rank 0 only); nothing of the
library runs on that path.
"""
import argparse
import contextlib
import hashlib
import re
import json
import os
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from nvfp4_moe_expert_topk_b200 import (nvfp4_global_scale, nvfp4_moe_calibrate, nvfp4_moe_forward,  # noqa: E402
                                        nvfp4_moe_forward_timed, nvfp4_moe_get_error, nvfp4_moe_plan)
from nvfp4_moe_expert_topk_b200 import prep  # noqa: E402
from nvfp4_moe_expert_topk_b200 import workloads as W  # noqa: E402

FP4_NOMINAL_TFLOPS = 9000.0            # dense FP4, NVIDIA public B200 figure
BF16_TO_FP4_NOMINAL_RATIO = 4.0        # 9 / 2.25 PFLOP/s dense
STAGES = ["global_scale", "route", "quantize_permute", "l1_gate_up_swiglu_quant", "l2_down", "combine"]
FRONT_STAGE = "front"                  # global scale of the batch + routing + quantise/permute
FUSED_STAGE = "l1_l2_fused"            # L1 and L2 as one launch (nvfp4_moe_plan)
PAIRS_STAGE = "l1_l2_fused_pairs"      # pair mode 1: the heavy experts' fused pair-tile launch
LIGHT_STAGE = "l1_l2_fused_light"      # pair mode 1: the fused 1-CTA launch over the other m-tiles
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
GEMM_SOURCES = ["gemm.cu", "ptx.cuh", "quant.cuh", "internal.h"]


# ---------------------------------------------------------------- helpers
def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(PEAKS_FALLBACK), "fallback"


def gemm_source_sha():
    """Hash of the GEMM kernels' code: gemm.cu, ptx.cuh, quant.cuh and, of
    internal.h, the GemmArgs struct the kernels take; comments and layout
    whitespace removed (a comment edit, or a declaration of another kernel in
    internal.h, does not invalidate the captured traffic)."""
    h = hashlib.sha256()
    for name in GEMM_SOURCES:
        with open(os.path.join(ROOT, "nvfp4_moe_expert_topk_b200", "csrc", name)) as f:
            text = f.read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        text = re.sub(r"//[^\n]*", "", text)
        if name == "internal.h":
            m = re.search(r"struct GemmArgs \{.*?\n\};", text, flags=re.S)
            text = m.group(0) if m else text
        h.update(" ".join(text.split()).encode())
    return h.hexdigest()[:16]


def ncu_traffic(kernel, workload):
    """DRAM bytes per launch from the committed ncu summary, if it was taken
    on the current GEMM sources (else None)."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.txt")
    if not os.path.exists(path):
        return None
    rows = {}
    with open(path) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                key, _, val = line.partition(":")
                rows[key.strip()] = val.strip()
    if rows.get("source_sha") != gemm_source_sha():
        return None
    v = rows.get(f"{workload}.{kernel}.dram_bytes_per_launch")
    return float(v) if v else None


class Clocks:
    """SM clock, power draw and clock-event reasons, sampled from NVML every
    5 ms by a background thread for the whole run (read-only queries: nothing
    is set).  Each timed region records its host interval (the device work
    inside it is bracketed by synchronisations), so every time reported
    carries the median SM clock it ran at.  Falls back to one nvidia-smi
    process sampling every 200 ms when NVML is unavailable."""
    REASONS = {"hw_slowdown": 0x8, "hw_thermal_slowdown": 0x40, "sw_thermal_slowdown": 0x20,
               "sw_power_cap": 0x4}
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device, period=0.005):
        self.device = device
        self.period = period
        self.samples = []               # (monotonic s, sm MHz, max MHz, power W, reason bits)
        self.regions = {}
        self.source = None
        self._stop = None
        self._thread = None
        self._proc = None

    def _uuid(self):
        try:
            return "GPU-" + str(torch.cuda.get_device_properties(self.device).uuid)
        except Exception:
            return None

    def start(self):
        import threading
        try:
            import pynvml as N
            N.nvmlInit()
            uid = self._uuid()
            h = N.nvmlDeviceGetHandleByUUID(uid) if uid else N.nvmlDeviceGetHandleByIndex(self.device.index or 0)
            mx = float(N.nvmlDeviceGetMaxClockInfo(h, N.NVML_CLOCK_SM))
        except Exception:
            return self._start_smi()
        self.source = "nvml"
        self._stop = threading.Event()

        def loop():
            while not self._stop.is_set():
                try:
                    self.samples.append((time.monotonic(), float(N.nvmlDeviceGetClockInfo(h, N.NVML_CLOCK_SM)), mx,
                                         N.nvmlDeviceGetPowerUsage(h) / 1000.0,
                                         int(N.nvmlDeviceGetCurrentClocksEventReasons(h))))
                except Exception:
                    pass
                self._stop.wait(self.period)

        self._thread = threading.Thread(target=loop, daemon=True)
        self._thread.start()

    def _start_smi(self):
        self.source = "nvidia-smi"
        self._file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        cmd = ["nvidia-smi", f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits", "-lms", "200"]
        uid = self._uuid()
        if uid:
            cmd[1:1] = ["-i", uid]
        self._t0 = time.monotonic()
        try:
            self._proc = subprocess.Popen(cmd, stdout=self._file, stderr=subprocess.DEVNULL)
        except OSError:
            self._proc = None

    def stop(self):
        if self._thread is not None:
            self._stop.set()
            self._thread.join(timeout=5)
            self._thread = None
        if self._proc is not None:
            time.sleep(0.25)
            self._proc.terminate()
            try:
                self._proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self._proc.kill()
            self._file.seek(0)
            rows = [[p.strip() for p in line.split(",")] for line in self._file.read().splitlines()]
            self._file.close()
            os.unlink(self._file.name)
            names = list(self.REASONS)
            for i, r in enumerate(r for r in rows if len(r) >= 9):
                try:
                    bits = sum(self.REASONS[names[j]] for j in range(4) if r[5 + j].lower() == "active")
                    # no per-sample timestamps: spread the samples 200 ms apart from the start
                    self.samples.append((self._t0 + 0.2 * i, float(r[1]), float(r[2]), float(r[3]), bits))
                except ValueError:
                    pass
            self._proc = None

    @contextlib.contextmanager
    def region(self, name):
        t0 = time.monotonic()
        try:
            yield
        finally:
            self.regions[name] = (t0, time.monotonic())

    def summary(self, names=None):
        """Median SM MHz, max MHz, median power and the clock-event reasons
        seen over the samples inside the named regions (all regions if None)."""
        spans = [self.regions[n] for n in (names or list(self.regions)) if n in self.regions]
        sel = [smp for smp in self.samples if any(a <= smp[0] <= b for a, b in spans)]
        if not sel:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples in the region"], "samples": 0,
                    "source": self.source}
        bits = 0
        for smp in sel:
            bits |= smp[4]
        return {"sm_mhz": float(np.median([smp[1] for smp in sel])), "sm_max_mhz": max(smp[2] for smp in sel),
                "power_w": round(float(np.median([smp[3] for smp in sel])), 1),
                "reasons": sorted(n for n, b in self.REASONS.items() if bits & b), "samples": len(sel),
                "source": self.source}

    def mhz(self, name):
        return self.summary([name])["sm_mhz"]


CLOCKS = None                           # the run's Clocks, started in run_ours / run_single


def clock_region(name):
    return CLOCKS.region(name) if CLOCKS is not None else contextlib.nullcontext()


def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(local)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(world, v):
    """Max of a per-rank scalar (a device time) over all ranks."""
    if world == 1:
        return v
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ---------------------------------------------------------------- workloads
class Workload:
    """A MoE config resident on the device: NVFP4 weights, one batch, inter_gs
    from the library's own warmup (nvfp4_moe_calibrate on the warmup batch)."""

    def __init__(self, cfg, dev):
        self.cfg = cfg
        self.dev = dev
        self.weights = prep.MoeWeights.synthetic(cfg, dev)
        x, ids, w = W.batch(cfg)
        self.x_cpu, self.ids_cpu, self.w_cpu = x, ids, w
        self.x, self.ids, self.w = x.to(dev), ids.to(dev), w.to(dev)
        self.x_gs = torch.empty(1, dtype=torch.float32, device=dev)
        self.ws = prep.workspace(cfg.T, cfg.k, cfg.E, cfg.H, cfg.I, dev)
        self.out = torch.empty(cfg.T, cfg.H, dtype=torch.bfloat16, device=dev)
        xw, idw, ww = W.batch(cfg, warmup=True)
        xw = xw.to(dev)
        gsw = torch.empty(1, dtype=torch.float32, device=dev)
        nvfp4_global_scale(xw, gsw)
        wsw = prep.workspace(cfg.warmup_T, cfg.k, cfg.E, cfg.H, cfg.I, dev)
        self.inter_gs = torch.empty(cfg.E, dtype=torch.float32, device=dev)
        nvfp4_moe_calibrate(xw, idw.to(dev), ww.to(dev), gsw, **self.weights.args(), inter_gs_out=self.inter_gs,
                            workspace=wsw)
        del wsw
        self.counts = np.bincount(ids.numpy().reshape(-1), minlength=cfg.E)
        self.rows = int(self.counts.sum())
        self.nonempty = int((self.counts > 0).sum())
        self.fused, self.pair_mode = nvfp4_moe_plan(cfg.T, cfg.k, cfg.E, cfg.H, cfg.I)
        self.launches_per_step = launches_per_step(self.fused, self.pair_mode)

    def fold(self, per_stage):
        return fold_stages(per_stage, self.fused, self.pair_mode)

    def step(self, events=None):
        # x_gs = None: the forward computes this batch's global scale itself
        if events is None:
            nvfp4_moe_forward(self.x, self.ids, self.w, None, **self.weights.args(), inter_gs=self.inter_gs,
                              out=self.out, workspace=self.ws)
        else:
            nvfp4_moe_forward_timed(self.x, self.ids, self.w, None, **self.weights.args(),
                                    inter_gs=self.inter_gs, out=self.out, workspace=self.ws, events=events)

    # algorithmic work (real rows only; weights of non-empty experts once)
    def flops(self):
        c = self.cfg
        return 2.0 * self.rows * 3 * c.H * c.I

    def kernel_bytes(self):
        """Algorithmic bytes of each stage the plan runs (stage_bytes)."""
        return stage_bytes(self.cfg, self.counts, self.fused, self.pair_mode)

    def step_bytes(self):
        """Algorithmic bytes of one step: non-empty experts' weights + x in + out + ids/weights."""
        c = self.cfg
        fp4 = 0.5 + 1.0 / 16
        return self.nonempty * 3 * c.H * c.I * fp4 + 2 * c.T * c.H * 2.0 + c.T * c.k * 8.0


FP4_BYTES = 0.5 + 1.0 / 16             # NVFP4 code + scale bytes per element


def launches_per_step(fused, pair_mode):
    """Launches of one forward: the front, the GEMMs, the combine."""
    gemm = {0: 1 if fused else 2, 1: 2, 2: 2}[pair_mode]
    return 2 + gemm


def fold_stages(per_stage, fused, pair_mode):
    """The timed forward's six stage slots (nvfp4_moe_forward_timed) keyed by
    what the plan runs there: the front (one launch: global scale, routing,
    quantise + permute) and then
      pair mode 0, fused   the fused 1-CTA L1 + L2 launch;
      pair mode 1          the heavy experts' fused pair launch, then the
                           fused 1-CTA launch over the other m-tiles (the
                           staged run records an event between them, so each
                           has its own stage; in the headline run, without
                           events, the 1-CTA CTAs take over SMs as pair CTAs
                           finish);
      otherwise            L1, then L2;
    and the combine."""
    d = dict(per_stage)
    d[FRONT_STAGE] = d.pop("global_scale") + d.pop("route") + d.pop("quantize_permute")
    if pair_mode == 1:
        d[PAIRS_STAGE] = d.pop("l1_gate_up_swiglu_quant")
        d[LIGHT_STAGE] = d.pop("l2_down")
    elif fused and pair_mode == 0:
        d[FUSED_STAGE] = d.pop("l1_gate_up_swiglu_quant") + d.pop("l2_down")
    return d


def tile_split(counts, pair_mode):
    """Per expert: (rows on pair tiles, rows on 1-CTA tiles), the rule the
    routing applies (pair mode 1: the full m-tile pairs of experts with two or
    more 128-row m-tiles; 2: everything)."""
    tiles = (counts + 127) // 128
    if pair_mode == 2:
        npair = (tiles + 1) // 2
    elif pair_mode == 1:
        npair = np.where(tiles >= 2, tiles // 2, 0)
    else:
        npair = np.zeros_like(tiles)
    pair_rows = np.minimum(counts, 256 * npair)
    return pair_rows, counts - pair_rows


def stage_bytes(cfg, counts, fused, pair_mode):
    """Algorithmic bytes per stage: each launch reads the weights of the
    experts it touches once, its activation rows once and writes its outputs
    once (real rows only; workspace traffic beyond that is implementation's)."""
    T, H, I, k, E = cfg.T, cfg.H, cfg.I, cfg.k, cfg.E
    R = int(counts.sum())

    def gemm(rows_e):
        n_exp = int((rows_e > 0).sum())
        r = int(rows_e.sum())
        l1 = n_exp * 2 * I * H * FP4_BYTES + r * H * FP4_BYTES + r * I * FP4_BYTES
        l2 = n_exp * H * I * FP4_BYTES + r * I * FP4_BYTES + r * H * 2.0
        return l1, l2

    d = {FRONT_STAGE: T * H * 2.0 + R * H * FP4_BYTES + T * k * 4.0 * 3 + E * 16.0,
         "combine": R * H * 2.0 + T * H * 2.0 + T * k * 12.0}
    pair_rows, light_rows = tile_split(counts, pair_mode)
    if pair_mode == 1:                          # each launch reads the experts it touches once
        d[PAIRS_STAGE] = sum(gemm(pair_rows))
        d[LIGHT_STAGE] = sum(gemm(light_rows))
    else:
        l1, l2 = gemm(counts)
        if fused and pair_mode == 0:
            d[FUSED_STAGE] = l1 + l2
        else:
            d["l1_gate_up_swiglu_quant"], d["l2_down"] = l1, l2
    return d


def _capture(fn):
    """A CUDA graph of everything fn() issues (captured on a side stream)."""
    stream = torch.cuda.current_stream()
    side = torch.cuda.Stream()
    side.wait_stream(stream)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(side):
        with torch.cuda.graph(g, stream=side):
            fn()
    stream.wait_stream(side)
    g.replay()                          # upload + warm
    torch.cuda.synchronize()
    return g


def time_steps(wl, steps, warmup, world, graph=True, tag="timed"):
    """Device time of `steps` steps: events on the launching stream, barrier +
    synchronize on both sides, max over ranks.  With graph=True the `steps`
    steps are captured once into a CUDA graph and the timed region is one
    replay of it -- the way a serving runtime issues the block (the pages'
    runner is cudagraph-safe); otherwise eager launches.  Per-stage mean
    durations come from a second run of the same steps with events recorded
    between the forward's stages (in the graph case a second graph, so that
    the event nodes, which also stop consecutive kernels from overlapping
    their launch, stay out of the headline time)."""
    stream = torch.cuda.current_stream()
    for _ in range(warmup):
        wl.step()
    torch.cuda.synchronize()
    ev = [[torch.cuda.Event(enable_timing=True, external=graph) for _ in range(7)] for _ in range(steps)]
    for row in ev:                      # create the CUDA events outside the timed region
        for e in row:
            e.record(stream)
    torch.cuda.synchronize()

    def issue_plain():
        for _ in range(steps):
            wl.step()

    def issue_staged():
        for i in range(steps):
            ev[i][0].record()
            wl.step(events=ev[i][1:])

    g = _capture(issue_plain) if graph else None
    g_staged = _capture(issue_staged) if graph else None
    barrier(world)
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    torch.cuda.nvtx.range_push(f"{tag}_{wl.cfg.name}")
    with clock_region(f"{tag}_{wl.cfg.name}"):
        t0.record(stream)
        if g is not None:
            g.replay()
        else:
            issue_plain()
        t1.record(stream)
        torch.cuda.synchronize()
    torch.cuda.nvtx.range_pop()
    barrier(world)
    ms = t0.elapsed_time(t1)
    if g_staged is not None:
        g_staged.replay()
    else:
        issue_staged()
    torch.cuda.synchronize()
    try:
        stage_ms = {name: float(np.mean([e[j].elapsed_time(e[j + 1]) for e in ev])) for j, name in enumerate(STAGES)}
    except Exception:                   # graph-recorded events not timeable here: time the stages eagerly
        stage_ms = None
    del g, g_staged
    if stage_ms is None:
        _, stage_ms = time_steps(wl, steps, 0, world, graph=False, tag="stages")
        return max_over_ranks(world, ms), stage_ms
    return max_over_ranks(world, ms), wl.fold(stage_ms)


def time_e2e(wl, steps, warmup, world):
    """The step through the public API from pinned host buffers, as a serving
    loop issues it: every step copies its x, ids and weights host -> device,
    runs nvfp4_moe_forward and copies its output device -> host, all inside
    the timed region.  Copies run on their own streams into two alternating
    device buffer sets, so step i+1's inputs upload and step i-1's output
    downloads while step i computes; events order each buffer's reuse."""
    dev = wl.x.device
    compute = torch.cuda.Stream(dev)
    up = torch.cuda.Stream(dev)
    down = torch.cuda.Stream(dev)
    hx = wl.x_cpu.pin_memory()
    hids = wl.ids_cpu.pin_memory()
    hw = wl.w_cpu.pin_memory()
    bufs = [dict(x=torch.empty_like(wl.x), ids=torch.empty_like(wl.ids), w=torch.empty_like(wl.w),
                 out=torch.empty_like(wl.out)) for _ in range(2)]
    houts = [torch.empty(wl.out.shape, dtype=wl.out.dtype, pin_memory=True) for _ in range(2)]
    n_all = warmup + steps
    ev = [{k: torch.cuda.Event() for k in ("in", "done", "down")} for _ in range(n_all)]

    def issue(i):
        b, e = bufs[i % 2], ev[i]
        with torch.cuda.stream(up):
            if i >= 2:
                up.wait_event(ev[i - 2]["done"])        # the forward two steps back has read this buffer set
            b["x"].copy_(hx, non_blocking=True)
            b["ids"].copy_(hids, non_blocking=True)
            b["w"].copy_(hw, non_blocking=True)
            e["in"].record(up)
        with torch.cuda.stream(compute):
            compute.wait_event(e["in"])
            if i >= 2:
                compute.wait_event(ev[i - 2]["down"])   # its output has left the device
            nvfp4_moe_forward(b["x"], b["ids"], b["w"], None, **wl.weights.args(), inter_gs=wl.inter_gs,
                              out=b["out"], workspace=wl.ws, stream=compute)
            e["done"].record(compute)
        with torch.cuda.stream(down):
            down.wait_event(e["done"])
            houts[i % 2].copy_(b["out"], non_blocking=True)
            e["down"].record(down)

    for i in range(warmup):
        issue(i)
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    with clock_region(f"e2e_{wl.cfg.name}"):
        t0.record(up)
        compute.wait_event(t0)
        down.wait_event(t0)
        for i in range(warmup, n_all):
            issue(i)
        up.wait_stream(down)
        up.wait_stream(compute)
        t1.record(up)
        torch.cuda.synchronize()
    barrier(world)
    ms = max_over_ranks(world, t0.elapsed_time(t1))
    h2d = hx.numel() * hx.element_size() + hids.numel() * 4 + hw.numel() * 4
    d2h = houts[0].numel() * houts[0].element_size()
    if not torch.isfinite(houts[(n_all - 1) % 2].float()).all():
        raise RuntimeError("non-finite output in the end-to-end run")
    if not torch.equal(houts[(n_all - 1) % 2], bufs[(n_all - 1) % 2]["out"].cpu()):
        raise RuntimeError("end-to-end output differs from the device result")
    return ms, h2d, d2h


# ---------------------------------------------------------------- MLA GEMMs
def graph_time(fns, reps, warmup, flush=None, region=None):
    """Per-call device times of a sequence of calls, issued back to back.
    `reps` repetitions of [flush(); ev0; fns[0](); ev1; fns[1](); ...] are
    captured into one CUDA graph (external event records, so the kernels run
    without host gaps between them) and replayed once after a warm replay;
    returns the mean milliseconds of each fns[j] over the repetitions.  With
    `flush` (a write of a buffer larger than L2) every repetition starts
    L2-cold; without it, repeated calls find their inputs in L2."""
    stream = torch.cuda.current_stream()
    for _ in range(warmup):
        for f in fns:
            f()
    torch.cuda.synchronize()
    ev = [[torch.cuda.Event(enable_timing=True, external=True) for _ in range(len(fns) + 1)] for _ in range(reps)]
    for row in ev:
        for e in row:
            e.record(stream)
    torch.cuda.synchronize()
    side = torch.cuda.Stream()
    side.wait_stream(stream)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(side):
        with torch.cuda.graph(g, stream=side):
            for row in ev:
                if flush is not None:
                    flush()
                row[0].record()
                for j, f in enumerate(fns):
                    f()
                    row[j + 1].record()
    stream.wait_stream(side)
    g.replay()
    torch.cuda.synchronize()
    with clock_region(region) if region else contextlib.nullcontext():
        g.replay()
        torch.cuda.synchronize()
    out = [float(np.mean([row[j].elapsed_time(row[j + 1]) for row in ev])) for j in range(len(fns))]
    del g
    return out


def graph_time_seq(fn, reps, region=None):
    """Mean milliseconds of one call of fn over `reps` calls issued back to
    back in one CUDA graph (one event pair around the replay)."""
    stream = torch.cuda.current_stream()
    for _ in range(3):
        fn()
    torch.cuda.synchronize()
    side = torch.cuda.Stream()
    side.wait_stream(stream)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(side):
        with torch.cuda.graph(g, stream=side):
            for _ in range(reps):
                fn()
    stream.wait_stream(side)
    g.replay()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with clock_region(region) if region else contextlib.nullcontext():
        a.record(stream)
        g.replay()
        b.record(stream)
        torch.cuda.synchronize()
    del g
    return a.elapsed_time(b) / reps


class L2Flush:
    """A 512 MB device buffer; calling the object overwrites it (4x the 126 MB L2)."""

    def __init__(self, dev):
        self.buf = torch.empty(512 << 20, dtype=torch.uint8, device=dev)
        self.i = 0

    def __call__(self):
        self.i = (self.i + 1) & 0xFF
        self.buf.fill_(self.i)


def time_router(cfg, dev, reps, warmup, flush):
    """The device top-k router (logits [T, E] fp32 -> top-k ids and
    renormalised sigmoid weights) on the batch's shape, one launch per call.
    Hot: logits L2-resident (the router GEMM has just written them); cold:
    after an L2 flush."""
    from nvfp4_moe_expert_topk_b200 import NVFP4_SCORING_SIGMOID, nvfp4_moe_topk
    logits = W.router_logits(cfg, dev)
    ids = torch.empty(cfg.T, cfg.k, dtype=torch.int32, device=dev)
    w = torch.empty(cfg.T, cfg.k, dtype=torch.float32, device=dev)

    def call():
        nvfp4_moe_topk(logits, cfg.k, ids, w, NVFP4_SCORING_SIGMOID)

    hot, = graph_time([call], reps, warmup, region="router_hot")
    cold, = graph_time([call], reps, 0, flush, region="router_cold")
    nbytes = cfg.T * cfg.E * 4 + cfg.T * cfg.k * 8
    return {"T": cfg.T, "E": cfg.E, "k": cfg.k, "scoring": "sigmoid", "us_per_call": round(hot * 1e3, 2),
            "us_per_call_cold": round(cold * 1e3, 2), "GB_s": round(nbytes / (hot * 1e-3) / 1e9, 1),
            "GB_s_cold": round(nbytes / (cold * 1e-3) / 1e9, 1), "bytes_per_call": nbytes, "launches": 1,
            "sm_mhz": CLOCKS.mhz("router_hot") if CLOCKS else None}


def time_variant_routing(wl, cfg, steps, warmup, world):
    """The prefill step on the same weights and tokens with another routing
    (pure Zipf: no expert forced empty), CUDA-graph timed like the headline."""
    _, ids, w = W.batch(cfg)
    saved = (wl.ids, wl.w)
    wl.ids, wl.w = ids.to(wl.dev), w.to(wl.dev)
    ms, stages = time_steps(wl, steps, warmup, world, graph=True, tag="variant")
    wl.ids, wl.w = saved
    counts = np.bincount(ids.numpy().reshape(-1), minlength=cfg.E)
    t = ms / steps / 1e3
    return {"workload": f"prefill_moe_E{cfg.E}_k{cfg.k}_T{cfg.T}_zipf{cfg.zipf_s}_pure",
            "ms_per_step": ms / steps, "tokens_per_s": world * cfg.T / t,
            "tflops": 2.0 * counts.sum() * 3 * cfg.H * cfg.I / t / 1e12,
            "empty_experts": int((counts == 0).sum()), "max_rows_per_expert": int(counts.max()),
            "m_tiles": int(np.ceil(counts / 128).sum()), "stage_ms": stages,
            "sm_mhz": CLOCKS.mhz(f"variant_{wl.cfg.name}") if CLOCKS else None}


def time_shared(dev, steps, warmup, flush, name="shared"):
    """A config whose weights fit in L2 -- the shared expert (one expert, 256
    tokens, 37 MB of weights) or the tiny MoE (0.4 MB): hot (back-to-back
    steps) and cold (L2 flushed before every step), CUDA-graph timed."""
    wl = Workload(W.MOE_CONFIGS[name], dev)
    hot, = graph_time([wl.step], steps, warmup, region=f"{name}_hot")
    cold, = graph_time([wl.step], steps, 0, flush, region=f"{name}_cold")
    if nvfp4_moe_get_error(wl.ws) != 0:
        raise RuntimeError("device error word after the shared-expert run")
    b, f = wl.step_bytes(), wl.flops()
    return {"workload": config_block(wl.cfg, 1)["workload"], "ms_hot": hot, "ms_cold": cold,
            "GB_s_hot": b / (hot * 1e-3) / 1e9, "GB_s_cold": b / (cold * 1e-3) / 1e9,
            "tflops_hot": f / (hot * 1e-3) / 1e12, "tflops_cold": f / (cold * 1e-3) / 1e12,
            "sm_mhz": CLOCKS.mhz(f"{name}_hot") if CLOCKS else None}


def time_shared_fold(dec, fold_cfg, dev, steps, warmup, hbm_gbs):
    """A routed batch plus the shared expert, two ways, CUDA-graph timed:
    folded in as one more group of the routed launches (every token's last
    slot is the shared expert with weight 1, as nvfp4_moe_topk_shared writes
    it), and run as its own one-group forward after the routed forward (two
    chains, two outputs to add)."""
    fold = Workload(fold_cfg, dev)
    c = dec.cfg
    sep = Workload(W.MoeConfig(f"shared_T{c.T}", E=1, k=1, T=c.T, H=c.H, I=c.I, routing="single",
                               outliers=c.outliers, warmup_T=min(c.T, 256)), dev)

    def separate():
        dec.step()
        sep.step()

    folded, = graph_time([fold.step], steps, warmup, region=f"{fold_cfg.name}_folded")
    both, = graph_time([separate], steps, warmup, region=f"{fold_cfg.name}_separate")
    for wl in (fold, sep):
        if nvfp4_moe_get_error(wl.ws) != 0:
            raise RuntimeError(f"device error word after the {wl.cfg.name} run")
    b = fold.step_bytes()
    return {"workload": config_block(fold.cfg, 1)["workload"], "ms_folded": folded,
            "ms_separate": both, "GB_s_folded": b / (folded * 1e-3) / 1e9,
            "hbm_frac_folded": b / (folded * 1e-3) / 1e9 / hbm_gbs,
            "algorithmic_bytes": b, "launches_folded": fold.launches_per_step,
            "launches_separate": dec.launches_per_step + sep.launches_per_step,
            "sm_mhz": CLOCKS.mhz(f"{fold_cfg.name}_folded") if CLOCKS else None}


def tma_stream_ceiling(wl):
    """The GEMM's weight-tile loads alone (nvfp4_tma_stream_ceiling): the
    prefill workload's stacked W13 codes as the matrix ([E*2I, H/2], 8.5 GB,
    the HBM read rate of the GEMM's access pattern), then its first 16384 rows
    (59 MB, L2-resident: the L2 -> shared-memory rate); 4 stages of 32 KB per
    SM as in the 1-CTA GEMM launch, 6 as a deeper ring."""
    from nvfp4_moe_expert_topk_b200 import nvfp4_tma_stream_ceiling
    c = wl.cfg
    m = wl.weights.w13_codes.view(c.E * 2 * c.I, c.H // 2)
    rows, row_bytes = m.shape
    work = rows // 256                                      # one pass over the full matrix
    err = torch.zeros(1, dtype=torch.int32, device=m.device)
    res = {"row_bytes": row_bytes, "box": "2 x 128 rows x 128 B per step, 128-byte swizzle"}
    for name, mat in (("hbm", m), ("l2", m[:16384])):
        for stages in (4, 6):
            region = f"tma_stream_{name}_{stages}"
            nvfp4_tma_stream_ceiling(mat, work, stages, err)
            torch.cuda.synchronize()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            ms = 1e9
            with clock_region(region):
                for _ in range(3):
                    a.record()
                    nvfp4_tma_stream_ceiling(mat, work, stages, err)
                    b.record()
                    torch.cuda.synchronize()
                    ms = min(ms, a.elapsed_time(b))
            res[f"{name}_{stages}_stages_gbs"] = work * 256 * row_bytes / (ms * 1e-3) / 1e9
            res[f"{name}_{stages}_stages_sm_mhz"] = CLOCKS.mhz(region) if CLOCKS else None
    if err.item() != 0:
        raise RuntimeError(f"TMA stream probe error word {err.item()}")
    return res


def fp4_ceiling(dev, sms):
    """Tensor-pipe ceiling of the FP4 MMA (nvfp4_fp4_mma_ceiling): one block
    per SM issues k-tiles of four M=128 K=64 MMAs for ~20 ms (long enough to
    reach the power-capped clock); TFLOP/s from CUDA events, cycles per MMA
    from the blocks' own clocks."""
    from nvfp4_moe_expert_topk_b200 import nvfp4_fp4_mma_ceiling
    res = {}
    for bn, iters in ((256, 50000), (128, 50000)):
        cycles = torch.zeros(sms, dtype=torch.int64, device=dev)
        err = torch.zeros(1, dtype=torch.int32, device=dev)
        nvfp4_fp4_mma_ceiling(bn, 2000, cycles, err)
        torch.cuda.synchronize()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        with clock_region(f"fp4_ceiling_n{bn}"):
            a.record()
            nvfp4_fp4_mma_ceiling(bn, iters, cycles, err)
            b.record()
            torch.cuda.synchronize()
        if err.item() != 0 or (cycles < 0).any():
            raise RuntimeError("FP4 ceiling probe: a bounded wait gave up")
        ms = a.elapsed_time(b)
        flops = sms * iters * 4 * 2.0 * 128 * bn * 64
        cyc = cycles.double()
        res[f"n{bn}"] = {"tflops": flops / (ms * 1e-3) / 1e12, "ms": ms,
                         "cycles_per_mma": float(cyc.mean()) / (iters * 4),
                         "cycles_per_mma_max": float(cyc.max()) / (iters * 4),
                         "implied_sm_mhz": float(cyc.mean()) / (ms * 1e3),
                         "sm_mhz": CLOCKS.mhz(f"fp4_ceiling_n{bn}") if CLOCKS else None}
    return res


def time_mla_gemms(dev, steps, warmup, peaks, flush, ceiling_tflops=None):
    """The MLA projections as separate dense NVFP4 GEMMs at M=2048 (weights
    quantised once; per step: activation global scale + quantisation + GEMM).
    Device times from CUDA events around CUDA-graph replays.  gemm_ms: the
    mean of `steps` GEMM calls issued back to back (hot: operands as the
    quantiser left them, weights L2-resident where they fit; each call's
    prologue overlaps the previous call's tail, as it overlaps the quantiser's
    in a step); gemm_ms_isolated: one call between two event records, so
    with no overlap; gemm_ms_cold: the same after a 512 MB L2 flush."""
    from nvfp4_moe_expert_topk_b200 import NVFP4_SCALES_MMA, nvfp4_gemm, nvfp4_quantize, nvfp4_scales_bytes
    res = {}
    fp4_peak = peaks["bf16_tflops_sustained"] * BF16_TO_FP4_NOMINAL_RATIO
    ridge = fp4_peak * 1e12 / (peaks["hbm_gbs"] * 1e9)
    stream = torch.cuda.current_stream()
    for idx, (name, cfg) in enumerate(W.MLA_GEMMS.items()):
        a, w = W.gemm_operands(cfg, idx, dev)
        M, N, K = cfg.M, cfg.N, cfg.K
        segs = list(cfg.seg_end)
        w_codes = torch.empty(N, K // 2, dtype=torch.uint8, device=dev)
        w_sc = torch.empty(nvfp4_scales_bytes(N, K, NVFP4_SCALES_MMA), dtype=torch.uint8, device=dev)
        w_gs = torch.empty(len(segs), dtype=torch.float32, device=dev)
        start = 0
        for i, end in enumerate(segs):
            nvfp4_global_scale(w[start:end], w_gs[i:i + 1])
            nvfp4_quantize(w[start:end], w_gs[i:i + 1], w_codes[start:end], w_sc[start * (K // 16):end * (K // 16)],
                           NVFP4_SCALES_MMA)
            start = end
        del w
        ad = a.to(dev)
        a_gs = torch.empty(1, dtype=torch.float32, device=dev)
        a_codes = torch.empty(M, K // 2, dtype=torch.uint8, device=dev)
        a_sc = torch.empty(nvfp4_scales_bytes(M, K, NVFP4_SCALES_MMA), dtype=torch.uint8, device=dev)
        out = torch.empty(M, N, dtype=torch.bfloat16, device=dev)

        def quant():
            nvfp4_global_scale(ad, a_gs)
            nvfp4_quantize(ad, a_gs, a_codes, a_sc, NVFP4_SCALES_MMA)

        def gemm():
            nvfp4_gemm(a_codes, a_sc, a_gs, w_codes, w_sc, w_gs, segs, out)

        quant_ms, gemm_iso_ms = graph_time([quant, gemm], steps, warmup, region=f"mla_{name}_isolated")
        gemm_ms = graph_time_seq(gemm, steps, region=f"mla_{name}")
        _, gemm_cold_ms = graph_time([quant, gemm], steps, 0, flush, region=f"mla_{name}_cold")
        step_ms = quant_ms + gemm_ms
        flops = 2.0 * M * N * K
        gbytes = (M * K + N * K) * (0.5 + 1 / 16) + M * N * 2.0
        ai = flops / gbytes
        tflops = flops / (gemm_ms * 1e-3) / 1e12
        gbs = gbytes / (gemm_ms * 1e-3) / 1e9
        bound = "tensor" if ai >= ridge else "hbm"
        res[name] = {"M": M, "N": N, "K": K, "ms_per_step": step_ms, "gemm_ms": gemm_ms,
                     "tflops": tflops, "gemm_ms_isolated": gemm_iso_ms,
                     "gemm_ms_cold": gemm_cold_ms, "tflops_cold": flops / (gemm_cold_ms * 1e-3) / 1e12,
                     "gbs": gbs, "arith_intensity": ai, "bound": bound,
                     "frac": (tflops / fp4_peak) if bound == "tensor" else (gbs / peaks["hbm_gbs"]),
                     "fp4_nominal_frac": tflops / FP4_NOMINAL_TFLOPS,
                     "sm_mhz": CLOCKS.mhz(f"mla_{name}") if CLOCKS else None}
        if ceiling_tflops:
            res[name]["fp4_ceiling_frac"] = tflops / ceiling_tflops
        del ad, a_codes, a_sc, out, w_codes, w_sc
        torch.cuda.empty_cache()
    return res


# ---------------------------------------------------------------- CPU oracle
def oracle_sample(cfg, tokens, dev, inter_gs_dev):
    """Oracle inputs for a token sample of a workload: the sampled tokens'
    experts regenerated from their seeds and quantised by the oracle."""
    import oracle as O
    x, ids, w = W.batch(cfg)
    xb = W.bf16_bits(x)
    x_gs = O.global_scale_bf16(xb)
    sub_ids = ids.numpy()[tokens]
    experts = sorted(set(sub_ids.reshape(-1).tolist()))
    lut = {e: i for i, e in enumerate(experts)}
    H, I, n = cfg.H, cfg.I, len(experts)
    w13c = np.empty((n, 2 * I, H // 2), np.uint8)
    w13s = np.empty((n, 2 * I, H // 16), np.uint8)
    w13g = np.empty((n, 2), np.float32)
    w2c = np.empty((n, H, I // 2), np.uint8)
    w2s = np.empty((n, H, I // 16), np.uint8)
    w2g = np.empty(n, np.float32)
    for i, e in enumerate(experts):
        b13 = W.bf16_bits(W.expert_w13(cfg, e, dev))
        for h in range(2):
            part = b13[h * I:(h + 1) * I]
            w13g[i, h] = O.global_scale_bf16(part)
            w13c[i, h * I:(h + 1) * I], w13s[i, h * I:(h + 1) * I] = O.quantize_bf16(part, w13g[i, h])
        b2 = W.bf16_bits(W.expert_w2(cfg, e, dev))
        w2g[i] = O.global_scale_bf16(b2)
        w2c[i], w2s[i] = O.quantize_bf16(b2, w2g[i])
    inter = None if inter_gs_dev is None else inter_gs_dev.cpu().numpy()[experts]
    remap = np.vectorize(lambda e: lut[e])(sub_ids).astype(np.int32)
    return dict(x_bits=xb[tokens], topk_ids=remap, topk_weights=w.numpy()[tokens], x_gs=x_gs,
                w13_codes=w13c, w13_scales=w13s, w13_gs=w13g, w2_codes=w2c, w2_scales=w2s, w2_gs=w2g,
                inter_gs=inter)


def run_oracle_tokens(sample, token_idx, slot=None):
    """Oracle seconds for the sampled tokens (or, with slot, for that one
    routed slot of one token: the other slots skipped)."""
    import oracle as O
    sel = np.atleast_1d(token_idx)
    kw = dict(sample)
    kw["x_bits"] = sample["x_bits"][sel]
    kw["topk_ids"] = sample["topk_ids"][sel]
    kw["topk_weights"] = sample["topk_weights"][sel]
    if slot is not None:
        ids = np.full_like(kw["topk_ids"], -1)
        ids[:, slot] = kw["topk_ids"][:, slot]
        kw["topk_ids"] = ids
    t0 = time.perf_counter()
    O.moe_forward(**kw)
    return time.perf_counter() - t0


def cpu_baseline(cfg, dev, inter_gs_dev, n_tokens=8, min_secs=10.0, max_passes=8):
    """The oracle on this host's cores over a fixed sample of the batch's
    tokens, passes repeated until at least min_secs of CPU work."""
    import oracle as O
    tokens = np.sort(np.random.default_rng(123).choice(cfg.T, n_tokens, replace=False))
    sample = oracle_sample(cfg, tokens, dev, inter_gs_dev)
    secs, passes = 0.0, 0
    while passes < max_passes and (passes == 0 or secs < min_secs):
        secs += run_oracle_tokens(sample, np.arange(n_tokens))
        passes += 1
    return {"value": passes * n_tokens / secs, "unit": "tokens/s", "cores": O.num_threads(), "kind": "oracle",
            "sample": f"{n_tokens} tokens of the {cfg.name} batch (their {sample['w13_codes'].shape[0]} experts), "
                      f"{passes} passes, {secs:.1f} s of CPU work; weight generation and quantisation excluded"}


# ---------------------------------------------------------------- arms
def config_block(cfg, world):
    return {"workload": f"{cfg.name}_moe_E{cfg.E}_k{cfg.k}_T{cfg.T}_H{cfg.H}_I{cfg.I}"
                        + ("_zipf1.1_16empty" if cfg.routing == "zipf" else ""),
            "experts": cfg.E, "top_k": cfg.k, "tokens_per_gpu": cfg.T, "hidden": cfg.H, "intermediate": cfg.I,
            "global_batch": cfg.T * world, "routing": cfg.routing, "outlier_channels": cfg.outliers,
            "weights": "NVFP4 (E2M1 + E4M3 per 16 + fp32 per tensor) from seeded N(0,0.02) bf16",
            "l2": "no flush: every step streams >= 1.7 GB of weights (> 126 MB L2)",
            "parallelism": "replicas" if world == 1 else f"dp{world} replicas (no data-path collective)"}


def compact(obj, digits=4):
    """Floats rounded to `digits` significant digits, recursively (keeps the
    one-line record short)."""
    if isinstance(obj, float):
        return float(f"{obj:.{digits}g}")
    if isinstance(obj, dict):
        return {k: compact(v, digits) for k, v in obj.items()}
    if isinstance(obj, (list, tuple)):
        return [compact(v, digits) for v in obj]
    return obj


def timed(ms, region):
    """A device time with the median SM clock of its region and their
    product (time x clock: comparable across runs at different clocks)."""
    mhz = CLOCKS.mhz(region) if CLOCKS else None
    return {"ms": ms, "sm_mhz": mhz, "ms_x_ghz": ms * mhz / 1e3 if mhz else None}


def run_ours(args):
    global CLOCKS
    world, rank, local = dist_setup()
    dev = torch.device("cuda", local)
    peaks, peak_src = load_peaks()
    steps, warmup = args.steps, max(3, args.warmup)
    CLOCKS = Clocks(dev)
    CLOCKS.start()
    try:
        if args.only != "all":
            return run_single(args.only, world, rank, dev, peaks, peak_src, steps, warmup)
        return _run_all(args, world, rank, dev, peaks, peak_src, steps, warmup)
    finally:
        CLOCKS.stop()
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


def _run_all(args, world, rank, dev, peaks, peak_src, steps, warmup):
    pre = Workload(W.MOE_CONFIGS["prefill"], dev)
    dec = Workload(W.MOE_CONFIGS["decode"], dev)
    torch.cuda.synchronize()

    mode = "eager" if args.eager else "timed"
    # decode first: timed right after the prefill it would run in the prefill's
    # power-cap tail (a decode step alone draws ~300 W and keeps the full clock)
    ms_dec, stages_dec = time_steps(dec, steps, warmup, world, graph=not args.eager)
    ms_dec_eager, _ = time_steps(dec, steps, warmup, world, graph=False, tag="eager")
    ms_pre, stages_pre = time_steps(pre, steps, warmup, world, graph=not args.eager)
    ms_pre_eager, _ = time_steps(pre, steps, warmup, world, graph=False, tag="eager")
    for wl in (pre, dec):
        err = nvfp4_moe_get_error(wl.ws)
        if err != 0:
            raise RuntimeError(f"device error word {err} after the {wl.cfg.name} run")
        if not torch.isfinite(wl.out.float()).all():
            raise RuntimeError(f"non-finite output in the {wl.cfg.name} run")
    e2e_ms, h2d, d2h = time_e2e(pre, steps, warmup, world)
    flush = L2Flush(dev)
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    ceiling = fp4_ceiling(dev, sms)
    stream_ceiling = tma_stream_ceiling(pre)
    mla = time_mla_gemms(dev, min(steps, 50), warmup, peaks, flush, ceiling["n256"]["tflops"])
    router = time_router(pre.cfg, dev, 50, warmup, flush)
    pure = time_variant_routing(pre, W.MOE_CONFIGS["prefill_zipf_pure"], min(steps, 50), warmup, world)
    shared = time_shared(dev, min(steps, 50), warmup, flush)
    tiny = time_shared(dev, min(steps, 50), warmup, flush, name="tiny")
    shared_fold = time_shared_fold(dec, W.MOE_CONFIGS["decode_shared"], dev, min(steps, 50), warmup, peaks["hbm_gbs"])

    t_step = ms_pre / steps / 1e3
    tokens_s = world * pre.cfg.T / t_step
    tflops = pre.flops() / t_step / 1e12
    fp4_measured = peaks["bf16_tflops_sustained"] * BF16_TO_FP4_NOMINAL_RATIO
    kb = pre.kernel_bytes()
    dominant = max(stages_pre, key=lambda s: stages_pre[s])
    dom_ms = stages_pre[dominant]
    achieved = kb[dominant] / (dom_ms / 1e3) / 1e9
    hbm = peaks["hbm_gbs"]
    traffic = ncu_traffic(dominant, "prefill")

    t_dec = ms_dec / steps / 1e3
    dec_gbs = dec.step_bytes() / t_dec / 1e9
    dec_kb = dec.kernel_bytes()
    dec_dom = max(stages_dec, key=lambda s: stages_dec[s])
    dec_ach = dec_kb[dec_dom] / (stages_dec[dec_dom] / 1e3) / 1e9
    r_pre, r_dec = f"{mode}_{pre.cfg.name}", f"{mode}_{dec.cfg.name}"

    line = {
        "metric": "moe_prefill_tokens_per_s",
        "value": tokens_s,
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": steps,
        "warmup": warmup,
        "ms_per_step": ms_pre / steps,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "nvfp4",
        "data": "synthetic",
        "config": config_block(pre.cfg, world),
        "tflops": tflops,
        "fp4_peak_frac": {"of_nominal_9000": tflops / FP4_NOMINAL_TFLOPS,
                          f"of_{peak_src}_bf16_sustained_x4": tflops / fp4_measured,
                          "of_measured_fp4_mma_ceiling": tflops / ceiling["n256"]["tflops"]},
        "hbm_gbs_step": pre.step_bytes() / t_step / 1e9,
        "hbm_frac_step": pre.step_bytes() / t_step / 1e9 / hbm,
        "stage_ms": stages_pre,
        "launch": "eager" if args.eager else "cuda_graph",
        "roofline": {"bound": "hbm", "kernel": dominant, "achieved": achieved, "peak": hbm, "unit": "GB/s",
                     "frac": achieved / hbm, "peak_source": f"{peak_src} hbm_gbs",
                     "algorithmic_bytes": kb[dominant], "traffic": traffic},
        "e2e": {"value": world * pre.cfg.T * steps / (e2e_ms / 1e3), "unit": "tokens/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms / steps},
        # this library's kernels launched in the headline's timed region (the
        # decode block counts its own)
        "gpu_launches": pre.launches_per_step * steps,
        "clocks": CLOCKS.summary([r_pre]),
        # every timed region with the median SM clock it ran at (time x clock compares runs)
        "timings": {"prefill": timed(ms_pre / steps, r_pre), "prefill_eager": timed(ms_pre_eager / steps,
                                                                                   f"eager_{pre.cfg.name}"),
                    "e2e_prefill": timed(e2e_ms / steps, f"e2e_{pre.cfg.name}"),
                    "decode": timed(ms_dec / steps, r_dec),
                    "decode_eager": timed(ms_dec_eager / steps, f"eager_{dec.cfg.name}")},
        "fp4_mma_ceiling": ceiling,
        "tma_stream_ceiling": stream_ceiling,
        "mla_gemms": mla,
        "router": router,
        "prefill_pure_zipf": pure,
        "shared_expert": shared,
        "tiny_moe": tiny,
        "decode_with_shared_expert": shared_fold,
    }
    if world == 1 and rank == 0 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(pre.cfg, dev, pre.inter_gs)
    # last, so that a record keeping only the end of the line still holds it
    line["decode"] = {
        "workload": config_block(dec.cfg, world)["workload"],
        "metric": "moe_decode_GB_per_s", "value": dec_gbs, "unit": "GB/s", "ms_per_step": ms_dec / steps,
        "hbm_frac": dec_gbs / hbm, "tokens_per_s": world * dec.cfg.T / t_dec,
        "eager_ms_per_step": ms_dec_eager / steps, "algorithmic_bytes_per_step": dec.step_bytes(),
        "stage_ms": stages_dec, "clocks": CLOCKS.summary([r_dec]), "gpu_launches": dec.launches_per_step * steps,
        "roofline": {"bound": "hbm", "kernel": dec_dom, "achieved": dec_ach, "peak": hbm, "unit": "GB/s",
                     "frac": dec_ach / hbm, "traffic": ncu_traffic(dec_dom, "decode")},
    }
    if rank == 0:
        print(json.dumps(compact(line)), flush=True)


def run_single(name, world, rank, dev, peaks, peak_src, steps, warmup):
    """One MoE workload alone (small cases for profiling: decode, prefill_ep48);
    for decode_shared / prefill_shared, the shared expert folded in against
    run as a second chain; mla: the three dense MLA projection GEMMs alone
    (per GEMM: `warmup` eager calls, then 2 x `steps` hot and 2 x `steps`
    L2-cold calls from CUDA graphs)."""
    if name == "mla":
        res = time_mla_gemms(dev, steps, warmup, peaks, L2Flush(dev))
        flops = sum(2.0 * v["M"] * v["N"] * v["K"] for v in res.values())
        ms = sum(v["gemm_ms"] for v in res.values())
        line = {"metric": "mla_gemm_TFLOP_per_s", "value": flops / (ms * 1e-3) / 1e12, "unit": "TFLOP/s",
                "n_gpus": world, "steps": steps, "warmup": warmup, "ms_per_step": ms, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "nvfp4", "data": "synthetic",
                "config": {"workload": "mla_projection_gemms_M2048", "l2": "hot; cold figures after a 512 MB flush"},
                "mla_gemms": res, "clocks": CLOCKS.summary([f"mla_{k}" for k in res])}
        if rank == 0:
            print(json.dumps(line), flush=True)
        return
    if name.endswith("_shared"):
        routed = Workload(W.MOE_CONFIGS[name[:-len("_shared")]], dev)
        res = time_shared_fold(routed, W.MOE_CONFIGS[name], dev, steps, warmup, peaks["hbm_gbs"])
        t = res["ms_folded"] / 1e3
        line = {"metric": f"moe_{name}_tokens_per_s", "value": world * routed.cfg.T / t, "unit": "tokens/s",
                "n_gpus": world, "steps": steps, "warmup": warmup, "ms_per_step": res["ms_folded"],
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "nvfp4",
                "data": "synthetic", "config": config_block(W.MOE_CONFIGS[name], world),
                "tokens_per_s_separate": world * routed.cfg.T / (res["ms_separate"] / 1e3), "shared_fold": res,
                "gpu_launches": (res["launches_folded"] + res["launches_separate"]) * steps}
        if rank == 0:
            print(json.dumps(line), flush=True)
        return
    dec = Workload(W.MOE_CONFIGS[name], dev)
    ms_dec, stages = time_steps(dec, steps, warmup, world, graph=False)
    err = nvfp4_moe_get_error(dec.ws)
    if err != 0:
        raise RuntimeError(f"device error word {err}")
    t = ms_dec / steps / 1e3
    gbs = dec.step_bytes() / t / 1e9
    kb = dec.kernel_bytes()
    dom = max(stages, key=lambda s: stages[s])
    achieved = kb[dom] / (stages[dom] / 1e3) / 1e9
    line = {"metric": f"moe_{name}_GB_per_s", "value": gbs, "unit": "GB/s", "n_gpus": world, "steps": steps,
            "warmup": warmup, "ms_per_step": ms_dec / steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "nvfp4", "data": "synthetic", "config": config_block(dec.cfg, world),
            "hbm_frac": gbs / peaks["hbm_gbs"], "stage_ms": stages,
            "roofline": {"bound": "hbm", "kernel": dom, "achieved": achieved, "peak": peaks["hbm_gbs"],
                         "unit": "GB/s", "frac": achieved / peaks["hbm_gbs"], "peak_source": f"{peak_src} hbm_gbs",
                         "algorithmic_bytes": kb[dom], "traffic": ncu_traffic(dom, name)},
            "gpu_launches": dec.launches_per_step * steps, "clocks": CLOCKS.summary([f"timed_{name}"])}
    if rank == 0:
        print(json.dumps(line), flush=True)


def run_reference(args):
    """The CPU oracle on this host's cores, one routed slot (one expert of one
    token, 1/k of a token's work) of the prefill batch per step, cycling
    through a fixed sample, so that the default run stays within minutes;
    rank 0 only."""
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return
    import oracle as O
    local = int(os.environ.get("LOCAL_RANK", "0"))
    dev = torch.device("cuda", local) if torch.cuda.is_available() else torch.device("cpu")
    cfg = W.MOE_CONFIGS["prefill"]
    steps, warmup = args.steps, max(3, args.warmup)
    tokens = np.sort(np.random.default_rng(321).choice(cfg.T, 4, replace=False))
    # nothing of the library on this path: the sampled tokens are the oracle's
    # own warmup batch for inter_gs (it sets the values, not the work)
    sample = oracle_sample(cfg, tokens, dev, None)
    sample["inter_gs"] = O.moe_warmup_inter_gs(**{key: v for key, v in sample.items() if key != "inter_gs"})
    k = cfg.k
    n_slots = len(tokens) * k
    for i in range(warmup):
        run_oracle_tokens(sample, (i % n_slots) // k, slot=i % k)
    total = 0.0
    for i in range(steps):
        total += run_oracle_tokens(sample, (i % n_slots) // k, slot=i % k)
    value = steps / k / total               # tokens/s: k slots make a token
    line = {"impl": "reference", "metric": "moe_prefill_tokens_per_s", "value": value, "unit": "tokens/s",
            "n_gpus": world, "steps": steps, "warmup": warmup, "ms_per_step": total / steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32/f64",
            "data": "synthetic", "config": config_block(cfg, 1),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": O.num_threads(), "kind": "oracle",
                             "sample": f"one routed slot (one expert of one token) of the prefill batch per step, "
                                       f"cycling over the {n_slots} slots of {len(tokens)} tokens"},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--eager", action="store_true", help="time eager launches instead of one CUDA-graph replay")
    ap.add_argument("--only", choices=["all", "decode", "prefill", "prefill_ep48", "prefill_front", "shared", "tiny",
                                       "decode_shared", "prefill_shared", "mla"], default="all",
                    help="one workload alone (small profiling cases)")
    args = ap.parse_args()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
