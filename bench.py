#!/usr/bin/env python3
"""Benchmark of the SIGE sparse-conv hot path on B200.

Workload (one step = one pass of the whole hot path over one edit): the
DDPM-style residual block at 256x256, C=128, bf16 storage / fp32 accumulation,
with a ~1.2% edit made of 1-3 seeded discs, in ONE launch
(sige_resblock_step):
    mask     : difference mask of x_orig vs x_edit -> 8x8 tile list (dilate 1)
    resblock : both layers on the tiles: gather(GN1 + SiLU) -> 3x3 conv1
               (+bias) -> y1 (into the cached y1, and on chip with a one-pixel
               ring) -> GN2 + SiLU -> 3x3 conv2 (+bias +x_edit) -> scatter
               into the cached out
Timed beside it: the same step as two launches (sige_reduce_mask, then
sige_resblock_fused: `two_launch_step_us`) and as three (the mask, then each
layer as its own fused-layer launch: `unfused_step_us`).
The caches (y1 and out of the original image, GroupNorm statistics of the
original) are computed once beforehand by the same library's dense conv, as
the engine pre-computes the original activations.

Timing: each call is captured in its own CUDA graph; every step starts with a
256 MiB write that flushes the 126 MB L2 followed by a 256 MiB read (so the
dirty lines are written back before, not during, the timed step), then CUDA
events on the launching stream bracket the three replays.  W warm-up steps, then exactly K timed
steps, barrier + synchronize on both sides, max over ranks.  More GPUs run
independent replicas (one edit each, no collective).

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl {sige,reference}]
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "sparse-conv layer latency (us) & % of roofline at 1.2% edit area vs dense conv"
WORKLOAD = "DDPM res block 256x256 C=128 bf16, GN(32)+SiLU -> conv3x3 -> GN+SiLU -> conv3x3 + residual, 8x8 tiles, 1.2% edit"
H = W = 256
C = 128
BLOCK = 8
THRESH = 1e-3
FLUSH_BYTES = 256 << 20
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}


# ------------------------------------------------------------------ helpers

def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    return {**FALLBACK_PEAKS, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def strip_c_comments(text: str) -> str:
    """C / C++ / CUDA source without its comments: each // or /* */ comment
    becomes one space (string and character literals are left alone), then
    trailing blanks and empty lines go."""
    out, i, n = [], 0, len(text)
    while i < n:
        ch = text[i]
        if ch in "\"'":
            j = i + 1
            while j < n and text[j] != ch and text[j] != "\n":
                j += 2 if text[j] == "\\" else 1
            out.append(text[i:j + 1])
            i = j + 1
        elif text.startswith("//", i):
            j = text.find("\n", i)
            i = n if j < 0 else j
            out.append(" ")
        elif text.startswith("/*", i):
            j = text.find("*/", i + 2)
            i = n if j < 0 else j + 2
            out.append(" ")
        else:
            out.append(ch)
            i += 1
    lines = (ln.rstrip() for ln in "".join(out).split("\n"))
    return "\n".join(ln for ln in lines if ln)


def code_sha(relpaths):
    """Hash of the sources' code (comments and blank lines left out), so that a
    traffic figure survives a comment edit and not a code edit."""
    h = hashlib.sha256()
    for rp in relpaths:
        with open(os.path.join(ROOT, rp), encoding="utf-8") as f:
            h.update(strip_c_comments(f.read()).encode())
        h.update(b"\0")
    return h.hexdigest()[:16]


def ncu_traffic(kernel):
    """DRAM bytes (read + write) per launch from the committed ncu summary, when
    it was taken on the current code of that kernel; else None."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f).get(kernel)
    if not d:
        return None
    try:
        if code_sha(d["sources"]) != d["code_sha"]:
            return None
    except (OSError, KeyError):
        return None
    return float(d["bytes_per_launch"])


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled while the timed loop runs.

    A reader thread stamps every sample with its arrival time.  `begin()` waits
    for the first sample (nvidia-smi takes a moment to start) and marks the
    start of the timed region, `stop()` marks its end and summarises the
    samples taken inside it.  A timed region shorter than the sampling period
    may hold none; then the last sample before it and the first after it
    (which bracket it) are reported, and `window` says so."""
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")
    PERIOD_MS = 50

    def __init__(self, device_index, cmd=None):
        import threading
        self.proc, self.lines, self.t0 = None, [], None
        self.lock = threading.Lock()
        try:
            if cmd is None:
                uuid = str(torch.cuda.get_device_properties(device_index).uuid)
                sel = uuid if uuid.startswith("GPU-") else f"GPU-{uuid}"
                cmd = ["nvidia-smi", "-i", sel, f"--query-gpu={self.FIELDS}",
                       "--format=csv,noheader,nounits", "-lms", str(self.PERIOD_MS)]
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self.reader = threading.Thread(target=self._read, daemon=True)
        self.reader.start()

    def _read(self):
        for ln in self.proc.stdout:
            with self.lock:
                self.lines.append((time.perf_counter(), ln))

    def _wait_lines(self, n, timeout):
        end = time.perf_counter() + timeout
        while time.perf_counter() < end:
            with self.lock:
                if len(self.lines) >= n:
                    return
            time.sleep(0.005)

    def begin(self):
        if self.proc is not None:
            self._wait_lines(1, 10.0)
        self.t0 = time.perf_counter()

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        t1 = time.perf_counter()
        with self.lock:
            n_at_end = len(self.lines)
        self._wait_lines(n_at_end + 1, 1.0)        # one sample after the region
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.reader.join(timeout=5)
        with self.lock:
            lines = list(self.lines)
        t0 = self.t0 if self.t0 is not None else t1
        inside = [ln for t, ln in lines if t0 <= t <= t1]
        window = "inside the timed region"
        if not inside:
            before = [ln for t, ln in lines if t < t0][-1:]
            after = [ln for t, ln in lines if t > t1][:1]
            inside = before + after
            window = "timed region shorter than the sampling period: the samples just before and after it"
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in inside:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 8:
                continue
            try:
                sm.append(float(f[0]))
                mx.append(float(f[1]))
            except ValueError:
                continue
            for nm, v in zip(names, f[4:8]):
                if v.lower() == "active":
                    reasons.add(nm)
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(sm), "window": window}


def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def max_over_ranks(vals, device):
    """Element-wise maximum of a list of floats over all ranks of the default
    process group (identity with one rank).  Every rank must call it with the
    same number of values, in the same order of calls."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return [float(v) for v in vals]
    t = torch.tensor([float(v) for v in vals], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


# ------------------------------------------------------------------ workload

def make_workload(seed, dev, area=0.012):
    import spatially_sparse_incremental_b200 as sige
    from spatially_sparse_incremental_b200 import inputs
    blk = inputs.make_cfg3(seed, H=H, W=W, C=C, area=area, block=BLOCK)
    d = {k: getattr(blk, k).to(dev) for k in ("x_orig", "x_edit", "w1", "b1", "w2", "b2", "g1", "be1", "g2", "be2")}
    cd = sige.conv_desc(3, 1, 1, C, C, BLOCK)
    cap = (H // BLOCK) * (W // BLOCK)
    # cache of the original image (computed once, untimed)
    gs1, gh1 = sige.sige_groupnorm_affine(d["x_orig"], 32, d["g1"], d["be1"])
    y1 = sige.sige_dense_conv(d["x_orig"], d["w1"], d["b1"], cd, gn_scale=gs1, gn_shift=gh1, silu=True)
    gs2, gh2 = sige.sige_groupnorm_affine(y1, 32, d["g2"], d["be2"])
    out = sige.sige_dense_conv(y1, d["w2"], d["b2"], cd, gn_scale=gs2, gn_shift=gh2, silu=True, residual=d["x_orig"])
    idx = torch.zeros((cap, 2), dtype=torch.int32, device=dev)
    cnt = torch.zeros(1, dtype=torch.int32, device=dev)
    mask_ws = sige.zeros_workspace(sige.sige_reduce_mask_workspace_bytes(sige.tensor_desc(d["x_orig"]),
                                                                         [(H, W, BLOCK, cap)]), dev)
    conv_ws = sige.zeros_workspace(sige.sige_conv_workspace_bytes(cd, 1, cap, H, W), dev)
    rb_ws = sige.zeros_workspace(sige.sige_workspace_bytes(sige.CALL_RESBLOCK, None, cap), dev)
    step_ws = sige.zeros_workspace(sige.sige_resblock_step_workspace_bytes(d["x_orig"], BLOCK), dev)
    d.update(cd=cd, cap=cap, gs1=gs1, gh1=gh1, gs2=gs2, gh2=gh2, y1=y1, out=out, idx=idx, cnt=cnt,
             mask_ws=mask_ws, conv_ws=conv_ws, rb_ws=rb_ws, step_ws=step_ws, blk=blk)
    return d


def step_calls(d, stream=None):
    """The step as one call (for graph capture)."""
    import spatially_sparse_incremental_b200 as sige

    def step():
        sige.sige_resblock_step(d["x_orig"], d["x_edit"], THRESH, d["w1"], d["b1"], (d["gs1"], d["gh1"]), d["w2"],
                                d["b2"], (d["gs2"], d["gh2"]), d["y1"], d["out"], d["cap"], idx=d["idx"],
                                count=d["cnt"], workspace=d["step_ws"], stream=stream)
    return {"step": step}


def two_launch_calls(d, stream=None):
    """The step as the mask call and the fused res-block call."""
    import spatially_sparse_incremental_b200 as sige

    def mask():
        sige.sige_reduce_mask(d["x_orig"], d["x_edit"], THRESH, [(H, W, BLOCK, d["cap"])], 1, idx=d["idx"],
                              counts=d["cnt"], workspace=d["mask_ws"], stream=stream)

    def resblock():
        sige.sige_resblock_fused(d["x_edit"], d["w1"], d["b1"], (d["gs1"], d["gh1"]), d["w2"], d["b2"],
                                 (d["gs2"], d["gh2"]), d["idx"], d["cnt"], d["cap"], d["y1"], d["out"],
                                 workspace=d["rb_ws"], stream=stream)
    return {"mask": mask, "resblock": resblock}


def unfused_calls(d, stream=None):
    """The same step with each layer as its own fused-layer launch."""
    import spatially_sparse_incremental_b200 as sige

    def mask():
        sige.sige_reduce_mask(d["x_orig"], d["x_edit"], THRESH, [(H, W, BLOCK, d["cap"])], 1, idx=d["idx"],
                              counts=d["cnt"], workspace=d["mask_ws"], stream=stream)

    def conv1():
        sige.sige_conv_fused(d["x_edit"], d["w1"], d["b1"], d["cd"], d["idx"], d["cnt"], d["cap"], d["y1"],
                             d["gs1"], d["gh1"], silu=True, workspace=d["conv_ws"], stream=stream)

    def conv2():
        sige.sige_conv_fused(d["y1"], d["w2"], d["b2"], d["cd"], d["idx"], d["cnt"], d["cap"], d["out"],
                             d["gs2"], d["gh2"], silu=True, residual=d["x_edit"], workspace=d["conv_ws"],
                             stream=stream)
    return {"mask": mask, "conv1": conv1, "conv2": conv2}


def dense_calls(d, stream=None):
    import spatially_sparse_incremental_b200 as sige
    y1d = torch.empty_like(d["y1"])
    outd = torch.empty_like(d["out"])

    def dense1():
        sige.sige_dense_conv(d["x_edit"], d["w1"], d["b1"], d["cd"], y=y1d, gn_scale=d["gs1"], gn_shift=d["gh1"],
                             silu=True, workspace=d["conv_ws"], stream=stream)

    def dense2():
        sige.sige_dense_conv(y1d, d["w2"], d["b2"], d["cd"], y=outd, gn_scale=d["gs2"], gn_shift=d["gh2"],
                             silu=True, residual=d["x_edit"], workspace=d["conv_ws"], stream=stream)
    return {"dense1": dense1, "dense2": dense2}


def capture(fn, stream):
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        fn()
    return g


class L2Flush:
    """Cold-L2 reset between timed steps: write a 256 MiB buffer (twice the
    126 MB L2), then stream-read another 256 MiB buffer so the write-backs of
    the dirty lines happen here, untimed, and the timed step starts from a
    cold but clean L2."""

    def __init__(self, dev):
        self.w = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
        self.r = torch.ones(FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
        self.sink = torch.empty((), dtype=torch.float32, device=dev)

    def __call__(self):
        self.w.zero_()
        torch.sum(self.r, dim=0, out=self.sink)


def timed_graph_steps(graphs, flush, steps, stream):
    """Per step: L2 flush, then events around each graph replay.  Returns per-
    call lists of durations (ms) and the per-step totals."""
    names = list(graphs)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(len(names) + 1)] for _ in range(steps)]
    with torch.cuda.stream(stream):
        for k in range(steps):
            flush()
            ev[k][0].record(stream)
            for i, nm in enumerate(names):
                graphs[nm].replay()
                ev[k][i + 1].record(stream)
    stream.synchronize()
    per = {nm: [ev[k][i].elapsed_time(ev[k][i + 1]) for k in range(steps)] for i, nm in enumerate(names)}
    tot = [ev[k][0].elapsed_time(ev[k][-1]) for k in range(steps)]
    return per, tot


def time_graph(g, flush, reps, stream, warm=False):
    """Device time (ms) of each replay of graph g, L2 flushed before each
    replay unless warm."""
    times = []
    with torch.cuda.stream(stream):
        for k in range(reps + 3):
            if not warm:
                flush()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            g.replay()
            e1.record(stream)
            if k >= 3:
                times.append((e0, e1))
    stream.synchronize()
    return [a.elapsed_time(b) for a, b in times]


FP32_ALU_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12   # FMA lanes x 2 x max SM clock
SFU_TEXP = 148 * 16 * 1.965e9 / 1e12                 # exp2 results per second (1e12): 16 per SM and clock


def layer_roofline(macs, nbytes, dtype_bits, peaks, us):
    """Roofline time of one sparse layer and the fraction reached: tensor (bf16)
    or FP32 ALU for the arithmetic, measured HBM copy bandwidth for the bytes."""
    if dtype_bits == 32:
        t_c, bound_c = 2 * macs / (FP32_ALU_TFLOPS * 1e12), "alu"
    else:
        t_c, bound_c = 2 * macs / (peaks["bf16_tflops"] * 1e12), "tensor"
    t_b = nbytes / (peaks["hbm_gbs"] * 1e9)
    t = max(t_c, t_b)
    return {"bound": bound_c if t_c >= t_b else "hbm", "roof_us": t * 1e6, "frac": t / (us * 1e-6)}


def measure_extras(dev, flush, stream, peaks, seed, step_graph):
    """Measurement rows beyond the headline step: warm-L2 step, the edit-area
    sweep with a linear fit of step latency on active tiles, and one sparse vs
    dense layer per shape of the other workloads (fp32 64x64x64, the SD-latent
    and GauGAN-shaped layers) at 1.2% edit."""
    import spatially_sparse_incremental_b200 as sige
    from spatially_sparse_incremental_b200 import inputs
    out = {}
    warm = time_graph(step_graph, flush, 50, stream, warm=True)
    out["warm_l2_step_us"] = float(np.median(warm)) * 1e3

    sweep = []
    for area in (0.005, 0.012, 0.05, 0.10, 0.20):
        d = make_workload(seed, dev, area=area)
        torch.cuda.synchronize()   # the workload is built on the default stream
        calls = step_calls(d, stream)
        with torch.cuda.stream(stream):
            calls["step"]()
        stream.synchronize()
        tiles = int(d["cnt"].item())

        def whole():
            for fn in calls.values():
                fn()
        g = capture(whole, stream)
        t = time_graph(g, flush, 40, stream)
        fl, by = step_work(tiles)
        t_roof = max(fl / (peaks["bf16_tflops"] * 1e12), by / (peaks["hbm_gbs"] * 1e9))
        med = float(np.median(t)) * 1e-3
        sweep.append({"area": area, "active_tiles": tiles, "step_us": med * 1e6,
                      "p90_us": float(np.percentile(t, 90)) * 1e3, "roof_us": t_roof * 1e6, "frac": t_roof / med,
                      "tensor_frac": fl / med / 1e12 / peaks["bf16_tflops"]})
        del g, d
    x = np.array([r["active_tiles"] for r in sweep], dtype=np.float64)
    y = np.array([r["step_us"] for r in sweep], dtype=np.float64)
    A = np.vstack([x, np.ones_like(x)]).T
    (slope, icpt), *_ = np.linalg.lstsq(A, y, rcond=None)
    pred = A @ np.array([slope, icpt])
    r2 = 1.0 - float(((y - pred) ** 2).sum()) / max(1e-30, float(((y - y.mean()) ** 2).sum()))
    out["area_sweep"] = {"rows": sweep, "fit": {"slope_us_per_tile": float(slope), "intercept_us": float(icpt),
                                                "r2": r2}}

    # the same step with the tile list from a 2-pixel dilation (exact for two
    # chained 3x3 convs) instead of one tile
    d = make_workload(seed, dev)
    torch.cuda.synchronize()
    calls = two_launch_calls(d, stream)

    def mask_px():
        sige.sige_reduce_mask_px(d["x_orig"], d["x_edit"], THRESH, [(H, W, BLOCK, d["cap"])], 2, idx=d["idx"],
                                 counts=d["cnt"], workspace=d["mask_ws"], stream=stream)
    with torch.cuda.stream(stream):
        mask_px()
    stream.synchronize()
    tiles_px = int(d["cnt"].item())

    def whole_px():
        mask_px()
        calls["resblock"]()
    g = capture(whole_px, stream)
    t = time_graph(g, flush, 40, stream)
    out["pixel_dilation_step"] = {"radius_px": 2, "active_tiles": tiles_px, "step_us": float(np.median(t)) * 1e3}
    del g, d

    rows = layer_rows(seed, dev, flush, stream, peaks)
    try:
        out["attention"] = attention_timing(seed, dev, flush, stream, peaks)
    except Exception as e:
        out["attention"] = {"error": str(e)[:200]}
    try:
        out["gather_scatter"] = gather_scatter_timing(seed, dev, flush, stream, peaks)
    except Exception as e:
        out["gather_scatter"] = {"error": str(e)[:200]}
    # edit-area sweeps of the SD-latent and GauGAN-shaped layers: active tiles,
    # sparse and dense time and the roofline fraction at every area
    sweeps = []
    for i, (h, w, c, b) in enumerate(inputs.CFG4_LAYERS):
        for area in inputs.CFG4_AREAS:
            sweeps.append((f"SD latent {h}x{w} C{c} 3x3 b{b}", area, inputs.make_cfg4_layer(seed, i, area=area)))
    for i, (h, w, ci, co, k, st, b) in enumerate(inputs.CFG5_LAYERS):
        for area in inputs.CFG5_AREAS:
            sweeps.append((f"GauGAN {h}x{w} {ci}->{co} {k}x{k} s{st} b{b}", area,
                           inputs.make_cfg5_layer(seed, i, area=area)))
    srows, dense_cache = [], {}
    for name, area, L in sweeps:
        try:
            r = layer_timing(L, 16, dev, flush, stream, peaks, reps=10, dense_us=dense_cache.get(name))
            dense_cache[name] = r["dense_us"]
            srows.append(dict(name=name, area=area, **r))
        except Exception as e:
            srows.append({"name": name, "area": area, "error": str(e)[:200]})
    out["layer_sweeps"] = srows
    out["layers"] = rows
    return out


def layer_rows(seed, dev, flush, stream, peaks, reps=30):
    """Every per-layer workload at its default edit: one fused call, sparse
    and dense, each in its own CUDA graph with L2 flushed."""
    from spatially_sparse_incremental_b200 import inputs
    layers = [("fp32 64x64 C64 3x3 b4", inputs.make_cfg1(seed), 32)]
    for i, (h, w, c, b) in enumerate(inputs.CFG4_LAYERS):
        layers.append((f"SD latent {h}x{w} C{c} 3x3 b{b}", inputs.make_cfg4_layer(seed, i), 16))
    for i, (h, w, ci, co, k, st, b) in enumerate(inputs.CFG5_LAYERS):
        layers.append((f"GauGAN {h}x{w} {ci}->{co} {k}x{k} s{st} b{b}", inputs.make_cfg5_layer(seed, i), 16))
    rows = []
    for name, L, bits in layers:
        try:
            rows.append(dict(name=name, **layer_timing(L, bits, dev, flush, stream, peaks, reps=reps)))
        except Exception as e:   # a failing row is reported, not fatal to the headline line
            rows.append({"name": name, "error": str(e)[:200]})
    # the 4x4-tile 3x3 layers with GroupNorm + SiLU on the input (a U-Net res block's convs)
    gn_layers = [(f"SD latent {h}x{w} C{c} 3x3 b{b}, GN+SiLU", inputs.make_cfg4_layer(seed, i))
                 for i, (h, w, c, b) in enumerate(inputs.CFG4_LAYERS) if b == 4]
    gn_layers += [(f"GauGAN {h}x{w} {ci}->{co} {k}x{k} s{st} b{b}, GN+SiLU", inputs.make_cfg5_layer(seed, i))
                  for i, (h, w, ci, co, k, st, b) in enumerate(inputs.CFG5_LAYERS) if b == 4 and k == 3]
    for name, L in gn_layers:
        try:
            rows.append(dict(name=name, **layer_timing(L, 16, dev, flush, stream, peaks, reps=reps, gn=True)))
        except Exception as e:
            rows.append({"name": name, "error": str(e)[:200]})
    for i, (h, w, ci, co, b) in enumerate(inputs.UPSAMPLE_LAYERS):
        name = f"GauGAN upsample {h}x{w}->{2 * h}x{2 * w} {ci}->{co} 3x3 transposed s2 b{b}"
        try:
            rows.append(dict(name=name, **ext_layer_timing(inputs.make_upsample_layer(seed, i), dev, flush, stream,
                                                           peaks, transposed=True, reps=min(20, reps))))
        except Exception as e:
            rows.append({"name": name, "error": str(e)[:200]})
    for i, (h, w, ci, co, b) in enumerate(inputs.SPADE_LAYERS):
        name = f"GauGAN SPADE {h}x{w} {ci}->{co} 3x3 b{b} LeakyReLU"
        try:
            rows.append(dict(name=name, **ext_layer_timing(inputs.make_spade_layer(seed, i), dev, flush, stream,
                                                           peaks, spade=True, reps=min(20, reps))))
        except Exception as e:
            rows.append({"name": name, "error": str(e)[:200]})
    return rows


def gather_scatter_timing(seed, dev, flush, stream, peaks, reps=30):
    """The unfused calls on the headline workload's tile list: the gather of
    conv1's 10x10 halos (GroupNorm1 + SiLU applied, bf16 blocks out) and the
    scatter of conv2's float32 blocks (+ bias + residual, bf16 into the cached
    output); each against the HBM roofline of its own bytes (halo pixels read
    once per tile, blocks written / read, outputs and residual)."""
    import spatially_sparse_incremental_b200 as sige
    d = make_workload(seed, dev)
    two_launch_calls(d)["mask"]()            # the step's tile list
    torch.cuda.synchronize()
    n = int(d["cnt"].item())
    assert n > 0, "the headline edit lists no tile"
    cd = d["cd"]
    b_in = (cd.block - 1) * cd.stride + cd.kernel
    blocks = torch.empty((max(d["cap"], 1), 1, b_in, b_in, C), dtype=torch.bfloat16, device=dev)
    oblk = torch.randn((max(d["cap"], 1), 1, BLOCK, BLOCK, C), generator=torch.Generator().manual_seed(seed)).to(dev)
    y = d["out"].clone()

    def gather():
        sige.sige_gather(d["x_edit"], cd, d["idx"], d["cnt"], d["cap"], d["gs1"], d["gh1"], silu=True, blocks=blocks,
                         stream=stream)

    def scatter():
        sige.sige_scatter(oblk, cd, d["idx"], d["cnt"], d["cap"], y, bias=d["b2"], residual=d["x_edit"],
                          stream=stream)
    res = {"active_tiles": n}
    for name, fn, nbytes in (("gather", gather, 2 * n * b_in * b_in * C * 2),
                             ("scatter", scatter, n * BLOCK * BLOCK * C * (4 + 2 + 2))):
        g = capture(fn, stream)
        t = time_graph(g, flush, reps, stream)
        us = float(np.median(t)) * 1e3
        res[name] = {"us": us, "bytes": nbytes, "gbs": nbytes / (us * 1e-6) / 1e9,
                     "frac": nbytes / (us * 1e-6) / 1e9 / peaks["hbm_gbs"]}
        del g
    return res


def layer_timing(L, bits, dev, flush, stream, peaks, reps=30, dense_us=None, gn=False):
    """One layer, sparse (its tile list at the layer's edit) and dense, each one
    call in its own graph with L2 flushed; gn: with a GroupNorm-style affine
    (seeded per-channel scale / shift) and SiLU on the input, as in a
    diffusion U-Net's res-block convs."""
    import spatially_sparse_incremental_b200 as sige
    xo, xe = L.x_orig.to(dev), L.x_edit.to(dev)
    wt, bias = L.weight.to(dev), L.bias.to(dev)
    N, Hi, Wi, ci = xo.shape
    co, k, st, b = wt.shape[0], L.kernel, L.stride, L.block
    cd = sige.conv_desc(k, st, L.pad, ci, co, b)
    gs = gh = None
    if gn:
        g = torch.Generator().manual_seed(ci * 7 + co)
        gs = (1.0 + 0.3 * torch.randn((N, ci), generator=g)).float().to(dev)
        gh = (0.1 * torch.randn((N, ci), generator=g)).float().to(dev)
    y0 = sige.sige_dense_conv(xo, wt, bias, cd)
    Ho, Wo = y0.shape[1], y0.shape[2]
    cap = -(-Ho // b) * -(-Wo // b)
    thr = L.meta.get("threshold", 1e-3) if L.meta else 1e-3
    idx, cnt, _ = sige.sige_reduce_mask(xo, xe, thr, [(Ho, Wo, b, cap)], 1)
    torch.cuda.synchronize()
    tiles = int(cnt.item())
    y = y0.clone()
    ws = sige.zeros_workspace(sige.sige_conv_workspace_bytes(cd, N, cap, Ho, Wo), dev)
    yd = torch.empty_like(y0)
    g_sp = capture(lambda: sige.sige_conv_fused(xe, wt, bias, cd, idx, cnt, cap, y, gs, gh, silu=gn, workspace=ws,
                                                stream=stream), stream)
    t_sp = float(np.median(time_graph(g_sp, flush, reps, stream))) * 1e3
    if dense_us is None:
        g_de = capture(lambda: sige.sige_dense_conv(xe, wt, bias, cd, y=yd, gn_scale=gs, gn_shift=gh, silu=gn,
                                                    workspace=ws, stream=stream), stream)
        t_de = float(np.median(time_graph(g_de, flush, reps, stream))) * 1e3
        del g_de
    else:
        t_de = dense_us
    esz = bits // 8
    bin_ = (b - 1) * st + k
    macs = tiles * b * b * ci * co * k * k
    nbytes = tiles * (bin_ * bin_ * ci + b * b * co) * esz + co * k * k * ci * esz + co * 4
    roof = layer_roofline(macs, nbytes, bits, peaks, t_sp)
    del g_sp
    return {"active_tiles": tiles, "tiles_total": cap, "sparse_us": t_sp, "dense_us": t_de,
            "speedup": t_de / t_sp, "path": "tcgen05" if sige.sige_conv_path(cd, L.x_orig.dtype) == 1 else "cuda-core",
            "roofline": roof}


def attention_timing(seed, dev, flush, stream, peaks, H_=64, W_=64, C_=320, heads=8, block=4, area=0.012, reps=20):
    """The SD-latent self-attention step with pruned queries: the tokens under
    the 4x4-tile list of a 1.2% edit (one rectangle plus discs at 64x64) attend
    to all 4096 keys; 8 heads of 40.  Sparse = sige_attention_core at those
    tokens; dense = the same call with every tile listed."""
    import spatially_sparse_incremental_b200 as sige
    from spatially_sparse_incremental_b200 import inputs
    L = inputs.make_cfg4_layer(seed, 0, area=area)            # the 64x64 C320 map and its edit
    q = L.x_edit.to(dev)
    g = torch.Generator().manual_seed(seed)
    k = torch.randn((1, H_ * W_, C_), generator=g).to(torch.bfloat16).to(dev)
    v = torch.randn((1, H_ * W_, C_), generator=g).to(torch.bfloat16).to(dev)
    cap = (H_ // block) * (W_ // block)
    idx, cnt, _ = sige.sige_reduce_mask(L.x_orig.to(dev), q, 1e-3, [(H_, W_, block, cap)], 1)
    every = torch.tensor([(h, w) for h in range(0, H_, block) for w in range(0, W_, block)], dtype=torch.int32,
                         device=dev)
    call = torch.tensor([cap], dtype=torch.int32, device=dev)
    torch.cuda.synchronize()
    tiles = int(cnt.item())
    o = torch.zeros((1, H_, W_, C_), dtype=torch.bfloat16, device=dev)
    g_sp = capture(lambda: sige.sige_attention_core(q, k, v, heads, idx, cnt, cap, block, o, stream), stream)
    g_de = capture(lambda: sige.sige_attention_core(q, k, v, heads, every, call, cap, block, o, stream), stream)
    t_sp = float(np.median(time_graph(g_sp, flush, reps, stream))) * 1e3
    t_de = float(np.median(time_graph(g_de, flush, max(3, reps // 4), stream))) * 1e3
    del g_sp, g_de
    m_tok = tiles * block * block
    flops = 2.0 * m_tok * H_ * W_ * (C_ + C_)
    nbytes = H_ * W_ * (C_ + C_) * 2 + m_tok * (C_ + C_) * 2
    exps = float(m_tok) * H_ * W_ * heads                      # one exponential per (query, key, head)
    t_tensor = flops / (peaks["bf16_tflops"] * 1e12)
    t_sfu = exps / (SFU_TEXP * 1e12)
    t_de_sfu = float(H_ * W_) * H_ * W_ * heads / (SFU_TEXP * 1e12)
    path = sige.sige_attention_path(q, C_, heads)
    return {"name": f"SD latent {H_}x{W_} C{C_} self-attention, {heads} heads, b{block}, {area:.1%} edit",
            "active_tiles": tiles, "query_tokens": m_tok, "keys": H_ * W_, "sparse_us": t_sp, "dense_us": t_de,
            "speedup": t_de / t_sp,
            "path": "tcgen05 (QK^T and PV on tensor cores, P bf16 in tensor memory)" if path == 1
                    else "cuda-core (fp32 online softmax)",
            "roofline": {"bound": "sfu", "exps": exps, "roof_us": t_sfu * 1e6, "frac": t_sfu / (t_sp * 1e-6),
                         "dense_frac": t_de_sfu / (t_de * 1e-6),
                         "tensor_roof_us": t_tensor * 1e6, "flops": flops, "bytes": nbytes}}


def ext_layer_timing(L, dev, flush, stream, peaks, transposed=False, spade=False, reps=20):
    """A GauGAN-style layer (transposed conv, or SPADE-modulated input with
    LeakyReLU) through sige_conv_fused_ext: sparse on the tiles of its edit
    vs the same call on every tile."""
    import spatially_sparse_incremental_b200 as sige
    xo, xe = L.x_orig.to(dev), L.x_edit.to(dev)
    wt, bias = L.weight.to(dev), L.bias.to(dev)
    N, Hi, Wi, ci = xo.shape
    co, k, b = wt.shape[0], L.kernel, L.block
    cd = sige.conv_desc(k, L.stride, L.pad, ci, co, b)
    kw = {}
    if transposed:
        kw = dict(transposed=True, output_padding=L.meta["output_padding"])
    if spade:
        ones = torch.ones(ci, device=dev)
        ns, nh = sige.sige_groupnorm_affine(xo, ci, ones, torch.zeros(ci, device=dev))
        kw = dict(gn_scale=ns, gn_shift=nh, spade_gamma=L.meta["gamma_edit"].to(dev),
                  spade_beta=L.meta["beta_edit"].to(dev), act=sige.ACT_LEAKY)
    y0 = sige.sige_conv_fused_ext(xo, wt, bias, cd, **kw)
    Ho, Wo = y0.shape[1], y0.shape[2]
    cap = -(-Ho // b) * -(-Wo // b)
    if transposed:
        # the output-resolution edit, as a mask image the library reduces
        eo = torch.from_numpy(L.meta["edit_out"].astype(np.uint8)).view(1, 1, Ho, Wo).to(dev)
        idx, cnt, _ = sige.sige_reduce_mask(torch.zeros_like(eo), eo, 0.0, [(Ho, Wo, b, cap)], 1, layout=sige.NCHW)
    else:
        idx, cnt, _ = sige.sige_reduce_mask(xo, xe, 1e-3, [(Ho, Wo, b, cap)], 1)
    torch.cuda.synchronize()
    tiles = int(cnt.item())
    y = y0.clone()
    ws = sige.zeros_workspace(sige.sige_conv_workspace_bytes(cd, N, cap, Ho, Wo), dev)
    yd = torch.empty_like(y0)
    g_sp = capture(lambda: sige.sige_conv_fused_ext(xe, wt, bias, cd, y=y, idx=idx, count=cnt, capacity=cap,
                                                    workspace=ws, stream=stream, **kw), stream)
    g_de = capture(lambda: sige.sige_conv_fused_ext(xe, wt, bias, cd, y=yd, workspace=ws, stream=stream, **kw),
                   stream)
    t_sp = float(np.median(time_graph(g_sp, flush, reps, stream))) * 1e3
    t_de = float(np.median(time_graph(g_de, flush, reps, stream))) * 1e3
    del g_sp, g_de
    # algorithmic work: the layer's own MACs at the tiles' pixels (for the
    # transposed conv the nonzero taps, k*k/s^2 per output pixel on average)
    taps = k * k / (L.stride ** 2) if transposed else k * k
    macs = tiles * b * b * ci * co * taps
    bin_in = (b // L.stride + 1) if transposed else (b - 1) * L.stride + k
    per_tile = bin_in * bin_in * ci * 2 + b * b * co * 2 + (2 * bin_in * bin_in * ci * 2 if spade else 0)
    nbytes = tiles * per_tile + co * k * k * ci * 2 + co * 4
    return {"active_tiles": tiles, "tiles_total": cap, "sparse_us": t_sp, "dense_us": t_de, "speedup": t_de / t_sp,
            "path": "tcgen05", "roofline": layer_roofline(macs, nbytes, 16, peaks, t_sp)}


# ------------------------------------------------------------------ roofline

def conv_work(n_tiles, residual):
    """Algorithmic FLOPs and bytes of one fused sparse conv launch on this workload."""
    macs = n_tiles * BLOCK * BLOCK * C * C * 9
    bin_ = BLOCK + 2
    gather = n_tiles * bin_ * bin_ * C * 2
    scatter = n_tiles * BLOCK * BLOCK * C * 2 * (2 if residual else 1)
    weights = C * 9 * C * 2 + C * 4
    return 2 * macs, gather + scatter + weights


def resblock_work(n_tiles):
    """Algorithmic FLOPs and bytes of one fused res-block launch: the two convs'
    MACs on the tiles (the ring of y1 that is recomputed is not counted); the x
    halo of each tile read once (12 x 12 pixels, which holds the residual), y1
    and out written at the tile, both weight tensors and the per-channel
    vectors once."""
    macs = 2 * n_tiles * BLOCK * BLOCK * C * C * 9
    halo = n_tiles * (BLOCK + 4) ** 2 * C * 2
    writes = 2 * n_tiles * BLOCK * BLOCK * C * 2
    weights = 2 * (C * 9 * C * 2) + 6 * C * 4
    return 2 * macs, halo + writes + weights


def step_work(n_tiles):
    """Algorithmic FLOPs and bytes of the one-launch step: both inputs read
    once by the mask (the halo of x_edit is read again from L2, not counted),
    the list written, y1 and out written at the tiles, both weight tensors and
    the per-channel vectors once; the two convs' MACs on the tiles."""
    flops, _ = resblock_work(n_tiles)
    writes = 2 * n_tiles * BLOCK * BLOCK * C * 2
    weights = 2 * (C * 9 * C * 2) + 6 * C * 4
    return flops, mask_work(n_tiles) + writes + weights


def mask_work(n_tiles):
    return 2 * H * W * C * 2 + n_tiles * 8 + 4


# ------------------------------------------------------------------ CPU oracle (baseline only)

class OracleStep:
    """The CPU oracle on the bench workload, for the CPU baseline and the
    reference arm.  The caches of the original image (GroupNorm statistics of
    x and of y1, the dense y1 and out) are built once with the oracle itself,
    untimed.  A step is the whole hot path on the full 256x256 image: pixel
    mask + tile list, then both tile-restricted sparse convs (the oracle's
    resblock_sparse).  ``dense_step`` is the oracle as defined: both layers
    dense over the image in double, then the listed tiles copied into the
    caches."""

    def __init__(self, seed, threads):
        import oracle
        from spatially_sparse_incremental_b200 import inputs
        self.oracle = oracle
        oracle.set_threads(threads)
        self.threads = threads
        blk = inputs.make_cfg3(seed, H=H, W=W, C=C, area=0.012, block=BLOCK)
        self.blk = blk
        self.g1 = oracle.gn_affine(blk.x_orig, 32, blk.g1, blk.be1)
        y1o = oracle.dense_conv(blk.x_orig, blk.w1, blk.b1, gn=self.g1, silu=True)
        self.g2 = oracle.gn_affine(y1o, 32, blk.g2, blk.be2)
        self.y1o, self.outo = oracle.resblock_dense(blk.x_orig, blk, self.g1, self.g2)

    def set_threads(self, n):
        self.oracle.set_threads(n)
        self.threads = n

    def step(self):
        o, b = self.oracle, self.blk
        idx = o.reduce_mask(b.x_orig, b.x_edit, THRESH, [(H, W, BLOCK)], 1)[0]
        o.resblock_sparse(b.x_edit, b, idx, self.y1o, self.outo, self.g1, self.g2)
        return len(idx)

    def dense_step(self):
        o, b = self.oracle, self.blk
        idx = o.reduce_mask(b.x_orig, b.x_edit, THRESH, [(H, W, BLOCK)], 1)[0]
        cov = np.zeros((H, W), dtype=bool)
        for h0, w0 in idx:
            cov[h0:h0 + BLOCK, w0:w0 + BLOCK] = True
        y1 = o.dense_conv(b.x_edit, b.w1, b.b1, gn=self.g1, silu=True)
        y1m = self.y1o.clone()
        y1m[:, torch.from_numpy(cov)] = y1[:, torch.from_numpy(cov)]
        out = o.dense_conv(y1m, b.w2, b.b2, gn=self.g2, silu=True, residual=b.x_edit)
        outm = self.outo.clone()
        outm[:, torch.from_numpy(cov)] = out[:, torch.from_numpy(cov)]
        return len(idx)

    def band_step(self, k, nbands=32):
        """1/nbands of a step: band k % nbands (H/nbands rows, full width) run
        as its own image, with the caches' rows of that band and the whole
        image's GroupNorm statistics."""
        o, b = self.oracle, self.blk
        rows = H // nbands
        r0 = (k % nbands) * rows
        xo = b.x_orig[:, r0:r0 + rows].contiguous()
        xe = b.x_edit[:, r0:r0 + rows].contiguous()
        idx = o.reduce_mask(xo, xe, THRESH, [(rows, W, BLOCK)], 1)[0]
        y1 = o.sparse_conv(xe, b.w1, b.b1, idx, self.y1o[:, r0:r0 + rows].contiguous(), block=BLOCK, gn=self.g1,
                           silu=True)
        o.sparse_conv(y1, b.w2, b.b2, idx, self.outo[:, r0:r0 + rows].contiguous(), block=BLOCK, gn=self.g2,
                      silu=True, residual=xe)
        return len(idx)

    def time_steps(self, n, dense=False):
        ts = []
        for _ in range(n):
            t0 = time.perf_counter()
            (self.dense_step if dense else self.step)()
            ts.append(time.perf_counter() - t0)
        return ts


def host_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


# ------------------------------------------------------------------ arms

def run_reference(args):
    ws, rank, _ = dist_env()
    if rank != 0:
        return 0
    cores = host_cores()
    t_build = time.perf_counter()
    orc_step = OracleStep(args.seed, cores)
    t_build = time.perf_counter() - t_build
    # W warm-up steps, then exactly K timed steps, each the whole hot path on
    # the full image (about 0.1-0.3 s each on a many-core host); when K of
    # those would take more than ~2 minutes, each step is one 1/32 band of the
    # image instead, scaled x32
    t0 = time.perf_counter()
    orc_step.time_steps(args.warmup)
    est = (time.perf_counter() - t0) / max(1, args.warmup)
    if est * args.steps <= 120.0:
        ts = orc_step.time_steps(args.steps)
        us = float(np.mean(ts)) * 1e6
        what = "the whole hot path on the full 256x256 image"
    else:
        ts = []
        for k in range(args.steps):
            t1 = time.perf_counter()
            orc_step.band_step(k)
            ts.append(time.perf_counter() - t1)
        us = float(np.mean(ts)) * 32e6
        what = "one 8-row band (1/32) of the 256x256 image run as its own image, scaled x32,"
    
    line = {
        "impl": "reference", "metric": METRIC, "value": us, "unit": "us", "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": us / 1e3, "higher_is_better": False, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD, "H": H, "W": W, "C": C, "block": BLOCK, "edit_area": 0.012},
        "cpu_baseline": {"value": us, "unit": "us", "cores": cores, "kind": "oracle",
                         "sample": f"each step = {what} (pixel mask + tile list, both tile-restricted sparse convs "
                                   f"of the res block), caches and GroupNorm statistics of the original built "
                                   f"once by the oracle ({t_build:.1f} s, untimed); {len(ts)} steps in "
                                   f"{sum(ts):.1f} s"},
        "e2e": {"value": us, "unit": "us", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def run_sige(args):
    import spatially_sparse_incremental_b200 as sige
    ws, rank, local = dist_env()
    if ws > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local if ws > 1 else torch.cuda.current_device())
    torch.cuda.set_device(dev)
    peaks = load_peaks()

    d = make_workload(args.seed + rank, dev)
    torch.cuda.synchronize()
    stream = torch.cuda.Stream(device=dev)
    calls = step_calls(d, stream)
    # eager warm-up of every call once (also counts kernels per call)
    with torch.cuda.stream(stream):
        launches = {}
        for nm, fn in calls.items():
            before = sige.sige_launch_count()
            fn()
            launches[nm] = sige.sige_launch_count() - before
    stream.synchronize()
    n_tiles = int(d["cnt"].item())

    def whole_step():
        for fn in calls.values():
            fn()
    step_graph = {"step": capture(whole_step, stream)}
    tcalls = two_launch_calls(d, stream)

    def whole_two():
        for fn in tcalls.values():
            fn()
    tgraph = {"two": capture(whole_two, stream)}
    graphs = {nm: capture(fn, stream) for nm, fn in tcalls.items()}
    ucalls = unfused_calls(d, stream)

    def whole_unfused():
        for fn in ucalls.values():
            fn()
    ugraph = {"unfused": capture(whole_unfused, stream)}
    ugraphs = {nm: capture(fn, stream) for nm, fn in ucalls.items()}
    dgraphs = {nm: capture(fn, stream) for nm, fn in dense_calls(d, stream).items()}
    flush = L2Flush(dev)
    stream.synchronize()

    # warm-up steps
    timed_graph_steps(step_graph, flush, args.warmup, stream)

    def barrier():
        if ws > 1:
            torch.distributed.barrier()
    sampler = ClockSampler(dev.index)
    sampler.begin()
    barrier()
    torch.cuda.synchronize()
    _, tot = timed_graph_steps(step_graph, flush, args.steps, stream)
    torch.cuda.synchronize()
    barrier()
    clocks = sampler.stop()
    step_ms = float(np.mean(tot))
    # the step as two launches, and each of them in a graph of its own (so
    # each number also carries one graph launch), same L2 flush before every step
    nu = max(10, min(args.steps, 200))
    timed_graph_steps(tgraph, flush, 3, stream)
    _, ttot = timed_graph_steps(tgraph, flush, nu, stream)
    two_ms = float(np.mean(ttot))
    timed_graph_steps(graphs, flush, 3, stream)
    per, _ = timed_graph_steps(graphs, flush, nu, stream)
    kern_ms = {nm: float(np.mean(v)) for nm, v in per.items()}
    # the same step with the layers as separate launches
    timed_graph_steps(ugraph, flush, 3, stream)
    _, utot = timed_graph_steps(ugraph, flush, nu, stream)
    uper, _ = timed_graph_steps(ugraphs, flush, nu, stream)
    unfused_ms = float(np.mean(utot))
    ukern_ms = {nm: float(np.mean(v)) for nm, v in uper.items()}
    red = max_over_ranks([step_ms, unfused_ms, two_ms] + [kern_ms[k] for k in kern_ms], dev)
    step_ms, unfused_ms, two_ms = red[0], red[1], red[2]
    kern_ms = {k: red[i + 3] for i, k in enumerate(kern_ms)}

    # dense comparison (same launch mode, L2 flushed)
    dper, dtot = timed_graph_steps(dgraphs, flush, max(10, min(args.steps, 50)), stream)
    dense_ms = {nm: float(np.mean(v)) for nm, v in dper.items()}

    # end to end through the public API: the pinned host input goes up whole
    # (the device finds the edit), the step runs, and the host copy of the
    # output (current before the edit: one full copy, untimed) takes the
    # step's tiles back through sige_download_tiles, which returns once the
    # host tensor is complete
    host_in = d["x_edit"].cpu().pin_memory()
    host_out = d["out"].cpu().pin_memory()
    dev_in = torch.empty_like(d["x_edit"])
    d_e2e = dict(d, x_edit=dev_in)
    ecalls = step_calls(d_e2e, stream)
    dl_bytes = sige.sige_download_tiles_bytes(d["out"], BLOCK, d["cap"])
    dl_dev = torch.empty(dl_bytes, dtype=torch.uint8, device=dev)
    dl_host = torch.empty(dl_bytes, dtype=torch.uint8).pin_memory()
    e2e_times = []
    for k in range(args.warmup + args.e2e_steps):
        with torch.cuda.stream(stream):
            flush()
            stream.synchronize()
            t0 = time.perf_counter()
            dev_in.copy_(host_in, non_blocking=True)
            for fn in ecalls.values():
                fn()
            sige.sige_download_tiles(d["out"], BLOCK, d["idx"], d["cnt"], d["cap"], host_out, staging=dl_dev,
                                     host_staging=dl_host, stream=stream)
            t1 = time.perf_counter()
        if k >= args.warmup:
            e2e_times.append((t1 - t0) * 1e3)
    e2e_ms = float(np.mean(e2e_times))
    e2e_ms = max_over_ranks([e2e_ms], dev)[0]
    out_ok = bool(torch.equal(host_out, d["out"].cpu()))
    tile_bytes = d["out"].shape[0] * BLOCK * BLOCK * d["out"].shape[3] * d["out"].element_size()
    e2e_d2h = 16 + 8 * d["cap"] + n_tiles * tile_bytes

    # roofline of the step's one kernel: the two inputs streamed once, the
    # list, y1 and out written at the tiles, the weights read once; the convs'
    # MACs on the tiles.  It is bound by the bytes.
    flops, nbytes = step_work(n_tiles)
    t_tc = flops / (peaks["bf16_tflops"] * 1e12)
    t_bw = nbytes / (peaks["hbm_gbs"] * 1e9)
    if t_bw >= t_tc:
        ach = nbytes / (step_ms * 1e-3) / 1e9
        roof = {"bound": "hbm", "achieved": ach, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": ach / peaks["hbm_gbs"], "peak_source": f"{peaks['source']} hbm_gbs"}
    else:
        ach = flops / (step_ms * 1e-3) / 1e12
        roof = {"bound": "tensor", "achieved": ach, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                "frac": ach / peaks["bf16_tflops"], "peak_source": f"{peaks['source']} bf16_tflops (burst)"}
    roof.update(traffic=ncu_traffic("k_resblock_step"), kernel="k_resblock<step>", algorithmic_bytes=nbytes,
                algorithmic_flops=flops, duration_us=step_ms * 1e3,
                tensor_frac=(flops / (step_ms * 1e-3) / 1e12) / peaks["bf16_tflops"])
    # the fused res block of the two-launch step against its own roofline
    f_rb, b_rb = resblock_work(n_tiles)
    t_rb = max(f_rb / (peaks["bf16_tflops"] * 1e12), b_rb / (peaks["hbm_gbs"] * 1e9))
    resblock_roof = {"kernel": "k_resblock", "roof_us": t_rb * 1e6, "us": kern_ms["resblock"] * 1e3,
                     "frac": t_rb / (kern_ms["resblock"] * 1e-3)}
    t_roof = max(t_tc, t_bw)
    sparse_conv_ms = kern_ms["resblock"]
    dense_conv_ms = dense_ms["dense1"] + dense_ms["dense2"]
    # the dense conv of the layer (GroupNorm + SiLU in, bias out) against the
    # tensor roofline: 2 * 256 * 256 * 128 * 128 * 9 FLOPs per conv
    dflops = 2.0 * H * W * C * C * 9
    dense_roof = {"flops_per_conv": dflops, "us": {k: v * 1e3 for k, v in dense_ms.items()},
                  "tflops": {k: dflops / (v * 1e-3) / 1e12 for k, v in dense_ms.items()},
                  "frac": {k: dflops / (v * 1e-3) / 1e12 / peaks["bf16_tflops"] for k, v in dense_ms.items()},
                  "peak_tflops": peaks["bf16_tflops"], "peak_source": f"{peaks['source']} bf16_tflops (burst)",
                  "l2": "cold (flushed before every call)"}

    extras = None
    if not args.no_extras:
        extras = measure_extras(dev, flush, stream, peaks, args.seed + rank, step_graph["step"])

    cpu = None
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        cores = host_cores()
        t_build = time.perf_counter()
        orc_step = OracleStep(args.seed, cores)
        t_build = time.perf_counter() - t_build
        orc_step.time_steps(1)
        ts, t_start = [], time.perf_counter()
        while time.perf_counter() - t_start < args.cpu_seconds or len(ts) < 3:
            ts += orc_step.time_steps(1)
        dense_ts = orc_step.time_steps(2, dense=True)
        orc_step.set_threads(1)
        one_ts = orc_step.time_steps(2)
        orc_step.set_threads(cores)
        cpu = {"value": float(np.mean(ts)) * 1e6, "unit": "us", "cores": cores, "kind": "oracle",
               "sample": f"{len(ts)} whole steps on the full 256x256 workload (pixel mask + tile list, both "
                         f"tile-restricted sparse convs of the res block) in {sum(ts):.1f} s on {cores} threads; "
                         f"caches and GroupNorm statistics of the original built once by the oracle "
                         f"({t_build:.1f} s, untimed)",
               "one_core_us": float(np.mean(one_ts)) * 1e6,
               "dense_definition_us": float(np.mean(dense_ts)) * 1e6,
               "dense_definition": "the oracle as defined: both layers dense over the image in double, then "
                                   "the listed tiles copied into the caches (2 steps, all threads)"}

    line = {
        "metric": METRIC, "value": step_ms * 1e3, "unit": "us", "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": step_ms, "higher_is_better": False, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": WORKLOAD, "H": H, "W": W, "C": C, "block": BLOCK, "edit_area": 0.012,
                   "active_tiles": n_tiles, "tile_fraction": n_tiles / d["cap"],
                   "l2": "cold: 256 MiB write then 256 MiB read (clean lines) before every step, untimed", "launch": "one CUDA graph per step holding the one-launch step kernel; breakdown_us: the two-launch form, one graph per call",
                   "parallelism": f"replicas x{ws}" if ws > 1 else "single GPU"},
        "step_p50_us": float(np.median(tot)) * 1e3, "step_p90_us": float(np.percentile(tot, 90)) * 1e3,
        "two_launch_step_us": two_ms * 1e3,
        "breakdown_us": {k: v * 1e3 for k, v in kern_ms.items()},
        "resblock_roofline": resblock_roof,
        "unfused_step_us": unfused_ms * 1e3,
        "unfused_breakdown_us": {k: v * 1e3 for k, v in ukern_ms.items()},
        "dense_conv_us": dense_conv_ms * 1e3, "dense_conv_roofline": dense_roof,
        "sparse_conv_us": sparse_conv_ms * 1e3,
        "speedup_vs_dense_conv": dense_conv_ms / sparse_conv_ms,
        "step_roofline_frac": t_roof / (step_ms * 1e-3),
        "roofline": roof,
        "cpu_baseline": cpu,
        "e2e": {"value": e2e_ms * 1e3, "unit": "us", "h2d_bytes_per_step": host_in.numel() * host_in.element_size(),
                "d2h_bytes_per_step": e2e_d2h,
                "api": "H2D of the edited input, sige_resblock_step, sige_download_tiles into the host copy of "
                       "the output (the list, then the step's tiles); host wall clock per step, pinned buffers",
                "host_output_matches_device": out_ok},
        "gpu_launches": sum(launches.values()) * args.steps,
        "clocks": clocks,
        "conv_path": "tcgen05" if sige.sige_conv_path(d["cd"], torch.bfloat16) == 1 else "cuda-core",
    }
    if extras is not None:
        line.update(extras)
    if rank == 0:
        print(json.dumps(line), flush=True)
    for gd in (graphs, dgraphs, step_graph, ugraph, ugraphs, tgraph):
        gd.clear()
    if ws > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["sige", "reference"], default="sige")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--e2e-steps", type=int, default=50)
    ap.add_argument("--cpu-seconds", type=float, default=8.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the area sweep, warm-L2 step and per-layer rows")
    ap.add_argument("--row", choices=["attention", "gather_scatter", "mask", "layers"],
                    help="time one component alone on one GPU and print its JSON (no headline line); "
                         "a small, self-contained run for profiling")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.row:
        return run_row(args)
    if args.impl == "reference":
        return run_reference(args)
    return run_sige(args)


def run_row(args):
    """One component of the extras, alone: the SD-latent attention step, the
    unfused gather and scatter, or the mask reduction (its own graph, L2
    flushed before each launch)."""
    dev = torch.device("cuda", torch.cuda.current_device())
    torch.cuda.set_device(dev)
    peaks = load_peaks()
    stream = torch.cuda.Stream(device=dev)
    flush = L2Flush(dev)
    with torch.cuda.stream(stream):
        if args.row == "attention":
            r = attention_timing(args.seed, dev, flush, stream, peaks, reps=max(3, args.steps))
        elif args.row == "layers":
            r = {"layers": layer_rows(args.seed, dev, flush, stream, peaks, reps=max(3, args.steps))}
        elif args.row == "gather_scatter":
            r = gather_scatter_timing(args.seed, dev, flush, stream, peaks, reps=max(3, args.steps))
        else:
            d = make_workload(args.seed, dev)
            g = capture(two_launch_calls(d, stream)["mask"], stream)
            t = time_graph(g, flush, max(3, args.steps), stream)
            us = float(np.median(t)) * 1e3
            nbytes = 2 * d["x_orig"].numel() * d["x_orig"].element_size()
            r = {"mask_us": us, "bytes": nbytes, "gbs": nbytes / (us * 1e-6) / 1e9,
                 "frac": nbytes / (us * 1e-6) / 1e9 / peaks["hbm_gbs"], "note": "graph time, launch included"}
    print(json.dumps({"row": args.row, **r}))
    return 0


if __name__ == "__main__":
    sys.exit(main())
