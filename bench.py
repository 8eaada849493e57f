#!/usr/bin/env python
"""Benchmark of the tile-binned differentiable Gaussian splatting rasterizer.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl native|reference]

One step = one training frame through the whole hot path for one camera:
project -> bin and sort -> forward blend -> L1 loss gradient -> backward blend
-> projection backward (gs_train_step, the `train_step` of the line, takes
the L1 loss in the forward's epilogue).  Default workload: a seeded synthetic 400k-Gaussian
scene (120 anisotropic clusters in a 10 m box, log-scales N(-4, 0.6), opacity
logits N(1, 1.5)) seen from 16 ring cameras at 980 x 545, f = 1000, L1 loss
against a seeded U(0, 1) target.  Inputs are resident in HBM; L2 (126 MB) is
flushed between timed steps by writing a 256 MB buffer outside the timed
events.  Each camera's step is captured once as a CUDA graph and replayed
(--no-graphs launches eagerly); per-kernel times for the roofline come from an
eager pass over the same steps with CUDA events around every launch.  Each
rank renders its own cameras (independent frames, no data-path
collective); the reported value is all frames over the slowest rank's device
time.  Prints one JSON line (rank 0).

--impl reference times the CPU oracle (double precision, every host core) on
a bounded sample of the same workload: full projection and brute-force
binning, the blend and its backward on a seeded sample of tiles, the frame
time extrapolated by tile count.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from scenes import SPECS, make_cameras, make_scene, make_target  # noqa: E402

TIGHT_TILES = 1  # gs_camera.flags bit of the opacity-aware tile cut (GS_FLAG_TIGHT_TILES)

DEFAULT_WORKLOAD = "train400k_half"
METRIC = "fwd and fwd+bwd frames/s at 400k Gaussians, 980x545; tile-pairs/s; % roofline"

# Algorithmic FP32-pipe operations per (pixel, list entry) evaluation,
# counted from the written formulas with a fused multiply-add as one
# operation (per-entry work done once per tile, such as the conic scaling,
# is not counted):
#   visited entry (forward and backward): dx, dy (2); sigma from the half
#     conic in FMA form (5); scale for exp (1); o G (1); min with 0.99 (1);
#     sigma < 0 test (1); alpha < 1/255 test (1)                      = 12
#   added entry, forward extra: T (1 - alpha) as one FMA (1); stop test (1);
#     w = alpha T (1); colour accumulation (3)                         = 6
#   added entry, backward extra: 1 - alpha (1); T_i = T r (1); w (1);
#     colour gradients w g (3); c - R (3); <c - R, g> (3); dL/dalpha (1);
#     R update (3); cap select (1); v = dL/dalpha alpha (1); the five
#     geometric products v dx, v dy, v dx^2, v dx dy, v dy^2 (5); the nine
#     per-Gaussian sums over pixels (9)                                = 32
# plus one MUFU ex2 per visit (and one rcp per backward addition).
OPS_VISIT = 12
OPS_FWD_ADD = 6
OPS_BWD_ADD = 32
# A per-evaluation estimate charges every visited entry the whole
# evaluation (forward about 21 FP32-pipe instructions, backward about 50),
# whether or not the entry passes the alpha test; reported beside the split
# above, which charges the add path only to the entries that take it.
OPS_EVAL_FWD = 21
OPS_EVAL_BWD = 50

# Algorithmic HBM bytes of the streaming stages (per Gaussian G, pair P):
#   project      56 B/G raw parameters read + 68 B/G records written
#   bin_count    16 B/G rectangles read (the count matrix is 4 B per CTA and
#                tile, small beside them)
#   emit         16 B/G rectangle + 16 B/G depth record read, 8 B/P keys written
#   tile_sort    8 B/P keys read, 8 B/P (id, tile) written
#   project_bwd  56 B/G raw parameters + 48 B/G 2D sums + 32 B/G records read,
#                48 B/G 2D gradients + 56 B/G raw gradients written
BYTES = {
    "project": lambda G, P: 124 * G,
    "bin_count": lambda G, P: 16 * G,
    "emit": lambda G, P: 32 * G + 8 * P,
    "tile_sort": lambda G, P: 16 * P,
    "project_bwd": lambda G, P: 240 * G,
}
# The same stages on the global binning path (GS_BIN_GLOBAL):
#   depth_sort   16 B/G rectangle + 16 B/G depth record read, 8 B/G keys written;
#                four passes of 4 B/G digit counts read + 8 B/G read, 8 B/G written
#   emit         rank sums and offsets: 2 x (4 B/G order + 16 B/G rectangle)
#                read, 4 B/G offsets written; the emit: 24 B/G read, 8 B/P written
#   tile_sort    per pass over the tile id's 8-bit digits: 4 B/P counts read,
#                8 B/P read and 8 B/P written
BYTES_GLOBAL = {
    "depth_sort": lambda G, P, tile_passes: 40 * G + 4 * 20 * G,
    "emit": lambda G, P, tile_passes: 68 * G + 8 * P,
    "tile_sort": lambda G, P, tile_passes: tile_passes * 20 * P,
}
ALU_KERNELS = ("render_fwd", "render_bwd")

# DRAM traffic per launch of render_bwd measured by ncu
# (dram__bytes_read.sum + dram__bytes_write.sum), valid only for the kernel
# source it was taken on.
# Taken on one frame of this workload (camera 0, 644,012 pairs): 42.42 MB
# read + 0.17 MB written; scaled to a launch by its pair count.
TRAFFIC = {"render_bwd": {"src_sha": "1babb3619e314df6", "bytes_per_pair": 66.13}}


def _binning_used(choice, max_pairs, spec) -> str:
    """The strategy gs_bin_and_sort takes (the automatic rule of include/gs.h)."""
    if choice != "auto":
        return choice
    tiles = ((spec.width + 15) // 16) * ((spec.height + 15) // 16)
    return "auto: " + ("global" if max_pairs >= 1024 * tiles and spec.n <= max_pairs else "per-tile")


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured", float(d.get("sm_max_mhz", 1965.0))
    except Exception:
        return 6650.0, "fallback", 1965.0


def _cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


def _src_sha(name):
    p = os.path.join(ROOT, "gaussian_splatting_differentiable_tile_b200", "csrc", name)
    return hashlib.sha256(open(p, "rb").read()).hexdigest()[:16]


class ClockSampler:
    """nvidia-smi samples every 200 ms while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_id: str | None):
        self.samples = []
        self.proc = None
        cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "200"]
        if device_id:
            cmd += ["-i", device_id]
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 9:
                self.samples.append(parts)

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm = [float(s[1]) for s in self.samples if s[1].replace(".", "").isdigit()]
        mx = [float(s[2]) for s in self.samples if s[2].replace(".", "").isdigit()]
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        reasons = sorted({names[k] for s in self.samples for k in range(4) if s[5 + k].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(self.samples)}


# ------------------------------------------------------------------ CPU side
def cpu_frame_time(params_np, cam, sample_tiles: int, seed: int = 0, bin_fraction: float = 1.0) -> dict:
    """The oracle, as it stands, on one frame: full projection, binning
    (brute force over every (Gaussian, tile) pair, so its time is linear in
    the Gaussians binned: with bin_fraction < 1 a seeded subset is binned and
    the time scaled up), blend and backward on `sample_tiles` seeded tiles,
    projection backward; returns the extrapolated seconds per frame."""
    import oracle as O

    tiles = cam.tiles
    mask = np.zeros(tiles, np.uint8)
    mask[np.random.default_rng(seed).choice(tiles, min(sample_tiles, tiles), replace=False)] = 1
    t = {}
    t0 = time.perf_counter()
    p = O.project(params_np, cam)
    t["project"] = time.perf_counter() - t0
    if bin_fraction < 1.0:
        n = p["rect"].shape[0]
        sub = np.sort(np.random.default_rng(seed + 2).choice(n, max(1, int(n * bin_fraction)), replace=False))
        t0 = time.perf_counter()
        O.bin_pairs(p["rect"][sub], p["valid"][sub], p["depth32"][sub], cam.width, cam.height)
        t["bin"] = (time.perf_counter() - t0) * n / len(sub)
    else:
        t0 = time.perf_counter()
        O.bin_pairs(p["rect"], p["valid"], p["depth32"], cam.width, cam.height)
        t["bin"] = time.perf_counter() - t0
    t0 = time.perf_counter()
    O.render(p, cam, tile_mask=mask)
    t["render_sample"] = time.perf_counter() - t0
    nc = O.channels(cam)
    dl = np.random.default_rng(seed + 1).normal(size=(cam.height, cam.width, nc)) / (nc * cam.pixels)
    t0 = time.perf_counter()
    g2, _ = O.render_bwd(p, cam, dl, tile_mask=mask)
    t["render_bwd_sample"] = time.perf_counter() - t0
    t0 = time.perf_counter()
    O.project_bwd(params_np, cam, g2)
    t["project_bwd"] = time.perf_counter() - t0
    scale = tiles / float(mask.sum())
    frame = t["project"] + t["bin"] + (t["render_sample"] + t["render_bwd_sample"]) * scale + t["project_bwd"]
    fwd = t["project"] + t["bin"] + t["render_sample"] * scale
    return {"frame_s": frame, "fwd_s": fwd, "parts": t, "sampled_tiles": int(mask.sum()), "tiles": tiles,
            "threads": O.default_threads()}


# gs_camera.flags bits of the pages' variants (GS_FLAG_* in include/gs.h)
VARIANT_FLAGS = {"3dgs": 0,
                 "gsplat": 4 | 16 | 32,           # inclusive stop test, per-axis opacity-aware radii
                 "gsplat-antialiased": 2 | 4 | 16 | 32,
                 "3dgs-depth": 64}                # a fourth channel: blended camera depth


# gs_bins.strategy (GS_BIN_* in include/gs.h): the same pairs either way
BINNING = {"auto": 0, "per-tile": 1, "global": 2}


def _cameras(spec, args):
    cams = make_cameras(spec)
    for c in cams:
        c.flags = (TIGHT_TILES if args.tiles == "cut" else 0) | VARIANT_FLAGS[args.variant]
    return cams


def run_reference(args, spec, rank, world):
    if rank != 0:
        return
    params = make_scene(spec)
    cams = _cameras(spec, args)
    frac = args.ref_bin_fraction
    for i in range(args.warmup):
        cpu_frame_time(params, cams[i % len(cams)], args.ref_sample_tiles, seed=i, bin_fraction=frac)
    times = []
    info = None
    wall0 = time.perf_counter()
    for i in range(args.steps):
        info = cpu_frame_time(params, cams[i % len(cams)], args.ref_sample_tiles, seed=100 + i, bin_fraction=frac)
        times.append(info["frame_s"])
    wall = time.perf_counter() - wall0
    fps = 1.0 / statistics.mean(times)
    sample = (f"per step one camera: full projection of {spec.n} Gaussians, brute-force binning of a seeded "
              f"{frac:g} of them (its time scaled by 1/{frac:g}: linear in the Gaussians binned), blend and "
              f"backward on {info['sampled_tiles']} of {info['tiles']} seeded tiles, frame time extrapolated "
              f"by tile count")
    out = {"impl": "reference", "metric": METRIC, "value": fps, "unit": "frames/s", "n_gpus": world,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000.0 * statistics.mean(times),
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
           "data": "synthetic", "config": _config(spec, None, args.tiles, False, args.variant),
           "cpu_baseline": {"value": fps, "unit": "frames/s", "cores": info["threads"], "cpu_model": _cpu_model(),
                            "kind": "oracle", "sample": sample},
           "e2e": {"value": fps, "unit": "frames/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
           # ms_per_step is the extrapolated time of a whole frame; the sampled
           # work this run actually did took wall_s
           "measured": {"wall_s": wall, "sampled_s_per_step": wall / max(1, args.steps),
                        "extrapolated_ms_per_step": 1000.0 * statistics.mean(times)}}
    print(json.dumps(out), flush=True)


def _config(spec, pairs, tiles, graphs=True, variant="3dgs", binning="auto"):
    return {"workload": spec.name, "n_gaussians": spec.n, "width": spec.width, "height": spec.height,
            "variant": variant,
            "focal": spec.focal, "cameras": f"{spec.n_cameras} {spec.cameras}", "pairs_per_frame": pairs,
            "tiles": ("3-sigma rectangle narrowed by the opacity-aware cut (same image)" if tiles == "cut"
                      else "3-sigma rectangle"),
            "l2": "flushed between timed steps (256 MB write outside the timed events)",
            "launch": "one CUDA graph per camera, replayed" if graphs else "eager launches",
            "binning": binning,
            "parallelism": "replicas (cameras split across ranks)"}


# ------------------------------------------------------------ rank logic
def my_cameras(cams, rank: int, world: int):
    """Replicas: rank r renders cameras r, r + world, ... (at least one, so
    that every rank takes the same collective steps)."""
    return [c for i, c in enumerate(cams) if i % world == rank] or cams[:1]


def max_over_ranks(values, world: int, device):
    """Elementwise max over ranks of per-rank timings (the whole job ends when
    the slowest rank does)."""
    import torch
    import torch.distributed as dist

    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


# ------------------------------------------------------------------ GPU side
def run_profile_frame(args, spec):
    """One eager frame (forward, L1 gradient, backward) of one camera for a
    profiler to capture: no sizing pass, no timing, about fifteen launches."""
    import torch

    import gaussian_splatting_differentiable_tile_b200 as G

    torch.cuda.set_device(0)
    params = {k: torch.from_numpy(v).cuda() for k, v in make_scene(spec).items()}
    cam = _cameras(spec, args)[args.profile_camera]
    # the pair list sized as the timed bench sizes it (1.05 K + 4096, so the
    # automatic binning strategy takes the same path), from a sizing call;
    # the profiled frame is the NVTX range "frame" (ncu --nvtx --nvtx-include frame/)
    r = G.Rasterizer(spec.n, spec.width, spec.height, strategy=BINNING[args.binning])
    G.gs_project(cam, params, r.proj)
    try:
        K = G.gs_bin_and_sort(cam, spec.n, r.proj, r.bins)
    except G.GSError as e:
        if e.code != G.GS_ERR_CAPACITY:
            raise
        K = e.n_pairs
    r.bins = G.Bins(spec.n, int(K * 1.05) + 4096, spec.width, spec.height, strategy=BINNING[args.binning])
    torch.cuda.synchronize()
    target = torch.from_numpy(make_target(spec.width, spec.height, channels=G.channels(cam))).cuda()
    r.image = torch.empty(tuple(target.shape), device="cuda")
    dl = torch.empty_like(r.image)
    loss = torch.zeros(1, device="cuda")
    torch.cuda.synchronize()
    # the bench's step: project, bin, forward, L1 loss, backward
    torch.cuda.nvtx.range_push("frame")
    G.gs_project(cam, params, r.proj)
    G.gs_bin_and_sort(cam, spec.n, r.proj, r.bins, sync=False)
    G.gs_render_fwd(cam, spec.n, r.proj, r.bins, r.image, r.T_final, r.last)
    G.gs_l1_loss_grad(r.image, target, dl, loss)
    r.backward(cam, params, dl)
    torch.cuda.nvtx.range_pop()
    torch.cuda.synchronize()
    print(json.dumps({"profile_frame": spec.name, "camera": args.profile_camera, "tiles": args.tiles,
                      "pairs": K, "binning": _binning_used(args.binning, r.bins.max_pairs, spec),
                      "loss": loss.item()}), flush=True)


def run_profile_train(args, spec):
    """One eager batched training step (4 cameras on 4 lanes, Adam) for a
    profiler to capture, in the NVTX range "train_step" (after a sizing pass
    and one warm-up step outside it)."""
    import torch

    import gaussian_splatting_differentiable_tile_b200 as G

    torch.cuda.set_device(0)
    params = {k: torch.from_numpy(v).cuda() for k, v in make_scene(spec).items()}
    cams = _cameras(spec, args)[:4]
    nc = G.channels(cams[0])
    tr = G.Trainer(spec.n, spec.width, spec.height, lanes=4, channels=nc)
    need = tr.fit_pairs(cams, params)
    tgt = torch.stack([torch.from_numpy(make_target(spec.width, spec.height, seed=i, channels=nc)).cuda()
                       for i in range(len(cams))])
    tr.step(cams, params, tgt)  # warm-up
    torch.cuda.synchronize()
    torch.cuda.nvtx.range_push("train_step")
    tr.step(cams, params, tgt)
    torch.cuda.nvtx.range_pop()
    torch.cuda.synchronize()
    print(json.dumps({"profile_train": spec.name, "cameras": len(cams), "lanes": 4, "max_pairs": need}),
          flush=True)


def run_native(args, spec, rank, world, local):
    import torch
    import torch.distributed as dist

    import gaussian_splatting_differentiable_tile_b200 as G

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    params_np = make_scene(spec)
    cams = _cameras(spec, args)
    mine = my_cameras(cams, rank, world)
    n = spec.n
    P = {k: torch.from_numpy(v).to(dev) for k, v in params_np.items()}
    nc = G.channels(cams[0])
    targets = [torch.from_numpy(make_target(spec.width, spec.height, seed=i, channels=nc)).to(dev)
               for i in range(len(mine))]
    ccams = [G.make_camera(c) for c in mine]

    # size the pair list from the cameras this rank renders
    r = G.Rasterizer(n, spec.width, spec.height, max_pairs=24 * n, device=dev)
    pairs, stats = [], []
    for c in mine:
        r.forward(c, P, sync=True)
        pairs.append(r.n_pairs)
        stats.append(G.gs_render_stats(c, n, r.proj, r.bins, r.last))
    bins = G.Bins(n, int(max(pairs) * 1.05) + 4096, spec.width, spec.height, device=dev,
                  strategy=BINNING[args.binning])
    proj = r.proj
    H, W = spec.height, spec.width
    image = torch.empty((H, W, nc), device=dev)
    T = torch.empty((H, W), device=dev)
    last = torch.empty((H, W), dtype=torch.int32, device=dev)
    dl = torch.empty_like(image)
    loss = torch.zeros(1, device=dev)
    grad2d = torch.empty((n, 12), device=dev)
    grads = {k: torch.empty_like(v) for k, v in P.items()}
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)

    def step_fwd(i):
        c = ccams[i % len(ccams)]
        G.gs_project(c, P, proj)
        G.gs_bin_and_sort(c, n, proj, bins, sync=False)
        G.gs_render_fwd(c, n, proj, bins, image, T, last)

    def step_full(i, params=P, tgt=None):
        c = ccams[i % len(ccams)]
        G.gs_project(c, params, proj)
        G.gs_bin_and_sort(c, n, proj, bins, sync=False)
        G.gs_render_fwd(c, n, proj, bins, image, T, last)
        G.gs_l1_loss_grad(image, targets[i % len(targets)] if tgt is None else tgt, dl, loss)
        G.gs_render_bwd(c, n, params, proj, bins, T, last, dl, grad2d, grads)

    def barrier():
        if world > 1:
            dist.barrier()

    def timed(fn, steps, warmup, profile=False):
        for i in range(warmup):
            fn(i)
        torch.cuda.synchronize()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        barrier()
        torch.cuda.synchronize()
        if profile:
            G.profile_begin(1 << 16)
        for i in range(steps):
            flush.zero_()
            ev[i][0].record()
            fn(i)
            ev[i][1].record()
        torch.cuda.synchronize()
        prof = G.profile_end() if profile else None
        barrier()
        ms = sum(a.elapsed_time(b) for a, b in ev)
        return ms, prof

    def graphed(fn, count):
        """One CUDA graph per camera of this rank: the step's launches replay
        without host work or per-launch gaps."""
        if args.no_graphs:
            return fn
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            for i in range(count):
                fn(i)
        torch.cuda.current_stream().wait_stream(side)
        graphs = []
        for i in range(count):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                fn(i)
            graphs.append(g)
        torch.cuda.synchronize()
        return lambda i: graphs[i % count].replay()

    device_id = None
    try:
        device_id = "GPU-" + str(torch.cuda.get_device_properties(local).uuid)
    except Exception:
        device_id = str(local)
    # per-kernel times (CUDA events around every launch), eager launches
    _, prof = timed(step_full, args.steps, args.warmup, profile=True)
    # the timed region: whole steps
    g_full = graphed(step_full, len(ccams))
    g_fwd = graphed(step_fwd, len(ccams))
    sampler = ClockSampler(device_id)
    full_ms, _ = timed(g_full, args.steps, args.warmup)
    clocks = sampler.stop()
    fwd_ms, _ = timed(g_fwd, args.steps, args.warmup)

    # end to end through the public API with host buffers: every step copies
    # its inputs (raw parameters, target) from pinned host memory and its
    # result (raw gradients, loss) back.  Steps are pipelined over three
    # streams and two buffer slots, so step i's copies overlap the work of
    # steps i - 1 and i + 1; the timed region spans all steps on the device.
    # each side's tensors live in one buffer (256-byte aligned views), so a
    # step is one copy in and one copy out
    def layout(shapes):
        offs, off = {}, 0
        for k, shp in shapes.items():
            offs[k] = off
            off += (int(np.prod(shp)) * 4 + 255) // 256 * 256
        return offs, off

    def views(buf, offs, shapes):
        return {k: buf[offs[k]:offs[k] + int(np.prod(shp)) * 4].view(torch.float32).view(shp)
                for k, shp in shapes.items()}

    in_shapes = {k: tuple(v.shape) for k, v in params_np.items()}
    in_shapes["target"] = tuple(targets[0].shape)
    in_offs, in_bytes = layout(in_shapes)
    out_shapes = {k: tuple(v.shape) for k, v in params_np.items()}
    out_shapes["loss"] = (1,)
    out_offs, out_bytes = layout(out_shapes)
    slots = 2
    host_in = [torch.empty(in_bytes, dtype=torch.uint8).pin_memory() for _ in range(len(targets))]
    for j, hb in enumerate(host_in):  # the camera's step inputs: parameters and its target
        hv = views(hb, in_offs, in_shapes)
        for k, v in params_np.items():
            hv[k].copy_(torch.from_numpy(v))
        hv["target"].copy_(targets[j].cpu())
    dev_inb = [torch.empty(in_bytes, dtype=torch.uint8, device=dev) for _ in range(slots)]
    dev_outb = [torch.empty(out_bytes, dtype=torch.uint8, device=dev) for _ in range(slots)]
    host_out = [torch.empty(out_bytes, dtype=torch.uint8).pin_memory() for _ in range(slots)]
    dev_in = [views(b, in_offs, in_shapes) for b in dev_inb]
    dev_o = [views(b, out_offs, out_shapes) for b in dev_outb]
    dev_tgt = [d.pop("target") for d in dev_in]
    dev_loss = [d.pop("loss") for d in dev_o]
    dev_grads = dev_o
    s_in, s_cmp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(slots)]   # the slot's inputs are on the device
    ev_cmp = [torch.cuda.Event() for _ in range(slots)]  # the slot's step is computed
    ev_out = [torch.cuda.Event() for _ in range(slots)]  # the slot's gradients are on the host

    def step_e2e(i):
        k = i % slots
        c = ccams[i % len(ccams)]
        with torch.cuda.stream(s_in):
            s_in.wait_event(ev_cmp[k])  # step i - 2 no longer reads the slot
            dev_inb[k].copy_(host_in[i % len(host_in)], non_blocking=True)
            ev_in[k].record(s_in)
        with torch.cuda.stream(s_cmp):
            s_cmp.wait_event(ev_in[k])
            s_cmp.wait_event(ev_out[k])  # step i - 2's gradients have left the slot
            flush.zero_()
            G.gs_project(c, dev_in[k], proj)
            G.gs_bin_and_sort(c, n, proj, bins, sync=False)
            G.gs_render_fwd(c, n, proj, bins, image, T, last)
            G.gs_l1_loss_grad(image, dev_tgt[k], dl, dev_loss[k])
            G.gs_render_bwd(c, n, dev_in[k], proj, bins, T, last, dl, grad2d, dev_grads[k])
            ev_cmp[k].record(s_cmp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_cmp[k])
            host_out[k].copy_(dev_outb[k], non_blocking=True)
            ev_out[k].record(s_out)

    for i in range(args.warmup):
        step_e2e(i)
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    e_start, e_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e_start.record(s_in)
    for i in range(args.steps):
        step_e2e(args.warmup + i)
    for st in (s_in, s_cmp, s_out):
        torch.cuda.current_stream().wait_stream(st)
    e_end.record()
    torch.cuda.synchronize()
    barrier()
    e2e_ms = e_start.elapsed_time(e_end)
    h2d = in_bytes
    d2h = out_bytes

    # the batched training step: B cameras per gs_train_step (lanes run
    # concurrently), then Adam on the mean gradient; one graph per camera group
    train = None
    if args.train_cams > 0:
        B = min(args.train_cams, len(mine))
        groups = [[(g * B + j) % len(mine) for j in range(B)] for g in range(max(1, len(mine) // B))]
        tr = G.Trainer(n, W, H, lanes=args.lanes, channels=nc, max_pairs=int(max(pairs) * 1.05) + 4096,
                       device=dev)
        Pt = {k: v.clone() for k, v in P.items()}  # Adam moves these, not the frames' parameters
        tcams = [[mine[j] for j in grp] for grp in groups]
        ttg = [torch.stack([targets[j] for j in grp]) for grp in groups]

        def step_train(i):
            tr.step(tcams[i % len(groups)], Pt, ttg[i % len(groups)])

        t_steps = max(1, args.steps // B)
        _, tprof = timed(step_train, t_steps, args.warmup, profile=True)
        # with several ranks the step all-reduces the gradient (data parallel)
        # and runs eagerly: no NCCL call inside a captured graph
        g_train = graphed(step_train, len(groups)) if world == 1 else step_train
        train_ms, _ = timed(g_train, t_steps, args.warmup)
        st = tr.cam_stats.cpu()
        if int(st[:, 0].abs().max()) != 0:
            raise RuntimeError(f"training step: pair list overflow {st.tolist()}")
        train = {"cameras_per_step": B, "lanes": args.lanes, "steps": t_steps, "ms": train_ms, "prof": tprof,
                 "slots": min(args.lanes, B) if world == 1 else 1}
    else:
        train_ms = 0.0

    # feature channels: F per-Gaussian values blended with the forward's
    # weights and their backward, per frame after that camera's forward
    feat = None
    if args.features > 0:
        F = args.features
        fts = torch.from_numpy(np.random.default_rng(5).uniform(-1, 1, (n, F)).astype(np.float32)).to(dev)
        fout = torch.empty((H, W, F), device=dev)
        fdl = torch.from_numpy(np.random.default_rng(6).normal(size=(H, W, F)).astype(np.float32) / (H * W * F)).to(dev)
        dfts = torch.empty_like(fts)
        f_fwd = f_bwd = 0.0
        f_steps = max(1, args.steps // 4)
        for i in range(args.warmup + f_steps):
            step_full(i)
            c = ccams[i % len(ccams)]
            e0, e1, e2 = (torch.cuda.Event(enable_timing=True) for _ in range(3))
            flush.zero_()
            e0.record()
            G.gs_render_features_fwd(c, n, proj, bins, fts, fout)
            e1.record()
            G.gs_render_features_bwd(c, n, P, proj, bins, T, last, fts, fdl, grad2d, dfts, grads)
            e2.record()
            torch.cuda.synchronize()
            if i >= args.warmup:
                f_fwd += e0.elapsed_time(e1)
                f_bwd += e1.elapsed_time(e2)
        feat = {"F": F, "frames": f_steps, "fwd_ms": f_fwd, "bwd_ms": f_bwd}
    feat_fwd_ms = feat["fwd_ms"] if feat else 0.0
    feat_bwd_ms = feat["bwd_ms"] if feat else 0.0

    full_ms, fwd_ms, e2e_ms, train_ms, feat_fwd_ms, feat_bwd_ms = max_over_ranks(
        [full_ms, fwd_ms, e2e_ms, train_ms, feat_fwd_ms, feat_bwd_ms], world, dev)
    frames = args.steps * world
    if rank != 0:
        return

    hbm_peak, peak_kind, sm_max = _peaks()
    sms = torch.cuda.get_device_properties(local).multi_processor_count
    clock_mhz = clocks["sm_max_mhz"] or sm_max
    alu_peak = sms * 128 * clock_mhz * 1e6 / 1e12  # T FP32 lane-ops/s
    # the same peak at the median SM clock sampled during the timed region
    alu_peak_sampled = sms * 128 * (clocks["sm_mhz"] or clock_mhz) * 1e6 / 1e12
    # work per timed step (cameras cycle through `mine`)
    sel = [i % len(mine) for i in range(args.steps)]
    pairs_steps = [pairs[i] for i in sel]
    fwd_visits = sum(stats[i]["fwd_visits"] for i in sel)
    bwd_visits = sum(stats[i]["bwd_visits"] for i in sel)
    contributions = sum(stats[i]["contributions"] for i in sel)
    fwd_ops = OPS_VISIT * fwd_visits + OPS_FWD_ADD * contributions
    bwd_ops = OPS_VISIT * bwd_visits + OPS_BWD_ADD * contributions
    work = {"steps": args.steps, "fwd_visits": fwd_visits, "bwd_visits": bwd_visits,
            "contributions": contributions,
            "ops": {"visit": OPS_VISIT, "fwd_add": OPS_FWD_ADD, "bwd_add": OPS_BWD_ADD},
            "fwd_ops": fwd_ops, "bwd_ops": bwd_ops,
            "formula": "fwd_ops = visit*fwd_visits + fwd_add*contributions; "
                       "bwd_ops = visit*bwd_visits + bwd_add*contributions; achieved = ops / summed kernel ms"}
    stages = {}
    gpu_launches = 0
    for name, (launches, ms) in (prof or {}).items():
        gpu_launches += launches
        entry = {"launches": launches, "ms_total": ms, "ms_per_step": ms / args.steps}
        global_path = "global" in _binning_used(args.binning, bins.max_pairs, spec)
        tiles_n = ((spec.width + 15) // 16) * ((spec.height + 15) // 16)
        tile_passes = 1 if tiles_n <= 256 else (2 if tiles_n <= 65536 else 3)
        if global_path and name in BYTES_GLOBAL:
            per_step = [BYTES_GLOBAL[name](n, pairs[i], tile_passes) for i in sel]
            total_bytes = sum(per_step)
            ach = total_bytes / (ms * 1e-3) / 1e9
            entry.update(bound="hbm", achieved=ach, peak=hbm_peak, unit="GB/s", frac=ach / hbm_peak)
        elif name in BYTES:
            per_step = [BYTES[name](n, pairs[i]) for i in sel]
            total_bytes = sum(per_step)
            ach = total_bytes / (ms * 1e-3) / 1e9
            entry.update(bound="hbm", achieved=ach, peak=hbm_peak, unit="GB/s", frac=ach / hbm_peak)
        elif name in ALU_KERNELS:
            ops = fwd_ops if name == "render_fwd" else bwd_ops
            ach = ops / (ms * 1e-3) / 1e12
            entry.update(bound="alu", achieved=ach, peak=alu_peak, unit="Tops/s", frac=ach / alu_peak,
                         ops=ops, frac_at_sampled_clock=ach / alu_peak_sampled)
            # the same work counted with the per-evaluation constants (every
            # visit charged the whole forward or backward evaluation)
            whole = (OPS_EVAL_FWD * fwd_visits if name == "render_fwd" else OPS_EVAL_BWD * bwd_visits)
            entry["frac_whole_eval"] = whole / (ms * 1e-3) / 1e12 / alu_peak
        stages[name] = entry
    dom = max(stages, key=lambda k: stages[k]["ms_total"]) if stages else None
    roof = None
    if dom and "bound" in stages[dom]:
        s = stages[dom]
        tr = TRAFFIC.get(dom)
        traffic = None
        if tr and tr.get("src_sha") == _src_sha("gs_render.cu"):
            traffic = tr["bytes_per_pair"] * statistics.mean(pairs_steps)
        roof = {"kernel": dom, "bound": s["bound"], "achieved": s["achieved"], "peak": s["peak"],
                "unit": s["unit"], "frac": s["frac"], "traffic": traffic,
                "peak_basis": (f"{sms} SMs x 128 FP32 lanes x {clock_mhz:.0f} MHz (FMA = 1 op)"
                               if s["bound"] == "alu" else f"{peak_kind} HBM copy bandwidth")}
        if s["bound"] == "alu":
            roof.update(kernel_ms_total=s["ms_total"], work=work,
                        frac_at_sampled_clock=s["frac_at_sampled_clock"],
                        sampled_sm_mhz=clocks["sm_mhz"])
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        info = cpu_frame_time(params_np, mine[0], args.cpu_sample_tiles)
        cpu = {"value": 1.0 / info["frame_s"], "unit": "frames/s", "cores": info["threads"],
               "cpu_model": _cpu_model(), "kind": "oracle",
               "sample": (f"one camera: full projection and brute-force binning of {n} Gaussians, blend and "
                          f"backward on {info['sampled_tiles']} of {info['tiles']} seeded tiles, frame time "
                          f"extrapolated by tile count ({info['frame_s']:.1f} s/frame)"),
               "fwd_frames_per_s": 1.0 / info["fwd_s"]}
    mean_pairs = statistics.mean(pairs_steps)
    train_out = None
    if train is not None:
        B, t_steps = train["cameras_per_step"], train["steps"]
        train_out = {"frames_per_s": B * t_steps * world / (train_ms * 1e-3), "ms_per_step": train_ms / t_steps,
                     "cameras_per_step": B, "lanes": train["lanes"],
                     "step": ("gs_train_step: per camera project, bin, blend, L1, backward into the lane's "
                              "gradient slot; Adam on the mean gradient; one CUDA graph per camera group"
                              if world == 1 else
                              "data parallel: each rank's gs_train_step (no Adam) over its cameras, one NCCL "
                              "all-reduce of the mean gradient, gs_adam_step; eager launches")}
        ad = (train["prof"] or {}).get("adam")
        if ad:
            launches, ms = ad
            # per value: p, m, v and each slot read; p, m, v and the mean gradient written
            abytes = 14 * n * 4 * (3 + train["slots"] + 4)
            kernels_per_step = launches / t_steps
            ach = abytes * t_steps / (ms * 1e-3) / 1e9
            train_out["adam"] = {"ms_per_step": ms / t_steps, "kernels_per_step": kernels_per_step,
                                 "bound": "hbm", "achieved": ach, "peak": hbm_peak, "unit": "GB/s",
                                 "frac": ach / hbm_peak, "bytes_per_step": abytes}
    feat_out = None
    if feat is not None:
        fr = feat["frames"]
        feat_out = {"channels": feat["F"], "fwd_ms_per_frame": feat_fwd_ms / fr, "bwd_ms_per_frame": feat_bwd_ms / fr,
                    "fwd_bwd_frames_per_s": fr * world / ((feat_fwd_ms + feat_bwd_ms) * 1e-3),
                    "passes": (f"{feat['F'] // 8} blend pass{'es' if feat['F'] // 8 != 1 else ''} of eight channels"
                               f"{' and one of four' if feat['F'] % 8 else ''} each way (forward weights recomputed per "
                               "pass, no background); backward adds into the frame's raw-parameter gradients")}
    out = {
        "metric": METRIC,
        "value": frames / (full_ms * 1e-3),
        "unit": "frames/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": full_ms / args.steps,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f32",
        "data": "synthetic",
        "config": _config(spec, int(mean_pairs), args.tiles, not args.no_graphs, args.variant,
                          _binning_used(args.binning, bins.max_pairs, spec)),
        "fwd_frames_per_s": frames / (fwd_ms * 1e-3),
        "fwd_ms_per_frame": fwd_ms / args.steps,
        "tile_pairs_per_s": mean_pairs * frames / (fwd_ms * 1e-3),
        "tiles_per_gaussian": mean_pairs / max(1, n),
        "roofline": roof,
        "stages": stages,
        "cpu_baseline": cpu,
        "e2e": {"value": frames / (e2e_ms * 1e-3), "unit": "frames/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h,
                "pipeline": "copy-in, compute and copy-out streams, two buffer slots; L2 flushed every step"},
        "gpu_launches": gpu_launches,
        "clocks": clocks,
        "train_step": train_out,
        "features": feat_out,
    }
    print(json.dumps(out), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=32)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("native", "reference"), default="native")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(SPECS))
    ap.add_argument("--cpu-sample-tiles", type=int, default=48)
    ap.add_argument("--ref-sample-tiles", type=int, default=8)
    ap.add_argument("--ref-bin-fraction", type=float, default=0.125,
                    help="fraction of the Gaussians the reference arm bins per step (time scaled up)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--train-cams", type=int, default=4,
                    help="cameras per batched training step (0: do not measure the training step)")
    ap.add_argument("--lanes", type=int, default=4, help="concurrent camera chains of the training step")
    ap.add_argument("--features", type=int, default=8,
                    help="feature channels per Gaussian to time (a multiple of 4; 0: skip)")
    ap.add_argument("--no-graphs", action="store_true", help="launch every kernel eagerly")
    ap.add_argument("--tiles", choices=("cut", "3sigma"), default="cut",
                    help="tile rectangles: 3-sigma narrowed by the opacity-aware cut, or plain 3-sigma")
    ap.add_argument("--variant", choices=sorted(VARIANT_FLAGS), default="3dgs",
                    help="the method's conventions: 3DGS (default), gsplat, gsplat with antialiasing, or 3DGS with a depth channel")
    ap.add_argument("--binning", choices=sorted(BINNING), default="auto",
                    help="binning strategy: automatic, per-tile sorts, or one depth sort and tile radix passes")
    ap.add_argument("--profile-frame", action="store_true",
                    help="run one eager frame of one camera and exit (for ncu); prints no bench line")
    ap.add_argument("--profile-camera", type=int, default=0)
    ap.add_argument("--profile-train", action="store_true",
                    help="run one eager batched training step (4 cameras, Adam) and exit (for ncu); no bench line")
    args = ap.parse_args()
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local = int(os.environ.get("LOCAL_RANK", 0))
    spec = SPECS[args.workload]
    if args.profile_frame:
        run_profile_frame(args, spec)
        return
    if args.profile_train:
        run_profile_train(args, spec)
        return
    if args.impl == "reference":
        run_reference(args, spec, rank, world)
        return
    if world > 1:
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", device_id=torch.device("cuda", local),
                                timeout=datetime.timedelta(seconds=300))
    try:
        run_native(args, spec, rank, world, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
