#!/usr/bin/env python
"""Benchmark of the differentiable EWA splatting path on B200.

One step of the default workload (train_1m_1080p: 1,000,000 SH3 Gaussians,
1920x1080, fx = fy = 1200, upstream image gradient N(0, 1e-2), synthetic and
seeded) is gs_project -> gs_bin_sort -> gs_rasterize_fwd -> gs_rasterize_bwd
(screen space) -> gs_project_bwd_adam (projection backward, densification
statistics and the Adam step in one launch; with N > 1 GPUs the gradients are
exchanged, so the tail is gs_project_bwd -> gs_densify_stats -> the sharded
Adam step). The metric is the step time and its pixel throughput (Mpix/s = rendered pixels /
step time). ``--workload`` selects one of the five workload shapes:

  fwd_1k_128        forward only (project, bin_sort, rasterize_fwd)
  fwd_100k_800      forward only
  train_1m_1080p    the full step above (default)
  train_6m_8x1080p  8 views, forward + backward + densify statistics summed
                    over the views; the sort's keys are 64-bit ((view << 32 |
                    depth) in the presort; the extras time the pages' own
                    (tile << 32 | depth) pair-key sort too)
  train_10m_4k      the full step

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--impl ours|reference]

N > 1 runs one process per GPU under torch.distributed (NCCL): each rank
renders its own view of the same Gaussians (views on an orbit of radius 8);
the flat gradient buffer is reduce-scattered, each rank runs Adam on its
1/N slice of the parameters, and an all-gather hands every rank the updated
parameters (weak scaling: one view per GPU).

Rank 0 prints one JSON line. ``--impl reference`` times the float64 CPU
oracle on the host cores on a bounded sample of the same workload instead.
"""

from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time
from typing import Optional

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "fwd+bwd train-step ms & Mpix/s at 1M Gaussians 1080p; % of roofline"

# workload -> what one step runs and its default sort mode
STEPS = {
    "fwd_1k_128": dict(kind="fwd", sort="presort"),
    "fwd_100k_800": dict(kind="fwd", sort="presort"),
    "train_1m_1080p": dict(kind="train", sort="presort"),
    "train_6m_8x1080p": dict(kind="fwdbwd", sort="presort"),
    "train_10m_4k": dict(kind="train", sort="presort"),
}
DEFAULT_WORKLOAD = "train_1m_1080p"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(STEPS))
    ap.add_argument("--sort-mode", default=None, choices=["presort", "full64"],
                    help="default: presort (depth presort, pairs placed per tile)")
    ap.add_argument("--n", type=int, default=None, help="override the Gaussian count")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-extras", action="store_true")
    ap.add_argument("--no-protocol", action="store_true",
                    help="skip the 20 + 100 step median measurement")
    ap.add_argument("--no-graphs", action="store_true",
                    help="launch every call's kernels from the host instead of replaying "
                         "one CUDA graph per call")
    args = ap.parse_args()
    if args.sort_mode is None:
        args.sort_mode = STEPS[args.workload]["sort"]
    return args


# ----------------------------------------------------------------- helpers

def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return dict(hbm_gbs=float(d["hbm_gbs"]), sm_max_mhz=float(d.get("sm_max_mhz", 1965.0)),
                    source="measured: MEASURED_PEAKS.json hbm_gbs (copy bandwidth)")
    except Exception:
        # no measured file: an earlier copy-bandwidth measurement on this GPU model
        return dict(hbm_gbs=6650.0, sm_max_mhz=1965.0,
                    source="fallback: 6650 GB/s copy bandwidth (no MEASURED_PEAKS.json)")


class ClockSampler:
    """nvidia-smi clock / throttle sampling during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(prefix="clocks_", suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.idx), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return dict(sm_mhz=None, sm_max_mhz=None, reasons=["nvidia-smi unavailable"])
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    smax.append(float(parts[2]))
                except ValueError:
                    continue
                for name, val in zip(names, parts[5:9]):
                    if val.lower().startswith("active"):
                        reasons.add(name)
        os.unlink(self.path)
        return dict(sm_mhz=statistics.median(sm) if sm else None,
                    sm_max_mhz=max(smax) if smax else None, reasons=sorted(reasons),
                    samples=len(sm))


# ----------------------------------------------------------------- work model

def sort_plan(sp, sort_mode: str) -> dict:
    """How gs_bin_sort treats this workload, as the library plans it
    (gs_bin_sort_plan): emission path, presort passes, pair passes and the
    tile-placement blocks per view."""
    from gaussian_splatting_differentiable_ewa_b200 import api
    mode = api.GS_SORT_FULL64 if sort_mode == "full64" else api.GS_SORT_PRESORT
    p = api.gs_bin_sort_plan(sp.n, sp.cams, sp.V, mode)
    tiles = sp.V * ((sp.W + 15) // 16) * ((sp.H + 15) // 16)
    path = {api.GS_PATH_TILES: "tiles", api.GS_PATH_COLUMNS: "columns",
            api.GS_PATH_TILE_ID: "tile_id"}[p.path]
    return dict(path=path, pre=p.presort_passes, pair=p.pair_passes, bpv=p.blocks_per_view,
                tiles=tiles, pair_sweep=bool(p.pair_single_sweep),
                count_ranges=bool(p.ranges_from_counts), key_bytes=int(p.pair_key_bytes))


# FP32 operations of the blend kernels (an FMA is one operation): per (pixel,
# list entry) evaluation, the evaluation form -- dx, dy, p1 and p2 (two FMAs
# each), zq (two FMAs) and the test zq <= 0; per contributing pixel in the
# forward, alpha = min(0.99, 2^-zq / 255) (multiply, min; the exp2 is an SFU
# op), T (1 - alpha) (FMA, multiply), w = alpha T and the three colour FMAs;
# in the backward, alpha, 1 - alpha and its reciprocal, T, w, the colour
# behind (3 differences, 3 FMAs), dL/dalpha (3 + 2), the clamp, dalpha/dmean
# through both eigen rows (6), the conic terms (5), opacity (1), colour (3),
# the absolute-gradient norm (3) and the ten per-pixel sums.
OPS_EVAL, OPS_FWD_CONTRIB, OPS_BWD_CONTRIB = 9, 8, 48


def algorithmic_work(sp, n_pairs: int, sort_mode: str, exps: float,
                     examined: Optional[int] = None, evals: Optional[float] = None) -> dict:
    """Algorithmic bytes (and exp evaluations) per launch of each call, from
    the per-unit figures of the hot-path scope table (its measurement part):

      project       the raw parameters read once ((11 + 3 K) floats: 236 B at
                    SH3) + 48 B written per Gaussian and view;
      bin_sort      full-64 keys: 24 B read per Gaussian and view, 12 B
                    emitted per pair, passes x 24 B + 8 B of histogram per
                    pair, 8 B per pair for the ranges; the presort paths
                    (depth presort, pairs placed per tile) move far fewer
                    bytes and are counted by their own model: every id written
                    once, the per-Gaussian depth keys counted (8 B) and sorted
                    (passes x 24 B),
                    the packed rectangles and the (tile, Gaussian block) count
                    table read and written once; the column path emits
                    key + id per pair and each rows pass reads and writes
                    them, with keys of the plan's width (4 B, or the row
                    alone in 1 or 2 B). Where the ranges come from the tile
                    counts (plan count_ranges), the last pass writes ids only
                    and nothing reads the keys for the ranges (a key's bytes
                    less twice per pair), and the rectangles are read once
                    more (16 B per Gaussian and view);
      raster fwd    4 B id + 40 B record per pair read + 20 B written per
                    pixel; the pairs read are the list entries the forward
                    examined (`examined`: a tile stops walking its list once
                    all its pixels have saturated), all pairs when not given;
      raster bwd    the same entries + 40 B of gradient atomics each + 12 B
                    of dL/dpixel per pixel; both blend kernels also count
                    FP32 operations (OPS_*): `evals` (pixel, entry)
                    evaluations -- 64 pixels for every 8x8 block an
                    examined entry's mask names -- and `exps` contributing
                    ones;
      project bwd   parameters read and gradients written once, 36 B of
                    screen-space gradients per Gaussian and view;
      densify       16 B per Gaussian and view + 24 B per Gaussian;
      adam          28 B per parameter (p, g, m, v read; p, m, v written);
      fused tail    (projection backward + statistics + Adam in one launch)
                    the parameters and both moments read and written once,
                    36 B of screen-space gradients per Gaussian and view,
                    24 B of statistics per Gaussian.

    Exps: the (pixel, Gaussian) evaluations with alpha >= 1/255 reached
    before the pixel stops (counted by the oracle on a pixel sample)."""
    n, V = sp.n, sp.V
    P = V * sp.W * sp.H
    walked = n_pairs if examined is None else examined
    ev = 0.0 if evals is None else float(evals)
    pbytes = (11 + 3 * sp.K) * 4
    plan = sort_plan(sp, sort_mode)
    pre, pair = plan["pre"], plan["pair"]
    cr = plan["count_ranges"]
    if sort_mode == "full64":
        sort_bytes = (V * n * (24 + (16 if cr else 0))
                      + n_pairs * (12 + pair * 24 + 8 + (-8 if cr else 8)))
    elif plan["path"] == "tiles":
        table = plan["tiles"] * plan["bpv"] * 4
        sort_bytes = (n_pairs * 4 + V * n * (16 + 12 + 8 + pre * 24 + 12 + 16 + 16)
                      + 3 * table + plan["tiles"] * 24)
    else:
        kb = plan["key_bytes"]
        sort_bytes = (n_pairs * ((kb + 4) + pair * 2 * (kb + 4) + (-kb if cr else kb))
                      + V * n * (16 + 8 + pre * 24 + 12 + (16 if cr else 0)))
    return {
        "gs_project": dict(bytes=n * pbytes + V * n * 48, exps=0.0),
        "gs_bin_sort": dict(bytes=sort_bytes, exps=0.0),
        "gs_rasterize_fwd": dict(bytes=walked * 44 + P * 20, exps=exps,
                                 ops=ev * OPS_EVAL + exps * OPS_FWD_CONTRIB),
        "gs_rasterize_bwd": dict(bytes=walked * (44 + 40) + P * 12, exps=exps,
                                 ops=ev * OPS_EVAL + exps * OPS_BWD_CONTRIB),
        "gs_project_bwd": dict(bytes=n * 2 * pbytes + V * n * 36, exps=0.0),
        "gs_densify_stats": dict(bytes=V * n * 16 + n * 24, exps=0.0),
        "gs_adam_step": dict(bytes=n * (pbytes // 4) * 28, exps=0.0),
        # fused tail: parameters read and written, both moments read and
        # written, the screen-space gradients, the statistics read and written
        "gs_project_bwd_adam": dict(bytes=n * 6 * pbytes + V * n * 36 + n * 24, exps=0.0),
    }


def launches_per_step(sp, sort_mode: str, kind: str = "train", fused: bool = False) -> int:
    """Library kernels launched by one step (memsets excluded); fused: the
    training step ends with the one-launch projection backward + statistics
    + Adam."""
    plan = sort_plan(sp, sort_mode)
    pre, pair = plan["pre"], plan["pair"]
    # the 64-bit sorts are single-sweep (a digit-count read + one kernel per
    # pass); the 32-bit row / tile passes are count, scan, scatter
    if sort_mode == "full64":
        # emit, digit counts, passes, ranges (from the keys, or the tile-count
        # histogram and its scan)
        sort = 1 + 1 + pair + (2 if plan["count_ranges"] else 1)
    elif plan["path"] == "tiles":
        sort = 1 + 1 + pre + 4                  # keys, presort, count, scan, base, place
    else:
        # row (columns) or tile-id passes: digit counts + one kernel each when
        # single-sweep, count + scan + scatter each otherwise
        passes = (1 + pair) if plan["pair_sweep"] else 3 * pair
        if plan["path"] == "columns":
            # ..., count, scan, emit, row passes, ranges (from the keys, or the
            # tile-count histogram and its scan)
            sort = 1 + 1 + pre + 3 + passes + (2 if plan["count_ranges"] else 1)
        else:
            sort = 1 + 1 + pre + 1 + passes + 1
    # project, sort, raster fwd (+ raster bwd, project bwd, densify (+ adam)),
    # or raster bwd + the fused tail
    tail = 2 if (kind == "train" and fused) else {"fwd": 0, "fwdbwd": 3, "train": 4}[kind]
    return 1 + sort + 1 + tail


# C call -> (kernel, source file) for the ncu traffic lookup
KERNEL_OF = {
    "gs_project": ("k_project", "project.cu"),
    "gs_rasterize_fwd": ("k_raster_fwd", "raster.cu"),
    "gs_rasterize_bwd": ("k_raster_bwd", "raster.cu"),
    "gs_project_bwd": ("k_project_bwd", "project.cu"),
    "gs_project_bwd_adam": ("k_project_bwd_fused", "project.cu"),
    "gs_adam_step": ("k_adam", "optim.cu"),
}


def profiled_traffic(call: str, workload: str):
    """DRAM bytes per launch (dram__bytes_read.sum + dram__bytes_write.sum) from
    the committed ncu summary of this kernel and workload, or None when there
    is none or the kernel's source changed since it was captured."""
    import hashlib
    import re
    if call not in KERNEL_OF:
        return None
    kernel, src = KERNEL_OF[call]
    prof = os.path.join(ROOT, "profiles", "%s_%s.md" % (kernel, workload))
    srcp = os.path.join(ROOT, "gaussian_splatting_differentiable_ewa_b200", "csrc", src)
    try:
        text = open(prof).read()
        sha = hashlib.sha256(open(srcp, "rb").read()).hexdigest()
    except OSError:
        return None
    m_sha = re.search(r"kernel_source_sha256:\s*([0-9a-f]{64})", text)
    m_t = re.search(r"traffic_bytes_per_launch:\s*([0-9]+)", text)
    if not m_sha or not m_t or m_sha.group(1) != sha:
        return None
    return int(m_t.group(1))


L2_BYTES = 126 * 1000 * 1000


def working_set_bytes(sp) -> int:
    """Device bytes one step touches: parameters, gradients and both moments,
    records, binning records, radii, pair ids, images and screen-space
    gradients."""
    n, V = sp.n, sp.V
    return int(4 * sp.flat_total * 4 + V * n * (64 + 16 + 4 + 48) + 4 * sp.capacity
               + V * sp.W * sp.H * (12 + 4 + 4 + 12))


def sfu_peak_gexps(sm_mhz: float, sms: int = 148) -> float:
    # MUFU.EX2: 16 results per SM per clock (4 per SM sub-partition)
    return sms * 16 * sm_mhz * 1e6 / 1e9


def alu_peak_gops(sm_mhz: float, sms: int = 148) -> float:
    # FP32: 128 lanes per SM, one operation (an FMA counting as one) per lane
    # per clock
    return sms * 128 * sm_mhz * 1e6 / 1e9


# ----------------------------------------------------------------- CPU oracle

def _subset(scene, m: int, seed: int = 3):
    """The scene restricted to m of its Gaussians (a seeded random subset)."""
    import copy
    if m >= scene.n:
        return scene
    idx = np.sort(np.random.default_rng(seed).choice(scene.n, m, replace=False))
    sub = copy.copy(scene)
    for k in ("means", "log_scales", "quats", "opacity_logit", "sh"):
        setattr(sub, k, np.ascontiguousarray(getattr(scene, k)[idx]))
    return sub


def cpu_baseline(scene, kind: str, sample_pixels: int = 2048, max_gauss: int = 250_000,
                 seed: int = 5):
    """Time the float64 oracle as it stands on the host cores over a bounded
    sample of one step and extrapolate to the full step:
      * projection, projection backward and Adam on a seeded subset of at
        most `max_gauss` Gaussians (all views), scaled by n / subset;
      * render (and render backward) of `sample_pixels` random pixels of view
        0 from the projection of every Gaussian into view 0 (its time is not
        counted again), scaled by the step's pixel count.
    Returns (dict, n_exp_mean) where n_exp_mean is the oracle's count of
    alpha >= 1/255 evaluations per pixel on the sample."""
    from oracle import oracle as O
    from gaussian_splatting_differentiable_ewa_b200 import scenes as S
    c = scene.cameras[0]
    n, V = scene.n, scene.n_views
    rng = np.random.default_rng(seed)
    pix = np.stack([np.zeros(sample_pixels, np.int64), rng.integers(0, c.width, sample_pixels),
                    rng.integers(0, c.height, sample_pixels)], 1).astype(np.int32)
    sub = _subset(scene, max_gauss)
    scale_g = n / sub.n
    t0 = time.perf_counter()
    projs_sub = O.project_views(sub)
    t1 = time.perf_counter()
    proj0 = [O.project(scene, c)]
    t2 = time.perf_counter()
    ref = O.render(proj0, scene.cameras[:1], scene.background, pix)
    t3 = time.perf_counter()
    t_bwd = t_pb = t_adam = 0.0
    if kind != "fwd":
        dL = S.make_upstream_grad(1, c.height, c.width, seed=1)
        gC = dL[0][:, pix[:, 2], pix[:, 1]].T
        O.render_bwd(proj0, scene.cameras[:1], scene.background, pix, gC)
        t4 = time.perf_counter()
        g2 = np.full((V, sub.n, 10), 1e-3)
        O.project_bwd(sub, projs_sub, g2)
        t5 = time.perf_counter()
        t_bwd, t_pb = t4 - t3, t5 - t4
        if kind == "train":
            p = np.zeros(59 * sub.n)
            O.adam(p, p + 1e-3, p, p, 1e-3, 1)
            t_adam = time.perf_counter() - t5
    P = V * c.width * c.height
    step_s = ((t1 - t0) + t_pb + t_adam) * scale_g + ((t3 - t2) + t_bwd) * P / sample_pixels
    measured = time.perf_counter() - t0
    out = dict(value=P / step_s / 1e6, unit="Mpix/s", cores=O.num_threads(), kind="oracle",
               sample=("float64 oracle: projection%s on %d of %d Gaussians (all %d views), "
                       "scaled by the Gaussian count; render%s on %d random pixels of view 0, "
                       "scaled to %d pixels" % (
                           "" if kind == "fwd" else ", projection backward" +
                           (" and Adam" if kind == "train" else ""),
                           sub.n, n, V, "" if kind == "fwd" else " + render backward",
                           sample_pixels, P)),
               step_s=step_s, measured_s=measured)
    return out, float(ref["n_exp"].mean())


def run_reference(args):
    """--impl reference: the oracle timed on the host, rank 0 only; each step
    a bounded sample of the workload (cpu_baseline's split), extrapolated."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    from oracle import oracle as O
    from gaussian_splatting_differentiable_ewa_b200 import scenes as S
    kind = STEPS[args.workload]["kind"]
    scene = S.make_scene(args.workload, n=args.n)
    c = scene.cameras[0]
    P = scene.n_views * c.width * c.height
    times = []
    cpu = None
    for it in range(args.warmup + args.steps):
        cpu, _ = cpu_baseline(scene, kind, sample_pixels=256, max_gauss=50_000, seed=7 + it)
        if it >= args.warmup:
            times.append(cpu["step_s"])
    ms = 1000.0 * float(np.mean(times))
    value = P / (ms / 1000.0) / 1e6
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "Mpix/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": args.workload, "gaussians": scene.n, "width": c.width,
                   "height": c.height, "sh_degree": scene.sh_degree,
                   "views_per_gpu": scene.n_views, "step": kind},
        "cpu_baseline": {"value": value, "unit": "Mpix/s", "cores": O.num_threads(),
                         "kind": "oracle", "sample": "per step: " + cpu["sample"]},
        "e2e": {"value": value, "unit": "Mpix/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------- our path

# FP32 peak of the part for the ALU-bound loss kernel: 148 SMs x 128 FP32
# lanes x 2 FLOP per FMA at the maximum SM clock.
FP32_LANES = 148 * 128


def measure_loss(sp, reps: int = 5) -> dict:
    """gs_l1_dssim (loss, and its gradient) on the Splatter's rendered frame
    against a seeded target of the same size, each launch timed with CUDA
    events after an L2 flush (a 256 MB write), mean over `reps` after an
    untimed launch. Algorithmic work per value: the separable 11-tap window
    applied along rows and columns to the four moments SSIM needs (x, y,
    xx + yy, xy) and to the three partial maps of the gradient,
    2 x 11 x 7 = 154 FMA (308 FLOP); traffic: x and y read, dL/dx written,
    12 bytes."""
    import torch
    from gaussian_splatting_differentiable_ewa_b200 import api
    from gaussian_splatting_differentiable_ewa_b200 import scenes as S
    V, H, W = sp.V, sp.H, sp.W
    _, tgt = S.make_image_pair(V, H, W, seed=4)
    target = torch.from_numpy(tgt).cuda()
    sp.loss(target)
    torch.cuda.synchronize()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ms = 0.0
    for _ in range(reps):
        flush.fill_(1)
        e0.record()
        sp.loss(target)
        e1.record()
        torch.cuda.synchronize()
        ms += e0.elapsed_time(e1) / reps
    values = 3 * V * H * W
    pk = peaks()
    tflops = values * 308 / (ms / 1e3) / 1e12
    fp32_peak = FP32_LANES * 2 * pk["sm_max_mhz"] * 1e6 / 1e12
    gbs = values * 12 / (ms / 1e3) / 1e9
    t = sp.loss_terms.cpu().numpy()
    return dict(ms=ms, values=values, tflops=tflops, fp32_peak_tflops=fp32_peak,
                alu_frac=tflops / fp32_peak, gbs=gbs, hbm_frac=gbs / pk["hbm_gbs"],
                loss=float(t[0, 0]), l1=float(t[0, 1]), ssim=float(t[0, 2]))


def measure_quant_adam(sp, reps: int = 5) -> dict:
    """gs_adam_step_sh_quant on the Splatter's SH (encoded once with
    gs_sh_quantize) and its SH gradient, 8- and 16-bit codes, nearest
    rounding, each launch after an L2 flush; mean of `reps` after an untimed
    launch. Beside it the float32 gs_adam_step of the same SH group.
    Algorithmic bytes per SH value: code read and written (1 or 2 B each),
    gradient 4 B, bfloat16 moments read and written 8 B; float32: 28 B."""
    import torch
    from gaussian_splatting_differentiable_ewa_b200 import api
    n = sp.n
    sh = dict(sp.param_list)["sh"]
    k3 = sh[0].numel()
    n_pad = -(-n // 256) * 256
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    pk = peaks()

    def timed(fn):
        fn()
        torch.cuda.synchronize()
        ms = 0.0
        for _ in range(reps):
            flush.fill_(1)
            e0.record()
            fn()
            e1.record()
            torch.cuda.synchronize()
            ms += e0.elapsed_time(e1) / reps
        return ms

    out = {}
    g = sp.grads["sh"]
    for bits in (8, 16):
        codes = torch.zeros((k3, n_pad), dtype=torch.uint8 if bits == 8 else torch.int16,
                            device="cuda")
        bounds = torch.zeros((k3, n_pad // 256, 2), dtype=torch.float32, device="cuda")
        q = api.sh_quant(codes, bounds, n, k3, bits)
        api.gs_sh_quantize(sh, q)
        m = torch.zeros((k3, n_pad), dtype=torch.int16, device="cuda")
        v = torch.zeros_like(m)
        step = [0]

        def run():
            step[0] += 1
            api.gs_adam_step_sh_quant(q, g, m, v, 2.5e-3, 0.9, 0.999, 1e-15, step[0])
        ms = timed(run)
        nbytes = n * k3 * (2 * bits // 8 + 4 + 8) + k3 * (n_pad // 256) * 16
        out["q%d" % bits] = dict(ms=ms, gbs=nbytes / (ms / 1e3) / 1e9,
                                 hbm_frac=nbytes / (ms / 1e3) / 1e9 / pk["hbm_gbs"],
                                 state_bytes=n * k3 * (bits // 8 + 4))
    m32, v32 = torch.zeros_like(sh), torch.zeros_like(sh)
    p32 = sh.clone()
    ms = timed(lambda: api.gs_adam_step([(p32, g, m32, v32, 2.5e-3)], 0.9, 0.999, 1e-15, 1))
    nbytes = n * k3 * 28
    out["f32"] = dict(ms=ms, gbs=nbytes / (ms / 1e3) / 1e9,
                      hbm_frac=nbytes / (ms / 1e3) / 1e9 / pk["hbm_gbs"], state_bytes=n * k3 * 12)
    return out


def measure_densify(sp) -> dict:
    """One gs_densify_and_prune call on the Splatter's accumulated statistics
    (absolute gradients, the page's threshold 0.0002), timed with CUDA events
    after an untimed call. Algorithmic bytes: 59 real floats of parameters,
    Adam m and v read per Gaussian plus its statistics and draws, and the same
    59 x 3 floats written per output Gaussian."""
    import torch
    from gaussian_splatting_differentiable_ewa_b200 import api
    n = sp.n
    names = [k for k, _ in sp.param_list]
    like = lambda t: torch.empty((2 * n,) + tuple(t.shape[1:]), dtype=t.dtype,  # noqa: E731
                                 device=t.device)
    out = [like(t) for _, t in sp.param_list]
    m_out = [like(t) for _, t in sp.param_list]
    v_out = [like(t) for _, t in sp.param_list]
    n_out = torch.zeros(1, dtype=torch.int64, device="cuda")
    codes = torch.empty(n, dtype=torch.int8, device="cuda")
    ws = torch.zeros((api.gs_densify_workspace_size(n) + 255) // 256 * 256 // 8,
                     dtype=torch.int64, device="cuda")
    gen = torch.Generator(device="cuda")
    gen.manual_seed(0)
    z = torch.randn((n, 2, 3), generator=gen, device="cuda")
    dp = api.densify_params(0.0002, 0.05, 0.005, 1.0)
    args = (sp.c_params, api.grads(*[sp.exp_avg[k] for k in names]),
            api.grads(*[sp.exp_avg_sq[k] for k in names]), sp.accum_abs, sp.denom, z, dp,
            api.grads(*out), api.grads(*m_out), api.grads(*v_out), 2 * n, n_out, codes, ws)
    api.gs_densify_and_prune(*args)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    api.gs_densify_and_prune(*args)
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1)
    m = int(n_out.item())
    counts = torch.bincount(codes.long(), minlength=4).cpu().tolist()
    nbytes = n * (59 * 4 * 3 + 4 + 4 + 24) + m * 59 * 4 * 3
    pk = peaks()
    return dict(ms=ms, gbs=nbytes / (ms / 1e3) / 1e9,
                hbm_frac=nbytes / (ms / 1e3) / 1e9 / pk["hbm_gbs"], n_in=n, n_out=m,
                pruned=counts[0], kept=counts[1], cloned=counts[2], split=counts[3])


def measure_full64_sort(scene, reps: int = 10) -> dict:
    """gs_bin_sort with 64-bit (global tile << 32 | depth bits) keys on the
    workload's projections: one emission of every pair's key, the stable
    least-significant-digit radix passes over the key bits, the tile ranges.
    Each launch after an L2 flush, mean of `reps` after an untimed one; bytes
    by the scope table's figures (see algorithmic_work)."""
    import torch
    from gaussian_splatting_differentiable_ewa_b200 import api
    from gaussian_splatting_differentiable_ewa_b200.pipeline import Splatter
    sp = Splatter(scene, sort_mode=api.GS_SORT_FULL64)
    sp.ensure_capacity()
    sp.project()
    sp.bin_sort()
    torch.cuda.synchronize()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ms = 0.0
    for _ in range(reps):
        flush.fill_(1)
        e0.record()
        sp.bin_sort()
        e1.record()
        torch.cuda.synchronize()
        ms += e0.elapsed_time(e1) / reps
    assert sp.status() == api.GS_OK
    n_pairs = int(sp.n_pairs.item())
    plan = sort_plan(sp, "full64")
    nbytes = algorithmic_work(sp, n_pairs, "full64", 0.0)["gs_bin_sort"]["bytes"]
    pk = peaks()
    out = dict(ms=ms, pairs=n_pairs, passes=plan["pair"], gbs=nbytes / (ms / 1e3) / 1e9,
               hbm_frac=nbytes / (ms / 1e3) / 1e9 / pk["hbm_gbs"], bytes=nbytes)
    del sp
    torch.cuda.empty_cache()
    return out


def run_ours(args):
    import torch
    import torch.distributed as dist
    from gaussian_splatting_differentiable_ewa_b200 import api
    from gaussian_splatting_differentiable_ewa_b200 import scenes as S
    from gaussian_splatting_differentiable_ewa_b200.pipeline import Splatter

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if not torch.cuda.is_available():
        raise RuntimeError("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    mode = api.GS_SORT_PRESORT if args.sort_mode == "presort" else api.GS_SORT_FULL64
    kind = STEPS[args.workload]["kind"]

    from gaussian_splatting_differentiable_ewa_b200 import dist as gdist
    scene = S.make_scene(args.workload, n=args.n)
    if world > 1:
        scene.cameras = [gdist.orbit_view(scene, rank, world)]
    c = scene.cameras[0]
    sp = Splatter(scene, sort_mode=mode)
    if world > 1 and kind == "train":
        sp.shard_optimizer(rank, world)
    sp.ensure_capacity()
    V = sp.V
    # the list entries a forward examines (the work model's raster units):
    # entry masks are 4-bit, so entries still holding 0xFF after one forward
    # were never reached (their tile had stopped)
    sp.project()
    sp.bin_sort()
    sp.warp_masks.fill_(0xFF)
    sp.rasterize_fwd()
    torch.cuda.synchronize()
    wm = sp.warp_masks[:int(sp.n_pairs.item())]
    wm = wm[wm != 0xFF].to(torch.int32)
    examined = int(wm.numel())
    # (pixel, entry) evaluations: 64 pixels per 8x8 block an entry's mask names
    evals = 64 * int(sum(((wm >> b) & 1).sum().item() for b in range(4)))
    # the parameters and moments the timed steps start from (Adam moves them;
    # the protocol run below starts from the same state)
    start_state = [t.clone() for t in (sp.param_flat, sp.m_flat, sp.v_flat)]
    dL_host = S.make_upstream_grad(V, c.height, c.width, seed=1)
    dL = torch.as_tensor(dL_host).cuda() if kind != "fwd" else None
    stream = torch.cuda.current_stream()
    pixels = V * c.width * c.height

    # a one-GPU training step ends with the fused tail (projection backward,
    # densification statistics and Adam in one launch); with N > 1 the
    # gradients are exchanged, so the tail stays three calls
    fused = kind == "train" and sp.fused_tail_ok()
    names = ["gs_project", "gs_bin_sort", "gs_rasterize_fwd"]
    if kind != "fwd":
        names += ["gs_rasterize_bwd"]
        names += ["gs_project_bwd_adam"] if fused else ["gs_project_bwd", "gs_densify_stats"]
    if kind == "train" and not fused:
        names += ["gs_adam_step" if world == 1 else "reduce_scatter+gs_adam_step+all_gather"]

    # one CUDA graph per call (not Adam, whose bias corrections follow the
    # step count): the call's kernels replay without host launch gaps
    graphs = None if args.no_graphs else sp.capture_calls(dL)
    torch.cuda.synchronize()

    def call(name, fn):
        if graphs is not None and name in graphs:
            graphs[name].replay()
        else:
            fn()

    def step(events=None):
        def mark(k):
            if events is not None:
                events[k].record(stream)
        mark(0)
        call("project", sp.project)
        mark(1)
        call("bin_sort", sp.bin_sort)
        mark(2)
        call("rasterize_fwd", sp.rasterize_fwd)
        mark(3)
        if kind == "fwd":
            return
        call("rasterize_bwd", lambda: sp.rasterize_bwd(dL, with_params=False))
        mark(4)
        if fused:
            sp.project_bwd_adam()  # not in a graph: the bias corrections follow the step
            mark(5)
            return
        call("project_bwd", sp.project_bwd)
        mark(5)
        call("densify_stats", sp.densify_stats)
        mark(6)
        if kind == "train":
            sp.adam_step()  # with N > 1: reduce-scatter, Adam on the slice, all-gather
            mark(7)

    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize()
    assert sp.status() == api.GS_OK, "device status after warm-up"

    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(len(names) + 1)]
          for _ in range(args.steps)]
    clocks = ClockSampler(local)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.3)
    # a working set that fits in L2 is flushed (a 256 MB write) before every
    # step, outside the step's events, and the step time is the sum of the
    # steps' own event intervals
    flush_l2 = working_set_bytes(sp) < L2_BYTES
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda") if flush_l2 else None
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for k in range(args.steps):
        if flush_l2:
            flush.fill_(1)
        step(ev[k])
    end.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    if world > 1:
        dist.barrier()
    if flush_l2:
        own = sum(ev[k][0].elapsed_time(ev[k][-1]) for k in range(args.steps))
        elapsed_ms = gdist.max_over_ranks(own, device="cuda")
    else:
        elapsed_ms = gdist.max_over_ranks(start.elapsed_time(end), device="cuda")
    per_call = {nm: float(np.mean([ev[k][i].elapsed_time(ev[k][i + 1]) for k in range(args.steps)]))
                for i, nm in enumerate(names)}
    ms = elapsed_ms / args.steps
    value = world * pixels / (ms / 1000.0) / 1e6
    n_pairs = int(sp.n_pairs.item())
    status = sp.status()

    # the measurement protocol of the scope table: 20 warm-up steps, then the
    # median of 100 steps, each timed by its own events (single GPU)
    protocol = None
    if world == 1 and not args.no_protocol:
        for dst, src in zip((sp.param_flat, sp.m_flat, sp.v_flat), start_state):
            dst.copy_(src)
        for _ in range(20):
            step()
        pev = [[torch.cuda.Event(enable_timing=True) for _ in range(len(names) + 1)]
               for _ in range(100)]
        for k in range(100):
            if flush_l2:
                flush.fill_(1)
            step(pev[k])
        torch.cuda.synchronize()
        st = np.array([pev[k][0].elapsed_time(pev[k][-1]) for k in range(100)])
        protocol = {"warmup": 20, "steps": 100, "median_ms": float(np.median(st)),
                    "mean_ms": float(st.mean()), "p10_ms": float(np.percentile(st, 10)),
                    "p90_ms": float(np.percentile(st, 90)),
                    "median_mpix_s": pixels / (float(np.median(st)) / 1000.0) / 1e6,
                    "per_call_median_ms": {
                        nm: float(np.median([pev[k][i].elapsed_time(pev[k][i + 1])
                                             for k in range(100)]))
                        for i, nm in enumerate(names)}}

    # end to end through the library's host-fed calls: every step uploads its
    # upstream gradient from pinned host memory (training) and downloads the
    # rendered image to it, on copy streams (one per direction) overlapping
    # the compute stream
    e2e = None
    if not args.no_e2e:
        h_out = torch.empty(sp.image.shape, dtype=torch.float32).pin_memory()
        sp.stream = torch.cuda.Stream()
        if kind == "fwd":
            run = lambda k: sp.render_to_host([h_out] * k)  # noqa: E731
            h2d = 88 * V  # the camera structs, passed by value with every launch
        else:
            h_in = torch.from_numpy(dL_host).pin_memory()
            run = lambda k: sp.train_from_host([h_in] * k, [h_out] * k,  # noqa: E731
                                               adam=(kind == "train"))
            h2d = int(h_in.numel() * 4)
        run(3)  # warm-up
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        e0.record(sp.stream)
        run(args.steps)
        e1.record(sp.stream)
        torch.cuda.synchronize()
        sp.stream = None
        e_ms = gdist.max_over_ranks(e0.elapsed_time(e1) / args.steps, device="cuda")
        e2e = {"value": world * pixels / (e_ms / 1000.0) / 1e6, "unit": "Mpix/s",
               "ms_per_step": e_ms, "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": int(h_out.numel() * 4)}

    # beside the step, on the default workload: densify_and_prune once on the
    # statistics the timed steps accumulated (it runs every few hundred
    # steps), the loss, the quantised-SH Adam step and the full-64 sort
    extras = {}
    if world == 1 and not args.no_extras:
        if args.workload == DEFAULT_WORKLOAD:
            extras["gs_densify_and_prune"] = measure_densify(sp)
            extras["gs_l1_dssim"] = measure_loss(sp)
            extras["gs_adam_step_sh_quant"] = measure_quant_adam(sp)
        if args.sort_mode != "full64" and kind != "fwd":
            extras["gs_bin_sort_full64"] = measure_full64_sort(scene)

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return 0

    # CPU baseline and the exp count of the blend kernels (oracle, rank 0, N=1)
    cpu = None
    exps = None
    if world == 1 and not args.no_cpu_baseline:
        cpu, nexp_mean = cpu_baseline(scene, kind)
        exps = nexp_mean * pixels
    pk = peaks()
    work = algorithmic_work(sp, n_pairs, args.sort_mode, exps or 0.0, examined, evals)
    if world > 1 and kind == "train":
        work["gs_adam_step"]["bytes"] /= world  # each rank updates its slice only
    kernels = {}
    sfu = sfu_peak_gexps(pk["sm_max_mhz"])
    alu = alu_peak_gops(pk["sm_max_mhz"])
    for nm in names:
        key = nm if nm in work else "gs_adam_step"
        if key not in work:
            continue
        t = per_call[nm] / 1000.0
        w = work[key]
        k = dict(ms=per_call[nm], bytes=w["bytes"], gbs=w["bytes"] / t / 1e9,
                 hbm_frac=w["bytes"] / t / 1e9 / pk["hbm_gbs"])
        bound_s = w["bytes"] / (pk["hbm_gbs"] * 1e9)
        if w["exps"]:
            k["gexps"] = w["exps"] / t / 1e9
            k["sfu_frac"] = k["gexps"] / sfu
            bound_s = max(bound_s, w["exps"] / (sfu * 1e9))
        if w.get("ops"):
            k["gops"] = w["ops"] / t / 1e9
            k["alu_frac"] = k["gops"] / alu
            bound_s = max(bound_s, w["ops"] / (alu * 1e9))
        k["bound_ms"] = bound_s * 1000.0
        k["roofline_frac"] = bound_s / t
        kernels[nm] = k
    dom = max(kernels, key=lambda k: kernels[k]["ms"])
    dk = "gs_adam_step" if dom not in work else dom
    t_hbm = work[dk]["bytes"] / (pk["hbm_gbs"] * 1e9)
    t_sfu = (work[dk]["exps"] / (sfu * 1e9)) if exps else 0.0
    t_alu = work[dk].get("ops", 0.0) / (alu * 1e9)
    if t_alu > max(t_hbm, t_sfu):
        ach = work[dk]["ops"] / (per_call[dom] / 1000.0) / 1e9
        roof = {"kernel": dom, "bound": "alu", "achieved": ach, "peak": alu, "unit": "Gop/s",
                "frac": ach / alu, "traffic": profiled_traffic(dk, args.workload),
                "peak_source": "148 SM x 128 FP32 lanes x %.0f MHz (max SM clock), FP32 "
                               "operations of the evaluation form" % pk["sm_max_mhz"]}
    elif t_sfu > t_hbm:
        ach = work[dk]["exps"] / (per_call[dom] / 1000.0) / 1e9
        roof = {"kernel": dom, "bound": "alu", "achieved": ach, "peak": sfu, "unit": "Gexp/s",
                "frac": ach / sfu, "traffic": profiled_traffic(dk, args.workload),
                "peak_source": "148 SM x 16 MUFU.EX2/clk x %.0f MHz (max SM clock)"
                               % pk["sm_max_mhz"]}
    else:
        ach = work[dk]["bytes"] / (per_call[dom] / 1000.0) / 1e9
        roof = {"kernel": dom, "bound": "hbm", "achieved": ach, "peak": pk["hbm_gbs"],
                "unit": "GB/s", "frac": ach / pk["hbm_gbs"],
                "traffic": profiled_traffic(dk, args.workload),
                "peak_source": pk["source"]}
    # step roofline: sum over calls of max(bytes / HBM, exps / SFU, ops / FP32)
    bound_ms = sum(k["bound_ms"] for k in kernels.values())
    n_launch = launches_per_step(sp, args.sort_mode, kind, fused)
    line = {
        "metric": METRIC, "value": value, "unit": "Mpix/s", "n_gpus": world,
        "steps": args.steps, "warmup": max(args.warmup, 3), "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic",
        "config": {"workload": args.workload, "step": kind, "gaussians": sp.n,
                   "width": c.width, "height": c.height, "views_per_gpu": V,
                   "sh_degree": sp.deg, "pairs": n_pairs, "pairs_examined": examined,
                   "sort_mode": args.sort_mode,
                   "sort_path": sort_plan(sp, args.sort_mode)["path"],
                   "launch": "host launches" if graphs is None else
                             "one CUDA graph per call (the step's Adam, fused or not, launched "
                             "from the host: its bias corrections follow the step)",
                   "l2": ("working set %.0f MB inside the 126 MB L2: flushed (256 MB write) "
                          "before every step, outside the step's own timing"
                          % (working_set_bytes(sp) / 1e6)) if flush_l2 else
                         ("working set %.0f MB, larger than the 126 MB L2"
                          % (working_set_bytes(sp) / 1e6)),
                   "parallelism": "dp%d (one view per GPU; gradient reduce-scatter, Adam on "
                                  "1/%d of the parameters, parameter all-gather)" % (world, world)
                   if world > 1 else "single GPU"},
        "roofline": roof,
        "step_roofline": {"bound_ms": bound_ms, "frac": bound_ms / ms},
        "kernels": kernels,
        "protocol": protocol,
        "extras": extras,
        "cpu_baseline": None if cpu is None else {k: cpu[k] for k in
                                                  ("value", "unit", "cores", "kind", "sample")},
        "e2e": e2e,
        "gpu_launches": n_launch * args.steps,
        "clocks": clk,
        "device_status": api.status_string(status),
    }
    print(json.dumps(line), flush=True)
    return 0


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
