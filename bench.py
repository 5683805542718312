#!/usr/bin/env python
"""Benchmark of the differentiable EWA splatting training step on B200.

One step = gs_project -> gs_bin_sort -> gs_rasterize_fwd -> gs_rasterize_bwd
(screen space) -> gs_project_bwd -> gs_densify_stats -> gs_adam_step, on the
1,000,000-Gaussian SH3 scene at 1920x1080 (fx = fy = 1200) with an upstream
image gradient N(0, 1e-2), synthetic and seeded. The metric is the step time
and its pixel throughput (Mpix/s = rendered pixels / step time).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

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

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

WORKLOAD = "train_1m_1080p"
METRIC = "fwd+bwd train-step ms & Mpix/s at 1M Gaussians 1080p; % of roofline"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--sort-mode", default="presort", choices=["presort", "full64"])
    ap.add_argument("--n", type=int, default=None, help="override the Gaussian count")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    return ap.parse_args()


# ----------------------------------------------------------------- helpers

def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return dict(hbm_gbs=float(d["hbm_gbs"]), sm_max_mhz=float(d.get("sm_max_mhz", 1965.0)),
                    source="measured")
    except Exception:
        return dict(hbm_gbs=6650.0, sm_max_mhz=1965.0, source="fallback")


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
                tiles=tiles)


def algorithmic_work(sp, n_pairs: int, sort_mode: str, exps: float) -> dict:
    """Algorithmic bytes (and exp evaluations) per launch of each call.

    Bytes count the data the definition has to move once: parameters read,
    outputs written, 59 real floats per Gaussian (pad lanes excluded); a radix
    pass reads and writes every key and value once; placing pairs straight at
    their positions writes every id once, reads every packed rectangle once
    and reads and writes the (tile, Gaussian block) count table once; the
    blend kernels read every list entry's id and record once."""
    n, V = sp.n, sp.V
    P = V * sp.W * sp.H
    rec = 48
    p59 = 59 * 4
    plan = sort_plan(sp, sort_mode)
    pre, pair = plan["pre"], plan["pair"]
    if sort_mode == "full64":
        sort_bytes = n_pairs * (12 + pair * 24 + 8) + V * n * 16
    elif plan["path"] == "tiles":
        table = plan["tiles"] * plan["bpv"] * 4
        sort_bytes = (n_pairs * 4 + V * n * (16 + 12 + pre * 24 + 12 + 16 + 16)
                      + 3 * table + plan["tiles"] * 24)
    else:
        sort_bytes = n_pairs * (8 + pair * 16 + 4) + V * n * (16 + pre * 24 + 12)
    return {
        "gs_project": dict(bytes=V * n * (p59 + rec + 16 + 4), exps=0.0),
        "gs_bin_sort": dict(bytes=sort_bytes, exps=0.0),
        "gs_rasterize_fwd": dict(bytes=n_pairs * (4 + rec) + P * 20, exps=exps),
        "gs_rasterize_bwd": dict(bytes=n_pairs * (4 + rec) + P * 20 + V * n * 48 * 2, exps=exps),
        "gs_project_bwd": dict(bytes=V * n * (p59 + 48 + 4) + n * p59, exps=0.0),
        "gs_densify_stats": dict(bytes=V * n * (12 + 4) + n * 24, exps=0.0),
        "gs_adam_step": dict(bytes=n * 59 * 28, exps=0.0),
    }


def launches_per_step(sp, sort_mode: str) -> int:
    """Library kernels launched by one step (memsets excluded)."""
    plan = sort_plan(sp, sort_mode)
    pre, pair = plan["pre"], plan["pair"]
    if sort_mode == "full64":
        sort = 1 + 3 * pair + 1                 # emit, passes, ranges
    elif plan["path"] == "tiles":
        sort = 1 + 3 * pre + 4                  # keys, presort, count, scan, base, place
    elif plan["path"] == "columns":
        sort = 1 + 3 * pre + 3 + 3 * pair + 1   # ..., count, scan, emit, row passes, ranges
    else:
        sort = 1 + 3 * pre + 1 + 3 * pair + 1
    return 1 + sort + 1 + 1 + 1 + 1 + 1


# C call -> (kernel, source file) for the ncu traffic lookup
KERNEL_OF = {
    "gs_project": ("k_project", "project.cu"),
    "gs_rasterize_fwd": ("k_raster_fwd", "raster.cu"),
    "gs_rasterize_bwd": ("k_raster_bwd", "raster.cu"),
    "gs_project_bwd": ("k_project_bwd", "project.cu"),
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


def sfu_peak_gexps(sm_mhz: float, sms: int = 148) -> float:
    # MUFU.EX2: 16 results per SM per clock (4 per SM sub-partition)
    return sms * 16 * sm_mhz * 1e6 / 1e9


# ----------------------------------------------------------------- CPU oracle

def cpu_baseline(scene, sample_pixels: int = 4096, seed: int = 5):
    """Time the float64 oracle as it stands on host cores over a bounded
    sample and extrapolate to one full step. Returns (dict, n_exp_mean)."""
    from oracle import oracle as O
    from gaussian_splatting_differentiable_ewa_b200 import scenes as S
    c = scene.cameras[0]
    rng = np.random.default_rng(seed)
    pix = np.stack([np.zeros(sample_pixels, np.int64), rng.integers(0, c.width, sample_pixels),
                    rng.integers(0, c.height, sample_pixels)], 1).astype(np.int32)
    t0 = time.perf_counter()
    projs = O.project_views(scene)
    t1 = time.perf_counter()
    ref = O.render(projs, scene.cameras, scene.background, pix)
    t2 = time.perf_counter()
    dL = S.make_upstream_grad(1, c.height, c.width, seed=1)
    gC = dL[0][:, pix[:, 2], pix[:, 1]].T
    g2 = O.render_bwd(projs, scene.cameras, scene.background, pix, gC)
    t3 = time.perf_counter()
    # the projection backward over every Gaussian (as in a full step)
    g2_full = g2.copy()
    g2_full[..., :9] += 1e-3
    O.project_bwd(scene, projs, g2_full)
    t4 = time.perf_counter()
    n = scene.n
    p = np.zeros(59 * n)
    O.adam(p, p + 1e-3, p, p, 1e-3, 1)
    t5 = time.perf_counter()
    P = c.width * c.height
    scale = P / sample_pixels
    step_s = (t1 - t0) + (t2 - t1 + t3 - t2) * scale + (t4 - t3) + (t5 - t4)
    out = dict(value=P / step_s / 1e6, unit="Mpix/s", cores=O.num_threads(), kind="oracle",
               sample=("float64 oracle: projection, projection backward and Adam over all %d "
                       "Gaussians; render + render backward on %d random pixels, extrapolated "
                       "linearly to %d pixels" % (n, sample_pixels, P)),
               step_s=step_s, measured_s=t5 - t0)
    return out, float(ref["n_exp"].mean())


def run_reference(args):
    """--impl reference: the oracle timed on the host, rank 0 only."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    from oracle import oracle as O
    from gaussian_splatting_differentiable_ewa_b200 import scenes as S
    scene = S.make_scene(WORKLOAD, n=args.n)
    c = scene.cameras[0]
    P = c.width * c.height
    n = scene.n
    sub = max(1, n // 16)
    small = S.make_scene(WORKLOAD, n=sub)
    projs_full = O.project_views(scene)
    rng = np.random.default_rng(7)
    dL = S.make_upstream_grad(1, c.height, c.width, seed=1)
    n_pix = 512
    times = []
    for it in range(args.warmup + args.steps):
        pix = np.stack([np.zeros(n_pix, np.int64), rng.integers(0, c.width, n_pix),
                        rng.integers(0, c.height, n_pix)], 1).astype(np.int32)
        gC = dL[0][:, pix[:, 2], pix[:, 1]].T
        t0 = time.perf_counter()
        pr = O.project_views(small)
        t1 = time.perf_counter()
        O.render(projs_full, scene.cameras, scene.background, pix)
        g2 = O.render_bwd(projs_full, scene.cameras, scene.background, pix, gC)
        t2 = time.perf_counter()
        g2s = np.full((1, sub, 10), 1e-3)
        O.project_bwd(small, pr, g2s)
        p = np.zeros(59 * sub)
        O.adam(p, p + 1e-3, p, p, 1e-3, 1)
        t3 = time.perf_counter()
        step = (t1 - t0) * n / sub + (t2 - t1) * P / n_pix + (t3 - t2) * n / sub
        if it >= args.warmup:
            times.append(step)
    ms = 1000.0 * float(np.mean(times))
    value = P / (ms / 1000.0) / 1e6
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "Mpix/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": WORKLOAD, "gaussians": n, "width": c.width, "height": c.height,
                   "sh_degree": 3, "views_per_gpu": 1},
        "cpu_baseline": {"value": value, "unit": "Mpix/s", "cores": O.num_threads(),
                         "kind": "oracle",
                         "sample": "per step: projection, projection backward and Adam on "
                                   "%d of %d Gaussians, render + backward on %d random pixels; "
                                   "each part extrapolated linearly to the full step"
                                   % (sub, n, n_pix)},
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

    from gaussian_splatting_differentiable_ewa_b200 import dist as gdist
    scene = S.make_scene(WORKLOAD, n=args.n)
    if world > 1:
        scene.cameras = [gdist.orbit_view(scene, rank, world)]
    c = scene.cameras[0]
    sp = Splatter(scene, sort_mode=mode)
    if world > 1:
        sp.shard_optimizer(rank, world)
    need = sp.ensure_capacity()
    dL_host = S.make_upstream_grad(1, c.height, c.width, seed=1)
    dL = torch.as_tensor(dL_host).cuda()
    stream = torch.cuda.current_stream()
    pixels = c.width * c.height

    def step(events=None):
        def mark(k):
            if events is not None:
                events[k].record(stream)
        mark(0)
        sp.project()
        mark(1)
        sp.bin_sort()
        mark(2)
        sp.rasterize_fwd()
        mark(3)
        sp.rasterize_bwd(dL, with_params=False)
        mark(4)
        sp.project_bwd()
        mark(5)
        sp.densify_stats()
        mark(6)
        sp.adam_step()  # with N > 1: reduce-scatter, Adam on the slice, all-gather
        mark(7)

    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize()
    assert sp.status() == api.GS_OK, "device status after warm-up"

    names = ["gs_project", "gs_bin_sort", "gs_rasterize_fwd", "gs_rasterize_bwd",
             "gs_project_bwd", "gs_densify_stats",
             "gs_adam_step" if world == 1 else "reduce_scatter+gs_adam_step+all_gather"]
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(len(names) + 1)]
          for _ in range(args.steps)]
    clocks = ClockSampler(local)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.3)
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for k in range(args.steps):
        step(ev[k])
    end.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    if world > 1:
        dist.barrier()
    elapsed_ms = gdist.max_over_ranks(start.elapsed_time(end), device="cuda")
    per_call = {nm: float(np.mean([ev[k][i].elapsed_time(ev[k][i + 1]) for k in range(args.steps)]))
                for i, nm in enumerate(names)}
    ms = elapsed_ms / args.steps
    value = world * pixels / (ms / 1000.0) / 1e6
    n_pairs = int(sp.n_pairs.item())
    status = sp.status()

    # end to end through the library's host-fed step (Splatter.train_from_host):
    # every step uploads its upstream gradient from pinned host memory and
    # downloads the rendered image to it, on a copy stream overlapping the
    # compute stream
    e2e = None
    if not args.no_e2e:
        h_in = torch.from_numpy(dL_host).pin_memory()
        h_out = torch.empty(sp.image.shape, dtype=torch.float32).pin_memory()
        sp.stream = torch.cuda.Stream()
        sp.train_from_host([h_in] * 3, [h_out] * 3)  # warm-up
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        e0.record(sp.stream)
        sp.train_from_host([h_in] * args.steps, [h_out] * args.steps)
        e1.record(sp.stream)
        torch.cuda.synchronize()
        sp.stream = None
        e_ms = gdist.max_over_ranks(e0.elapsed_time(e1) / args.steps, device="cuda")
        e2e = {"value": world * pixels / (e_ms / 1000.0) / 1e6, "unit": "Mpix/s",
               "ms_per_step": e_ms, "h2d_bytes_per_step": int(h_in.numel() * 4),
               "d2h_bytes_per_step": int(h_out.numel() * 4)}

    # densify_and_prune once, on the statistics the timed steps accumulated
    # (not part of the step: it runs every few hundred steps)
    extras = {}
    if world == 1:
        extras["gs_densify_and_prune"] = measure_densify(sp)
        extras["gs_l1_dssim"] = measure_loss(sp)
        extras["gs_adam_step_sh_quant"] = measure_quant_adam(sp)

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return 0

    # CPU baseline and the exp count of the blend kernels (oracle, rank 0, N=1)
    cpu = None
    exps = None
    if world == 1 and not args.no_cpu_baseline:
        cpu, nexp_mean = cpu_baseline(scene)
        exps = nexp_mean * pixels
    pk = peaks()
    work = algorithmic_work(sp, n_pairs, args.sort_mode, exps or 0.0)
    if world > 1:
        work["gs_adam_step"]["bytes"] /= world  # each rank updates its slice only
    kernels = {}
    for nm in names:
        if nm not in work:
            continue
        t = per_call[nm] / 1000.0
        w = work[nm]
        kernels[nm] = dict(ms=per_call[nm], gbs=w["bytes"] / t / 1e9,
                           hbm_frac=w["bytes"] / t / 1e9 / pk["hbm_gbs"])
        if w["exps"]:
            kernels[nm]["gexps"] = w["exps"] / t / 1e9
    dom = max(kernels, key=lambda k: kernels[k]["ms"])
    sm_for_peak = pk["sm_max_mhz"]
    t_hbm = work[dom]["bytes"] / (pk["hbm_gbs"] * 1e9)
    t_sfu = (work[dom]["exps"] / (sfu_peak_gexps(sm_for_peak) * 1e9)) if exps else 0.0
    if t_sfu > t_hbm:
        peak = sfu_peak_gexps(sm_for_peak)
        ach = work[dom]["exps"] / (per_call[dom] / 1000.0) / 1e9
        roof = {"kernel": dom, "bound": "alu", "achieved": ach, "peak": peak, "unit": "Gexp/s",
                "frac": ach / peak, "traffic": profiled_traffic(dom, WORKLOAD),
                "peak_source": "148 SM x 16 MUFU.EX2/clk x %.0f MHz (max SM clock)" % sm_for_peak}
    else:
        ach = work[dom]["bytes"] / (per_call[dom] / 1000.0) / 1e9
        roof = {"kernel": dom, "bound": "hbm", "achieved": ach, "peak": pk["hbm_gbs"],
                "unit": "GB/s", "frac": ach / pk["hbm_gbs"],
                "traffic": profiled_traffic(dom, WORKLOAD),
                "peak_source": pk["source"] + " (MEASURED_PEAKS.json copy bandwidth)"}
    # step roofline: sum over calls of max(bytes / HBM, exps / SFU)
    bound_s = 0.0
    for nm, w in work.items():
        bound_s += max(w["bytes"] / (pk["hbm_gbs"] * 1e9),
                       (w["exps"] / (sfu_peak_gexps(sm_for_peak) * 1e9)) if w["exps"] else 0.0)
    n_launch = launches_per_step(sp, args.sort_mode)
    line = {
        "metric": METRIC, "value": value, "unit": "Mpix/s", "n_gpus": world,
        "steps": args.steps, "warmup": max(args.warmup, 3), "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic",
        "config": {"workload": WORKLOAD, "gaussians": sp.n, "width": c.width, "height": c.height,
                   "sh_degree": 3, "views_per_gpu": 1, "pairs": n_pairs,
                   "sort_mode": args.sort_mode,
                   "sort_path": sort_plan(sp, args.sort_mode)["path"],
                   "l2": "working set larger than L2 (0.7 GB of parameters and Adam state "
                         "rewritten every step)",
                   "parallelism": "dp%d (one view per GPU; gradient reduce-scatter, Adam on "
                                  "1/%d of the parameters, parameter all-gather)" % (world, world)
                   if world > 1 else "single GPU"},
        "roofline": roof,
        "step_roofline": {"bound_ms": bound_s * 1000.0, "frac": bound_s * 1000.0 / ms},
        "kernels": kernels,
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
