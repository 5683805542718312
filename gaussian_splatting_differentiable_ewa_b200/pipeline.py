"""Buffers and call sequence of one training step, on top of the C ABI.

``Splatter`` owns the device buffers (allocated with torch, which is used for
nothing else besides streams and the collectives of the multi-GPU step) and
runs the calls in order: gs_project -> gs_bin_sort -> gs_rasterize_fwd ->
[gs_l1_dssim against a target image] -> gs_rasterize_bwd -> gs_densify_stats
-> gs_adam_step (or, with quantised SH, gs_adam_step_sh_quant for the SH), and
gs_densify_and_prune when asked. Every step of the computation runs in
libgs_b200.so.
"""

from __future__ import annotations

import contextlib
import math
from typing import Optional

import numpy as np
import torch

from . import api
from . import dist as gdist

# Per-group Adam learning rates of the 10M-Gaussian training workload.
DEFAULT_LR = dict(means=1.6e-4, sh=2.5e-3, opacity_logit=5e-2, log_scales=5e-3, quats=1e-3)

# The flat parameter / gradient / moment buffers are padded to a multiple of
# this many floats, so that they split into 16-byte aligned equal slices for
# any power-of-two number of ranks up to 256.
FLAT_PAD = 1024


class Splatter:
    def __init__(self, scene, device="cuda", sort_mode: int = api.GS_SORT_PRESORT,
                 pair_capacity: Optional[int] = None, headroom: float = 1.25,
                 lr: Optional[dict] = None, stream: Optional[torch.cuda.Stream] = None,
                 sh_bits: Optional[int] = None, sh_rounding: int = 0, sh_seed: int = 0):
        self.device = torch.device(device)
        self.sh_bits = sh_bits
        self.sh_rounding = int(sh_rounding)
        self.sh_seed = int(sh_seed)
        self._shard = None
        self.scene = scene
        self.n = int(scene.n)
        self.V = int(scene.n_views)
        self.deg = int(scene.sh_degree)
        self.K = (self.deg + 1) ** 2
        self.W = int(scene.cameras[0].width)
        self.H = int(scene.cameras[0].height)
        self.sort_mode = int(sort_mode)
        self.headroom = headroom
        self.lr = dict(DEFAULT_LR if lr is None else lr)
        self.stream = stream
        self.cams = api.cameras(scene.cameras)
        self.bg = [float(x) for x in scene.background]
        dev = self.device
        f32 = torch.float32

        def up(a, shape=None):
            t = torch.as_tensor(np.ascontiguousarray(a, np.float32))
            return (t if shape is None else t.reshape(shape)).to(dev).contiguous()

        self._alloc_gaussians(up(scene.means), up(scene.log_scales), up(scene.quats),
                              up(scene.opacity_logit), up(scene.sh, (self.n, self.K, 3)))
        V = self.V
        self.image = torch.empty((V, 3, self.H, self.W), dtype=f32, device=dev)
        self.final_T = torch.empty((V, self.H, self.W), dtype=f32, device=dev)
        self.n_contrib = torch.empty((V, self.H, self.W), dtype=torch.int32, device=dev)
        tiles = ((self.W + 15) // 16) * ((self.H + 15) // 16) * V
        self.ranges = torch.empty((tiles, 2), dtype=torch.int64, device=dev)
        self.n_pairs = torch.zeros(1, dtype=torch.int64, device=dev)
        self.capacity = 0
        self.ids = None
        self.ws = None
        self.step_count = 0
        self.loss_terms = None
        self._alloc_pairs(int(pair_capacity) if pair_capacity is not None else 0)

    # ------------------------------------------------------------ buffers
    def _alloc_gaussians(self, means, log_scales, quats, opacity_logit, sh, exp_avg=None,
                         exp_avg_sq=None, sh_state=None) -> None:
        """Adopt the given parameter values (and Adam moments, zero if None) and
        (re)allocate every buffer whose size follows the Gaussian count. With
        quantised SH, sh_state = (codes, bounds, exp_avg16, exp_avg_sq16) is
        adopted as the SH state (else sh is quantised afresh).

        Parameters, gradients and both moments each live in one flat buffer,
        every group at a 16-byte aligned offset (the same offsets in all four)
        and the total padded to a multiple of FLAT_PAD floats, so that one
        collective moves a whole buffer and equal 16-byte aligned slices of
        it can be handed to ranks."""
        dev, f32 = self.device, torch.float32
        self._gen = getattr(self, "_gen", 0) + 1
        src = [("means", means), ("log_scales", log_scales), ("quats", quats),
               ("opacity_logit", opacity_logit), ("sh", sh)]
        self.n = n = int(means.shape[0])
        V = self.V
        offs, total = gdist.flat_layout([(k, t.numel()) for k, t in src], FLAT_PAD)
        self.flat_offsets = offs
        self.flat_sizes = {k: t.numel() for k, t in src}
        self.flat_total = total

        def views(buf, names):
            return {k: buf[offs[k]:offs[k] + t.numel()].view(t.shape)
                    for k, t in src if k in names}

        names = [k for k, _ in src]
        self.param_flat = torch.zeros(total, dtype=f32, device=dev)
        P = views(self.param_flat, names)
        for k, t in src:
            P[k].copy_(t)
        self.means, self.log_scales, self.quats = P["means"], P["log_scales"], P["quats"]
        self.opacity_logit, self.sh = P["opacity_logit"], P["sh"]
        self.param_list = [(k, P[k]) for k in names]
        self.records = torch.empty((V, n, api.GS_RECORD_FLOATS), dtype=f32, device=dev)
        self.bins = torch.empty((V, n, 4), dtype=f32, device=dev)
        self.radii = torch.empty((V, n), dtype=torch.int32, device=dev)
        self.grad2d = torch.empty((V, n, api.GS_GRAD2D_FLOATS), dtype=f32, device=dev)
        self.grad_flat = torch.zeros(total, dtype=f32, device=dev)
        self.grads = views(self.grad_flat, names)
        # the moments: with quantised SH the SH moments live beside the codes,
        # so the float32 moment buffers stop before the SH group
        m_names = names[:-1] if self.sh_bits is not None else names
        m_total = offs["sh"] if self.sh_bits is not None else total
        self.m_flat = torch.zeros(max(m_total, 4), dtype=f32, device=dev)
        self.v_flat = torch.zeros(max(m_total, 4), dtype=f32, device=dev)
        self.exp_avg = views(self.m_flat, m_names)
        self.exp_avg_sq = views(self.v_flat, m_names)
        for given, mine in ((exp_avg, self.exp_avg), (exp_avg_sq, self.exp_avg_sq)):
            if given is not None:
                for k in m_names:
                    mine[k].copy_(given[k])
        if self.sh_bits is not None:
            self.exp_avg["sh"] = self.exp_avg_sq["sh"] = None
        if self.sh_bits is not None:
            self._quantise_sh(sh_state)
        self.accum_plain = torch.zeros(n, dtype=f32, device=dev)
        self.accum_abs = torch.zeros(n, dtype=f32, device=dev)
        self.denom = torch.zeros(n, dtype=torch.int32, device=dev)
        # with quantised SH the kernels read the codes themselves
        quant = self.sh_bits is not None
        self.c_params = api.params(self.means, self.log_scales, self.quats, self.opacity_logit,
                                   None if quant else self.sh, self.deg,
                                   sh_quant=self.sh_q if quant else None)
        self.c_grads = api.grads(*[self.grads[k] for k, _ in self.param_list])
        self.c_m = api.grads(*[self.exp_avg[k] for k, _ in self.param_list])
        self.c_v = api.grads(*[self.exp_avg_sq[k] for k, _ in self.param_list])
        self.c_proj = api.projected(self.records, self.bins, self.radii)
        if getattr(self, "_shard", None) is not None:
            self._plan_shard()  # the slices follow the buffer size
        if getattr(self, "ws", None) is not None:
            self._alloc_pairs(self.capacity)  # the workspace follows the count too

    def _quantise_sh(self, state=None) -> None:
        """Quantised SH state: the SH live as codes with per-256 bounds and
        bfloat16 Adam moments, which the projection and its backward decode
        where they use them; ``self.sh`` holds the decoded float32 values
        for inspection (refresh_sh_float)."""
        if self.sh_bits not in (8, 16):
            raise ValueError("sh_bits must be 8 or 16")
        n, k3, dev = self.n, 3 * self.K, self.device
        n_pad = -(-n // api.GS_QUANT_GROUP) * api.GS_QUANT_GROUP
        if state is None:
            self.sh_codes = torch.zeros((k3, n_pad), device=dev,
                                        dtype=torch.uint8 if self.sh_bits == 8 else torch.int16)
            self.sh_bounds = torch.zeros((k3, n_pad // api.GS_QUANT_GROUP, 2),
                                         dtype=torch.float32, device=dev)
            self.sh_m16 = torch.zeros((k3, n_pad), dtype=torch.int16, device=dev)
            self.sh_v16 = torch.zeros((k3, n_pad), dtype=torch.int16, device=dev)
        else:
            self.sh_codes, self.sh_bounds, self.sh_m16, self.sh_v16 = state
        self.sh_q = api.sh_quant(self.sh_codes, self.sh_bounds, n, k3, self.sh_bits)
        if state is None:
            api.gs_sh_quantize(self.sh, self.sh_q, self.stream)
        self.refresh_sh_float()

    def refresh_sh_float(self) -> None:
        """Quantised SH: decode the codes into ``self.sh``."""
        api.gs_sh_dequantize(self.sh_q, self.sh, self.stream)

    def _alloc_pairs(self, capacity: int) -> None:
        self._gen = getattr(self, "_gen", 0) + 1  # captured graphs name the old buffers
        self.capacity = int(capacity)
        self.ids = torch.empty(max(self.capacity, 1), dtype=torch.int32, device=self.device)
        # the forward's per-entry warp masks, reused by the backward
        self.warp_masks = torch.empty(max(self.capacity, 1), dtype=torch.uint8, device=self.device)
        nbytes = api.gs_workspace_size(self.n, self.cams, self.V, self.capacity, self.sort_mode)
        if nbytes == 0:
            raise ValueError("invalid workspace request")
        self.ws = torch.zeros((nbytes + 255) // 256 * 256 // 8, dtype=torch.int64,
                              device=self.device)
        self.c_bins = api.binned(self.ids, self.ranges, self.n_pairs, self.capacity)

    def workspace_bytes(self) -> int:
        return int(self.ws.numel() * 8)

    def ensure_capacity(self) -> int:
        """Project and bin once, growing the pair buffers until they fit."""
        self.project()
        self.bin_sort()
        torch.cuda.synchronize(self.device)
        need = int(self.n_pairs.item())
        api.gs_get_status(self.ws, self.stream)  # clear a capacity flag from sizing
        if need > self.capacity:
            self._alloc_pairs(int(math.ceil(need * self.headroom)) + 1024)
            self.project()
            self.bin_sort()
        return need

    # ------------------------------------------------------------ the calls
    def project(self):
        api.gs_project(self.c_params, self.cams, self.V, self.c_proj, self.ws, self.stream)

    def bin_sort(self):
        api.gs_bin_sort(self.c_proj, self.cams, self.V, self.n, self.sort_mode, self.c_bins,
                        self.ws, self.stream)

    def rasterize_fwd(self, image: Optional[torch.Tensor] = None):
        """Render into ``self.image`` (or `image`, a tensor of its shape)."""
        api.gs_rasterize_fwd(self.c_proj, self.c_bins, self.cams, self.V, self.n, self.bg,
                             self.image if image is None else image, self.final_T,
                             self.n_contrib, self.ws, self.stream, warp_masks=self.warp_masks)

    def rasterize_bwd(self, dL_dimage: torch.Tensor, with_params: bool = True):
        api.gs_rasterize_bwd(self.c_params, self.c_proj, self.c_bins, self.cams, self.V, self.bg,
                             dL_dimage, self.final_T, self.n_contrib, self.grad2d,
                             self.c_grads if with_params else None, self.ws, self.stream,
                             warp_masks=self.warp_masks)

    def project_bwd(self):
        api.gs_project_bwd(self.c_params, self.cams, self.V, self.radii, self.grad2d,
                           self.c_grads, self.stream)

    def fused_tail_ok(self) -> bool:
        """Whether project_bwd_adam can end a step: one GPU's optimiser over
        float32 SH."""
        return self._shard is None and self.sh_bits is None

    def project_bwd_adam(self, beta1=0.9, beta2=0.999, eps=1e-15, stats: bool = True):
        """The step's tail in one launch (gs_project_bwd_adam): projection
        backward from ``self.grad2d``, densification statistics (unless
        stats is False) and the Adam step, the parameters updated in place;
        the gradients are not materialised."""
        if not self.fused_tail_ok():
            raise ValueError("the fused tail needs an unsharded optimiser and float32 SH")
        self.step_count += 1
        names = [k for k, _ in self.param_list]
        api.gs_project_bwd_adam(self.c_params, self.cams, self.V, self.radii, self.grad2d,
                                self.c_m, self.c_v, [self.lr[k] for k in names], beta1, beta2,
                                eps, self.step_count, self.accum_plain if stats else None,
                                self.accum_abs if stats else None,
                                self.denom if stats else None, self.stream)

    def densify_stats(self):
        api.gs_densify_stats(self.grad2d, self.radii, self.V, self.n, self.accum_plain,
                             self.accum_abs, self.denom, self.stream)

    def adam_step(self, beta1=0.9, beta2=0.999, eps=1e-15):
        self.step_count += 1
        if self._shard is not None:
            self._sharded_adam_step(beta1, beta2, eps)
            return
        quant = self.sh_bits is not None
        groups = [(t, self.grads[k], self.exp_avg[k], self.exp_avg_sq[k], self.lr[k])
                  for k, t in self.param_list if not (quant and k == "sh")]
        api.gs_adam_step(groups, beta1, beta2, eps, self.step_count, self.stream)
        if quant:
            api.gs_adam_step_sh_quant(self.sh_q, self.grads["sh"], self.sh_m16, self.sh_v16,
                                      self.lr["sh"], beta1, beta2, eps, self.step_count,
                                      self.sh_rounding, self.sh_seed, self.stream)

    # ------------------------------------------------------------ sharded optimiser
    def shard_optimizer(self, rank: int, world: int, group=None) -> None:
        """Shard the Adam step over `world` ranks that each render their own
        views of the same Gaussians (torch.distributed initialised, NCCL on
        GPUs). adam_step then reduce-scatters the flat gradient buffer (every
        rank gets the sum over ranks of its slice), runs Adam on this rank's
        contiguous slice of the flat parameter buffer only, and all-gathers
        the parameters, so every rank ends the step with the same parameters.
        The moments outside the slice are not kept current on this rank;
        densify_and_prune gathers them first. world == 1 needs no process
        group and runs the same slice logic over the whole buffer."""
        if self.sh_bits is not None:
            raise NotImplementedError("sharded optimiser with quantised SH state")
        self._shard = dict(rank=int(rank), world=int(world), group=group)
        self._plan_shard()

    def _plan_shard(self) -> None:
        sh = self._shard
        lo, hi = gdist.shard_bounds(self.flat_total, sh["rank"], sh["world"])
        sh["lo"], sh["hi"] = lo, hi
        sh["slices"] = gdist.shard_slices(self.flat_offsets, self.flat_sizes, lo, hi)
        if sh["world"] > 1:
            self._grad_shard = torch.empty(hi - lo, dtype=torch.float32, device=self.device)
            self._param_shard = torch.empty(hi - lo, dtype=torch.float32, device=self.device)

    def _torch_stream(self):
        return (torch.cuda.stream(self.stream) if self.stream is not None
                else contextlib.nullcontext())

    def _sharded_adam_step(self, beta1, beta2, eps) -> None:
        import torch.distributed as dist
        sh = self._shard
        lo, hi, world, group = sh["lo"], sh["hi"], sh["world"], sh["group"]
        if world > 1:
            with self._torch_stream():
                dist.reduce_scatter_tensor(self._grad_shard, self.grad_flat, group=group)
            gsl = self._grad_shard
        else:
            gsl = self.grad_flat[lo:hi]
        groups = [(self.param_flat[a:b], gsl[a - lo:b - lo], self.m_flat[a:b], self.v_flat[a:b],
                   self.lr[k]) for k, a, b in sh["slices"]]
        if groups:
            api.gs_adam_step(groups, beta1, beta2, eps, self.step_count, self.stream)
        if world > 1:
            with self._torch_stream():
                self._param_shard.copy_(self.param_flat[lo:hi])
                dist.all_gather_into_tensor(self.param_flat, self._param_shard, group=group)

    def _gather_for_densify(self) -> None:
        """Before densify_and_prune on several ranks: the summed view-space
        statistics and, when the optimiser is sharded, every rank's slice of
        the moments (gdist.gather_for_densify)."""
        sh = self._shard
        with self._torch_stream():
            gdist.gather_for_densify(
                (self.accum_plain, self.accum_abs, self.denom), (self.m_flat, self.v_flat),
                None if sh is None else (sh["lo"], sh["hi"]),
                None if sh is None else sh["group"])

    def _graph_of(self, fn) -> "torch.cuda.CUDAGraph":
        """A CUDA graph of one fixed-shape call: run once outside capture (on
        a capture stream ordered after the current one), then captured."""
        saved = self.stream
        cap = torch.cuda.Stream(device=self.device)
        cap.wait_stream(torch.cuda.current_stream(self.device))
        if saved is not None:
            cap.wait_stream(saved)
        try:
            with torch.cuda.stream(cap):
                self.stream = cap
                fn()
            cap.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=cap):
                self.stream = cap
                fn()
        finally:
            self.stream = saved
        torch.cuda.current_stream(self.device).wait_stream(cap)
        if saved is not None:
            saved.wait_stream(cap)
        return g

    def capture_calls(self, dL_dimage: Optional[torch.Tensor] = None) -> dict:
        """CUDA graphs of this Splatter's fixed-shape calls: 'project',
        'bin_sort', 'rasterize_fwd' and, given an upstream gradient,
        'rasterize_bwd' (screen space), 'project_bwd' and 'densify_stats'.
        Every size and pointer of those calls is fixed once ensure_capacity has
        sized the buffers, so a graph replays the call's kernels with no host
        launch gaps between them (gs_bin_sort alone is up to 17 launches).
        Replays run on the current stream. The Adam step (fused or not) is not
        captured: its bias corrections follow the step count, a host value of
        the call. The graphs stay valid until a buffer is reallocated
        (ensure_capacity growing the pairs, densify_and_prune)."""
        calls = {"project": self.project, "bin_sort": self.bin_sort,
                 "rasterize_fwd": self.rasterize_fwd}
        if dL_dimage is not None:
            calls["rasterize_bwd"] = lambda: self.rasterize_bwd(dL_dimage, with_params=False)
            calls["project_bwd"] = self.project_bwd
            calls["densify_stats"] = self.densify_stats
        return {name: self._graph_of(fn) for name, fn in calls.items()}

    def forward(self):
        self.project()
        self.bin_sort()
        self.rasterize_fwd()

    def _backward_tail(self, dL_dimage: torch.Tensor, adam: bool) -> None:
        # with Adam on one GPU and float SH: screen-space backward, then the
        # fused projection backward + statistics + Adam (no gradient arrays)
        if adam and self.fused_tail_ok():
            self.rasterize_bwd(dL_dimage, with_params=False)
            self.project_bwd_adam()
            return
        self.rasterize_bwd(dL_dimage)
        self.densify_stats()
        if adam:
            self.adam_step()

    def train_step(self, dL_dimage: torch.Tensor, adam: bool = True):
        """Render, backward, densification statistics and (with adam) the
        Adam step; ``self.grads`` is written only on the unfused path
        (adam False, a sharded optimiser or quantised SH)."""
        self.forward()
        self._backward_tail(dL_dimage, adam)

    def loss(self, target: torch.Tensor, lam: float = 0.2, grad: bool = True) -> torch.Tensor:
        """(1 - lam) L1 + lam (1 - SSIM) of the rendered image against
        `target` ([V, 3, H, W] float32 on the device). Leaves the per-view
        terms (loss, mean L1, mean SSIM) in ``self.loss_terms`` and, with
        `grad`, dL/dimage in ``self.dL_loss``; returns ``self.loss_terms``."""
        if tuple(target.shape) != tuple(self.image.shape) or target.dtype != torch.float32:
            raise ValueError("target must be float32 of the image's shape")
        if self.loss_terms is None:
            self.loss_terms = torch.empty((self.V, 3), dtype=torch.float64, device=self.device)
            self.dL_loss = torch.empty_like(self.image)
            nb = api.gs_l1_dssim_workspace_size(self.V)
            self._loss_ws = torch.empty((nb + 7) // 8, dtype=torch.float64, device=self.device)
        api.gs_l1_dssim(self.image, target.contiguous(), self.V, self.H, self.W, lam,
                        self.loss_terms, self.dL_loss if grad else None, self._loss_ws,
                        self.stream)
        return self.loss_terms

    def train_step_target(self, target: torch.Tensor, lam: float = 0.2, adam: bool = True):
        """One training step on target images: render, the L1 + D-SSIM loss
        and its image gradient, then the backward, statistics and Adam."""
        self.forward()
        self.loss(target, lam)
        self._backward_tail(self.dL_loss, adam)

    def train_from_host(self, dL_host, image_host, adam: bool = True, grad_hook=None) -> None:
        """Training steps fed from host memory, copies overlapped with compute.

        Step k uploads ``dL_host[k]`` (pinned, [V][3][H][W] float32), runs one
        training step and downloads the rendered image into ``image_host[k]``
        (pinned). The copies run on two streams of their own, one per
        direction, so that an upload and a download proceed together: step
        k + 1's gradient uploads (into the other of two device buffers) as
        soon as step k - 1's backward is done with that buffer, and step k's
        image downloads while its backward runs; events order the next
        forward after that download and each backward after its upload.
        Everything is enqueued; the caller synchronises. ``self.stream`` must
        be a stream other than the legacy default stream (which would
        serialise them). ``grad_hook()``, if given, runs on the compute
        stream between the backward and the statistics (e.g. a gradient clip;
        the multi-GPU exchange is part of adam_step once shard_optimizer was
        called)."""
        comp = self.stream
        if comp is None:
            raise ValueError("train_from_host needs Splatter(stream=...) on a created stream")
        n = len(dL_host)
        if n != len(image_host):
            raise ValueError("one image buffer per gradient")
        if getattr(self, "_copy_streams", None) is None:
            self._copy_streams = (torch.cuda.Stream(device=self.device),
                                  torch.cuda.Stream(device=self.device))
            self._dL_dev = [torch.empty((self.V, 3, self.H, self.W), dtype=torch.float32,
                                        device=self.device) for _ in range(2)]
        up, down = self._copy_streams
        # one CUDA graph per fixed-shape call (two for the backward, one per
        # gradient buffer), kept until a buffer is reallocated
        hg = getattr(self, "_host_graphs", None)
        if hg is None or hg[0] != self._gen:
            gr = {"project": self._graph_of(self.project),
                  "bin_sort": self._graph_of(self.bin_sort),
                  "rasterize_fwd": self._graph_of(self.rasterize_fwd)}
            for b in range(2):
                gr["bwd%d" % b] = self._graph_of(
                    lambda b=b: self.rasterize_bwd(self._dL_dev[b], with_params=False))
            self._host_graphs = hg = (self._gen, gr)
        gr = hg[1]

        def run(name, fn):
            with torch.cuda.stream(comp):
                gr[name].replay() if name in gr else fn()

        uploaded = [torch.cuda.Event(), torch.cuda.Event()]
        consumed = [torch.cuda.Event(), torch.cuda.Event()]
        rendered = torch.cuda.Event()
        downloaded = torch.cuda.Event()
        up.wait_stream(comp)  # nothing earlier on the compute stream is overtaken
        down.wait_stream(comp)
        with torch.cuda.stream(up):
            self._dL_dev[0].copy_(dL_host[0], non_blocking=True)
            uploaded[0].record(up)
        for k in range(n):
            buf = k & 1
            if k + 1 < n:  # the next step's gradient, once its buffer is free
                if k >= 1:
                    up.wait_event(consumed[buf ^ 1])  # step k - 1's backward is done with it
                with torch.cuda.stream(up):
                    self._dL_dev[buf ^ 1].copy_(dL_host[k + 1], non_blocking=True)
                    uploaded[buf ^ 1].record(up)
            run("project", self.project)
            run("bin_sort", self.bin_sort)
            if k > 0:
                comp.wait_event(downloaded)  # the previous image has left
            run("rasterize_fwd", self.rasterize_fwd)
            rendered.record(comp)
            down.wait_event(rendered)
            with torch.cuda.stream(down):
                image_host[k].copy_(self.image, non_blocking=True)
                downloaded.record(down)
            comp.wait_event(uploaded[buf])
            # without a hook on the gradients the tail is the fused one
            fused = adam and grad_hook is None and self.fused_tail_ok()
            if fused:
                run("bwd%d" % buf, None)
            else:
                self.rasterize_bwd(self._dL_dev[buf])
            consumed[buf].record(comp)
            if fused:
                self.project_bwd_adam()
                continue
            if grad_hook is not None:
                with torch.cuda.stream(comp):
                    grad_hook()
            self.densify_stats()
            if adam:
                self.adam_step()
        comp.wait_event(downloaded)  # the last image is on the host when comp is done

    def render_to_host(self, image_host) -> None:
        """Forward renders delivered to host memory, copies overlapped with
        compute: step k renders into one of two device image buffers and
        downloads it into ``image_host[k]`` (pinned, [V][3][H][W] float32) on a
        second stream while step k + 1 projects, sorts and renders into the
        other buffer; a render waits only for the download of the buffer it
        reuses (step k - 1's). The calls replay as CUDA graphs, kept until a
        buffer is reallocated. Everything is enqueued; the caller
        synchronises; ``self.image`` ends up holding the last image.
        ``self.stream`` must be a created stream (see train_from_host)."""
        comp = self.stream
        if comp is None:
            raise ValueError("render_to_host needs Splatter(stream=...) on a created stream")
        if getattr(self, "_copy_stream", None) is None:
            self._copy_stream = torch.cuda.Stream(device=self.device)
        cs = self._copy_stream
        rg = getattr(self, "_render_graphs", None)
        if rg is None or rg[0] != self._gen:
            imgs = [self.image, torch.empty_like(self.image)]
            gr = {"project": self._graph_of(self.project),
                  "bin_sort": self._graph_of(self.bin_sort)}
            for b in range(2):
                gr["fwd%d" % b] = self._graph_of(lambda b=b: self.rasterize_fwd(imgs[b]))
            self._render_graphs = rg = (self._gen, gr, imgs)
        gr, imgs = rg[1], rg[2]
        rendered = torch.cuda.Event()
        downloaded = [torch.cuda.Event(), torch.cuda.Event()]
        cs.wait_stream(comp)
        n = len(image_host)
        with torch.cuda.stream(comp):
            for k in range(n):
                b = k & 1
                gr["project"].replay()
                gr["bin_sort"].replay()
                if k > 1:
                    comp.wait_event(downloaded[b])  # step k - 2's image has left this buffer
                gr["fwd%d" % b].replay()
                rendered.record(comp)
                cs.wait_event(rendered)
                with torch.cuda.stream(cs):
                    image_host[k].copy_(imgs[b], non_blocking=True)
                    downloaded[b].record(cs)
            if n > 0:
                if (n - 1) & 1:
                    self.image.copy_(imgs[1])
                comp.wait_event(downloaded[(n - 1) & 1])

    def densify_and_prune(self, grad_threshold: float = 0.0002, scale_split: float = 0.05,
                          min_opacity: float = 0.005, max_scale: float = 1.0,
                          split_shrink: float = 1.6, use_abs: bool = True, z=None,
                          seed: int = 0) -> torch.Tensor:
        """Clone, split and prune (gs_densify_and_prune) with this Splatter's
        accumulated view-space gradient statistics (the absolute ones when
        use_abs, else the plain ones), then adopt the new Gaussian set: every
        per-Gaussian buffer is reallocated and the statistics restart from
        zero. z: standard normal draws float32 [n][2][3] for the split
        children (drawn on the device from `seed` when None). Returns the
        per-Gaussian codes (0 pruned, 1 kept, 2 cloned, 3 split). With
        quantised SH, gs_densify_sh_quant builds the new SH state from the
        codes (decoded values gathered, groups encoded anew)."""
        quant = self.sh_bits is not None
        self._gather_for_densify()
        n, dev = self.n, self.device
        if z is None:
            gen = torch.Generator(device=dev)
            gen.manual_seed(int(seed))
            z = torch.randn((n, 2, 3), generator=gen, device=dev, dtype=torch.float32)
        cap = 2 * n
        names = [k for k, _ in self.param_list]

        def like(t):
            return torch.empty((cap,) + tuple(t.shape[1:]), dtype=t.dtype, device=dev)

        out = {k: like(t) for k, t in self.param_list}
        m_out = {k: like(t) for k, t in self.param_list if not (quant and k == "sh")}
        v_out = {k: like(t) for k, t in self.param_list if not (quant and k == "sh")}
        grads_of = lambda d: api.grads(*[d.get(k) for k in names])  # noqa: E731
        n_out = torch.zeros(1, dtype=torch.int64, device=dev)
        codes = torch.empty(max(n, 1), dtype=torch.int8, device=dev)
        ws = torch.zeros((api.gs_densify_workspace_size(n) + 255) // 256 * 256 // 8,
                         dtype=torch.int64, device=dev)
        dp = api.densify_params(grad_threshold, scale_split, min_opacity, max_scale, split_shrink)
        api.gs_densify_and_prune(self.c_params, grads_of(self.exp_avg), grads_of(self.exp_avg_sq),
                                 self.accum_abs if use_abs else self.accum_plain, self.denom,
                                 z, dp, grads_of(out), grads_of(m_out), grads_of(v_out), cap,
                                 n_out, codes, ws, self.stream)
        st = api.gs_get_status(ws, self.stream)
        if st != api.GS_OK:
            raise api.GsError(st, "gs_densify_and_prune")
        m = int(n_out.item())
        keep = lambda d: {k: d[k][:m] for k in d}  # noqa: E731
        o, mo, vo = keep(out), keep(m_out), keep(v_out)
        sh_state = None
        if quant:
            k3 = 3 * self.K
            m_pad = -(-m // api.GS_QUANT_GROUP) * api.GS_QUANT_GROUP
            state = (torch.zeros((k3, m_pad), device=dev, dtype=self.sh_codes.dtype),
                     torch.zeros((k3, m_pad // api.GS_QUANT_GROUP, 2), dtype=torch.float32,
                                 device=dev),
                     torch.zeros((k3, m_pad), dtype=torch.int16, device=dev),
                     torch.zeros((k3, m_pad), dtype=torch.int16, device=dev))
            q_out = api.sh_quant(state[0], state[1], m, k3, self.sh_bits)
            ws2 = torch.zeros((api.gs_densify_sh_quant_workspace_size(n, m) + 255) // 256 * 256
                              // 8, dtype=torch.int64, device=dev)
            api.gs_densify_sh_quant(self.sh_q, self.sh_m16, self.sh_v16, codes, q_out, state[2],
                                    state[3], ws2, self.stream)
            st = api.gs_get_status(ws2, self.stream)
            if st != api.GS_OK:
                raise api.GsError(st, "gs_densify_sh_quant")
            sh_state = state  # o["sh"] is not written: the decode of the new codes fills it
        self._alloc_gaussians(o["means"], o["log_scales"], o["quats"], o["opacity_logit"],
                              o["sh"], mo, vo, sh_state=sh_state)
        return codes[:n]

    def status(self) -> int:
        return api.gs_get_status(self.ws, self.stream)
