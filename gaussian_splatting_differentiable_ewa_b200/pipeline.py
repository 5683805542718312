"""Buffers and call sequence of one training step, on top of the C ABI.

``Splatter`` owns the device buffers (allocated once with torch, the only
thing torch is used for besides streams) and runs the six calls in order:
gs_project -> gs_bin_sort -> gs_rasterize_fwd -> gs_rasterize_bwd ->
gs_densify_stats -> gs_adam_step. Every step of the computation runs in
libgs_b200.so.
"""

from __future__ import annotations

import math
from typing import Optional

import numpy as np
import torch

from . import api

# Per-group Adam learning rates of the 10M-Gaussian training workload.
DEFAULT_LR = dict(means=1.6e-4, sh=2.5e-3, opacity_logit=5e-2, log_scales=5e-3, quats=1e-3)


class Splatter:
    def __init__(self, scene, device="cuda", sort_mode: int = api.GS_SORT_PRESORT,
                 pair_capacity: Optional[int] = None, headroom: float = 1.25,
                 lr: Optional[dict] = None, stream: Optional[torch.cuda.Stream] = None):
        self.device = torch.device(device)
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

        self.means = up(scene.means)
        self.log_scales = up(scene.log_scales)
        self.quats = up(scene.quats)
        self.opacity_logit = up(scene.opacity_logit)
        self.sh = up(scene.sh, (self.n, self.K, 3))
        self.param_list = [("means", self.means), ("log_scales", self.log_scales),
                           ("quats", self.quats), ("opacity_logit", self.opacity_logit),
                           ("sh", self.sh)]
        n, V = self.n, self.V
        self.records = torch.empty((V, n, api.GS_RECORD_FLOATS), dtype=f32, device=dev)
        self.bins = torch.empty((V, n, 4), dtype=f32, device=dev)
        self.radii = torch.empty((V, n), dtype=torch.int32, device=dev)
        self.image = torch.empty((V, 3, self.H, self.W), dtype=f32, device=dev)
        self.final_T = torch.empty((V, self.H, self.W), dtype=f32, device=dev)
        self.n_contrib = torch.empty((V, self.H, self.W), dtype=torch.int32, device=dev)
        self.grad2d = torch.empty((V, n, api.GS_GRAD2D_FLOATS), dtype=f32, device=dev)
        # gradients live in one flat buffer (one all-reduce across ranks), each
        # group at a 16-byte aligned offset
        offs, total = {}, 0
        for k, t in self.param_list:
            offs[k] = total
            total += (t.numel() + 3) // 4 * 4
        self.grad_flat = torch.zeros(max(total, 4), dtype=f32, device=dev)
        self.grads = {k: self.grad_flat[offs[k]:offs[k] + t.numel()].view(t.shape)
                      for k, t in self.param_list}
        self.exp_avg = {k: torch.zeros_like(t) for k, t in self.param_list}
        self.exp_avg_sq = {k: torch.zeros_like(t) for k, t in self.param_list}
        self.accum_plain = torch.zeros(n, dtype=f32, device=dev)
        self.accum_abs = torch.zeros(n, dtype=f32, device=dev)
        self.denom = torch.zeros(n, dtype=torch.int32, device=dev)
        tiles = ((self.W + 15) // 16) * ((self.H + 15) // 16) * V
        self.ranges = torch.empty((tiles, 2), dtype=torch.int64, device=dev)
        self.n_pairs = torch.zeros(1, dtype=torch.int64, device=dev)
        self.capacity = 0
        self.ids = None
        self.ws = None
        self.step_count = 0
        self.c_params = api.params(self.means, self.log_scales, self.quats, self.opacity_logit,
                                   self.sh, self.deg)
        self.c_grads = api.grads(*[self.grads[k] for k, _ in self.param_list])
        self.c_proj = api.projected(self.records, self.bins, self.radii)
        self._alloc_pairs(int(pair_capacity) if pair_capacity is not None else 0)

    # ------------------------------------------------------------ buffers
    def _alloc_pairs(self, capacity: int) -> None:
        self.capacity = int(capacity)
        self.ids = torch.empty(max(self.capacity, 1), dtype=torch.int32, device=self.device)
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
        api.gs_project(self.c_params, self.cams, self.V, self.c_proj, self.stream)

    def bin_sort(self):
        api.gs_bin_sort(self.c_proj, self.cams, self.V, self.n, self.sort_mode, self.c_bins,
                        self.ws, self.stream)

    def rasterize_fwd(self):
        api.gs_rasterize_fwd(self.c_proj, self.c_bins, self.cams, self.V, self.n, self.bg,
                             self.image, self.final_T, self.n_contrib, self.stream)

    def rasterize_bwd(self, dL_dimage: torch.Tensor, with_params: bool = True):
        api.gs_rasterize_bwd(self.c_params, self.c_proj, self.c_bins, self.cams, self.V, self.bg,
                             dL_dimage, self.final_T, self.n_contrib, self.grad2d,
                             self.c_grads if with_params else None, self.stream)

    def project_bwd(self):
        api.gs_project_bwd(self.c_params, self.cams, self.V, self.radii, self.grad2d,
                           self.c_grads, self.stream)

    def densify_stats(self):
        api.gs_densify_stats(self.grad2d, self.radii, self.V, self.n, self.accum_plain,
                             self.accum_abs, self.denom, self.stream)

    def adam_step(self, beta1=0.9, beta2=0.999, eps=1e-15):
        self.step_count += 1
        groups = [(t, self.grads[k], self.exp_avg[k], self.exp_avg_sq[k], self.lr[k])
                  for k, t in self.param_list]
        api.gs_adam_step(groups, beta1, beta2, eps, self.step_count, self.stream)

    def forward(self):
        self.project()
        self.bin_sort()
        self.rasterize_fwd()

    def train_step(self, dL_dimage: torch.Tensor, adam: bool = True):
        self.forward()
        self.rasterize_bwd(dL_dimage)
        self.densify_stats()
        if adam:
            self.adam_step()

    def train_from_host(self, dL_host, image_host, adam: bool = True, grad_hook=None) -> None:
        """Training steps fed from host memory, copies overlapped with compute.

        Step k uploads ``dL_host[k]`` (pinned, [V][3][H][W] float32), runs one
        training step and downloads the rendered image into ``image_host[k]``
        (pinned). The copies run on a second stream: step k + 1's gradient
        uploads (into the other of two device buffers) while step k computes,
        and step k's image downloads while its backward runs; events order the
        next forward after that download and each upload after the backward
        that last read its buffer. Everything is enqueued; the caller
        synchronises. ``self.stream`` must be a stream other than the legacy
        default stream (which would serialise the two). ``grad_hook()``, if
        given, runs on the compute stream between the backward and the
        statistics (e.g. the gradient all-reduce of a multi-GPU step)."""
        comp = self.stream
        if comp is None:
            raise ValueError("train_from_host needs Splatter(stream=...) on a created stream")
        n = len(dL_host)
        if n != len(image_host):
            raise ValueError("one image buffer per gradient")
        if getattr(self, "_copy_stream", None) is None:
            self._copy_stream = torch.cuda.Stream(device=self.device)
            self._dL_dev = [torch.empty((self.V, 3, self.H, self.W), dtype=torch.float32,
                                        device=self.device) for _ in range(2)]
        cs = self._copy_stream
        uploaded = [torch.cuda.Event(), torch.cuda.Event()]
        consumed = [torch.cuda.Event(), torch.cuda.Event()]
        rendered = torch.cuda.Event()
        downloaded = torch.cuda.Event()
        cs.wait_stream(comp)  # nothing earlier on the compute stream is overtaken
        with torch.cuda.stream(cs):
            self._dL_dev[0].copy_(dL_host[0], non_blocking=True)
            uploaded[0].record(cs)
        for k in range(n):
            buf = k & 1
            self.project()
            self.bin_sort()
            if k > 0:
                comp.wait_event(downloaded)  # the previous image has left
            self.rasterize_fwd()
            rendered.record(comp)
            cs.wait_event(rendered)
            with torch.cuda.stream(cs):
                image_host[k].copy_(self.image, non_blocking=True)
                downloaded.record(cs)
                if k + 1 < n:
                    if k >= 1:
                        cs.wait_event(consumed[buf ^ 1])  # step k - 1's backward is done with it
                    self._dL_dev[buf ^ 1].copy_(dL_host[k + 1], non_blocking=True)
                    uploaded[buf ^ 1].record(cs)
            comp.wait_event(uploaded[buf])
            self.rasterize_bwd(self._dL_dev[buf])
            consumed[buf].record(comp)
            if grad_hook is not None:
                with torch.cuda.stream(comp):
                    grad_hook()
            self.densify_stats()
            if adam:
                self.adam_step()
        comp.wait_event(downloaded)  # the last image is on the host when comp is done

    def status(self) -> int:
        return api.gs_get_status(self.ws, self.stream)
