"""ctypes binding of ``libgs_b200.so`` -- the C ABI declared in ``include/gs.h``.

Argument marshalling only: every step of the path runs in the library's CUDA
kernels. The structs mirror gs.h field for field; the functions keep the C
names. Loading fails loudly when the library has not been built -- there is
no fallback implementation.
"""

from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libgs_b200.so")

GS_OK = 0
GS_ERR_INVALID_ARG = 1
GS_ERR_CAPACITY = 2
GS_ERR_OVERFLOW = 3
GS_ERR_DEVICE_TIMEOUT = 4
GS_ERR_NONFINITE = 5
GS_ERR_CUDA = 6

GS_SORT_FULL64 = 0
GS_SORT_PRESORT = 1

# bits of the device status word
GS_STATUS_BIT_CAPACITY = 1
GS_STATUS_BIT_TIMEOUT = 2
GS_STATUS_BIT_BOUNDS = 4
GS_STATUS_BIT_NONFINITE = 8

# gs_debug_stall sites
GS_STALL_NONE, GS_STALL_EMIT_LOOKBACK, GS_STALL_RASTER_FWD, GS_STALL_RASTER_BWD = 0, 1, 2, 3
GS_STALL_SORT_LOOKBACK = 4

GS_TILE = 16
GS_MAX_VIEWS = 32
GS_RECORD_FLOATS = 16
GS_GRAD2D_FLOATS = 12

_c = ctypes
_vp = _c.c_void_p


class GsCamera(_c.Structure):
    _fields_ = [("viewmat", _c.c_float * 12), ("fx", _c.c_float), ("fy", _c.c_float),
                ("cx", _c.c_float), ("cy", _c.c_float), ("width", _c.c_int32),
                ("height", _c.c_int32), ("campos", _c.c_float * 3), ("reserved", _c.c_float)]


class GsParams(_c.Structure):
    _fields_ = [("means", _vp), ("log_scales", _vp), ("quats", _vp), ("opacity_logit", _vp),
                ("sh", _vp), ("sh_degree", _c.c_int32), ("reserved", _c.c_int32),
                ("n", _c.c_int64), ("sh_quant", _vp)]


class GsGrads(_c.Structure):
    _fields_ = [("means", _vp), ("log_scales", _vp), ("quats", _vp), ("opacity_logit", _vp),
                ("sh", _vp)]


class GsProjected(_c.Structure):
    _fields_ = [("records", _vp), ("bins", _vp), ("radii", _vp)]


class GsBinned(_c.Structure):
    _fields_ = [("ids", _vp), ("ranges", _vp), ("n_pairs", _vp), ("pair_capacity", _c.c_int64)]


class GsAdamGroup(_c.Structure):
    _fields_ = [("param", _vp), ("grad", _vp), ("exp_avg", _vp), ("exp_avg_sq", _vp),
                ("count", _c.c_int64), ("lr", _c.c_float), ("reserved", _c.c_float)]


class GsDensifyParams(_c.Structure):
    _fields_ = [("grad_threshold", _c.c_float), ("log_scale_split", _c.c_float),
                ("logit_min_opacity", _c.c_float), ("log_max_scale", _c.c_float),
                ("log_split_shrink", _c.c_float), ("reserved", _c.c_int32)]


# (name, restype, argtypes) for every symbol gs.h declares
SIGNATURES = [
    ("gs_abi_version", _c.c_int32, []),
    ("gs_status_string", _c.c_char_p, [_c.c_int]),
    ("gs_workspace_size", _c.c_size_t,
     [_c.c_int64, _c.c_int32, _c.POINTER(GsCamera), _c.c_int64, _c.c_int32]),
    ("gs_project", _c.c_int,
     [_c.POINTER(GsParams), _c.POINTER(GsCamera), _c.c_int32, _c.POINTER(GsProjected), _vp,
      _vp]),
    ("gs_bin_sort", _c.c_int,
     [_c.POINTER(GsProjected), _c.POINTER(GsCamera), _c.c_int32, _c.c_int64, _c.c_int32,
      _c.POINTER(GsBinned), _vp, _c.c_size_t, _vp]),
    ("gs_rasterize_fwd", _c.c_int,
     [_c.POINTER(GsProjected), _c.POINTER(GsBinned), _c.POINTER(GsCamera), _c.c_int32,
      _c.c_int64, _c.POINTER(_c.c_float), _vp, _vp, _vp, _vp, _vp, _vp]),
    ("gs_rasterize_bwd", _c.c_int,
     [_c.POINTER(GsParams), _c.POINTER(GsProjected), _c.POINTER(GsBinned),
      _c.POINTER(GsCamera), _c.c_int32, _c.POINTER(_c.c_float), _vp, _vp, _vp, _vp, _vp,
      _c.POINTER(GsGrads), _vp, _vp]),
    ("gs_project_bwd", _c.c_int,
     [_c.POINTER(GsParams), _c.POINTER(GsCamera), _c.c_int32, _vp, _vp, _c.POINTER(GsGrads),
      _vp]),
    ("gs_project_bwd_adam", _c.c_int,
     [_c.POINTER(GsParams), _c.POINTER(GsCamera), _c.c_int32, _vp, _vp, _c.POINTER(GsGrads),
      _c.POINTER(GsGrads), _c.POINTER(_c.c_float), _c.c_float, _c.c_float, _c.c_float,
      _c.c_int64, _vp, _vp, _vp, _vp]),
    ("gs_densify_stats", _c.c_int,
     [_vp, _vp, _c.c_int32, _c.c_int64, _vp, _vp, _vp, _vp]),
    ("gs_adam_step", _c.c_int,
     [_c.POINTER(GsAdamGroup), _c.c_int32, _c.c_float, _c.c_float, _c.c_float, _c.c_int64, _vp]),
    ("gs_get_status", _c.c_int, [_vp, _vp]),
    ("gs_densify_workspace_size", _c.c_size_t, [_c.c_int64]),
    ("gs_densify_params_from_cutoffs", _c.c_int,
     [_c.c_double, _c.c_double, _c.c_double, _c.c_double, _c.c_double,
      _c.POINTER(GsDensifyParams)]),
    ("gs_densify_and_prune", _c.c_int,
     [_c.POINTER(GsParams), _c.POINTER(GsGrads), _c.POINTER(GsGrads), _vp, _vp, _vp,
      _c.POINTER(GsDensifyParams), _c.POINTER(GsGrads), _c.POINTER(GsGrads), _c.POINTER(GsGrads),
      _c.c_int64, _vp, _vp, _vp, _c.c_size_t, _vp]),
    ("gs_l1_dssim_workspace_size", _c.c_size_t, [_c.c_int32]),
    ("gs_l1_dssim", _c.c_int,
     [_vp, _vp, _c.c_int32, _c.c_int32, _c.c_int32, _c.c_float, _vp, _vp, _vp, _c.c_size_t,
      _vp]),
    ("gs_sh_quantize", _c.c_int, [_vp, _c.c_void_p, _vp]),
    ("gs_sh_dequantize", _c.c_int, [_c.c_void_p, _vp, _vp]),
    ("gs_adam_step_sh_quant", _c.c_int,
     [_c.c_void_p, _vp, _vp, _vp, _c.c_float, _c.c_float, _c.c_float, _c.c_float, _c.c_int64,
      _c.c_int32, _c.c_uint64, _vp]),
    ("gs_densify_sh_quant_workspace_size", _c.c_size_t, [_c.c_int64, _c.c_int64]),
    ("gs_densify_sh_quant", _c.c_int,
     [_c.c_void_p, _vp, _vp, _vp, _c.c_void_p, _vp, _vp, _vp, _c.c_size_t, _vp]),
    ("gs_bin_sort_plan", _c.c_int,
     [_c.c_int64, _c.c_int32, _c.POINTER(GsCamera), _c.c_int32, _c.c_void_p]),
    ("gs_debug_stall", _c.c_int, [_c.c_int32, _c.c_int64, _c.c_double]),
    ("gs_bin_sort_noalloc", _c.c_int,
     [_c.POINTER(GsProjected), _c.POINTER(GsCamera), _c.c_int32, _c.c_int64, _c.c_int32,
      _c.POINTER(GsBinned), _vp, _vp]),
]

GS_NOALLOC_SCRATCH_BYTES = 32 << 20

_LIB = None


class GsError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__("%s failed: %s (status %d)" % (where, status_string(status), status))
        self.status = status


def lib():
    """Load libgs_b200.so (no fallback: raises if it was not built)."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError("libgs_b200.so is not built (run "
                               "gaussian_splatting_differentiable_ewa_b200/build.py)")
        L = _c.CDLL(LIB_PATH)
        for name, res, args in SIGNATURES:
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _LIB = L
    return _LIB


def status_string(status: int) -> str:
    try:
        return lib().gs_status_string(int(status)).decode()
    except Exception:  # library not loadable
        return "status %d" % status


def _check(status: int, where: str) -> None:
    if status != GS_OK:
        raise GsError(status, where)


def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    return int(t.data_ptr())


def _stream(stream) -> Optional[int]:
    if stream is None:
        return None
    h = getattr(stream, "cuda_stream", stream)
    return int(h) if h else None


def cameras(cams: Sequence) -> ctypes.Array:
    """Array of GsCamera from objects with viewmat/fx/fy/cx/cy/width/height/campos."""
    arr = (GsCamera * len(cams))()
    for k, c in enumerate(cams):
        d = c if isinstance(c, dict) else c.as_dict()
        vm = [float(x) for x in np.asarray(d["viewmat"], np.float32).reshape(12)]
        arr[k].viewmat[:] = vm
        arr[k].fx, arr[k].fy = float(d["fx"]), float(d["fy"])
        arr[k].cx, arr[k].cy = float(d["cx"]), float(d["cy"])
        arr[k].width, arr[k].height = int(d["width"]), int(d["height"])
        arr[k].campos[:] = [float(x) for x in d["campos"]]
    return arr


def params(means, log_scales, quats, opacity_logit, sh, sh_degree: int,
           sh_quant=None) -> GsParams:
    """sh_quant (a GsShQuant) replaces sh: pass sh=None with it."""
    p = GsParams(_ptr(means), _ptr(log_scales), _ptr(quats), _ptr(opacity_logit), _ptr(sh),
                 int(sh_degree), 0, int(means.shape[0]),
                 _c.cast(_c.pointer(sh_quant), _vp) if sh_quant is not None else None)
    p._sh_quant_ref = sh_quant  # the descriptor outlives the pointer to it
    return p


def grads(means, log_scales, quats, opacity_logit, sh) -> GsGrads:
    return GsGrads(_ptr(means), _ptr(log_scales), _ptr(quats), _ptr(opacity_logit), _ptr(sh))


def projected(records, bins, radii) -> GsProjected:
    return GsProjected(_ptr(records), _ptr(bins), _ptr(radii))


def binned(ids, ranges, n_pairs, capacity: int) -> GsBinned:
    return GsBinned(_ptr(ids), _ptr(ranges), _ptr(n_pairs), int(capacity))


def _floats3(bg) -> ctypes.Array:
    a = (_c.c_float * 3)()
    a[:] = [float(x) for x in bg]
    return a


# ---------------------------------------------------------------- C calls

def gs_abi_version() -> int:
    return int(lib().gs_abi_version())


def gs_workspace_size(n: int, cams_arr, n_views: int, pair_capacity: int, sort_mode: int) -> int:
    return int(lib().gs_workspace_size(int(n), int(n_views), cams_arr, int(pair_capacity),
                                       int(sort_mode)))


def gs_project(p: GsParams, cams_arr, n_views: int, out: GsProjected, ws, stream=None) -> None:
    _check(lib().gs_project(_c.byref(p), cams_arr, int(n_views), _c.byref(out), _ptr(ws),
                            _stream(stream)), "gs_project")


def gs_bin_sort(proj: GsProjected, cams_arr, n_views: int, n: int, sort_mode: int,
                out: GsBinned, ws, stream=None) -> None:
    _check(lib().gs_bin_sort(_c.byref(proj), cams_arr, int(n_views), int(n), int(sort_mode),
                             _c.byref(out), _ptr(ws), int(ws.numel() * ws.element_size()),
                             _stream(stream)), "gs_bin_sort")


def gs_rasterize_fwd(proj: GsProjected, bins: GsBinned, cams_arr, n_views: int, n: int, bg,
                     image, final_T, n_contrib, ws, stream=None, warp_masks=None) -> None:
    """warp_masks: optional uint8 [pair_capacity] the backward can reuse."""
    _check(lib().gs_rasterize_fwd(_c.byref(proj), _c.byref(bins), cams_arr, int(n_views), int(n),
                                  _floats3(bg), _ptr(image), _ptr(final_T), _ptr(n_contrib),
                                  _ptr(warp_masks), _ptr(ws), _stream(stream)),
           "gs_rasterize_fwd")


def gs_rasterize_bwd(p: GsParams, proj: GsProjected, bins: GsBinned, cams_arr, n_views: int, bg,
                     dL_dimage, final_T, n_contrib, grad2d, g: Optional[GsGrads], ws,
                     stream=None, warp_masks=None) -> None:
    """warp_masks: the forward's (same lists), or None to test every entry again."""
    _check(lib().gs_rasterize_bwd(_c.byref(p), _c.byref(proj), _c.byref(bins), cams_arr,
                                  int(n_views), _floats3(bg), _ptr(dL_dimage), _ptr(final_T),
                                  _ptr(n_contrib), _ptr(warp_masks), _ptr(grad2d),
                                  None if g is None else _c.byref(g), _ptr(ws), _stream(stream)),
           "gs_rasterize_bwd")


def gs_debug_stall(site: int, index: int = -1, wait_limit_s: float = 0.0) -> None:
    """Test hook: make one device-side wait run out (see include/gs.h)."""
    _check(lib().gs_debug_stall(int(site), int(index), float(wait_limit_s)), "gs_debug_stall")


def gs_project_bwd(p: GsParams, cams_arr, n_views: int, radii, grad2d, g: GsGrads,
                   stream=None) -> None:
    _check(lib().gs_project_bwd(_c.byref(p), cams_arr, int(n_views), _ptr(radii), _ptr(grad2d),
                                _c.byref(g), _stream(stream)), "gs_project_bwd")


def gs_project_bwd_adam(p: GsParams, cams_arr, n_views: int, radii, grad2d, exp_avg: GsGrads,
                        exp_avg_sq: GsGrads, lr, beta1: float, beta2: float, eps: float,
                        step: int, accum_plain=None, accum_abs=None, denom=None,
                        stream=None) -> None:
    """lr: the five group learning rates (means, log_scales, quats,
    opacity_logit, sh); the parameters of p are updated in place."""
    lr5 = (_c.c_float * 5)(*[float(x) for x in lr])
    _check(lib().gs_project_bwd_adam(_c.byref(p), cams_arr, int(n_views), _ptr(radii),
                                     _ptr(grad2d), _c.byref(exp_avg), _c.byref(exp_avg_sq), lr5,
                                     float(beta1), float(beta2), float(eps), int(step),
                                     _ptr(accum_plain), _ptr(accum_abs), _ptr(denom),
                                     _stream(stream)), "gs_project_bwd_adam")


def gs_densify_stats(grad2d, radii, n_views: int, n: int, accum_plain, accum_abs, denom,
                     stream=None) -> None:
    _check(lib().gs_densify_stats(_ptr(grad2d), _ptr(radii), int(n_views), int(n),
                                  _ptr(accum_plain), _ptr(accum_abs), _ptr(denom),
                                  _stream(stream)), "gs_densify_stats")


def gs_adam_step(groups: Sequence[tuple], beta1: float, beta2: float, eps: float, step: int,
                 stream=None) -> None:
    """groups: (param, grad, exp_avg, exp_avg_sq, lr) tensors / float."""
    arr = (GsAdamGroup * len(groups))()
    for k, (p, g, m, v, lr) in enumerate(groups):
        arr[k] = GsAdamGroup(_ptr(p), _ptr(g), _ptr(m), _ptr(v), int(p.numel()), float(lr), 0.0)
    _check(lib().gs_adam_step(arr, len(groups), float(beta1), float(beta2), float(eps), int(step),
                              _stream(stream)), "gs_adam_step")


def gs_get_status(ws, stream=None) -> int:
    return int(lib().gs_get_status(_ptr(ws), _stream(stream)))


def densify_params(grad_threshold: float, scale_split: float, min_opacity: float,
                   max_scale: float, split_shrink: float = 1.6) -> GsDensifyParams:
    """gs_densify_params from cut-offs stated as scales and an opacity (the
    library converts them to log-scales and a logit)."""
    dp = GsDensifyParams()
    _check(lib().gs_densify_params_from_cutoffs(float(grad_threshold), float(scale_split),
                                                float(min_opacity), float(max_scale),
                                                float(split_shrink), _c.byref(dp)),
           "gs_densify_params_from_cutoffs")
    return dp


def gs_densify_workspace_size(n: int) -> int:
    return int(lib().gs_densify_workspace_size(int(n)))


def gs_densify_and_prune(params: GsParams, m_in: GsGrads, v_in: GsGrads, accum, denom, z,
                         dp: GsDensifyParams, out: GsGrads, m_out: GsGrads, v_out: GsGrads,
                         out_capacity: int, n_out, codes, ws, stream=None) -> None:
    _check(lib().gs_densify_and_prune(_c.byref(params), _c.byref(m_in), _c.byref(v_in),
                                      _ptr(accum), _ptr(denom), _ptr(z), _c.byref(dp),
                                      _c.byref(out), _c.byref(m_out), _c.byref(v_out),
                                      int(out_capacity), _ptr(n_out), _ptr(codes), _ptr(ws),
                                      int(ws.numel() * ws.element_size()), _stream(stream)),
           "gs_densify_and_prune")


def gs_l1_dssim_workspace_size(n_views: int) -> int:
    return int(lib().gs_l1_dssim_workspace_size(int(n_views)))


def gs_l1_dssim(image, target, n_views: int, height: int, width: int, lam: float, terms,
                dL_dimage, ws, stream=None) -> None:
    """(1 - lam) L1 + lam (1 - SSIM) per view; terms [V, 3] float64 (loss,
    mean L1, mean SSIM), dL_dimage like image or None."""
    _check(lib().gs_l1_dssim(_ptr(image), _ptr(target), int(n_views), int(height), int(width),
                             float(lam), _ptr(terms), _ptr(dL_dimage), _ptr(ws),
                             int(ws.numel() * ws.element_size()), _stream(stream)),
           "gs_l1_dssim")


GS_QUANT_GROUP = 256


GS_QUANT_PLANAR, GS_QUANT_PACKED = 0, 1


class GsShQuant(_c.Structure):
    _fields_ = [("codes", _vp), ("bounds", _vp), ("n", _c.c_int64), ("k3", _c.c_int32),
                ("bits", _c.c_int32), ("layout", _c.c_int32), ("reserved", _c.c_int32)]


def sh_quant(codes, bounds, n: int, k3: int, bits: int, layout: int = GS_QUANT_PLANAR
             ) -> GsShQuant:
    """Descriptor of a quantised SH state: codes uint8/int16 [k3, n_pad]
    (planar) or int16 [k3, n_pad // 32, 3, 32] (packed blocks of codes and
    both moments), bounds float32 [k3, n_pad // 256, 2]."""
    return GsShQuant(_ptr(codes), _ptr(bounds), int(n), int(k3), int(bits), int(layout), 0)


def gs_sh_quantize(sh, q: GsShQuant, stream=None) -> None:
    _check(lib().gs_sh_quantize(_ptr(sh), _c.byref(q), _stream(stream)), "gs_sh_quantize")


def gs_sh_dequantize(q: GsShQuant, sh, stream=None) -> None:
    _check(lib().gs_sh_dequantize(_c.byref(q), _ptr(sh), _stream(stream)), "gs_sh_dequantize")


def gs_adam_step_sh_quant(q: GsShQuant, grad_sh, exp_avg, exp_avg_sq, lr: float, beta1: float,
                          beta2: float, eps: float, step: int, rounding: int = 0, seed: int = 0,
                          stream=None) -> None:
    """Planar state: exp_avg / exp_avg_sq int16 [k3, n_pad]; packed: None."""
    _check(lib().gs_adam_step_sh_quant(_c.byref(q), _ptr(grad_sh), _ptr(exp_avg),
                                       _ptr(exp_avg_sq), float(lr), float(beta1), float(beta2),
                                       float(eps), int(step), int(rounding), int(seed),
                                       _stream(stream)), "gs_adam_step_sh_quant")


def gs_densify_sh_quant_workspace_size(n_in: int, n_out: int) -> int:
    return int(lib().gs_densify_sh_quant_workspace_size(int(n_in), int(n_out)))


def gs_densify_sh_quant(q_in: GsShQuant, m_in, v_in, decisions, q_out: GsShQuant, m_out, v_out,
                        ws, stream=None) -> None:
    """Quantised SH of densify_and_prune's output (planar moments as int16
    [k3, n_pad] tensors, None for packed state)."""
    _check(lib().gs_densify_sh_quant(_c.byref(q_in), _ptr(m_in), _ptr(v_in), _ptr(decisions),
                                     _c.byref(q_out), _ptr(m_out), _ptr(v_out), _ptr(ws),
                                     int(ws.numel() * ws.element_size()), _stream(stream)),
           "gs_densify_sh_quant")


GS_PATH_TILE_ID, GS_PATH_COLUMNS, GS_PATH_TILES = 0, 1, 2


class GsSortPlan(_c.Structure):
    _fields_ = [("path", _c.c_int32), ("presort_passes", _c.c_int32),
                ("pair_passes", _c.c_int32), ("gaussians_per_block", _c.c_int32),
                ("pair_single_sweep", _c.c_int32), ("ranges_from_counts", _c.c_int32),
                ("blocks_per_view", _c.c_int64), ("pair_key_bytes", _c.c_int32),
                ("reserved", _c.c_int32)]


def gs_bin_sort_plan(n: int, cams_arr, n_views: int, sort_mode: int) -> GsSortPlan:
    """How gs_bin_sort orders the pairs of this request (host only)."""
    plan = GsSortPlan()
    _check(lib().gs_bin_sort_plan(int(n), int(n_views), cams_arr, int(sort_mode),
                                  _c.addressof(plan)), "gs_bin_sort_plan")
    return plan


def gs_bin_sort_noalloc(proj: GsProjected, cams_arr, n_views: int, n: int, sort_mode: int,
                        out: GsBinned, device_status=None, stream=None) -> None:
    """gs_bin_sort without a workspace argument, for callers that cannot
    allocate device memory: the library's fixed scratch array is used instead
    (see include/gs.h for its size limit and the no-overlap rule)."""
    _check(lib().gs_bin_sort_noalloc(_c.byref(proj), cams_arr, int(n_views), int(n),
                                     int(sort_mode), _c.byref(out), _ptr(device_status),
                                     _stream(stream)), "gs_bin_sort_noalloc")
