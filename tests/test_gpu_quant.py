"""Quantised SH state on the GPU (through the C ABI) against the oracle.

Encoding from float32 input is a float32 decision on both sides: codes and
bounds bit-exact. Decoding: within 2 ulps of the group's largest magnitude.
The fused Adam step re-encodes parameters that the kernel computes in float32
and the oracle in float64, so a code may land one step away where the value
sits on a rounding boundary: |code difference| <= 1 everywhere and equal for
all but a small fraction; bfloat16 moments equal or one unit apart; bounds
within float32 rounding of the oracle's.
"""

import numpy as np
import pytest
import torch

from gaussian_splatting_differentiable_ewa_b200 import api
from oracle import oracle as O

pytestmark = pytest.mark.gpu


def _state(n, k3, bits):
    n_pad = -(-n // 256) * 256
    dt = torch.uint8 if bits == 8 else torch.int16
    codes = torch.zeros((k3, n_pad), dtype=dt, device="cuda")
    bounds = torch.zeros((k3, n_pad // 256, 2), dtype=torch.float32, device="cuda")
    return codes, bounds, api.sh_quant(codes, bounds, n, k3, bits)


def _codes_np(codes, bits):
    c = codes.cpu().numpy()
    return c.view(np.uint16) if bits == 16 else c


@pytest.mark.parametrize("bits", [8, 16])
@pytest.mark.parametrize("n,K", [(10000, 16), (777, 9), (256, 1), (1, 4)])
def test_quantize_and_dequantize_match_oracle(bits, n, K):
    rng = np.random.default_rng(n + K + bits)
    sh = rng.normal(0, 0.6, (n, K, 3)).astype(np.float32)
    if n > 300:
        sh[:256, 0, 0] = 1.5                 # a constant group
    k3 = 3 * K
    codes, bounds, q = _state(n, k3, bits)
    api.gs_sh_quantize(torch.from_numpy(sh).cuda(), q)
    out = torch.full((n, K, 3), float("nan"), device="cuda")
    api.gs_sh_dequantize(q, out)
    torch.cuda.synchronize()
    want_c, want_b = O.sh_quantize(sh, bits)
    got_c = _codes_np(codes, bits)
    assert np.array_equal(got_c[:, :n], want_c[:, :n])
    assert np.array_equal(bounds.cpu().numpy(), want_b)
    dec = O.dequantize_groups(want_c, want_b, n, bits).T.reshape(n, K, 3)
    mag = np.maximum(np.abs(want_b[..., 0]), np.abs(want_b[..., 1]))
    tol = 2.0 ** -22 * mag[:, np.arange(n) // 256].T.reshape(n, K, 3) + 1e-30
    assert np.all(np.abs(out.cpu().numpy() - dec) <= tol)


def _adam_case(n, K, bits, rounding, seed=5, step=7):
    rng = np.random.default_rng(seed)
    sh = rng.normal(0, 0.5, (n, K, 3)).astype(np.float32)
    k3 = 3 * K
    c0, b0 = O.sh_quantize(sh, bits)
    n_pad = c0.shape[1]
    m16 = O.to_bf16(rng.normal(0, 1e-3, (k3, n_pad)))
    v16 = O.to_bf16(rng.uniform(0, 1e-6, (k3, n_pad)))
    grad = rng.normal(0, 1e-3, (n, K, 3)).astype(np.float32)
    codes, bounds, q = _state(n, k3, bits)
    codes.copy_(torch.from_numpy(c0.view(np.int16) if bits == 16 else c0))
    bounds.copy_(torch.from_numpy(b0))
    m = torch.from_numpy(m16.view(np.int16).copy()).cuda()
    v = torch.from_numpy(v16.view(np.int16).copy()).cuda()
    api.gs_adam_step_sh_quant(q, torch.from_numpy(grad).cuda(), m, v, 2.5e-3, 0.9, 0.999, 1e-15,
                              step, rounding, seed=99)
    torch.cuda.synchronize()
    want = O.adam_sh_quant(c0, b0, grad, m16, v16, n, bits, 2.5e-3, step, rounding=rounding,
                           seed=99)
    got = (_codes_np(codes, bits), bounds.cpu().numpy(), m.cpu().numpy().view(np.uint16),
           v.cpu().numpy().view(np.uint16))
    return got, want


@pytest.mark.parametrize("bits", [8, 16])
@pytest.mark.parametrize("rounding", [0, 1])
def test_adam_on_quantised_state_matches_oracle(bits, rounding):
    n, K = 5000, 16
    (gc, gb, gm, gv), (wc, wb, wm, wv, p_new) = _adam_case(n, K, bits, rounding)
    for got, want in ((gm, wm), (gv, wv)):
        d = np.abs(got[:, :n].astype(np.int32) - want[:, :n].astype(np.int32))
        assert d.max() <= 1 and (d > 0).mean() < 1e-2
        assert np.array_equal(got[:, n:], want[:, n:])      # padding untouched
    # bounds: min / max of the new float32 parameters
    scale = np.abs(wb).max()
    assert np.abs(gb - wb).max() <= 1e-6 * scale
    d = np.abs(gc[:, :n].astype(np.int64) - wc[:, :n].astype(np.int64))
    assert d.max() <= 1
    assert (d > 0).mean() < 1e-2
    # the decoded parameters track the float64 Adam step within one code step
    x = O.dequantize_groups(gc, gb, n, bits)
    step = (gb[..., 1] - gb[..., 0]).astype(np.float64) / ((1 << bits) - 1)
    assert np.all(np.abs(x - p_new) <= 1.05 * step[:, np.arange(n) // 256] + 1e-6)


def test_quant_rejects_bad_descriptors_and_accepts_empty():
    codes, bounds, q = _state(300, 12, 8)
    sh = torch.zeros((300, 4, 3), device="cuda")
    for bad in (api.sh_quant(codes, bounds, 300, 12, 12), api.sh_quant(codes, bounds, 300, 5, 8),
                api.sh_quant(codes, bounds, -1, 12, 8)):
        with pytest.raises(api.GsError):
            api.gs_sh_quantize(sh, bad)
    m = torch.zeros((12, 512), dtype=torch.int16, device="cuda")
    with pytest.raises(api.GsError):
        api.gs_adam_step_sh_quant(q, sh, m, m, 1e-3, 0.9, 0.999, 1e-15, 1, rounding=2)
    with pytest.raises(api.GsError):
        api.gs_adam_step_sh_quant(q, sh, m, m, 1e-3, 0.9, 0.999, 1e-15, 0)
    empty = api.sh_quant(None, None, 0, 12, 8)
    api.gs_sh_quantize(None, empty)
    api.gs_adam_step_sh_quant(empty, None, None, None, 1e-3, 0.9, 0.999, 1e-15, 1)
    torch.cuda.synchronize()


def _train_losses(sh_bits, rounding, steps=30):
    from gaussian_splatting_differentiable_ewa_b200 import scenes as S
    from gaussian_splatting_differentiable_ewa_b200.pipeline import Splatter
    sc = S.make_scene("fwd_1k_128")
    outs = O.render_all(sc)
    H, W = sc.cameras[0].height, sc.cameras[0].width
    tgt = np.stack([o[1]["color"].reshape(H, W, 3).transpose(2, 0, 1) for o in outs])
    tgt = torch.from_numpy(np.ascontiguousarray(tgt, np.float32)).cuda()
    rng = np.random.default_rng(1)
    sc2 = S.make_scene("fwd_1k_128")
    sc2.sh[:, 0, :] += rng.normal(0, 0.2, size=sc2.sh[:, 0, :].shape).astype(np.float32)
    sp = Splatter(sc2, lr=dict(means=1.6e-4, sh=1e-2, opacity_logit=5e-2, log_scales=5e-3,
                               quats=1e-3), sh_bits=sh_bits, sh_rounding=rounding, sh_seed=3)
    sp.ensure_capacity()
    first = None
    for _ in range(steps):
        sp.train_step_target(tgt)
        if first is None:
            first = float(sp.loss_terms[0, 0].item())
    sp.forward()
    last = float(sp.loss(tgt, grad=False)[0, 0].item())
    assert sp.status() == api.GS_OK
    return first, last


def test_training_with_quantised_sh_state():
    """The Splatter with its SH kept only as codes (decoded before each
    projection, Adam on the codes): 16-bit nearest and 8-bit stochastic
    rounding both lower the loss toward an oracle-rendered target about as
    far as the float32 state does."""
    f0, l32 = _train_losses(None, 0)
    for bits, rounding in ((16, 0), (8, 1)):
        f, last = _train_losses(bits, rounding)
        assert abs(f - f0) < 0.02 * f0 + 1e-3      # the same start, up to the encoding
        assert last < 0.85 * f
        assert last < 1.25 * l32 + 1e-3, (bits, last, l32)


# ---------------------------------------------------------------- packed layout

def _packed_state(n, k3):
    n_pad = -(-n // 256) * 256
    words = torch.zeros((k3, n_pad // 32, 3, 32), dtype=torch.int16, device="cuda")
    bounds = torch.zeros((k3, n_pad // 256, 2), dtype=torch.float32, device="cuda")
    return words, bounds


def _pack(codes, m, v, bits):
    """Planar codes [k3][n_pad] and moments -> packed words [k3][n_pad/32][3][32]."""
    k3, n_pad = codes.shape
    c16 = codes.to(torch.int16) if bits == 8 else codes
    return torch.stack([c16.view(k3, n_pad // 32, 32), m.view(k3, n_pad // 32, 32),
                        v.view(k3, n_pad // 32, 32)], dim=2).contiguous()


@pytest.mark.parametrize("bits", [8, 16])
@pytest.mark.parametrize("rounding", [0, 1])
def test_packed_layout_gives_the_planar_results(bits, rounding):
    # the packed optimiser block (codes and both moments of 32 Gaussians in
    # one 192-byte block) changes where the words live, not what they hold
    n, K = 3000, 16
    k3 = 3 * K
    rng = np.random.default_rng(bits + rounding)
    sh = torch.from_numpy(rng.normal(0, 0.5, (n, K, 3)).astype(np.float32)).cuda()
    codes, bounds, q = _state(n, k3, bits)
    words, pbounds = _packed_state(n, k3)
    qp = api.sh_quant(words, pbounds, n, k3, bits, api.GS_QUANT_PACKED)
    api.gs_sh_quantize(sh, q)
    api.gs_sh_quantize(sh, qp)
    n_pad = codes.shape[1]
    m = torch.from_numpy(O.to_bf16(rng.normal(0, 1e-3, (k3, n_pad))).view(np.int16).copy()).cuda()
    v = torch.from_numpy(O.to_bf16(rng.uniform(0, 1e-6, (k3, n_pad))).view(np.int16).copy()).cuda()
    torch.cuda.synchronize()
    assert torch.equal(words[:, :, 0, :].reshape(k3, n_pad)[:, :n],
                       codes.to(torch.int16)[:, :n] if bits == 8 else codes[:, :n])
    assert torch.equal(pbounds, bounds)
    words[:, :, 1:, :] = _pack(codes, m, v, bits)[:, :, 1:, :]
    grad = torch.from_numpy(rng.normal(0, 1e-3, (n, K, 3)).astype(np.float32)).cuda()
    for step in (1, 2):
        api.gs_adam_step_sh_quant(q, grad, m, v, 2.5e-3, 0.9, 0.999, 1e-15, step, rounding, seed=7)
        api.gs_adam_step_sh_quant(qp, grad, None, None, 2.5e-3, 0.9, 0.999, 1e-15, step, rounding,
                                  seed=7)
    out_p = torch.empty((n, K, 3), device="cuda")
    out_q = torch.empty((n, K, 3), device="cuda")
    api.gs_sh_dequantize(q, out_q)
    api.gs_sh_dequantize(qp, out_p)
    torch.cuda.synchronize()
    want = _pack(codes, m, v, bits)
    got = words.clone()
    # padding Gaussians past n are never written in either layout
    mask = torch.zeros((k3, n_pad), dtype=torch.bool, device="cuda")
    mask[:, :n] = True
    mask = mask.view(k3, n_pad // 32, 1, 32).expand_as(got)
    assert torch.equal(got[mask], want[mask])
    assert torch.equal(pbounds, bounds)
    assert torch.equal(out_p, out_q)
    with pytest.raises(api.GsError):   # packed moments travel in the blocks
        api.gs_adam_step_sh_quant(qp, grad, m, v, 2.5e-3, 0.9, 0.999, 1e-15, 3)


# ------------------------------------------------- projection reads the codes

def _quant_of(sp, bits, layout):
    n, k3 = sp.n, 3 * sp.K
    if layout == api.GS_QUANT_PACKED:
        codes, bounds = _packed_state(n, k3)
    else:
        codes, bounds, _ = _state(n, k3, bits)
    q = api.sh_quant(codes, bounds, n, k3, bits, layout)
    api.gs_sh_quantize(sp.sh, q)
    api.gs_sh_dequantize(q, sp.sh)     # the float path sees the decoded values
    return q, (codes, bounds)


@pytest.mark.parametrize("bits,layout", [(8, api.GS_QUANT_PLANAR), (16, api.GS_QUANT_PLANAR),
                                         (8, api.GS_QUANT_PACKED), (16, api.GS_QUANT_PACKED)])
@pytest.mark.parametrize("case", [("train_6m_8x1080p", 1), ("train_6m_8x1080p", 3),
                                  ("fwd_1k_128", 1)])
def test_projection_from_codes_equals_projection_of_decoded_sh(bits, layout, case):
    # SH degree 3 with one view (gradients staged in place) and three views,
    # and degree 0
    from gaussian_splatting_differentiable_ewa_b200 import scenes as S
    from gaussian_splatting_differentiable_ewa_b200.pipeline import Splatter
    name, views = case
    if name == "fwd_1k_128":
        sc = S.make_scene(name)
    else:
        sc = S.make_scene(name, n=3000, width=320, height=180, n_views=views)
    sp = Splatter(sc)
    q, keep = _quant_of(sp, bits, layout)
    sp.ensure_capacity()
    sp.forward()
    rec, bins, radii = sp.records.clone(), sp.bins.clone(), sp.radii.clone()
    pq = api.params(sp.means, sp.log_scales, sp.quats, sp.opacity_logit, None, sp.deg,
                    sh_quant=q)
    api.gs_project(pq, sp.cams, sp.V, sp.c_proj, sp.ws)
    torch.cuda.synchronize()
    assert torch.equal(sp.records, rec) and torch.equal(sp.bins, bins)
    assert torch.equal(sp.radii, radii)
    # backward: the SH gradients and the colour -> direction chain use the codes
    dL = torch.randn_like(sp.image) * 1e-2
    sp.rasterize_bwd(dL, with_params=False)
    g_f = {k: torch.zeros_like(t) for k, t in sp.param_list}
    g_q = {k: torch.zeros_like(t) for k, t in sp.param_list}
    names = [k for k, _ in sp.param_list]
    api.gs_project_bwd(sp.c_params, sp.cams, sp.V, sp.radii, sp.grad2d,
                       api.grads(*[g_f[k] for k in names]))
    api.gs_project_bwd(pq, sp.cams, sp.V, sp.radii, sp.grad2d, api.grads(*[g_q[k] for k in names]))
    torch.cuda.synchronize()
    for k in names:
        assert torch.equal(g_f[k], g_q[k]), k
    assert sp.status() == api.GS_OK
    # exactly one SH source
    both = api.params(sp.means, sp.log_scales, sp.quats, sp.opacity_logit, sp.sh, sp.deg,
                      sh_quant=q)
    with pytest.raises(api.GsError):
        api.gs_project(both, sp.cams, sp.V, sp.c_proj, sp.ws)


# ------------------------------------------------------ densify of the codes

def _unpack(words, n_pad):
    k3 = words.shape[0]
    return [words[:, :, r, :].reshape(k3, n_pad) for r in range(3)]


@pytest.mark.parametrize("bits,layout", [(8, api.GS_QUANT_PLANAR), (16, api.GS_QUANT_PLANAR),
                                         (8, api.GS_QUANT_PACKED), (16, api.GS_QUANT_PACKED)])
def test_densify_of_quantised_sh_equals_encoding_the_gathered_values(bits, layout):
    # output o takes the decoded SH of the input it comes from (kept: itself;
    # cloned: itself then a copy; split: two children), in densify order, and
    # its groups are encoded anew; moments kept for a kept Gaussian and a
    # clone's first copy, zero otherwise
    n, K = 3000, 16
    k3 = 3 * K
    rng = np.random.default_rng(bits * 3 + layout)
    sh = rng.normal(0, 0.5, (n, K, 3)).astype(np.float32)
    dec = rng.integers(0, 4, n).astype(np.int8)
    counts = np.array([0, 1, 2, 2])[dec]
    n_out = int(counts.sum())
    n_pad, m_pad = -(-n // 256) * 256, -(-n_out // 256) * 256
    m_np = O.to_bf16(rng.normal(0, 1e-3, (k3, n_pad))).view(np.int16)
    v_np = O.to_bf16(rng.uniform(0, 1e-6, (k3, n_pad))).view(np.int16)
    packed = layout == api.GS_QUANT_PACKED
    if packed:
        codes, bounds = _packed_state(n, k3)
        ocodes, obounds = _packed_state(n_out, k3)
    else:
        codes, bounds, _ = _state(n, k3, bits)
        ocodes, obounds, _ = _state(n_out, k3, bits)
    q_in = api.sh_quant(codes, bounds, n, k3, bits, layout)
    q_out = api.sh_quant(ocodes, obounds, n_out, k3, bits, layout)
    # the input state comes from the oracle's encoder
    c0, b0 = O.sh_quantize(sh, bits)
    c0_t = torch.from_numpy(c0.view(np.int16) if bits == 16 else c0).cuda()
    bounds.copy_(torch.from_numpy(b0))
    m_in = torch.from_numpy(m_np.copy()).cuda()
    v_in = torch.from_numpy(v_np.copy()).cuda()
    m_out = torch.zeros((k3, m_pad), dtype=torch.int16, device="cuda")
    v_out = torch.zeros_like(m_out)
    if packed:
        codes.copy_(_pack(c0_t, m_in, v_in, bits))
    else:
        codes.copy_(c0_t)
    ws = torch.zeros((api.gs_densify_sh_quant_workspace_size(n, n_out) + 255) // 256 * 32,
                     dtype=torch.int64, device="cuda")
    decisions = torch.from_numpy(dec).cuda()
    if packed:
        api.gs_densify_sh_quant(q_in, None, None, decisions, q_out, None, None, ws)
    else:
        api.gs_densify_sh_quant(q_in, m_in, v_in, decisions, q_out, m_out, v_out, ws)
    assert api.gs_get_status(ws, None) == api.GS_OK
    # expected, from the oracle's float32 decoding of the input codes
    src, zero = [], []
    for i, c in enumerate(dec):
        if c == 1:
            src += [i]; zero += [False]
        elif c == 2:
            src += [i, i]; zero += [False, True]
        elif c == 3:
            src += [i, i]; zero += [True, True]
    src, zero = np.array(src), np.array(zero)
    decoded = O.dequantize_groups_f32(c0, b0, n, bits).T.reshape(n, K, 3)
    want_c, want_b = O.sh_quantize(decoded[src], bits)
    want_m = np.where(zero[None, :], 0, m_np[:, src])
    want_v = np.where(zero[None, :], 0, v_np[:, src])
    if packed:
        gc, gm, gv = [t.cpu().numpy() for t in _unpack(ocodes, m_pad)]
        gc = gc.view(np.uint16)
        want_c = want_c.astype(np.uint16)
    else:
        gc, gm, gv = _codes_np(ocodes, bits), m_out.cpu().numpy(), v_out.cpu().numpy()
    assert np.array_equal(gc[:, :n_out], want_c[:, :n_out])
    assert np.array_equal(obounds.cpu().numpy(), want_b)
    assert np.array_equal(gm[:, :n_out], want_m)
    assert np.array_equal(gv[:, :n_out], want_v)
    # a count that does not match the decisions writes nothing and reports
    q_bad = api.sh_quant(ocodes, obounds, n_out - 1, k3, bits, layout)
    before = ocodes.clone()
    if packed:
        api.gs_densify_sh_quant(q_in, None, None, decisions, q_bad, None, None, ws)
    else:
        api.gs_densify_sh_quant(q_in, m_in, v_in, decisions, q_bad, m_out, v_out, ws)
    assert api.gs_get_status(ws, None) == api.GS_ERR_CAPACITY
    assert torch.equal(ocodes, before)


def test_training_and_densify_with_quantised_sh_state():
    """Splatter with 16-bit codes: a few steps, densify_and_prune on the
    codes, more steps; the new state decodes to the gathered values."""
    from gaussian_splatting_differentiable_ewa_b200 import scenes as S
    from gaussian_splatting_differentiable_ewa_b200.pipeline import Splatter
    sc = S.make_scene("fwd_100k_800", n=4000, width=256, height=256)
    sp = Splatter(sc, sh_bits=16)
    sp.ensure_capacity()
    dL = torch.randn((1, 3, 256, 256), device="cuda") * 1e-3
    for _ in range(3):
        sp.forward()
        sp.rasterize_bwd(dL)
        sp.densify_stats()
        sp.adam_step()
    sp.refresh_sh_float()
    before = sp.sh.clone()
    codes = sp.densify_and_prune(grad_threshold=1e-7, scale_split=0.02)
    c = codes.cpu().numpy()
    assert (c == 2).any() or (c == 3).any()
    src = np.concatenate([[i] * {0: 0, 1: 1, 2: 2, 3: 2}[int(k)] for i, k in enumerate(c)])
    assert sp.n == len(src)
    want = torch.empty((sp.n, sp.K, 3), device="cuda")
    wc, wb = torch.zeros_like(sp.sh_codes), torch.zeros_like(sp.sh_bounds)
    q = api.sh_quant(wc, wb, sp.n, 3 * sp.K, 16)
    api.gs_sh_quantize(before[torch.from_numpy(src).cuda()].contiguous(), q)
    api.gs_sh_dequantize(q, want)
    torch.cuda.synchronize()
    assert torch.equal(sp.sh, want)
    sp.ensure_capacity()
    for _ in range(2):
        sp.forward()
        sp.rasterize_bwd(dL)
        sp.adam_step()
    assert sp.status() == api.GS_OK
