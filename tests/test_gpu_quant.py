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
