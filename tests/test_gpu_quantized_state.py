"""The quantised-state baseline on the GPU (rssm_conventional_step_quantized).

A layer whose state is stored in FP8 or NVFP4 and rounded again at every token
is the design a read copy replaces ("ReplaySSM: Rethinking State Storage for
Faster Hybrid-Model Decoding", deskofai.com summary, paragraph 4).

* Each step is checked against the oracle applied to the GPU's own state
  before the step (decoded on the CPU): the output within the bf16 tolerance,
  the new state within one quantisation of the exact update, and its codes
  equal to the oracle's quantisation of that update except where fp32 and fp64
  arithmetic fall on either side of a rounding boundary.
* Over many tokens its output error exceeds that of a read-copy layer (fp32
  recurrence, low-precision reads) by more than 2x; the fp64 oracle alone puts
  the ratio at 4.1 to 4.6 for these layers and formats.
"""
import numpy as np
import pytest
import torch

import seeded_inputs as si
from gpu_common import DEV, GDN_KEYS, M2_KEYS, dev_inputs, gdn_layer, m2_layer, rel_err, tok64
from hybrid_ssm_decode_replayssm_b200 import rssm
from oracle import codecs as oc
from oracle import gdn as og
from oracle import mamba2 as om
from oracle import quantized_state as qs

pytestmark = pytest.mark.gpu

FMTS = {rssm.RSSM_READ_FP8_E4M3_ROW: "fp8_e4m3_row", rssm.RSSM_READ_NVFP4: "nvfp4"}


def _decode(fmt, codes, scales):
    """GPU state codes -> (fp64 values, element codes)."""
    codes, scales = codes.cpu().numpy(), scales.cpu().numpy()
    if fmt == rssm.RSSM_READ_FP8_E4M3_ROW:
        return oc.fp8_row_dequantize(codes, scales), codes
    el = np.stack([codes & 0xF, codes >> 4], axis=-1).reshape(codes.shape[:-1] + (-1,))
    return oc.nvfp4_dequantize(el, scales), el


def _bound(fmt, x):
    """Largest |quantised - x| elementwise for one rounding of x.  The 1.15 and the
    1e-6 of the row maximum allow the GPU's fp32 update to round a block or row
    scale one E4M3 step (12.5%) away from the fp64 update's."""
    r = np.abs(np.asarray(x, np.float32)).astype(np.float64)
    slack = 1e-6 * r.max(-1, keepdims=True)
    if fmt == rssm.RSSM_READ_FP8_E4M3_ROW:
        s = r.max(-1, keepdims=True) / 448.0
        return np.maximum(r * 2.0 ** -4, s * 2.0 ** -10) * 1.15 + slack
    blk = r.reshape(r.shape[:-1] + (-1, 16))
    sv = oc.e4m3_decode(oc.e4m3_encode(blk.max(-1, keepdims=True) / 6.0))
    q = blk / np.where(sv == 0, 1, sv)
    half = np.where(q < 2, 0.25, np.where(q < 4, 0.5, 1.0)) + np.maximum(q - 6, 0)
    return np.where(sv == 0, blk, half * sv).reshape(r.shape) * 1.15 + slack


def _layer(kind, fmt, L=16):
    if kind == "mamba2":
        shape = si.Mamba2Layer(batch=2, nheads=8, headdim=64, dstate=128, ngroups=2, window=L,
                               dtype="bf16", state_std=0.1, max_draft=1)
        layer, A, D, h0 = m2_layer(shape, read_fmt=fmt)
        step = lambda S, tok: om.step(S, tok["x"], tok["B"], tok["C"], tok["dt"], A, D)
        return layer, shape, h0.double().numpy(), step, M2_KEYS, lambda t: si.mamba2_tokens(shape, t, seed=3)
    shape = si.GDNLayer(batch=2, nheads=4, dk=128, dv=128, window=L, dtype="bf16", state_std=0.05, max_draft=1)
    layer, S0 = gdn_layer(shape, read_fmt=fmt)
    step = lambda S, tok: og.step(S, tok["q"], tok["k"], tok["v"], tok["alpha"], tok["beta"])
    return layer, shape, S0.double().numpy(), step, GDN_KEYS, lambda t: si.gdn_tokens(shape, t, seed=3)


def _state_from_read_copy(layer):
    """Quantised-state buffers holding the layer's read copy (its quantised checkpoint)."""
    codes, scales = layer.quantized_state_buffers()
    rc_codes, rc_scales = layer.read_copy_views()
    codes.copy_(rc_codes)
    scales.copy_(rc_scales)
    return codes, scales


@pytest.mark.parametrize("fmt", list(FMTS))
@pytest.mark.parametrize("kind", ["mamba2", "gdn"])
def test_quantized_state_step_matches_oracle(kind, fmt):
    layer, shape, _, step, keys, tokens = _layer(kind, fmt)
    codes, scales = _state_from_read_copy(layer)
    out_shape = (2, 8, 64) if kind == "mamba2" else (2, 4, 128)
    out = torch.empty(out_shape, device=DEV)
    for t in range(6):
        before, _ = _decode(fmt, codes, scales)
        tok = tokens(t)
        layer.conventional_step_quantized(codes, scales, codes, scales, dev_inputs(tok, keys), out)   # in place
        exact, y = step(before, tok64(tok))
        assert rel_err(out.cpu(), y) < 2e-3, f"{kind} {FMTS[fmt]} step {t}: output"
        after, el = _decode(fmt, codes, scales)
        assert np.all(np.abs(after - exact) <= _bound(fmt, exact)), f"step {t}: state off by more than one rounding"
        _, el_oracle = _decode_oracle(fmt, exact)
        agree = np.mean(el == el_oracle)
        assert agree > 0.999, f"step {t}: only {agree:.5f} of the codes agree with the oracle's"


def _decode_oracle(fmt, exact):
    rows = np.asarray(exact, np.float32)
    if fmt == rssm.RSSM_READ_FP8_E4M3_ROW:
        c, s = oc.fp8_row_quantize(rows)
        return oc.fp8_row_dequantize(c, s), c
    c, s = oc.nvfp4_quantize(rows)
    return oc.nvfp4_dequantize(c, s), c


@pytest.mark.parametrize("fmt", list(FMTS))
@pytest.mark.parametrize("kind", ["mamba2", "gdn"])
def test_stored_state_rounding_compounds_read_copy_does_not(kind, fmt):
    T, L = 512, 16
    base_layer, shape, S0, step, keys, tokens = _layer(kind, fmt, L)
    rc_layer, _, _, _, _, _ = _layer(kind, fmt, L)
    codes, scales = _state_from_read_copy(base_layer)
    out_shape = (2, 8, 64) if kind == "mamba2" else (2, 4, 128)
    yb = torch.empty(out_shape, device=DEV)
    yr = torch.empty_like(yb)
    exact = S0.copy()
    eb, er = [], []
    for t in range(T):
        tok = tokens(t)
        ins = dev_inputs(tok, keys)
        base_layer.conventional_step_quantized(codes, scales, codes, scales, ins, yb)
        rc_layer.decode_step(ins, yr)
        exact, y = step(exact, tok64(tok))
        rms = np.sqrt(np.mean(y ** 2))
        eb.append(np.sqrt(np.mean((yb.cpu().double().numpy() - y) ** 2)) / rms)
        er.append(np.sqrt(np.mean((yr.cpu().double().numpy() - y) ** 2)) / rms)
    assert rc_layer.get_status() == 0
    b = float(np.sqrt(np.mean(np.square(eb[-256:]))))
    r = float(np.sqrt(np.mean(np.square(er[-256:]))))
    print(f"\n{kind} {FMTS[fmt]}: rms output error over the last 256 of {T} steps: "
          f"stored low-precision state {b:.3e}, read copy {r:.3e} (ratio {b / r:.2f})")
    assert b > 2.0 * r, f"stored-state error {b:.3e} not above twice the read copy's {r:.3e}"
