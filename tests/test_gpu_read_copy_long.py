"""Long-run output error of the low-precision read copies (2048 decode steps).

"ReplaySSM: Rethinking State Storage for Faster Hybrid-Model Decoding"
(deskofai.com summary, paragraph 4): the recurrence stays in high precision
while a low-precision copy serves the reads, so the rounding of the copy does
not compound over the decode.  Every fold works from the fp32 checkpoint and
rebuilds the copy from it; the output error over the last 256 of 2048 steps
must therefore stay at the level of the first 256, and the fp32 checkpoint
must track the exact fp64 state to fp32 accuracy throughout.

Narrow layers (2 sequences, a few heads, the serving head sizes) keep the
fp64 oracle fast; the error per element depends on the head sizes, not on
the number of heads.  `pytest -s` prints the measured error per case.
"""
import numpy as np
import pytest
import torch

import seeded_inputs as si
from gpu_common import DEV, GDN_KEYS, M2_KEYS, dev_inputs, gdn_layer, m2_layer, rel_err, to64, tok64
from hybrid_ssm_decode_replayssm_b200 import rssm
from oracle import gdn as og
from oracle import mamba2 as om

pytestmark = pytest.mark.gpu

STEPS = 2048
EDGE = 256
FMT_NAME = {rssm.RSSM_READ_FP8_E4M3_ROW: "fp8_e4m3_row", rssm.RSSM_READ_NVFP4: "nvfp4"}


def _scaled_errors(got, want):
    """Per-step max and rms of |g - o| / rms(o) (rms over the step's outputs)."""
    rms = np.sqrt(np.mean(want ** 2)) + 1e-300
    d = np.abs(got - want) / rms
    return float(d.max()), float(np.sqrt(np.mean(d ** 2)))


def _run(kind, fmt, L):
    if kind == "mamba2":
        shape = si.Mamba2Layer(batch=2, nheads=8, headdim=64, dstate=128, ngroups=2, window=L,
                               dtype="bf16", state_std=0.1, max_draft=1)
        layer, A, D, h0 = m2_layer(shape, read_fmt=fmt)
        state = h0.double().numpy()
        out = torch.empty(2, 8, 64, device=DEV)
        keys = M2_KEYS

        def oracle(st, tok):
            t = tok64(tok)
            return om.step(st, t["x"], t["B"], t["C"], t["dt"], A, D)

        tokens = lambda t: si.mamba2_tokens(shape, t, seed=3)
    else:
        shape = si.GDNLayer(batch=2, nheads=4, dk=128, dv=128, window=L, dtype="bf16",
                            state_std=0.05, max_draft=1)
        layer, S0 = gdn_layer(shape, read_fmt=fmt)
        state = S0.double().numpy()
        out = torch.empty(2, 4, 128, device=DEV)
        keys = GDN_KEYS

        def oracle(st, tok):
            t = tok64(tok)
            return og.step(st, t["q"], t["k"], t["v"], t["alpha"], t["beta"])

        tokens = lambda t: si.gdn_tokens(shape, t, seed=3)

    emax, erms, ck_err = [], [], 0.0
    for t in range(STEPS):
        tok = tokens(t)
        layer.decode_step(dev_inputs(tok, keys), out)
        state, want = oracle(state, tok)
        mx, rm = _scaled_errors(out.cpu().double().numpy(), want)
        emax.append(mx)
        erms.append(rm)
        if (t + 1) % L == 0:   # a fold just ran: the fp32 checkpoint holds the state after t
            ck_err = max(ck_err, rel_err(to64(layer.ckpt), state))
    assert layer.get_status() == 0
    return np.array(emax), np.array(erms), ck_err


@pytest.mark.parametrize("L", [1, 16])
@pytest.mark.parametrize("fmt", [rssm.RSSM_READ_FP8_E4M3_ROW, rssm.RSSM_READ_NVFP4])
@pytest.mark.parametrize("kind", ["mamba2", "gdn"])
def test_read_copy_error_does_not_compound(kind, fmt, L):
    emax, erms, ck_err = _run(kind, fmt, L)
    first, last = emax[:EDGE].max(), emax[-EDGE:].max()
    print(f"\n{kind} {FMT_NAME[fmt]} L={L}: max scaled error first {EDGE} steps {first:.3e}, "
          f"last {EDGE} {last:.3e}; rms over {STEPS} steps {np.sqrt(np.mean(erms ** 2)):.3e}; "
          f"fp32 checkpoint vs fp64 {ck_err:.2e}")
    # the fp32 recurrence: folds from the fp32 checkpoint keep it within fp32 rounding
    assert ck_err < 2e-3, f"fp32 checkpoint drifted from the exact state: {ck_err:.3e}"
    # no compounding: the late error is of the same size as the early error
    assert last <= 2.0 * first, f"error grew: first {first:.3e}, last {last:.3e}"
    # and it is the error of one rounding of the state, not of a drifting one
    assert np.sqrt(np.mean(erms[-EDGE:] ** 2)) <= 1.5 * np.sqrt(np.mean(erms[:EDGE] ** 2)) + 1e-6
