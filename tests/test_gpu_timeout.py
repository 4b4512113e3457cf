"""Bounded waits that run out.

Every wait of the replay kernels (a stage's asynchronous copies landing, the
consumer warps releasing a stage) gives up after a limit, sets
RSSM_STATUS_TIMEOUT and lets the launch end early with the device context
intact.  The test arms the kernels' self-test (rssm_arm_timeout_test: the
consumer warps of the first CTA wait for a shared flag that nothing sets) with
a short limit (rssm_set_wait_limit, 20000 SM cycles), so that wait runs out on
purpose -- no fault, trap or endless loop is involved -- and the rest of the
CTA takes the same abort path a copy that never lands would.  After rssm_reset
(which also clears the per-sequence arrival counters an aborted launch may
leave behind) the same layer decodes correctly again.
"""
import pytest
import torch

import seeded_inputs as si
from gpu_common import (DEV, GDN_KEYS, KDA_KEYS, M2_KEYS, assert_close, dev_inputs, gdn_layer, kda_layer,
                        m2_layer, tok64)
from hybrid_ssm_decode_replayssm_b200 import rssm
from oracle import gdn as og
from oracle import kda as ok
from oracle import mamba2 as om

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("kind", ["mamba2", "gdn", "kda"])
def test_short_wait_limit_times_out_then_layer_recovers(kind):
    if kind == "mamba2":
        shape = si.Mamba2Layer(batch=64, nheads=16, headdim=64, dstate=128, ngroups=2, window=16,
                               dtype="bf16", state_std=0.1)
        layer, A, D, h0 = m2_layer(shape, seed=4)
        tokens = lambda t: si.mamba2_tokens(shape, t, seed=4)
        keys, out_shape = M2_KEYS, (64, 16, 64)
        step = lambda S, t: om.step(S, t["x"], t["B"], t["C"], t["dt"], A, D)
    elif kind == "gdn":
        shape = si.GDNLayer(batch=64, nheads=8, dk=128, dv=128, window=16, dtype="bf16", state_std=0.05)
        layer, h0 = gdn_layer(shape, seed=4)
        tokens = lambda t: si.gdn_tokens(shape, t, seed=4)
        keys, out_shape = GDN_KEYS, (64, 8, 128)
        step = lambda S, t: og.step(S, t["q"], t["k"], t["v"], t["alpha"], t["beta"])
    else:   # the KDA decode serving kernel (bf16 inputs)
        shape = si.KDALayer(batch=64, nheads=8, dk=128, dv=128, window=16, dtype="bf16", state_std=0.05)
        layer, h0 = kda_layer(shape, seed=4)
        tokens = lambda t: si.kda_tokens(shape, t, seed=4)
        keys, out_shape = KDA_KEYS, (64, 8, 128)
        step = lambda S, t: ok.step(S, t["q"], t["k"], t["v"], t["alpha"], t["beta"])
    L = rssm.lib()
    out = torch.empty(out_shape, device=DEV)
    assert L.rssm_set_wait_limit(layer.handle, 20000) == rssm.RSSM_OK
    assert L.rssm_arm_timeout_test(layer.handle) == rssm.RSSM_OK
    layer.decode_step(dev_inputs(tokens(0), keys), out)
    torch.cuda.synchronize()                      # the launch ended: no error, no hang
    assert layer.get_status(clear=True) & rssm.RSSM_STATUS_TIMEOUT
    assert torch.equal(layer.ckpt, h0.to(DEV)), "a decode that does not fold never writes the checkpoint"
    # back to the default limit; reset the pointers and counters and decode again
    assert L.rssm_set_wait_limit(layer.handle, 0) == rssm.RSSM_OK
    assert L.rssm_set_wait_limit(layer.handle, -1) == rssm.RSSM_ERR_INVALID_ARG
    layer.reset()
    S = h0.double().numpy()
    for t in range(18):                           # one fold at the 16th token
        tok = tokens(t)
        layer.decode_step(dev_inputs(tok, keys), out)
        S, want = step(S, tok64(tok))
        assert_close(out.cpu(), want, 2e-3, f"{kind} token {t} after the reset")
    assert layer.get_status() == 0
