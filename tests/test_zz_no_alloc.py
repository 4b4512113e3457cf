"""rssm_decode_step_static_scratch against rssm_decode_step.

The static-scratch entry point exists for callers that cannot hand the
library extra device memory when they decode: code recording decode steps
into a CUDA graph (nothing may be allocated inside a capture), serving
engines that reserve all device memory when they start, and tight loops that
cannot pay for cudaMalloc's implicit synchronisation.  It keeps the replay
kernel's per-sequence arrival counters in an array inside the library.  It
runs the same kernel on the same inputs as the ordinary decode step, so its
outputs, ring pointers and checkpoint must be bit-identical to that call's,
call after call, for every layer type (the counters expect a different number
of arrivals per sequence in each: groups x head chunks for Mamba-2, head chunks
for Gated DeltaNet, heads for KDA).

This file is collected last on purpose (its name sorts after the others), so
a run that stops at the first failure has run every other test first.
"""
import ctypes as C

import pytest
import torch

import seeded_inputs as si
from gpu_common import DEV, GDN_KEYS, KDA_KEYS, M2_KEYS, dev_inputs, gdn_layer, kda_layer, m2_layer
from hybrid_ssm_decode_replayssm_b200 import rssm

pytestmark = pytest.mark.gpu


def _static_scratch_decode(layer, inputs, out):
    arr = (C.c_void_p * len(inputs))(*[t.data_ptr() for t in inputs])
    rssm.check(rssm.lib().rssm_decode_step_static_scratch(
        layer.handle, arr, out.data_ptr(), torch.cuda.current_stream().cuda_stream))


def _pair(kind):
    """Two identical layers (same seeds), their token function, keys and output shape.
    Window 2: the second call fills the window and folds it into the checkpoint."""
    if kind == "mamba2":
        # 64 sequences x 4 groups = 256 items: more items than resident CTAs, so every
        # CTA works through several items and 4 CTAs meet on each sequence's counter.
        shape = si.Mamba2Layer(batch=64, nheads=16, headdim=64, dstate=128, ngroups=4, window=2,
                               dtype="bf16", state_std=0.1, max_draft=2)
        make = lambda: m2_layer(shape, seed=3)[0]
        return make(), make(), (lambda t: si.mamba2_tokens(shape, t, seed=3)), M2_KEYS, (64, 16, 64)
    if kind == "gdn":
        shape = si.GDNLayer(batch=64, nheads=8, dk=128, dv=128, window=2, dtype="bf16", state_std=0.05,
                            max_draft=2)
        make = lambda: gdn_layer(shape, seed=3)[0]
        return make(), make(), (lambda t: si.gdn_tokens(shape, t, seed=3)), GDN_KEYS, (64, 8, 128)
    shape = si.KDALayer(batch=16, nheads=8, dk=128, dv=128, window=2, dtype="bf16", state_std=0.05)
    make = lambda: kda_layer(shape, seed=3)[0]
    return make(), make(), (lambda t: si.kda_tokens(shape, t, seed=3)), KDA_KEYS, (16, 8, 128)


@pytest.mark.parametrize("kind", ["mamba2", "gdn", "kda"])
def test_static_scratch_decode_matches_decode_step(kind):
    ref, nal, tokens, keys, out_shape = _pair(kind)
    y_ref = torch.empty(out_shape, device=DEV)
    y_nal = torch.full_like(y_ref, float("nan"))
    for t in range(2):                       # two calls in a row
        ins = dev_inputs(tokens(t), keys)
        ref.decode_step(ins, y_ref)
        _static_scratch_decode(nal, ins, y_nal)
        torch.cuda.synchronize()
        assert torch.equal(y_nal, y_ref), f"call {t}: outputs differ"
        assert torch.equal(nal.get_bookkeeping(), ref.get_bookkeeping()), f"call {t}: ring pointers"
    assert torch.equal(nal.ckpt, ref.ckpt), "checkpoint after the fold"
    assert int(ref.get_bookkeeping()[3].min()) == 1, "the second call must fold every sequence"
    assert nal.get_status() == 0 and ref.get_status() == 0


def test_static_scratch_rejects_oversize_batch():
    shape = si.Mamba2Layer(batch=rssm.RSSM_STATIC_SCRATCH_MAX_BATCH + 1, nheads=1, headdim=64,
                           dstate=64, ngroups=1, window=2, dtype="f32", state_std=0.0, max_draft=1)
    d = rssm.make_desc(rssm.RSSM_MAMBA2, shape.batch, 1, 64, 64, ngroups=1, window=2, max_draft=1,
                       in_dtype=rssm.RSSM_F32)
    h = C.c_void_p()
    fake = 1 << 20                     # the call must refuse before touching any pointer
    L = rssm.lib()
    assert L.rssm_create(C.byref(d), fake, fake, None, fake, C.byref(h)) == rssm.RSSM_OK
    try:
        L.rssm_set_params(h, fake, fake)
        arr = (C.c_void_p * 4)(fake, fake, fake, fake)
        assert L.rssm_decode_step_static_scratch(h, arr, fake, None) == rssm.RSSM_ERR_INVALID_ARG
        assert b"static scratch" in L.rssm_last_error_string()
    finally:
        L.rssm_destroy(h)
