"""State export / import to host (the serving-side half of a multi-layer decode
loop: a preempted request's layers are moved off the GPU and back).

The blob is raw bytes of the layer's checkpoint slots, read copy, ring buffers
and pointers, so export -> more decoding -> import must put the layer back
exactly: decoding the same tokens again gives bit-identical outputs,
checkpoints and pointers.  Checked for a branching Mamba-2 layer with an NVFP4
read copy (branched before the export) and a GDN layer.  The continuation
after the import is also compared with the fp64 oracle run without any
interruption: outputs (fp32 reads) and the checkpoint each sequence reads
(every layer: the recurrence stays fp32) within 2e-3.
"""
import numpy as np
import pytest
import torch

import seeded_inputs as si
from gpu_common import DEV, GDN_KEYS, M2_KEYS, assert_close, dev_inputs, gdn_layer, m2_layer, tok64
from oracle import branch as obr

pytestmark = pytest.mark.gpu


def _run(layer, toks, keys, out_shape):
    outs = []
    for tok in toks:
        out = torch.empty(out_shape, device=DEV)
        layer.decode_step(dev_inputs(tok, keys), out)
        outs.append(out)
    torch.cuda.synchronize()
    return outs


@pytest.mark.parametrize("kind", ["mamba2", "gdn"])
def test_export_import_round_trip(kind):
    if kind == "mamba2":
        shape = si.Mamba2Layer(batch=4, nheads=16, headdim=64, dstate=128, ngroups=2, window=4, dtype="bf16",
                               state_std=0.1, max_draft=1)
        from hybrid_ssm_decode_replayssm_b200 import rssm
        layer, A, D, h0 = m2_layer(shape, read_fmt=rssm.RSSM_READ_NVFP4, branching=True)
        toks = [si.mamba2_tokens(shape, t, seed=8) for t in range(12)]
        keys, out_shape = M2_KEYS, (4, 16, 64)
        model = obr.mamba2_rows(h0.double().numpy(), shape.window, int(layer.layout.cap), A, D)
    else:
        shape = si.GDNLayer(batch=4, nheads=4, dk=128, dv=128, window=4, dtype="bf16", state_std=0.05,
                            max_draft=1)
        layer, S0 = gdn_layer(shape)
        toks = [si.gdn_tokens(shape, t, seed=8) for t in range(12)]
        keys, out_shape = GDN_KEYS, (4, 4, 128)
        model = obr.gdn_rows(S0.double().numpy(), shape.window, int(layer.layout.cap))
    _run(layer, toks[:5], keys, out_shape)
    for tok in toks[:5]:
        model.decode(tok64(tok))
    if kind == "mamba2":
        parent = [0, 0, 3, 1]
        layer.branch(torch.tensor(parent, dtype=torch.int32, device=DEV))
        model.branch(parent)
    blob = layer.export_state()
    assert blob.numel() == layer.state_bytes()
    first = _run(layer, toks[5:], keys, out_shape)            # folds happen in here
    ck1, bk1 = layer.ckpt.clone(), layer.get_bookkeeping().clone()
    layer.import_state(blob)
    second = _run(layer, toks[5:], keys, out_shape)
    for a, b in zip(first, second):
        assert torch.equal(a, b)
    assert torch.equal(layer.ckpt, ck1)
    assert torch.equal(layer.get_bookkeeping(), bk1)
    assert layer.get_status() == 0
    # the continuation equals the oracle's uninterrupted recurrence
    for t, (tok, out) in enumerate(zip(toks[5:], second)):
        want = model.decode(tok64(tok))
        if kind == "gdn":
            assert_close(out.cpu(), want, 2e-3, f"output {t} after import vs oracle")
    assert_close(layer.checkpoint_rows().cpu(), model.checkpoint(), 2e-3, "checkpoints after import vs oracle")
    assert np.array_equal(layer.get_bookkeeping().cpu().numpy(), np.array(model.book.snapshot()))
