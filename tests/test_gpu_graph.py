"""A multi-layer decode step captured once in a CUDA graph and replayed.

A decode step of a hybrid model runs several SSM layers back to back
("ReplaySSM: Rethinking State Storage for Faster Hybrid-Model Decoding",
deskofai.com summary, paragraphs 2-3: every layer keeps a checkpoint and a
buffer and decodes from them).  The replay kernels read each sequence's ring
pointers from device memory and decide on the device whether a row folds, so
one captured step is valid at every window position: replaying it must give,
bit for bit, what the same calls made eagerly give, through several folds, and
every layer's replayed outputs and folded checkpoints must equal the fp64
oracle's token-by-token recurrence of that layer (tolerance 2e-3, bf16 inputs).
"""
import pytest
import torch

import seeded_inputs as si
from gpu_common import DEV, GDN_KEYS, M2_KEYS, assert_close, dev_inputs, gdn_layer, m2_layer, tok64
from oracle import gdn as og
from oracle import mamba2 as om

pytestmark = pytest.mark.gpu

M2 = si.Mamba2Layer(batch=6, nheads=16, headdim=64, dstate=128, ngroups=2, window=8, dtype="bf16",
                    state_std=0.1, max_draft=2)
GDN = si.GDNLayer(batch=6, nheads=4, dk=128, dv=128, window=8, dtype="bf16", state_std=0.05, max_draft=2)


def _stack(seed):
    """Two Mamba-2 layers and one GDN layer, each with its own state."""
    return [m2_layer(M2, seed=seed)[0], m2_layer(M2, seed=seed + 1)[0], gdn_layer(GDN, seed=seed + 2)[0]]


def _oracle_stack(seed):
    """The same three layers as fp64 oracle states and step functions."""
    res = []
    for k in range(2):
        _, A, D, h0 = m2_layer(M2, seed=seed + k)
        res.append([h0.double().numpy(),
                    lambda h, t, A=A, D=D: om.step(h, t["x"], t["B"], t["C"], t["dt"], A, D)])
    _, S0 = gdn_layer(GDN, seed=seed + 2)
    res.append([S0.double().numpy(), lambda S, t: og.step(S, t["q"], t["k"], t["v"], t["alpha"], t["beta"])])
    return res


def _tokens(t):
    return [si.mamba2_tokens(M2, t, seed=11), si.mamba2_tokens(M2, t, seed=12), si.gdn_tokens(GDN, t, seed=13)]


KEYS = [M2_KEYS, M2_KEYS, GDN_KEYS]
OUT = [(6, 16, 64), (6, 16, 64), (6, 4, 128)]


def test_graph_replay_equals_eager_through_folds():
    eager, graphed = _stack(0), _stack(0)
    oracle = _oracle_stack(0)
    # static device buffers the graph reads its tokens from and writes outputs to
    static_in = [dev_inputs(tok, keys) for tok, keys in zip(_tokens(0), KEYS)]
    static_out = [torch.empty(s, device=DEV) for s in OUT]
    eager_out = [torch.empty(s, device=DEV) for s in OUT]

    def step(layers, ins, outs):
        for layer, i, o in zip(layers, ins, outs):
            layer.decode_step(i, o)

    # token 0 eagerly on both stacks, then capture the step of the graphed one
    step(eager, static_in, eager_out)
    step(graphed, static_in, static_out)
    torch.cuda.synchronize()

    def check_oracle(t, folded):
        for k, (o, tok) in enumerate(zip(oracle, _tokens(t))):
            o[0], want = o[1](o[0], tok64(tok))
            assert_close(static_out[k].cpu(), want, 2e-3, f"layer {k}, token {t}: output vs oracle")
            if folded:
                assert_close(graphed[k].ckpt.cpu(), o[0], 2e-3, f"layer {k}, token {t}: checkpoint vs oracle")

    check_oracle(0, False)
    g = torch.cuda.CUDAGraph()
    # "relaxed": besides the kernel launch, a step makes host-side calls (the
    # kernel's shared-memory attribute, an occupancy query) that this mode
    # leaves unchecked
    with torch.cuda.graph(g, capture_error_mode="relaxed"):
        step(graphed, static_in, static_out)
    # capture records, it does not run: token 1 onwards replays the graph
    for t in range(1, 30):   # window 8: folds at tokens 7, 15, 23
        toks = [dev_inputs(tok, keys) for tok, keys in zip(_tokens(t), KEYS)]
        for dst, src in zip(static_in, toks):
            for d, s_ in zip(dst, src):
                d.copy_(s_)
        g.replay()
        step(eager, toks, eager_out)
        torch.cuda.synchronize()
        for k in range(3):
            assert torch.equal(static_out[k], eager_out[k]), f"layer {k}, token {t}: outputs differ"
        check_oracle(t, t % 8 == 7)
    for k in range(3):
        assert torch.equal(graphed[k].ckpt, eager[k].ckpt), f"layer {k}: checkpoints differ"
        assert torch.equal(graphed[k].get_bookkeeping(), eager[k].get_bookkeeping())
        assert graphed[k].get_status() == 0
    del g
