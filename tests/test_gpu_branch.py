"""Branch / fork and restore-to-position on the GPU, against the oracle.

Beam search, best-of-n and tree search spawn several continuations of one
prefix ("ReplaySSM: Rethinking State Storage for Faster Hybrid-Model
Decoding", nexus-ai-blog.com guide, §"The State-Storage Bottleneck in
Branching Workloads"), and the decode loop can return a sequence to the state
it had at an earlier position (same guide, §"What a Replay-First Design Implies").  A branching
layer lets rows share a checkpoint slot and copies only windows; folds move a
row to a free slot.  Here random sequences of decode, branch, restore and
flush calls run on the GPU and on the oracle (oracle.branch) side by side:

* every output and every row's checkpoint (through its slot) within the
  bf16-input tolerance of the fp64 recurrence, fp32 reads;
* pointers (start, len, pending, flushes) bit-exact against the oracle's
  window book, refused rows included;
* read-copy layers: the fp32 checkpoints as above, each row's read copy equal
  to the oracle's quantisation of its fp32 checkpoint, and outputs within the
  read copy's error;
* a shared slot is never written: rows that shared a slot and fold at
  different times (after restores) keep their own results.
"""
import numpy as np
import pytest
import torch

import seeded_inputs as si
from gpu_common import DEV, GDN_KEYS, M2_KEYS, assert_close, dev_inputs, gdn_layer, m2_layer, to64, tok64
from hybrid_ssm_decode_replayssm_b200 import rssm
from oracle import branch as ob
from oracle import codecs as oc

pytestmark = pytest.mark.gpu

TOL = 2e-3   # bf16 inputs, fp32 state
M2 = si.Mamba2Layer(batch=6, nheads=16, headdim=64, dstate=128, ngroups=2, window=4, dtype="bf16",
                    state_std=0.1, max_draft=1)
GDN = si.GDNLayer(batch=6, nheads=4, dk=128, dv=128, window=4, dtype="bf16", state_std=0.05, max_draft=1)


def _setup(kind, fmt):
    if kind == "mamba2":
        layer, A, D, h0 = m2_layer(M2, read_fmt=fmt, branching=True)
        rows = ob.mamba2_rows(to64(h0), M2.window, layer.layout.cap, A, D)
        return layer, rows, M2_KEYS, (M2.batch, M2.nheads, M2.headdim), lambda t: si.mamba2_tokens(M2, t, seed=4)
    layer, S0 = gdn_layer(GDN, read_fmt=fmt, branching=True)
    rows = ob.gdn_rows(to64(S0), GDN.window, layer.layout.cap)
    return layer, rows, GDN_KEYS, (GDN.batch, GDN.nheads, GDN.dv), lambda t: si.gdn_tokens(GDN, t, seed=4)


def _book(layer):
    return [list(map(int, r)) for r in layer.get_bookkeeping().cpu().numpy()]


def _read_copy_matches(layer, fmt):
    """Each row's read copy is the oracle's quantisation of its fp32 checkpoint."""
    slots = layer.get_slots().cpu().numpy()
    ck = layer.ckpt.cpu().numpy()[slots]
    codes, scales = layer.read_copy_views()
    codes, scales = codes.cpu().numpy()[slots], scales.cpu().numpy()[slots]
    if fmt == rssm.RSSM_READ_FP8_E4M3_ROW:
        wc, ws = oc.fp8_row_quantize(ck)
        np.testing.assert_array_equal(codes, wc)
        np.testing.assert_array_equal(scales.view(np.uint32), ws.view(np.uint32))
    else:
        wc, ws = oc.nvfp4_quantize(ck)
        el = np.stack([codes & 0xF, codes >> 4], axis=-1).reshape(codes.shape[:-1] + (-1,))
        np.testing.assert_array_equal(el, wc)
        np.testing.assert_array_equal(scales, ws)


OPS = (["decode"] * 3 + ["branch", "decode", "restore"]) * 6 + ["flush", "decode", "branch0", "decode",
                                                                  "decode", "badbranch", "badrestore", "decode"]


@pytest.mark.parametrize("fmt", [rssm.RSSM_READ_FP32, rssm.RSSM_READ_FP8_E4M3_ROW, rssm.RSSM_READ_NVFP4])
@pytest.mark.parametrize("kind", ["mamba2", "gdn"])
def test_branch_restore_decode_against_oracle(kind, fmt):
    layer, rows, keys, out_shape, tokens = _setup(kind, fmt)
    B = rows.batch
    out = torch.empty(out_shape, device=DEV)
    rng = np.random.default_rng(7)
    worst, t = 0.0, 0
    for i, op in enumerate(OPS):
        status = 0
        if op == "decode":
            tok = tokens(t)
            t += 1
            layer.decode_step(dev_inputs(tok, keys), out)
            y = rows.decode(tok64(tok))
            if fmt == rssm.RSSM_READ_FP32:
                worst = max(worst, assert_close(out.cpu(), y, TOL, f"{op} {i}: output"))
            else:   # reads from FP8 / NVFP4: the read copy's error, not the tolerance
                g = out.cpu().double().numpy()
                rms = np.sqrt(np.mean((g - y) ** 2)) / np.sqrt(np.mean(y ** 2))
                assert rms < (0.05 if fmt == rssm.RSSM_READ_FP8_E4M3_ROW else 0.15), f"{op} {i}: rms {rms:.3e}"
        elif op in ("branch", "branch0", "badbranch"):
            parent = si.branch_parents(B, i, seed=9).numpy()
            if op == "branch0":
                parent[:] = 0                      # best-of-n: every row from row 0
            if op == "badbranch":
                parent[1], parent[4] = B + 3, -1   # refused rows keep their own state
                status = rssm.RSSM_STATUS_STATE
            layer.branch(torch.from_numpy(parent).to(DEV))
            rows.branch(parent)
        elif op in ("restore", "badrestore"):
            keep = [int(rng.integers(0, n + 1)) for n in rows.book.len]
            if op == "badrestore":
                keep[2] = rows.book.len[2] + 1
                status = rssm.RSSM_STATUS_STATE
            layer.restore(torch.tensor(keep, dtype=torch.int32, device=DEV))
            rows.restore(keep)
        elif op == "flush":
            mask = [1, 0, 1, 1, 0, 1]
            layer.flush(torch.tensor(mask, dtype=torch.int32, device=DEV))
            rows.flush(mask)
        assert layer.get_status(clear=True) == status, f"{op} {i}: status"
        assert _book(layer) == [list(x) for x in rows.book.snapshot()], f"{op} {i}: pointers"
        assert_close(layer.checkpoint_rows().cpu(), rows.checkpoint(), TOL, f"{op} {i}: checkpoints")
    if fmt != rssm.RSSM_READ_FP32:
        _read_copy_matches(layer, fmt)
    assert sum(rows.book.flushes) > B, "the sequence must fold rows several times"
    print(f"\n{kind} fmt {fmt}: worst output error {worst:.2e}")


def test_no_slot_shared_with_a_fold():
    """Rows sharing a slot fold at different steps (restores leave them at
    different window lengths): each fold moves its row to a slot no other row
    reads, and the rows that still share the old slot keep reading it."""
    layer, rows, keys, out_shape, tokens = _setup("mamba2", rssm.RSSM_READ_FP32)
    B = rows.batch
    out = torch.empty(out_shape, device=DEV)
    for t in range(2):
        tok = tokens(t)
        layer.decode_step(dev_inputs(tok, keys), out)
        rows.decode(tok64(tok))
    layer.branch(torch.zeros(B, dtype=torch.int32, device=DEV))
    rows.branch(np.zeros(B, np.int32))
    assert len(set(layer.get_slots().cpu().tolist())) == 1
    keep = [2, 1, 0, 2, 1, 0]
    layer.restore(torch.tensor(keep, dtype=torch.int32, device=DEV))
    rows.restore(keep)
    for t in range(2, 9):
        tok = tokens(t)
        layer.decode_step(dev_inputs(tok, keys), out)
        y = rows.decode(tok64(tok))
        assert_close(out.cpu(), y, TOL, f"token {t}")
        slots = layer.get_slots().cpu().tolist()
        assert all(0 <= s < 2 * B for s in slots)
        # rows with different histories never share a slot
        ck = rows.checkpoint()
        for a in range(B):
            for b in range(B):
                if slots[a] == slots[b]:
                    np.testing.assert_array_equal(ck[a], ck[b])
    assert_close(layer.checkpoint_rows().cpu(), rows.checkpoint(), TOL, "checkpoints")
    assert layer.get_status() == 0
