"""Kimi Delta Attention on the GPU against the fp64 oracle (oracle.kda).

KDA is the third SSM layer type the pages name ("ReplaySSM: Rethinking State
Storage for Faster Hybrid-Model Decoding", babnews.org teaser); it is read as
the gated delta rule with one gate per key channel.  The replay kernel keeps
the fp32 checkpoint plus a window of inputs and cached w rows, folds the
window when it fills, and must give the recurrence's outputs and states:

* every output and the checkpoint after every fold, fp32 inputs (1e-4) over
  window lengths 1..32 and bf16 inputs (2e-3);
* the conventional per-token kernel (the in-run baseline) against the oracle;
* explicit masked flush, restore to a position, and branching (rows sharing
  checkpoint slots) against the oracle's window rules;
* speculative verify of k drafts with rollback to the accepted prefix against
  the oracle's round (oracle.speculative.kda_round), and its refusals;
* FP8-row / NVFP4 read copies: the copy is always the oracle codec's quantisation
  of the fp32 checkpoint (code for code), the outputs are the recurrence from
  the copy's values, and every fold solves the window again from the fp32
  checkpoint, which tracks the exact state.
"""
import numpy as np
import pytest
import torch

import seeded_inputs as si
from gpu_common import DEV, KDA_KEYS, assert_close, dev_inputs, kda_layer, to64, tok64
from hybrid_ssm_decode_replayssm_b200 import rssm
from oracle import bookkeeping as obk
from oracle import branch as ob
from oracle import codecs as oc
from oracle import kda as ok
from oracle import speculative as osp

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-4, "bf16": 2e-3}


def _step(S, tok):
    return ok.step(S, tok["q"], tok["k"], tok["v"], tok["alpha"], tok["beta"])


@pytest.mark.parametrize("L,dtype", [(1, "f32"), (4, "f32"), (16, "f32"), (32, "f32"), (16, "bf16")])
def test_decode_and_folds_against_oracle(L, dtype):
    shape = si.KDALayer(batch=3, nheads=4, dk=128, dv=128, window=L, dtype=dtype, state_std=0.05)
    layer, S0 = kda_layer(shape)
    S = to64(S0)
    out = torch.empty((3, 4, 128), device=DEV)
    T = max(40, 2 * L + 3)
    ck = S.copy()
    for t in range(T):
        tok = si.kda_tokens(shape, t, seed=2)
        layer.decode_step(dev_inputs(tok, KDA_KEYS), out)
        S, y = _step(S, tok64(tok))
        assert_close(out.cpu(), y, TOL[dtype], f"L={L} step {t}: output")
        if (t + 1) % L == 0:
            ck = S.copy()
        if t % 7 == 0 or (t + 1) % L == 0:
            assert_close(layer.ckpt.cpu(), ck, TOL[dtype], f"L={L} step {t}: checkpoint")
    layer.flush()
    assert_close(layer.ckpt.cpu(), S, TOL[dtype], "checkpoint after the final flush")
    assert layer.get_status() == 0


def test_conventional_kernel_against_oracle():
    shape = si.KDALayer(batch=4, nheads=8, dk=128, dv=128, window=16, dtype="bf16", state_std=0.05)
    layer, S0 = kda_layer(shape)
    state = S0.to(DEV).contiguous()
    out = torch.empty((4, 8, 128), device=DEV)
    S = to64(S0)
    for t in range(6):
        tok = si.kda_tokens(shape, t, seed=3)
        layer.conventional_step(state, state, dev_inputs(tok, KDA_KEYS), out)
        S, y = _step(S, tok64(tok))
        assert_close(out.cpu(), y, TOL["bf16"], f"conventional y step {t}")
    assert_close(state.cpu(), S, TOL["bf16"], "conventional state")


def test_flush_restore_branch_against_oracle():
    shape = si.KDALayer(batch=6, nheads=4, dk=128, dv=128, window=4, dtype="bf16", state_std=0.05)
    layer, S0 = kda_layer(shape, branching=True)
    rows = ob.BranchingRows(to64(S0), 4, layer.layout.cap, _step)
    out = torch.empty((6, 4, 128), device=DEV)
    rng = np.random.default_rng(3)
    ops = ["decode", "decode", "branch", "decode", "restore", "decode", "decode", "flush", "decode",
           "branch", "decode", "decode", "decode", "restore", "decode", "decode", "decode", "decode"]
    for i, op in enumerate(ops):
        if op == "decode":
            tok = si.kda_tokens(shape, i, seed=5)
            layer.decode_step(dev_inputs(tok, KDA_KEYS), out)
            y = rows.decode(tok64(tok))
            assert_close(out.cpu(), y, TOL["bf16"], f"{op} {i}")
        elif op == "branch":
            parent = si.branch_parents(6, i, seed=2).numpy()
            layer.branch(torch.from_numpy(parent).to(DEV))
            rows.branch(parent)
        elif op == "restore":
            keep = [int(rng.integers(0, n + 1)) for n in rows.book.len]
            layer.restore(torch.tensor(keep, dtype=torch.int32, device=DEV))
            rows.restore(keep)
        else:
            mask = [1, 1, 0, 1, 0, 1]
            layer.flush(torch.tensor(mask, dtype=torch.int32, device=DEV))
            rows.flush(mask)
        assert layer.get_status(clear=True) == 0, f"{op} {i}: status"
        bk = [list(map(int, r)) for r in layer.get_bookkeeping().cpu().numpy()]
        assert bk == [list(x) for x in rows.book.snapshot()], f"{op} {i}: pointers"
        assert_close(layer.checkpoint_rows().cpu(), rows.checkpoint(), TOL["bf16"], f"{op} {i}: checkpoints")


def _bk(layer):
    return [list(map(int, r)) for r in layer.get_bookkeeping().cpu().numpy()]


@pytest.mark.parametrize("k,L,dtype", [(1, 1, "f32"), (3, 4, "f32"), (4, 16, "bf16"), (8, 8, "bf16"),
                                       (8, 32, "f32")])
def test_verify_rollback(k, L, dtype):
    """Verify rounds of k seeded drafts with seeded acceptance, decode steps in
    between: every draft output is the recurrence's output after drafts 0..j,
    the accepted prefix becomes committed window entries (their cached w rows
    are what later decodes and folds read), and a round that does not fit is
    folded first.  With bf16 inputs the decodes in between run on the serving
    kernel, which reads the ring the verify kernel wrote."""
    shape = si.KDALayer(batch=5, nheads=2, dk=128, dv=128, window=L, dtype=dtype, state_std=0.05)
    layer, S0 = kda_layer(shape, seed=k, max_draft=k)
    S = to64(S0)
    book = obk.WindowBook(5, L, int(layer.layout.cap))
    o = torch.empty(5, 2, 128, device=DEV)
    outk = torch.empty(5, k, 2, 128, device=DEV)
    for r in range(10):
        drafts = si.kda_drafts(shape, r, k, seed=k)
        acc = si.accept_counts(5, r, k, seed=k)
        layer.verify(k, dev_inputs(drafts, KDA_KEYS), outk)
        book.verify(k)
        want, S_next = osp.kda_round(S, tok64(drafts), acc.numpy())
        assert_close(outk.cpu(), want, TOL[dtype], f"verify round {r}")
        n_reject = (k - acc).to(torch.int32)
        layer.rollback(n_reject.to(DEV))
        book.rollback(n_reject.tolist())
        S = S_next
        assert _bk(layer) == [list(x) for x in book.snapshot()], f"pointers after round {r}"
        if r % 2 == 1:
            tok = si.kda_tokens(shape, 500 + r, seed=k)
            layer.decode_step(dev_inputs(tok, KDA_KEYS), o)
            book.decode()
            S, y = _step(S, tok64(tok))
            assert_close(o.cpu(), y, TOL[dtype], f"decode after round {r}")
    layer.flush()
    book.flush()
    assert_close(layer.ckpt.cpu(), S, TOL[dtype], "checkpoint after the rounds")
    assert _bk(layer) == [list(x) for x in book.snapshot()]
    assert layer.get_status() == 0


def test_verify_refusals():
    """A verify over a row whose drafts are still pending sets STATE; with
    auto_flush off, drafts that do not fit in the window set CAPACITY.  Refused
    rows keep their pointers and their checkpoint."""
    shape = si.KDALayer(batch=2, nheads=4, dk=128, dv=128, window=4, dtype="bf16", state_std=0.05)
    layer, S0 = kda_layer(shape, auto_flush=False, max_draft=3)
    outk = torch.empty(2, 3, 4, 128, device=DEV)
    layer.verify(3, dev_inputs(si.kda_drafts(shape, 0, 3), KDA_KEYS), outk)
    before = _bk(layer)
    layer.verify(3, dev_inputs(si.kda_drafts(shape, 1, 3), KDA_KEYS), outk)
    assert layer.get_status(clear=True) == rssm.RSSM_STATUS_STATE
    assert _bk(layer) == before
    layer.rollback(torch.zeros(2, dtype=torch.int32, device=DEV))   # 3 committed of 4
    before = _bk(layer)
    layer.verify(2, dev_inputs(si.kda_drafts(shape, 2, 2), KDA_KEYS), outk[:, :2].contiguous())
    assert layer.get_status(clear=True) == rssm.RSSM_STATUS_CAPACITY
    assert _bk(layer) == before
    assert_close(layer.ckpt.cpu(), to64(S0), 0.0, "checkpoint untouched")


FMTS = [rssm.RSSM_READ_FP8_E4M3_ROW, rssm.RSSM_READ_NVFP4]


def _read_view(layer, fmt, what):
    """The layer's read copy checked code for code against the oracle codec applied
    to its fp32 checkpoint; returns the copy's values (fp64), what the reads see."""
    codes, scales = (t.cpu().numpy() for t in layer.read_copy_views())
    if fmt == rssm.RSSM_READ_NVFP4:
        codes = np.stack([codes & 0xF, codes >> 4], axis=-1).reshape(codes.shape[:-1] + (-1,))
        want_codes, want_scales = oc.nvfp4_quantize(layer.ckpt.cpu().numpy())
        deq = oc.nvfp4_dequantize(want_codes, want_scales)
        np.testing.assert_array_equal(scales, want_scales, err_msg=what)
    else:
        want_codes, want_scales = oc.fp8_row_quantize(layer.ckpt.cpu().numpy())
        deq = oc.fp8_row_dequantize(want_codes, want_scales)
        np.testing.assert_array_equal(scales.view(np.uint32), want_scales.view(np.uint32), err_msg=what)
    np.testing.assert_array_equal(codes, want_codes, err_msg=what)
    return np.asarray(deq, dtype=np.float64)


def _rows(mask):
    return np.asarray(mask, dtype=bool)[:, None, None, None]


@pytest.mark.parametrize("fmt", FMTS)
def test_read_copy_reads_and_fp32_folds(fmt):
    """Decodes and verify rounds (seeded acceptance) on a layer with a read copy,
    rows folding at different calls (window full, or drafts that do not fit), then
    a flush.  The reads see the copy: every output equals the recurrence started
    from the copy's values R (after a pre-fold, from the new copy).  The copy is
    the quantised fp32 checkpoint at all times, and after each fold that
    checkpoint equals the exact state S of the committed tokens."""
    B, L, k = 3, 6, 3
    shape = si.KDALayer(batch=B, nheads=4, dk=128, dv=128, window=L, dtype="bf16", state_std=0.05)
    layer, S0 = kda_layer(shape, max_draft=k, read_fmt=fmt)
    S = to64(S0)
    R = _read_view(layer, fmt, "copy at creation")
    book = obk.WindowBook(B, L, int(layer.layout.cap))
    o = torch.empty(B, 4, 128, device=DEV)
    ov = torch.empty(B, k, 4, 128, device=DEV)
    ops = "ddvdvddvvdddvdvddvd"
    pre_seen = post_seen = 0
    for i, op in enumerate(ops):
        if op == "d":
            tok = si.kda_tokens(shape, 100 + i, seed=7)
            plan = book.decode()
            layer.decode_step(dev_inputs(tok, KDA_KEYS), o)
            pre = [p[1] for p in plan]
            post = [p[3] for p in plan]
            C = _read_view(layer, fmt, f"copy after call {i}")
            start = np.where(_rows(pre), C, R)
            R_next, y = _step(start, tok64(tok))
            assert_close(o.cpu(), y, TOL["bf16"], f"{fmt} decode {i}: outputs from the copy")
            S_next, _ = _step(S, tok64(tok))
            for b in range(B):
                if post[b]:
                    assert_close(layer.ckpt[b].cpu(), S_next[b], TOL["f32"], f"decode {i} row {b}: folded checkpoint")
                elif pre[b]:
                    assert_close(layer.ckpt[b].cpu(), S[b], TOL["f32"], f"decode {i} row {b}: pre-folded checkpoint")
            pre_seen += sum(pre)
            post_seen += sum(post)
            R = np.where(_rows(post), C, R_next)
            S = S_next
        else:
            drafts = si.kda_drafts(shape, i, k, seed=7)
            acc = si.accept_counts(B, i, k, seed=5)   # (this seed leaves some rows full before a decode)
            plan = book.verify(k)
            layer.verify(k, dev_inputs(drafts, KDA_KEYS), ov)
            pre = [p[1] for p in plan]
            C = _read_view(layer, fmt, f"copy after call {i}")
            want, R_next = osp.kda_round(np.where(_rows(pre), C, R), tok64(drafts), acc.numpy())
            assert_close(ov.cpu(), want, TOL["bf16"], f"{fmt} verify {i}: outputs from the copy")
            for b in range(B):
                if pre[b]:
                    assert_close(layer.ckpt[b].cpu(), S[b], TOL["f32"], f"verify {i} row {b}: pre-folded checkpoint")
            _, S = osp.kda_round(S, tok64(drafts), acc.numpy())
            n_reject = (k - acc).to(torch.int32)
            layer.rollback(n_reject.to(DEV))
            book.rollback(n_reject.tolist())
            R = R_next
        assert _bk(layer) == [list(x) for x in book.snapshot()], f"pointers after call {i}"
    assert pre_seen > 0 and post_seen > 0, (pre_seen, post_seen)
    layer.flush()
    book.flush()
    assert_close(layer.ckpt.cpu(), S, TOL["f32"], "checkpoint after the final flush")
    _read_view(layer, fmt, "copy after the final flush")
    assert layer.get_status() == 0
