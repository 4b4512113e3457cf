"""Mamba-2 CUDA path vs the fp64 oracle, through the C ABI.

Tolerances: the scaled error |g - o| / (|o| + rms(o)) must stay below 1e-4
for fp32 inputs and 2e-3 for bf16 inputs with an fp32 checkpoint (the oracle
consumes the same bf16 values, widened exactly, so the measured error is
fp32 rounding only and far below either bound).  Pointer bookkeeping is
compared bit for bit with the oracle's window rules.
"""
import numpy as np
import pytest
import torch

import seeded_inputs as si
from gpu_common import DEV, M2_KEYS, assert_close, dev_inputs, m2_layer, rel_err, to64, tok64
from hybrid_ssm_decode_replayssm_b200 import rssm
from oracle import bookkeeping as ob
from oracle import codecs as oc
from oracle import mamba2 as om
from oracle import speculative as osp

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-4, "bf16": 2e-3}


def _bk(layer):
    return [list(r) for r in layer.get_bookkeeping().cpu().numpy()]


def _oracle_step(h, tok, A, D):
    t = tok64(tok)
    return om.step(h, t["x"], t["B"], t["C"], t["dt"], A, D)


def test_tiny_f32_every_step_every_element():
    """Mamba-2, fp32 throughout, B=4 H=8 P=64 N=64 G=1 L=16, 64 steps from zero."""
    shape = si.MAMBA2_TINY_F32
    layer, A, D, h0 = m2_layer(shape)
    h = h0.double().numpy()
    book = ob.WindowBook(shape.batch, shape.window, int(layer.layout.cap))
    out = torch.empty(shape.batch, shape.nheads, shape.headdim, device=DEV)
    worst = 0.0
    for t in range(64):
        tok = si.mamba2_tokens(shape, t)
        before = layer.ckpt.clone()
        layer.decode_step(dev_inputs(tok, M2_KEYS), out)
        flags = book.decode()
        h, y = _oracle_step(h, tok, A, D)
        worst = max(worst, assert_close(out.cpu(), y, TOL["f32"], f"y step {t}"))
        if flags[0][3]:                                     # window full: folded
            assert_close(layer.ckpt.cpu(), h, TOL["f32"], f"checkpoint after step {t}")
        else:                                               # the state is never written
            assert torch.equal(layer.ckpt, before), f"checkpoint written at step {t}"
    assert _bk(layer) == [list(x) for x in book.snapshot()]
    assert layer.get_status() == 0
    print(f"max scaled error {worst:.2e}")


@pytest.mark.parametrize("L", [1, 2, 3, 5, 16, 32])
@pytest.mark.parametrize("dtype,N", [("f32", 64), ("bf16", 128)])
def test_window_sweep_ragged_tail(L, dtype, N):
    shape = si.Mamba2Layer(batch=3, nheads=4, headdim=64, dstate=N, ngroups=2, window=L,
                           dtype=dtype, state_std=0.1, max_draft=min(4, L))
    layer, A, D, h0 = m2_layer(shape, seed=L)
    h = h0.double().numpy()
    book = ob.WindowBook(shape.batch, L, int(layer.layout.cap))
    out = torch.empty(3, 4, 64, device=DEV)
    for t in range(2 * L + 3):
        tok = si.mamba2_tokens(shape, t, seed=L)
        layer.decode_step(dev_inputs(tok, M2_KEYS), out)
        book.decode()
        h, y = _oracle_step(h, tok, A, D)
        assert_close(out.cpu(), y, TOL[dtype], f"L={L} step {t}")
    layer.flush()
    book.flush()
    assert_close(layer.ckpt.cpu(), h, TOL[dtype], "checkpoint after final flush")
    assert _bk(layer) == [list(x) for x in book.snapshot()]


@pytest.mark.parametrize("shape", [si.MAMBA2_TINY_F32,
                                   si.Mamba2Layer(2, 16, 64, 128, 4, dtype="bf16", state_std=0.1)])
def test_conventional_kernel(shape):
    layer, A, D, h0 = m2_layer(shape)
    state = h0.to(DEV).contiguous()
    h = h0.double().numpy()
    out = torch.empty(shape.batch, shape.nheads, shape.headdim, device=DEV)
    for t in range(24):
        tok = si.mamba2_tokens(shape, t)
        layer.conventional_step(state, state, dev_inputs(tok, M2_KEYS), out)
        h, y = _oracle_step(h, tok, A, D)
        assert_close(out.cpu(), y, TOL[shape.dtype], f"conventional y step {t}")
    assert_close(state.cpu(), h, TOL[shape.dtype], "conventional state")


def test_window_one_equals_conventional_update():
    """L = 1: every decode folds, so replay must track the conventional kernel."""
    shape = si.Mamba2Layer(2, 8, 64, 128, 2, window=1, dtype="bf16", state_std=0.1, max_draft=1)
    layer, A, D, h0 = m2_layer(shape)
    state = h0.to(DEV).contiguous()
    y1 = torch.empty(2, 8, 64, device=DEV)
    y2 = torch.empty_like(y1)
    for t in range(20):
        ins = dev_inputs(si.mamba2_tokens(shape, t), M2_KEYS)
        layer.decode_step(ins, y1)
        layer.conventional_step(state, state, ins, y2)
        assert rel_err(y1.cpu(), y2.cpu()) < 1e-6
        assert rel_err(layer.ckpt.cpu(), state.cpu()) < 1e-6


@pytest.mark.parametrize("k", [1, 3, 4])
def test_verify_rollback(k):
    """Rounds of verify(k) + rollback with seeded acceptance, decode steps in
    between; window 8 so that pre-folds and window-full folds both happen."""
    shape = si.Mamba2Layer(5, 4, 64, 128, 2, window=8, dtype="bf16", state_std=0.1, max_draft=4)
    layer, A, D, h0 = m2_layer(shape, seed=k)
    h = h0.double().numpy()
    book = ob.WindowBook(shape.batch, shape.window, int(layer.layout.cap))
    y = torch.empty(5, 4, 64, device=DEV)
    yk = torch.empty(5, k, 4, 64, device=DEV)
    for r in range(14):
        drafts = si.mamba2_drafts(shape, r, k, seed=k)
        acc = si.accept_counts(shape.batch, r, k, seed=k)
        layer.verify(k, dev_inputs(drafts, M2_KEYS), yk)
        book.verify(k)
        want, h_next = osp.mamba2_round(h, tok64(drafts), acc.numpy(), A, D)
        assert_close(yk.cpu(), want, TOL["bf16"], f"verify round {r}")
        assert _bk(layer) == [list(x) for x in book.snapshot()]
        n_reject = (k - acc).to(torch.int32)
        layer.rollback(n_reject.to(DEV))
        book.rollback(n_reject.tolist())
        h = h_next
        assert _bk(layer) == [list(x) for x in book.snapshot()]
        if r % 3 == 2:
            tok = si.mamba2_tokens(shape, 1000 + r, seed=k)
            layer.decode_step(dev_inputs(tok, M2_KEYS), y)
            book.decode()
            h, yy = _oracle_step(h, tok, A, D)
            assert_close(y.cpu(), yy, TOL["bf16"], f"decode after round {r}")
    layer.flush()
    book.flush()
    assert_close(layer.ckpt.cpu(), h, TOL["bf16"], "checkpoint after rounds")
    assert _bk(layer) == [list(x) for x in book.snapshot()]
    assert layer.get_status() == 0


def test_masked_flush_and_status_bits():
    shape = si.Mamba2Layer(4, 4, 64, 64, 1, window=4, dtype="f32", state_std=0.1, max_draft=2)
    layer, A, D, h0 = m2_layer(shape, auto_flush=False)
    h = h0.double().numpy()
    book = ob.WindowBook(4, 4, int(layer.layout.cap), auto_flush=False)
    out = torch.empty(4, 4, 64, device=DEV)
    for t in range(4):
        tok = si.mamba2_tokens(shape, t)
        layer.decode_step(dev_inputs(tok, M2_KEYS), out)
        book.decode()
        h, _ = _oracle_step(h, tok, A, D)
    out.fill_(float("nan"))
    layer.decode_step(dev_inputs(si.mamba2_tokens(shape, 99), M2_KEYS), out)   # window full, no auto flush
    book.decode()
    assert torch.isnan(out).all(), "a refused row must not be written"
    assert layer.get_status(clear=True) == rssm.RSSM_STATUS_CAPACITY
    mask = torch.tensor([1, 0, 1, 0], dtype=torch.int32, device=DEV)
    before = layer.ckpt.clone()
    layer.flush(mask)
    book.flush([1, 0, 1, 0])
    assert _bk(layer) == [list(x) for x in book.snapshot()]
    assert_close(layer.ckpt[[0, 2]].cpu(), h[[0, 2]], TOL["f32"], "flushed rows")
    assert torch.equal(layer.ckpt[[1, 3]], before[[1, 3]])
    # drafts pending: decode and flush are refused, an oversize rollback too
    layer.flush()
    book.flush()
    layer.verify(2, dev_inputs(si.mamba2_drafts(shape, 0, 2), M2_KEYS), torch.empty(4, 2, 4, 64, device=DEV))
    book.verify(2)
    layer.decode_step(dev_inputs(si.mamba2_tokens(shape, 7), M2_KEYS), out)
    book.decode()
    assert layer.get_status(clear=True) == rssm.RSSM_STATUS_STATE
    layer.rollback(torch.tensor([3, 0, 1, 2], dtype=torch.int32, device=DEV))
    book.rollback([3, 0, 1, 2])
    assert layer.get_status(clear=True) == rssm.RSSM_STATUS_STATE
    assert _bk(layer) == [list(x) for x in book.snapshot()]


# --------------------------------------------------------------- read copies
FMTS = [rssm.RSSM_READ_FP8_E4M3_ROW, rssm.RSSM_READ_NVFP4]


def _oracle_read_copy(fmt, rows):
    if fmt == rssm.RSSM_READ_FP8_E4M3_ROW:
        codes, scales = oc.fp8_row_quantize(rows)
        return codes, scales, oc.fp8_row_dequantize(codes, scales)
    codes, scales = oc.nvfp4_quantize(rows)
    return codes, scales, oc.nvfp4_dequantize(codes, scales)


def _gpu_codes(layer, fmt):
    codes, scales = layer.read_copy_views()
    codes, scales = codes.cpu().numpy(), scales.cpu().numpy()
    if fmt == rssm.RSSM_READ_NVFP4:                      # element 2i in the low nibble
        codes = np.stack([codes & 0xF, codes >> 4], axis=-1).reshape(codes.shape[:-1] + (-1,))
    return codes, scales


@pytest.mark.parametrize("fmt", FMTS)
def test_read_copy_codes_bit_exact(fmt):
    shape = si.Mamba2Layer(8, 16, 64, 128, 2, dtype="bf16", state_std=0.1)
    layer, A, D, h0 = m2_layer(shape, read_fmt=fmt)
    codes, scales = _gpu_codes(layer, fmt)
    want_codes, want_scales, _ = _oracle_read_copy(fmt, h0.numpy())
    np.testing.assert_array_equal(codes, want_codes)
    if fmt == rssm.RSSM_READ_FP8_E4M3_ROW:
        np.testing.assert_array_equal(scales.view(np.uint32), want_scales.view(np.uint32))
    else:
        np.testing.assert_array_equal(scales, want_scales)


@pytest.mark.parametrize("fmt", FMTS)
def test_quantized_reads_within_first_window(fmt):
    """Before the first fold the read copy is the quantised seeded checkpoint: the
    outputs must equal the recurrence started from its dequantised values."""
    shape = si.Mamba2Layer(4, 16, 64, 128, 4, window=16, dtype="bf16", state_std=0.1)
    layer, A, D, h0 = m2_layer(shape, read_fmt=fmt)
    _, _, deq = _oracle_read_copy(fmt, h0.numpy())
    h = deq
    out = torch.empty(4, 16, 64, device=DEV)
    for t in range(15):
        tok = si.mamba2_tokens(shape, t)
        layer.decode_step(dev_inputs(tok, M2_KEYS), out)
        h, y = _oracle_step(h, tok, A, D)
        assert_close(out.cpu(), y, TOL["bf16"], f"{fmt} step {t}")


@pytest.mark.parametrize("fmt", FMTS)
def test_read_copy_keeps_fp32_recurrence(fmt):
    """The fp32 checkpoint trajectory with and without a read copy agrees to fp32
    rounding (both fold the same fp32 checkpoint and inputs; the fp32-read layer
    folds on the tensor cores with an exact three-part split, the read-copy
    layer on the CUDA cores, so only the order of the fp32 additions differs),
    and the read-copy output error stays within the quantisation bound."""
    shape = si.Mamba2Layer(4, 16, 64, 128, 4, window=16, dtype="bf16", state_std=0.1)
    lq, A, D, h0 = m2_layer(shape, read_fmt=fmt)
    lf, _, _, _ = m2_layer(shape)
    yq = torch.empty(4, 16, 64, device=DEV)
    yf = torch.empty_like(yq)
    h_exact = h0.double().numpy()
    h_ckpt = h_exact.copy()          # exact state at the last fold
    book = ob.WindowBook(4, 16, int(lq.layout.cap))
    window_toks = []
    for t in range(40):
        tok = si.mamba2_tokens(shape, t)
        ins = dev_inputs(tok, M2_KEYS)
        lq.decode_step(ins, yq)
        lf.decode_step(ins, yf)
        assert rel_err(lq.ckpt.cpu(), lf.ckpt.cpu()) < 1e-6, f"fp32 checkpoints diverged at step {t}"
        h_exact, y = _oracle_step(h_exact, tok, A, D)
        window_toks.append(tok64(tok))
        # bound: e^{G_t} sum_n |dh[p,n]| |C_n| with the per-element code-grid bound on dh
        rows = h_ckpt.astype(np.float32)
        if fmt == rssm.RSSM_READ_FP8_E4M3_ROW:
            s = np.abs(rows).max(-1, keepdims=True) / 448.0
            dh = np.maximum(np.abs(rows) * 2.0 ** -4, s * 2.0 ** -10)
        else:
            blk = rows.reshape(rows.shape[:-1] + (-1, 16))
            sv = oc.e4m3_decode(oc.e4m3_encode(np.abs(blk).max(-1, keepdims=True) / 6.0))
            # half the E2M1 spacing at |x|/s (0.25, 0.5, 1) and up to 1/16 relative scale rounding
            q = np.abs(blk) / np.where(sv == 0, 1, sv)
            half = np.where(q < 2, 0.25, np.where(q < 4, 0.5, 1.0)) + np.maximum(q - 6, 0)
            dh = np.where(sv == 0, np.abs(blk), half * sv).reshape(rows.shape)
        Gt = sum(wt["dt"] for wt in window_toks) * A[None, :]
        g = om.head_groups(16, 4)
        Ct = window_toks[-1]["C"][:, g, :]
        bound = np.exp(Gt)[..., None] * np.einsum("bhpn,bhn->bhp", dh, np.abs(Ct))
        err = np.abs(yq.cpu().numpy() - y)
        # 1.15: the bound's scales come from the exact state, the GPU's from its fp32
        # checkpoint, which may round a block scale one E4M3 step (12.5%) differently
        slack = 1e-4 * (np.abs(y) + np.sqrt(np.mean(y ** 2)))
        assert np.all(err <= 1.15 * bound + slack), f"step {t}: bound exceeded"
        if book.decode()[0][3]:
            h_ckpt = h_exact.copy()
            window_toks = []


@pytest.mark.parametrize("fmt", [rssm.RSSM_READ_FP32, rssm.RSSM_READ_FP8_E4M3_ROW, rssm.RSSM_READ_NVFP4])
def test_many_items_per_cta(fmt):
    """One head per group (G = H) and enough sequences that every persistent CTA
    works through several items, so the copies requested ahead cross item
    boundaries; verify rounds with ragged acceptance make rows fold at
    different calls of the same launch."""
    shape = si.Mamba2Layer(batch=96, nheads=8, headdim=64, dstate=128, ngroups=8, window=6,
                           dtype="bf16", state_std=0.1, max_draft=3)
    layer, A, D, h0 = m2_layer(shape, read_fmt=fmt)
    h = h0.double().numpy()
    book = ob.WindowBook(96, 6, int(layer.layout.cap))
    yk = torch.empty(96, 3, 8, 64, device=DEV)
    y = torch.empty(96, 8, 64, device=DEV)
    for r in range(8):
        drafts = si.mamba2_drafts(shape, r, 3, seed=5)
        acc = si.accept_counts(96, r, 3, seed=5)
        layer.verify(3, dev_inputs(drafts, M2_KEYS), yk)
        book.verify(3)
        want, h_next = osp.mamba2_round(h, tok64(drafts), acc.numpy(), A, D)
        if fmt == rssm.RSSM_READ_FP32:
            assert_close(yk.cpu(), want, TOL["bf16"], f"verify round {r}")
        else:   # low-precision reads: bounded by the quantisation, checked elsewhere
            assert rel_err(yk.cpu(), want) < (0.1 if fmt == rssm.RSSM_READ_FP8_E4M3_ROW else 0.5)
        n_reject = (3 - acc).to(torch.int32)
        layer.rollback(n_reject.to(DEV))
        book.rollback(n_reject.tolist())
        h = h_next
        tok = si.mamba2_tokens(shape, 500 + r, seed=5)
        layer.decode_step(dev_inputs(tok, M2_KEYS), y)
        book.decode()
        h, yy = _oracle_step(h, tok, A, D)
        assert _bk(layer) == [list(x) for x in book.snapshot()]
    layer.flush()
    book.flush()
    assert_close(layer.ckpt.cpu(), h, TOL["bf16"], "checkpoint")
    assert _bk(layer) == [list(x) for x in book.snapshot()]
    assert layer.get_status() == 0


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


@pytest.mark.parametrize("fmt", FMTS)
def test_read_copy_view_through_folds(fmt):
    """Decodes (the read-copy decode kernel) and verify rounds with seeded
    acceptance, rows folding at different calls: after the window fills, and
    before a token or drafts that do not fit (a pre-fold, after which the reads
    see the copy the fold just wrote).  Every output equals the recurrence from
    the copy's values R; the copy is the quantised fp32 checkpoint after every
    call, and after each fold that checkpoint equals the exact state S."""
    B, L, k = 3, 6, 3
    shape = si.Mamba2Layer(batch=B, nheads=16, headdim=64, dstate=128, ngroups=2, window=L, dtype="bf16",
                           state_std=0.1, max_draft=k)
    layer, A, D, h0 = m2_layer(shape, read_fmt=fmt)
    S = h0.double().numpy()
    R = _read_view(layer, fmt, "copy at creation")
    book = ob.WindowBook(B, L, int(layer.layout.cap))
    y = torch.empty(B, 16, 64, device=DEV)
    yk = torch.empty(B, k, 16, 64, device=DEV)
    rows = lambda m: np.asarray(m, dtype=bool)[:, None, None, None]
    pre_seen = post_seen = 0
    for i, op in enumerate("ddvdvddvvdddvdvddvd"):
        if op == "d":
            tok = si.mamba2_tokens(shape, 100 + i, seed=7)
            plan = book.decode()
            layer.decode_step(dev_inputs(tok, M2_KEYS), y)
            pre, post = [p[1] for p in plan], [p[3] for p in plan]
            C = _read_view(layer, fmt, f"copy after call {i}")
            R_next, want = _oracle_step(np.where(rows(pre), C, R), tok, A, D)
            assert_close(y.cpu(), want, TOL["bf16"], f"{fmt} decode {i}: outputs from the copy")
            S_next, _ = _oracle_step(S, tok, A, D)
            for b in range(B):
                if post[b]:
                    assert_close(layer.ckpt[b].cpu(), S_next[b], TOL["f32"], f"decode {i} row {b}: folded checkpoint")
                elif pre[b]:
                    assert_close(layer.ckpt[b].cpu(), S[b], TOL["f32"], f"decode {i} row {b}: pre-folded checkpoint")
            pre_seen += sum(pre)
            post_seen += sum(post)
            R = np.where(rows(post), C, R_next)
            S = S_next
        else:
            drafts = si.mamba2_drafts(shape, i, k, seed=7)
            acc = si.accept_counts(B, i, k, seed=5)   # (this seed leaves some rows full before a decode)
            plan = book.verify(k)
            layer.verify(k, dev_inputs(drafts, M2_KEYS), yk)
            pre = [p[1] for p in plan]
            C = _read_view(layer, fmt, f"copy after call {i}")
            want, R_next = osp.mamba2_round(np.where(rows(pre), C, R), tok64(drafts), acc.numpy(), A, D)
            assert_close(yk.cpu(), want, TOL["bf16"], f"{fmt} verify {i}: outputs from the copy")
            for b in range(B):
                if pre[b]:
                    assert_close(layer.ckpt[b].cpu(), S[b], TOL["f32"], f"verify {i} row {b}: pre-folded checkpoint")
            _, S = osp.mamba2_round(S, tok64(drafts), acc.numpy(), A, D)
            n_reject = (k - acc).to(torch.int32)
            layer.rollback(n_reject.to(DEV))
            book.rollback(n_reject.tolist())
            R = R_next
        assert _bk(layer) == [list(x) for x in book.snapshot()], f"pointers after call {i}"
    assert post_seen > 0 and pre_seen > 0, (post_seen, pre_seen)
    layer.flush()
    book.flush()
    assert_close(layer.ckpt.cpu(), S, TOL["f32"], "checkpoint after the final flush")
    _read_view(layer, fmt, "copy after the final flush")
    assert layer.get_status() == 0
