"""Serving-shape parity: every sequence of the batch, in the launch configuration
the bench times, against the fp64 oracle.

* Decode: Mamba-2 (batch 256, 128 heads, P 64, N 128, G 8) and Gated DeltaNet /
  KDA (batch 256, 32 heads, d 128), bf16 inputs, fp32 checkpoint, L = 16.  All
  256 sequences are compared element by element for the first 32 calls (two
  window-full folds included, checkpoints compared after each), then 16
  sequences spread over the batch for every call up to 1024.  Between folds the
  checkpoint must stay byte-identical (the state is never written by a read).
* Speculative verify: k = 4 drafts per round, a seeded accepted prefix
  U{0..4} per sequence, the rest rolled back by pointer, 32 rounds over the
  full batch: the 4 outputs of every round, the checkpoint of every sequence
  that folds before its drafts, the final checkpoint after a flush, and the
  pointers after every round (bit for bit) against the oracle's rules.

The oracle runs in worker processes (``oracle_workers``), one per block of 16
sequences.  Tolerance 2e-3 (bf16 inputs, fp32 state), scaled error
|g - o| / (|o| + rms(o)).
"""
import numpy as np
import pytest
import torch

import seeded_inputs as si
from gpu_common import DEV, GDN_KEYS, KDA_KEYS, M2_KEYS, dev_inputs, gdn_layer, kda_layer, m2_layer
from oracle import bookkeeping as ob
from oracle_workers import OracleWorkers

pytestmark = pytest.mark.gpu

TOL = 2e-3
FULL_CALLS = 32
CALLS = 1024
TRACKED = [16 * w + (5 * w + 3) % 16 for w in range(16)]   # one sequence per block of 16


def _np(tok):
    return {k: v.float().numpy() for k, v in tok.items()}


def _bk(layer):
    return [list(r) for r in layer.get_bookkeeping().cpu().numpy()]


def _decode_run(kind, layer, state0, tokens_fn, keys, params=None):
    """Decode CALLS tokens; compare with the oracle workers as described above."""
    L = layer.desc.window
    B = state0.shape[0]
    book = ob.WindowBook(B, L, int(layer.layout.cap))
    workers = OracleWorkers(kind, state0.numpy(), params=params)
    out = torch.empty((B, layer.desc.nheads, layer.desc.headdim), device=DEV)
    ck_after_fold = layer.ckpt.clone()
    try:
        for t in range(CALLS):
            tok = tokens_fn(t)
            layer.decode_step(dev_inputs(tok, keys), out)
            flags = book.decode()
            folded = [b for b in range(B) if flags[b][3]]
            assert folded in ([], list(range(B))), "all sequences share one window position"
            rows = workers.rows()
            ck = None
            if folded:
                ck = layer.ckpt[rows].cpu().numpy()
                ck_after_fold.copy_(layer.ckpt)
            else:
                assert torch.equal(layer.ckpt, ck_after_fold), f"checkpoint written by call {t}"
            workers.decode(f"call {t}", _np(tok), out[rows].cpu().numpy(), ck, TOL)
            if t == FULL_CALLS - 1:
                workers.narrow(TRACKED)
        assert _bk(layer) == [list(x) for x in book.snapshot()]
        assert layer.get_status() == 0
    finally:
        worst, failures = workers.finish()
    assert not failures, failures
    assert worst.get("output", 1.0) <= TOL and worst.get("checkpoint", 1.0) <= TOL
    print(f"{kind}: worst scaled errors {worst}")


def test_mamba2_serving_every_sequence():
    shape = si.MAMBA2_SERVING
    layer, A, D, h0 = m2_layer(shape)
    _decode_run("mamba2", layer, h0, lambda t: si.mamba2_tokens(shape, t), M2_KEYS, {"A": A, "D": D})


def test_gdn_serving_every_sequence():
    shape = si.GDN_SERVING
    layer, S0 = gdn_layer(shape)
    _decode_run("gdn", layer, S0, lambda t: si.gdn_tokens(shape, t), GDN_KEYS)


def test_kda_serving_every_sequence():
    shape = si.KDA_SERVING
    layer, S0 = kda_layer(shape)
    _decode_run("kda", layer, S0, lambda t: si.kda_tokens(shape, t), KDA_KEYS)


ROUNDS = 32


def _verify_run(kind, layer, state0, drafts_fn, keys, params=None, k=4):
    L = layer.desc.window
    B = state0.shape[0]
    book = ob.WindowBook(B, L, int(layer.layout.cap))
    workers = OracleWorkers(kind, state0.numpy(), params=params)
    yk = torch.empty((B, k, layer.desc.nheads, layer.desc.headdim), device=DEV)
    nfolds = 0
    try:
        for r in range(ROUNDS):
            drafts = drafts_fn(r)
            acc = si.accept_counts(B, r, k)
            layer.verify(k, dev_inputs(drafts, keys), yk)
            flags = book.verify(k)
            folded = [b for b in range(B) if flags[b][1]]     # folded before appending the drafts
            nfolds += len(folded)
            assert _bk(layer) == [list(x) for x in book.snapshot()], f"pointers after verify {r}"
            ck = layer.ckpt[folded].cpu().numpy() if folded else None
            workers.verify(f"round {r}", _np(drafts), acc.numpy(), yk.cpu().numpy(), folded, ck, TOL)
            n_reject = (k - acc).to(torch.int32)
            layer.rollback(n_reject.to(DEV))
            book.rollback(n_reject.tolist())
            assert _bk(layer) == [list(x) for x in book.snapshot()], f"pointers after rollback {r}"
        layer.flush()
        book.flush()
        workers.checkpoint("final flush", layer.ckpt.cpu().numpy(), TOL)
        assert _bk(layer) == [list(x) for x in book.snapshot()]
        assert layer.get_status() == 0
    finally:
        worst, failures = workers.finish()
    assert not failures, failures
    assert nfolds > B, "the rounds must fold most sequences at least once"
    assert worst.get("verify output", 1.0) <= TOL and worst.get("checkpoint", 1.0) <= TOL
    print(f"{kind} verify: {nfolds} folds, worst scaled errors {worst}")


def test_mamba2_verify_serving_every_sequence():
    shape = si.MAMBA2_SERVING
    layer, A, D, h0 = m2_layer(shape)
    _verify_run("mamba2", layer, h0, lambda r: si.mamba2_drafts(shape, r, 4), M2_KEYS, {"A": A, "D": D})


def test_gdn_verify_serving_every_sequence():
    shape = si.GDN_SERVING
    layer, S0 = gdn_layer(shape)
    _verify_run("gdn", layer, S0, lambda r: si.gdn_drafts(shape, r, 4), GDN_KEYS)
