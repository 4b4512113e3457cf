"""The worker-process oracle used by the full-batch GPU parity tests: on CPU,
fed the oracle's own results it reports zero error, and fed a result with one
wrong element it reports the failure."""
import numpy as np

import seeded_inputs as si
from oracle import gdn as og
from oracle import mamba2 as om
from oracle import speculative as osp
from oracle_workers import OracleWorkers


def _np(tok):
    return {k: v.float().numpy() for k, v in tok.items()}


def test_decode_stream_matches_in_process_oracle_and_flags_a_planted_error():
    shape = si.Mamba2Layer(batch=6, nheads=4, headdim=8, dstate=16, ngroups=2, dtype="bf16")
    A, D = (t.double().numpy() for t in si.mamba2_params(shape))
    h0 = si.mamba2_checkpoint(shape)
    w = OracleWorkers("mamba2", h0.numpy(), nblocks=3, params={"A": A, "D": D})
    h = h0.double().numpy()
    for t in range(5):
        tok = _np(si.mamba2_tokens(shape, t))
        h, y = om.step(h, *(tok[k].astype(np.float64) for k in ("x", "B", "C", "dt")), A, D)
        y_sent = y.copy()
        if t == 3:
            y_sent[4, 1, 2] += 1.0           # one wrong element, in the third block
        w.decode(f"call {t}", tok, y_sent[w.rows()], h[w.rows()] if t == 2 else None, 2e-3)
        if t == 2:
            w.narrow([1, 4])
    worst, failures = w.finish()
    assert len(failures) == 1 and "call 3" in failures[0]
    assert worst["checkpoint"] < 1e-12


def test_verify_stream_matches_in_process_oracle():
    shape = si.GDNLayer(batch=4, nheads=2, dk=8, dv=8, dtype="bf16")
    S0 = si.gdn_checkpoint(shape)
    w = OracleWorkers("gdn", S0.numpy(), nblocks=2)
    S = S0.double().numpy()
    for r in range(3):
        drafts = _np(si.gdn_drafts(shape, r, 3))
        acc = si.accept_counts(4, r, 3).numpy()
        before = S.copy()
        y, S = osp.gdn_round(S, {k: v.astype(np.float64) for k, v in drafts.items()}, acc)
        w.verify(f"round {r}", drafts, acc, y, [0, 3], before[[0, 3]], 2e-3)
    w.checkpoint("end", S, 2e-3)
    worst, failures = w.finish()
    assert not failures, failures
    assert worst["verify output"] < 1e-12 and worst["checkpoint"] < 1e-12
