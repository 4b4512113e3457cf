"""The fp64 oracle spread over worker processes, for full-batch parity tests.

Test infrastructure.  A serving-shape layer (256 sequences, a 1 GiB fp32
checkpoint) makes the single-process numpy oracle take minutes per comparison
run, so the tests split the batch into blocks of sequences, one spawned worker
process per block (spawned, not forked: the parent holds a CUDA context).
Each worker owns the fp64 state of its sequences and advances it with the
oracle's own functions (``oracle.mamba2.step``, ``oracle.gdn.step``,
``oracle.kda.step``, ``oracle.speculative``); the parent streams it the same
token inputs the GPU consumed and the GPU's results for its sequences, and the
worker compares them.  The oracle's arithmetic is not changed: sequences are
independent in every recurrence, so a block of them is the same computation.

Error measure, per comparison and per block: max over elements of
|g - o| / (|o| + rms(o)), rms over the block's compared tensor (the measure
the parity tolerances bound).
"""
from __future__ import annotations

import multiprocessing as mp
import traceback

import numpy as np


def scaled_error(got, want):
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    if want.size == 0:
        return 0.0
    rms = np.sqrt(np.mean(want ** 2))
    return float(np.max(np.abs(got - want) / (np.abs(want) + rms + 1e-300)))


def _worker(conn, kind, state0, params, out_scale):
    from oracle import gdn as og
    from oracle import kda as ok
    from oracle import mamba2 as om
    from oracle import speculative as osp

    state = np.asarray(state0, np.float64)
    worst = {}
    failures = []
    series = []

    def note(what, err, tol, tag):
        worst[what] = max(worst.get(what, 0.0), err)
        if err > tol and len(failures) < 5:
            failures.append(f"{what} at {tag}: scaled error {err:.3e} > {tol:.1e}")

    def step(S, tok):
        t = {k: np.asarray(v, np.float64) for k, v in tok.items()}
        if kind == "mamba2":
            return om.step(S, t["x"], t["B"], t["C"], t["dt"], params["A"], params["D"])
        if kind == "gdn":
            return og.step(S, t["q"], t["k"], t["v"], t["alpha"], t["beta"], out_scale)
        return ok.step(S, t["q"], t["k"], t["v"], t["alpha"], t["beta"], out_scale)

    def verify_round(S, drafts, accept):
        d = {k: np.asarray(v, np.float64) for k, v in drafts.items()}
        if kind == "mamba2":
            return osp.mamba2_round(S, d, accept, params["A"], params["D"])
        return osp.gdn_round(S, d, accept, out_scale)

    try:
        while True:
            msg = conn.recv()
            op = msg[0]
            if op == "decode":
                _, tag, tok, y_gpu, ck_gpu, tol = msg
                state, y = step(state, tok)
                if y_gpu is not None:
                    note("output", scaled_error(y_gpu, y), tol, tag)
                if ck_gpu is not None:
                    note("checkpoint", scaled_error(ck_gpu, state), tol, tag)
            elif op == "decode_bound":
                # per element |g - o| <= bound + slack * (|o| + rms(o)); keeps per-call
                # max and mean-square of |g - o| / rms(o) and the worst ratio to the bound
                _, tag, tok, y_gpu, bound, slack, ck_gpu, tol = msg
                state, y = step(state, tok)
                y_gpu = np.asarray(y_gpu, np.float64)
                rms = np.sqrt(np.mean(y ** 2)) + 1e-300
                err = np.abs(y_gpu - y)
                allowed = np.asarray(bound, np.float64) + slack * (np.abs(y) + rms)
                ratio = float(np.max(err / allowed))
                worst["bound ratio"] = max(worst.get("bound ratio", 0.0), ratio)
                if ratio > 1.0 and len(failures) < 5:
                    failures.append(f"error bound exceeded at {tag}: ratio {ratio:.3f}")
                series.append((float(np.max(err) / rms), float(np.mean((err / rms) ** 2))))
                if ck_gpu is not None:
                    note("checkpoint", scaled_error(ck_gpu, state), tol, tag)
            elif op == "verify":
                _, tag, drafts, accept, y_gpu, fold_local, ck_gpu, tol = msg
                if len(fold_local):   # a row folded before its drafts: checkpoint = committed state
                    note("checkpoint", scaled_error(ck_gpu, state[fold_local]), tol, tag)
                y, state = verify_round(state, drafts, np.asarray(accept))
                note("verify output", scaled_error(y_gpu, y), tol, tag)
            elif op == "checkpoint":
                _, tag, ck_gpu, tol = msg
                note("checkpoint", scaled_error(ck_gpu, state), tol, tag)
            elif op == "narrow":
                state = state[msg[1]]
            elif op == "done":
                conn.send({"worst": worst, "failures": failures, "series": series, "error": None})
                return
    except Exception:   # report, do not hang the parent
        conn.send({"worst": worst, "failures": failures, "series": series, "error": traceback.format_exc()})


class OracleWorkers:
    """One spawned oracle process per block of sequences.

    state0: fp32 numpy [B, ...] (the GPU's initial checkpoint); params: Mamba-2
    {"A": [H], "D": [H]} fp64.  All arrays passed to the methods are indexed by
    the global sequence index; the class slices them per block.
    """

    def __init__(self, kind, state0, nblocks=16, params=None, out_scale=1.0):
        ctx = mp.get_context("spawn")
        B = state0.shape[0]
        self.blocks = [list(b) for b in np.array_split(np.arange(B), min(nblocks, B))]
        self.active = [list(b) for b in self.blocks]
        self.conns, self.procs = [], []
        for blk in self.blocks:
            parent, child = ctx.Pipe()
            p = ctx.Process(target=_worker, args=(child, kind, np.ascontiguousarray(state0[blk]), params, out_scale),
                            daemon=True)
            p.start()
            self.conns.append(parent)
            self.procs.append(p)

    def rows(self):
        """Global indices of the sequences still compared, in block order."""
        return [r for a in self.active for r in a]

    def _split(self, arr_rows):
        """Split an array over self.rows() into per-block pieces."""
        out, i = [], 0
        for a in self.active:
            out.append(None if arr_rows is None else arr_rows[i:i + len(a)])
            i += len(a)
        return out

    def decode(self, tag, tok, y_rows, ck_rows, tol):
        """tok: full-batch token arrays; y_rows / ck_rows: the GPU output / checkpoint at
        self.rows() (None: not compared this step)."""
        ys, cks = self._split(y_rows), self._split(ck_rows)
        for c, a, y, ck in zip(self.conns, self.active, ys, cks):
            if a:
                c.send(("decode", tag, {k: v[a] for k, v in tok.items()}, y, ck, tol))

    def decode_bound(self, tag, tok, y_rows, bound_rows, slack, ck_rows, tol):
        """As decode, with a per-element error bound (arrays at self.rows())."""
        ys, bs, cks = self._split(y_rows), self._split(bound_rows), self._split(ck_rows)
        for c, a, y, bd, ck in zip(self.conns, self.active, ys, bs, cks):
            if a:
                c.send(("decode_bound", tag, {k: v[a] for k, v in tok.items()}, y, bd, slack, ck, tol))

    def verify(self, tag, drafts, accept, y_rows, folded, ck_folded, tol):
        """drafts: full-batch [B, k, ...]; accept [B]; y_rows: GPU outputs at self.rows();
        folded: global rows that folded before their drafts this round, ck_folded
        their GPU checkpoints (same order)."""
        ys = self._split(y_rows)
        pos = {r: i for i, r in enumerate(folded)}
        for c, a, y in zip(self.conns, self.active, ys):
            if not a:
                continue
            loc = [i for i, r in enumerate(a) if r in pos]
            ck = np.stack([ck_folded[pos[a[i]]] for i in loc]) if loc else None
            c.send(("verify", tag, {k: v[a] for k, v in drafts.items()}, np.asarray(accept)[a], y, loc, ck, tol))

    def checkpoint(self, tag, ck_rows, tol):
        for c, a, ck in zip(self.conns, self.active, self._split(ck_rows)):
            if a:
                c.send(("checkpoint", tag, ck, tol))

    def narrow(self, keep):
        """Keep comparing only the global rows in `keep`."""
        keep = set(int(r) for r in keep)
        for i, (c, a) in enumerate(zip(self.conns, self.active)):
            if not a:
                continue
            loc = [j for j, r in enumerate(a) if r in keep]
            c.send(("narrow", loc))
            self.active[i] = [a[j] for j in loc]

    def finish(self, timeout=1800):
        """Collect every worker's worst errors and failures; returns (worst, failures).
        The per-call error series of decode_bound calls, one list per worker, is
        left in self.series."""
        worst, failures = {}, []
        self.series = []
        for c, p in zip(self.conns, self.procs):
            c.send(("done",))
            if not c.poll(timeout):
                failures.append("oracle worker did not answer")
                p.kill()
                continue
            r = c.recv()
            p.join(60)
            if r["error"]:
                failures.append(r["error"])
            failures += r["failures"]
            self.series.append(r.get("series", []))
            for k, v in r["worst"].items():
                worst[k] = max(worst.get(k, 0.0), v)
        return worst, failures
