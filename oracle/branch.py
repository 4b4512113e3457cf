"""Branch / fork and restore-to-position reference (oracle; test infrastructure).

[guide §"The State-Storage Bottleneck in Branching Workloads"]: beam search,
best-of-n sampling and tree-structured reasoning spawn several continuations
of one prefix, and at a branch point each continuation needs the prefix's
state as its own.  [guide §"What a Replay-First Design Implies"]: the decode
loop can return a sequence to the state it had at an earlier position p.

Readings the library implements:

* branch(parent): every row b at once continues from the state row parent[b]
  held *before* the call (a gather; parent[b] == b keeps the row).  A row whose
  parent is out of range or has pending drafts is refused (STATE) and left as
  it is.  The child takes the parent's whole window: entries, pointers,
  pending count (0) and fold count.
* restore(keep): row b returns to its state after the first keep[b] committed
  tokens of its current window (the tokens since its last fold);
  0 <= keep <= len, and no pending drafts, else the row is refused (STATE).

The expected values are the plain definition: each row holds its fp64 state
history since its last fold (hist[0] = the checkpoint, hist[i] = the state
after the window's i-th committed token); decode is the conventional
recurrence; branch copies histories; restore truncates one.  Window pointers
come from ``bookkeeping.WindowBook`` (its ``branch`` and ``restore``).
"""
from __future__ import annotations

import numpy as np

from . import bookkeeping, gdn, mamba2

OK, ERR_STATE = bookkeeping.OK, bookkeeping.ERR_STATE


class BranchingRows:
    """Per-row fp64 state histories of one layer, with the window book beside them.

    ``step(S, tok)`` maps states [B, ...] and one token per row to
    (new states, outputs); it is the conventional recurrence of the layer.
    """

    def __init__(self, S0, window, capacity, step):
        S0 = np.asarray(S0, np.float64)
        self.book = bookkeeping.WindowBook(S0.shape[0], window, capacity, auto_flush=True)
        self.hist = [[S0[b].copy()] for b in range(S0.shape[0])]
        self.step_fn = step

    @property
    def batch(self):
        return len(self.hist)

    def state(self):
        """Current state of every row [B, ...]."""
        return np.stack([h[-1] for h in self.hist])

    def checkpoint(self):
        """The state each row's window starts from (its checkpoint) [B, ...]."""
        return np.stack([h[0] for h in self.hist])

    def decode(self, tok):
        """One token per row; returns the outputs [B, ...] (rows refused by the
        book give NaN)."""
        new, y = self.step_fn(self.state(), tok)
        res = self.book.decode()
        y = np.array(y, np.float64)
        for b, (st, pre, _, post) in enumerate(res):
            if st != OK:
                y[b] = np.nan
                continue
            if pre:
                self.hist[b] = [self.hist[b][-1]]
            self.hist[b].append(new[b])
            if post:
                self.hist[b] = [new[b]]
        return y

    def branch(self, parent):
        res = self.book.branch(parent)
        old = [list(h) for h in self.hist]
        for b, st in enumerate(res):
            if st == OK:
                self.hist[b] = [s.copy() for s in old[int(parent[b])]]
        return res

    def flush(self, mask=None):
        res = self.book.flush(mask)
        for b, (st, folded) in enumerate(res):
            if st == OK and folded:
                self.hist[b] = [self.hist[b][-1]]
        return res

    def restore(self, keep):
        res = self.book.restore(keep)
        for b, st in enumerate(res):
            if st == OK:
                self.hist[b] = self.hist[b][: int(keep[b]) + 1]
        return res


def mamba2_rows(h0, window, capacity, A, D):
    def step(h, tok):
        return mamba2.step(h, tok["x"], tok["B"], tok["C"], tok["dt"], A, D)
    return BranchingRows(h0, window, capacity, step)


def gdn_rows(S0, window, capacity, out_scale=1.0):
    def step(S, tok):
        return gdn.step(S, tok["q"], tok["k"], tok["v"], tok["alpha"], tok["beta"], out_scale)
    return BranchingRows(S0, window, capacity, step)
