"""Window pointer bookkeeping (oracle; test infrastructure).

[summary ¶3]: inputs are cached and folded into the checkpoint ("flush") when
the buffer fills; speculative drafts are appended to the buffer and rejected
ones are discarded by moving a pointer, without per-token state snapshots.
The pages leave the exact rule open; this module is the reading the library
implements, written per sequence in plain integers:

* A sequence's window lives in a ring of ``capacity`` slots.  ``start`` is the
  ring slot of its oldest entry, ``len`` the number of committed entries and
  ``pending`` the number of draft entries after them.  Entry i (0-based) is in
  slot (start + i) mod capacity.  ``flushes`` counts folds.
* A fold moves ``start`` past the committed entries and sets ``len`` to 0.
* decode (one token): refused (STATE) while drafts are pending.  If the token
  does not fit (len + 1 > L) the committed entries are folded first (with
  auto-flush; otherwise CAPACITY and the row is left alone).  The token is
  written to slot (start + len) and committed.  When len reaches L (window
  full) the window is folded right away (auto-flush).
* verify (k drafts): refused (STATE) while drafts are pending.  If
  len + k > L the committed entries are folded first (auto-flush; otherwise
  CAPACITY).  The drafts go to slots (start + len + j), j < k, as pending.
* rollback (n_reject): refused (STATE) unless 0 <= n_reject <= pending; else
  len += pending - n_reject and pending = 0.  Nothing else moves.
* flush: refused (STATE) while drafts are pending; folds a non-empty window.
* branch (parent): row b takes row parent[b]'s pointers from before the call
  (refused, STATE, if the parent is out of range or has pending drafts).
* restore (keep): len = keep, for 0 <= keep <= len with no pending drafts
  (else refused, STATE); the dropped entries are simply overwritten later.

With capacity >= L + max(k, 1) the slots a call writes never overlap the slots
a fold in the same call reads, and len + pending never exceeds L.
"""
from __future__ import annotations

OK, ERR_STATE, ERR_CAPACITY = 0, 1, 2


class WindowBook:
    def __init__(self, batch: int, window: int, capacity: int, auto_flush: bool = True):
        if window < 1 or capacity < window + 1:
            raise ValueError("need window >= 1 and capacity >= window + 1")
        self.L, self.cap, self.auto = int(window), int(capacity), bool(auto_flush)
        self.start = [0] * batch
        self.len = [0] * batch
        self.pending = [0] * batch
        self.flushes = [0] * batch

    @property
    def batch(self) -> int:
        return len(self.start)

    def _fold(self, b: int) -> None:
        self.start[b] = (self.start[b] + self.len[b]) % self.cap
        self.len[b] = 0
        self.flushes[b] += 1

    def decode(self):
        """Returns per row (status, pre_fold, slot, post_fold)."""
        out = []
        for b in range(self.batch):
            if self.pending[b]:
                out.append((ERR_STATE, False, None, False))
                continue
            pre = self.len[b] + 1 > self.L
            if pre and not self.auto:
                out.append((ERR_CAPACITY, False, None, False))
                continue
            if pre:
                self._fold(b)
            slot = (self.start[b] + self.len[b]) % self.cap
            self.len[b] += 1
            post = self.auto and self.len[b] == self.L
            if post:
                self._fold(b)
            out.append((OK, pre, slot, post))
        return out

    def verify(self, k: int):
        """Returns per row (status, pre_fold, slots)."""
        if not 1 <= k <= self.L or self.L + k > self.cap:
            raise ValueError("draft count out of range")
        out = []
        for b in range(self.batch):
            if self.pending[b]:
                out.append((ERR_STATE, False, None))
                continue
            pre = self.len[b] + k > self.L
            if pre and not self.auto:
                out.append((ERR_CAPACITY, False, None))
                continue
            if pre:
                self._fold(b)
            slots = [(self.start[b] + self.len[b] + j) % self.cap for j in range(k)]
            self.pending[b] = k
            out.append((OK, pre, slots))
        return out

    def rollback(self, n_reject):
        out = []
        for b in range(self.batch):
            n = int(n_reject[b])
            if n < 0 or n > self.pending[b]:
                out.append(ERR_STATE)
                continue
            self.len[b] += self.pending[b] - n
            self.pending[b] = 0
            out.append(OK)
        return out

    def flush(self, mask=None):
        out = []
        for b in range(self.batch):
            if mask is not None and not mask[b]:
                out.append((OK, False))
                continue
            if self.pending[b]:
                out.append((ERR_STATE, False))
                continue
            folded = self.len[b] > 0
            if folded:
                self._fold(b)
            out.append((OK, folded))
        return out

    def branch(self, parent):
        """Row b takes the pointers of row parent[b] as they were before the call
        [guide §"The State-Storage Bottleneck in Branching Workloads"].  Refused
        (STATE) if the parent is out of range or has pending drafts."""
        old = self.snapshot()
        out = []
        for b in range(self.batch):
            p = int(parent[b])
            if not 0 <= p < self.batch or old[2][p]:
                out.append(ERR_STATE)
                continue
            self.start[b], self.len[b] = old[0][p], old[1][p]
            self.pending[b], self.flushes[b] = old[2][p], old[3][p]
            out.append(OK)
        return out

    def restore(self, keep):
        """Keep only the first keep[b] committed entries of row b's window
        [guide §"What a Replay-First Design Implies": restore to position p].
        Refused (STATE) unless 0 <= keep <= len and no drafts are pending."""
        out = []
        for b in range(self.batch):
            k = int(keep[b])
            if self.pending[b] or not 0 <= k <= self.len[b]:
                out.append(ERR_STATE)
                continue
            self.len[b] = k
            out.append(OK)
        return out

    def snapshot(self):
        return (list(self.start), list(self.len), list(self.pending), list(self.flushes))
