"""The ReplaySSM replay form in fp64 (oracle; test infrastructure).

[summary ¶2-3]: a layer's state is kept as a checkpoint plus a buffer of the
most recent inputs; every decode step computes its output by reading the
checkpoint and replaying the buffered inputs, the state itself is not written,
and once the buffer holds L inputs they are folded into the checkpoint (a
"flush").  The pages print no formula; the forms below are the recurrences of
``mamba2`` and ``gdn`` unrolled over the window, which is the plainest reading
(and the one the test suite checks against the recurrence).

Notation for a window of l entries s = 1..l on top of checkpoint h_c:
    seg(s, t) = sum_{r=s+1..t} a_r   (direct suffix sum of log-decays)
    G_t       = seg(0, t)
Mamba-2 (a_r = dt_r * A):
    y_t  = e^{G_t} h_c C_t + sum_{s<=t} e^{seg(s,t)} dt_s (B_s . C_t) x_s + D x_t
    flush: h_c <- e^{G_l} h_c + sum_{s<=l} e^{seg(s,l)} dt_s x_s B_s^T
Gated DeltaNet (a_r = ln alpha_r), the WY/UT form:
    u_t  = h_c k_t
    w_t  = beta_t (v_t - e^{G_t} u_t - sum_{s<t} e^{seg(s,t)} (k_s . k_t) w_s)
    o_t  = e^{G_t} h_c q_t + sum_{s<=t} e^{seg(s,t)} (k_s . q_t) w_s
    flush: h_c <- e^{G_l} h_c + sum_{s<=l} e^{seg(s,l)} w_s k_s^T
The w_s solve the unit-lower-triangular system of the window (forward
substitution); they depend only on h_c and entries 1..s, so later tokens never
change them.
"""
from __future__ import annotations

import numpy as np

from .mamba2 import head_groups


def _suffix_segments(a):
    """seg[s][t] for 0 <= s <= t < l as direct sums over a list of [B,H] arrays.

    Entry indices are 0-based here: seg[s][t] = sum_{r=s+1..t} a[r], and the
    decay from the checkpoint to entry t is exp(sum_{r=0..t} a[r]).
    """
    l = len(a)
    seg = [[None] * l for _ in range(l)]
    for t in range(l):
        for s in range(t + 1):
            acc = np.zeros_like(a[0])
            for r in range(s + 1, t + 1):
                acc = acc + a[r]
            seg[s][t] = acc
    return seg


def _total(a, t):
    acc = np.zeros_like(a[0])
    for r in range(t + 1):
        acc = acc + a[r]
    return acc


class Mamba2Replay:
    """Checkpoint + window for a whole batch (every row shares one length)."""

    def __init__(self, hc, A, D, ngroups, window):
        self.hc = np.array(hc, dtype=np.float64, copy=True)
        self.A, self.D = np.asarray(A, np.float64), np.asarray(D, np.float64)
        self.groups = head_groups(self.hc.shape[1], ngroups)
        self.L = int(window)
        self.entries = []

    def _output(self, C_t, x_t):
        e = self.entries
        a = [en["dt"] * self.A[None, :] for en in e]
        seg = _suffix_segments(a)
        t = len(e) - 1
        Ch = C_t[:, self.groups, :]
        y = np.exp(_total(a, t))[:, :, None] * np.einsum("bhpn,bhn->bhp", self.hc, Ch)
        for s in range(t + 1):
            bc = np.einsum("bhn,bhn->bh", e[s]["B"][:, self.groups, :], Ch)
            coef = np.exp(seg[s][t]) * e[s]["dt"] * bc
            y = y + coef[:, :, None] * e[s]["x"]
        return y + self.D[None, :, None] * x_t

    def flush(self):
        e = self.entries
        if not e:
            return
        a = [en["dt"] * self.A[None, :] for en in e]
        seg = _suffix_segments(a)
        t = len(e) - 1
        h = np.exp(_total(a, t))[:, :, None, None] * self.hc
        for s in range(t + 1):
            w = np.exp(seg[s][t]) * e[s]["dt"]
            Bh = e[s]["B"][:, self.groups, :]
            h = h + w[:, :, None, None] * e[s]["x"][:, :, :, None] * Bh[:, :, None, :]
        self.hc = h
        self.entries = []

    def decode(self, tok):
        """Append one token, return its output; flush when the window is full."""
        self.entries.append({"x": tok["x"], "B": tok["B"], "dt": tok["dt"]})
        y = self._output(tok["C"], tok["x"])
        if len(self.entries) == self.L:
            self.flush()
        return y


class GDNReplay:
    """Checkpoint + window (with the solved w_s) for a whole batch."""

    def __init__(self, Sc, window, out_scale=1.0):
        self.Sc = np.array(Sc, dtype=np.float64, copy=True)
        self.L = int(window)
        self.out_scale = float(out_scale)
        self.entries = []

    def decode(self, tok):
        e = self.entries
        e.append({"k": tok["k"], "v": tok["v"], "a": np.log(tok["alpha"]),
                  "beta": tok["beta"]})
        a = [en["a"] for en in e]
        seg = _suffix_segments(a)
        t = len(e) - 1
        Gt = np.exp(_total(a, t))
        u = np.einsum("bhij,bhj->bhi", self.Sc, e[t]["k"])
        rhs = tok["v"] - Gt[:, :, None] * u
        for s in range(t):
            kk = np.einsum("bhj,bhj->bh", e[s]["k"], e[t]["k"])
            rhs = rhs - (np.exp(seg[s][t]) * kk)[:, :, None] * e[s]["w"]
        e[t]["w"] = tok["beta"][:, :, None] * rhs
        o = Gt[:, :, None] * np.einsum("bhij,bhj->bhi", self.Sc, tok["q"])
        for s in range(t + 1):
            kq = np.einsum("bhj,bhj->bh", e[s]["k"], tok["q"])
            o = o + (np.exp(seg[s][t]) * kq)[:, :, None] * e[s]["w"]
        if len(e) == self.L:
            self.flush()
        return self.out_scale * o

    def flush(self):
        e = self.entries
        if not e:
            return
        a = [en["a"] for en in e]
        seg = _suffix_segments(a)
        t = len(e) - 1
        S = np.exp(_total(a, t))[:, :, None, None] * self.Sc
        for s in range(t + 1):
            S = S + np.exp(seg[s][t])[:, :, None, None] * e[s]["w"][:, :, :, None] * e[s]["k"][:, :, None, :]
        self.Sc = S
        self.entries = []
