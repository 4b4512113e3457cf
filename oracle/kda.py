"""Kimi Delta Attention (KDA) in fp64: conventional rule and replay form
(oracle; test infrastructure).

The pages name KDA as the third SSM layer type a hybrid model may carry
([teaser]) and give no formula.  Reading taken: KDA is the gated delta rule
with the scalar gate replaced by a per-key-channel gate alpha_t in (0, 1)^dk
(a diagonal decay), with S in R^{dv x dk} mapping keys to values, for one
(batch, head):

    S <- S Diag(alpha_t)                          (channel-wise decay)
    u  = S k_t
    S <- S + beta_t (v_t - u) k_t^T               (delta-rule write)
    o_t = out_scale * S q_t

equivalently S_t = S_{t-1} Diag(alpha_t) (I - beta_t k_t k_t^T) + beta_t v_t k_t^T;
with every channel of alpha_t equal it is the gated delta rule of ``gdn``.

Replay form (the recurrence unrolled over a window of l entries on top of the
checkpoint S_c; g_r = ln alpha_r per channel, seg(s,t) = sum_{r=s+1..t} g_r as a
direct suffix sum per channel, G_t = seg(0,t), and x (.) y the elementwise
product):

    w_t = beta_t (v_t - S_c (e^{G_t} (.) k_t) - sum_{s<t} ((k_s (.) e^{seg(s,t)}) . k_t) w_s)
    o_t = out_scale (S_c (e^{G_t} (.) q_t) + sum_{s<=t} ((k_s (.) e^{seg(s,t)}) . q_t) w_s)
    flush: S_c <- S_c Diag(e^{G_l}) + sum_{s<=l} w_s (k_s (.) e^{seg(s,l)})^T

since S_{t-1} Diag(alpha_t) = S_c Diag(e^{G_t}) + sum_{s<t} w_s (k_s (.) e^{seg(s,t)})^T.
"""
from __future__ import annotations

import numpy as np


def step(S, q, k, v, alpha, beta, out_scale=1.0):
    """One token for every (batch, head); returns (new state, o).

    S [B,H,dv,dk], q/k/alpha [B,H,dk], v [B,H,dv], beta [B,H]; all fp64.
    """
    S = S * alpha[:, :, None, :]
    u = np.einsum("bhij,bhj->bhi", S, k)
    S = S + beta[:, :, None, None] * (v - u)[:, :, :, None] * k[:, :, None, :]
    o = out_scale * np.einsum("bhij,bhj->bhi", S, q)
    return S, o


def run(S0, tokens, out_scale=1.0):
    """The rule over a list of token dicts {q, k, v, alpha, beta}; (final state, os [T,B,H,dv])."""
    S = np.array(S0, dtype=np.float64, copy=True)
    outs = []
    for tok in tokens:
        S, o = step(S, tok["q"], tok["k"], tok["v"], tok["alpha"], tok["beta"], out_scale)
        outs.append(o)
    return S, np.stack(outs) if outs else np.zeros((0,) + S.shape[:3])


class KDAReplay:
    """Checkpoint + window for a whole batch (every row shares one length): the
    replay form above, step by step (w solved once per entry, by forward
    substitution, and kept)."""

    def __init__(self, Sc, window, out_scale=1.0):
        self.Sc = np.array(Sc, dtype=np.float64, copy=True)
        self.L, self.scale = int(window), float(out_scale)
        self.k, self.g, self.w = [], [], []

    def _seg(self, s, t):
        """seg(s, t) per channel [B,H,dk], entries 0-based: sum of g[r], s < r <= t."""
        acc = np.zeros_like(self.g[0])
        for r in range(s + 1, t + 1):
            acc = acc + self.g[r]
        return acc

    def _total(self, t):
        acc = np.zeros_like(self.g[0])
        for r in range(t + 1):
            acc = acc + self.g[r]
        return acc

    def decode(self, q, k, v, alpha, beta):
        self.k.append(np.asarray(k, np.float64))
        self.g.append(np.log(np.asarray(alpha, np.float64)))
        t = len(self.k) - 1
        Gt = np.exp(self._total(t))
        r = np.asarray(v, np.float64) - np.einsum("bhij,bhj->bhi", self.Sc, Gt * k)
        for s in range(t):
            r = r - np.sum(self.k[s] * np.exp(self._seg(s, t)) * k, -1)[:, :, None] * self.w[s]
        self.w.append(np.asarray(beta, np.float64)[:, :, None] * r)
        o = np.einsum("bhij,bhj->bhi", self.Sc, Gt * q)
        for s in range(t + 1):
            o = o + np.sum(self.k[s] * np.exp(self._seg(s, t)) * q, -1)[:, :, None] * self.w[s]
        if len(self.k) == self.L:
            self.flush()
        return self.scale * o

    def flush(self):
        l = len(self.k)
        if l == 0:
            return
        Sc = self.Sc * np.exp(self._total(l - 1))[:, :, None, :]
        for s in range(l):
            Sc = Sc + self.w[s][:, :, :, None] * (self.k[s] * np.exp(self._seg(s, l - 1)))[:, :, None, :]
        self.Sc = Sc
        self.k, self.g, self.w = [], [], []

    def state(self):
        """The current state (checkpoint with the window folded in), without folding."""
        l = len(self.k)
        if l == 0:
            return self.Sc.copy()
        S = self.Sc * np.exp(self._total(l - 1))[:, :, None, :]
        for s in range(l):
            S = S + self.w[s][:, :, :, None] * (self.k[s] * np.exp(self._seg(s, l - 1)))[:, :, None, :]
        return S
