"""Speculative verify / rollback reference (oracle; test infrastructure).

[summary ¶3]: draft inputs are appended to the buffer, all drafts are verified
in one pass, and rejected drafts are dropped by moving a pointer;
[guide §"Example 3: Speculative decoding and rollback"]: after verification the
longest accepted prefix is kept and the rest is rolled back.  Whatever the
storage does, the committed state after a round must be the state reached by
decoding only the accepted tokens, and the output for draft j must be the
output of the plain recurrence after drafts 1..j.  So each round is computed
here as: copy the committed state, run the k drafts through the conventional
recurrence (giving the k expected outputs), then advance every sequence's
committed state by its own accepted-prefix length.
"""
from __future__ import annotations

import numpy as np

from . import gdn, kda, mamba2


def _draft(tokens, j):
    return {name: arr[:, j] for name, arr in tokens.items()}


def mamba2_round(h, drafts, accept, A, D):
    """h [B,H,P,N] committed; drafts {x[B,k,H,P], B/C[B,k,G,N], dt[B,k,H]};
    accept [B] ints in 0..k.  Returns (outputs [B,k,H,P], new committed state)."""
    k = drafts["x"].shape[1]
    states, ys, cur = [h], [], h
    for j in range(k):
        tok = _draft(drafts, j)
        cur, y = mamba2.step(cur, tok["x"], tok["B"], tok["C"], tok["dt"], A, D)
        states.append(cur)
        ys.append(y)
    new = np.stack([states[int(accept[b])][b] for b in range(h.shape[0])])
    return np.stack(ys, axis=1), new


def gdn_round(S, drafts, accept, out_scale=1.0):
    """S [B,H,dv,dk] committed; drafts {q,k[B,k,H,dk], v[B,k,H,dv], alpha,beta[B,k,H]}."""
    k = drafts["q"].shape[1]
    states, outs, cur = [S], [], S
    for j in range(k):
        tok = _draft(drafts, j)
        cur, o = gdn.step(cur, tok["q"], tok["k"], tok["v"], tok["alpha"], tok["beta"], out_scale)
        states.append(cur)
        outs.append(o)
    new = np.stack([states[int(accept[b])][b] for b in range(S.shape[0])])
    return np.stack(outs, axis=1), new


def kda_round(S, drafts, accept, out_scale=1.0):
    """S [B,H,dv,dk] committed; drafts {q,k,alpha[B,k,H,dk], v[B,k,H,dv], beta[B,k,H]}
    (alpha one gate per key channel)."""
    k = drafts["q"].shape[1]
    states, outs, cur = [S], [], S
    for j in range(k):
        tok = _draft(drafts, j)
        cur, o = kda.step(cur, tok["q"], tok["k"], tok["v"], tok["alpha"], tok["beta"], out_scale)
        states.append(cur)
        outs.append(o)
    new = np.stack([states[int(accept[b])][b] for b in range(S.shape[0])])
    return np.stack(outs, axis=1), new
