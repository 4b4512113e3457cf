"""Conventional gated delta rule in fp64 (oracle; test infrastructure).

Gated DeltaNet is one of the SSM layers the pages accelerate ([teaser];
[summary ¶7]).  The pages give no formula, so this is the standard gated delta
rule (Yang, Kautz & Hatamizadeh, "Gated Delta Networks", 2024), with the
state S in R^{dv x dk} mapping keys to values, for one (batch, head):

    S <- alpha_t * S                              (gate, alpha in (0, 1))
    u  = S k_t                                    (current prediction for k_t)
    S <- S + beta_t * (v_t - u) k_t^T             (delta-rule write, beta in (0, 1))
    o_t = out_scale * S q_t

equivalently S_t = alpha_t S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T.
The layer's short convolutions, output gate and norm are not modelled.
"""
from __future__ import annotations

import numpy as np


def step(S, q, k, v, alpha, beta, out_scale=1.0):
    """One token for every (batch, head); returns (new state, o).

    S [B,H,dv,dk], q/k [B,H,dk], v [B,H,dv], alpha/beta [B,H]; all fp64.
    """
    S = alpha[:, :, None, None] * S
    u = np.einsum("bhij,bhj->bhi", S, k)
    S = S + beta[:, :, None, None] * (v - u)[:, :, :, None] * k[:, :, None, :]
    o = out_scale * np.einsum("bhij,bhj->bhi", S, q)
    return S, o


def run(S0, tokens, out_scale=1.0):
    """Run the rule over a list of token dicts {q, k, v, alpha, beta} (fp64).

    Returns (final state, os [T,B,H,dv]).
    """
    S = np.array(S0, dtype=np.float64, copy=True)
    outs = []
    for tok in tokens:
        S, o = step(S, tok["q"], tok["k"], tok["v"], tok["alpha"], tok["beta"], out_scale)
        outs.append(o)
    return S, np.stack(outs) if outs else np.zeros((0,) + S.shape[:3])
