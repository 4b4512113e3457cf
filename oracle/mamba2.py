"""Conventional Mamba-2 SSM recurrence in fp64 (oracle; test infrastructure).

The layer is one of the SSM layers the pages accelerate ([teaser]; [summary
¶7]).  The pages give no formula for it, so this is the standard Mamba-2
selective-state-space update with a scalar-times-identity A per head (Dao &
Gu, "Transformers are SSMs", 2024, the SSD recurrence), read as follows for
one (batch b, head h) reading group g(h) = h // (H / G):

    dA_t = exp(dt_t * A_h)
    h_t  = dA_t * h_{t-1} + dt_t * x_t B_t^T          h in R^{P x N}
    y_t  = h_t C_t + D_h * x_t

dt arrives already passed through softplus (no dt bias), and the layer's
short convolution, z-gate and norm are outside the SSM recurrence and are not
modelled.  This conventional update (read and rewrite the full state every
token) is what [summary ¶3] says ReplaySSM stops doing; its outputs are what
ReplaySSM must reproduce.
"""
from __future__ import annotations

import numpy as np


def head_groups(nheads: int, ngroups: int) -> np.ndarray:
    """Group index of every head: contiguous blocks of H/G heads."""
    if ngroups <= 0 or nheads % ngroups:
        raise ValueError("nheads must be a positive multiple of ngroups")
    return np.arange(nheads) // (nheads // ngroups)


def step(h, x, Bm, C, dt, A, D):
    """One token for every (batch, head); returns (new state, y).

    h [B,H,P,N], x [B,H,P], Bm/C [B,G,N], dt [B,H], A/D [H]; all fp64.
    """
    g = head_groups(h.shape[1], Bm.shape[1])
    Bh = Bm[:, g, :]                                  # [B,H,N]
    Ch = C[:, g, :]
    dA = np.exp(dt * A[None, :])                      # [B,H]
    h = dA[:, :, None, None] * h + (dt[:, :, None, None] * x[:, :, :, None]) * Bh[:, :, None, :]
    y = np.einsum("bhpn,bhn->bhp", h, Ch) + D[None, :, None] * x
    return h, y


def run(h0, tokens, A, D):
    """Run the recurrence over a list of token dicts {x, B, C, dt} (fp64 arrays).

    Returns (final state, ys [T,B,H,P]).
    """
    h = np.array(h0, dtype=np.float64, copy=True)
    ys = []
    for tok in tokens:
        h, y = step(h, tok["x"], tok["B"], tok["C"], tok["dt"], A, D)
        ys.append(y)
    return h, np.stack(ys) if ys else np.zeros((0,) + h.shape[:3])
