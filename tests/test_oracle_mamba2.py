"""Pins for the fp64 Mamba-2 oracle against results fixed by the mathematics.

Each pin is independent of the oracle's code: an unrolled closed form written
out with Python loops, a geometric series, and a reduction to causal linear
attention computed with a cumulative sum.
"""
import math

import numpy as np
import pytest

from oracle import mamba2


def _rand_case(rng, B, H, G, P, N, T):
    A = -np.exp(rng.uniform(0, math.log(16), H))
    D = rng.standard_normal(H)
    h0 = rng.standard_normal((B, H, P, N)) * 0.3
    toks = [{"x": rng.standard_normal((B, H, P)), "B": rng.standard_normal((B, G, N)),
             "C": rng.standard_normal((B, G, N)),
             "dt": np.log1p(np.exp(rng.normal(-1, 0.5, (B, H))))} for _ in range(T)]
    return A, D, h0, toks


@pytest.mark.parametrize("P,N", [(1, 1), (2, 4), (4, 2), (4, 4)])
def test_unrolled_closed_form(P, N):
    """y_t = D x_t + e^{sum_{r<=t} a_r} h0 C_t + sum_{s<=t} e^{sum_{s<r<=t} a_r} dt_s (B_s.C_t) x_s."""
    rng = np.random.default_rng(10 + P * 7 + N)
    B, H, G, T = 2, 4, 2, 7
    A, D, h0, toks = _rand_case(rng, B, H, G, P, N, T)
    hT, ys = mamba2.run(h0, toks, A, D)
    for b in range(B):
        for h in range(H):
            g = h // (H // G)
            a = [toks[t]["dt"][b, h] * A[h] for t in range(T)]
            for t in range(T):
                for p in range(P):
                    y = D[h] * toks[t]["x"][b, h, p]
                    dec0 = math.exp(sum(a[: t + 1]))
                    y += dec0 * sum(h0[b, h, p, n] * toks[t]["C"][b, g, n] for n in range(N))
                    for s in range(t + 1):
                        bc = sum(toks[s]["B"][b, g, n] * toks[t]["C"][b, g, n] for n in range(N))
                        y += math.exp(sum(a[s + 1: t + 1])) * toks[s]["dt"][b, h] * bc * toks[s]["x"][b, h, p]
                    assert abs(ys[t, b, h, p] - y) <= 1e-12 * (1 + abs(y))
            for p in range(P):
                for n in range(N):
                    want = math.exp(sum(a)) * h0[b, h, p, n]
                    for s in range(T):
                        want += (math.exp(sum(a[s + 1:])) * toks[s]["dt"][b, h]
                                 * toks[s]["x"][b, h, p] * toks[s]["B"][b, g, n])
                    assert abs(hT[b, h, p, n] - want) <= 1e-12 * (1 + abs(want))


def test_scalar_geometric_series():
    """P = N = 1, constant inputs: h_T = q^T h0 + c (1 - q^T) / (1 - q)."""
    A, D = np.array([-2.0]), np.array([0.0])
    dt, x, Bv, C = 0.3, 1.7, -0.8, 1.0
    h0 = np.full((1, 1, 1, 1), 0.25)
    T = 9
    tok = {"x": np.full((1, 1, 1), x), "B": np.full((1, 1, 1), Bv),
           "C": np.full((1, 1, 1), C), "dt": np.full((1, 1), dt)}
    hT, ys = mamba2.run(h0, [tok] * T, A, D)
    q, c = math.exp(dt * A[0]), dt * x * Bv
    for t in range(1, T + 1):
        want = q ** t * 0.25 + c * (1 - q ** t) / (1 - q)
        assert abs(ys[t - 1, 0, 0, 0] - want * C) < 1e-14
    assert abs(hT[0, 0, 0, 0] - (q ** T * 0.25 + c * (1 - q ** T) / (1 - q))) < 1e-14


def test_zero_decay_is_causal_linear_attention():
    """A = 0, dt = 1: h_t = h0 + cumsum_s x_s B_s^T and y_t = h_t C_t + D x_t."""
    rng = np.random.default_rng(3)
    B, H, G, P, N, T = 2, 4, 2, 3, 5, 6
    _, D, h0, toks = _rand_case(rng, B, H, G, P, N, T)
    for t in toks:
        t["dt"] = np.ones((B, H))
    A = np.zeros(H)
    _, ys = mamba2.run(h0, toks, A, D)
    g = np.arange(H) // (H // G)
    outer = np.stack([t["x"][:, :, :, None] * t["B"][:, g, None, :] for t in toks])
    hs = h0[None] + np.cumsum(outer, axis=0)
    Cs = np.stack([t["C"][:, g, :] for t in toks])
    Xs = np.stack([t["x"] for t in toks])
    want = np.einsum("tbhpn,tbhn->tbhp", hs, Cs) + D[None, None, :, None] * Xs
    np.testing.assert_allclose(ys, want, rtol=1e-13, atol=1e-13)


def test_groups_are_contiguous_head_blocks():
    """Heads 2, 3 of H=4, G=2 read group 1: zeroing that group's B leaves them pure decay."""
    rng = np.random.default_rng(5)
    B, H, G, P, N, T = 1, 4, 2, 2, 3, 4
    A, D, h0, toks = _rand_case(rng, B, H, G, P, N, T)
    for t in toks:
        t["B"][:, 1, :] = 0.0
    hT, _ = mamba2.run(h0, toks, A, D)
    decay = np.exp(sum(t["dt"] for t in toks) * A[None, :])
    np.testing.assert_allclose(hT[:, 2:], decay[:, 2:, None, None] * h0[:, 2:], rtol=1e-14)
    assert not np.allclose(hT[:, :2], decay[:, :2, None, None] * h0[:, :2])
    with pytest.raises(ValueError):
        mamba2.head_groups(6, 4)
