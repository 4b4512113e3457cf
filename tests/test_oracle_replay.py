"""The replay form (checkpoint + replayed window, flush every L tokens) equals
the sequential recurrence for every window length, in fp64."""
import math

import numpy as np
import pytest

from oracle import gdn, mamba2, replay

WINDOWS = [1, 2, 3, 4, 8, 16, 32]


def _m2_case(rng, B, H, G, P, N, T):
    A = -np.exp(rng.uniform(0, math.log(16), H))
    D = rng.standard_normal(H)
    h0 = rng.standard_normal((B, H, P, N)) * 0.1
    toks = [{"x": rng.standard_normal((B, H, P)), "B": rng.standard_normal((B, G, N)),
             "C": rng.standard_normal((B, G, N)),
             "dt": np.log1p(np.exp(rng.normal(-1, 0.5, (B, H))))} for _ in range(T)]
    return A, D, h0, toks


@pytest.mark.parametrize("L", WINDOWS)
def test_mamba2_replay_equals_recurrence(L):
    rng = np.random.default_rng(100 + L)
    B, H, G, P, N = 2, 4, 2, 3, 5
    T = 2 * L + 3                        # several flushes and a ragged tail
    A, D, h0, toks = _m2_case(rng, B, H, G, P, N, T)
    hT, ys = mamba2.run(h0, toks, A, D)
    rp = replay.Mamba2Replay(h0, A, D, G, L)
    got = np.stack([rp.decode(t) for t in toks])
    np.testing.assert_allclose(got, ys, rtol=1e-12, atol=1e-12)
    assert len(rp.entries) == T % L
    rp.flush()
    np.testing.assert_allclose(rp.hc, hT, rtol=1e-12, atol=1e-12)


def test_mamba2_replay_never_touches_checkpoint_between_flushes():
    rng = np.random.default_rng(1)
    A, D, h0, toks = _m2_case(rng, 1, 2, 1, 2, 3, 5)
    rp = replay.Mamba2Replay(h0, A, D, 1, 16)
    for t in toks:
        rp.decode(t)
        assert np.array_equal(rp.hc, h0)


def _gdn_case(rng, B, H, dk, dv, T):
    def unit(v):
        return v / np.linalg.norm(v, axis=-1, keepdims=True)
    S0 = rng.standard_normal((B, H, dv, dk)) * 0.05
    toks = [{"q": unit(rng.standard_normal((B, H, dk))), "k": unit(rng.standard_normal((B, H, dk))),
             "v": rng.standard_normal((B, H, dv)),
             "alpha": np.exp(-0.1 * np.log1p(np.exp(rng.standard_normal((B, H))))),
             "beta": 1 / (1 + np.exp(-rng.standard_normal((B, H))))} for _ in range(T)]
    return S0, toks


@pytest.mark.parametrize("L", WINDOWS)
def test_gdn_replay_equals_recurrence(L):
    rng = np.random.default_rng(200 + L)
    B, H, dk, dv = 2, 3, 6, 5
    T = 2 * L + 3
    S0, toks = _gdn_case(rng, B, H, dk, dv, T)
    ST, outs = gdn.run(S0, toks, out_scale=1.0)
    rp = replay.GDNReplay(S0, L)
    got = np.stack([rp.decode(t) for t in toks])
    np.testing.assert_allclose(got, outs, rtol=1e-12, atol=1e-12)
    rp.flush()
    np.testing.assert_allclose(rp.Sc, ST, rtol=1e-12, atol=1e-12)


def test_gdn_strong_decay_window_32():
    """Small alphas over a 32-entry window: products of decays far below fp32 range
    stay exact because segments are direct sums of logs."""
    rng = np.random.default_rng(4)
    S0, toks = _gdn_case(rng, 1, 2, 4, 4, 40)
    for t in toks:
        t["alpha"] = np.full((1, 2), 0.02)
    ST, outs = gdn.run(S0, toks)
    rp = replay.GDNReplay(S0, 32)
    got = np.stack([rp.decode(t) for t in toks])
    np.testing.assert_allclose(got, outs, rtol=1e-11, atol=1e-12)
