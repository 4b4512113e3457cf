"""Pins for the fp64 KDA oracle (oracle.kda) against results fixed by the
mathematics, independent of its code: the gated delta rule it reduces to when
every channel of the gate is equal, the explicit product of per-token
transition matrices (written with Python loops over d x d matrices), pure
channel-wise decay when beta = 0, exact key/value memorisation, and the replay
form equal to the recurrence for every window length."""
import numpy as np
import pytest

from oracle import gdn, kda


def _unit(v):
    return v / np.linalg.norm(v, axis=-1, keepdims=True)


def _tokens(rng, B, H, d, T, alpha_lo=0.5):
    return [{"q": _unit(rng.standard_normal((B, H, d))), "k": _unit(rng.standard_normal((B, H, d))),
             "v": rng.standard_normal((B, H, d)), "alpha": rng.uniform(alpha_lo, 1.0, (B, H, d)),
             "beta": rng.uniform(0.05, 0.95, (B, H))} for _ in range(T)]


def test_equal_channel_gates_are_the_gated_delta_rule():
    rng = np.random.default_rng(41)
    B, H, d = 2, 3, 5
    S = rng.standard_normal((B, H, d, d))
    for tok in _tokens(rng, B, H, d, 6):
        a = tok["alpha"][:, :, 0]
        S1, o1 = kda.step(S, tok["q"], tok["k"], tok["v"], np.repeat(a[:, :, None], d, -1), tok["beta"])
        S2, o2 = gdn.step(S, tok["q"], tok["k"], tok["v"], a, tok["beta"])
        np.testing.assert_allclose(S1, S2, rtol=1e-14, atol=1e-14)
        np.testing.assert_allclose(o1, o2, rtol=1e-14, atol=1e-14)
        S = S1


@pytest.mark.parametrize("d", [1, 2, 4])
def test_product_of_transitions(d):
    """S_T = S_0 M_1 ... M_T + sum_s beta_s v_s k_s^T M_{s+1} ... M_T,
    M_t = Diag(alpha_t) (I - beta_t k_t k_t^T); o_t = S_t q_t."""
    rng = np.random.default_rng(42 + d)
    T = 6
    S0 = rng.standard_normal((1, 1, d, d))
    toks = _tokens(rng, 1, 1, d, T)
    Sk, os_ = kda.run(S0, toks)
    M = []
    for tok in toks:
        a, k, b = tok["alpha"][0, 0], tok["k"][0, 0], tok["beta"][0, 0]
        Mt = np.zeros((d, d))
        for i in range(d):
            for j in range(d):
                Mt[i, j] = a[i] * ((1.0 if i == j else 0.0) - b * k[i] * k[j])
        M.append(Mt)
    for t in range(1, T + 1):
        S = S0[0, 0].copy()
        for r in range(t):
            S = S @ M[r]
        for s in range(t):
            tok = toks[s]
            term = tok["beta"][0, 0] * np.outer(tok["v"][0, 0], tok["k"][0, 0])
            for r in range(s + 1, t):
                term = term @ M[r]
            S = S + term
        np.testing.assert_allclose(os_[t - 1, 0, 0], S @ toks[t - 1]["q"][0, 0], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(Sk[0, 0], S, rtol=1e-12, atol=1e-12)


def test_beta_zero_is_channel_decay():
    rng = np.random.default_rng(44)
    B, H, d = 2, 2, 4
    S0 = rng.standard_normal((B, H, d, d))
    toks = _tokens(rng, B, H, d, 5)
    for tok in toks:
        tok["beta"] = np.zeros((B, H))
    S, _ = kda.run(S0, toks)
    prod = np.prod(np.stack([t["alpha"] for t in toks]), 0)       # [B,H,d] per key channel
    np.testing.assert_allclose(S, S0 * prod[:, :, None, :], rtol=1e-13, atol=1e-13)


def test_orthonormal_keys_memorise():
    rng = np.random.default_rng(45)
    d = 4
    Q, _ = np.linalg.qr(rng.standard_normal((d, d)))
    S = rng.standard_normal((1, 1, d, d))
    vs = []
    for i in range(d):
        v = rng.standard_normal((1, 1, d))
        vs.append(v[0, 0])
        S, _ = kda.step(S, Q[:, i][None, None], Q[:, i][None, None], v, np.ones((1, 1, d)), np.ones((1, 1)))
    for i in range(d):
        np.testing.assert_allclose(S[0, 0] @ Q[:, i], vs[i], rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("L", [1, 2, 3, 4, 8, 16, 32])
def test_replay_equals_recurrence(L):
    rng = np.random.default_rng(50 + L)
    B, H, d, T = 2, 2, 4, 40
    S0 = rng.standard_normal((B, H, d, d)) * 0.3
    toks = _tokens(rng, B, H, d, T, alpha_lo=0.05)   # strong decays: e^{G} down to ~1e-40 at L = 32
    rep = kda.KDAReplay(S0, L)
    S = S0
    for t, tok in enumerate(toks):
        o = rep.decode(tok["q"], tok["k"], tok["v"], tok["alpha"], tok["beta"])
        S, o_ref = kda.step(S, tok["q"], tok["k"], tok["v"], tok["alpha"], tok["beta"])
        np.testing.assert_allclose(o, o_ref, rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(rep.state(), S, rtol=1e-12, atol=1e-12)
    rep.flush()
    np.testing.assert_allclose(rep.Sc, S, rtol=1e-12, atol=1e-12)
