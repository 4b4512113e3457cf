"""Pins for the fp64 gated-delta-rule oracle against results fixed by the mathematics."""
import numpy as np
import pytest

from oracle import gdn


def _unit(v):
    return v / np.linalg.norm(v, axis=-1, keepdims=True)


def _rand_tokens(rng, B, H, dk, dv, T):
    return [{"q": _unit(rng.standard_normal((B, H, dk))), "k": _unit(rng.standard_normal((B, H, dk))),
             "v": rng.standard_normal((B, H, dv)),
             "alpha": np.exp(-0.1 * np.log1p(np.exp(rng.standard_normal((B, H))))),
             "beta": 1 / (1 + np.exp(-rng.standard_normal((B, H))))} for _ in range(T)]


@pytest.mark.parametrize("d", [1, 2, 3, 4])
def test_product_of_transitions(d):
    """S_t = S_0 prod_r alpha_r (I - beta_r k_r k_r^T) + sum_s beta_s v_s k_s^T prod_{r>s} (...)."""
    rng = np.random.default_rng(20 + d)
    B, H, T = 2, 3, 6
    S0 = rng.standard_normal((B, H, d, d))
    toks = _rand_tokens(rng, B, H, d, d, T)
    ST, outs = gdn.run(S0, toks, out_scale=0.7)
    for b in range(B):
        for h in range(H):
            M = [toks[t]["alpha"][b, h] * (np.eye(d) - toks[t]["beta"][b, h]
                                           * np.outer(toks[t]["k"][b, h], toks[t]["k"][b, h]))
                 for t in range(T)]
            for t in range(T):
                S = S0[b, h].copy()
                for r in range(t + 1):
                    S = S @ M[r]
                for s in range(t + 1):
                    term = toks[s]["beta"][b, h] * np.outer(toks[s]["v"][b, h], toks[s]["k"][b, h])
                    for r in range(s + 1, t + 1):
                        term = term @ M[r]
                    S = S + term
                np.testing.assert_allclose(outs[t, b, h], 0.7 * S @ toks[t]["q"][b, h], rtol=1e-12, atol=1e-12)
                if t == T - 1:
                    np.testing.assert_allclose(ST[b, h], S, rtol=1e-12, atol=1e-12)


def test_beta_zero_is_pure_decay():
    rng = np.random.default_rng(7)
    B, H, d, T = 2, 2, 5, 8
    S0 = rng.standard_normal((B, H, d, d))
    toks = _rand_tokens(rng, B, H, d, d, T)
    for t in toks:
        t["beta"] = np.zeros((B, H))
    ST, _ = gdn.run(S0, toks)
    decay = np.prod([t["alpha"] for t in toks], axis=0)
    np.testing.assert_allclose(ST, decay[:, :, None, None] * S0, rtol=1e-13)


def test_orthonormal_keys_are_memorised():
    """alpha = beta = 1, orthonormal keys: after writing (k_i, v_i), S = sum_i v_i k_i^T."""
    rng = np.random.default_rng(9)
    d, dv = 4, 3
    Q, _ = np.linalg.qr(rng.standard_normal((d, d)))
    S0 = rng.standard_normal((1, 1, dv, d))
    vs = rng.standard_normal((d, dv))
    toks = [{"q": Q[:, i][None, None], "k": Q[:, i][None, None], "v": vs[i][None, None],
             "alpha": np.ones((1, 1)), "beta": np.ones((1, 1))} for i in range(d)]
    ST, outs = gdn.run(S0, toks)
    for i in range(d):
        np.testing.assert_allclose(ST[0, 0] @ Q[:, i], vs[i], atol=1e-12)
        np.testing.assert_allclose(outs[i, 0, 0], vs[i], atol=1e-12)
    np.testing.assert_allclose(ST[0, 0], sum(np.outer(vs[i], Q[:, i]) for i in range(d)), atol=1e-12)
