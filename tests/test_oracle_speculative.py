"""Pin for the speculative reference: rolling back rejected drafts must leave the
state reached by decoding only the accepted tokens from scratch."""
import math

import numpy as np

from oracle import gdn, kda, mamba2, speculative


def test_mamba2_rollback_equals_accepted_prefix():
    rng = np.random.default_rng(11)
    B, H, G, P, N, k, R = 3, 4, 2, 2, 3, 4, 5
    A = -np.exp(rng.uniform(0, math.log(16), H))
    D = rng.standard_normal(H)
    h0 = rng.standard_normal((B, H, P, N)) * 0.1
    h = h0
    accepted = [[] for _ in range(B)]
    for r in range(R):
        drafts = {"x": rng.standard_normal((B, k, H, P)), "B": rng.standard_normal((B, k, G, N)),
                  "C": rng.standard_normal((B, k, G, N)),
                  "dt": np.log1p(np.exp(rng.normal(-1, 0.5, (B, k, H))))}
        acc = rng.integers(0, k + 1, B)
        ys, h = speculative.mamba2_round(h, drafts, acc, A, D)
        for b in range(B):
            for j in range(k):
                # output of draft j: the recurrence over accepted tokens so far, then drafts 0..j
                seq = accepted[b] + [{n: drafts[n][b:b + 1, i] for n in drafts} for i in range(j + 1)]
                _, yy = mamba2.run(h0[b:b + 1], seq, A, D)
                np.testing.assert_allclose(ys[b, j], yy[-1, 0], rtol=1e-12, atol=1e-12)
            accepted[b] += [{n: drafts[n][b:b + 1, i] for n in drafts} for i in range(int(acc[b]))]
    for b in range(B):
        hb, _ = mamba2.run(h0[b:b + 1], accepted[b], A, D)
        np.testing.assert_allclose(h[b], hb[0], rtol=1e-12, atol=1e-12)


def test_gdn_rollback_equals_accepted_prefix():
    rng = np.random.default_rng(12)
    B, H, d, k, R = 2, 3, 4, 3, 6

    def unit(v):
        return v / np.linalg.norm(v, axis=-1, keepdims=True)
    S0 = rng.standard_normal((B, H, d, d)) * 0.05
    S = S0
    accepted = [[] for _ in range(B)]
    for r in range(R):
        drafts = {"q": unit(rng.standard_normal((B, k, H, d))), "k": unit(rng.standard_normal((B, k, H, d))),
                  "v": rng.standard_normal((B, k, H, d)),
                  "alpha": np.exp(-0.1 * np.log1p(np.exp(rng.standard_normal((B, k, H))))),
                  "beta": 1 / (1 + np.exp(-rng.standard_normal((B, k, H))))}
        acc = rng.integers(0, k + 1, B)
        outs, S = speculative.gdn_round(S, drafts, acc)
        for b in range(B):
            seq = accepted[b] + [{n: drafts[n][b:b + 1, i] for n in drafts} for i in range(k)]
            _, oo = gdn.run(S0[b:b + 1], seq)
            np.testing.assert_allclose(outs[b], oo[len(accepted[b]):, 0], rtol=1e-12, atol=1e-12)
            accepted[b] += seq[len(accepted[b]): len(accepted[b]) + int(acc[b])]
    for b in range(B):
        Sb, _ = gdn.run(S0[b:b + 1], accepted[b])
        np.testing.assert_allclose(S[b], Sb[0], rtol=1e-12, atol=1e-12)


def test_kda_rollback_equals_accepted_prefix():
    rng = np.random.default_rng(13)
    B, H, d, k, R = 2, 3, 4, 3, 6

    def unit(v):
        return v / np.linalg.norm(v, axis=-1, keepdims=True)
    S0 = rng.standard_normal((B, H, d, d)) * 0.05
    S = S0
    accepted = [[] for _ in range(B)]
    for r in range(R):
        drafts = {"q": unit(rng.standard_normal((B, k, H, d))), "k": unit(rng.standard_normal((B, k, H, d))),
                  "v": rng.standard_normal((B, k, H, d)),
                  "alpha": np.exp(-0.1 * np.log1p(np.exp(rng.standard_normal((B, k, H, d))))),
                  "beta": 1 / (1 + np.exp(-rng.standard_normal((B, k, H))))}
        acc = rng.integers(0, k + 1, B)
        outs, S = speculative.kda_round(S, drafts, acc)
        for b in range(B):
            seq = accepted[b] + [{n: drafts[n][b:b + 1, i] for n in drafts} for i in range(k)]
            _, oo = kda.run(S0[b:b + 1], seq)
            np.testing.assert_allclose(outs[b], oo[len(accepted[b]):, 0], rtol=1e-12, atol=1e-12)
            accepted[b] += seq[len(accepted[b]): len(accepted[b]) + int(acc[b])]
    for b in range(B):
        Sb, _ = kda.run(S0[b:b + 1], accepted[b])
        np.testing.assert_allclose(S[b], Sb[0], rtol=1e-12, atol=1e-12)


def test_kda_round_with_equal_channel_gates_is_gdn_round():
    """A per-channel gate that is the same on every channel is the gated delta rule's
    scalar gate: the KDA round must give the GDN round's outputs and state."""
    rng = np.random.default_rng(14)
    B, H, d, k = 2, 2, 5, 4
    S0 = rng.standard_normal((B, H, d, d)) * 0.05
    a = np.exp(-0.1 * np.log1p(np.exp(rng.standard_normal((B, k, H)))))
    drafts = {"q": rng.standard_normal((B, k, H, d)), "k": rng.standard_normal((B, k, H, d)) / d,
              "v": rng.standard_normal((B, k, H, d)), "beta": 1 / (1 + np.exp(-rng.standard_normal((B, k, H))))}
    acc = np.array([1, 3])
    og, Sg = speculative.gdn_round(S0, dict(drafts, alpha=a), acc)
    ok_, Sk = speculative.kda_round(S0, dict(drafts, alpha=np.repeat(a[..., None], d, axis=-1)), acc)
    np.testing.assert_allclose(ok_, og, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(Sk, Sg, rtol=1e-12, atol=1e-12)
