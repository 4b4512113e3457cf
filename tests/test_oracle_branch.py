"""Pins for the branch / restore reference (oracle.branch, oracle.bookkeeping).

The pins do not use the oracle's history lists: every row's state is rebuilt
from its own token lineage (the tokens it has seen since the start, copied
whole at a branch and cut back at a restore) by running the conventional
recurrence over that lineage from its origin row's initial state.  A parent
map read the wrong way round, a gather that sees rows already overwritten in
the same call, or a restore that keeps one token too many or too few makes
the two disagree.
"""
import math

import numpy as np
import pytest

import seeded_inputs as si
from oracle import bookkeeping, branch, gdn, mamba2


def _m2_case(rng, B, H, G, P, N):
    A = -np.exp(rng.uniform(0, math.log(16), H))
    D = rng.standard_normal(H)
    h0 = rng.standard_normal((B, H, P, N)) * 0.3

    def tok():
        return {"x": rng.standard_normal((B, H, P)), "B": rng.standard_normal((B, G, N)),
                "C": rng.standard_normal((B, G, N)), "dt": np.log1p(np.exp(rng.normal(-1, 0.5, (B, H))))}

    def run(h, toks):
        return mamba2.run(h, toks, A, D)
    return h0, tok, run, lambda L, cap: branch.mamba2_rows(h0, L, cap, A, D)


def _gdn_case(rng, B, H, d):
    S0 = rng.standard_normal((B, H, d, d)) * 0.2

    def unit(v):
        return v / np.linalg.norm(v, axis=-1, keepdims=True)

    def tok():
        return {"q": unit(rng.standard_normal((B, H, d))), "k": unit(rng.standard_normal((B, H, d))),
                "v": rng.standard_normal((B, H, d)), "alpha": np.exp(-0.1 * np.log1p(np.exp(rng.standard_normal((B, H))))),
                "beta": 1 / (1 + np.exp(-rng.standard_normal((B, H))))}
    return S0, tok, lambda S, toks: gdn.run(S, toks), lambda L, cap: branch.gdn_rows(S0, L, cap)


def _row(tok, b):
    return {n: v[b:b + 1] for n, v in tok.items()}


@pytest.mark.parametrize("kind", ["mamba2", "gdn"])
def test_states_and_outputs_follow_token_lineage(kind):
    rng = np.random.default_rng(31 if kind == "mamba2" else 32)
    B, L = 5, 3
    if kind == "mamba2":
        S0, tok, run, make = _m2_case(rng, B, 2, 1, 3, 4)
    else:
        S0, tok, run, make = _gdn_case(rng, B, 2, 4)
    rows = make(L, L + 1)
    origin = list(range(B))
    lineage = [[] for _ in range(B)]
    inwin = [0] * B                       # tokens since the row's last fold, counted here
    for t in range(40):
        op = rng.choice(["decode", "decode", "branch", "restore"])
        if op == "decode":
            tk = tok()
            y = rows.decode(tk)
            for b in range(B):
                lineage[b].append(_row(tk, b))
                inwin[b] = (inwin[b] + 1) % L
                _, ys = run(S0[origin[b]][None], lineage[b])
                np.testing.assert_allclose(y[b], ys[-1, 0], rtol=1e-12, atol=1e-12)
        elif op == "branch":
            parent = si.branch_parents(B, t, seed=5).numpy() if t % 3 else np.zeros(B, np.int32)
            res = rows.branch(parent)
            assert res == [bookkeeping.OK] * B
            origin = [origin[p] for p in parent]
            lineage = [list(lineage[p]) for p in parent]
            inwin = [inwin[p] for p in parent]
        else:
            keep = [int(rng.integers(0, inwin[b] + 2)) for b in range(B)]   # one past len: refused
            res = rows.restore(keep)
            for b in range(B):
                if keep[b] <= inwin[b]:
                    assert res[b] == bookkeeping.OK
                    del lineage[b][len(lineage[b]) - (inwin[b] - keep[b]):]
                    inwin[b] = keep[b]
                else:
                    assert res[b] == bookkeeping.ERR_STATE
        st = rows.state()
        for b in range(B):
            want, _ = run(S0[origin[b]][None], lineage[b]) if lineage[b] else (S0[origin[b]][None], None)
            np.testing.assert_allclose(st[b], want[0], rtol=1e-12, atol=1e-12)
        assert rows.book.len == inwin


def test_special_cases():
    rng = np.random.default_rng(33)
    B, L = 4, 4
    S0, tok, run, make = _m2_case(rng, B, 2, 2, 2, 2)
    rows = make(L, L + 1)
    rows.decode(tok())
    rows.decode(tok())
    before = rows.state().copy()
    assert rows.branch(np.arange(B)) == [bookkeeping.OK] * B          # identity: nothing moves
    np.testing.assert_array_equal(rows.state(), before)
    assert rows.restore([2] * B) == [bookkeeping.OK] * B              # keep the whole window
    np.testing.assert_array_equal(rows.state(), before)
    rows.branch(np.full(B, 2))                                        # best-of-n: all from row 2
    for b in range(B):
        np.testing.assert_array_equal(rows.state()[b], before[2])
    rows.restore([0] * B)                                             # back to the checkpoint
    np.testing.assert_array_equal(rows.state(), np.stack([S0[2]] * B))
    assert rows.book.len == [0] * B


def test_bookkeeping_hand_trace():
    """Three rows, L = 4, capacity 5, traced by hand."""
    wb = bookkeeping.WindowBook(3, 4, 5)
    wb.decode(); wb.decode()
    assert wb.snapshot() == ([0, 0, 0], [2, 2, 2], [0, 0, 0], [0, 0, 0])
    assert wb.restore([1, 2, 0]) == [0, 0, 0]
    assert wb.len == [1, 2, 0]
    assert wb.branch([1, 1, 0]) == [0, 0, 0]          # row 2 takes row 0's len from before the call
    assert wb.len == [2, 2, 1]
    wb.decode(); wb.decode()                          # row 0/1 reach 4 -> fold; row 2 reaches 3
    assert wb.snapshot() == ([4, 4, 0], [0, 0, 3], [0, 0, 0], [1, 1, 0])
    assert wb.branch([2, 0, 7]) == [0, 0, bookkeeping.ERR_STATE]   # parent 7 out of range
    assert wb.snapshot() == ([0, 4, 0], [3, 0, 3], [0, 0, 0], [0, 1, 0])
    wb.verify(1)                                      # drafts pending on every row
    assert wb.branch([1, 1, 1]) == [bookkeeping.ERR_STATE] * 3
    assert wb.restore([0, 0, 0]) == [bookkeeping.ERR_STATE] * 3


def test_branch_parents_generator():
    p = si.branch_parents(1000, 3, seed=1)
    assert p.dtype.is_floating_point is False and p.min() >= 0 and p.max() < 1000
    own = (p == np.arange(1000)).float().mean().item()
    assert 0.4 < own < 0.6
    assert np.array_equal(p.numpy(), si.branch_parents(1000, 3, seed=1).numpy())
