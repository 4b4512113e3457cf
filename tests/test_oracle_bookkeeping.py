"""Pins for the window pointer rules: a hand-traced fixture and an explicit
list-of-tokens model that the pointer arithmetic must always agree with."""
import os
import random

import pytest

from oracle.bookkeeping import ERR_CAPACITY, ERR_STATE, OK, WindowBook

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_hand_traced_fixture():
    book = WindowBook(batch=1, window=4, capacity=6)
    with open(os.path.join(GOLDEN, "bookkeeping_trace.txt")) as f:
        lines = [l for l in f if l.strip() and not l.startswith("#")]
    for line in lines:
        op, expect, slots = [p.strip() for p in line.split("|")]
        name, arg = op.split()
        status, start, length, pending, flushes = map(int, expect.split())
        if name == "decode":
            st, _, slot, _ = book.decode()[0]
            got_slots = [slot] if st == OK else []
        elif name == "verify":
            st, _, sl = book.verify(int(arg))[0]
            got_slots = sl if st == OK else []
        elif name == "rollback":
            st = book.rollback([int(arg)])[0]
            got_slots = []
        else:
            st, _ = book.flush()[0]
            got_slots = []
        assert st == status, line
        assert (book.start[0], book.len[0], book.pending[0], book.flushes[0]) == \
            (start, length, pending, flushes), line
        assert got_slots == ([] if slots == "-" else [int(s) for s in slots.split()]), line


class ListModel:
    """The window as explicit Python lists of token ids (obviously correct)."""

    def __init__(self, L):
        self.L, self.committed, self.drafts, self.folded = L, [], [], []

    def fold(self):
        self.folded.append(list(self.committed))
        self.committed = []


@pytest.mark.parametrize("L,k", [(1, 1), (4, 2), (16, 4), (5, 5), (32, 4)])
def test_pointer_rules_agree_with_list_model(L, k):
    rnd = random.Random(L * 100 + k)
    cap = L + k
    book = WindowBook(batch=1, window=L, capacity=cap)
    model = ListModel(L)
    ring = [None] * cap
    next_id = 0
    for _ in range(3000):
        op = rnd.choice(["decode", "verify", "rollback", "rollback", "flush"])
        folds_before = book.flushes[0]
        if op == "decode":
            st, pre, slot, post = book.decode()[0]
            if model.drafts:
                assert st == ERR_STATE
                continue
            assert st == OK
            if len(model.committed) + 1 > L:
                assert pre
                model.fold()
            ring[slot] = next_id
            model.committed.append(next_id)
            next_id += 1
            if len(model.committed) == L:
                assert post
                model.fold()
        elif op == "verify":
            st, pre, slots = book.verify(k)[0]
            if model.drafts:
                assert st == ERR_STATE
                continue
            assert pre == (len(model.committed) + k > L)
            if pre:
                model.fold()
            for s in slots:
                # a draft never overwrites a committed entry
                assert ring[s] not in model.committed
                ring[s] = next_id
                model.drafts.append(next_id)
                next_id += 1
        elif op == "rollback":
            n = rnd.randint(-1, k + 1)
            st = book.rollback([n])[0]
            if n < 0 or n > len(model.drafts):
                assert st == ERR_STATE
                continue
            model.committed += model.drafts[: len(model.drafts) - n]
            model.drafts = []
        else:
            st, folded = book.flush()[0]
            if model.drafts:
                assert st == ERR_STATE
                continue
            assert folded == bool(model.committed)
            if model.committed:
                model.fold()
        # pointer view == list view
        assert book.flushes[0] - folds_before in (0, 1, 2)
        assert book.flushes[0] == len(model.folded)
        assert book.len[0] == len(model.committed) and book.pending[0] == len(model.drafts)
        assert book.len[0] + book.pending[0] <= L
        view = [ring[(book.start[0] + i) % cap] for i in range(book.len[0] + book.pending[0])]
        assert view == model.committed + model.drafts


def test_capacity_error_without_auto_flush():
    book = WindowBook(batch=2, window=2, capacity=4, auto_flush=False)
    book.decode()
    book.decode()
    st = book.decode()
    assert [s[0] for s in st] == [ERR_CAPACITY, ERR_CAPACITY]
    assert book.len == [2, 2] and book.flushes == [0, 0]
    assert [s[0] for s in book.verify(1)] == [ERR_CAPACITY] * 2
    book.flush(mask=[1, 0])
    assert book.len == [0, 2] and book.flushes == [1, 0]
