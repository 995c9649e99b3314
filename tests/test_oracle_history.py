"""Pins of the oracle's weight-free history drafts: values planted by hand
(key occurrences, rewards, groups) and the one-hot draft rows."""
import numpy as np

import oracle


def _hist(rows, lens=None, width=64):
    H = len(rows)
    t = np.full((H, width), 7777, dtype=np.int32)
    for h, r in enumerate(rows):
        t[h, :len(r)] = r
    return t, np.array([len(r) for r in rows] if lens is None else lens, dtype=np.int32)


def _seqs(rows, width=32):
    s = np.zeros((len(rows), width), dtype=np.int32)
    for b, r in enumerate(rows):
        s[b, :len(r)] = r
    return s, np.array([len(r) for r in rows], dtype=np.int32)


KEY = [11, 12, 13]


def test_planted_key_gives_the_following_tokens():
    ht, hl = _hist([[1, 2, 3, 4, 5] + KEY + [100, 101, 102, 103, 104]])
    st, sl = _seqs([[9, 9] + KEY])
    d, n, _ = oracle.history_draft(ht, hl, [0.5], [0], st, sl, [0], 3, 4)
    assert d.tolist() == [[100, 101, 102, 103]] and n.tolist() == [4]


def test_highest_reward_then_lowest_index_then_first_position():
    rows = [KEY + [1, 1], [0] + KEY + [2, 2] + KEY + [3, 3], KEY + [4, 4]]
    ht, hl = _hist(rows)
    st, sl = _seqs([KEY])
    d, n, _ = oracle.history_draft(ht, hl, [0.2, 0.9, 0.9], [0, 0, 0], st, sl, [0], 3, 2)
    assert d.tolist() == [[2, 2]] and n.tolist() == [2]      # response 1 (reward 0.9, lower index), first position


def test_own_group_first_then_any_group():
    rows = [KEY + [5, 5], KEY + [6, 6]]
    ht, hl = _hist(rows)
    st, sl = _seqs([KEY, KEY])
    d, n, _ = oracle.history_draft(ht, hl, [0.1, 0.9], [0, 1], st, sl, [0, 2], 3, 2)
    assert d.tolist() == [[5, 5], [6, 6]]                   # group 0 finds its own; group 2 falls back to the best
    assert n.tolist() == [2, 2]


def test_truncation_padding_and_misses():
    rows = [[0, 0] + KEY + [8]]
    ht, hl = _hist(rows)
    st, sl = _seqs([KEY, [11, 99, 13], [12, 13]])
    d, n, p = oracle.history_draft(ht, hl, [1.0], [0], st, sl, [0, 0, 0], 3, 4, vocab=10)
    assert d.tolist() == [[8, 0, 0, 0], [0, 0, 0, 0], [0, 0, 0, 0]]
    assert n.tolist() == [1, 0, 0]                          # one token after the key; no match; too short
    # one-hot rows at the (padded) draft tokens
    assert p.shape == (3, 4, 10) and (p.sum(-1) == 1).all() and p[0, 0, 8] == 1 and p[1, 2, 0] == 1


def test_key_must_leave_a_token_after_it():
    ht, hl = _hist([[0] + KEY])                             # the key ends the response
    st, sl = _seqs([KEY])
    d, n, _ = oracle.history_draft(ht, hl, [1.0], [0], st, sl, [0], 3, 2)
    assert n.tolist() == [0]
