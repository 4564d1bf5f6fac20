"""The parity checkers themselves (CPU): the structural selection check must
accept every row the oracle's top-n produces and reject rows with a planted
mistake (a forced block dropped, an index out of range, the order or the
padding broken, a wrong count)."""
import numpy as np

import oracle
from helpers import selection_valid, selection_ok


def _cfg(**kw):
    c = dict(B=1, T=700, H=4, G=1, dk=16, dv=8, l=32, d=16, lp=64, n=5, fi=1, fl=2, w=64)
    c.update(kw)
    return c


def test_oracle_rows_are_valid_and_planted_mistakes_are_not():
    c = _cfg()
    rng = np.random.default_rng(11)
    rows = np.arange(c["T"])
    NS = oracle.num_sel_blocks(c, c["T"])
    idx = oracle.topn(c, rows, rng.random((c["T"], 1, NS)))
    for t in rows:
        assert selection_valid(c, t, idx[t, 0]) is None, (t, idx[t, 0])
    t = 650                                             # b_t = 10: blocks 0, 9, 10 forced
    row = list(idx[t, 0])
    assert selection_valid(c, t, row) is None
    assert 0 in row and 9 in row and 10 in row
    free = [j for j in range(1, 9) if j not in row]
    bad_forced = sorted([j for j in row if j != 9] + [free[0]])
    assert "forced" in selection_valid(c, t, bad_forced)
    assert selection_valid(c, t, row[:-1] + [11]) is not None           # beyond b_t
    assert selection_valid(c, t, [row[1], row[0]] + row[2:]) is not None  # order
    assert selection_valid(c, t, row[:-1] + [-1]) is not None            # count
    short = list(idx[100, 0])                                             # b_t = 1: 2 blocks
    assert short == [0, 1, -1, -1, -1]
    assert selection_valid(c, 100, [0, 1, 1, -1, -1]) is not None
    assert selection_valid(c, 100, [0, -1, 1, -1, -1]) is not None


def test_near_tie_acceptance_needs_a_valid_row():
    c = _cfg()
    t = 650
    pg = np.ones(11)                        # every candidate ties
    want = np.array([0, 1, 2, 9, 10])
    assert selection_ok(c, t, pg, np.array([0, 1, 3, 9, 10]), want, 0.0)           # one swap at a tie
    # a forced block traded for a tied candidate is rejected, however its score compares
    assert not selection_ok(c, t, pg, np.array([0, 1, 2, 3, 10]), want, 0.0)
    # below the slack: a lower-scoring block in place of the oracle's is rejected
    pg2 = pg.copy()
    pg2[3] = 0.5
    assert not selection_ok(c, t, pg2, np.array([0, 1, 3, 9, 10]), want, 0.0)
