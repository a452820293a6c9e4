"""Pins of the list-validity checker (oracle/list_check.py) on hand-built rows.

The checker decides which GPU lists count as correct, so each of its rules
is exercised here with a row whose answer follows from the definition of
the top-p selection ("FVAttn" digest, sections 00 and 02): exact rows must
match, borderline rows (mass within 1e-5 of p at the cut) may take any count
between the counts at p -/+ 1e-5 but must stay a top-count set, near-tie rows
may swap tied tiles, and everything else is a mismatch."""
import numpy as np

from oracle import fvattn_oracle as O
from oracle.list_check import check_lists, merge


def res_for(S, top_p, k_min):
    S = np.asarray(S, np.float64)
    counts, idx, border = O.select_blocks(S, top_p, k_min)
    return dict(S=S, s_abs=np.ones_like(S), counts=counts, idx=idx, border=border)


def as_lists(rows, n):
    counts = np.array([len(r) for r in rows])
    idx = np.full((len(rows), n), -1)
    for i, r in enumerate(rows):
        idx[i, :len(r)] = r
    return counts, idx


def test_oracle_lists_are_equal_on_every_row():
    rng = np.random.default_rng(0)
    S = rng.normal(size=(12, 12)) * 3
    r = res_for(S, 0.9, 2)
    out = check_lists(r, r["counts"], r["idx"], 0.9, 2)
    assert out["equal"] == 12 and out["mismatch"] == 0


def test_borderline_row_accepts_either_count_but_only_top_sets():
    # probabilities 0.5, 0.3, 0.15, 0.05: the mass of the top three is p = 0.95
    S = np.log([[0.5, 0.3, 0.15, 0.05]])
    r = res_for(S, 0.95, 1)
    assert r["border"][0]
    for cand in ([0, 1, 2], [0, 1, 2, 3]):
        c, i = as_lists([cand], 4)
        out = check_lists(r, c, i, 0.95, 1)
        assert out["mismatch"] == 0 and out["borderline"] == 1, cand
    # the same counts with a non-top set, an unsorted list or a count outside [3, 4] fail
    for cand in ([0, 1, 3], [1, 0, 2], [0, 1]):
        c, i = as_lists([cand], 4)
        assert check_lists(r, c, i, 0.95, 1)["mismatch"] == 1, cand


def test_near_tie_row_may_keep_either_tied_tile():
    # logits 2, 1, 1, 0 with k_min 2: tiles 1 and 2 tie at the cut, the oracle keeps tile 1
    S = np.array([[2.0, 1.0, 1.0, 0.0]])
    r = res_for(S, 0.5, 2)
    assert list(r["idx"][0, :r["counts"][0]]) == [0, 1]
    c, i = as_lists([[0, 2]], 4)
    out = check_lists(r, c, i, 0.5, 2)
    assert out["mismatch"] == 0 and out["near_tie"] == 1 and out["near_tie_differ"] == 1
    # a near-tie row must still keep the oracle's count and the untied top tile
    for cand in ([0, 1, 2], [1, 2]):
        c, i = as_lists([cand], 4)
        assert check_lists(r, c, i, 0.5, 2)["mismatch"] == 1, cand


def test_other_rows_must_match_exactly():
    S = np.array([[3.0, 1.0, 0.0, -1.0], [0.0, 0.5, 4.0, 0.2]])
    r = res_for(S, 0.5, 1)
    assert not r["border"].any()
    c, i = as_lists([[1], [2]], 4)
    out = check_lists(r, c, i, 0.5, 1)
    assert out["mismatch"] == 1 and out["equal"] == 1 and out["bad_rows"] == [0]


def test_merge_sums_heads():
    a = dict(rows=4, equal=3, mismatch=1, bad_rows=[2])
    b = dict(rows=4, equal=4, mismatch=0, bad_rows=[])
    t = merge(merge({}, a), b)
    assert t["rows"] == 8 and t["equal"] == 7 and t["mismatch"] == 1 and t["bad_rows"] == [2]
