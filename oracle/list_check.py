"""Validity of a candidate block list against the oracle's top-p selection.

TEST INFRASTRUCTURE ONLY, like the rest of ``oracle/``: used by ``tests/``
and by the CPU-baseline leg of ``bench.py`` to compare the lists the CUDA
path wrote with the oracle's, never by the library.

The selection ("FVAttn" digest, sections 00 and 02: top-p routing with a
top-k safety floor) keeps, per query-tile row, the fewest tiles whose
probabilities summed in descending order reach p, at least k_min of them.
The oracle evaluates it in float64; a float32 evaluation may legitimately
differ on two kinds of rows, and on those rows several lists are correct:

* borderline rows: the cumulative mass at the cut lies within 1e-5 of p
  (``select_blocks``'s ``border`` flag), so the count may be any value
  between the counts at p - 1e-5 and p + 1e-5;
* near-tie rows: the last kept and the first dropped logits are closer
  than the float32 rounding bound of their dot products, so either tile
  may be kept.

On those rows a differing list is accepted when it is *valid*: ids in
range, strictly ascending, a count in the allowed range, and a top-count
set of the row's logits up to the rounding bound.  Every other row must
equal the oracle's list exactly.
"""
from __future__ import annotations

import numpy as np

from oracle.fvattn_oracle import BORDER, near_tie_rows, select_blocks

# float32 rounding bound of one pooled logit, relative to the magnitude of
# its terms scale * |Qp| . |Kp| (a 128-term dot product carries at most a few
# 2^-24 relative errors per term; 1e-5 leaves a wide margin).
TIE_REL = 1e-5


def _valid_set(S_row, sel, tol, n_tiles):
    """ids in range, strictly ascending, and a top-|sel| set of S_row up to tol."""
    if len(sel) == 0:
        return False
    if sel.min() < 0 or sel.max() >= n_tiles or (len(sel) > 1 and not (np.diff(sel) > 0).all()):
        return False
    rest = np.setdiff1d(np.arange(n_tiles), sel)
    if len(rest) == 0:
        return True
    return bool(S_row[sel].min() >= S_row[rest].max() - tol)


def check_lists(res: dict, gpu_counts, gpu_idx, top_p: float, k_min: int, equal_rows=None) -> dict:
    """Compare one head's candidate lists with the oracle's selection.

    ``res`` is ``coarse_head``'s result (S, s_abs, counts, idx, border);
    ``gpu_counts`` [nT] and ``gpu_idx`` [nT, >= count] are the candidate's
    counts and ascending ids.  Returns counts of rows: ``rows``, ``equal``,
    ``borderline`` (flagged by the oracle), ``borderline_differ`` (flagged,
    differing and valid), ``near_tie`` (flagged, not borderline),
    ``near_tie_differ`` (flagged, differing and valid), ``mismatch`` (every
    other differing row, and flagged rows whose list is not valid), and
    ``bad_rows`` (the first few mismatching row ids).  ``equal_rows``, a
    boolean array of one entry per row if given, is set where the lists are
    identical."""
    S, counts, idx, border = res["S"], res["counts"], res["idx"], res["border"]
    rows, nT = S.shape
    tol = TIE_REL * res["s_abs"].max(axis=1)
    near = near_tie_rows(S, counts, tol)
    lo = hi = None
    if border.any():
        lo = select_blocks(S, top_p - BORDER, k_min)[0]
        hi = select_blocks(S, top_p + BORDER, k_min)[0]
    out = dict(rows=rows, equal=0, borderline=int(border.sum()), borderline_differ=0,
               near_tie=int((near & ~border).sum()), near_tie_differ=0, mismatch=0, bad_rows=[])
    gpu_counts = np.asarray(gpu_counts)
    gpu_idx = np.asarray(gpu_idx)
    for r in range(rows):
        c = int(gpu_counts[r])
        sel = gpu_idx[r, :max(c, 0)].astype(np.int64)
        same = c == counts[r] and np.array_equal(sel, idx[r, :counts[r]])
        if equal_rows is not None:
            equal_rows[r] = same
        if same:
            out["equal"] += 1
            continue
        ok = False
        if border[r]:
            ok = lo[r] <= c <= hi[r] and _valid_set(S[r], sel, tol[r], nT)
            out["borderline_differ"] += int(ok)
        elif near[r]:
            ok = c == counts[r] and _valid_set(S[r], sel, tol[r], nT)
            out["near_tie_differ"] += int(ok)
        if not ok:
            out["mismatch"] += 1
            if len(out["bad_rows"]) < 8:
                out["bad_rows"].append(r)
    return out


def merge(totals: dict, one: dict) -> dict:
    """Sum the row counts of several heads (bad_rows keeps the first few)."""
    for key, val in one.items():
        if key == "bad_rows":
            totals.setdefault(key, [])
            totals[key] = (totals[key] + val)[:8]
        else:
            totals[key] = totals.get(key, 0) + val
    return totals
