"""Pins for the timestep schedule of (top_p, k_min) and for slack-aware
augmentation: closed forms and endpoints of the schedule; for augmentation,
the makespan of the kept work list never grows (and every CTA is filled to it
when no cap binds), lists only grow, the added tiles are the best outside
tiles by brute force, and the degenerate cases (one CTA, one item per CTA,
empty rows)."""
import numpy as np

from oracle import fvattn_oracle as O


def test_timestep_schedule_closed_forms():
    assert O.timestep_params(0, 10, 0.99, 0.9, 4, 8, dense_steps=2) == (1.0, 4)
    assert O.timestep_params(1, 10, 0.99, 0.9, 4, 8, dense_steps=2) == (1.0, 4)
    p, k = O.timestep_params(2, 10, 0.99, 0.9, 4, 8, dense_steps=2)
    assert abs(p - 0.99) < 1e-15 and k == 4
    p, k = O.timestep_params(9, 10, 0.99, 0.9, 4, 8, dense_steps=2)
    assert abs(p - 0.9) < 1e-15 and k == 8
    p, k = O.timestep_params(5, 11, 0.9, 0.5, 8, 9)          # halfway: 0.7, 8.5 rounds up
    assert abs(p - 0.7) < 1e-15 and k == 9
    ps = [O.timestep_params(s, 50, 0.99, 0.8, 2, 16, dense_steps=5)[0] for s in range(50)]
    assert all(a >= b for a, b in zip(ps, ps[1:]))
    assert O.timestep_params(0, 1, 0.95, 0.5, 8, 8) == (0.95, 8)   # a single step


def _case(BH=3, nT=9, seed=0, density=0.3, empty=()):
    rng = np.random.default_rng(seed)
    S = rng.standard_normal((BH, nT, nT))
    counts = np.zeros((BH, nT), np.int64)
    idx = np.zeros((BH, nT, nT), np.int64)
    for bh in range(BH):
        for r in range(nT):
            if (bh, r) in empty:
                continue
            sel = np.flatnonzero(rng.random(nT) < density)
            if sel.size == 0:
                sel = np.array([r])
            counts[bh, r] = sel.size
            idx[bh, r, :sel.size] = sel
    return S, counts, idx


def _loads(counts, idx, order, G, nT):
    costs = [max(1, len(u)) for u in O.item_unions(counts, idx, nT)]
    return [sum(costs[order[t]] for t in range(c, len(order), G)) for c in range(G)]


def test_makespan_is_kept_and_ctas_fill_up_to_it():
    S, counts, idx = _case(BH=4, nT=12, seed=1, density=0.2)
    nT = 12
    for G in (2, 5, 7):
        c2, i2, added, order = O.augment_lists(S, counts, idx, G)
        before = _loads(counts, idx, order, G, nT)
        after = _loads(c2, i2, order, G, nT)
        assert max(after) == max(before)
        # no cap binds at this density: every CTA is filled exactly to the makespan
        assert all(a == max(before) for a in after)
        assert sum(added) == sum(max(before) - b for b in before)


def test_lists_only_grow_and_added_tiles_are_the_best_outside_tiles():
    S, counts, idx = _case(BH=2, nT=10, seed=2, density=0.25)
    nT, P = 10, 5
    c2, i2, added, order = O.augment_lists(S, counts, idx, 3)
    unions = O.item_unions(counts, idx, nT)
    for bh in range(2):
        for r in range(nT):
            old = set(idx[bh, r, :counts[bh, r]].tolist())
            new = i2[bh, r, :c2[bh, r]].tolist()
            assert new == sorted(set(new)) and old <= set(new)
    for item, u in enumerate(unions):
        bh, q = divmod(item, P)
        rows = [r for r in (2 * q, 2 * q + 1) if r < nT and counts[bh, r] > 0]
        got = set()
        for r in rows:
            got |= set(i2[bh, r, :c2[bh, r]].tolist()) - set(idx[bh, r, :counts[bh, r]].tolist())
        got -= u
        assert len(got) == added[item]
        outside = [j for j in range(nT) if j not in u]
        score = {j: max(S[bh, r, j] for r in rows) for j in outside} if rows else {}
        for j in got:                          # brute force: nothing better was left out
            for o in outside:
                if o not in got:
                    assert (score[j], -j) > (score[o], -o)
        for r in rows:                          # every live row of the item gets the same tiles
            assert got <= set(i2[bh, r, :c2[bh, r]].tolist())


def test_degenerate_cases():
    S, counts, idx = _case(BH=2, nT=8, seed=3, density=0.3, empty={(0, 3), (1, 6), (1, 7)})
    c1, i1, added, _ = O.augment_lists(S, counts, idx, 1)   # one CTA: no slack
    assert np.array_equal(c1, counts) and sum(added) == 0
    items = 2 * 4
    c2, i2, added, order = O.augment_lists(S, counts, idx, items)   # one item per CTA
    costs = [max(1, len(u)) for u in O.item_unions(counts, idx, 8)]
    for item, u in enumerate(O.item_unions(counts, idx, 8)):
        bh, q = divmod(item, 4)
        live = any(counts[bh, r] > 0 for r in (2 * q, 2 * q + 1))
        want = min(max(costs) - costs[item], 8 - len(u)) if live else 0
        assert added[item] == want
    assert c2[0, 3] == 0 and c2[1, 6] == 0 and c2[1, 7] == 0   # empty rows stay empty


def test_hand_worked_split_of_the_slack():
    """Items of costs 5, 3, 2, 1 on two CTAs: CTA 0 runs items 0 and 2 (load
    7), CTA 1 items 1 and 3 (load 4), so CTA 1's slack of 3 gives its first
    item in slot order 2 extra tiles and the second 1."""
    nT = 8
    counts = np.zeros((1, nT), np.int64)
    idx = np.zeros((1, nT, nT), np.int64)
    lists = {0: [0, 1, 2], 1: [3, 4], 2: [0, 1], 3: [2], 4: [5], 5: [6], 6: [7], 7: [7]}
    for r, lst in lists.items():
        counts[0, r] = len(lst)
        idx[0, r, :len(lst)] = lst
    S = np.zeros((1, nT, nT))
    S[0, 2] = S[0, 3] = np.arange(nT)[::-1]       # item 1 prefers low tile ids
    S[0, 6] = S[0, 7] = np.arange(nT)             # item 3 prefers high tile ids
    c2, i2, added, order = O.augment_lists(S, counts, idx, 2)
    assert order == [0, 1, 2, 3]
    assert added == [0, 2, 0, 1]
    assert i2[0, 2, :c2[0, 2]].tolist() == [0, 1, 3, 4] and i2[0, 3, :c2[0, 3]].tolist() == [2, 3, 4]
    assert i2[0, 6, :c2[0, 6]].tolist() == [6, 7] and i2[0, 7, :c2[0, 7]].tolist() == [6, 7]


def _hand_lists():
    nT = 8
    counts = np.zeros((1, nT), np.int64)
    idx = np.zeros((1, nT, nT), np.int64)
    lists = {0: [0, 1, 2], 1: [3, 4], 2: [0, 1], 3: [2], 4: [5], 5: [6], 6: [7], 7: [7]}
    for r, lst in lists.items():
        counts[0, r] = len(lst)
        idx[0, r, :len(lst)] = lst
    return counts, idx


def test_measured_slack_hand_worked():
    """The same four items (costs 5, 3, 2, 1; CTA 0 runs items 0 and 2, CTA 1
    items 1 and 3; 11 union entries in all) with measured busy times.
    CTA 0 at 500 ns and CTA 1 at 600 ns: CTA 1 is the slower one although it
    has fewer entries, so CTA 0 gets the slack, (600 - 500) * 11 * 100 /
    (100 * 1100) = 1 entry, on its first item (item 0, rows 0 and 1, union
    {0..4}); all logits are equal, so the lowest outside tile, 5, is added to
    both rows.  At 700 / 400 ns with fill 50%: CTA 1's slack is
    floor(300 * 11 * 50 / (100 * 1100)) = floor(1.5) = 1, on item 1 (rows 2
    and 3, union {0, 1, 2}): tile 3 is added to both rows."""
    counts, idx = _hand_lists()
    S = np.zeros((1, 8, 8))
    c2, i2, added, order = O.augment_lists(S, counts, idx, 2, cta_busy_ns=[500, 600])
    assert order == [0, 1, 2, 3] and added == [1, 0, 0, 0]
    assert i2[0, 0, :c2[0, 0]].tolist() == [0, 1, 2, 5] and i2[0, 1, :c2[0, 1]].tolist() == [3, 4, 5]
    assert np.array_equal(c2[0, 2:], counts[0, 2:])
    c3, i3, added3, _ = O.augment_lists(S, counts, idx, 2, cta_busy_ns=[700, 400], fill_percent=50)
    assert added3 == [0, 1, 0, 0]
    assert i3[0, 2, :c3[0, 2]].tolist() == [0, 1, 3] and i3[0, 3, :c3[0, 3]].tolist() == [2, 3]


def test_measured_slack_proportional_to_entries_matches_entry_slack():
    """Busy times proportional to the CTAs' entry loads give back the entry
    slack exactly; fill 0 adds nothing."""
    S, counts, idx = _case(BH=4, nT=12, seed=5, density=0.2)
    for G in (3, 7):
        c1, i1, added1, order = O.augment_lists(S, counts, idx, G)
        busy = [1000 * ld for ld in _loads(counts, idx, order, G, 12)]
        c2, i2, added2, _ = O.augment_lists(S, counts, idx, G, cta_busy_ns=busy)
        assert added1 == added2 and np.array_equal(c1, c2) and np.array_equal(i1, i2)
        c3, _, added3, _ = O.augment_lists(S, counts, idx, G, cta_busy_ns=busy, fill_percent=0)
        assert sum(added3) == 0 and np.array_equal(c3, counts)
