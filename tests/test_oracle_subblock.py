"""Pins of the oracle's hierarchical (sub-block) scoring ("DFSAttn" digest,
section 2: a block is split into smaller sub-blocks whose scores are summed
into the block's importance).  CPU only."""
import itertools
import math

import numpy as np
import pytest

from oracle import fvattn_oracle as O

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def test_subblocks_are_aligned_2x2x2_cubes():
    grid = (8, 8, 12)
    for order in ("raster", "hilbert"):
        pos = O.positions(grid, order)
        ct = O.to_tiled(O.token_coords(grid), pos)
        ids = O.subblock_ids(ct)
        for t in range(ct.shape[0] // 64):
            rows = slice(64 * t, 64 * t + 64)
            c, i = ct[rows], ids[rows]
            assert sorted(np.bincount(i, minlength=8)) == [8] * 8
            for s in range(8):
                sc = c[i == s]
                # the 8 tokens form one aligned 2x2x2 cube
                assert (sc // 2 == sc[0] // 2).all()
                assert len({tuple(x) for x in sc}) == 8


def test_one_subblock_per_tile_is_the_plain_coarse_softmax():
    rng = np.random.default_rng(1)
    grid, d = (8, 8, 8), 16
    q, k = rng.normal(size=(512, d)), rng.normal(size=(512, d))
    for order in ("raster", "hilbert"):
        plain = O.coarse_head(q, k, grid, order, 0.6, 2, 0.3)
        whole = O.coarse_head_subblock(q, k, grid, order, 0.6, 2, 0.3, sub=(4, 4, 4))
        assert np.allclose(np.exp(whole["logP"]), plain["P"], rtol=0, atol=1e-14)
        assert np.array_equal(whole["counts"], plain["counts"])
        assert np.array_equal(whole["idx"], plain["idx"])


def test_brute_force_sum_of_subblock_softmax_masses():
    rng = np.random.default_rng(2)
    grid, d, scale = (4, 4, 8), 4, 0.7                     # 2 tiles x 8 sub-blocks
    q, k = rng.normal(size=(128, d)), rng.normal(size=(128, d))
    r = O.coarse_head_subblock(q, k, grid, "raster", 0.5, 1, scale)
    coords = O.token_coords(grid)

    def members(tile, sub):
        out = []
        for n, (t, h, w) in enumerate(coords):
            if w // 4 == tile and (t % 4) // 2 * 4 + (h % 4) // 2 * 2 + (w % 4) // 2 == sub:
                out.append(n)
        return out

    mean = lambda x, rows: [sum(x[r][c] for r in rows) / len(rows) for c in range(d)]  # noqa: E731
    qs = {(i, a): mean(q, members(i, a)) for i in range(2) for a in range(8)}
    ks = {(j, b): mean(k, members(j, b)) for j in range(2) for b in range(8)}
    for i in range(2):
        P = [0.0, 0.0]
        for a in range(8):
            logits = {(j, b): scale * sum(x * y for x, y in zip(qs[i, a], ks[j, b]))
                      for j in range(2) for b in range(8)}
            m = max(logits.values())
            z = sum(math.exp(v - m) for v in logits.values())
            for (j, b), v in logits.items():
                P[j] += math.exp(v - m) / z / 8
        assert np.allclose(np.exp(r["logP"][i]), P, rtol=1e-13, atol=0)


def test_rows_sum_to_one_and_relabelling_subblocks_changes_nothing():
    rng = np.random.default_rng(3)
    nT, S, d = 6, 8, 8
    qs, ks = rng.normal(size=(nT, S, d)) * 2, rng.normal(size=(nT, S, d)) * 2
    logP = O.subblock_tile_logprob(qs, ks, 0.5)
    assert np.allclose(np.exp(logP).sum(axis=1), 1.0, atol=1e-13)
    perm_q = np.stack([rng.permutation(S) for _ in range(nT)])
    perm_k = np.stack([rng.permutation(S) for _ in range(nT)])
    qs2 = np.take_along_axis(qs, perm_q[:, :, None], axis=1)
    ks2 = np.take_along_axis(ks, perm_k[:, :, None], axis=1)
    assert np.allclose(O.subblock_tile_logprob(qs2, ks2, 0.5), logP, atol=1e-12)


def test_raster_and_hilbert_give_the_same_tile_probabilities():
    rng = np.random.default_rng(4)
    grid, d = (8, 8, 16), 8
    q, k = rng.normal(size=(1024, d)), rng.normal(size=(1024, d))
    res = {}
    for order in ("raster", "hilbert"):
        r = O.coarse_head_subblock(q, k, grid, order, 0.7, 2, 0.4)
        cubes = [tuple(c) for c in O.tile_cubes(grid, r["pos"])]
        res[order] = {(cubes[i], cubes[j]): r["P"][i, j] for i in range(len(cubes)) for j in range(len(cubes))}
    for key, v in res["raster"].items():
        assert abs(res["hilbert"][key] - v) < 1e-13


def test_hidden_detail_closed_form():
    """Query tile 0 has one sub-cube whose 8 queries are (c, 0); key tile 2 has
    one sub-cube whose 8 keys are (1, 0); every other vector is 0 (scale 1).
    Sub-block scoring: the seven flat query sub-blocks spread their mass evenly
    (1/3 per tile) and the sharp one gives tile 2 (e^c + 7) / (e^c + 23), so
    P[0, 2] = (7/3 + (e^c + 7)/(e^c + 23)) / 8 and P[0, 0] = P[0, 1] =
    (7/3 + 8/(e^c + 23)) / 8.  Pooled tile means see only a logit of c/64."""
    grid, c = (4, 4, 12), 8.0
    coords = O.token_coords(grid)
    q = np.zeros((192, 2))
    k = np.zeros((192, 2))
    sub0 = (coords[:, 0] < 2) & (coords[:, 1] < 2) & (coords[:, 2] % 4 < 2)
    q[sub0 & (coords[:, 2] // 4 == 0), 0] = c
    k[sub0 & (coords[:, 2] // 4 == 2), 0] = 1.0
    ec = math.exp(c)
    want = np.array([7 / 3 + 8 / (ec + 23), 7 / 3 + 8 / (ec + 23), 7 / 3 + (ec + 7) / (ec + 23)]) / 8
    r = O.coarse_head_subblock(q, k, grid, "raster", 0.40, 1, 1.0)
    assert np.allclose(r["P"][0], want, rtol=1e-13, atol=0)
    plain = O.coarse_head(q, k, grid, "raster", 0.40, 1, 1.0)
    e = math.exp(c / 64)
    assert np.allclose(plain["P"][0], [1 / (e + 2), 1 / (e + 2), e / (e + 2)], rtol=1e-13, atol=0)
    # p = 0.40: sub-block scores keep tile 2 alone (0.416 >= 0.40); the pooled
    # means need a second tile (0.362 < 0.40; ties to the lower id)
    assert r["counts"][0] == 1 and list(r["idx"][0, :1]) == [2]
    assert plain["counts"][0] == 2 and list(plain["idx"][0, :2]) == [0, 2]


def test_selection_on_tile_logprob_matches_brute_force_subsets():
    rng = np.random.default_rng(5)
    nT, S, d = 7, 8, 6
    qs, ks = rng.normal(size=(nT, S, d)) * 3, rng.normal(size=(nT, S, d)) * 3
    logP = O.subblock_tile_logprob(qs, ks, 0.5)
    P = np.exp(logP)
    for p, kmin in ((0.5, 1), (0.8, 2), (0.95, 3)):
        counts, idx, _ = O.select_blocks(logP, p, kmin)
        for r in range(nT):
            best = None
            for size in range(1, nT + 1):
                for sub in itertools.combinations(range(nT), size):
                    if P[r, list(sub)].sum() >= p:
                        best = size
                        break
                if best:
                    break
            assert counts[r] == min(nT, max(best, kmin))
            assert P[r, idx[r, :counts[r]]].sum() >= p - 1e-12 or counts[r] == kmin
