"""Pins for the oracle's token orders (raster-cube and 3D Hilbert).

Raster-cube: hand-derived positions (golden fixture) and the bijection.
Hilbert: bijection, unit steps between consecutive indices on 2^k cubes, every
aligned 2^j sub-cube visited contiguously (the recursive property that makes
a Hilbert curve, and that a boustrophedon or Morton order breaks), and each
run of 64 valid tokens being one aligned 4x4x4 cube on the workloads' grids.
"""
import json
import os

import numpy as np
import pytest

from oracle import fvattn_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_raster_cube_golden_positions():
    with open(os.path.join(GOLDEN, "raster_cube_positions.json")) as f:
        fx = json.load(f)
    for case in fx["cases"]:
        T, Hg, W = case["grid"]
        t, h, w = case["thw"]
        pos = O.raster_cube_positions((T, Hg, W))
        assert pos[(t * Hg + h) * W + w] == case["position"], case


@pytest.mark.parametrize("grid", [(4, 4, 4), (8, 16, 16), (20, 32, 52), (4, 8, 12)])
def test_raster_cube_bijection_and_cubes(grid):
    pos = O.raster_cube_positions(grid)
    assert np.array_equal(np.sort(pos), np.arange(pos.size))
    cubes = O.tile_cubes(grid, pos)
    # raster order over the tile grid
    nh, nw = grid[1] // 4, grid[2] // 4
    rank = (cubes[:, 0] * nh + cubes[:, 1]) * nw + cubes[:, 2]
    assert np.array_equal(rank, np.arange(len(cubes)))


def test_partial_tiles_rejected():
    with pytest.raises(ValueError):
        O.raster_cube_positions((4, 4, 6))
    with pytest.raises(ValueError):
        O.hilbert_positions((6, 4, 4))


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_hilbert_bijection_and_unit_steps(bits):
    n = 1 << bits
    c = O.token_coords((n, n, n))
    key = O.hilbert_index_3d(c, bits)
    assert np.array_equal(np.sort(key), np.arange(n ** 3))
    path = c[np.argsort(key)]
    steps = np.abs(np.diff(path, axis=0)).sum(axis=1)
    assert (steps == 1).all()
    assert (path[0] == 0).all()


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_hilbert_visits_aligned_subcubes_contiguously(bits):
    n = 1 << bits
    c = O.token_coords((n, n, n))
    path = c[np.argsort(O.hilbert_index_3d(c, bits))]
    for j in range(1, bits):
        side = 1 << j
        cube_id = path // side
        runs = cube_id.reshape(-1, side ** 3, 3)
        assert (runs == runs[:, :1, :]).all(), f"level {j}"


def test_morton_order_fails_the_pins():
    """Control: a Z-order curve is a bijection that visits aligned sub-cubes
    contiguously but does not take unit steps, so the step pin discriminates."""
    bits, n = 3, 8
    c = O.token_coords((n, n, n))
    morton = np.zeros(len(c), np.int64)
    for b in range(bits - 1, -1, -1):
        for a in range(3):
            morton = (morton << 1) | ((c[:, a] >> b) & 1)
    path = c[np.argsort(morton)]
    assert (np.abs(np.diff(path, axis=0)).sum(axis=1) > 1).any()


@pytest.mark.parametrize("grid", [(8, 16, 16), (20, 32, 52), (20, 48, 80), (12, 8, 20)])
def test_hilbert_tiles_are_aligned_cubes(grid):
    pos = O.hilbert_positions(grid)
    assert np.array_equal(np.sort(pos), np.arange(pos.size))
    cubes = O.tile_cubes(grid, pos)          # raises if a run is not a cube
    nT = pos.size // 64
    assert len({tuple(x) for x in cubes}) == nT


def test_hilbert_tile_path_mostly_adjacent():
    """On a 2^k grid consecutive tiles are face neighbours; on the 720p grid
    most are (the skipped part of the enclosing cube breaks a few steps)."""
    pos = O.hilbert_positions((16, 16, 16))
    cubes = O.tile_cubes((16, 16, 16), pos)
    assert (np.abs(np.diff(cubes, axis=0)).sum(axis=1) == 1).all()
    pos = O.hilbert_positions((20, 48, 80))
    cubes = O.tile_cubes((20, 48, 80), pos)
    steps = np.abs(np.diff(cubes, axis=0)).sum(axis=1)
    assert (steps == 1).mean() > 0.9


def test_tiled_roundtrip():
    rng = np.random.default_rng(0)
    x = rng.standard_normal((2, 8 * 8 * 8, 3))
    for order in ("raster", "hilbert"):
        pos = O.positions((8, 8, 8), order)
        assert np.array_equal(O.from_tiled(O.to_tiled(x, pos), pos), x)
