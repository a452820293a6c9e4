"""Pins for the oracle's arithmetic: RoPE, bf16 rounding, pooling, softmax,
selection (brute force over subsets), the fine stage (independent O(N^2)
loops and torch SDPA), lse closed forms and a hand-derived worked example."""
import itertools
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest

from block_sparse_spatiotemporal_b200.inputs import bf16_bits_to_f32, f32_to_bf16_bits
from oracle import fvattn_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------- RoPE ----

def _rand(shape, seed=0):
    return np.random.default_rng(seed).standard_normal(shape)


def test_rope_preserves_pair_norms_and_identity_at_origin():
    x = _rand((50, 128))
    coords = np.random.default_rng(1).integers(0, 80, (50, 3))
    y = O.rope_3d(x, coords)
    assert np.allclose(np.hypot(y[:, 0::2], y[:, 1::2]), np.hypot(x[:, 0::2], x[:, 1::2]),
                       rtol=0, atol=1e-12)
    assert np.allclose(O.rope_3d(x, np.zeros_like(coords)), x, rtol=0, atol=0)


def test_rope_dot_depends_only_on_relative_position():
    """(R_m q).(R_n k) = (R_{m+s} q).(R_{n+s} k) for any shift s per axis."""
    q, k = _rand((1, 128), 2), _rand((1, 128), 3)
    rng = np.random.default_rng(4)
    for _ in range(20):
        m = rng.integers(0, 60, (1, 3))
        n = rng.integers(0, 60, (1, 3))
        s = rng.integers(-20, 20, (1, 3))
        a = O.rope_3d(q, m) @ O.rope_3d(k, n).T
        b = O.rope_3d(q, m + s) @ O.rope_3d(k, n + s).T
        assert abs(a - b).max() < 1e-9


def test_rope_axis_groups_are_independent():
    """Moving only the t coordinate leaves the h and w groups untouched."""
    x = _rand((4, 128), 5)
    c0 = np.array([[0, 3, 7]] * 4)
    c1 = np.array([[9, 3, 7]] * 4)
    a, b = O.rope_3d(x, c0), O.rope_3d(x, c1)
    assert np.array_equal(a[:, 44:], b[:, 44:])
    assert not np.allclose(a[:, :44], b[:, :44])


def test_rope_first_pair_turns_one_radian_per_step():
    """Pair 0 of every axis group has frequency base^0 = 1."""
    x = np.zeros((1, 128))
    x[0, 0] = 1.0
    x[0, 44] = 1.0
    x[0, 86] = 1.0
    y = O.rope_3d(x, np.array([[1, 2, 3]]))
    for off, pos in ((0, 1), (44, 2), (86, 3)):
        assert math.isclose(math.atan2(y[0, off + 1], y[0, off]), math.remainder(pos, 2 * math.pi),
                            abs_tol=1e-12)


# ------------------------------------------------------------ bf16 ----

def test_round_bf16_matches_bit_rounding_and_torch():
    import torch
    rng = np.random.default_rng(6)
    x = (rng.standard_normal(200000) * np.exp(rng.uniform(-20, 20, 200000))).astype(np.float32)
    # exact halfway cases
    x[:1000] = bf16_bits_to_f32(f32_to_bf16_bits(x[:1000])) + np.float32(0.0)
    u = x[1000:3000].view(np.uint32) & np.uint32(0xFFFF0000) | np.uint32(0x8000)
    x[1000:3000] = u.view(np.float32)
    ref_bits = bf16_bits_to_f32(f32_to_bf16_bits(x)).astype(np.float64)
    ref_torch = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    got = O.round_bf16(x.astype(np.float64))
    assert np.array_equal(got, ref_bits)
    assert np.array_equal(got, ref_torch)


# ------------------------------------------------------- pool/softmax ----

def test_pool_is_mean_of_64_rows_bruteforce():
    x = _rand((4 * 64, 5), 7)
    p = O.pool_tiles(x)
    for i in range(4):
        for c in range(5):
            assert math.isclose(p[i, c], math.fsum(x[i * 64 + r, c] for r in range(64)) / 64,
                                rel_tol=0, abs_tol=1e-14)


def test_coarse_softmax_rows_sum_to_one():
    qp, kp = _rand((40, 64), 8) * 5, _rand((40, 64), 9) * 5
    P = O.coarse_probabilities(qp, kp, 0.125)
    assert (P >= 0).all()
    assert np.abs(P.sum(axis=1) - 1).max() < 1e-12
    # invariant to a shared shift of the logits of a row: shift Kp along Qp
    assert np.allclose(P, O.coarse_probabilities(qp, kp, 0.125), atol=0)


def test_coarse_softmax_matches_exp_normalisation_small():
    qp, kp = _rand((3, 4), 10), _rand((5, 4), 11)
    P = O.coarse_probabilities(qp, kp, 0.5)
    for i in range(3):
        logits = [0.5 * sum(qp[i, c] * kp[j, c] for c in range(4)) for j in range(5)]
        z = math.fsum(math.exp(v) for v in logits)
        for j in range(5):
            assert math.isclose(P[i, j], math.exp(logits[j]) / z, rel_tol=1e-13)


# ------------------------------------------------------------ select ----

def _brute_force_count(prob, p, k_min):
    nT = len(prob)
    if p >= 1:
        return nT
    best = None
    for size in range(1, nT + 1):
        for sub in itertools.combinations(range(nT), size):
            if math.fsum(prob[j] for j in sub) >= p:
                best = size
                break
        if best is not None:
            break
    if best is None:
        best = nT
    return min(nT, max(best, k_min, 1))


@pytest.mark.parametrize("seed", range(6))
def test_select_matches_brute_force_over_subsets(seed):
    rng = np.random.default_rng(100 + seed)
    nT = 9
    P = rng.dirichlet(np.full(nT, 0.5), size=6)
    for p in (0.0, 0.3, 0.5, 0.8, 0.9, 0.95, 0.99, 1.0):
        for k_min in (0, 1, 2, 4, 12):
            counts, idx, border = O.select_blocks(np.log(P), p, k_min)
            for r in range(P.shape[0]):
                c = counts[r]
                assert c == _brute_force_count(P[r], p, k_min), (p, k_min, r)
                sel = idx[r, :c]
                assert (np.diff(sel) > 0).all() and (idx[r, c:] == -1).all()
                rest = np.setdiff1d(np.arange(nT), sel)
                # the selected set is the top-c set (ties to the lower index)
                for a in sel:
                    for b in rest:
                        assert P[r, a] > P[r, b] or (P[r, a] == P[r, b] and a < b)
                if p < 1 and c > max(k_min, 1):
                    assert P[r, sel].sum() >= p - 1e-12


def test_select_ties_go_to_lower_index_and_fixed_topk():
    P = np.array([[0.25, 0.25, 0.25, 0.25], [0.1, 0.4, 0.1, 0.4]])
    counts, idx, _ = O.select_blocks(np.log(P), 0.5, 1)
    assert counts.tolist() == [2, 2]
    assert idx[0, :2].tolist() == [0, 1] and idx[1, :2].tolist() == [1, 3]
    counts, idx, _ = O.select_blocks(np.log(P), 0.0, 3)
    assert counts.tolist() == [3, 3]
    assert idx[0, :3].tolist() == [0, 1, 2] and idx[1, :3].tolist() == [0, 1, 3]


def test_select_ranks_underflowing_tiles_by_logit():
    """Probabilities exp(-900) and exp(-800) are both 0.0 in float64, yet the
    tile with the larger logit is the more probable one and ranks first."""
    S = np.array([[0.0, -900.0, -800.0, -5.0]])
    P = O.row_softmax(S)
    assert P[0, 1] == 0.0 and P[0, 2] == 0.0
    counts, idx, _ = O.select_blocks(S, 0.0, 3)
    assert counts.tolist() == [3] and idx[0, :3].tolist() == [0, 2, 3]
    assert O.near_tie_rows(S, counts, np.array([1e-3])).tolist() == [False]
    S2 = np.array([[0.0, -900.0, -5.0 - 1e-7, -5.0]])
    c2, _, _ = O.select_blocks(S2, 0.0, 2)
    assert O.near_tie_rows(S2, c2, np.array([1e-6])).tolist() == [True]


def test_select_borderline_flag():
    P = np.array([[0.6, 0.3, 0.1], [0.5, 0.3 + 4e-6, 0.2 - 4e-6]])
    _, _, border = O.select_blocks(np.log(P), 0.8, 1)
    assert border.tolist() == [False, True]
    # with a k_min floor above both candidate counts the row is not borderline
    _, _, border = O.select_blocks(np.log(P), 0.8, 3)
    assert border.tolist() == [False, False]


# ------------------------------------------------------------ fine ----

def _constructed_case(fx):
    T, Hg, W = fx["grid"]
    d = fx["head_dim"]
    N = T * Hg * W
    probs = np.array(fx["probs"])
    pos = O.raster_cube_positions((T, Hg, W))
    q = np.zeros((N, d)); q[:, 0] = 2.0
    k = np.zeros((N, d)); v = np.zeros((N, d))
    tile_of = pos // 64
    k[:, 0] = np.log(probs[tile_of])
    v[np.arange(N), tile_of] = tile_of + 1.0
    return q, k, v, probs


def test_worked_example_selection_output_and_lse():
    with open(os.path.join(GOLDEN, "topp_constructed.json")) as f:
        fx = json.load(f)
    q, k, v, probs = _constructed_case(fx)
    for case in fx["cases"]:
        res = O.forward_head(q.astype(np.float32), k.astype(np.float64), v, tuple(fx["grid"]),
                             "raster", case["top_p"], case["k_min"], "f64")
        assert (res["counts"] == len(case["selected"])).all()
        for r in range(len(probs)):
            assert res["idx"][r, :res["counts"][r]].tolist() == case["selected"]
        want = np.array([float(Fraction(s)) for s in case["out"]])
        assert np.abs(res["out"] - want[None, :]).max() < 1e-12, case
        assert np.abs(res["lse"] - math.log(float(Fraction(case["lse_arg"])))).max() < 1e-12


def test_dense_p1_equals_independent_loop():
    grid = (4, 4, 8)          # 128 tokens, 2 tiles
    rng = np.random.default_rng(12)
    q, k, v = (rng.standard_normal((128, 8)) for _ in range(3))
    res = O.forward_head(q, k, v, grid, "raster", 1.0, 1, "f64")
    assert (res["counts"] == 2).all()
    out, lse = O.dense_attention_loop(q.tolist(), k.tolist(), v.tolist(), 1 / math.sqrt(8))
    assert np.abs(res["out"] - np.array(out)).max() < 1e-12
    assert np.abs(res["lse"] - np.array(lse)).max() < 1e-12


def test_dense_p1_matches_torch_sdpa():
    import torch
    grid = (8, 8, 8)
    rng = np.random.default_rng(13)
    q, k, v = (rng.standard_normal((512, 64)) * 2 for _ in range(3))
    for order in ("raster", "hilbert"):
        res = O.forward_head(q, k, v, grid, order, 1.0, 1, "f64")
        ref = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(q)[None], torch.from_numpy(k)[None], torch.from_numpy(v)[None])[0]
        assert np.abs(res["out"] - ref.numpy()).max() < 1e-12
        s = torch.from_numpy(q) @ torch.from_numpy(k).T / 8.0
        assert np.abs(res["lse"] - torch.logsumexp(s, dim=1).numpy()).max() < 1e-12


def test_zero_queries_give_mean_of_selected_values():
    grid = (4, 8, 8)           # 4 tiles
    rng = np.random.default_rng(14)
    q = np.zeros((256, 16)); k = rng.standard_normal((256, 16)); v = rng.standard_normal((256, 16))
    counts = np.array([1, 2, 4, 3])
    idx = np.array([[2, -1, -1, -1], [0, 3, -1, -1], [0, 1, 2, 3], [1, 2, 3, -1]])
    res = O.forward_head(q, k, v, grid, "raster", 0.5, 1, "f64", blocks=(counts, idx))
    vt = v  # raster order of this grid: tile j = rows of cube j
    pos = O.raster_cube_positions(grid)
    vt = O.to_tiled(v, pos)
    for i in range(4):
        rows = np.concatenate([np.arange(j * 64, j * 64 + 64) for j in idx[i, :counts[i]]])
        want = vt[rows].mean(axis=0)
        got = res["out_tiled"][i * 64:(i + 1) * 64]
        assert np.abs(got - want).max() < 1e-12
        assert np.abs(res["lse_tiled"][i * 64:(i + 1) * 64] - math.log(64 * counts[i])).max() < 1e-12


def test_order_invariance_raster_vs_hilbert():
    """Same tile contents in both orders: dense outputs agree, and the sparse
    selections agree as sets of cubes."""
    grid = (8, 8, 16)
    rng = np.random.default_rng(15)
    q, k, v = (rng.standard_normal((1024, 32)) for _ in range(3))
    a = O.forward_head(q, k, v, grid, "raster", 1.0, 1, "f64")
    b = O.forward_head(q, k, v, grid, "hilbert", 1.0, 1, "f64")
    assert np.abs(a["out"] - b["out"]).max() < 1e-12
    a = O.forward_head(q, k, v, grid, "raster", 0.7, 2, "f64")
    b = O.forward_head(q, k, v, grid, "hilbert", 0.7, 2, "f64")
    ca = O.tile_cubes(grid, a["pos"])
    cb = O.tile_cubes(grid, b["pos"])
    sets_a = {tuple(ca[i]): {tuple(ca[j]) for j in a["idx"][i, :a["counts"][i]]} for i in range(len(ca))}
    sets_b = {tuple(cb[i]): {tuple(cb[j]) for j in b["idx"][i, :b["counts"][i]]} for i in range(len(cb))}
    assert sets_a == sets_b
    assert np.abs(a["out"] - b["out"]).max() < 1e-12


def test_rope_bf16_operand_rounding_only_in_fine_stage():
    """With RoPE on a bf16 workload the pooled scores use unrounded rotated
    values; the fine stage sees them rounded to bf16."""
    grid = (4, 4, 8)
    rng = np.random.default_rng(16)
    q32 = rng.standard_normal((128, 128)).astype(np.float32)
    k32 = rng.standard_normal((128, 128)).astype(np.float32)
    v32 = rng.standard_normal((128, 128)).astype(np.float32)
    q, k, v = f32_to_bf16_bits(q32), f32_to_bf16_bits(k32), f32_to_bf16_bits(v32)
    rope = dict(dims=(44, 42, 42), base=10000.0)
    res = O.forward_head(q, k, v, grid, "raster", 1.0, 1, "bf16", rope=rope)
    coords = O.token_coords(grid)
    qr = O.rope_3d(O.as_f64(q, "bf16"), coords)
    kr = O.rope_3d(O.as_f64(k, "bf16"), coords)
    assert np.abs(res["qp"] - O.pool_tiles(O.to_tiled(qr, res["pos"]))).max() == 0
    qr32 = O.rope_3d_f32(O.as_f64(q, "bf16"), coords).astype(np.float64)
    kr32 = O.rope_3d_f32(O.as_f64(k, "bf16"), coords).astype(np.float64)
    out, lse = O.dense_attention_loop(O.round_bf16(qr32).tolist(), O.round_bf16(kr32).tolist(),
                                      O.as_f64(v, "bf16").tolist(), 1 / math.sqrt(128))
    assert np.abs(res["out"] - np.array(out)).max() < 1e-12


def test_rope_f32_rotation_is_the_float32_evaluation_of_the_rotation():
    """rope_3d_f32 (the fine stage's operand rotation) against the float64
    rotation: identical at position 0 (cos 1, sin 0 exactly), within two
    float32 rounding errors of the float64 value elsewhere, pair norms kept
    to float32 precision, and equal to a scalar loop that rounds every
    intermediate through struct's IEEE single format."""
    import struct
    rng = np.random.default_rng(21)
    x = rng.standard_normal((6, 128)).astype(np.float32).astype(np.float64)
    coords = np.array([[0, 0, 0], [1, 2, 3], [19, 47, 79], [5, 0, 9], [0, 11, 0], [7, 7, 7]])
    y = O.rope_3d_f32(x, coords)
    assert y.dtype == np.float32
    assert np.array_equal(y[0], x[0].astype(np.float32))
    ref = O.rope_3d(x, coords)
    mag = np.abs(x[:, 0::2]) + np.abs(x[:, 1::2])
    err = np.maximum(np.abs(y[:, 0::2] - ref[:, 0::2]), np.abs(y[:, 1::2] - ref[:, 1::2]))
    assert (err <= 2 * 2.0 ** -23 * mag + 1e-30).all()
    n0, n1 = x[:, 0::2] ** 2 + x[:, 1::2] ** 2, y[:, 0::2].astype(np.float64) ** 2 + y[:, 1::2].astype(np.float64) ** 2
    assert np.abs(n1 - n0).max() <= 1e-5 * n0.max()
    f = lambda v: struct.unpack("f", struct.pack("f", v))[0]   # noqa: E731
    r, dim = 2, 50                                             # token 2, h-axis pair j = 3
    da, j = 42, 3
    ang = coords[r, 1] * 10000.0 ** (-2.0 * j / da)
    c, s = f(math.cos(ang)), f(math.sin(ang))
    x0, x1 = f(x[r, dim]), f(x[r, dim + 1])
    assert y[r, dim] == f(f(x0 * c) - f(x1 * s))
    assert y[r, dim + 1] == f(f(x0 * s) + f(x1 * c))


def test_rope_each_axis_group_matches_library_1d_rotary():
    """Restricted to one axis, each group is the standard 1D rotary encoding
    with adjacent pairs; pinned against the GPT-J rotary routine shipped in
    transformers (float32, hence the 1e-4 bound)."""
    import torch
    from transformers.models.gptj import modeling_gptj as gptj
    rng = np.random.default_rng(17)
    x = rng.standard_normal((60, 128))
    for axis, (off, da) in enumerate(((0, 44), (44, 42), (86, 42))):
        coords = np.zeros((60, 3), np.int64)
        coords[:, axis] = np.arange(60)
        ours = O.rope_3d(x, coords)[:, off:off + da]
        table = gptj.create_sinusoidal_positions(60, da)
        sin, cos = torch.split(table, da // 2, dim=-1)
        t = torch.from_numpy(x[:, off:off + da]).float()[None, :, None, :]
        ref = gptj.apply_rotary_pos_emb(t, sin[None], cos[None])[0, :, 0, :].double().numpy()
        assert np.abs(ours - ref).max() < 1e-4, axis
