"""GPU parity of each kernel against the oracle on small seeded inputs that
span several tiles and a ragged tail, plus the edge cases of the method.

Bars: bit-exact for the reorder, block lists and work list (borderline rows
exempt and counted); bf16 outputs within 2e-2 max-abs and 2e-3 mean-abs;
fp32 within 1e-4."""
import numpy as np
import pytest
import torch

from block_sparse_spatiotemporal_b200 import fvattn as F
from block_sparse_spatiotemporal_b200.inputs import f32_to_bf16_bits, Workload, WORKLOADS, make_inputs
from oracle import fvattn_oracle as O
from tests.gpu_util import (assert_close, compare_blocks, sum_checks, oracle_coarse, oracle_rope, rope_of, shape_of,
                            to_dev, to_host)

pytestmark = pytest.mark.gpu


def small(grid, heads=2, d=128, dtype="bf16", order="raster", rope=False, gen="per_head", seed=7,
          top_p=0.9, k_min=2):
    return Workload(f"small{grid}", grid, heads, d, dtype, seed, top_p, k_min, order, rope, gen)


def _blocks_host(counts, idx):
    return counts.cpu().numpy(), idx.cpu().numpy()


def test_wait_cap_reports_status_instead_of_hanging():
    ws = torch.zeros(1 << 12, dtype=torch.uint8, device="cuda")
    F.selftest_wait_timeout(ws, 1000)
    assert F.device_status(ws) == 2
    assert F.device_status(ws) == 0      # reading clears it


@pytest.mark.parametrize("order", ["raster", "hilbert"])
@pytest.mark.parametrize("grid", [(4, 4, 12), (8, 16, 16), (12, 8, 20)])
def test_tile_reorder_is_the_oracle_permutation(order, grid):
    wl = small(grid, heads=3, order=order)
    shape = shape_of(wl)
    ws = F.workspace(shape)
    N = wl.tokens
    x = torch.arange(3 * N * 128, dtype=torch.int32, device="cuda").view(1, 3, N, 128).to(torch.int16)
    x = x.view(torch.bfloat16)
    y = F.tile_reorder(shape, x, ws)
    pos = O.positions(grid, order)
    xh = x.view(torch.int16).cpu().numpy()
    want = O.to_tiled(xh, pos)
    assert np.array_equal(y.view(torch.int16).cpu().numpy(), want)
    back = F.tile_reorder(shape, y, ws, inverse=True)
    assert torch.equal(back.view(torch.int16), x.view(torch.int16))
    # 4-byte rows (lse layout)
    l = torch.randn(1, 3, N, device="cuda")
    lt = F.tile_reorder(shape, l, ws)
    assert np.array_equal(lt.cpu().numpy(), O.to_tiled(l.cpu().numpy()[..., None], pos)[..., 0])


def _pool_select_case(wl, layout=F.NATURAL, top_p=None, k_min=None):
    top_p = wl.top_p if top_p is None else top_p
    k_min = wl.k_min if k_min is None else k_min
    q, k, v = make_inputs(wl)
    shape = shape_of(wl, layout)
    rope = rope_of(wl)
    ws = F.workspace(shape, rope)
    qd, kd = to_dev(q, wl.dtype), to_dev(k, wl.dtype)
    if layout == F.TILED:
        qd, kd = F.tile_reorder(shape, qd, ws), F.tile_reorder(shape, kd, ws)
    counts, idx = F.pool_select(shape, qd, kd, ws, top_p, k_min, rope=rope)
    assert F.device_status(ws) == 0
    gc, gi = _blocks_host(counts, idx)
    res = oracle_coarse(wl, q, k, top_p, k_min)
    tot = sum_checks([compare_blocks(r, gc[0, h], gi[0, h], top_p, k_min) for h, r in enumerate(res)])
    assert tot["mismatch"] == 0, tot
    return q, k, v, res, gc, gi


@pytest.mark.parametrize("case", [
    dict(grid=(8, 16, 16), dtype="f32", d=64, gen="fixed"),
    dict(grid=(8, 16, 16), dtype="bf16", d=128),
    dict(grid=(4, 8, 12), dtype="bf16", d=128, top_p=0.5, k_min=1),
    dict(grid=(8, 8, 16), dtype="bf16", d=128, order="hilbert", rope=True),
    dict(grid=(8, 8, 12), dtype="f32", d=128, order="hilbert", rope=True),
])
@pytest.mark.parametrize("layout", [F.NATURAL, F.TILED])
def test_pool_select_lists_bit_exact(case, layout):
    wl = small(case["grid"], d=case["d"], dtype=case["dtype"], order=case.get("order", "raster"),
               rope=case.get("rope", False), gen=case.get("gen", "per_head"), top_p=case.get("top_p", 0.9),
               k_min=case.get("k_min", 2))
    _pool_select_case(wl, layout)


@pytest.mark.parametrize("top_p,k_min", [(1.0, 1), (0.0, 3), (0.0, 1), (0.5, 100), (0.99, 0), (0.3, 2)])
def test_pool_select_special_cases(top_p, k_min):
    wl = small((4, 8, 16), heads=3)
    _, _, _, res, gc, gi = _pool_select_case(wl, top_p=top_p, k_min=k_min)
    nT = wl.num_tiles
    if top_p >= 1.0:
        assert (gc == nT).all()
    if top_p <= 0.0:
        assert (gc == min(max(k_min, 1), nT)).all()
    assert (gc >= min(max(k_min, 1), nT)).all()


def _fine_case(wl, layout, top_p=None, k_min=None):
    """Fine stage fed the oracle's own lists; every output row compared."""
    top_p = wl.top_p if top_p is None else top_p
    k_min = wl.k_min if k_min is None else k_min
    q, k, v = make_inputs(wl)
    shape = shape_of(wl, layout)
    rope = rope_of(wl)
    ws = F.workspace(shape, rope)
    nT = wl.num_tiles
    pos = O.positions(wl.grid, wl.order)
    counts = np.zeros((1, wl.heads, nT), np.int32)
    idx = np.full((1, wl.heads, nT, nT), -1, np.int32)
    want_out = np.zeros((wl.heads, wl.tokens, wl.head_dim))
    want_lse = np.zeros((wl.heads, wl.tokens))
    for h in range(wl.heads):
        r = O.forward_head(q[0, h], k[0, h], v[0, h], wl.grid, wl.order, top_p, k_min, wl.dtype,
                           rope=oracle_rope(wl))
        counts[0, h] = r["counts"]
        idx[0, h] = r["idx"]
        if layout == F.TILED:
            want_out[h], want_lse[h] = r["out_tiled"], r["lse_tiled"]
        else:
            want_out[h], want_lse[h] = r["out"], r["lse"]
    qd, kd, vd = (to_dev(x, wl.dtype) for x in (q, k, v))
    if layout == F.TILED:
        qd, kd, vd = (F.tile_reorder(shape, x, ws) for x in (qd, kd, vd))
    cd, idd = torch.from_numpy(counts).cuda(), torch.from_numpy(idx).cuda()
    out, lse = F.block_sparse_fwd(shape, qd, kd, vd, cd, idd, ws, rope=rope)
    assert F.device_status(ws) == 0
    assert_close(to_host(out)[0], want_out, wl.dtype, "out")
    assert_close(to_host(lse)[0], want_lse, wl.dtype, "lse")


@pytest.mark.parametrize("case", [
    dict(grid=(8, 16, 16), dtype="f32", d=64, gen="fixed", top_p=0.9, k_min=2),
    dict(grid=(4, 8, 8), dtype="bf16", d=128, top_p=1.0, k_min=1),                 # dense, two items
    dict(grid=(4, 4, 12), dtype="bf16", d=128, top_p=1.0, k_min=1),                # odd nT: single-tile item
    dict(grid=(8, 16, 16), dtype="bf16", d=128, top_p=0.9, k_min=2),
    dict(grid=(8, 16, 16), dtype="bf16", d=128, top_p=0.0, k_min=5),               # fixed top-k
    dict(grid=(8, 8, 12), dtype="bf16", d=128, order="hilbert", rope=True, top_p=0.9, k_min=3),
    dict(grid=(8, 8, 12), dtype="f32", d=128, order="hilbert", rope=True, top_p=0.9, k_min=3),
    dict(grid=(4, 4, 20), dtype="bf16", d=128, top_p=0.9, k_min=2),                # nT = 5: a one-tile quad
    dict(grid=(4, 8, 12), dtype="bf16", d=128, top_p=0.5, k_min=1),                # nT = 6: a two-tile quad
    dict(grid=(4, 4, 28), dtype="bf16", d=128, top_p=0.7, k_min=1),                # nT = 7: a three-tile quad
])
@pytest.mark.parametrize("layout", [F.NATURAL, F.TILED])
def test_block_sparse_fwd_matches_oracle(case, layout):
    wl = small(case["grid"], d=case["d"], dtype=case["dtype"], order=case.get("order", "raster"),
               rope=case.get("rope", False), gen=case.get("gen", "per_head"))
    _fine_case(wl, layout, case["top_p"], case["k_min"])


def test_late_large_logits_rescale():
    """Keys of the last tile scaled by 2^4 (exact in bf16): with dense lists
    every row meets logits far above its first tile's only at the last step,
    so the running max moves up there (O, l and the step's P rescaled)."""
    wl = small((4, 8, 16), heads=2)                 # nT = 8
    q, k, v = make_inputs(wl)
    k = k.copy()
    pos = O.positions(wl.grid, wl.order)
    last = pos // 64 == wl.num_tiles - 1
    big = O.as_f64(k[:, :, last], "bf16") * 16.0
    k[:, :, last] = f32_to_bf16_bits(big.astype(np.float32))
    shape = shape_of(wl)
    ws = F.workspace(shape)
    nT = wl.num_tiles
    counts = torch.full((1, wl.heads, nT), nT, dtype=torch.int32, device="cuda")
    idx = torch.arange(nT, dtype=torch.int32, device="cuda").repeat(1, wl.heads, nT, 1)
    out, lse = F.block_sparse_fwd(shape, to_dev(q, "bf16"), to_dev(k, "bf16"), to_dev(v, "bf16"), counts, idx, ws)
    assert F.device_status(ws) == 0
    full = (np.full(nT, nT), np.tile(np.arange(nT), (nT, 1)))
    for h in range(wl.heads):
        r = O.forward_head(q[0, h], k[0, h], v[0, h], wl.grid, wl.order, 1.0, 1, "bf16", blocks=full)
        s = O.default_scale(wl.head_dim) * np.abs(O.as_f64(q[0, h], "bf16") @ O.as_f64(k[0, h], "bf16").T)
        assert s.max() * 1.4427 > 64          # the jump exceeds the kernel's headroom somewhere
        assert_close(to_host(out)[0, h], r["out"], "bf16", f"out head {h}")
        assert_close(to_host(lse)[0, h], r["lse"], "bf16", f"lse head {h}")


def test_single_tile_grid():
    wl = small((4, 4, 4), heads=2, gen="fixed")     # one tile: no room for two sink tiles
    _fine_case(wl, F.NATURAL, 0.9, 1)


def test_empty_rows_and_bad_block_ids():
    """A row with count 0 gives out = 0 and lse = -inf; an out-of-range id is
    reported through the status word and never read."""
    wl = small((4, 8, 8), heads=1)
    q, k, v = make_inputs(wl)
    shape = shape_of(wl)
    ws = F.workspace(shape)
    nT = wl.num_tiles
    counts = torch.tensor([[[0, 2, 1, 4]]], dtype=torch.int32, device="cuda")
    idx = torch.full((1, 1, nT, nT), -1, dtype=torch.int32, device="cuda")
    idx[0, 0, 1, :2] = torch.tensor([0, 3])
    idx[0, 0, 2, 0] = 2
    idx[0, 0, 3, :] = torch.arange(4)
    out, lse = F.block_sparse_fwd(shape, to_dev(q, "bf16"), to_dev(k, "bf16"), to_dev(v, "bf16"), counts, idx, ws)
    assert F.device_status(ws) == 0
    pos = O.positions(wl.grid, wl.order)
    tile_of = pos // 64
    o, l = to_host(out)[0, 0], to_host(lse)[0, 0]
    assert (o[tile_of == 0] == 0).all() and np.isneginf(l[tile_of == 0]).all()
    r = O.forward_head(q[0, 0], k[0, 0], v[0, 0], wl.grid, "raster", 0.9, 1, "bf16",
                       blocks=(np.array([1, 2, 1, 4]), np.array([[0, -1, -1, -1], [0, 3, -1, -1],
                                                                 [2, -1, -1, -1], [0, 1, 2, 3]])))
    rows = tile_of != 0
    assert_close(o[rows], r["out"][rows], "bf16", "out")
    bad = idx.clone()
    bad[0, 0, 2, 0] = 77
    F.block_sparse_fwd(shape, to_dev(q, "bf16"), to_dev(k, "bf16"), to_dev(v, "bf16"), counts, bad, ws)
    assert F.device_status(ws) == 1
    unsorted = idx.clone()
    unsorted[0, 0, 1, :2] = torch.tensor([3, 0])
    F.block_sparse_fwd(shape, to_dev(q, "bf16"), to_dev(k, "bf16"), to_dev(v, "bf16"), counts, unsorted, ws)
    assert F.device_status(ws) == 1


def test_worklist_is_longest_union_first():
    wl = small((8, 8, 20), heads=4)         # nT = 20 tiles: 10 items per head
    _worklist_case(wl)
    _worklist_case(small((4, 4, 12), heads=3))   # nT = 3: the last item has one tile


def _worklist_case(wl):
    q, k, v, res, gc, gi = _pool_select_case(wl)
    shape = shape_of(wl)
    ws = F.workspace(shape)
    nT = wl.num_tiles
    oc = np.stack([r["counts"] for r in res])[None].astype(np.int32)
    oi = np.stack([r["idx"] for r in res])[None].astype(np.int32)
    cd, idd = torch.from_numpy(oc).cuda(), torch.from_numpy(oi).cuda()
    got = F.build_worklist(shape, cd, idd, ws).cpu().numpy()
    P = (nT + 1) // 2
    cost = []
    for h, r in enumerate(res):
        for p in range(P):
            u = set()
            for t in range(2 * p, min(2 * p + 2, nT)):
                u |= set(r["idx"][t, :r["counts"][t]].tolist())
            cost.append(len(u))
    cost = np.array(cost)
    want = np.lexsort((np.arange(len(cost)), -cost))
    assert np.array_equal(got, want)


def test_forward_cache_reuse_and_mismatch():
    wl = small((8, 8, 16), heads=2)
    q, k, v = make_inputs(wl)
    shape = shape_of(wl)
    ws = F.workspace(shape)
    cache, cc, ci = F.new_cache(shape)
    qd, kd, vd = (to_dev(x, "bf16") for x in (q, k, v))
    with pytest.raises(F.FvattnError):
        F.forward(shape, qd, kd, vd, ws, 0.9, 2, cache=cache, reuse_mask=True)
    out0, _ = F.forward(shape, qd, kd, vd, ws, 0.9, 2, cache=cache)
    assert cache.valid == 1
    # reuse with different q/k: output uses the cached lists
    q2, k2 = q[:, ::-1].copy(), k[:, ::-1].copy()
    out1, lse1 = F.forward(shape, to_dev(q2, "bf16"), to_dev(k2, "bf16"), vd, ws, 0.5, 1, cache=cache,
                           reuse_mask=True)
    assert F.device_status(ws) == 0
    for h in range(wl.heads):
        step0 = O.forward_head(q[0, h], k[0, h], v[0, h], wl.grid, "raster", 0.9, 2, "bf16")
        r = O.forward_head(q2[0, h], k2[0, h], v[0, h], wl.grid, "raster", 0.5, 1, "bf16",
                           blocks=(step0["counts"], step0["idx"]))
        assert_close(to_host(out1)[0, h], r["out"], "bf16", "out")
        assert_close(to_host(lse1)[0, h], r["lse"], "bf16", "lse")
    other = F.make_shape(1, 2, 128, (8, 8, 20))
    ws2 = F.workspace(other)
    z = torch.zeros(1, 2, 8 * 8 * 20, 128, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(F.FvattnError) as e:
        F.forward(other, z, z, z, ws2, 0.9, 2, cache=cache, reuse_mask=True)
    assert e.value.status == -6


def test_forward_equals_tiled_path():
    """forward on natural tensors == reorder + pool_select + block_sparse_fwd
    in tiled layout + inverse reorder (same kernels, other data path)."""
    wl = small((8, 8, 16), heads=2, order="hilbert")
    q, k, v = make_inputs(wl)
    shape_n, shape_t = shape_of(wl, F.NATURAL), shape_of(wl, F.TILED)
    ws = F.workspace(shape_n)
    qd, kd, vd = (to_dev(x, "bf16") for x in (q, k, v))
    out_n, lse_n = F.forward(shape_n, qd, kd, vd, ws, 0.9, 2)
    qt, kt, vt = (F.tile_reorder(shape_t, x, ws) for x in (qd, kd, vd))
    c, i = F.pool_select(shape_t, qt, kt, ws, 0.9, 2)
    out_t, lse_t = F.block_sparse_fwd(shape_t, qt, kt, vt, c, i, ws)
    back = F.tile_reorder(shape_t, out_t, ws, inverse=True)
    assert_close(to_host(back), to_host(out_n), "bf16", "out")
    lse_back = F.tile_reorder(shape_t, lse_t.contiguous(), ws, inverse=True)
    assert_close(to_host(lse_back), to_host(lse_n), "bf16", "lse")
