"""GPU parity of hierarchical sub-block scoring ("DFSAttn" digest, section 2)
through the C ABI: block lists of fvattn_pool_select_subblock against the
oracle's, and the fine stage on those lists against the oracle's forward."""
import numpy as np
import pytest

from block_sparse_spatiotemporal_b200 import fvattn as F
from block_sparse_spatiotemporal_b200.inputs import Workload, WORKLOADS, make_inputs
from oracle import fvattn_oracle as O
from tests.gpu_util import assert_close, compare_blocks, sum_checks, oracle_rope, rope_of, shape_of, to_dev, to_host

pytestmark = pytest.mark.gpu


def small(grid, heads=2, d=128, dtype="bf16", order="raster", rope=False, gen="per_head", seed=11,
          top_p=0.9, k_min=2):
    return Workload(f"small{grid}", grid, heads, d, dtype, seed, top_p, k_min, order, rope, gen)


def oracle_sub(wl, q, k, top_p, k_min, heads=None):
    """Oracle sub-block coarse stage per head, repackaged for compare_blocks:
    the ranking key is the tile log-probability; the float32 tolerance scale is
    the row's largest scale * |Qs| . |Ks|."""
    pos = O.positions(wl.grid, wl.order)
    out = []
    for h in (range(wl.heads) if heads is None else heads):
        r = O.coarse_head_subblock(O.as_f64(q[0, h], wl.dtype), O.as_f64(k[0, h], wl.dtype), wl.grid, wl.order,
                                   top_p, k_min, O.default_scale(wl.head_dim), oracle_rope(wl), pos)
        out.append(dict(S=r["logP"], counts=r["counts"], idx=r["idx"], border=r["border"],
                        s_abs=r["s_abs_row"][:, None], logP=r["logP"]))
    return out


def run_sub(wl, top_p, k_min, layout=F.NATURAL, heads=None):
    q, k, v = make_inputs(wl)
    shape = shape_of(wl, layout)
    rope = rope_of(wl)
    ws = F.workspace(shape, rope, subblock=True)
    qd, kd = to_dev(q, wl.dtype), to_dev(k, wl.dtype)
    if layout == F.TILED:
        qd, kd = F.tile_reorder(shape, qd, ws), F.tile_reorder(shape, kd, ws)
    counts, idx = F.pool_select_subblock(shape, qd, kd, ws, top_p, k_min, rope=rope)
    assert F.device_status(ws) == 0
    gc, gi = counts.cpu().numpy(), idx.cpu().numpy()
    res = oracle_sub(wl, q, k, top_p, k_min, heads)
    tot = sum_checks([compare_blocks(res[n], gc[0, h], gi[0, h], top_p, k_min)
                      for n, h in enumerate(range(wl.heads) if heads is None else heads)])
    mism, border, ties = tot["mismatch"], tot["borderline"], tot["near_tie"]
    return dict(q=q, k=k, v=v, shape=shape, rope=rope, ws=ws, counts=counts, idx=idx, gc=gc, gi=gi, res=res,
                mism=mism, border=border, ties=ties)


@pytest.mark.parametrize("case", [
    dict(grid=(8, 16, 16), dtype="f32", d=64, gen="fixed"),
    dict(grid=(8, 16, 16), dtype="bf16", d=128),
    dict(grid=(4, 4, 12), dtype="bf16", d=128, top_p=0.5, k_min=1),              # nT = 3
    dict(grid=(8, 16, 24), dtype="bf16", d=128, order="hilbert", rope=True),
    dict(grid=(12, 8, 20), dtype="bf16", d=128, order="hilbert", top_p=0.95, k_min=4),
])
@pytest.mark.parametrize("layout", [F.NATURAL, F.TILED])
def test_subblock_lists_bit_exact(case, layout):
    wl = small(case["grid"], d=case["d"], dtype=case["dtype"], order=case.get("order", "raster"),
               rope=case.get("rope", False), gen=case.get("gen", "per_head"), top_p=case.get("top_p", 0.9),
               k_min=case.get("k_min", 2))
    r = run_sub(wl, wl.top_p, wl.k_min, layout)
    assert r["mism"] == 0, f"{r['mism']} rows differ (border {r['border']}, near ties {r['ties']})"


@pytest.mark.parametrize("top_p,k_min", [(1.0, 1), (0.0, 3), (0.5, 100), (0.99, 0)])
def test_subblock_special_cases(top_p, k_min):
    wl = small((4, 8, 16), heads=3)
    r = run_sub(wl, top_p, k_min)
    assert r["mism"] == 0
    nT = wl.num_tiles
    if top_p >= 1.0:
        assert (r["gc"] == nT).all()
    if top_p <= 0.0:
        assert (r["gc"] == min(max(k_min, 1), nT)).all()
    assert (r["gc"] >= min(max(k_min, 1), nT)).all()


def test_subblock_lists_480p_eight_heads():
    wl = WORKLOADS["wan480p"]
    heads = [0, 5, 11, 17, 23, 29, 35, 39]
    r = run_sub(wl, wl.top_p, wl.k_min, heads=heads)
    print(f"480p sub-block: border rows {r['border']}, near-tie rows {r['ties']}")
    assert r["mism"] == 0


def test_subblock_lists_then_fine_stage_match_the_oracle_forward():
    """The whole sub-block path through the C ABI (pool_select_subblock then
    block_sparse_fwd) against the oracle's own sub-block lists and forward.
    On this case every GPU row equals the oracle's, so the comparison is of
    the same computation; the oracle never sees a GPU result."""
    wl = small((8, 16, 16), heads=2)
    r = run_sub(wl, wl.top_p, wl.k_min)
    assert r["mism"] == 0
    shape, q, k, v = r["shape"], r["q"], r["k"], r["v"]
    for h in range(wl.heads):
        res = r["res"][h]
        for row in range(wl.num_tiles):
            c = res["counts"][row]
            assert r["gc"][0, h, row] == c and np.array_equal(r["gi"][0, h, row, :c], res["idx"][row, :c])
    out, lse = F.block_sparse_fwd(shape, to_dev(q, "bf16"), to_dev(k, "bf16"), to_dev(v, "bf16"),
                                  r["counts"], r["idx"], r["ws"])
    assert F.device_status(r["ws"]) == 0
    go, gl = to_host(out), to_host(lse)
    for h in range(wl.heads):
        res = r["res"][h]
        want = O.forward_head(q[0, h], k[0, h], v[0, h], wl.grid, wl.order, wl.top_p, wl.k_min, "bf16",
                              blocks=(res["counts"], res["idx"]))
        assert_close(go[0, h], want["out"], "bf16", f"out head {h}")
        assert_close(gl[0, h], want["lse"], "bf16", f"lse head {h}")
