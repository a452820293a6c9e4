"""GPU parity on the five benchmark workloads at full size, in the launch
configuration bench.py times (fvattn_forward on natural-layout tensors).

Block lists: every row of every head is compared with the oracle.  Rows
whose cumulative mass lies within 1e-5 of top_p at the cut (borderline) and
rows whose last kept and first dropped logits are within the float32
rounding bound (near ties) may differ from the oracle's list, but only with
a valid list (oracle/list_check.py); their numbers are counted and printed.
Outputs and lse: every row of every head for the small workloads; for the
large ones every row of whole heads chosen from the oracle's lists (the
densest head, the head whose mass is most concentrated on one key tile --
the sink-dominated head -- and seeded others) plus a seeded sample of query
tiles in every other head, always on rows whose lists match the oracle's."""
import numpy as np
import pytest
import torch

from block_sparse_spatiotemporal_b200 import fvattn as F
from block_sparse_spatiotemporal_b200.inputs import WORKLOADS, make_inputs, perturb_steps, sweep_points
from oracle import fvattn_oracle as O
from tests.gpu_util import (assert_close, compare_blocks, oracle_coarse, oracle_rope, rope_of, sample_tiles,
                            shape_of, sum_checks, to_dev, to_host)

pytestmark = pytest.mark.gpu

_INPUTS = {}


def inputs(name):
    if name not in _INPUTS:
        _INPUTS.clear()
        _INPUTS[name] = make_inputs(WORKLOADS[name])
    return _INPUTS[name]


def run_forward(wl, q, k, v, top_p, k_min, cache=None, reuse=False, dev_inputs=None):
    shape = shape_of(wl)
    rope = rope_of(wl)
    ws = F.workspace(shape, rope)
    if cache is None:
        cache, _, _ = F.new_cache(shape)
    qd, kd, vd = dev_inputs if dev_inputs is not None else (to_dev(x, wl.dtype) for x in (q, k, v))
    out, lse = F.forward(shape, qd, kd, vd, ws, top_p, k_min, rope=rope, cache=cache, reuse_mask=reuse)
    assert F.device_status(ws) == 0
    return out, lse, cache


def whole_heads(res, extra, seed):
    """Heads compared on every row: the densest (most selected pairs), the
    sink-dominated one (largest mean probability that the rows give one key
    tile) and `extra` seeded others."""
    dens = [int(r["counts"].sum()) for r in res]
    sink = [float(r["P"].mean(axis=0).max()) for r in res]
    pick = [int(np.argmax(dens)), int(np.argmax(sink))]
    rng = np.random.default_rng(seed)
    rest = [h for h in range(len(res)) if h not in pick]
    pick += [int(h) for h in rng.choice(rest, size=min(extra, len(rest)), replace=False)]
    return sorted(set(pick))


def check_workload(wl, q, k, v, top_p, k_min, tiles_per_head=None, full_heads=0, seed=0):
    """tiles_per_head None: every row of every head; otherwise every row of the
    whole heads (whole_heads with `full_heads` extra ones) and a seeded
    sample of query tiles in the others."""
    shape = shape_of(wl)
    cache, counts_d, idx_d = F.new_cache(shape)
    out, lse, _ = run_forward(wl, q, k, v, top_p, k_min, cache=cache)
    gc, gi = counts_d.cpu().numpy(), idx_d.cpu().numpy()
    o, l = to_host(out), to_host(lse)
    res = oracle_coarse(wl, q, k, top_p, k_min)
    nT = wl.num_tiles
    pos = O.positions(wl.grid, wl.order)
    tile_of = pos // 64
    checks = [compare_blocks(r, gc[0, h], gi[0, h], top_p, k_min) for h, r in enumerate(res)]
    tot = sum_checks(checks)
    assert tot["mismatch"] == 0, f"block-list rows differ: {tot}"
    full = set(range(wl.heads)) if tiles_per_head is None else set(whole_heads(res, full_heads, seed))
    worst = (0.0, 0.0)
    compared = 0
    for h, r in enumerate(res):
        tiles = range(nT) if h in full else sample_tiles(nT, tiles_per_head, seed + h)
        tiles = [i for i in tiles if checks[h]["equal_rows"][i]]
        if not tiles:
            continue
        f = O.forward_head(q[0, h], k[0, h], v[0, h], wl.grid, wl.order, top_p, k_min, wl.dtype,
                           rope=oracle_rope(wl), blocks=(r["counts"], r["idx"]), rows=tiles)
        rows = np.isin(tile_of, tiles)
        mx, mean = assert_close(o[0, h][rows], f["out"][rows], wl.dtype, f"out head {h}")
        assert_close(l[0, h][rows], f["lse"][rows], wl.dtype, f"lse head {h}")
        worst = (max(worst[0], mx), max(worst[1], mean))
        compared += len(tiles)
    print(f"{wl.name} top_p={top_p} k_min={k_min}: lists {tot}; whole heads {sorted(full)[:8]}; "
          f"{compared} query tiles compared, worst max-abs {worst[0]:.3g}, worst mean-abs {worst[1]:.3g}")
    return gc, gi, res, tot


def test_tiny_fp32_full():
    wl = WORKLOADS["tiny_fp32"]
    q, k, v = inputs(wl.name)
    check_workload(wl, q, k, v, wl.top_p, wl.k_min)


def test_grid16k_full():
    wl = WORKLOADS["grid16k"]
    q, k, v = inputs(wl.name)
    check_workload(wl, q, k, v, wl.top_p, wl.k_min)


def test_wan480p_sampled():
    wl = WORKLOADS["wan480p"]
    q, k, v = inputs(wl.name)
    _, _, _, tot = check_workload(wl, q, k, v, wl.top_p, wl.k_min, tiles_per_head=6, full_heads=2)
    assert tot["rows"] == wl.heads * wl.num_tiles


def test_wan720p_hilbert_rope_sampled():
    wl = WORKLOADS["wan720p_hilbert_rope"]
    q, k, v = inputs(wl.name)
    gc, _, _, _ = check_workload(wl, q, k, v, wl.top_p, wl.k_min, tiles_per_head=4, full_heads=0)
    per_head = gc[0].mean(axis=1)
    assert per_head.max() > 4 * per_head.min()     # strongly varying selected-block counts


@pytest.mark.parametrize("top_p,k_min", sweep_points())
def test_wan480p_sweep_point(top_p, k_min):
    wl = WORKLOADS["wan480p_sweep"]
    q, k, v = inputs(wl.name)
    gc, _, _, _ = check_workload(wl, q, k, v, top_p, k_min, tiles_per_head=2, seed=int(top_p * 100) + k_min)
    if top_p >= 1.0:
        assert (gc == wl.num_tiles).all()
    if top_p <= 0.0:
        assert (gc == k_min).all()


def test_wan480p_cached_mask_steps():
    """Step 0 selects and fills the cache; each of the ten further steps
    perturbs Q/K by 0.05*N(0,1) (cumulatively) and reuses the step-0 lists.
    Every step is compared with the oracle's forward on the step-0 lists."""
    wl = WORKLOADS["wan480p_sweep"]
    q, k, v, masters = make_inputs(wl, keep_f32_masters=True)
    shape = shape_of(wl)
    cache, counts_d, idx_d = F.new_cache(shape)
    vd = to_dev(v, wl.dtype)
    run_forward(wl, q, k, v, wl.top_p, wl.k_min, cache=cache, dev_inputs=(to_dev(q, "bf16"), to_dev(k, "bf16"), vd))
    step0 = oracle_coarse(wl, q, k, wl.top_p, wl.k_min)
    gc, gi = counts_d.cpu().numpy(), idx_d.cpu().numpy()
    checks = [compare_blocks(r, gc[0, h], gi[0, h], wl.top_p, wl.k_min) for h, r in enumerate(step0)]
    assert sum_checks(checks)["mismatch"] == 0
    equal = [c["equal_rows"] for c in checks]
    pos = O.positions(wl.grid, wl.order)
    tile_of = pos // 64
    for t, (qt, kt) in enumerate(perturb_steps(wl, masters, steps=10), start=1):
        out, lse, _ = run_forward(wl, qt, kt, v, 0.5, 1, cache=cache, reuse=True,
                                  dev_inputs=(to_dev(qt, "bf16"), to_dev(kt, "bf16"), vd))
        assert torch.equal(counts_d.cpu(), torch.from_numpy(gc))      # the cache is read, not rewritten
        o, l = to_host(out), to_host(lse)
        for h in range(0, wl.heads, 5):
            tiles = [i for i in sample_tiles(wl.num_tiles, 2, 50 * t + h) if equal[h][i]]
            f = O.forward_head(qt[0, h], kt[0, h], v[0, h], wl.grid, wl.order, wl.top_p, wl.k_min, "bf16",
                               blocks=(step0[h]["counts"], step0[h]["idx"]), rows=tiles)
            rows = np.isin(tile_of, tiles)
            assert_close(o[0, h][rows], f["out"][rows], "bf16", f"step {t} out head {h}")
            assert_close(l[0, h][rows], f["lse"][rows], "bf16", f"step {t} lse head {h}")
