"""GPU parity of slack-aware augmentation (fvattn_augment_lists) and of the
fine stage run with its work list (fvattn_block_sparse_fwd_worklist),
through the C ABI, against the oracle.  Base lists are the oracle's own
selection (an input to both sides).  The work list is integer logic and must
match exactly; the added tiles must match the oracle's, except where the
last tile taken and the first one left out are within the float32 rounding
of the coarse logits (then the GPU's pick must still be a best set within
that bound)."""
import numpy as np
import pytest
import torch

from block_sparse_spatiotemporal_b200 import fvattn as F
from block_sparse_spatiotemporal_b200.inputs import Workload, WORKLOADS, make_inputs
from oracle import fvattn_oracle as O
from tests.gpu_util import assert_close, oracle_coarse, oracle_rope, rope_of, shape_of, to_dev, to_host

pytestmark = pytest.mark.gpu


def base_lists(wl, q, k, top_p, k_min):
    res = oracle_coarse(wl, q, k, top_p, k_min)
    nT = wl.num_tiles
    counts = np.stack([r["counts"] for r in res]).astype(np.int32)
    idx = np.zeros((wl.heads, nT, nT), np.int32)
    for h, r in enumerate(res):
        idx[h, :, :r["idx"].shape[1]] = r["idx"]
    S = np.stack([r["S"] for r in res])
    tol = np.stack([1e-5 * r["s_abs"].max(axis=1) for r in res])        # per row
    return counts, idx, S, tol


def compare(wl, counts, idx, S, tol, G, gc, gi, gw, busy=None, fill=100):
    nT, P = wl.num_tiles, (wl.num_tiles + 1) // 2
    oc, oi, added, order = O.augment_lists(S, counts, idx, G, cta_busy_ns=busy, fill_percent=fill)
    assert np.array_equal(gw, np.array(order)), "work list"
    unions = O.item_unions(counts, idx, nT)
    ties = 0
    for item, u in enumerate(unions):
        h, q = divmod(item, P)
        rows = [r for r in (2 * q, 2 * q + 1) if r < nT]
        live = [r for r in rows if counts[h, r] > 0]
        for r in rows:
            if counts[h, r] == 0:
                assert gc[0, h, r] == 0
        if not live:
            continue
        g_add = set(gi[0, h, live[0], :gc[0, h, live[0]]].tolist()) - u
        o_add = set(oi[h, live[0], :oc[h, live[0]]].tolist()) - u
        for r in live:       # every live row carries its base list plus the same picks
            assert gi[0, h, r, :gc[0, h, r]].tolist() == sorted(set(idx[h, r, :counts[h, r]].tolist()) | g_add)
        assert len(g_add) == len(o_add) == added[item]
        if g_add != o_add:   # near tie: the GPU's picks must be a best set within the rounding bound
            ties += 1
            score = {j: max(S[h, r, j] for r in live) for j in range(nT) if j not in u}
            t = max(tol[h, r] for r in live)
            worst_in = min(score[j] for j in g_add)
            best_out = max([score[j] for j in score if j not in g_add], default=-np.inf)
            assert worst_in >= best_out - t, (item, worst_in, best_out)
    if busy is not None:      # slack from measured time: the entry loads may move either way
        return oc, oi, ties
    # the kept work list's critical path did not grow
    costs_b = [max(1, len(x)) for x in unions]
    costs_a = [max(1, len(x)) for x in O.item_unions(gc[0], gi[0], nT)]
    Gc = min(G, len(order))
    load = lambda costs: max(sum(costs[order[t]] for t in range(c, len(order), Gc)) for c in range(Gc))  # noqa: E731
    assert load(costs_a) == load(costs_b)
    return oc, oi, ties


@pytest.mark.parametrize("case", [
    dict(grid=(8, 16, 24), heads=4, G=3, p=0.9, k_min=2),
    dict(grid=(8, 16, 24), heads=4, G=16, p=0.8, k_min=1, order="hilbert", rope=True),
    dict(grid=(4, 8, 12), heads=2, G=200, p=0.5, k_min=1),        # more CTAs than items
    dict(grid=(4, 4, 20), heads=3, G=2, p=0.6, k_min=1),          # nT = 5: the last item has one row
])
def test_augment_small(case):
    wl = Workload("aug", case["grid"], case["heads"], 128, "bf16", 17, case["p"], case["k_min"],
                  case.get("order", "raster"), case.get("rope", False), "per_head")
    q, k, v = make_inputs(wl)
    counts, idx, S, tol = base_lists(wl, q, k, wl.top_p, wl.k_min)
    shape = shape_of(wl)
    rope = rope_of(wl)
    ws = F.workspace(shape, rope)
    qd, kd, vd = to_dev(q, "bf16"), to_dev(k, "bf16"), to_dev(v, "bf16")
    cd = torch.from_numpy(counts[None]).cuda()
    idd = torch.from_numpy(idx[None]).cuda()
    ac, ai, wlist = F.augment_lists(shape, qd, kd, ws, cd, idd, num_ctas=case["G"], rope=rope)
    assert F.device_status(ws) == 0
    gc, gi, gw = ac.cpu().numpy(), ai.cpu().numpy(), wlist.cpu().numpy()
    oc, oi, ties = compare(wl, counts, idx, S, tol, case["G"], gc, gi, gw)
    assert ties == 0
    # the fine stage on the augmented lists with the kept work list
    out, lse = F.block_sparse_fwd_worklist(shape, qd, kd, vd, ac, ai, wlist, ws, num_ctas=case["G"], rope=rope)
    assert F.device_status(ws) == 0
    got, glse = to_host(out)[0], lse.cpu().numpy()[0]
    for h in range(wl.heads):
        ref = O.forward_head(q[0, h], k[0, h], v[0, h], wl.grid, wl.order, wl.top_p, wl.k_min, "bf16",
                             rope=oracle_rope(wl), blocks=(oc[h], oi[h]))
        assert_close(got[h], ref["out"], "bf16", f"out h{h}")
        assert_close(glse[h], ref["lse"], "bf16", f"lse h{h}")


@pytest.mark.parametrize("G,fill", [(16, 100), (16, 37), (5, 0), (200, 60)])
def test_augment_measured_slack(G, fill):
    """Slack from per-CTA busy times (seeded synthetic nanoseconds, the same
    array on both sides) instead of entry counts: work list exact, the same
    tiles added per item as the oracle's."""
    wl = Workload("aug", (8, 16, 24), 4, 128, "bf16", 23, 0.85, 2, "raster", False, "per_head")
    q, k, v = make_inputs(wl)
    counts, idx, S, tol = base_lists(wl, q, k, wl.top_p, wl.k_min)
    items = wl.heads * ((wl.num_tiles + 1) // 2)
    Gc = min(G, items)
    busy = np.random.default_rng(G * 1000 + fill).integers(1_000_000, 3_000_000, Gc).tolist()
    shape = shape_of(wl)
    ws = F.workspace(shape)
    qd, kd = to_dev(q, "bf16"), to_dev(k, "bf16")
    cd = torch.from_numpy(counts[None]).cuda()
    idd = torch.from_numpy(idx[None]).cuda()
    ac, ai, wlist = F.augment_lists(shape, qd, kd, ws, cd, idd, num_ctas=G, cta_busy_ns=busy, fill_percent=fill)
    assert F.device_status(ws) == 0
    gc, gi, gw = ac.cpu().numpy(), ai.cpu().numpy(), wlist.cpu().numpy()
    _, _, ties = compare(wl, counts, idx, S, tol, Gc, gc, gi, gw, busy=busy, fill=fill)
    assert ties == 0
    if fill == 0:
        assert np.array_equal(gc[0], counts)


def test_augment_480p_full():
    """The 480p workload with the oracle's top-p lists and one CTA per SM:
    work list exact, picks as the oracle's up to rounding ties, the critical
    path unchanged; the fine stage on the augmented lists runs clean."""
    wl = WORKLOADS["wan480p"]
    q, k, v = make_inputs(wl)
    counts, idx, S, tol = base_lists(wl, q, k, wl.top_p, wl.k_min)
    G = torch.cuda.get_device_properties(0).multi_processor_count
    shape = shape_of(wl)
    ws = F.workspace(shape)
    qd, kd, vd = to_dev(q, "bf16"), to_dev(k, "bf16"), to_dev(v, "bf16")
    cd = torch.from_numpy(counts[None]).cuda()
    idd = torch.from_numpy(idx[None]).cuda()
    ac, ai, wlist = F.augment_lists(shape, qd, kd, ws, cd, idd, num_ctas=G)
    assert F.device_status(ws) == 0
    gc, gi, gw = ac.cpu().numpy(), ai.cpu().numpy(), wlist.cpu().numpy()
    _, _, ties = compare(wl, counts, idx, S, tol, G, gc, gi, gw)
    assert ties <= 20
    assert gc.sum() > counts.sum()                       # there was slack to fill
    out, lse = F.block_sparse_fwd_worklist(shape, qd, kd, vd, ac, ai, wlist, ws, num_ctas=G)
    assert F.device_status(ws) == 0
    assert torch.isfinite(out.float()).all() and torch.isfinite(lse).all()
