"""GPU parity of the fine-stage backward pass (fvattn_block_sparse_bwd)
through the C ABI against the oracle's gradients.

Lists are inputs to both sides: seeded random lists, or the oracle's own
selection on the seeded workload; the GPU computes out and lse with its own
forward (fvattn_block_sparse_fwd on those lists), the oracle recomputes
everything from q, k, v, dout.

Tolerance, from the arithmetic: the kernels round P and dS to bf16 for the
tensor cores (relative 2^-9 each), take p from the forward's fp32 lse and D
from its bf16 output, accumulate in fp32 and round each gradient once to
bf16.  With a_rk = p_rk (|dp_rk| + sum_c |dout_rc out_rc|) the error of dS
is at most ~2^-7 a, so per element
  dq, dk: |gpu - exact| <= 2^-8 |exact| + 2^-6 * scale * (a |k| or a^T |q|)
  dv:     |gpu - exact| <= 2^-8 |exact| + 2^-7 * (p^T |dout|)
(factor 2 of margin on the derived terms)."""
import numpy as np
import pytest
import torch

from block_sparse_spatiotemporal_b200 import fvattn as F
from block_sparse_spatiotemporal_b200.inputs import WORKLOADS, make_inputs
from oracle import fvattn_oracle as O
from tests.gpu_util import to_dev, to_host

pytestmark = pytest.mark.gpu


def random_lists(nT, density, seed, empty_rows=(), unused_cols=()):
    rng = np.random.default_rng(seed)
    counts = np.zeros(nT, np.int32)
    idx = np.zeros((nT, nT), np.int32)
    for i in range(nT):
        if i in empty_rows:
            continue
        sel = [j for j in np.flatnonzero(rng.random(nT) < density) if j not in unused_cols]
        if not sel:
            sel = [j for j in range(nT) if j not in unused_cols][:1]
        counts[i] = len(sel)
        idx[i, :len(sel)] = sel
    return counts, idx


def run_gpu(q, k, v, g, counts, idx, grid, heads):
    """q, k, v, g: bf16 bit patterns [1, H, N, 128] in tiled order;
    counts [H, nT], idx [H, nT, nT]."""
    shape = F.make_shape(1, heads, 128, grid, dtype=F.BF16, layout=F.TILED)
    ws = torch.empty(max(F.workspace_size(shape), F.workspace_size_bwd(shape)), dtype=torch.uint8, device="cuda")
    qd, kd, vd, gd = (to_dev(x, "bf16") for x in (q, k, v, g))
    cd = torch.from_numpy(counts[None].astype(np.int32)).cuda()
    idd = torch.from_numpy(idx[None].astype(np.int32)).cuda()
    out, lse = F.block_sparse_fwd(shape, qd, kd, vd, cd, idd, ws)
    assert F.device_status(ws) == 0
    dq, dk, dv = F.block_sparse_bwd(shape, qd, kd, vd, out, gd, lse, cd, idd, ws)
    assert F.device_status(ws) == 0
    return to_host(dq)[0], to_host(dk)[0], to_host(dv)[0]


def check(got, ref, scale_elem, frac, label):
    tol = 2.0 ** -8 * np.abs(ref) + frac * scale_elem
    err = np.abs(got - ref)
    bad = err > tol
    assert not bad.any(), (label, int(bad.sum()), float((err - tol).max()), float(err.max()))
    # and on average far inside the bound
    assert err.mean() <= 0.25 * tol.mean(), (label, float(err.mean()), float(tol.mean()))


def oracle_grads(q, k, v, g, counts, idx, scale, rows=None):
    """Oracle gradients and error scales of one head (float64 inputs, tiled);
    with ``rows`` only those query tiles contribute."""
    c = counts.copy()
    if rows is not None:
        keep = np.zeros(len(c), bool)
        keep[list(rows)] = True
        c[~keep] = 0
    out, _ = O.fine_head(q, k, v, c, idx, scale, rows=[i for i in range(len(c)) if c[i] > 0])
    out = np.nan_to_num(out)
    grads = O.fine_head_backward(q, k, v, g, c, idx, scale)
    scales = O.fine_head_backward_scales(q, k, v, g, out, c, idx, scale)
    return grads, scales


def seeded(shape, seed):
    rng = np.random.default_rng(seed)
    from block_sparse_spatiotemporal_b200.inputs import f32_to_bf16_bits
    return f32_to_bf16_bits(rng.standard_normal(shape).astype(np.float32))


@pytest.mark.parametrize("case", [
    dict(grid=(8, 8, 16), heads=2, density=0.35, seed=1),                       # nT = 16
    dict(grid=(4, 4, 12), heads=1, density=0.7, seed=2),                        # nT = 3: a missing second tile
    dict(grid=(4, 8, 8), heads=2, density=1.0, seed=3),                         # dense
    dict(grid=(8, 8, 8), heads=1, density=0.3, seed=4, empty=(2,), unused=(5,)),  # empty row, unselected key tile
])
def test_backward_matches_oracle_small(case):
    grid, H = case["grid"], case["heads"]
    N = grid[0] * grid[1] * grid[2]
    nT = N // 64
    q, k, v, g = (seeded((1, H, N, 128), case["seed"] * 10 + t) for t in range(4))
    counts = np.zeros((H, nT), np.int32)
    idx = np.zeros((H, nT, nT), np.int32)
    for h in range(H):
        counts[h], idx[h] = random_lists(nT, case["density"], case["seed"] * 100 + h, case.get("empty", ()),
                                         case.get("unused", ()))
    dq, dk, dv = run_gpu(q, k, v, g, counts, idx, grid, H)
    scale = O.default_scale(128)
    for h in range(H):
        args = [O.as_f64(x[0, h], "bf16") for x in (q, k, v, g)]
        (rq, rk, rv), (sq, sk, sv) = oracle_grads(*args, counts[h], idx[h], scale)
        check(dq[h], rq, sq, 2.0 ** -6, f"dq h{h}")
        check(dk[h], rk, sk, 2.0 ** -6, f"dk h{h}")
        check(dv[h], rv, sv, 2.0 ** -7, f"dv h{h}")
        for e in case.get("empty", ()):
            assert not dq[h, 64 * e:64 * e + 64].any()
        for u in case.get("unused", ()):
            assert not dk[h, 64 * u:64 * u + 64].any() and not dv[h, 64 * u:64 * u + 64].any()


def test_backward_480p_sampled():
    """The 480p workload (40 heads, 33,280 tokens, tiled raster-cube order)
    with the oracle's own top-p lists, in the launch configuration the
    benchmark times.  Six heads are checked on two query tiles (dq) and two
    key tiles (dk, dv) each, every query tile that selected those key tiles
    contributing; all heads are checked on the softmax-gradient identities
    (dk sums to zero over keys, dv sums to the sum of dout)."""
    wl = WORKLOADS["wan480p"]
    q, k, v = make_inputs(wl)
    N, H, nT = wl.tokens, wl.heads, wl.num_tiles
    pos = O.positions(wl.grid, wl.order)
    scale = O.default_scale(128)
    counts = np.zeros((H, nT), np.int32)
    idx = np.zeros((H, nT, nT), np.int32)
    for h in range(H):
        r = O.coarse_head(O.as_f64(q[0, h], "bf16"), O.as_f64(k[0, h], "bf16"), wl.grid, wl.order, wl.top_p,
                          wl.k_min, scale, None, pos)
        counts[h], idx[h] = r["counts"], r["idx"]
    g = seeded((1, H, N, 128), 77)
    til = lambda x: O.to_tiled(x, pos)                       # natural -> tiled rows  # noqa: E731
    qt, kt, vt = til(q), til(k), til(v)
    gt = g                                                  # dout drawn directly in tiled order
    dq, dk, dv = run_gpu(qt, kt, vt, gt, counts, idx, wl.grid, H)
    # identities on every head
    for h in range(H):
        live = np.repeat(counts[h] > 0, 64)
        gsum = O.as_f64(gt[0, h], "bf16")[live].sum(axis=0)
        assert np.abs(dk[h].sum(axis=0)).max() <= 1e-2 * np.abs(dk[h]).sum(axis=0).max() + 1e-3
        assert np.abs(dv[h].sum(axis=0) - gsum).max() <= 1e-2 * np.abs(dv[h]).sum(axis=0).max() + 1e-3
    rng = np.random.default_rng(5)
    for h in rng.choice(H, 6, replace=False):
        I = sorted({0, nT - 1} if h % 2 else set(rng.choice(nT, 2, replace=False).tolist()))
        J = sorted(set(rng.choice(nT, 2, replace=False).tolist()))
        users = {i for i in range(nT) for j in J if j in idx[h, i, :counts[h, i]]}
        args = [O.as_f64(x[0, h], "bf16") for x in (qt, kt, vt, gt)]
        (rq, rk, rv), (sq, sk, sv) = oracle_grads(*args, counts[h], idx[h], scale, rows=set(I) | users)
        for i in I:
            sl = slice(64 * i, 64 * i + 64)
            check(dq[h, sl], rq[sl], sq[sl], 2.0 ** -6, f"dq h{h} tile {i}")
        for j in J:
            sl = slice(64 * j, 64 * j + 64)
            check(dk[h, sl], rk[sl], sk[sl], 2.0 ** -6, f"dk h{h} tile {j}")
            check(dv[h, sl], rv[sl], sv[sl], 2.0 ** -7, f"dv h{h} tile {j}")


def test_backward_rejects_natural_layout_and_f32():
    grid = (4, 4, 8)
    shape = F.make_shape(1, 1, 128, grid, dtype=F.BF16, layout=F.NATURAL)
    ws = torch.empty(F.workspace_size_bwd(shape), dtype=torch.uint8, device="cuda")
    x = torch.zeros((1, 1, 128, 128), dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros((1, 1, 128), dtype=torch.float32, device="cuda")
    c = torch.ones((1, 1, 2), dtype=torch.int32, device="cuda")
    i = torch.zeros((1, 1, 2, 2), dtype=torch.int32, device="cuda")
    with pytest.raises(F.FvattnError):
        F.block_sparse_bwd(shape, x, x, x, x, x, lse, c, i, ws)
    f32 = F.make_shape(1, 1, 128, grid, dtype=F.F32, layout=F.TILED)
    with pytest.raises(F.FvattnError):
        F.block_sparse_bwd(f32, x, x, x, x, x, lse, c, i, ws)
