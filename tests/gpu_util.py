"""Helpers for the GPU parity tests: host<->device conversion of the seeded
inputs and comparisons against the oracle (which always runs on the CPU on
its own inputs; nothing computed by the CUDA path is fed to it)."""
from __future__ import annotations

import numpy as np
import torch

from block_sparse_spatiotemporal_b200 import fvattn as F
from block_sparse_spatiotemporal_b200.inputs import Workload
from oracle import fvattn_oracle as O

BF16_MAX_ABS, BF16_MEAN_ABS = 2e-2, 2e-3
F32_ABS = 1e-4


def to_dev(x: np.ndarray, dtype: str) -> torch.Tensor:
    if dtype == "bf16":
        return torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).cuda()


def to_host(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def shape_of(wl: Workload, layout=F.NATURAL) -> F.Shape:
    return F.make_shape(wl.batch, wl.heads, wl.head_dim, wl.grid,
                        dtype=F.BF16 if wl.dtype == "bf16" else F.F32,
                        order=F.HILBERT if wl.order == "hilbert" else F.RASTER_CUBE, layout=layout)


def rope_of(wl: Workload):
    return F.make_rope(wl.rope_dims, wl.rope_base) if wl.rope else None


def oracle_rope(wl: Workload):
    return dict(dims=wl.rope_dims, base=wl.rope_base) if wl.rope else None


def oracle_coarse(wl: Workload, q, k, top_p, k_min, b=0, heads=None):
    """Oracle steps 1-5 for every head: list of per-head result dicts."""
    pos = O.positions(wl.grid, wl.order)
    out = []
    for h in (range(wl.heads) if heads is None else heads):
        out.append(O.coarse_head(O.as_f64(q[b, h], wl.dtype), O.as_f64(k[b, h], wl.dtype), wl.grid, wl.order,
                                 top_p, k_min, O.default_scale(wl.head_dim), oracle_rope(wl), pos))
    return out


def compare_blocks(res: dict, gpu_counts: np.ndarray, gpu_idx: np.ndarray, top_p: float):
    """Compare one head's GPU lists with the oracle's.

    Returns (n_mismatch, n_border, n_neartie_checked, equal_rows).  Rows whose
    cumulative mass lies within 1e-5 of top_p at the cut are exempt (counted).
    Near-tie rows -- the last kept and first dropped logits closer than the
    float32 rounding bound of a 128-term dot product (1e-5 of the row's
    largest scale * |Qp|.|Kp|) -- may select either tile, but the GPU set must
    still be a top-count set within that bound.  Any other difference is a
    mismatch."""
    S, counts, idx, border = res["S"], res["counts"], res["idx"], res["border"]
    nT = S.shape[0]
    tol = 1e-5 * res["s_abs"].max(axis=1)
    near = O.near_tie_rows(S, counts, tol)
    mism = 0
    ntie = 0
    equal = np.zeros(nT, bool)
    for r in range(nT):
        c = int(gpu_counts[r])
        same = c == counts[r] and np.array_equal(gpu_idx[r, :c], idx[r, :counts[r]])
        equal[r] = same
        if same or border[r]:
            continue
        if near[r] and c == counts[r]:
            sel = gpu_idx[r, :c]
            ok = len(set(sel.tolist())) == c and (np.diff(sel) > 0).all()
            rest = np.setdiff1d(np.arange(nT), sel)
            if ok and len(rest):
                ok = S[r, sel].min() >= S[r, rest].max() - tol[r]
            ntie += 1
            if ok:
                continue
        mism += 1
    return mism, int(border.sum()), ntie, equal


def assert_close(got: np.ndarray, want: np.ndarray, dtype: str, what: str):
    mask = ~np.isnan(want)
    assert mask.any(), what
    diff = np.abs(got[mask] - want[mask])
    assert np.isfinite(got[mask]).all(), f"{what}: non-finite values"
    if dtype == "bf16":
        assert diff.max() <= BF16_MAX_ABS, f"{what}: max abs {diff.max():.3g}"
        assert diff.mean() <= BF16_MEAN_ABS, f"{what}: mean abs {diff.mean():.3g}"
    else:
        assert diff.max() <= F32_ABS, f"{what}: max abs {diff.max():.3g}"
    return float(diff.max()), float(diff.mean())


def sample_tiles(nT: int, n: int, seed: int):
    """Seeded sample of query tiles, always including the first and last."""
    rng = np.random.default_rng(seed)
    pick = set(rng.choice(nT, size=min(n, nT), replace=False).tolist()) | {0, nT - 1}
    return sorted(pick)
