"""Helpers for the GPU parity tests: host<->device conversion of the seeded
inputs and comparisons against the oracle (which always runs on the CPU on
its own inputs; nothing computed by the CUDA path is fed to it)."""
from __future__ import annotations

import numpy as np
import torch

from block_sparse_spatiotemporal_b200 import fvattn as F
from block_sparse_spatiotemporal_b200.inputs import Workload
from oracle import fvattn_oracle as O
from oracle.list_check import check_lists, merge

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


def compare_blocks(res: dict, gpu_counts: np.ndarray, gpu_idx: np.ndarray, top_p: float, k_min: int):
    """Compare one head's GPU lists with the oracle's (oracle/list_check.py).

    Returns the checker's row counts plus ``equal_rows`` (bool per row).
    Borderline rows (cumulative mass within 1e-5 of top_p at the cut) and
    near-tie rows (last kept and first dropped logits within the float32
    rounding bound) may differ from the oracle's list but must be valid:
    ids ascending and in range, the count between the counts at
    top_p -/+ 1e-5 (borderline) or equal to the oracle's (near tie), and a
    top-count set of the row's logits up to the rounding bound.  Any other
    difference is a mismatch."""
    equal = np.zeros(len(gpu_counts), bool)
    out = check_lists(res, gpu_counts, gpu_idx, top_p, k_min, equal_rows=equal)
    out["equal_rows"] = equal
    return out


def sum_checks(checks):
    """Row counts of several heads' compare_blocks results, summed."""
    tot = {}
    for c in checks:
        merge(tot, {k: v for k, v in c.items() if k != "equal_rows"})
    return tot


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
