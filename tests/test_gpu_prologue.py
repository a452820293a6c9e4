"""GPU parity of the attention prologue (QKV projection fused with the 3D
rotary encoding, "Causal-RoPE SP" digest, sections 2.2-2.3) through the C
ABI: every output of small cases, and sampled tokens of the full 720p-shaped
projection, against the oracle.

Tolerance, from the arithmetic: the kernel sums exact bf16 products in fp32
and rotates in fp32, then rounds once to bf16; the oracle rounds the exact
value.  So |gpu - exact| <= 1/2 ulp_bf16 + delta, delta = 2^-16 * sum|x w|
(+ |bias|) per output (per rotated pair, the larger of the two, times
sqrt 2): fp32 summation error of any order over K <= 65536 terms stays far
below it in practice, and it is still 6x below half a bf16 ulp of a
unit-scale output at C = 5120.  At least 99% of the outputs must round to
the oracle's bf16 value exactly."""
import math

import numpy as np
import pytest
import torch

from block_sparse_spatiotemporal_b200 import fvattn as F
from block_sparse_spatiotemporal_b200.inputs import make_projection_inputs
from oracle import fvattn_oracle as O
from tests.gpu_util import to_dev, to_host

pytestmark = pytest.mark.gpu

ROPE_DIMS, ROPE_BASE = (44, 42, 42), 10000.0


def _ulp_bf16(x):
    a = np.maximum(np.abs(x), 2.0 ** -126)
    return 2.0 ** (np.floor(np.log2(a)) - 7)


def check(got, raw, bound, label):
    """got: GPU bf16 values (float64); raw: exact oracle values; bound: the
    oracle's |x||w| scale of each output."""
    ref = O.round_bf16(raw)
    tol = 0.5 * _ulp_bf16(np.maximum(np.abs(raw), np.abs(got))) + math.sqrt(2.0) * 2.0 ** -16 * bound
    err = np.abs(got - raw)
    bad = err > tol
    assert not bad.any(), (label, int(bad.sum()), float((err - tol).max()))
    exact = float((got == ref).mean())
    assert exact >= 0.99, (label, exact)
    return exact


def run(grid, B, H, C, layout, order, rope, t_offset, bias=True, seed=21):
    T, Hg, W = grid
    N = T * Hg * W
    x, w, b = make_projection_inputs(B, N, C, H, 128, seed, bias)
    shape = F.make_shape(B, H, 128, grid, dtype=F.BF16, order=F.HILBERT if order == "hilbert" else F.RASTER_CUBE,
                         layout=layout)
    rp = F.make_rope(ROPE_DIMS, ROPE_BASE) if rope else None
    ws = torch.empty(F.workspace_size_qkv(shape, rp), dtype=torch.uint8, device="cuda")
    xd, wd = to_dev(x, "bf16"), to_dev(w, "bf16")
    bd = torch.from_numpy(b).cuda() if b is not None else None
    q, k, v = F.qkv_rope(shape, xd, wd, ws, bias=bd, rope=rp, t_offset=t_offset)
    assert F.device_status(ws) == 0
    return x, w, b, (q, k, v)


CASES = [
    # grid, B, H, C, layout, order, rope, t_offset, bias
    ((4, 4, 20), 1, 3, 192, F.NATURAL, "raster", True, 0, True),      # M = 320: one full tile + 64 rows; H odd
    ((4, 8, 12), 2, 2, 64, F.TILED, "raster", True, 5, True),         # one k block; tiles span both batches
    ((8, 8, 12), 1, 1, 320, F.TILED, "hilbert", True, 3, False),      # five k blocks: the stage ring wraps
    ((4, 12, 8), 1, 2, 128, F.NATURAL, "raster", False, 0, True),     # no rotation
    ((8, 16, 32), 1, 8, 256, F.TILED, "hilbert", True, 11, True),     # 192 tiles: several per CTA
]


@pytest.mark.parametrize("case", CASES, ids=[f"g{c[0]}_B{c[1]}H{c[2]}C{c[3]}_{c[5]}{c[4]}_r{int(c[6])}s{c[7]}"
                                              for c in CASES])
def test_prologue_matches_oracle(case):
    grid, B, H, C, layout, order, rope, s, bias = case
    x, w, b, out = run(grid, B, H, C, layout, order, rope, s, bias)
    xf, wf = O.as_f64(x, "bf16"), O.as_f64(w, "bf16")
    bf = None if b is None else b.astype(np.float64)
    orope = dict(dims=ROPE_DIMS, base=ROPE_BASE) if rope else None
    raw = O.qkv_rope(xf, wf, bf, grid, H, 128, orope, t_offset=s, rounded=False)
    bound = O.qkv_abs_bound(xf, wf, bf, H, 128)
    pos = O.positions(grid, order) if layout == F.TILED else None
    for i, name in enumerate("qkv"):
        got = to_host(out[i])
        if pos is not None:
            got = got[..., pos, :]        # back to natural order
        check(got, raw[i], bound[i], name)


def test_prologue_tiled_equals_reorder_of_natural():
    """The tiled output is bit-identical to fvattn_tile_reorder of the
    natural output (same arithmetic, rows permuted in the epilogue)."""
    grid, B, H, C = (8, 8, 16), 1, 2, 128
    T, Hg, W = grid
    x, w, b = make_projection_inputs(B, T * Hg * W, C, H, 128, 4)
    rp = F.make_rope(ROPE_DIMS, ROPE_BASE)
    xd, wd, bd = to_dev(x, "bf16"), to_dev(w, "bf16"), torch.from_numpy(b).cuda()
    outs = {}
    for layout in (F.NATURAL, F.TILED):
        shape = F.make_shape(B, H, 128, grid, dtype=F.BF16, order=F.HILBERT, layout=layout)
        ws = torch.empty(max(F.workspace_size_qkv(shape, rp), F.workspace_size(shape)), dtype=torch.uint8,
                         device="cuda")
        outs[layout] = (shape, ws, F.qkv_rope(shape, xd, wd, ws, bias=bd, rope=rp, t_offset=2))
    shape, ws, nat = outs[F.NATURAL]
    til = outs[F.TILED][2]
    for a, t in zip(nat, til):
        assert torch.equal(F.tile_reorder(shape, a, ws), t)


def test_prologue_rejects_bad_arguments():
    grid = (4, 4, 4)
    shape = F.make_shape(1, 1, 128, grid, dtype=F.BF16)
    ws = torch.empty(F.workspace_size_qkv(shape), dtype=torch.uint8, device="cuda")
    x = torch.zeros((1, 64, 64), dtype=torch.bfloat16, device="cuda")
    w = torch.zeros((384, 64), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(F.FvattnError):          # channels not a multiple of 64
        F.qkv_rope(shape, x[..., :32].contiguous(), w[:, :32].contiguous(), ws)
    with pytest.raises(F.FvattnError):          # negative start frame
        F.qkv_rope(shape, x, w, ws, t_offset=-1)
    f32 = F.make_shape(1, 1, 128, grid, dtype=F.F32)
    with pytest.raises(F.FvattnError):          # bf16 only
        F.qkv_rope(f32, x, w, ws)
    with pytest.raises(F.FvattnError):          # workspace too small
        F.qkv_rope(shape, x, w, ws[:16])
    q, k, v = F.qkv_rope(shape, x, w, ws)       # zero inputs, no bias: zero outputs
    assert not q.any() and not k.any() and not v.any()


def test_prologue_full_720p_sampled_tokens():
    """The 720p-shaped projection (76,800 tokens x 5120 channels -> 40 heads
    of Q, K and V, tiled in Hilbert order, RoPE at start frame 0) in the
    launch configuration the benchmark times; 96 sampled tokens (the first
    and last, tile and frame boundaries, random) checked in every head."""
    grid, B, H, C, s = (20, 48, 80), 1, 40, 5120, 0
    T, Hg, W = grid
    N = T * Hg * W
    x, w, b, out = run(grid, B, H, C, F.TILED, "hilbert", True, s, seed=3)
    rng = np.random.default_rng(0)
    toks = np.unique(np.concatenate([[0, 1, 63, 64, N - 1, N - 64, Hg * W - 1, Hg * W],
                                     rng.integers(0, N, 88)]))
    xf, wf = O.as_f64(x[:, toks], "bf16"), O.as_f64(w, "bf16")
    bf = b.astype(np.float64)
    raw = O.qkv_rope(xf, wf, bf, grid, H, 128, dict(dims=ROPE_DIMS, base=ROPE_BASE), t_offset=s, tokens=toks,
                     rounded=False, gathered=True)
    bound = O.qkv_abs_bound(xf, wf, bf, H, 128)
    pos = O.positions(grid, "hilbert")
    rows = torch.from_numpy(pos[toks]).cuda()
    for i, name in enumerate("qkv"):
        got = to_host(out[i][:, :, rows, :])
        check(got, raw[i], bound[i], name)
