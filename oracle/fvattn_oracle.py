"""CPU oracle for adaptive block-sparse spatiotemporal attention.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path imports, calls or links
this module: only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of ``bench.py`` may use it.  It shares no code with the CUDA path; the
only common module is the seeded input generator, which holds none of the
method's arithmetic.

Plain, slow and written to be checked by eye: numpy in float64, one step per
function, in the order the pages give the method.  Library primitives
(matmul, stable argsort, cumsum, exp) serve as steps; there is no blocking,
fusion or reordering beyond the definitions below.

Sources (page title, section):
  * "VSA" digest (aibr.jp), section 3 "core technical elements": tokens are
    grouped into small (4,4,4) cubes, a coarse stage pools each cube and
    predicts per-tile importance, the fine stage runs token-level attention
    only inside the selected tiles.
  * "FVAttn" digest (iselia-ai.com), sections 00 and 02: the routing front end
    is top-p routing with a top-k safety floor; ranks off the critical path
    spend spare time on extra, somewhat important blocks (slack-aware
    augmentation).
  * "VSA" digest, section 3, also: the coarse and fine stages are trained end
    to end (hence the fine stage's backward pass).
  * "DFSAttn" digest (gist.science 2605.23445), section 1 "Hilbert shuffle":
    tokens are reordered along a 3D Hilbert curve before blocking; section 2
    "sub-block scores": a block is split into smaller sub-blocks, each scored,
    and the fine scores are summed into the block's importance; section 3
    "smart cache": the previous step's selection is reused, and sparsity is
    low at the early, noisy steps and rises as the video sharpens.
  * "Causal-RoPE SP" digest (gist.science 2603.06664), sections 2.2-2.3: 3D
    rotary position encoding with precomputed frequencies, the global frame
    index t + s of a block starting at frame s, and the QKV projection fused
    with the rotation.

Readings where the pages are silent:
  * pooling is the mean over the 64 tokens of a tile;
  * coarse logits are scale * Qp . Kp with scale = 1/sqrt(d); normalisation is
    a softmax over the key tiles of each query-tile row;
  * top-p keeps the fewest tiles (at least one) whose cumulative mass, summed
    in descending order, reaches p (``>= p``); tiles are ranked by their
    coarse logit (the probability order, without the ties that underflowing
    probabilities would create), ties to the lower tile index;
    count = min(nT, max(m, k_min)); p >= 1 keeps every tile;
  * the output is the fine stage only (the coarse stage only routes); so the
    backward pass is the gradient of the fine stage for fixed lists (the
    selection is piecewise constant in Q and K and passes no gradient);
  * lse is the natural log of the softmax normaliser;
  * RoPE: per-axis groups of 44/42/42 head dims for (t, h, w), adjacent pairs
    (2j, 2j+1) inside each group, angle = pos * base^(-2j/d_axis); pooling uses
    the rotated values unrounded (float64 here), the fine stage uses them as
    its tensor-core operands hold them: rotated in float32 and, for a bf16
    workload, rounded to bf16 (the rounding is a quantisation, so it is taken
    from the same float32 values as the kernel's, see ``rope_3d_f32``);
  * Hilbert order: Skilling's transposed-axes Hilbert index ("Programming the
    Hilbert curve", AIP Conf. Proc. 707, 2004) on the enclosing 2^k cube with
    axes (t, h, w), valid tokens ordered by index;
  * sub-block scoring: a 4x4x4 tile is split into the eight 2x2x2 sub-cubes of
    its grid coordinates; Q and K are pooled per sub-cube; every query
    sub-block takes a softmax over all key sub-blocks of the head; the
    importance of key tile j for query tile i is the mean, over the eight
    query sub-blocks of i, of the probability mass they give to the eight
    key sub-blocks of j (the sum of the fine scores, normalised so that each
    row sums to one); top-p and k_min then act on these tile probabilities,
    ranked by their logarithm (no underflow ties);
  * timestep schedule: optional dense first steps, then (top_p, k_min)
    linear in the step from their start to their end values;
  * slack-aware augmentation: see ``augment_lists`` (the persistent fine
    stage's CTAs play the pages' ranks; costs are union entries);
  * prologue: Q | K | V = X W^T + b, one linear layer whose 3*H*d output
    rows are Q heads, then K heads, then V heads (head h of each at rows
    h*d..h*d+d-1); Q and K are rotated by the 3D RoPE above at
    (t + s, h, w), s the start frame of the block ("Causal-RoPE SP" digest,
    section 2.2), V is not; the results are rounded once to bf16.

Every function below is pinned by ``tests/test_oracle_*.py`` against brute
force, closed forms, invariants or library routines; each test's docstring
names what it pins.
"""
from __future__ import annotations

import math

import numpy as np

TILE = (4, 4, 4)


# ----------------------------------------------------------------------------
# token layout and the two orders
# ----------------------------------------------------------------------------

def token_coords(grid):
    """(t, h, w) of every token in natural (raster) order, int64 [N, 3]."""
    T, Hg, W = grid
    n = np.arange(T * Hg * W, dtype=np.int64)
    return np.stack([n // (Hg * W), (n // W) % Hg, n % W], axis=1)


def check_grid(grid, tile=TILE):
    for g, t in zip(grid, tile):
        if g % t != 0:
            raise ValueError(f"grid {grid} is not a multiple of the tile {tile}")


def raster_cube_positions(grid, tile=TILE):
    """Raster-cube order: position of each natural token in the tiled layout.

    Tiles are ranked in raster order over the tile grid; inside a tile the
    64 tokens are ranked in raster order of (t%4, h%4, w%4)."""
    check_grid(grid, tile)
    c = token_coords(grid)
    nh, nw = grid[1] // tile[1], grid[2] // tile[2]
    tile_rank = ((c[:, 0] // tile[0]) * nh + c[:, 1] // tile[1]) * nw + c[:, 2] // tile[2]
    intra = ((c[:, 0] % tile[0]) * tile[1] + c[:, 1] % tile[1]) * tile[2] + c[:, 2] % tile[2]
    return tile_rank * (tile[0] * tile[1] * tile[2]) + intra


def hilbert_index_3d(coords, bits):
    """Hilbert index of each 3D point (int64 [P, 3], each coordinate < 2^bits).

    Skilling's method: convert the axes to the "transposed" Hilbert form
    (undo the excess rotations from the top bit down, then Gray-encode), then
    read the index out by interleaving one bit of each axis per level, most
    significant level first."""
    X = [np.asarray(coords[:, a], dtype=np.int64).copy() for a in range(3)]
    n = 3
    top = 1 << (bits - 1)
    q = top
    while q > 1:
        low = q - 1
        for i in range(n):
            hit = (X[i] & q) != 0
            if i == 0:
                X[0] = np.where(hit, X[0] ^ low, X[0])
                continue
            swap = (X[0] ^ X[i]) & low
            new0 = np.where(hit, X[0] ^ low, X[0] ^ swap)
            newi = np.where(hit, X[i], X[i] ^ swap)
            X[0], X[i] = new0, newi
        q >>= 1
    for i in range(1, n):
        X[i] = X[i] ^ X[i - 1]
    flip = np.zeros_like(X[0])
    q = top
    while q > 1:
        flip = np.where((X[n - 1] & q) != 0, flip ^ (q - 1), flip)
        q >>= 1
    for i in range(n):
        X[i] = X[i] ^ flip
    idx = np.zeros_like(X[0])
    for b in range(bits - 1, -1, -1):
        for i in range(n):
            idx = (idx << 1) | ((X[i] >> b) & 1)
    return idx


def hilbert_bits(grid):
    return max(1, int(math.ceil(math.log2(max(grid)))))


def hilbert_positions(grid, tile=TILE):
    """3D Hilbert order: position of each natural token when the valid tokens
    are sorted by their Hilbert index on the enclosing 2^k cube."""
    check_grid(grid, tile)
    key = hilbert_index_3d(token_coords(grid), hilbert_bits(grid))
    order = np.argsort(key, kind="stable")
    pos = np.empty_like(order)
    pos[order] = np.arange(order.size)
    return pos


def positions(grid, order, tile=TILE):
    if order == "raster":
        return raster_cube_positions(grid, tile)
    if order == "hilbert":
        return hilbert_positions(grid, tile)
    raise ValueError(order)


def tile_cubes(grid, pos, tile=TILE):
    """Cube coordinate (ct, ch, cw) of every tile rank; raises if a run of 64
    consecutive positions is not exactly one aligned 4x4x4 cube."""
    c = token_coords(grid)
    tsz = tile[0] * tile[1] * tile[2]
    inv = np.empty_like(pos)
    inv[pos] = np.arange(pos.size)
    cube = c[inv] // np.array(tile)
    cube = cube.reshape(-1, tsz, 3)
    if not (cube == cube[:, :1, :]).all():
        raise AssertionError("a tile is not one aligned cube")
    return cube[:, 0, :]


def to_tiled(x, pos):
    """x[..., N, d] in natural order -> tiled order (row pos[n] <- row n)."""
    y = np.empty_like(x)
    y[..., pos, :] = x
    return y


def from_tiled(y, pos):
    return y[..., pos, :]


# ----------------------------------------------------------------------------
# 3D rotary position encoding
# ----------------------------------------------------------------------------

def rope_3d(x, coords, dims=(44, 42, 42), base=10000.0):
    """Rotate x [N, d] (float64) by each token's (t, h, w) coordinate.

    Head dims are split into one group per axis; inside a group of size d_a,
    pair j = dims (2j, 2j+1) is rotated by angle pos_a * base^(-2j/d_a)."""
    assert sum(dims) == x.shape[-1]
    y = np.array(x, dtype=np.float64, copy=True)
    off = 0
    for axis, da in enumerate(dims):
        j = np.arange(da // 2, dtype=np.float64)
        theta = base ** (-2.0 * j / da)
        ang = coords[:, axis:axis + 1].astype(np.float64) * theta[None, :]
        c, s = np.cos(ang), np.sin(ang)
        x0 = x[:, off + 0:off + da:2].astype(np.float64)
        x1 = x[:, off + 1:off + da:2].astype(np.float64)
        y[:, off + 0:off + da:2] = x0 * c - x1 * s
        y[:, off + 1:off + da:2] = x0 * s + x1 * c
        off += da
    return y


def rope_3d_f32(x, coords, dims=(44, 42, 42), base=10000.0):
    """The rotation of ``rope_3d`` evaluated in float32, the precision of the
    values that become the fine stage's tensor-core operands: each (cos, sin)
    entry is the float64 value of pos * base^(-2j/d_a) rounded to float32,
    and each product and the sum or difference is rounded to float32 on its
    own (numpy float32 arithmetic, no fused multiply-add).  Rounding these
    values to bf16 is a quantisation; taking it from float32 values that the
    kernel reproduces exactly makes the two sides round identically, where
    float64 values would round differently whenever one sits within a float32
    rounding error of a bf16 boundary.  Returns float32 [N, d]."""
    assert sum(dims) == x.shape[-1]
    xf = np.asarray(x, dtype=np.float32)
    y = np.array(xf, copy=True)
    off = 0
    for axis, da in enumerate(dims):
        j = np.arange(da // 2, dtype=np.float64)
        theta = base ** (-2.0 * j / da)
        ang = coords[:, axis:axis + 1].astype(np.float64) * theta[None, :]
        c, s = np.cos(ang).astype(np.float32), np.sin(ang).astype(np.float32)
        x0, x1 = xf[:, off + 0:off + da:2], xf[:, off + 1:off + da:2]
        y[:, off + 0:off + da:2] = (x0 * c) - (x1 * s)
        y[:, off + 1:off + da:2] = (x0 * s) + (x1 * c)
        off += da
    return y


def fine_operands(q, k, grid, dtype, rope=None, pos=None):
    """Tiled q, k as the fine stage consumes them: the inputs as given
    (float64 of the bf16 / float32 values), or with RoPE the float32
    rotation of ``rope_3d_f32``, rounded to bf16 for bf16 workloads."""
    if pos is None:
        pos = positions(grid, "raster")
    if rope is None:
        return to_tiled(q, pos), to_tiled(k, pos)
    coords = token_coords(grid)
    qr = rope_3d_f32(q, coords, rope["dims"], rope["base"]).astype(np.float64)
    kr = rope_3d_f32(k, coords, rope["dims"], rope["base"]).astype(np.float64)
    if dtype == "bf16":
        qr, kr = round_bf16(qr), round_bf16(kr)
    return to_tiled(qr, pos), to_tiled(kr, pos)


def round_bf16(x):
    """Round float64 values to the nearest bf16 value (ties to even)."""
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)                     # x = m * 2^e, 0.5 <= |m| < 1
    scaled = np.ldexp(m, 8)                # 8 significant bits
    r = np.round(scaled)                   # numpy rounds half to even
    return np.ldexp(r, e - 8)


# ----------------------------------------------------------------------------
# prologue: QKV projection fused with the 3D rotary encoding
# ----------------------------------------------------------------------------

def project_qkv(x, w, bias=None):
    """Linear projection of token features to Q | K | V columns.

    x [..., C] float64, w [3*H*d, C] float64 (output rows first, as a linear
    layer stores them), bias [3*H*d] or None.  Returns x @ w^T + bias."""
    y = np.asarray(x, np.float64) @ np.asarray(w, np.float64).T
    if bias is not None:
        y = y + np.asarray(bias, np.float64)
    return y


def qkv_rope(x, w, bias, grid, heads, head_dim, rope=None, t_offset=0,
             order=None, tokens=None, rounded=True, gathered=False):
    """The attention prologue ("Causal-RoPE SP" digest, section 2.3: QKV
    projection and the rotary encoding as one operator; section 2.2: a token
    at local frame t of a block that starts at frame s is encoded at global
    frame t + s).

    x [B, N, C] float64 in natural token order; w [3*H*d, C]; bias or None.
    Output columns o = which*H*d + h*d + j: which 0/1/2 = Q/K/V, head h,
    head dim j.  Q and K of token n are rotated by ``rope_3d`` at
    (t + t_offset, h, w); V is not rotated.  ``rounded`` rounds the results
    once to bf16.  Returns q, k, v [B, H, N, d] in natural order, or in the
    tiled order ``order`` ("raster" / "hilbert") when given.  ``tokens``
    (natural indices) restricts the result to those tokens, returned as
    [B, H, len(tokens), d] in the given order (``order`` must then be None);
    with ``gathered`` x holds only those tokens' rows, [B, len(tokens), C]."""
    x = np.asarray(x, np.float64)
    B = x.shape[0]
    N = grid[0] * grid[1] * grid[2]
    H, d = heads, head_dim
    if gathered and tokens is None:
        raise ValueError("gathered needs tokens")
    if tokens is None:
        tok = np.arange(N)
    else:
        if order is not None:
            raise ValueError("tokens and order are exclusive")
        tok = np.asarray(tokens, np.int64)
    y = project_qkv(x if gathered else x[:, tok, :], w, bias)  # [B, n, 3*H*d]
    y = y.reshape(B, len(tok), 3, H, d).transpose(2, 0, 3, 1, 4)  # [3, B, H, n, d]
    q, k, v = y[0].copy(), y[1].copy(), y[2].copy()
    if rope is not None:
        coords = token_coords(grid)[tok].copy()
        coords[:, 0] += t_offset
        for b in range(B):
            for h in range(H):
                q[b, h] = rope_3d(q[b, h], coords, rope["dims"], rope["base"])
                k[b, h] = rope_3d(k[b, h], coords, rope["dims"], rope["base"])
    if rounded:
        q, k, v = round_bf16(q), round_bf16(k), round_bf16(v)
    if order is not None:
        pos = positions(grid, order)
        q, k, v = to_tiled(q, pos), to_tiled(k, pos), to_tiled(v, pos)
    return q, k, v


def qkv_abs_bound(x, w, bias, heads, head_dim, tokens=None):
    """Sum over the contraction of |x_c * w_oc| (+ |bias_o|) per output, as
    [3, B, H, n, d]: the scale of the rounding error of any summation order
    of the projection (RoPE mixes the two members of a pair, so the bound of a
    rotated pair is the larger of the two)."""
    x = np.abs(np.asarray(x, np.float64))
    if tokens is not None:
        x = x[:, np.asarray(tokens, np.int64), :]
    y = x @ np.abs(np.asarray(w, np.float64)).T
    if bias is not None:
        y = y + np.abs(np.asarray(bias, np.float64))
    B, n, _ = y.shape
    y = y.reshape(B, n, 3, heads, head_dim).transpose(2, 0, 3, 1, 4)
    pair = np.maximum(y[..., 0::2], y[..., 1::2])
    y = y.copy()
    y[..., 0::2] = pair
    y[..., 1::2] = pair
    return y


# ----------------------------------------------------------------------------
# coarse stage: pool, score, softmax, select
# ----------------------------------------------------------------------------

def pool_tiles(x_tiled, tile_tokens=64):
    """Mean of each run of 64 tiled rows: [N, d] -> [nT, d]."""
    N, d = x_tiled.shape
    return np.asarray(x_tiled, np.float64).reshape(N // tile_tokens, tile_tokens, d).mean(axis=1)


def coarse_logits(qp, kp, scale):
    """Pooled coarse logits scale * Qp Kp^T: [nT, nT]."""
    return scale * (qp @ kp.T)


def row_softmax(S):
    s = S - S.max(axis=1, keepdims=True)
    e = np.exp(s)
    return e / e.sum(axis=1, keepdims=True)


def coarse_probabilities(qp, kp, scale):
    """Row softmax of the pooled logits scale * Qp Kp^T: [nT, nT]."""
    return row_softmax(coarse_logits(qp, kp, scale))


BORDER = 1e-5


def select_blocks(S, top_p, k_min):
    """Top-p selection with a k_min floor for each row of the coarse logits
    S [nT, nT] (probabilities P = row softmax of S).

    Tiles are ranked by probability, descending, ties to the lower tile id.
    The ranking is taken on the logits: softmax is monotone in the logit, so
    the order is the same, but tiles whose probability underflows to zero
    keep their true order instead of becoming spurious ties.

    Returns counts [nT], idx [nT, nT] (ascending tile ids, -1 padded) and
    a boolean [nT] marking borderline rows, whose count could change if the
    cumulative masses moved by 1e-5."""
    P = row_softmax(S)
    nT = P.shape[1]
    order = np.argsort(-S, axis=1, kind="stable")       # desc, ties -> lower id
    cum = np.cumsum(np.take_along_axis(P, order, axis=1), axis=1)

    def count_for(p):
        if p >= 1.0:
            return np.full(P.shape[0], nT, np.int64)
        reach = cum >= p
        m = np.where(reach.any(axis=1), reach.argmax(axis=1) + 1, nT)
        return np.minimum(nT, np.maximum(m, max(k_min, 1)))

    counts = count_for(top_p)
    if top_p >= 1.0:
        border = np.zeros(P.shape[0], bool)
    else:
        border = count_for(top_p + BORDER) != count_for(top_p - BORDER)
    idx = np.full(P.shape, -1, np.int64)
    for r in range(P.shape[0]):
        idx[r, :counts[r]] = np.sort(order[r, :counts[r]])
    return counts, idx, border


# ----------------------------------------------------------------------------
# hierarchical (sub-block) scoring
# ----------------------------------------------------------------------------

SUB = (2, 2, 2)


def subblock_ids(coords_tiled, tile=TILE, sub=SUB):
    """Sub-block of every tiled row (0 .. S-1, S = tile/sub per axis product),
    from the token's grid coordinates: raster order of the sub-cube inside its
    tile.  coords_tiled [N, 3] are the (t, h, w) of the tiled rows."""
    per = [t // s for t, s in zip(tile, sub)]
    c = (np.asarray(coords_tiled) % np.array(tile)) // np.array(sub)
    return (c[:, 0] * per[1] + c[:, 1]) * per[2] + c[:, 2]


def pool_subblocks(x_tiled, coords_tiled, tile=TILE, sub=SUB):
    """Mean of each sub-block of each tile: [N, d] -> [nT, S, d]."""
    tsz = tile[0] * tile[1] * tile[2]
    nsub = tsz // (sub[0] * sub[1] * sub[2])
    N, d = x_tiled.shape
    nT = N // tsz
    ids = subblock_ids(coords_tiled, tile, sub)
    x = np.asarray(x_tiled, np.float64)
    out = np.zeros((nT, nsub, d))
    cnt = np.zeros((nT, nsub))
    tiles = np.arange(N) // tsz
    np.add.at(out, (tiles, ids), x)
    np.add.at(cnt, (tiles, ids), 1.0)
    return out / cnt[:, :, None]


def _logsumexp(a, axis):
    m = np.max(a, axis=axis, keepdims=True)
    m = np.where(np.isfinite(m), m, 0.0)
    return np.squeeze(m, axis=axis) + np.log(np.sum(np.exp(a - m), axis=axis))


def subblock_tile_logprob(qs, ks, scale):
    """Tile log-probabilities from sub-block scores: qs [nT, S, d], ks [nT, S, d]
    -> logP [nT, nT] with P[i, j] = (1/S) sum_a sum_b softmax_{(j', b')}(scale *
    qs[i, a] . ks[j', b'])[j, b], evaluated in the log domain."""
    nT, S, d = qs.shape
    L = scale * (qs.reshape(nT * S, d) @ ks.reshape(nT * S, d).T)       # [(i,a), (j,b)]
    L = L.reshape(nT, S, nT, S)
    T = _logsumexp(L, axis=3)                                           # [i, a, j]: mass of key tile j
    Z = _logsumexp(T, axis=2)                                           # [i, a]: row normaliser
    return _logsumexp(T - Z[:, :, None], axis=1) - math.log(S)          # [i, j]


def coarse_head_subblock(q, k, grid, order, top_p, k_min, scale, rope=None, pos=None, sub=SUB):
    """Steps 1-4 for one head with sub-block scoring; q, k [N, d] float64 in
    natural order.  Returns the tile log-probabilities (the ranking key),
    counts, idx, borderline flags and a per-row magnitude of the sub-block
    logits' terms (for the float32 near-tie bound)."""
    if pos is None:
        pos = positions(grid, order)
    coords = token_coords(grid)
    if rope is not None:
        q = rope_3d(q, coords, rope["dims"], rope["base"])
        k = rope_3d(k, coords, rope["dims"], rope["base"])
    qt, kt = to_tiled(q, pos), to_tiled(k, pos)
    ct = to_tiled(coords, pos)
    qs, ks = pool_subblocks(qt, ct, sub=sub), pool_subblocks(kt, ct, sub=sub)
    logP = subblock_tile_logprob(qs, ks, scale)
    counts, idx, border = select_blocks(logP, top_p, k_min)
    nT, S, d = qs.shape
    s_abs = scale * (np.abs(qs.reshape(nT * S, d)) @ np.abs(ks.reshape(nT * S, d)).T)
    s_abs = s_abs.reshape(nT, S, nT, S).max(axis=(1, 2, 3))
    return dict(logP=logP, P=np.exp(logP), counts=counts, idx=idx, border=border,
                qs=qs, ks=ks, s_abs_row=s_abs, pos=pos)


def near_tie_rows(S, counts, tol):
    """Rows whose last kept and first dropped logits differ by at most
    tol[r] (the rounding error a float32 evaluation of the row may carry)."""
    nT = S.shape[1]
    srt = -np.sort(-S, axis=1)
    out = np.zeros(S.shape[0], bool)
    for r in range(S.shape[0]):
        c = counts[r]
        if 0 < c < nT:
            out[r] = srt[r, c - 1] - srt[r, c] <= tol[r]
    return out


# ----------------------------------------------------------------------------
# fine stage
# ----------------------------------------------------------------------------

def fine_tile(q_tile, k_tiled, v_tiled, tiles, scale, tile_tokens=64):
    """Attention of the 64 query rows of one tile over the keys of the given
    key tiles: out [64, d] and lse [64] (natural log)."""
    rows = (np.asarray(tiles)[:, None] * tile_tokens + np.arange(tile_tokens)[None, :]).ravel()
    ks = np.asarray(k_tiled[rows], np.float64)
    vs = np.asarray(v_tiled[rows], np.float64)
    s = scale * (np.asarray(q_tile, np.float64) @ ks.T)
    m = s.max(axis=1, keepdims=True)
    e = np.exp(s - m)
    l = e.sum(axis=1, keepdims=True)
    return (e @ vs) / l, (m + np.log(l))[:, 0]


def fine_head(q_tiled, k_tiled, v_tiled, counts, idx, scale, rows=None, tile_tokens=64):
    """Fine stage of one head in tiled order.  ``rows`` restricts the query
    tiles computed (others are left NaN)."""
    N, d = q_tiled.shape
    out = np.full((N, d), np.nan)
    lse = np.full(N, np.nan)
    nT = N // tile_tokens
    for i in (range(nT) if rows is None else rows):
        sl = slice(i * tile_tokens, (i + 1) * tile_tokens)
        out[sl], lse[sl] = fine_tile(q_tiled[sl], k_tiled, v_tiled,
                                     idx[i, :counts[i]], scale, tile_tokens)
    return out, lse


# ----------------------------------------------------------------------------
# timestep schedule and slack-aware augmentation
# ----------------------------------------------------------------------------

def timestep_params(step, num_steps, p_start, p_end, k_start, k_end, dense_steps=0):
    """(top_p, k_min) for diffusion step ``step`` of ``num_steps`` ("DFSAttn"
    digest, section 3: sparsity is low while the frames are still noise and
    rises as the video sharpens).  The first ``dense_steps`` steps keep every
    tile (top_p = 1); over the remaining steps top_p and k_min move linearly
    from (p_start, k_start) to (p_end, k_end), k_min rounded half up."""
    if step < dense_steps:
        return 1.0, int(k_start)
    span = num_steps - dense_steps - 1
    f = 0.0 if span <= 0 else (step - dense_steps) / span
    f = min(max(f, 0.0), 1.0)
    p = p_start + (p_end - p_start) * f
    k = int(math.floor(k_start + (k_end - k_start) * f + 0.5))
    return p, k


def item_unions(counts, idx, nT):
    """Key-tile union of each work item (query tiles 2q, 2q+1 of one head):
    counts [BH, nT], idx [BH, nT, cap] -> list over items (b*H + h)*P + q of
    sets; the item's cost is max(1, len(set)) (an empty union still takes one
    masked step)."""
    BH = counts.shape[0]
    P = (nT + 1) // 2
    out = []
    for bh in range(BH):
        for q in range(P):
            u = set()
            for r in (2 * q, 2 * q + 1):
                if r < nT:
                    u.update(int(j) for j in idx[bh, r, :counts[bh, r]])
            out.append(u)
    return out


def lpt_order(costs):
    """Items by cost descending, ties by ascending item code."""
    return sorted(range(len(costs)), key=lambda i: (-costs[i], i))


def augment_lists(S, counts, idx, num_ctas, cta_busy_ns=None, fill_percent=100):
    """Slack-aware augmentation on one GPU ("FVAttn" digest, section 02: ranks
    off the critical path spend their spare time on extra, somewhat
    important blocks), with the persistent fine stage's CTAs as the ranks.

    The work list is the longest-first order of the items' union costs; CTA c
    of ``num_ctas`` runs the items at slots c, c + G, ...; its slack is the
    largest CTA load minus its own.  The slack is split evenly over the CTA's
    items (the first ones in slot order take the remainder); an item receives
    that many extra key tiles, at most the tiles outside its union, only if
    one of its rows has a list: the outside tiles with the largest logit max
    over the item's rows with a list (ties to the lower tile), added to each
    of those rows.  S [BH, nT, nT] are the coarse logits.

    With ``cta_busy_ns`` (one measured busy time per CTA, from a run of the
    same work list on the unaugmented lists) a CTA's slack is its measured
    idle time instead, turned into union entries at the run's mean time per
    entry and scaled by ``fill_percent``:
    floor((max busy - busy_c) * total entries * fill / (100 * total busy)),
    in exact integer arithmetic (the spare time the digest's ranks spend is
    time, which entry counts only approximate).

    Returns (counts, idx, extra, worklist): the augmented lists (ascending),
    the tiles added per item, and the work list the fine stage keeps (the
    order of the unaugmented costs)."""
    BH, nT = counts.shape
    P = (nT + 1) // 2
    unions = item_unions(counts, idx, nT)
    costs = [max(1, len(u)) for u in unions]
    order = lpt_order(costs)
    G = max(1, min(num_ctas, len(order)))
    loads = [sum(costs[order[t]] for t in range(c, len(order), G)) for c in range(G)]
    top = max(loads)
    if cta_busy_ns is not None:
        busy = [int(b) for b in cta_busy_ns[:G]]
        total_busy, total_load, top_busy = sum(busy), sum(loads), max(busy)
        slacks = [((top_busy - b) * total_load * int(fill_percent)) // (100 * total_busy) if total_busy > 0 else 0
                  for b in busy]
    else:
        slacks = [top - ld for ld in loads]
    extra = [0] * len(order)
    for c in range(G):
        slots = list(range(c, len(order), G))
        slack, n = slacks[c], len(slots)
        for u, t in enumerate(slots):
            extra[order[t]] = slack // n + (1 if u < slack % n else 0)
    new_counts = counts.copy()
    new_idx = np.zeros((BH, nT, nT), dtype=idx.dtype)
    for bh in range(BH):
        for r in range(nT):
            new_idx[bh, r, :counts[bh, r]] = idx[bh, r, :counts[bh, r]]
    added = [0] * len(order)
    for item in range(len(order)):
        bh, q = divmod(item, P)
        rows = [r for r in (2 * q, 2 * q + 1) if r < nT and counts[bh, r] > 0]
        e = min(extra[item], nT - len(unions[item])) if rows else 0
        if e <= 0:
            continue
        cand = [j for j in range(nT) if j not in unions[item]]
        score = {j: max(S[bh, r, j] for r in rows) for j in cand}
        pick = sorted(cand, key=lambda j: (-score[j], j))[:e]
        added[item] = len(pick)
        for r in rows:
            lst = sorted(set(int(j) for j in idx[bh, r, :counts[bh, r]]) | set(pick))
            new_counts[bh, r] = len(lst)
            new_idx[bh, r, :len(lst)] = lst
    return new_counts, new_idx, added, order


# ----------------------------------------------------------------------------
# backward pass of the fine stage
# ----------------------------------------------------------------------------

def fine_tile_backward(q_tile, k_tiled, v_tiled, do_tile, tiles, scale, tile_tokens=64):
    """Gradients of L = sum(out * dout) for the 64 query rows of one tile
    attending over the tokens of the given key tiles ("VSA" digest, section 3:
    the fine stage is token-level softmax attention inside the selected tiles;
    it is trained end to end, which needs these gradients).

    With s = scale * q k^T, p = softmax_rows(s), out = p v:
      dv = p^T dout,  dp = dout v^T,  ds = p * (dp - rowsum(p * dp)),
      dq = scale * ds k,  dk = scale * ds^T q.
    Returns (dq [64, d], rows, dk [len(rows), d], dv [len(rows), d]) where
    ``rows`` are the key token rows the tile attends to (tiled order)."""
    rows = (np.asarray(tiles)[:, None] * tile_tokens + np.arange(tile_tokens)[None, :]).ravel()
    q = np.asarray(q_tile, np.float64)
    ks = np.asarray(k_tiled[rows], np.float64)
    vs = np.asarray(v_tiled[rows], np.float64)
    g = np.asarray(do_tile, np.float64)
    s = scale * (q @ ks.T)
    e = np.exp(s - s.max(axis=1, keepdims=True))
    p = e / e.sum(axis=1, keepdims=True)
    dv = p.T @ g
    dp = g @ vs.T
    ds = p * (dp - (p * dp).sum(axis=1, keepdims=True))
    return scale * (ds @ ks), rows, scale * (ds.T @ q), dv


def fine_head_backward(q_tiled, k_tiled, v_tiled, do_tiled, counts, idx, scale, tile_tokens=64):
    """dq, dk, dv [N, d] of one head in tiled order: each query tile's
    gradients (``fine_tile_backward``), the key and value parts summed over
    every query tile that selected the key's tile.  A query tile with an empty
    list has zero output and contributes nothing."""
    N, d = q_tiled.shape
    dq = np.zeros((N, d))
    dk = np.zeros((N, d))
    dv = np.zeros((N, d))
    for i in range(N // tile_tokens):
        if counts[i] == 0:
            continue
        sl = slice(i * tile_tokens, (i + 1) * tile_tokens)
        gq, rows, gk, gv = fine_tile_backward(q_tiled[sl], k_tiled, v_tiled, do_tiled[sl],
                                              idx[i, :counts[i]], scale, tile_tokens)
        dq[sl] = gq
        np.add.at(dk, rows, gk)
        np.add.at(dv, rows, gv)
    return dq, dk, dv


def fine_head_backward_scales(q_tiled, k_tiled, v_tiled, do_tiled, out_tiled, counts, idx, scale,
                              tile_tokens=64):
    """Magnitude of the terms behind each gradient element, the scale of the
    rounding error of any evaluation that rounds p and ds to bf16:
    with a_rk = p_rk * (|dp_rk| + sum_c |dout_rc * out_rc|),
      dq: scale * a |k|,  dk: scale * a^T |q|,  dv: p^T |dout|."""
    N, d = q_tiled.shape
    sq = np.zeros((N, d))
    sk = np.zeros((N, d))
    sv = np.zeros((N, d))
    for i in range(N // tile_tokens):
        if counts[i] == 0:
            continue
        sl = slice(i * tile_tokens, (i + 1) * tile_tokens)
        rows = (np.asarray(idx[i, :counts[i]])[:, None] * tile_tokens + np.arange(tile_tokens)[None, :]).ravel()
        q = np.asarray(q_tiled[sl], np.float64)
        ks = np.asarray(k_tiled[rows], np.float64)
        vs = np.asarray(v_tiled[rows], np.float64)
        g = np.asarray(do_tiled[sl], np.float64)
        s = scale * (q @ ks.T)
        e = np.exp(s - s.max(axis=1, keepdims=True))
        p = e / e.sum(axis=1, keepdims=True)
        a = p * (np.abs(g @ vs.T) + np.abs(g * np.asarray(out_tiled[sl], np.float64)).sum(axis=1, keepdims=True))
        sq[sl] = scale * (a @ np.abs(ks))
        np.add.at(sk, rows, scale * (a.T @ np.abs(q)))
        np.add.at(sv, rows, p.T @ np.abs(g))
    return sq, sk, sv


# ----------------------------------------------------------------------------
# whole forward pass
# ----------------------------------------------------------------------------

def as_f64(x, dtype):
    """Input tensor (bf16 bit patterns as uint16, or float32) -> float64."""
    if dtype == "bf16":
        return _bf16_to_f64(x)
    return np.asarray(x, np.float64)


def _bf16_to_f64(x):
    u = np.asarray(x, np.uint16).astype(np.uint32) << np.uint32(16)
    return u.view(np.float32).astype(np.float64)


def default_scale(d):
    return 1.0 / math.sqrt(d)


def coarse_head(q, k, grid, order, top_p, k_min, scale, rope=None, pos=None):
    """Steps 1-4 for one head; q, k [N, d] float64 in natural order.

    Returns a dict with the tiled (and, with RoPE, rotated) q/k, pooled
    Qp/Kp, probabilities, counts, idx and borderline flags."""
    if pos is None:
        pos = positions(grid, order)
    if rope is not None:
        coords = token_coords(grid)
        q = rope_3d(q, coords, rope["dims"], rope["base"])
        k = rope_3d(k, coords, rope["dims"], rope["base"])
    qt, kt = to_tiled(q, pos), to_tiled(k, pos)
    qp, kp = pool_tiles(qt), pool_tiles(kt)
    S = coarse_logits(qp, kp, scale)
    counts, idx, border = select_blocks(S, top_p, k_min)
    # magnitude of the terms of each logit: scale * |Qp| . |Kp|
    s_abs = scale * (np.abs(qp) @ np.abs(kp).T)
    return dict(q_tiled=qt, k_tiled=kt, qp=qp, kp=kp, S=S, P=row_softmax(S), s_abs=s_abs,
                counts=counts, idx=idx, border=border, pos=pos)


def forward_head(q, k, v, grid, order, top_p, k_min, dtype, scale=None,
                 rope=None, blocks=None, rows=None):
    """Whole path for one head, natural order in and out.

    q, k, v: [N, d] as given to the library (bf16 bit patterns or float32).
    ``blocks`` = (counts, idx) reuses a cached selection (steps 2-4 skipped).
    ``rows`` restricts the fine stage to the given query tiles."""
    N, d = q.shape[-2:]
    if scale is None:
        scale = default_scale(d)
    qf, kf, vf = as_f64(q, dtype), as_f64(k, dtype), as_f64(v, dtype)
    pos = positions(grid, order)
    res = {}
    if blocks is None:
        res = coarse_head(qf, kf, grid, order, top_p, k_min, scale, rope, pos)
        counts, idx = res["counts"], res["idx"]
    else:
        counts, idx = blocks
    qt, kt = fine_operands(qf, kf, grid, dtype, rope, pos)
    vt = to_tiled(vf, pos)
    out_t, lse_t = fine_head(qt, kt, vt, counts, idx, scale, rows)
    res.update(out=from_tiled(out_t, pos), lse=lse_t[pos], out_tiled=out_t,
               lse_tiled=lse_t, counts=counts, idx=idx, pos=pos)
    return res


def dense_attention_loop(q, k, v, scale):
    """Independent O(N^2) dense softmax attention with plain Python loops
    (tiny inputs only): out [N, d], lse [N]."""
    N, d = len(q), len(q[0])
    out, lse = [], []
    for i in range(N):
        logits = [scale * sum(q[i][c] * k[j][c] for c in range(d)) for j in range(N)]
        m = max(logits)
        w = [math.exp(x - m) for x in logits]
        z = math.fsum(w)
        out.append([math.fsum(w[j] * v[j][c] for j in range(N)) / z for c in range(d)])
        lse.append(m + math.log(z))
    return out, lse
