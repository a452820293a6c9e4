"""Seeded synthetic inputs for adaptive block-sparse 3D video attention.

This module is the only code shared by the CPU oracle and the CUDA path, and it
holds none of the method's arithmetic: it draws Q, K and V tensors with the
shape and structure of the workloads the pages describe (video-DiT latents
with spatially local attention), and nothing else.

The pages measure on real Wan / Mochi activations ("FVAttn" page, section 03;
"CalibAtt" page, "Demonstrated performance"), which are not available here.
These tensors stand in for them.

Recipe (numpy generators; every stream is seeded, so the tensors do not
depend on the number of threads that draw them):

1. Head parameters, from ``default_rng(seed)`` in this order, head by head:
   a. concentration s_h and bandwidth sigma_h: fixed (s=3, sigma=0.15) for
      the "fixed" generator, else s_h = exp(U[log 1, log 6]) then
      sigma_h = U[0.05, 0.3];
   b. frequencies omega_h, shape [D, 3], drawn N(0, 1/sigma_h^2) (D = d);
   c. phases b_h, shape [D], drawn U[0, 2*pi);
   d. with sinks: 2 distinct sink tiles, ``choice(nT, 2, replace=False)``
      over raster-cube tile ids.
2. Noise: tensor t (0 = Q noise, 1 = K noise, 2 = V) of head h of batch b is
   [N, d] standard normal (float32) from
   ``default_rng(SeedSequence([seed, 1 + t, b, h]))``.
3. phi(x)_j = cos(omega_j . x + b_j) with x = (t, h, w) / max(extent - 1, 1)
   the normalised coordinate of the token (unnormalised features, so that
   logits are large and attention is spatially local).
4. Q = s_h * phi + 0.3 * Qnoise,  K = s_h * phi + 0.3 * Knoise.
5. Sinks: every K row of a sink tile is multiplied by 3.
6. bf16 workloads are rounded to bf16 (round to nearest even); fp32 ones
   stay float32.

Perturbed steps for the cached-mask mode: Q_t = Q_{t-1} + 0.05 * N(0,1) and
K_t likewise (cumulative over t, float32 masters), V fixed; the noise of
step t, tensor t' (0 = Q, 1 = K), head h comes from
``default_rng(SeedSequence([seed, 100 + t, t', b, h]))``; each step is
rounded to bf16 on its own.

Token layout: natural order is raster order over the latent grid (T, Hg, W),
index n = (t * Hg + h) * W + w, tensors are [B, H, N, d] with B = 1.

Prologue inputs (the QKV projection before attention): token features
X [B, N, C] ~ N(0, 1) (the scale of normalised DiT activations), weights
W [3*H*d, C] ~ N(0, 1/C) (fan-in initialisation, so projected values are
about N(0, 1)) and bias [3*H*d] ~ N(0, 0.1^2), all rounded to bf16 except the
float32 bias.  X rows are drawn in chunks of 4096 tokens, chunk c of batch b
from ``default_rng(SeedSequence([seed, 200, b, c]))``; W and bias from
``default_rng(SeedSequence([seed, 201]))`` and ``[seed, 202]``.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

__all__ = ["Workload", "WORKLOADS", "make_inputs", "perturb_steps",
           "f32_to_bf16_bits", "bf16_bits_to_f32", "sweep_points",
           "make_projection_inputs"]


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic workload: latent grid, heads, dtype and routing knobs."""
    name: str
    grid: tuple          # (T, Hg, W) latent tokens
    heads: int
    head_dim: int
    dtype: str           # "f32" or "bf16"
    seed: int
    top_p: float
    k_min: int
    order: str           # "raster" or "hilbert"
    rope: bool
    generator: str       # "fixed" (s=3, sigma=0.15) or "per_head" (+ 2 sinks)
    batch: int = 1
    tile: tuple = (4, 4, 4)
    rope_dims: tuple = (44, 42, 42)
    rope_base: float = 10000.0

    @property
    def tokens(self) -> int:
        T, Hg, W = self.grid
        return T * Hg * W

    @property
    def num_tiles(self) -> int:
        return self.tokens // (self.tile[0] * self.tile[1] * self.tile[2])


WORKLOADS = {
    "tiny_fp32": Workload("tiny_fp32", (8, 16, 16), 2, 64, "f32", 0, 0.9, 2,
                          "raster", False, "fixed"),
    "grid16k": Workload("grid16k", (16, 32, 32), 12, 128, "bf16", 1, 0.9, 4,
                        "raster", False, "fixed"),
    "wan480p": Workload("wan480p", (20, 32, 52), 40, 128, "bf16", 2, 0.95, 8,
                        "raster", False, "per_head"),
    "wan720p_hilbert_rope": Workload("wan720p_hilbert_rope", (20, 48, 80), 40,
                                     128, "bf16", 3, 0.95, 8, "hilbert", True,
                                     "per_head"),
    "wan480p_sweep": Workload("wan480p_sweep", (20, 32, 52), 40, 128, "bf16",
                              4, 0.95, 8, "raster", False, "per_head"),
}


def sweep_points():
    """(top_p, k_min) points of the 480p sweep: top-p values with k_min=8,
    then fixed top-k (top_p = 0, k_min = k)."""
    pts = [(p, 8) for p in (0.5, 0.8, 0.9, 0.95, 0.99, 1.0)]
    pts += [(0.0, k) for k in (8, 32, 128)]
    return pts


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (nearest even); returns uint16 bit patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    bias = np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))
    return ((u + bias) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns (uint16) to float32 exactly."""
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32)
            << np.uint32(16)).view(np.float32)


def _coords(grid):
    T, Hg, W = grid
    t, h, w = np.meshgrid(np.arange(T), np.arange(Hg), np.arange(W), indexing="ij")
    return np.stack([t.ravel(), h.ravel(), w.ravel()], axis=1)


def _head_params(rng, wl: Workload):
    D = wl.head_dim
    params = []
    for _ in range(wl.heads):
        if wl.generator == "per_head":
            s = math.exp(rng.uniform(math.log(1.0), math.log(6.0)))
            sigma = rng.uniform(0.05, 0.3)
        else:
            s, sigma = 3.0, 0.15
        omega = rng.normal(0.0, 1.0 / sigma, size=(D, 3))
        phase = rng.uniform(0.0, 2.0 * math.pi, size=D)
        sinks = None
        if wl.generator == "per_head":
            sinks = rng.choice(wl.num_tiles, 2, replace=False)
        params.append((s, sigma, omega, phase, sinks))
    return params


def _sink_rows(wl: Workload, tile_ids):
    """Natural token indices of the given raster-cube tile ids."""
    T, Hg, W = wl.grid
    tt, th, tw = wl.tile
    nh, nw = Hg // th, W // tw
    rows = []
    for tid in tile_ids:
        ct, rem = divmod(int(tid), nh * nw)
        ch, cw = divmod(rem, nw)
        t, h, w = np.meshgrid(np.arange(ct * tt, ct * tt + tt),
                              np.arange(ch * th, ch * th + th),
                              np.arange(cw * tw, cw * tw + tw), indexing="ij")
        rows.append(((t * Hg + h) * W + w).ravel())
    return np.concatenate(rows)


def _finish(x32, wl):
    return f32_to_bf16_bits(x32) if wl.dtype == "bf16" else x32.astype(np.float32)


def _noise(seed_words, shape):
    return np.random.default_rng(np.random.SeedSequence(seed_words)).standard_normal(shape, dtype=np.float32)


def _parallel(fn, items):
    import concurrent.futures
    import os
    workers = max(1, min(len(items), os.cpu_count() or 1))
    with concurrent.futures.ThreadPoolExecutor(workers) as ex:
        list(ex.map(fn, items))


def make_inputs(wl: Workload, keep_f32_masters: bool = False):
    """Draw (q, k, v) for a workload, shapes [B, H, N, d].

    bf16 workloads return uint16 arrays of bf16 bit patterns, fp32 workloads
    float32 arrays.  With ``keep_f32_masters`` the float32 Q/K before rounding
    are returned too (for the perturbed steps)."""
    rng = np.random.default_rng(wl.seed)
    params = _head_params(rng, wl)
    T, Hg, W = wl.grid
    N, d, H, B = wl.tokens, wl.head_dim, wl.heads, wl.batch
    x = _coords(wl.grid).astype(np.float64)
    x /= np.maximum(np.array([T, Hg, W], dtype=np.float64) - 1.0, 1.0)

    out_dtype = np.uint16 if wl.dtype == "bf16" else np.float32
    q = np.empty((B, H, N, d), out_dtype)
    k = np.empty((B, H, N, d), out_dtype)
    v = np.empty((B, H, N, d), out_dtype)
    qm = np.empty((B, H, N, d), np.float32) if keep_f32_masters else None
    km = np.empty((B, H, N, d), np.float32) if keep_f32_masters else None
    sink_rows = [None if p[4] is None else _sink_rows(wl, p[4]) for p in params]

    def one(bh):
        b, h = bh
        s, _, omega, phase, _ = params[h]
        phi = (s * np.cos(x @ omega.T + phase)).astype(np.float32)
        qh = phi + np.float32(0.3) * _noise([wl.seed, 1, b, h], (N, d))
        kh = phi + np.float32(0.3) * _noise([wl.seed, 2, b, h], (N, d))
        if sink_rows[h] is not None:
            kh[sink_rows[h]] *= np.float32(3.0)
        if keep_f32_masters:
            qm[b, h] = qh
            km[b, h] = kh
        q[b, h] = _finish(qh, wl)
        k[b, h] = _finish(kh, wl)
        v[b, h] = _finish(_noise([wl.seed, 3, b, h], (N, d)), wl)

    _parallel(one, [(b, h) for b in range(B) for h in range(H)])
    if keep_f32_masters:
        return q, k, v, dict(q_f32=qm, k_f32=km)
    return q, k, v


def perturb_steps(wl: Workload, masters: dict, steps: int = 10):
    """Yield (q_t, k_t) for t = 1..steps: cumulative 0.05*N(0,1) perturbation
    of the float32 masters returned by ``make_inputs(..., keep_f32_masters=True)``."""
    qm = masters["q_f32"].copy()
    km = masters["k_f32"].copy()
    B, H, N, d = qm.shape
    for t in range(1, steps + 1):
        def one(bh, t=t):
            b, h = bh
            qm[b, h] += np.float32(0.05) * _noise([wl.seed, 100 + t, 0, b, h], (N, d))
            km[b, h] += np.float32(0.05) * _noise([wl.seed, 100 + t, 1, b, h], (N, d))
        _parallel(one, [(b, h) for b in range(B) for h in range(H)])
        yield _finish(qm, wl), _finish(km, wl)


def make_projection_inputs(batch: int, tokens: int, channels: int, heads: int, head_dim: int,
                           seed: int, bias: bool = True):
    """Draw (x, w, b) for the QKV projection: x [B, N, C] and w [3*H*d, C] as
    bf16 bit patterns (uint16), b [3*H*d] float32 or None."""
    chunk = 4096
    x = np.empty((batch, tokens, channels), np.uint16)

    def one(item):
        b, c = item
        lo, hi = c * chunk, min(tokens, (c + 1) * chunk)
        x[b, lo:hi] = f32_to_bf16_bits(_noise([seed, 200, b, c], (hi - lo, channels)))

    _parallel(one, [(b, c) for b in range(batch) for c in range((tokens + chunk - 1) // chunk)])
    rows = 3 * heads * head_dim
    w32 = _noise([seed, 201], (rows, channels)) * np.float32(1.0 / math.sqrt(channels))
    w = f32_to_bf16_bits(w32)
    bv = (_noise([seed, 202], (rows,)) * np.float32(0.1)).astype(np.float32) if bias else None
    return x, w, bv
