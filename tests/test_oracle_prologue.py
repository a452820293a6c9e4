"""Pins for the oracle's attention prologue (QKV projection fused with the 3D
rotary encoding, "Causal-RoPE SP" digest, sections 2.2-2.3): brute force with
complex-number rotations on a tiny case, identity weights, the start-frame
offset as a shift of the grid, the relative-position invariance of Q.K, pair
norms, and the tiled order."""
import cmath
import math

import numpy as np

from block_sparse_spatiotemporal_b200.inputs import make_projection_inputs
from oracle import fvattn_oracle as O

ROPE = {"dims": (44, 42, 42), "base": 10000.0}


def _inputs(B, N, C, H, seed, bias=True):
    x, w, b = make_projection_inputs(B, N, C, H, 128, seed, bias)
    return O.as_f64(x, "bf16"), O.as_f64(w, "bf16"), (None if b is None else b.astype(np.float64))


def test_brute_force_complex_rotation():
    """Every output of a tiny case from scalar loops: the projection as an
    explicit sum, the rotation as multiplication of the complex number
    y_{2i} + i*y_{2i+1} by exp(i * (pos + offset on the axis) * base^(-2i'/d_a))."""
    grid, B, C, H, d, s = (4, 4, 4), 2, 8, 1, 128, 5
    N = 64
    x, w, b = _inputs(B, N, C, H, 11)
    q, k, v = O.qkv_rope(x, w, b, grid, H, d, ROPE, t_offset=s, rounded=False)
    T, Hg, W = grid
    groups = [(0, 44, 0), (44, 42, 1), (86, 42, 2)]     # (first dim, size, axis)
    for bi in range(B):
        for n in range(N):
            t, rem = divmod(n, Hg * W)
            hh, ww = divmod(rem, W)
            pos = (t + s, hh, ww)
            for which, got in enumerate((q, k, v)):
                y = [math.fsum(x[bi, n, c] * w[which * H * d + j, c] for c in range(C)) + b[which * H * d + j]
                     for j in range(d)]
                if which < 2:
                    r = list(y)
                    for first, size, axis in groups:
                        for i in range(size // 2):
                            z = complex(y[first + 2 * i], y[first + 2 * i + 1])
                            z *= cmath.exp(1j * pos[axis] * 10000.0 ** (-2.0 * i / size))
                            r[first + 2 * i], r[first + 2 * i + 1] = z.real, z.imag
                    y = r
                assert np.allclose(got[bi, 0, n], y, rtol=0, atol=1e-12), (bi, n, which)


def test_identity_weights_split_heads_in_order():
    """C = H*d and W = [I; 2I; 3I]: Q is the rotated input, K twice it, V
    three times the unrotated input, head h = feature columns h*d..h*d+d-1."""
    grid, H, d = (4, 4, 8), 2, 128
    N, C = 128, H * d
    x = np.random.default_rng(3).standard_normal((1, N, C))
    eye = np.eye(C)
    w = np.concatenate([eye, 2 * eye, 3 * eye])
    q, k, v = O.qkv_rope(x, w, None, grid, H, d, ROPE, rounded=False)
    coords = O.token_coords(grid)
    for h in range(H):
        xh = x[0, :, h * d:(h + 1) * d]
        assert np.allclose(v[0, h], 3 * xh, rtol=0, atol=1e-12)
        assert np.allclose(k[0, h], 2 * q[0, h], rtol=0, atol=1e-12)
        assert np.allclose(np.hypot(q[0, h, :, 0::2], q[0, h, :, 1::2]), np.hypot(xh[:, 0::2], xh[:, 1::2]),
                           rtol=0, atol=1e-12)
        # frame 0, row 0, column 0 is at the origin: no rotation
        assert np.allclose(q[0, h, 0], xh[0], rtol=0, atol=0)
        assert not np.allclose(q[0, h, 1:], xh[1:])
    assert (coords[0] == 0).all()


def test_start_frame_offset_is_a_shift_of_the_grid():
    """Block at start frame s of a (T, Hg, W) grid == frames s.. of the
    same tokens placed after s blank frames of a (T + s, Hg, W) grid."""
    T, Hg, W, s = 4, 4, 4, 3
    H, d, C = 1, 128, 16
    x, w, b = _inputs(1, T * Hg * W, C, H, 5)
    blank = np.zeros((1, s * Hg * W, C))
    big = np.concatenate([blank, x], axis=1)
    got = O.qkv_rope(x, w, b, (T, Hg, W), H, d, ROPE, t_offset=s, rounded=False)
    ref = O.qkv_rope(big, w, b, (T + s, Hg, W), H, d, ROPE, t_offset=0, rounded=False)
    for g, r in zip(got, ref):
        assert np.allclose(g, r[:, :, s * Hg * W:], rtol=0, atol=1e-12)
    # and the offset matters
    q0 = O.qkv_rope(x, w, b, (T, Hg, W), H, d, ROPE, t_offset=0, rounded=False)[0]
    assert not np.allclose(q0, got[0])


def test_offset_keeps_qk_dot_products():
    """RoPE encodes relative position: shifting every frame by s leaves
    Q.K between any two tokens unchanged, although Q and K change."""
    grid, H, d, C = (4, 4, 4), 2, 128, 32
    x, w, b = _inputs(1, 64, C, H, 7)
    q0, k0, v0 = O.qkv_rope(x, w, b, grid, H, d, ROPE, t_offset=0, rounded=False)
    q1, k1, v1 = O.qkv_rope(x, w, b, grid, H, d, ROPE, t_offset=17, rounded=False)
    for h in range(H):
        assert np.allclose(q0[0, h] @ k0[0, h].T, q1[0, h] @ k1[0, h].T, rtol=0, atol=1e-9)
    assert not np.allclose(q0, q1)
    assert np.array_equal(v0, v1)


def test_rope_keeps_pair_norms_and_spares_v():
    grid, H, d, C = (4, 8, 4), 2, 128, 64
    x, w, b = _inputs(2, 128, C, H, 9)
    plain = O.qkv_rope(x, w, b, grid, H, d, None, rounded=False)
    rot = O.qkv_rope(x, w, b, grid, H, d, ROPE, t_offset=2, rounded=False)
    for p, r in zip(plain[:2], rot[:2]):
        assert np.allclose(np.hypot(r[..., 0::2], r[..., 1::2]), np.hypot(p[..., 0::2], p[..., 1::2]),
                           rtol=0, atol=1e-12)
    assert np.array_equal(plain[2], rot[2])


def test_tiled_order_token_subset_and_rounding():
    grid, H, d, C = (4, 8, 8), 1, 128, 32
    x, w, b = _inputs(1, 256, C, H, 13)
    nat = O.qkv_rope(x, w, b, grid, H, d, ROPE, t_offset=1)
    for order in ("raster", "hilbert"):
        pos = O.positions(grid, order)
        til = O.qkv_rope(x, w, b, grid, H, d, ROPE, t_offset=1, order=order)
        for a, c in zip(nat, til):
            assert np.array_equal(c[..., pos, :], a)
    toks = np.array([0, 5, 77, 255])
    sub = O.qkv_rope(x, w, b, grid, H, d, ROPE, t_offset=1, tokens=toks)
    gat = O.qkv_rope(x[:, toks], w, b, grid, H, d, ROPE, t_offset=1, tokens=toks, gathered=True)
    for a, c, g in zip(nat, sub, gat):
        assert np.array_equal(c, a[..., toks, :])
        assert np.array_equal(g, c)
    raw = O.qkv_rope(x, w, b, grid, H, d, ROPE, t_offset=1, rounded=False)
    for a, r in zip(nat, raw):
        assert np.array_equal(a, O.round_bf16(r))
        assert np.abs(a - r).max() <= np.abs(r).max() * 2.0 ** -8


def test_abs_bound_bounds_every_output():
    grid, H, d, C = (4, 4, 4), 2, 128, 64
    x, w, b = _inputs(1, 64, C, H, 15)
    raw = O.qkv_rope(x, w, b, grid, H, d, ROPE, t_offset=4, rounded=False)
    bound = O.qkv_abs_bound(x, w, b, H, d)
    for i in range(3):
        assert (np.abs(raw[i]) <= math.sqrt(2.0) * bound[i] * (1 + 1e-12)).all()
