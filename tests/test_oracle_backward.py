"""Pins for the oracle's fine-stage backward pass: central finite differences
of the oracle's own forward, torch autograd (float64) of dense attention when
every tile is selected and of additively masked dense attention for a sparse
selection, and the identities of the softmax gradient (keys' dk sum to zero,
dv sums to the sum of dout)."""
import numpy as np
import torch

from oracle import fvattn_oracle as O


def _case(nT=5, d=32, seed=0, density=0.5):
    rng = np.random.default_rng(seed)
    N = 64 * nT
    q, k, v, g = (rng.standard_normal((N, d)) for _ in range(4))
    counts = np.zeros(nT, np.int64)
    idx = np.zeros((nT, nT), np.int64)
    for i in range(nT):
        sel = np.flatnonzero(rng.random(nT) < density)
        if sel.size == 0:
            sel = np.array([i])
        counts[i] = sel.size
        idx[i, :sel.size] = sel
    return q, k, v, g, counts, idx


def _loss(q, k, v, g, counts, idx, scale):
    out, _ = O.fine_head(q, k, v, counts, idx, scale)
    return float((out * g).sum())


def test_finite_differences():
    q, k, v, g, counts, idx = _case()
    scale = 0.3
    dq, dk, dv = O.fine_head_backward(q, k, v, g, counts, idx, scale)
    rng = np.random.default_rng(9)
    h = 1e-5
    for name, x, grad in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        for _ in range(3):
            dirn = rng.standard_normal(x.shape)
            args = {"q": q, "k": k, "v": v}
            plus = dict(args, **{name: x + h * dirn})
            minus = dict(args, **{name: x - h * dirn})
            fd = (_loss(plus["q"], plus["k"], plus["v"], g, counts, idx, scale)
                  - _loss(minus["q"], minus["k"], minus["v"], g, counts, idx, scale)) / (2 * h)
            an = float((grad * dirn).sum())
            assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (name, fd, an)


def _torch_masked(q, k, v, g, mask, scale):
    qt, kt, vt = (torch.tensor(x, dtype=torch.float64, requires_grad=True) for x in (q, k, v))
    s = scale * qt @ kt.T
    s = s.masked_fill(~torch.tensor(mask), float("-inf"))
    out = torch.softmax(s, dim=-1) @ vt
    (out * torch.tensor(g, dtype=torch.float64)).sum().backward()
    return qt.grad.numpy(), kt.grad.numpy(), vt.grad.numpy()


def test_dense_selection_matches_torch_autograd():
    q, k, v, g, _, _ = _case(nT=3, d=16, seed=1)
    nT = 3
    counts = np.full(nT, nT)
    idx = np.tile(np.arange(nT), (nT, 1))
    scale = 1 / 4
    got = O.fine_head_backward(q, k, v, g, counts, idx, scale)
    qt, kt, vt = (torch.tensor(x, dtype=torch.float64, requires_grad=True) for x in (q, k, v))
    out = torch.nn.functional.scaled_dot_product_attention(qt[None], kt[None], vt[None], scale=scale)[0]
    (out * torch.tensor(g)).sum().backward()
    for a, b in zip(got, (qt.grad, kt.grad, vt.grad)):
        assert np.allclose(a, b.numpy(), rtol=0, atol=1e-10)


def test_sparse_selection_matches_masked_dense_autograd():
    q, k, v, g, counts, idx = _case(nT=6, d=24, seed=2, density=0.4)
    scale = 0.2
    N = q.shape[0]
    mask = np.zeros((N, N), bool)
    for i in range(6):
        for j in idx[i, :counts[i]]:
            mask[64 * i:64 * i + 64, 64 * j:64 * j + 64] = True
    got = O.fine_head_backward(q, k, v, g, counts, idx, scale)
    ref = _torch_masked(q, k, v, g, mask, scale)
    for a, b in zip(got, ref):
        assert np.allclose(a, b, rtol=0, atol=1e-10)


def test_softmax_gradient_identities():
    """Shifting every key by one vector leaves each row's softmax unchanged,
    so the dk of all keys sums to zero; each row's probabilities sum to one,
    so the dv of all keys sums to the sum of dout over rows with a list."""
    q, k, v, g, counts, idx = _case(nT=6, d=16, seed=3)
    counts[2] = 0                             # an empty row contributes nothing
    dq, dk, dv = O.fine_head_backward(q, k, v, g, counts, idx, 0.5)
    assert np.allclose(dk.sum(axis=0), 0, atol=1e-10)
    live = np.repeat(counts > 0, 64)
    assert np.allclose(dv.sum(axis=0), g[live].sum(axis=0), atol=1e-10)
    assert not dq[128:192].any()


def test_error_scales_bound_the_gradients():
    q, k, v, g, counts, idx = _case(nT=4, d=16, seed=4)
    out, _ = O.fine_head(q, k, v, counts, idx, 0.5)
    grads = O.fine_head_backward(q, k, v, g, counts, idx, 0.5)
    scales = O.fine_head_backward_scales(q, k, v, g, out, counts, idx, 0.5)
    for a, sc in zip(grads, scales):
        assert (np.abs(a) <= sc * (1 + 1e-12) + 1e-15).all()
