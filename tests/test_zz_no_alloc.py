"""fvattn_pool_select_noalloc: the pool/select step for callers that cannot
allocate device memory (for example a plugin whose host application owns
every device allocation and only passes in its tensors).  Its scratch is a
fixed 32 MiB array inside the library instead of a caller workspace.

Checked through the C ABI against fvattn_pool_select on the same inputs, on
two calls in a row (the second call reuses the array the first one left
behind), for bf16 and fp32 inputs with and without RoPE; block lists are
integer results, so the bar is bit-exact.  After each call the status word
of the library's array (fvattn_pool_select_noalloc_status) must read 0.
Kept in a file of its own that pytest collects last."""
import ctypes

import numpy as np
import pytest
import torch

from block_sparse_spatiotemporal_b200 import fvattn as F
from block_sparse_spatiotemporal_b200.inputs import Workload, make_inputs

pytestmark = pytest.mark.gpu


def _dev(x, dtype):
    if dtype == "bf16":
        return torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).cuda()


def _same_lists(c0, i0, c1, i1):
    assert torch.equal(c0, c1)
    c = c0.cpu().numpy()
    a, b = i0.cpu().numpy(), i1.cpu().numpy()
    for bh in np.ndindex(c.shape):
        n = c[bh]
        assert np.array_equal(a[bh][:n], b[bh][:n]), bh


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("rope", [False, True])
def test_noalloc_pool_select_matches_workspace_entry_point(dtype, rope):
    """bf16 and fp32 inputs, with and without the RoPE table in the shared
    array (Hilbert order with RoPE, so the token table is used too)."""
    order = "hilbert" if rope else "raster"
    wl = Workload("noalloc", (8, 16, 24), 4, 128, dtype, 21, 0.9, 2, order, rope, "per_head")
    q, k, _ = make_inputs(wl)
    qd, kd = _dev(q, dtype), _dev(k, dtype)
    shape = F.make_shape(1, wl.heads, wl.head_dim, wl.grid, dtype=F.BF16 if dtype == "bf16" else F.F32,
                         order=F.HILBERT if rope else F.RASTER_CUBE)
    rp = F.make_rope() if rope else None
    assert F.workspace_size(shape, rp) <= 32 << 20
    ws = F.workspace(shape, rp)
    lib = F.lib()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for top_p, k_min in ((0.9, 2), (0.5, 4)):          # two calls in a row
        ref_counts, ref_idx = F.pool_select(shape, qd, kd, ws, top_p, k_min, rope=rp)
        assert F.device_status(ws) == 0
        counts, idx, blocks = F.new_blocks(shape)
        counts.fill_(-7)
        st = lib.fvattn_pool_select_noalloc(ctypes.byref(shape), ctypes.c_void_p(qd.data_ptr()),
                                            ctypes.c_void_p(kd.data_ptr()), ctypes.byref(rp) if rp else None,
                                            top_p, k_min, ctypes.byref(blocks), stream)
        assert st == 0, lib.fvattn_status_string(st)
        status = ctypes.c_int32(-1)
        assert lib.fvattn_pool_select_noalloc_status(stream, ctypes.byref(status)) == 0
        assert status.value == 0
        _same_lists(ref_counts, ref_idx, counts, idx)


def test_noalloc_rejects_shapes_beyond_its_scratch():
    big = F.make_shape(1, 40, 128, (20, 32, 52))         # needs 144 MiB of scratch
    x = torch.zeros(16, dtype=torch.bfloat16, device="cuda")
    _, _, blocks = F.new_blocks(F.make_shape(1, 1, 128, (4, 4, 4)))
    st = F.lib().fvattn_pool_select_noalloc(ctypes.byref(big), ctypes.c_void_p(x.data_ptr()),
                                            ctypes.c_void_p(x.data_ptr()), None, 0.9, 2, ctypes.byref(blocks),
                                            None)
    assert st == -8
