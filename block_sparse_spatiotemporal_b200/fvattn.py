"""Thin Python binding of libfvattn.so (argument marshalling only).

Every step of the path runs in the library's CUDA kernels; this module only
builds the C structs, passes torch device pointers and the current CUDA
stream, and turns status codes into exceptions.  There is no fallback: if
the library is missing or the device is not an sm_100 GPU, calls raise.

Names follow the C ABI in include/fvattn.h.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

__all__ = [
    "FvattnError", "Shape", "Rope", "Blocks", "MaskCache", "lib", "library_path",
    "F32", "BF16", "RASTER_CUBE", "HILBERT", "NATURAL", "TILED",
    "make_shape", "make_rope", "num_tiles", "workspace_size", "workspace", "workspace_size_subblock",
    "pool_select_subblock",
    "tile_reorder", "pool_select", "build_worklist", "block_sparse_fwd", "forward",
    "device_status", "selftest_wait_timeout", "new_blocks", "new_cache", "profile_enable", "profile_read",
    "STAGES", "pool_select_noalloc", "noalloc_status", "profile_cta_times", "workspace_size_qkv", "qkv_rope", "workspace_size_bwd", "block_sparse_bwd",
    "augment_lists", "block_sparse_fwd_worklist", "timestep_params",
]

F32, BF16 = 0, 1
RASTER_CUBE, HILBERT = 0, 1
NATURAL, TILED = 0, 1

_HERE = os.path.dirname(os.path.abspath(__file__))


def library_path() -> str:
    return os.path.join(_HERE, "libfvattn.so")


class FvattnError(RuntimeError):
    def __init__(self, fn: str, status: int):
        msg = lib().fvattn_status_string(status).decode()
        super().__init__(f"{fn} failed with status {status}: {msg}")
        self.status = status


class Dims(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int32), ("H", ctypes.c_int32), ("W", ctypes.c_int32)]


class Tile(ctypes.Structure):
    _fields_ = [("t", ctypes.c_int32), ("h", ctypes.c_int32), ("w", ctypes.c_int32)]


class Rope(ctypes.Structure):
    _fields_ = [("enabled", ctypes.c_int32), ("dt", ctypes.c_int32), ("dh", ctypes.c_int32),
                ("dw", ctypes.c_int32), ("base", ctypes.c_float)]


class Shape(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("grid", Dims), ("tile", Tile), ("dtype", ctypes.c_int), ("order", ctypes.c_int),
                ("layout", ctypes.c_int), ("scale", ctypes.c_float)]


class Blocks(ctypes.Structure):
    _fields_ = [("counts", ctypes.c_void_p), ("idx", ctypes.c_void_p), ("cap", ctypes.c_int32)]


class MaskCache(ctypes.Structure):
    _fields_ = [("blocks", Blocks), ("shape", Shape), ("top_p", ctypes.c_float),
                ("k_min", ctypes.c_int32), ("valid", ctypes.c_int32)]


_LIB = None

_SIGS = {
    "fvattn_num_tiles": [ctypes.POINTER(Shape), ctypes.POINTER(ctypes.c_int64)],
    "fvattn_workspace_size": [ctypes.POINTER(Shape), ctypes.POINTER(Rope), ctypes.POINTER(ctypes.c_size_t)],
    "fvattn_tile_reorder": [ctypes.POINTER(Shape), ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int32,
                            ctypes.c_int, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p],
    "fvattn_pool_select": [ctypes.POINTER(Shape), ctypes.c_void_p, ctypes.c_void_p, ctypes.POINTER(Rope),
                           ctypes.c_float, ctypes.c_int32, ctypes.POINTER(Blocks), ctypes.c_void_p,
                           ctypes.c_size_t, ctypes.c_void_p],
    "fvattn_workspace_size_subblock": [ctypes.POINTER(Shape), ctypes.POINTER(Rope), ctypes.POINTER(ctypes.c_size_t)],
    "fvattn_pool_select_subblock": [ctypes.POINTER(Shape), ctypes.c_void_p, ctypes.c_void_p, ctypes.POINTER(Rope),
                                    ctypes.c_float, ctypes.c_int32, ctypes.POINTER(Blocks), ctypes.c_void_p,
                                    ctypes.c_size_t, ctypes.c_void_p],
    "fvattn_pool_select_noalloc": [ctypes.POINTER(Shape), ctypes.c_void_p, ctypes.c_void_p, ctypes.POINTER(Rope),
                                   ctypes.c_float, ctypes.c_int32, ctypes.POINTER(Blocks), ctypes.c_void_p],
    "fvattn_pool_select_noalloc_status": [ctypes.c_void_p, ctypes.POINTER(ctypes.c_int32)],
    "fvattn_profile_cta_times": [ctypes.POINTER(Shape), ctypes.POINTER(Rope), ctypes.c_void_p, ctypes.c_void_p,
                                 ctypes.POINTER(ctypes.c_int64), ctypes.c_int32, ctypes.POINTER(ctypes.c_int32)],
    "fvattn_build_worklist": [ctypes.POINTER(Shape), ctypes.POINTER(Blocks), ctypes.c_void_p, ctypes.c_void_p,
                              ctypes.c_size_t, ctypes.c_void_p],
    "fvattn_block_sparse_fwd": [ctypes.POINTER(Shape), ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                ctypes.POINTER(Rope), ctypes.POINTER(Blocks), ctypes.c_void_p, ctypes.c_void_p,
                                ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p],
    "fvattn_forward": [ctypes.POINTER(Shape), ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                       ctypes.POINTER(Rope), ctypes.c_float, ctypes.c_int32, ctypes.POINTER(MaskCache),
                       ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t,
                       ctypes.c_void_p],
    "fvattn_augment_lists": [ctypes.POINTER(Shape), ctypes.c_void_p, ctypes.c_void_p, ctypes.POINTER(Rope),
                             ctypes.POINTER(Blocks), ctypes.c_int32, ctypes.c_void_p, ctypes.c_int32,
                             ctypes.POINTER(Blocks), ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t,
                             ctypes.c_void_p],
    "fvattn_block_sparse_fwd_worklist": [ctypes.POINTER(Shape), ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                         ctypes.POINTER(Rope), ctypes.POINTER(Blocks), ctypes.c_void_p,
                                         ctypes.c_int32, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                         ctypes.c_size_t, ctypes.c_void_p],
    "fvattn_timestep_params": [ctypes.c_int32, ctypes.c_int32, ctypes.c_float, ctypes.c_float, ctypes.c_int32,
                               ctypes.c_int32, ctypes.c_int32, ctypes.POINTER(ctypes.c_float),
                               ctypes.POINTER(ctypes.c_int32)],
    "fvattn_workspace_size_bwd": [ctypes.POINTER(Shape), ctypes.POINTER(ctypes.c_size_t)],
    "fvattn_block_sparse_bwd": [ctypes.POINTER(Shape), ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.POINTER(Blocks),
                                ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t,
                                ctypes.c_void_p],
    "fvattn_workspace_size_qkv": [ctypes.POINTER(Shape), ctypes.POINTER(Rope), ctypes.POINTER(ctypes.c_size_t)],
    "fvattn_qkv_rope": [ctypes.POINTER(Shape), ctypes.c_void_p, ctypes.c_int32, ctypes.c_void_p, ctypes.c_void_p,
                        ctypes.POINTER(Rope), ctypes.c_int32, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                        ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p],
    "fvattn_get_device_status": [ctypes.c_void_p, ctypes.c_void_p, ctypes.POINTER(ctypes.c_int32)],
    "fvattn_selftest_wait_timeout": [ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int64, ctypes.c_void_p],
    "fvattn_profile_enable": [ctypes.c_int],
    "fvattn_profile_read": [ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_int64)],
    "fvattn_status_string": [ctypes.c_int],
}

STAGES = ("tables", "reorder", "pool", "select", "schedule", "fine", "prologue", "bwd_prep", "bwd_kv", "bwd_q")


def lib():
    """Load libfvattn.so (raises if it has not been built)."""
    global _LIB
    if _LIB is None:
        path = library_path()
        if not os.path.exists(path):
            raise RuntimeError(f"{path} is missing: build it with `python -m block_sparse_spatiotemporal_b200.build`")
        h = ctypes.CDLL(path)
        for name, args in _SIGS.items():
            fn = getattr(h, name)
            fn.argtypes = args
            fn.restype = ctypes.c_char_p if name == "fvattn_status_string" else ctypes.c_int
        _LIB = h
    return _LIB


def _check(fn: str, status: int):
    if status != 0:
        raise FvattnError(fn, status)


def _stream(stream: Optional[torch.cuda.Stream]):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return ctypes.c_void_p(t.data_ptr())


def make_shape(batch, heads, head_dim, grid, dtype=BF16, order=RASTER_CUBE, layout=NATURAL, scale=0.0) -> Shape:
    T, Hg, W = grid
    return Shape(batch, heads, head_dim, Dims(T, Hg, W), Tile(4, 4, 4), dtype, order, layout, float(scale))


def make_rope(dims=(44, 42, 42), base=10000.0, enabled=True) -> Rope:
    return Rope(1 if enabled else 0, dims[0], dims[1], dims[2], float(base))


def _rope_ptr(rope: Optional[Rope]):
    return ctypes.byref(rope) if rope is not None else None


def num_tiles(shape: Shape) -> int:
    n = ctypes.c_int64()
    _check("fvattn_num_tiles", lib().fvattn_num_tiles(ctypes.byref(shape), ctypes.byref(n)))
    return n.value


def workspace_size(shape: Shape, rope: Optional[Rope] = None) -> int:
    n = ctypes.c_size_t()
    _check("fvattn_workspace_size", lib().fvattn_workspace_size(ctypes.byref(shape), _rope_ptr(rope), ctypes.byref(n)))
    return n.value


def workspace(shape: Shape, rope: Optional[Rope] = None, device="cuda", subblock=False) -> torch.Tensor:
    """A device workspace of the size the library asks for (caller-owned);
    ``subblock`` sizes it for pool_select_subblock as well."""
    n = workspace_size_subblock(shape, rope) if subblock else workspace_size(shape, rope)
    return torch.empty(n, dtype=torch.uint8, device=device)


def workspace_size_subblock(shape: Shape, rope: Optional[Rope] = None) -> int:
    n = ctypes.c_size_t()
    _check("fvattn_workspace_size_subblock",
           lib().fvattn_workspace_size_subblock(ctypes.byref(shape), _rope_ptr(rope), ctypes.byref(n)))
    return n.value


def new_blocks(shape: Shape, device="cuda"):
    """Caller-owned block-list buffers: (counts [B,H,nT], idx [B,H,nT,nT], Blocks)."""
    nT = num_tiles(shape)
    counts = torch.empty((shape.batch, shape.heads, nT), dtype=torch.int32, device=device)
    idx = torch.empty((shape.batch, shape.heads, nT, nT), dtype=torch.int32, device=device)
    return counts, idx, Blocks(counts.data_ptr(), idx.data_ptr(), nT)


def new_cache(shape: Shape, device="cuda"):
    """A mask cache with its own block buffers: (cache, counts, idx)."""
    counts, idx, blocks = new_blocks(shape, device)
    cache = MaskCache()
    cache.blocks = blocks
    cache.valid = 0
    return cache, counts, idx


def tile_reorder(shape: Shape, x: torch.Tensor, ws: torch.Tensor, inverse=False, out=None, stream=None):
    """Permute token rows of x [B,H,N,...] between natural and tiled layout."""
    y = torch.empty_like(x) if out is None else out
    row_bytes = x[0, 0, 0].numel() * x.element_size() if x.dim() == 4 else x.element_size()
    _check("fvattn_tile_reorder", lib().fvattn_tile_reorder(ctypes.byref(shape), _ptr(x), _ptr(y), row_bytes,
                                                            1 if inverse else 0, _ptr(ws), ws.numel(),
                                                            _stream(stream)))
    return y


def pool_select(shape: Shape, q, k, ws, top_p: float, k_min: int, rope: Optional[Rope] = None, blocks=None,
                stream=None):
    """Steps 2-5: returns (counts, idx) int32 device tensors."""
    if blocks is None:
        counts, idx, b = new_blocks(shape, q.device)
    else:
        counts, idx, b = blocks
    _check("fvattn_pool_select", lib().fvattn_pool_select(ctypes.byref(shape), _ptr(q), _ptr(k), _rope_ptr(rope),
                                                          float(top_p), int(k_min), ctypes.byref(b), _ptr(ws),
                                                          ws.numel(), _stream(stream)))
    return counts, idx


def pool_select_subblock(shape: Shape, q, k, ws, top_p: float, k_min: int, rope: Optional[Rope] = None,
                         blocks=None, stream=None):
    """Steps 2-5 with hierarchical sub-block scoring (ws from
    ``workspace(..., subblock=True)``): returns (counts, idx)."""
    if blocks is None:
        counts, idx, b = new_blocks(shape, q.device)
    else:
        counts, idx, b = blocks
    _check("fvattn_pool_select_subblock",
           lib().fvattn_pool_select_subblock(ctypes.byref(shape), _ptr(q), _ptr(k), _rope_ptr(rope), float(top_p),
                                             int(k_min), ctypes.byref(b), _ptr(ws), ws.numel(), _stream(stream)))
    return counts, idx


def pool_select_noalloc(shape: Shape, q, k, top_p: float, k_min: int, rope: Optional[Rope] = None, blocks=None,
                        stream=None):
    """Steps 2-5 with the library's static scratch instead of a workspace
    (for callers that cannot allocate); returns (counts, idx)."""
    if blocks is None:
        counts, idx, b = new_blocks(shape, q.device)
    else:
        counts, idx, b = blocks
    _check("fvattn_pool_select_noalloc",
           lib().fvattn_pool_select_noalloc(ctypes.byref(shape), _ptr(q), _ptr(k), _rope_ptr(rope), float(top_p),
                                            int(k_min), ctypes.byref(b), _stream(stream)))
    return counts, idx


def noalloc_status(stream=None) -> int:
    """Read and clear the device status word of pool_select_noalloc
    (synchronises the stream)."""
    v = ctypes.c_int32(0)
    _check("fvattn_pool_select_noalloc_status", lib().fvattn_pool_select_noalloc_status(_stream(stream),
                                                                                       ctypes.byref(v)))
    return int(v.value)


def _blocks_of(counts, idx):
    return Blocks(counts.data_ptr(), idx.data_ptr(), idx.shape[-1])


def build_worklist(shape: Shape, counts, idx, ws, stream=None):
    P = (num_tiles(shape) + 1) // 2
    wl = torch.empty(shape.batch * shape.heads * P, dtype=torch.int32, device=counts.device)
    b = _blocks_of(counts, idx)
    _check("fvattn_build_worklist", lib().fvattn_build_worklist(ctypes.byref(shape), ctypes.byref(b), _ptr(wl),
                                                                _ptr(ws), ws.numel(), _stream(stream)))
    return wl


def block_sparse_fwd(shape: Shape, q, k, v, counts, idx, ws, rope: Optional[Rope] = None, out=None, lse=None,
                     stream=None):
    """Step 6: returns (out, lse) in shape.layout."""
    out = torch.empty_like(q) if out is None else out
    if lse is None:
        lse = torch.empty(q.shape[:-1], dtype=torch.float32, device=q.device)
    b = _blocks_of(counts, idx)
    _check("fvattn_block_sparse_fwd",
           lib().fvattn_block_sparse_fwd(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _rope_ptr(rope),
                                         ctypes.byref(b), _ptr(out), _ptr(lse), _ptr(ws), ws.numel(),
                                         _stream(stream)))
    return out, lse


def forward(shape: Shape, q, k, v, ws, top_p: float, k_min: int, rope: Optional[Rope] = None,
            cache: Optional[MaskCache] = None, reuse_mask=False, out=None, lse=None, stream=None):
    """Whole path on natural-layout tensors: returns (out, lse)."""
    out = torch.empty_like(q) if out is None else out
    if lse is None:
        lse = torch.empty(q.shape[:-1], dtype=torch.float32, device=q.device)
    _check("fvattn_forward",
           lib().fvattn_forward(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _rope_ptr(rope), float(top_p),
                                int(k_min), ctypes.byref(cache) if cache is not None else None,
                                1 if reuse_mask else 0, _ptr(out), _ptr(lse), _ptr(ws), ws.numel(),
                                _stream(stream)))
    return out, lse


def augment_lists(shape: Shape, q, k, ws, counts, idx, num_ctas: int = 0, rope: Optional[Rope] = None, out=None,
                  stream=None, cta_busy_ns=None, fill_percent: int = 100):
    """Slack-aware augmentation of (counts, idx): returns (counts, idx,
    worklist) -- the augmented lists and the work list to run them with.
    cta_busy_ns: None, or one measured busy time (ns) per CTA of a run of the
    same work list on the unaugmented lists (a host sequence of ints)."""
    if out is None:
        oc, oi, ob = new_blocks(shape, q.device)
    else:
        oc, oi = out
        ob = _blocks_of(oc, oi)
    wl = torch.empty(shape.batch * shape.heads * ((num_tiles(shape) + 1) // 2), dtype=torch.int32, device=q.device)
    base = _blocks_of(counts, idx)
    busy = None
    if cta_busy_ns is not None:
        vals = [int(x) for x in cta_busy_ns]
        busy = (ctypes.c_int64 * max(1, len(vals)))(*vals)
    _check("fvattn_augment_lists",
           lib().fvattn_augment_lists(ctypes.byref(shape), _ptr(q), _ptr(k), _rope_ptr(rope), ctypes.byref(base),
                                      int(num_ctas), busy, int(fill_percent), ctypes.byref(ob), _ptr(wl), _ptr(ws),
                                      ws.numel(), _stream(stream)))
    return oc, oi, wl


def block_sparse_fwd_worklist(shape: Shape, q, k, v, counts, idx, worklist, ws, num_ctas: int = 0,
                              rope: Optional[Rope] = None, out=None, lse=None, stream=None):
    """Step 6 with a given work list and persistent grid: returns (out, lse)."""
    out = torch.empty_like(q) if out is None else out
    if lse is None:
        lse = torch.empty(q.shape[:-1], dtype=torch.float32, device=q.device)
    b = _blocks_of(counts, idx)
    _check("fvattn_block_sparse_fwd_worklist",
           lib().fvattn_block_sparse_fwd_worklist(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _rope_ptr(rope),
                                                  ctypes.byref(b), _ptr(worklist), int(num_ctas), _ptr(out),
                                                  _ptr(lse), _ptr(ws), ws.numel(), _stream(stream)))
    return out, lse


def timestep_params(step: int, num_steps: int, p_start: float, p_end: float, k_start: int, k_end: int,
                    dense_steps: int = 0):
    """(top_p, k_min) of a diffusion step (host arithmetic in the library)."""
    p = ctypes.c_float()
    km = ctypes.c_int32()
    _check("fvattn_timestep_params",
           lib().fvattn_timestep_params(int(step), int(num_steps), float(p_start), float(p_end), int(k_start),
                                        int(k_end), int(dense_steps), ctypes.byref(p), ctypes.byref(km)))
    return p.value, km.value


def workspace_size_bwd(shape: Shape) -> int:
    n = ctypes.c_size_t()
    _check("fvattn_workspace_size_bwd", lib().fvattn_workspace_size_bwd(ctypes.byref(shape), ctypes.byref(n)))
    return n.value


def block_sparse_bwd(shape: Shape, q, k, v, out, dout, lse, counts, idx, ws, grads=None, stream=None):
    """Backward of step 6 (tiled layout, bf16): returns (dq, dk, dv)."""
    if grads is None:
        grads = tuple(torch.empty_like(q) for _ in range(3))
    dq, dk, dv = grads
    b = _blocks_of(counts, idx)
    _check("fvattn_block_sparse_bwd",
           lib().fvattn_block_sparse_bwd(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(dout),
                                         _ptr(lse), ctypes.byref(b), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(ws),
                                         ws.numel(), _stream(stream)))
    return dq, dk, dv


def workspace_size_qkv(shape: Shape, rope: Optional[Rope] = None) -> int:
    n = ctypes.c_size_t()
    _check("fvattn_workspace_size_qkv",
           lib().fvattn_workspace_size_qkv(ctypes.byref(shape), _rope_ptr(rope), ctypes.byref(n)))
    return n.value


def qkv_rope(shape: Shape, x, w, ws, bias=None, rope: Optional[Rope] = None, t_offset: int = 0, out=None,
             stream=None):
    """Prologue: x [B, N, C] bf16, w [3*H*d, C] bf16, bias [3*H*d] float32
    or None -> (q, k, v) [B, H, N, d] bf16 in shape.layout, Q and K rotated
    at frame t + t_offset."""
    B, N, C = x.shape
    if out is None:
        out = tuple(torch.empty((shape.batch, shape.heads, N, shape.head_dim), dtype=torch.bfloat16,
                                device=x.device) for _ in range(3))
    q, k, v = out
    _check("fvattn_qkv_rope",
           lib().fvattn_qkv_rope(ctypes.byref(shape), _ptr(x), int(C), _ptr(w), _ptr(bias), _rope_ptr(rope),
                                 int(t_offset), _ptr(q), _ptr(k), _ptr(v), _ptr(ws), ws.numel(), _stream(stream)))
    return q, k, v


def device_status(ws, stream=None) -> int:
    """Synchronise, read and clear the workspace status word (0 = no error)."""
    st = ctypes.c_int32()
    _check("fvattn_get_device_status", lib().fvattn_get_device_status(_ptr(ws), _stream(stream), ctypes.byref(st)))
    return st.value


def selftest_wait_timeout(ws, cap_iterations: int, stream=None):
    _check("fvattn_selftest_wait_timeout",
           lib().fvattn_selftest_wait_timeout(_ptr(ws), ws.numel(), int(cap_iterations), _stream(stream)))


def profile_enable(on: bool = True):
    """Record CUDA events around every library kernel (per-stage timing)."""
    _check("fvattn_profile_enable", lib().fvattn_profile_enable(1 if on else 0))


def profile_cta_times(shape: Shape, ws, rope: Optional[Rope] = None, stream=None):
    """(start, end) nanoseconds of every CTA of the last profiled fine-stage
    launch that used `ws`, as an [n, 2] int64 numpy array (synchronises)."""
    import numpy as np
    cap = 1024
    buf = (ctypes.c_int64 * (2 * cap))()
    n = ctypes.c_int32(0)
    _check("fvattn_profile_cta_times", lib().fvattn_profile_cta_times(ctypes.byref(shape), _rope_ptr(rope), _ptr(ws),
                                                                        _stream(stream), buf, cap, ctypes.byref(n)))
    m = min(n.value, cap)
    return np.frombuffer(buf, dtype=np.int64, count=2 * m).reshape(m, 2).copy()


def profile_read():
    """{stage: (ms, launches)} summed since the last read (synchronises)."""
    ms = (ctypes.c_double * len(STAGES))()
    n = (ctypes.c_int64 * len(STAGES))()
    _check("fvattn_profile_read", lib().fvattn_profile_read(ms, n))
    return {name: (ms[i], n[i]) for i, name in enumerate(STAGES)}
