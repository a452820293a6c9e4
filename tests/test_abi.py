"""The C-ABI library loads, exports every symbol the header declares, and its
host-side validation returns the documented status codes (no GPU needed:
these calls fail before any CUDA work is enqueued)."""
import ctypes
import os
import re

import pytest

from block_sparse_spatiotemporal_b200 import fvattn as F

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names |= set(re.findall(r"\b(fvattn_\w+)\s*\(", src))
    return names


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(F.library_path()):
        from block_sparse_spatiotemporal_b200 import build
        build.build()
    return F.lib()


def test_every_declared_symbol_is_exported(lib):
    names = _declared()
    assert len(names) >= 10
    for n in sorted(names):
        assert hasattr(lib, n), n
    assert set(F._SIGS) == names


def test_struct_layouts_match_the_c_header(tmp_path):
    """sizeof/offsetof of every ABI struct, compiled from include/fvattn.h by
    the C compiler, against the ctypes mirror."""
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    probes = {
        "fvattn_shape": (F.Shape, ["batch", "heads", "head_dim", "grid", "tile", "dtype", "order", "layout",
                                   "scale"]),
        "fvattn_rope": (F.Rope, ["enabled", "dt", "dh", "dw", "base"]),
        "fvattn_blocks": (F.Blocks, ["counts", "idx", "cap"]),
        "fvattn_mask_cache": (F.MaskCache, ["blocks", "shape", "top_p", "k_min", "valid"]),
    }
    lines = ["#include <stdio.h>", "#include <stddef.h>", '#include "fvattn.h"', "int main(void){"]
    for cname, (_, fields) in probes.items():
        lines.append(f'printf("{cname} %zu\\n", sizeof({cname}));')
        for f in fields:
            lines.append(f'printf("{cname}.{f} %zu\\n", offsetof({cname}, {f}));')
    lines.append("return 0;}")
    src = tmp_path / "probe.c"
    src.write_text("\n".join(lines))
    exe = tmp_path / "probe"
    subprocess.run([cc, "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)], check=True)
    got = dict(line.split() for line in subprocess.run([str(exe)], capture_output=True, text=True,
                                                        check=True).stdout.splitlines())
    for cname, (cls, fields) in probes.items():
        assert int(got[cname]) == ctypes.sizeof(cls), cname
        for f in fields:
            assert int(got[f"{cname}.{f}"]) == getattr(cls, f).offset, (cname, f)


def _status(shape):
    n = ctypes.c_int64()
    return F.lib().fvattn_num_tiles(ctypes.byref(shape), ctypes.byref(n)), n.value


def test_num_tiles_and_shape_validation(lib):
    assert _status(F.make_shape(1, 40, 128, (20, 32, 52))) == (0, 520)
    assert _status(F.make_shape(1, 40, 128, (20, 48, 80)))[1] == 1200
    assert _status(F.make_shape(1, 2, 64, (8, 16, 16), dtype=F.F32)) == (0, 32)
    assert _status(F.make_shape(1, 1, 128, (4, 4, 6)))[0] == -2          # partial tile
    assert _status(F.make_shape(1, 1, 128, (0, 4, 4)))[0] == -2
    assert _status(F.make_shape(1, 1, 96, (4, 4, 4)))[0] == -2           # head dim
    assert _status(F.make_shape(1, 1, 64, (4, 4, 4)))[0] == -9           # bf16 d=64 not built
    assert _status(F.make_shape(1, 1, 64, (4, 4, 4), dtype=F.F32))[0] == 0
    assert _status(F.make_shape(1, 1, 128, (256, 64, 64)))[0] == -2      # nT > 4096
    assert _status(F.make_shape(0, 1, 128, (4, 4, 4)))[0] == -2
    bad = F.make_shape(1, 1, 128, (4, 4, 4))
    bad.dtype = 7
    assert _status(bad)[0] == -3
    bad = F.make_shape(1, 1, 128, (4, 4, 4))
    bad.scale = -1.0
    assert _status(bad)[0] == -1
    bad = F.make_shape(1, 1, 128, (4, 4, 4))
    bad.tile = F.Tile(2, 4, 4)
    assert _status(bad)[0] == -2


def test_workspace_size_grows_with_rope_and_heads(lib):
    s1 = F.make_shape(1, 4, 128, (8, 16, 16))
    s2 = F.make_shape(1, 8, 128, (8, 16, 16))
    a, b = F.workspace_size(s1), F.workspace_size(s2)
    assert 0 < a < b
    assert F.workspace_size(s1, F.make_rope()) > a
    n = ctypes.c_size_t()
    bad_rope = F.make_rope((44, 42, 40))
    assert lib.fvattn_workspace_size(ctypes.byref(s1), ctypes.byref(bad_rope), ctypes.byref(n)) == -1
    odd_rope = F.make_rope((43, 43, 42))
    assert lib.fvattn_workspace_size(ctypes.byref(s1), ctypes.byref(odd_rope), ctypes.byref(n)) == -1


def test_argument_errors_before_any_device_work(lib):
    s = F.make_shape(1, 1, 128, (4, 4, 8))
    b = F.Blocks(None, None, 2)
    # null tensors
    assert lib.fvattn_pool_select(ctypes.byref(s), None, None, None, 0.9, 1, ctypes.byref(b), None, 0, None) == -1
    assert lib.fvattn_block_sparse_fwd(ctypes.byref(s), None, None, None, None, ctypes.byref(b), None, None,
                                       None, 0, None) == -1
    assert lib.fvattn_forward(ctypes.byref(s), None, None, None, None, 0.9, 1, None, 0, None, None, None, 0,
                              None) == -1
    assert lib.fvattn_tile_reorder(ctypes.byref(s), None, None, 256, 0, None, 0, None) == -1
    assert lib.fvattn_get_device_status(None, None, None) == -1
    assert lib.fvattn_selftest_wait_timeout(None, 0, 10, None) == -1
    # misaligned tensor pointers are rejected on the host
    fake = ctypes.c_void_p(0x1000 + 8)
    assert lib.fvattn_pool_select(ctypes.byref(s), fake, fake, None, 0.9, 1, ctypes.byref(b), None, 0,
                                  None) == -1
    # NaN top_p and negative k_min
    al = ctypes.c_void_p(0x100000)
    assert lib.fvattn_pool_select(ctypes.byref(s), al, al, None, float("nan"), 1, ctypes.byref(b), None, 0,
                                  None) == -1
    assert lib.fvattn_pool_select(ctypes.byref(s), al, al, None, 0.9, -1, ctypes.byref(b), None, 0, None) == -1


def test_status_strings(lib):
    for code in range(-9, 1):
        assert lib.fvattn_status_string(code)
    assert b"unknown" in lib.fvattn_status_string(42)


def test_new_entry_points_reject_bad_arguments_on_the_host(lib):
    """Prologue, backward and augmentation: argument, dtype, layout and shape
    errors are returned before any device call (fake aligned pointers)."""
    al = ctypes.c_void_p(0x100000)
    s = F.make_shape(1, 1, 128, (4, 4, 8), layout=F.TILED)
    # prologue: null input, channels not a multiple of 64, negative start frame, fp32
    assert lib.fvattn_qkv_rope(ctypes.byref(s), None, 64, al, None, None, 0, al, al, al, al, 1 << 20, None) == -1
    assert lib.fvattn_qkv_rope(ctypes.byref(s), al, 96, al, None, None, 0, al, al, al, al, 1 << 20, None) == -2
    assert lib.fvattn_qkv_rope(ctypes.byref(s), al, 64, al, None, None, -1, al, al, al, al, 1 << 20, None) == -1
    f32 = F.make_shape(1, 1, 128, (4, 4, 8), dtype=F.F32, layout=F.TILED)
    assert lib.fvattn_qkv_rope(ctypes.byref(f32), al, 64, al, None, None, 0, al, al, al, al, 1 << 20, None) == -3
    # backward: natural layout is not built, fp32 is not a backward dtype, null gradient
    b = F.Blocks(al.value, al.value, 2)
    nat = F.make_shape(1, 1, 128, (4, 4, 8))
    args = (al, al, al, al, al, ctypes.cast(al, ctypes.c_void_p), ctypes.byref(b), al, al, al, al, 1 << 30, None)
    assert lib.fvattn_block_sparse_bwd(ctypes.byref(nat), *args) == -9
    assert lib.fvattn_block_sparse_bwd(ctypes.byref(f32), *args) == -3
    assert lib.fvattn_block_sparse_bwd(ctypes.byref(s), al, al, al, al, al, al, ctypes.byref(b), None, al, al, al,
                                       1 << 30, None) == -1
    # augmentation: more than 1024 CTAs, null work list, fill outside [0, 100] with measured busy times
    assert lib.fvattn_augment_lists(ctypes.byref(s), al, al, None, ctypes.byref(b), 2048, None, 100,
                                    ctypes.byref(b), al, al, 1 << 30, None) == -1
    assert lib.fvattn_augment_lists(ctypes.byref(s), al, al, None, ctypes.byref(b), 0, None, 100,
                                    ctypes.byref(b), None, al, 1 << 30, None) == -1
    busy = (ctypes.c_int64 * 4)(1, 2, 3, 4)
    for fill in (-1, 101):
        assert lib.fvattn_augment_lists(ctypes.byref(s), al, al, None, ctypes.byref(b), 4, busy, fill,
                                        ctypes.byref(b), al, al, 1 << 30, None) == -1
    assert lib.fvattn_block_sparse_fwd_worklist(ctypes.byref(s), al, al, al, None, ctypes.byref(b), None, 0, al, al,
                                                al, 1 << 30, None) == -1
    # workspace sizes of the new entry points
    n = ctypes.c_size_t()
    assert lib.fvattn_workspace_size_bwd(ctypes.byref(s), ctypes.byref(n)) == 0 and n.value > 0
    assert lib.fvattn_workspace_size_qkv(ctypes.byref(s), None, ctypes.byref(n)) == 0 and n.value > 0
