"""C-ABI checks that need no GPU: the library loads, exports every function
include/fathom.h declares, and its host-only functions answer correctly."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fathom.h")


@pytest.fixture(scope="module")
def libpath():
    from bit_plane_key_b200 import build
    return build.build()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\**\s+(fathom_[a-z0-9_]+)\s*\(", src, flags=re.M)
    return sorted(set(names))


def test_header_declares_the_boundary():
    names = declared_functions()
    for must in ("fathom_pack_bitplanes", "fathom_alloc_depths", "fathom_scan_topk", "fathom_sparse_attend",
                 "fathom_scan_scores", "fathom_topk", "fathom_planes_bytes", "fathom_scales_bytes",
                 "fathom_scan_workspace_bytes", "fathom_last_device_status", "fathom_decode_step",
                 "fathom_decode_workspace_bytes"):
        assert must in names


def test_library_exports_every_declared_symbol(libpath):
    out = subprocess.run(["nm", "-D", "--defined-only", libpath], capture_output=True, text=True, check=True).stdout
    exported = set(re.findall(r"\sT\s(\S+)$", out, flags=re.M))
    missing = [n for n in declared_functions() if n not in exported]
    assert not missing, missing
    lib = ctypes.CDLL(libpath)
    for n in declared_functions():
        assert hasattr(lib, n)


def test_host_only_functions(libpath):
    from bit_plane_key_b200 import fathom as F
    L = F.lib()
    assert F.n_pad(1) == 1024 and F.n_pad(1024) == 1024 and F.n_pad(4097) == 5120
    assert L.fathom_planes_bytes(8, 128, 131072) == 8 * 128 * 4 * 131072 // 8
    assert L.fathom_scales_bytes(8, 128, 131072) == 8 * 128 * (131072 // 64) * 2
    assert L.fathom_planes_bytes(8, 100, 1000) == 0      # d not a multiple of 32
    assert L.fathom_planes_bytes(0, 128, 1000) == 0
    assert L.fathom_topk_workspace_bytes(1000, 4, 5000) == 0   # k above the maximum
    assert L.fathom_topk_workspace_bytes(1000, 4, 64) > 0
    assert L.fathom_status_string(0) == b"ok"
    assert L.fathom_status_string(2) == b"workspace or buffer too small"


def test_null_arguments_rejected_before_any_cuda_call(libpath):
    from bit_plane_key_b200 import fathom as F
    L = F.lib()
    assert L.fathom_pack_bitplanes(None, 0, 1, 10, 32, None, None, None) == F.EINVAL
    assert L.fathom_alloc_depths(None, 0, None, 1, 1, 32, 10, 0, None, None) == F.EINVAL
    assert L.fathom_topk(None, None, 10, 10, 1, 1, None, None, None, 0, None) == F.EINVAL
    assert L.fathom_scan_topk(None, None, 0, None, 1, 1, None, None, None, 0, None) == F.EINVAL
    assert L.fathom_sparse_attend(None, 0, None, None, 128, 0, None, 1, 1, 10, 128, 1, None, None) == F.EINVAL
    assert L.fathom_decode_step(None, None, 0, None, 4, 92, 0, 16, None, None, 10, 128, 0, 1, None, None, None,
                                None, None, 0, None) == F.EINVAL
    assert L.fathom_sparse_attend_partial(None, 0, None, None, 128, 0, 0, None, 1, 1, 10, 128, 1, None,
                                          None) == F.EINVAL
    assert L.fathom_attend_merge(None, 1, 1, 128, None, None) == F.EINVAL
    # non-null but impossible sizes are rejected before the pointers are looked at
    fake = ctypes.c_void_p(16)
    assert L.fathom_sparse_attend_partial(fake, 0, fake, fake, 128, 0, -1, fake, 1, 1, 10, 128, 1, fake,
                                          None) == F.EINVAL
    assert L.fathom_attend_merge(fake, 0, 1, 128, fake, None) == F.EINVAL


def test_decode_workspace_sizes(libpath):
    from bit_plane_key_b200 import fathom as F
    st = F.fathom_store(8, 128, 1 << 20, F.n_pad(1 << 20), 1, 0, None, None)
    one = F.lib().fathom_decode_workspace_bytes(ctypes.byref(st), 32, 2048, 1)
    four = F.lib().fathom_decode_workspace_bytes(ctypes.byref(st), 32, 2048, 4)
    assert one >= 4 * 32 * F.n_pad(1 << 20) and four >= 4 * 32 * F.n_pad(1 << 20)
    assert four < one            # one top-k workspace, sized for a group's rows
    assert F.lib().fathom_decode_workspace_bytes(ctypes.byref(st), 32, 2048, 3) == 0    # 3 does not divide 8
    assert F.lib().fathom_decode_workspace_bytes(ctypes.byref(st), 32, 5000, 1) == 0    # k above the maximum
    assert F.lib().fathom_decode_workspace_bytes(ctypes.byref(st), 30, 2048, 1) == 0    # Hq not a multiple of Hkv
