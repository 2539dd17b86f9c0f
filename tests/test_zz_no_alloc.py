"""The allocation-free scan + top-k entry point against the regular one.

fathom_scan_topk_noalloc serves callers that cannot allocate device memory:
an inference engine that hands all of its device memory to its own pool up
front, or a plug-in whose host program forbids cudaMalloc/cudaFree on the
serving path (both calls synchronise the device and would stall every other
stream).  It takes its scratch from a fixed array inside the library instead
of a caller workspace.

This test calls it through the C ABI on several decode steps in a row and
checks every result against fathom_scan_topk given a normal workspace, bit for
bit: both calls run the same kernels on the same inputs.  The steps are chosen
so that each top-k path keeps its state in the shared scratch array in turn:
rows of at most 131072 keys (one cluster kernel, no top-k buffers), rows of
200000 keys twice with different budgets and k (the histogram path: row
state, histograms and candidate lists, which the second step must not inherit
from the first), and rows of 600000 keys at k = 64 (the block-maxima path).
The file is named so that pytest collects it last.
"""
import ctypes

import numpy as np
import pytest

import synth

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA GPU", allow_module_level=True)

from bit_plane_key_b200 import fathom as F  # noqa: E402

DEV = torch.device("cuda:0")


def _inputs(layer, n, B, d=128):
    inp = synth.layer_inputs(2, layer=layer, n=n, n_kv_heads=2, n_q_heads=8, d=d)
    q = torch.from_numpy(inp["q_bf16"].view(np.int16)).to(DEV).view(torch.bfloat16)
    st = F.pack_bitplanes(torch.from_numpy(inp["K"]).to(DEV))
    dep = F.alloc_depths(q, torch.from_numpy(inp["sigma2"]).to(DEV), B)
    return st, q, dep


def _regular(st, q, dep, k):
    ws = torch.empty(F.scan_workspace_bytes(st, q.shape[0], k), dtype=torch.uint8, device=DEV)
    idx, top = F.scan_topk(st, q, dep, k, workspace=ws)
    torch.cuda.synchronize()
    return idx, top


def _noalloc_c_abi(st, q, dep, k):
    idx = torch.full((q.shape[0], k), -7, dtype=torch.int32, device=DEV)
    top = torch.full((q.shape[0], k), float("nan"), dtype=torch.float32, device=DEV)
    rc = F.lib().fathom_scan_topk_noalloc(
        st.c, ctypes.c_void_p(q.data_ptr()), F.BF16, ctypes.c_void_p(dep.data_ptr()), q.shape[0], k,
        ctypes.c_void_p(idx.data_ptr()), ctypes.c_void_p(top.data_ptr()),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == F.OK, rc
    torch.cuda.synchronize()
    return idx, top


# (layer, n, budget, k, d, top-k path taken)
STEPS = [
    (0, 20000, 92, 2048, 128, "cluster"),
    (1, 200000, 92, 2048, 64, "histogram"),
    (2, 200000, 46, 1000, 64, "histogram"),
    (3, 600000, 68, 64, 64, "block maxima"),
    (4, 9000, 46, 512, 128, "cluster"),
]


def test_noalloc_matches_regular_entry_point_on_consecutive_steps():
    for layer, n, B, k, d, path in STEPS:
        st, q, dep = _inputs(layer, n, B, d)
        need = F.scan_workspace_bytes(st, q.shape[0], k)
        assert 0 < need <= F.noalloc_scratch_bytes(), (path, need)
        want_idx, want_top = _regular(st, q, dep, k)
        got_idx, got_top = _noalloc_c_abi(st, q, dep, k)
        assert torch.equal(got_idx, want_idx), path
        assert torch.equal(got_top.view(torch.int32), want_top.view(torch.int32)), path
        del st, q, dep
        torch.cuda.empty_cache()
    assert F.last_device_status() == 0


def test_noalloc_rejects_steps_beyond_its_scratch():
    st, q, dep = _inputs(5, 4096, 64)
    big = F.Store(st.planes, st.scales, st.n)
    # describe a store far larger than the scratch array can score (sizes only:
    # the size check comes before any pointer is looked at)
    big._c.n = 1 << 22
    big._c.n_pad = F.n_pad(1 << 22)
    idx = torch.empty((8, 16), dtype=torch.int32, device=DEV)
    rc = F.lib().fathom_scan_topk_noalloc(big.c, ctypes.c_void_p(q.data_ptr()), F.BF16,
                                          ctypes.c_void_p(dep.data_ptr()), 8, 16, ctypes.c_void_p(idx.data_ptr()),
                                          None, ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == F.ENOMEM
