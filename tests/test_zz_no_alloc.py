"""The allocation-free scan + top-k entry point against the regular one.

fathom_scan_topk_noalloc serves callers that cannot allocate device memory
(an engine that hands all its memory to its own pool, a plug-in whose host
forbids cudaMalloc/cudaFree on the serving path): it takes its scratch from
a fixed array inside the library instead of a caller workspace.  This test
calls it through the C ABI twice in a row, on two different decode steps, and
checks each result against fathom_scan_topk given a normal workspace.  The
second call also shows that whatever the first call left in the shared array
does not leak into the next result.  The file is named so that pytest
collects it last.
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
SCORE_RTOL = 1e-4   # the score tolerance the parity tests use


def _inputs(layer, n, B):
    inp = synth.layer_inputs(2, layer=layer, n=n, n_kv_heads=2, n_q_heads=8)
    q = torch.from_numpy(inp["q_bf16"].view(np.int16)).to(DEV).view(torch.bfloat16)
    st = F.pack_bitplanes(torch.from_numpy(inp["K"]).to(DEV))
    dep = F.alloc_depths(q, torch.from_numpy(inp["sigma2"]).to(DEV), B)
    return st, q, dep


def _regular(st, q, dep, k):
    ws = torch.empty(F.scan_workspace_bytes(st, q.shape[0], k), dtype=torch.uint8, device=DEV)
    idx, top = F.scan_topk(st, q, dep, k, workspace=ws)
    torch.cuda.synchronize()
    return idx.cpu().numpy(), top.cpu().numpy()


def _noalloc_c_abi(st, q, dep, k):
    idx = torch.full((q.shape[0], k), -7, dtype=torch.int32, device=DEV)
    top = torch.full((q.shape[0], k), float("nan"), dtype=torch.float32, device=DEV)
    rc = F.lib().fathom_scan_topk_noalloc(
        st.c, ctypes.c_void_p(q.data_ptr()), F.BF16, ctypes.c_void_p(dep.data_ptr()), q.shape[0], k,
        ctypes.c_void_p(idx.data_ptr()), ctypes.c_void_p(top.data_ptr()),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == F.OK, rc
    torch.cuda.synchronize()
    return idx.cpu().numpy(), top.cpu().numpy()


def test_noalloc_matches_regular_entry_point_twice_in_a_row():
    steps = [(_inputs(0, 20000, 92), 2048), (_inputs(1, 9000, 46), 512)]
    for (st, q, dep), k in steps:
        need = F.scan_workspace_bytes(st, q.shape[0], k)
        assert 0 < need <= F.noalloc_scratch_bytes()
        want_idx, want_top = _regular(st, q, dep, k)
        got_idx, got_top = _noalloc_c_abi(st, q, dep, k)
        assert np.array_equal(got_idx, want_idx)
        np.testing.assert_allclose(got_top, want_top, rtol=SCORE_RTOL, atol=0)
    assert F.last_device_status() == 0


def test_noalloc_rejects_steps_beyond_its_scratch():
    st, q, dep = _inputs(2, 4096, 64)
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
