"""The one-call decode step (fathom_decode_step) against the separate calls.

The step pipelines groups of KV heads over two streams; every kernel is the
separate entry points' kernel on a slice of the same arrays, so depths, top-k
indices and scores, and the attention output must equal fathom_alloc_depths +
fathom_scan_topk + fathom_sparse_attend bit for bit, for every group count,
residency and GQA ratio.  The separate calls are themselves checked against
the oracle in test_gpu_parity.py; one case here also checks the attention
output against the oracle directly.
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


def _layer(n, Hkv, Hq, d=128, config=2, layer=0):
    inp = synth.layer_inputs(config, layer=layer, n=n, n_kv_heads=Hkv, n_q_heads=Hq, d=d, with_values=True)
    q = torch.from_numpy(inp["q_bf16"].view(np.int16)).to(DEV).view(torch.bfloat16)
    s2 = torch.from_numpy(inp["sigma2"]).to(DEV)
    st = F.pack_bitplanes(torch.from_numpy(inp["K"]).to(DEV))
    Kr = torch.from_numpy(inp["K_rows"].view(np.int16)).to(DEV).view(torch.bfloat16)
    Vr = torch.from_numpy(inp["V_rows"].view(np.int16)).to(DEV).view(torch.bfloat16)
    return inp, q, s2, st, Kr, Vr


def _separate(st, q, s2, B, k, Kr, Vr):
    dep = F.alloc_depths(q, s2, B)
    idx, top = F.scan_topk(st, q, dep, k)
    out = F.sparse_attend(q, Kr, Vr, idx)
    torch.cuda.synchronize()
    return dep.cpu(), idx.cpu(), top.cpu(), out.cpu()


@pytest.mark.parametrize("n,Hkv,Hq,groups,host", [
    (20000, 8, 32, 1, False), (20000, 8, 32, 2, False), (20000, 8, 32, 8, False),
    (9001, 4, 8, 4, False), (9001, 4, 8, 2, True), (40000, 8, 32, 4, True),
    (200001, 4, 16, 1, False), (200001, 4, 16, 2, True)])
def test_decode_step_equals_separate_calls(n, Hkv, Hq, groups, host):
    """Rows of up to 131072 keys take the cluster top-k over the scores, the
    200001-key rows the cluster top-k over the block maxima."""
    inp, q, s2, st, Kr, Vr = _layer(n, Hkv, Hq)
    B, k = 92, 512
    if host:   # host-resident store and interleaved host rows
        st = st.to_host()
        Ki, Vi = F.kv_rows(Hkv, n, 128, pin_memory=True)
        Ki.copy_(Kr)
        Vi.copy_(Vr)
        Kr, Vr = Ki, Vi
    want = _separate(st, q, s2, B, k, Kr, Vr)
    got = F.decode_step(st, q, s2, B, k, Kr, Vr, kv_groups=groups)
    torch.cuda.synchronize()
    for name, a, b in zip(("depths", "idx", "top", "out"), want, [t.cpu() for t in got]):
        assert torch.equal(a, b), name
    assert F.last_device_status() == 0


def test_decode_step_fixed_r_without_top_scores_and_oracle_attention(ref):
    n, Hkv, Hq, k = 5000, 2, 8, 300
    inp, q, s2, st, Kr, Vr = _layer(n, Hkv, Hq, layer=3)
    dep, idx, top, out = F.decode_step(st, q, s2, 0, k, Kr, Vr, fixed_r=16, kv_groups=2, want_top_scores=False)
    assert top is None
    dep_h, idx_h, out_h = dep.cpu().numpy(), idx.cpu().numpy(), out.cpu().numpy()
    assert np.array_equal(dep_h, ref.alloc_depths(inp["q"], inp["sigma2"], 0, fixed_r=16))
    want = ref.attend(inp["q"], inp["K_rows"], inp["V_rows"], idx_h)
    for h in range(Hq):
        assert np.linalg.norm(out_h[h] - want[h]) <= 1e-3 * np.linalg.norm(want[h]), h


def test_decode_step_in_a_cuda_graph():
    n, Hkv, Hq, k, B = 20000, 8, 32, 256, 68
    inp, q, s2, st, Kr, Vr = _layer(n, Hkv, Hq, layer=5)
    want = _separate(st, q, s2, B, k, Kr, Vr)
    bufs = dict(depths=torch.empty((Hq, 128), dtype=torch.uint8, device=DEV),
                idx=torch.empty((Hq, k), dtype=torch.int32, device=DEV),
                top_scores=torch.empty((Hq, k), dtype=torch.float32, device=DEV),
                out=torch.empty((Hq, 128), dtype=torch.float32, device=DEV),
                workspace=torch.empty(F.decode_workspace_bytes(st, Hq, k, 4), dtype=torch.uint8, device=DEV))
    F.decode_step(st, q, s2, B, k, Kr, Vr, kv_groups=4, **bufs)   # creates the auxiliary stream before capture
    torch.cuda.synchronize()
    for v in bufs.values():
        v.zero_()
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            F.decode_step(st, q, s2, B, k, Kr, Vr, kv_groups=4, stream=s, **bufs)
    g.replay()
    torch.cuda.synchronize()
    for name, a in zip(("depths", "idx", "top_scores", "out"), want):
        assert torch.equal(a, bufs[name].cpu()), name
    del g


def test_decode_step_rejects_bad_groups_and_small_workspace():
    n, Hkv, Hq, k = 3000, 4, 16, 64
    inp, q, s2, st, Kr, Vr = _layer(n, Hkv, Hq)
    with pytest.raises(F.FathomError) as e:
        F.decode_step(st, q, s2, 92, k, Kr, Vr, kv_groups=3)
    assert e.value.status == F.EINVAL
    ws = torch.empty(F.decode_workspace_bytes(st, Hq, k, 2) - 256, dtype=torch.uint8, device=DEV)
    with pytest.raises(F.FathomError) as e:
        F.decode_step(st, q, s2, 92, k, Kr, Vr, kv_groups=2, workspace=ws)
    assert e.value.status == F.ENOMEM
