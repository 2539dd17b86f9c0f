"""Decode-time append (fathom_append_keys) and stores with spare capacity.

A growing cache is a store whose arrays have room for more keys than it holds
(n_pad = capacity, the row stride).  Appending keys must leave the store
exactly as packing all keys at once would (bit for bit over the scanned
range), and every call that reads a store must give the same results for a
store with spare capacity as for one packed to size.
"""
import numpy as np
import pytest

import synth

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA GPU", allow_module_level=True)

from bit_plane_key_b200 import fathom as F  # noqa: E402

DEV = torch.device("cuda:0")


def _keys(n, Hkv=2, Hq=8, d=128, layer=0):
    inp = synth.layer_inputs(2, layer=layer, n=n, n_kv_heads=Hkv, n_q_heads=Hq, d=d, with_values=True)
    q = torch.from_numpy(inp["q_bf16"].view(np.int16)).to(DEV).view(torch.bfloat16)
    return inp, torch.from_numpy(inp["K"]).to(DEV), q, torch.from_numpy(inp["sigma2"]).to(DEV)


@pytest.mark.parametrize("host", [False, True])
def test_append_equals_packing_everything(ref, host):
    n_final, cap = 5000, 9000
    inp, K, q, s2 = _keys(n_final)
    st = F.Store.empty(2, 128, cap, device=DEV, host_resident=host)
    assert st.n_pad == F.n_pad(cap) and st.n == 0
    prev = 0
    for n in (700, 701, 702, 703, 764, 765, 1030, 2048, 2049, 3100, 4999, 5000):
        t = (prev // 64) * 64
        F.append_keys(st, K[:, t:n].contiguous(), n)
        torch.cuda.synchronize()
        assert st.n == n
        planes_ref, scales_ref = ref.pack(inp["K"][:, :n])
        npad = F.n_pad(n)
        P = st.planes.cpu().numpy().view(np.uint32)
        S = st.scales.cpu().numpy().view(np.uint16)
        assert np.array_equal(P[..., :npad // 32], planes_ref), n
        assert np.array_equal(S[..., :npad // 64], scales_ref), n
        prev = n
    # the scan of the grown store equals the scan of a store packed to size
    dep = F.alloc_depths(q, s2, 92)
    fresh = F.pack_bitplanes(K)
    if host:
        fresh = fresh.to_host()
    assert torch.equal(F.scan_scores(st, q, dep), F.scan_scores(fresh, q, dep))
    i1, t1 = F.scan_topk(st, q, dep, 300)
    i2, t2 = F.scan_topk(fresh, q, dep, 300)
    assert torch.equal(i1, i2) and torch.equal(t1, t2)
    assert F.last_device_status() == 0


def test_append_one_key_at_a_time_bf16():
    n0, steps = 1000, 70   # crosses a block boundary (1024) on the way
    inp, K, q, s2 = _keys(n0 + steps, layer=1)
    Kb = K.to(torch.bfloat16)
    st = F.Store.empty(2, 128, 4096, device=DEV)
    F.append_keys(st, Kb[:, :n0].contiguous(), n0)
    for n in range(n0 + 1, n0 + steps + 1):
        t = ((n - 1) // 64) * 64
        F.append_keys(st, Kb[:, t:n].contiguous(), n)
    fresh = F.pack_bitplanes(Kb)
    npad = F.n_pad(n0 + steps)
    assert torch.equal(st.planes[..., :npad // 32], fresh.planes)
    assert torch.equal(st.scales[..., :npad // 64], fresh.scales)


def test_append_rejects_bad_requests():
    inp, K, q, s2 = _keys(3000, layer=2)
    st = F.Store.empty(2, 128, 2048, device=DEV)
    F.append_keys(st, K[:, :1500].contiguous(), 1500)
    with pytest.raises(F.FathomError) as e:          # beyond the capacity
        F.append_keys(st, K[:, 1472:2100].contiguous(), 2100)
    assert e.value.status == F.EINVAL
    with pytest.raises(F.FathomError) as e:          # not growing
        F.append_keys(st, K[:, 1472:1500].contiguous(), 1500)
    assert e.value.status == F.EINVAL
    assert st.n == 1500


def test_decode_step_on_a_growing_cache(ref):
    """A store and K/V rows with spare capacity: the one-call step equals the
    separate calls, and the attention over capacity-strided rows is exact."""
    n, cap, Hkv, Hq, k = 6000, 8192, 2, 8, 256
    inp, K, q, s2 = _keys(n, layer=3)
    st = F.Store.empty(Hkv, 128, cap, device=DEV)
    F.append_keys(st, K, n)
    Kr, Vr = F.kv_rows(Hkv, cap, 128, device=DEV)   # rows at capacity; only the first n are used
    Kr.zero_()
    Vr.zero_()
    Kr[:, :n].copy_(torch.from_numpy(inp["K_rows"].view(np.int16)).to(DEV).view(torch.bfloat16))
    Vr[:, :n].copy_(torch.from_numpy(inp["V_rows"].view(np.int16)).to(DEV).view(torch.bfloat16))
    dep = F.alloc_depths(q, s2, 92)
    idx, top = F.scan_topk(st, q, dep, k)
    out = F.sparse_attend(q, Kr, Vr, idx)
    got = F.decode_step(st, q, s2, 92, k, Kr, Vr, kv_groups=2)
    torch.cuda.synchronize()
    for a, b in zip((dep, idx, top, out), got):
        assert torch.equal(a, b)
    want = ref.attend(inp["q"], inp["K_rows"], inp["V_rows"], idx.cpu().numpy())
    o = out.cpu().numpy()
    for h in range(Hq):
        assert np.linalg.norm(o[h] - want[h]) <= 1e-3 * np.linalg.norm(want[h])
