"""Key-range sharding, emulated on one GPU: the layer's keys are split into
four 1024-aligned ranges, each range is packed and scanned on its own and
takes its local top-k, the lists are laid side by side as the all-gather
would lay them, and fathom_topk_merge must return exactly the top-k of the
unsplit layer (indices and scores, bit for bit).  Attention over the
selected keys then runs per range on that range's rows, and
fathom_attend_merge of the ranges' partials must give the unsplit
attention up to fp32 rounding."""
import numpy as np
import pytest

import synth

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA GPU", allow_module_level=True)

from bit_plane_key_b200 import fathom as F  # noqa: E402
from bit_plane_key_b200.shard import empty_partials, local_topk, shard_range  # noqa: E402

DEV = torch.device("cuda:0")


@pytest.mark.parametrize("n,world,k,host", [(20000, 4, 2048, False), (9000, 3, 512, True), (3000, 4, 1500, False)])
def test_sharded_topk_equals_unsplit(n, world, k, host):
    inp = synth.layer_inputs(2, layer=7, n=n, n_kv_heads=2, n_q_heads=8, needles=0)
    K = torch.from_numpy(inp["K"]).to(DEV)
    q = torch.from_numpy(inp["q_bf16"].view(np.int16)).to(DEV).view(torch.bfloat16)
    dep = F.alloc_depths(q, torch.from_numpy(inp["sigma2"]).to(DEV), 92)
    whole = F.pack_bitplanes(K)
    if host:
        whole = whole.to_host()
    want_idx, want_top = F.scan_topk(whole, q, dep, k)
    tops, idxs = [], []
    for r in range(world):
        k0, k1 = shard_range(n, world, r)
        shard = F.pack_bitplanes(K[:, k0:k1].contiguous()) if k1 > k0 else None
        if host and shard is not None:
            shard = shard.to_host()
        t, i = local_topk(shard, k0, q, dep, k)
        tops.append(t)
        idxs.append(i)
    idx, top = F.topk_merge(torch.cat(tops, dim=1).contiguous(), torch.cat(idxs, dim=1).contiguous(), k)
    assert torch.equal(idx, want_idx)
    assert torch.equal(top, want_top)
    assert F.last_device_status() == 0


def test_topk_merge_rejects_bad_sizes():
    s = torch.zeros((2, 100), dtype=torch.float32, device=DEV)
    i = torch.zeros((2, 100), dtype=torch.int32, device=DEV)
    with pytest.raises(F.FathomError) as e:
        F.topk_merge(s, i, 101)
    assert e.value.status == F.EINVAL


def _rows(inp, dev_or_host, interleaved):
    """bf16 K and V row views [Hkv][n][d] of the layer (one interleaved buffer,
    or two arrays), on the device or page-locked on the host."""
    Kb = torch.from_numpy(inp["K_rows"].view(np.int16)).view(torch.bfloat16)
    Vb = torch.from_numpy(inp["V_rows"].view(np.int16)).view(torch.bfloat16)
    host = dev_or_host == "host"
    Hkv, n, d = Kb.shape
    if interleaved:
        Kr, Vr = F.kv_rows(Hkv, n, d, device=None if host else DEV, pin_memory=host)
        Kr.copy_(Kb)
        Vr.copy_(Vb)
        return Kr, Vr
    if host:
        return Kb.pin_memory(), Vb.pin_memory()
    return Kb.to(DEV), Vb.to(DEV)


def _range_rows(inp, k0, k1, where, interleaved):
    sub = dict(K_rows=np.ascontiguousarray(inp["K_rows"][:, k0:k1]), V_rows=np.ascontiguousarray(inp["V_rows"][:, k0:k1]))
    return _rows(sub, where, interleaved)


def _rel_err(got, want):
    return float(((got - want).norm(dim=1) / want.norm(dim=1).clamp_min(1e-30)).max())


@pytest.mark.parametrize("n,world,k,where,interleaved", [(20000, 4, 2048, "device", False),
                                                          (9000, 3, 512, "host", True),
                                                          (3000, 4, 1500, "device", True)])
def test_sharded_attention_equals_unsplit(ref, n, world, k, where, interleaved):
    inp = synth.layer_inputs(2, layer=5, n=n, n_kv_heads=2, n_q_heads=8, needles=0, with_values=True)
    q = torch.from_numpy(inp["q_bf16"].view(np.int16)).to(DEV).view(torch.bfloat16)
    dep = F.alloc_depths(q, torch.from_numpy(inp["sigma2"]).to(DEV), 92)
    idx, _ = F.scan_topk(F.pack_bitplanes(torch.from_numpy(inp["K"]).to(DEV)), q, dep, k)
    Kf, Vf = _rows(inp, where, interleaved)
    want = F.sparse_attend(q, Kf, Vf, idx)
    parts = []
    for r in range(world):
        k0, k1 = shard_range(n, world, r)
        if k1 <= k0:
            parts.append(empty_partials(8, 128, DEV))
            continue
        Kl, Vl = _range_rows(inp, k0, k1, where, interleaved)
        parts.append(F.sparse_attend_partial(q, Kl, Vl, idx, k0))
    got = F.attend_merge(torch.stack(parts))
    assert _rel_err(got, want) <= 1e-5
    # and against the oracle's fp64 attention over the same rows
    oref = ref.attend(synth.bf16_bits_to_f32(inp["q_bf16"]), inp["K_rows"], inp["V_rows"], idx.cpu().numpy())
    assert _rel_err(got.cpu().double(), torch.from_numpy(oref)) <= 1e-3
    assert F.last_device_status() == 0


def test_attend_merge_empty_ranges_and_padding():
    """Heads whose rows all lie in one range (the other ranges contribute
    m = -inf, l = 0), and -1 padding, which a partial skips."""
    n, k = 5000, 64
    inp = synth.layer_inputs(2, layer=6, n=n, n_kv_heads=1, n_q_heads=4, needles=0, with_values=True)
    q = torch.from_numpy(inp["q_bf16"].view(np.int16)).to(DEV).view(torch.bfloat16)
    rng = np.random.default_rng(4)
    idx = np.stack([np.arange(k), 3072 + np.arange(k), rng.choice(n, k, replace=False),
                    rng.choice(n, k, replace=False)]).astype(np.int32)
    idx[3, -10:] = -1
    idx_d = torch.from_numpy(idx).to(DEV)
    Kf, Vf = _rows(inp, "device", True)
    want = torch.cat([F.sparse_attend(q[h:h + 1], Kf, Vf, idx_d[h:h + 1].contiguous()) for h in range(3)])
    want3 = F.sparse_attend(q[3:], Kf, Vf, idx_d[3:, :k - 10].contiguous())
    parts = []
    for k0, k1 in ((0, 3072), (3072, n)):
        Kl, Vl = _range_rows(inp, k0, k1, "device", True)
        parts.append(F.sparse_attend_partial(q, Kl, Vl, idx_d, k0))
    assert float(parts[1][0, 128]) == float("-inf") and float(parts[1][0, 129]) == 0.0
    assert float(parts[0][1, 128]) == float("-inf") and float(parts[0][1, 129]) == 0.0
    got = F.attend_merge(torch.stack(parts))
    assert _rel_err(got[:3], want) <= 1e-5
    assert _rel_err(got[3:], want3) <= 1e-5
    assert F.last_device_status() == 0
