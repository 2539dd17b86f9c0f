"""Key-range sharding, emulated on one GPU: the layer's keys are split into
four 1024-aligned ranges, each range is packed and scanned on its own and
takes its local top-k, the lists are laid side by side as the all-gather
would lay them, and fathom_topk_merge must return exactly the top-k of the
unsplit layer (indices and scores, bit for bit)."""
import numpy as np
import pytest

import synth

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA GPU", allow_module_level=True)

from bit_plane_key_b200 import fathom as F  # noqa: E402
from bit_plane_key_b200.shard import local_topk, shard_range  # noqa: E402

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
