"""The fidelity harness of bench.py (fidelity_refs, fidelity_of) against the oracle.

The harness measures a read policy's decode step against exact attention:
the softmax mass of the selected keys, the recall of the exact top-k (the k
largest q.k over the bf16 keys) and the relative error of the attention output
against dense attention over all keys.  It computes its references in fp32 on
the GPU.  Here the same metrics are computed on the CPU in fp64, with the
oracle's attention (dense: all keys selected) and its sort-based top-k, for the
same GPU decode step of a small layer, and the two must agree.
"""
import numpy as np
import pytest

import synth

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA GPU", allow_module_level=True)

import bench  # noqa: E402
from bit_plane_key_b200 import fathom as F  # noqa: E402

DEV = torch.device("cuda:0")


def _bf16_dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(DEV).view(torch.bfloat16)


@pytest.mark.parametrize("B,fixed_r", [(46, 0), (92, 0), (0, 16)])
def test_fidelity_metrics_match_oracle(ref, B, fixed_r):
    n, Hkv, Hq, d, k = 4096, 2, 8, 128, 256
    G = Hq // Hkv
    inp = synth.layer_inputs(2, n=n, n_kv_heads=Hkv, n_q_heads=Hq, d=d, with_values=True)
    q = _bf16_dev(inp["q_bf16"])
    Kr, Vr = _bf16_dev(inp["K_rows"]), _bf16_dev(inp["V_rows"])
    st = F.pack_bitplanes(torch.from_numpy(inp["K"]).to(DEV))
    _, idx, _, out = F.decode_step(st, q, torch.from_numpy(inp["sigma2"]).to(DEV), B, k, Kr, Vr, fixed_r=fixed_r)
    refs = bench.fidelity_refs(torch, q, Kr, Vr, k, G)
    m = bench.fidelity_of(torch, refs, idx, out)

    idx_h, out_h = idx.cpu().numpy(), out.cpu().numpy().astype(np.float64)
    qf = inp["q"].astype(np.float64)                                    # bf16 queries, widened
    Kf = synth.bf16_bits_to_f32(inp["K_rows"]).astype(np.float64)
    dense = ref.attend(inp["q"], inp["K_rows"], inp["V_rows"], np.tile(np.arange(n, dtype=np.int32), (Hq, 1)))
    exact_h = refs["exact_idx"].cpu().numpy()
    for h in range(Hq):
        g = h // G
        s = Kf[g] @ qf[h]                                               # exact scores, fp64
        exact = ref.topk(s, k)
        # the harness's exact top-k: the oracle's, except keys tied with the k-th score to fp32 rounding
        kth = s[exact[-1]]
        diff = set(exact_h[h].tolist()) ^ set(exact.tolist())
        assert all(abs(s[i] - kth) <= 1e-5 * np.abs(Kf[g][i] * qf[h]).sum() for i in diff), h
        z = s / np.sqrt(d)
        p = np.exp(z - z.max())
        p /= p.sum()
        mass = p[idx_h[h]].sum()
        assert abs(m["mass"][h] - mass) <= 1e-5, (h, m["mass"][h], mass)
        if not diff:
            assert m["recall"][h] == len(set(idx_h[h].tolist()) & set(exact.tolist())) / k
        err = np.linalg.norm(out_h[h] - dense[h]) / np.linalg.norm(dense[h])
        assert abs(m["err_dense"][h] - err) <= 1e-5 + 1e-3 * err, (h, m["err_dense"][h], err)
