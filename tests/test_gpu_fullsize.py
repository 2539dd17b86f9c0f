"""Parity at the workloads' full sizes, in the launch configuration bench.py times.

Inputs come from synth's GPU generator (seeded).  The oracle checks sampled
outputs: 64-aligned windows of keys are packed by the oracle from the same
synthetic keys (block scales depend only on a block's own keys), scored in
fp64 and compared key by key with the scan's scores.  The top-k is checked as
a property of the scan's own scores (it must be exactly the k largest, ties to
the lower index) and, where the workload plants them, by needle recall.
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
SCORE_RTOL = 1e-4
WINDOW = 1024


def windows(n, count, rng):
    starts = sorted(set(int(x) for x in rng.integers(0, max(1, (n - WINDOW) // 64), count) * 64))
    return [(s0, min(n, s0 + WINDOW)) for s0 in starts] + [((n - 1) // 64 * 64, n)]   # plus the ragged tail


def check_windows(ref, K_dev, q, dep_h, scores_h, n, rng, count=3, kv_heads=(0,), G=4, k_head_offset=0):
    """fp64 oracle scores of sampled key windows against the scan's scores.
    K_dev holds KV heads k_head_offset.. of the layer; q, dep_h, scores_h all query heads."""
    for g in kv_heads:
        for (i0, i1) in windows(n, count, rng):
            Kw = K_dev[g - k_head_offset:g - k_head_offset + 1, i0:i1].cpu().numpy()
            planes, scales = ref.pack(Kw)
            hs = slice(g * G, (g + 1) * G)
            s_ref, a_ref = ref.scores(planes, scales, i1 - i0, q[hs], dep_h[hs], with_abs=True)
            err = np.abs(scores_h[hs, i0:i1].astype(np.float64) - s_ref)
            assert np.all(err <= SCORE_RTOL * a_ref + 1e-30), (g, i0)


def check_topk_property(scores_row, idx_row, k):
    """idx must be the k largest of the row, ordered (score desc, index asc)."""
    n = scores_row.size
    s = scores_row.astype(np.float64)
    sel = s[idx_row]
    assert len(set(idx_row.tolist())) == k
    order = np.lexsort((idx_row, -sel))
    assert np.array_equal(order, np.arange(k))
    mask = np.ones(n, bool)
    mask[idx_row] = False
    kth = sel[-1]
    rest = s[mask]
    assert not np.any(rest > kth)
    ties = np.nonzero(mask & (s == kth))[0]
    assert ties.size == 0 or ties.min() > idx_row[sel == kth].max()


@pytest.mark.parametrize("budget,fixed_r", [(46, 0), (68, 0), (92, 0), (136, 0), (0, 16), (0, 32)])
def test_config2_layer_n131072(ref, budget, fixed_r):
    """Qwen3-8B-shaped layer, n = 131072, HBM-resident: B sweep and the fixed 68/136-bit scans."""
    rng = np.random.default_rng(budget + fixed_r)
    inp = synth.layer_inputs_cuda(2, n=131072, device=DEV, with_values=False)
    st = F.pack_bitplanes(inp["K"])
    dep = F.alloc_depths(inp["q_dev"], inp["sigma2_dev"], budget, fixed_r=fixed_r)
    dep_h = dep.cpu().numpy()
    assert np.array_equal(dep_h, ref.alloc_depths(inp["q"], inp["sigma2"], budget, fixed_r=fixed_r))
    ws = torch.empty(F.scan_workspace_bytes(st, 32, 2048), dtype=torch.uint8, device=DEV)
    idx, top = F.scan_topk(st, inp["q_dev"], dep, 2048, workspace=ws)
    scores = F.scan_scores_view(ws, 32, st.n_pad).cpu().numpy()[:, :131072]
    check_windows(ref, inp["K"], inp["q"], dep_h, scores, 131072, rng, kv_heads=[0, 5])
    idx_h = idx.cpu().numpy()
    for h in (0, 13, 31):
        check_topk_property(scores[h], idx_h[h], 2048)


def test_config3_layer_n1M_host_resident_needles(ref):
    """n = 2^20, planes in page-locked host memory, B = 92, k = 2048, 16 needles."""
    rng = np.random.default_rng(3)
    n = 1 << 20
    inp = synth.layer_inputs_cuda(3, n=n, device=DEV, with_values=False)
    st = F.pack_bitplanes(inp["K"]).to_host()
    dep = F.alloc_depths(inp["q_dev"], inp["sigma2_dev"], 92)
    dep_h = dep.cpu().numpy()
    assert np.array_equal(dep_h, ref.alloc_depths(inp["q"], inp["sigma2"], 92))
    ws = torch.empty(F.scan_workspace_bytes(st, 32, 2048), dtype=torch.uint8, device=DEV)
    idx, top = F.scan_topk(st, inp["q_dev"], dep, 2048, workspace=ws)
    scores = F.scan_scores_view(ws, 32, st.n_pad).cpu().numpy()[:, :n]
    check_windows(ref, inp["K"], inp["q"], dep_h, scores, n, rng, count=2, kv_heads=[0, 7])
    idx_h = idx.cpu().numpy()
    for h in (0, 31):
        check_topk_property(scores[h], idx_h[h], 2048)
    assert set(inp["needles"].tolist()) <= set(idx_h[0].tolist())   # every needle of query head 0 is found


def test_config4_sixteen_sessions_host_resident(ref):
    """16 sessions, n ~ U[64k, 512k] (multiples of 64), per-session sigma, B = 68, k = 1024, one batched call."""
    rng = synth.rng_for(4, 0, 9)
    lengths = (rng.integers(65536 // 64, 524288 // 64 + 1, 16) * 64).tolist()
    stores, qs, s2s, Ks, inps = [], [], [], [], []
    for sidx, n in enumerate(lengths):
        inp = synth.layer_inputs_cuda(4, layer=sidx, n=n, device=DEV, with_values=False)
        stores.append(F.pack_bitplanes(inp["K"]).to_host())
        qs.append(inp["q_dev"])
        s2s.append(inp["sigma2_dev"])
        Ks.append(inp["K"][:1].clone())  # KV head 0 kept for the oracle windows
        inps.append(inp)
        del inp["K"]
    q = torch.stack(qs)
    dep = F.alloc_depths(q.view(-1, 128), torch.cat(s2s), 68).view(16, 32, 128)
    ws = torch.empty(F.scan_batched_workspace_bytes(stores, 32, 1024), dtype=torch.uint8, device=DEV)
    idx, top = F.scan_topk_batched(stores, q, dep, 1024, workspace=ws)
    idx_h = idx.cpu().numpy()
    npr = np.random.default_rng(4)
    off = 0
    for sidx, n in enumerate(lengths):
        npad = F.n_pad(n)
        sc = ws[off: off + 4 * 32 * npad].view(torch.float32).view(32, npad).cpu().numpy()[:, :n]
        off += (4 * 32 * npad + 255) // 256 * 256
        if sidx % 4 == 0:
            dep_h = dep[sidx].cpu().numpy()
            check_windows(ref, Ks[sidx], inps[sidx]["q"], dep_h, sc, n, npr, count=1, kv_heads=[0])
        check_topk_property(sc[sidx % 32], idx_h[sidx, sidx % 32], 1024)
    assert F.last_device_status() == 0


def test_config5_decode_step_sampled_layers(ref):
    """36-layer decode step at n = 2^20, per-layer B ~ U[46, 136]: layers 0, 17, 35 checked end to end
    (depths, sampled scores, top-k property, exact attention over the selected rows)."""
    n = 1 << 20
    budgets = synth.rng_for(5, 0, 8).integers(46, 137, 36)
    for layer in (0, 17, 35):
        B = int(budgets[layer])
        inp = synth.layer_inputs_cuda(5, layer=layer, n=n, device=DEV, with_values=True)
        st = F.pack_bitplanes(inp["K"]).to_host()
        Kr, Vr = F.kv_rows(8, n, 128, pin_memory=True)   # interleaved host rows, as a server keeps them
        Kr.copy_(inp["K_rows"])
        Vr.copy_(inp["V_rows"])
        dep = F.alloc_depths(inp["q_dev"], inp["sigma2_dev"], B)
        dep_h = dep.cpu().numpy()
        assert np.array_equal(dep_h, ref.alloc_depths(inp["q"], inp["sigma2"], B))
        ws = torch.empty(F.scan_workspace_bytes(st, 32, 2048), dtype=torch.uint8, device=DEV)
        idx, top = F.scan_topk(st, inp["q_dev"], dep, 2048, workspace=ws)
        out = F.sparse_attend(inp["q_dev"], Kr, Vr, idx).cpu().numpy()
        scores = F.scan_scores_view(ws, 32, st.n_pad).cpu().numpy()[:, :n]
        check_windows(ref, inp["K"], inp["q"], dep_h, scores, n, np.random.default_rng(layer), count=1,
                      kv_heads=[layer % 8])
        idx_h = idx.cpu().numpy()
        check_topk_property(scores[layer % 32], idx_h[layer % 32], 2048)
        # exact attention of two heads, oracle on the gathered rows (bf16 bits)
        for h in (0, 29):
            g = h // 4
            rows = np.sort(idx_h[h])
            Kh = inp["K_rows"][g, torch.from_numpy(rows).to(DEV)].cpu().view(torch.int16).numpy().view(np.uint16)
            Vh = inp["V_rows"][g, torch.from_numpy(rows).to(DEV)].cpu().view(torch.int16).numpy().view(np.uint16)
            pos = {int(r): j for j, r in enumerate(rows)}
            local = np.array([[pos[int(r)] for r in idx_h[h]]], np.int32)
            o_ref = ref.attend(inp["q"][h:h + 1], Kh[None], Vh[None], local)[0]
            assert np.linalg.norm(out[h] - o_ref) <= 1e-3 * np.linalg.norm(o_ref)
        del inp, st, Kr, Vr
        torch.cuda.empty_cache()
    assert F.last_device_status() == 0


def test_config3_decode_step_as_benchmarked(ref):
    """The call bench.py times, at its size: one fathom_decode_step on the n = 2^20 layer with the planes, the
    scales and the interleaved K|V rows in page-locked host memory, B = 92, k = 2048, one KV-head group (the
    top-k takes its block-maxima path: 16384 blocks >= 8k).  Depths bit-exact; sampled scores of every KV head
    against fp64; the complete top-k property of all 32 heads on the scan's own scores; every needle found;
    exact attention of heads in four KV groups against fp64; the one-call step equal to the separate calls."""
    n, k, B = 1 << 20, 2048, 92
    inp = synth.layer_inputs_cuda(3, n=n, device=DEV, with_values=True)
    q = inp["q_dev"]
    st = F.pack_bitplanes(inp["K"]).to_host()
    Kr, Vr = F.kv_rows(8, n, 128, pin_memory=True)
    Kr.copy_(inp["K_rows"])
    Vr.copy_(inp["V_rows"])
    dep, idx, top, out = F.decode_step(st, q, inp["sigma2_dev"], B, k, Kr, Vr, kv_groups=1)
    torch.cuda.synchronize()
    dep_h = dep.cpu().numpy()
    assert np.array_equal(dep_h, ref.alloc_depths(inp["q"], inp["sigma2"], B))

    # the same step as separate calls: bit for bit
    bmax = F.block_max_buffer(32, n, DEV)
    scores = F.scan_scores(st, q, dep, block_max=bmax)
    idx2, top2 = F.scan_topk(st, q, dep, k)
    out2 = F.sparse_attend(q, Kr, Vr, idx2)
    assert torch.equal(idx, idx2)
    assert torch.equal(top.view(torch.int32), top2.view(torch.int32))
    assert torch.equal(out.view(torch.int32), out2.view(torch.int32))

    scores_h = scores.cpu().numpy()[:, :n]
    check_windows(ref, inp["K"], inp["q"], dep_h, scores_h, n, np.random.default_rng(33), count=1,
                  kv_heads=list(range(8)))
    idx_h = idx.cpu().numpy()
    for h in range(32):
        check_topk_property(scores_h[h], idx_h[h], k)
    assert set(inp["needles"].tolist()) <= set(idx_h[0].tolist())

    o = out.cpu().numpy()
    for h in (0, 9, 18, 27):
        g = h // 4
        rows = np.sort(idx_h[h])
        sel = torch.from_numpy(rows).to(DEV)
        Kh = inp["K_rows"][g, sel].cpu().view(torch.int16).numpy().view(np.uint16)
        Vh = inp["V_rows"][g, sel].cpu().view(torch.int16).numpy().view(np.uint16)
        pos = {int(r): j for j, r in enumerate(rows)}
        local = np.array([[pos[int(r)] for r in idx_h[h]]], np.int32)
        o_ref = ref.attend(inp["q"][h:h + 1], Kh[None], Vh[None], local)[0]
        assert np.linalg.norm(o[h] - o_ref) <= 1e-3 * np.linalg.norm(o_ref), h
    assert F.last_device_status() == 0
