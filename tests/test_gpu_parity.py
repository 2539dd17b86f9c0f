"""GPU parity: every step of the path through the C ABI against the oracle.

Bit-exact: packing (planes and scales), depths, top-k indices of given
scores.  Tolerance: scan scores, |s_gpu - s_ref| <= 1e-4 * sum_c |q_c khat_c|
(fp32 accumulation of at most 2d terms; worst case a few 1e-5); attention,
||o - o_ref|| <= 1e-3 ||o_ref||.  Top-k of the scan against the fp64 oracle:
equal index sets except keys whose fp64 score lies within the score
tolerance of the k-th score.
"""
import ctypes
import json
import os

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
GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def dev(a):
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).to(DEV)
    if a.dtype == np.uint32:
        return torch.from_numpy(a.view(np.int32)).to(DEV)
    return torch.from_numpy(a).to(DEV)


def bf16(a_bits):
    return dev(a_bits).view(torch.bfloat16)


def host(t, dtype=None):
    a = t.detach().cpu().numpy()
    return a.view(dtype) if dtype is not None else a


def make(config=1, n=None, Hkv=None, Hq=None, d=None, q_bf16=None, values=False, needles=None, layer=0):
    inp = synth.layer_inputs(config, layer=layer, n=n, n_kv_heads=Hkv, n_q_heads=Hq, d=d, with_values=values,
                             needles=needles)
    if q_bf16 is not None and q_bf16 and "q_bf16" not in inp:
        inp["q_bf16"] = synth.f32_to_bf16_bits(inp["q"])
        inp["q"] = synth.bf16_bits_to_f32(inp["q_bf16"])
    return inp


def q_dev(inp):
    return bf16(inp["q_bf16"]) if "q_bf16" in inp else dev(inp["q"])


def check_scores(ref, planes_np, scales_np, n, q, dep, s_gpu, i0=0, i1=None):
    i1 = n if i1 is None else i1
    s_ref, a_ref = ref.scores(planes_np, scales_np, n, q, dep, i0, i1, with_abs=True)
    err = np.abs(s_gpu[:, i0:i1].astype(np.float64) - s_ref)
    tol = SCORE_RTOL * a_ref + 1e-30
    bad = err > tol
    assert not bad.any(), "score mismatch at %s: gpu %s ref %s" % (
        np.argwhere(bad)[:5].tolist(), s_gpu[:, i0:i1][bad][:5], s_ref[bad][:5])
    return s_ref, a_ref


# --------------------------------------------------------------------------
# a0: packing, bit-exact
# --------------------------------------------------------------------------
@pytest.mark.parametrize("n,Hkv,d", [(4096, 1, 128), (1, 1, 32), (63, 2, 64), (64, 1, 32), (4097, 2, 128),
                                     (1000, 3, 256), (130, 1, 96)])
def test_pack_bit_exact(ref, n, Hkv, d):
    inp = make(1, n=n, Hkv=Hkv, Hq=Hkv, d=d)
    K = inp["K"]
    K[0, : min(n, 64), 0] = 0.0          # an all-zero block: Delta = 0
    st = F.pack_bitplanes(dev(K))
    planes, scales = ref.pack(K)
    assert np.array_equal(host(st.planes, np.uint32), planes)
    assert np.array_equal(host(st.scales, np.uint16), scales)


def test_pack_bf16_input(ref):
    inp = make(1, n=777, Hkv=2, Hq=2, d=128)
    kb = synth.f32_to_bf16_bits(inp["K"])
    st = F.pack_bitplanes(bf16(kb))
    planes, scales = ref.pack(synth.bf16_bits_to_f32(kb))
    assert np.array_equal(host(st.planes, np.uint32), planes)
    assert np.array_equal(host(st.scales, np.uint16), scales)


def test_pack_edge_values(ref):
    """Keys at cell edges, +-amax, tiny and huge magnitudes."""
    rng = np.random.default_rng(5)
    n, d = 256, 32
    K = (rng.standard_normal((1, n, d)) * 10.0 ** rng.integers(-6, 6, (1, 1, d))).astype(np.float32)
    for c in range(d):
        amax = np.max(np.abs(K[0, :64, c]))
        delta = np.float32(np.float16(amax / np.float32(8)))
        K[0, 1:17, c] = (np.arange(-8, 8) * delta).astype(np.float32)   # exact cell edges
        K[0, 17, c] = -amax
    st = F.pack_bitplanes(dev(K))
    planes, scales = ref.pack(K)
    assert np.array_equal(host(st.planes, np.uint32), planes)
    assert np.array_equal(host(st.scales, np.uint16), scales)


# --------------------------------------------------------------------------
# a1-a2, a7: depths, bit-exact
# --------------------------------------------------------------------------
@pytest.mark.parametrize("d", [32, 128, 256])
@pytest.mark.parametrize("qtype", ["f32", "bf16"])
def test_depths_bit_exact(ref, d, qtype):
    rng = np.random.default_rng(d)
    Hkv, G = 2, 4
    sig = synth.channel_sigma(rng, Hkv, d)
    s2 = (sig * sig).astype(np.float32)
    q = rng.standard_normal((Hkv * G, d)).astype(np.float32)
    q[0, :5] = 0.0
    q[1] = 1.0                          # equal importances: tie rule
    if qtype == "bf16":
        qb = synth.f32_to_bf16_bits(q)
        qd, qf = bf16(qb), synth.bf16_bits_to_f32(qb)
    else:
        qd, qf = dev(q), q
    s2d = dev(s2)
    for B in (0, 1, 7, 46, 64, 68, 92, 136, 4 * d - 1, 4 * d, 4 * d + 50):
        got = host(F.alloc_depths(qd, s2d, B))
        want = ref.alloc_depths(qf, s2, B)
        assert np.array_equal(got, want), B
        assert np.all(got.sum(1) == min(B, 4 * d))
    for r in (1, 16, 32, d):
        got = host(F.alloc_depths(qd, s2d, 0, fixed_r=r))
        assert np.array_equal(got, ref.alloc_depths(qf, s2, 0, fixed_r=r)), r


def test_depths_extreme_importance(ref):
    """Subnormal, zero and huge importances keep the exact order."""
    d = 128
    rng = np.random.default_rng(1)
    q = rng.standard_normal((4, d)).astype(np.float32)
    s2 = np.exp(rng.uniform(-100, 80, (1, d))).astype(np.float32)
    s2[0, :4] = [0.0, 1e-45, 3e38, 1e-40]
    for B in (10, 92, 300):
        got = host(F.alloc_depths(dev(q), dev(s2), B))
        assert np.array_equal(got, ref.alloc_depths(q, s2, B)), B


@pytest.mark.parametrize("G", [1, 2, 4, 8])
def test_pooled_depths_bit_exact(ref, G):
    """Group-pooled depths (the comparison variant) equal the oracle's, and the
    scan over them reads exactly min(B, 4d) plane bits per key."""
    rng = np.random.default_rng(50 + G)
    Hkv, d = 2, 128
    sig = synth.channel_sigma(rng, Hkv, d)
    s2 = (sig * sig).astype(np.float32)
    qb = synth.f32_to_bf16_bits(rng.standard_normal((Hkv * G, d)).astype(np.float32))
    qd, qf = bf16(qb), synth.bf16_bits_to_f32(qb)
    for B in (0, 5, 46, 92, 136, 4 * d, 4 * d + 9):
        got = host(F.alloc_depths_pooled(qd, dev(s2), B))
        assert np.array_equal(got, ref.alloc_depths_pooled(qf, s2, B)), B
        assert np.all(got.reshape(Hkv, G, d) == got.reshape(Hkv, G, d)[:, :1])
        assert np.all(got.sum(1) == min(B, 4 * d))


# --------------------------------------------------------------------------
# a4: scan scores within tolerance (+ the basis rule at every depth)
# --------------------------------------------------------------------------
@pytest.mark.parametrize("case", ["config1", "gqa_ragged", "d256_g2", "g8", "depth_mix", "depth_mix_g8",
                                  "depth_mix_g2_tail", "depth_mix_g1"])
def test_scan_scores(ref, case):
    if case == "config1":
        inp = make(1)                                       # Hkv=1, n=4096, d=128, f32 q
        B = 64
    elif case == "gqa_ragged":
        inp = make(2, n=5000, Hkv=2, Hq=8, d=128)           # bf16 q, GQA 4, ragged tail
        B = 92
    elif case == "d256_g2":
        inp = make(1, n=3000, Hkv=2, Hq=4, d=256)
        B = 136
    elif case == "g8":
        inp = make(2, n=1100, Hkv=1, Hq=8, d=64)
        B = 46
    elif case == "depth_mix":
        inp = make(1, n=2100, Hkv=1, Hq=4, d=128)
        B = None
    elif case == "depth_mix_g8":                            # two head groups of 4 per KV head
        inp = make(2, n=7000, Hkv=2, Hq=16, d=96)
        B = None
    elif case == "depth_mix_g2_tail":                       # several full tiles and a half tile
        inp = make(2, n=9217, Hkv=3, Hq=6, d=64)
        B = None
    else:
        inp = make(1, n=4100, Hkv=2, Hq=2, d=256)
        B = None
    K, q = inp["K"], inp["q"]
    n = K.shape[1]
    st = F.pack_bitplanes(dev(K))
    planes, scales = ref.pack(K)
    if B is None:   # arbitrary depths 0..4 in every head: heads read less than the union
        dep = np.random.default_rng(3).integers(0, 5, q.shape).astype(np.uint8)
    else:
        dep = ref.alloc_depths(q, inp["sigma2"], B)
    s = host(F.scan_scores(st, q_dev(inp), dev(dep)))
    assert s.shape == (q.shape[0], F.n_pad(n))
    assert np.all(np.isneginf(s[:, n:]))
    check_scores(ref, planes, scales, n, q, dep, s)


@pytest.mark.parametrize("Hkv,Hq", [(64, 64), (52, 208)])
def test_scan_scores_wide_grid(ref, Hkv, Hq):
    """Many KV heads (64 heads of one query, 52 heads of four): grids of
    1820-2240 CTAs, more than the SMs hold at once, so tiles of one head run
    in different waves; each head's last 2048-key tile is a half tile and its
    last block ragged, and depths 0..4 vary per channel and head.  Device- and
    host-resident stores give the same scores."""
    inp = make(2, n=70000, Hkv=Hkv, Hq=Hq, d=32)
    st = F.pack_bitplanes(dev(inp["K"]))
    planes, scales = ref.pack(inp["K"])
    dep = np.random.default_rng(5).integers(0, 5, inp["q"].shape).astype(np.uint8)
    s = host(F.scan_scores(st, q_dev(inp), dev(dep)))
    assert np.all(np.isneginf(s[:, 70000:]))
    check_scores(ref, planes, scales, 70000, inp["q"], dep, s)
    assert np.array_equal(host(F.scan_scores(st.to_host(), q_dev(inp), dev(dep))), s)


def test_scan_all_depths_uniform(ref):
    """t = 0..4 for every channel: full-depth and zero-depth corners."""
    inp = make(1, n=700, Hkv=1, Hq=1, d=128)
    st = F.pack_bitplanes(dev(inp["K"]))
    planes, scales = ref.pack(inp["K"])
    for t in range(5):
        dep = np.full((1, 128), t, np.uint8)
        s = host(F.scan_scores(st, dev(inp["q"]), dev(dep)))
        if t == 0:
            assert np.all(s[:, :700] == 0.0)
        check_scores(ref, planes, scales, 700, inp["q"], dep, s)


def test_scan_bad_depth_flagged(ref):
    inp = make(1, n=256, Hkv=1, Hq=1, d=32)
    st = F.pack_bitplanes(dev(inp["K"]))
    dep = np.full((1, 32), 2, np.uint8)
    dep[0, 3] = 9
    F.last_device_status()
    s = host(F.scan_scores(st, dev(inp["q"]), dev(dep)))
    assert F.last_device_status() & F.DEV_BAD_DEPTH
    planes, scales = ref.pack(inp["K"])
    dep[0, 3] = 0            # the bad channel is skipped
    check_scores(ref, planes, scales, 256, inp["q"], dep, s)
    assert F.last_device_status() == 0


def test_six_key_example_on_gpu():
    with open(os.path.join(GOLDEN, "six_key_example.json")) as f:
        ex = json.load(f)
    K = np.array(ex["keys_x"], np.float32)[None]
    q = np.array(ex["q"], np.float32)[None]
    s2 = np.array(ex["sigma2"], np.float32)[None]
    # d must be a multiple of 32: pad channels with zero keys, zero q, zero sigma2
    Kp = np.zeros((1, 6, 32), np.float32)
    Kp[:, :, :4] = K
    qp = np.zeros((1, 32), np.float32)
    qp[:, :4] = q
    s2p = np.zeros((1, 32), np.float32)
    s2p[:, :4] = s2
    st = F.pack_bitplanes(dev(Kp))
    for B, want in ex["expected_scores"].items():
        dep = host(F.alloc_depths(dev(qp), dev(s2p), int(B)))
        assert dep[0, :4].tolist() == ex["expected_depths"][B]
        s = host(F.scan_scores(st, dev(qp), dev(dep)))[0, :6]
        np.testing.assert_allclose(s, want, rtol=0, atol=1e-5)
        idx, _ = F.scan_topk(st, dev(qp), dev(dep), 3)
        assert host(idx)[0].tolist() == ex["expected_top3"][B]


# --------------------------------------------------------------------------
# a5: top-k, bit-exact on given scores
# --------------------------------------------------------------------------
@pytest.mark.parametrize("n,rows,k,kind", [
    (100, 3, 1, "normal"), (100, 3, 100, "normal"), (4096, 2, 64, "normal"), (20000, 4, 2048, "normal"),
    (131072, 2, 2048, "normal"), (200000, 2, 4096, "ties"), (50000, 2, 2048, "equal"),
    (70000, 2, 1000, "narrow"), (4096, 1, 4096, "ties"), (9000, 1, 4096, "ties"),
    (300000, 2, 2048, "normal"), (140000, 2, 1000, "narrow"), (140000, 1, 3000, "equal")])
def test_topk_bit_exact(ref, n, rows, k, kind):
    """Rows up to 131072 keys take the one-kernel cluster path (1, 2, 4 or 8
    CTAs per row), longer rows the multi-pass histogram path."""
    rng = np.random.default_rng(n + k)
    if kind == "normal":
        s = rng.standard_normal((rows, n)).astype(np.float32)
    elif kind == "ties":
        s = np.round(rng.standard_normal((rows, n)), 1).astype(np.float32)
    elif kind == "equal":
        s = np.full((rows, n), 1.5, np.float32)
        s[:, ::7] = -2.0
    else:  # one octave, 12-bit bins overflow: forces the deeper levels
        s = (1.0 + rng.random((rows, n)) * 1e-3).astype(np.float32)
    ld = n + 5
    sd = torch.full((rows, ld), float("nan"), device=DEV)
    sd[:, :n] = dev(s)
    idx, top = F.topk(sd, n, k)
    idx, top = host(idx), host(top)
    for r in range(rows):
        want = ref.topk(s[r], k)
        assert np.array_equal(idx[r], want), r
        assert np.array_equal(top[r], s[r][want])
    assert F.last_device_status() == 0


@pytest.mark.parametrize("n,B,k", [(20000, 92, 2048), (5000, 46, 700), (70000, 0, 1024), (131072, 136, 4096),
                                    (3000, 92, 3000), (131072, 92, 2048), (100000, 68, 1500), (4096, 92, 64),
                                    (65536, 46, 512), (300000, 92, 2048), (150001, 46, 777), (1 << 20, 68, 4096),
                                    (200000, 0, 1000), (524288, 136, 64), (131073, 92, 2048), (131073, 92, 3000)])
def test_topk_from_block_maxima_equals_full_selection(n, B, k):
    """The scan's block maxima let top-k read only the blocks that can hold a
    selected key; the result must equal the selection over the whole rows bit
    for bit (B = 0: every score ties, the candidates overflow and the full-row
    path takes the lowest indices)."""
    inp = make(2, n=n, Hkv=2, Hq=8, layer=B)
    st = F.pack_bitplanes(dev(inp["K"]))
    dep = F.alloc_depths(q_dev(inp), dev(inp["sigma2"]), B)
    bm = F.block_max_buffer(8, n, DEV)
    sc = F.scan_scores(st, q_dev(inp), dep, block_max=bm)
    i_blk, t_blk = F.topk(sc, n, k, block_max=bm)
    i_all, t_all = F.topk(sc, n, k)
    assert torch.equal(i_blk, i_all) and torch.equal(t_blk, t_all)
    i_st, t_st = F.scan_topk(st, q_dev(inp), dep, k)
    assert torch.equal(i_st, i_all) and torch.equal(t_st, t_all)
    if B == 0:
        assert np.array_equal(host(i_blk), np.tile(np.arange(k, dtype=np.int32), (8, 1)))
    assert F.last_device_status() == 0


def _ordered_keys(s):
    """Order-preserving u32 keys of fp32 scores (the block-maximum format)."""
    u = np.ascontiguousarray(s, dtype=np.float32).view(np.uint32).copy()
    u[u == 0x80000000] = 0
    neg = (u & 0x80000000) != 0
    return np.where(neg, ~u, u | np.uint32(0x80000000)).astype(np.uint32)


@pytest.mark.parametrize("long_rows", [False, True])
@pytest.mark.parametrize("case", ["ties_at_bound", "k_equals_blocks", "top_in_one_block", "ragged_tail",
                                  "all_equal", "rounded_ties"])
def test_topk_block_maxima_bound_edge_cases(ref, case, long_rows):
    """Rows with at least k blocks, given block maxima computed here.  Short
    rows (<= 131072 keys) take the one-kernel cluster path over the scores;
    long rows the cluster path over the block maxima, which keeps the keys at
    or above the 24-bit bin of the k-th largest block maximum.  Scores built so
    that all selected keys tie at the k-th block maximum, the top keys sit in
    one block or in a ragged last block, every score is equal (the candidates
    overflow and the row is selected exactly from all its keys), or scores are
    rounded so that ties pile up; checked against the oracle bit for bit."""
    rng = np.random.default_rng(11)
    rows, n = 2, 131072
    if case == "ragged_tail":
        n = 100003
    if long_rows:
        n = 4 * n + 17
    nbk = -(-n // 64)
    s = rng.uniform(-1.0, 1.0, (rows, n)).astype(np.float32)
    if case == "ties_at_bound":
        k = min(nbk, 4096)
        s[:, ::64] = 5.0                     # every block's maximum is 5.0: the top k all tie there
    elif case == "k_equals_blocks":
        k = min(nbk, 4096)
        s[:, ::64] = rng.uniform(2.0, 3.0, (rows, nbk)).astype(np.float32)
    elif case == "top_in_one_block":
        k = 1000
        s[:, 64:128] = 10.0 + np.arange(64, dtype=np.float32)
    elif case == "all_equal":
        k = 1000
        s[:] = 1.5
    elif case == "rounded_ties":
        k = 2048
        s = np.round(rng.standard_normal((rows, n)), 1).astype(np.float32)
    else:
        k = 1563
        s[:, -3:] = 7.0                      # the partial last block holds the largest keys
    ld = ((n + 1023) // 1024) * 1024
    sd = torch.full((rows, ld), float("-inf"), device=DEV)
    sd[:, :n] = dev(s)
    pad = np.full((rows, nbk * 64), -np.inf, np.float32)
    pad[:, :n] = s
    bm = np.zeros((rows, ld // 64), np.uint32)
    bm[:, :nbk] = _ordered_keys(pad.reshape(rows, nbk, 64).max(axis=2))
    idx, top = F.topk(sd, n, k, block_max=dev(bm))
    idx, top = host(idx), host(top)
    for r in range(rows):
        want = ref.topk(s[r], k)
        assert np.array_equal(idx[r], want), (case, r)
        assert np.array_equal(top[r], s[r][want])
    assert F.last_device_status() == 0


@pytest.mark.parametrize("kind", ["normal", "ties", "narrow"])
@pytest.mark.parametrize("n", [65536, 262144])
def test_topk_repeatable_under_load(ref, kind, n):
    """The same rows, 20 launches back to back with many rows in flight: every
    launch must give the oracle's exact answer (a race in the selection or the
    final sort shows up as a launch that differs)."""
    rng = np.random.default_rng(7)
    rows, k = 32, 2048
    if kind == "normal":
        s = rng.standard_normal((rows, n)).astype(np.float32)
    elif kind == "ties":
        s = np.round(rng.standard_normal((rows, n)), 1).astype(np.float32)
    else:
        s = (1.0 + rng.random((rows, n)) * 1e-3).astype(np.float32)
    sd = dev(s)
    ws = torch.empty(F.topk_workspace_bytes(n, rows, k), dtype=torch.uint8, device=DEV)
    outs = [F.topk(sd, n, k, workspace=ws) for _ in range(20)]
    want = np.stack([ref.topk(s[r], k) for r in range(rows)])
    for idx, top in outs:
        assert np.array_equal(host(idx), want)
    assert F.last_device_status() == 0


# --------------------------------------------------------------------------
# a4 + a5 against the fp64 oracle
# --------------------------------------------------------------------------
def topk_sets_agree(ref, s_ref, a_ref, idx_gpu, k):
    """Equal sets, except keys whose fp64 score is within tolerance of the k-th."""
    want = ref.topk(s_ref, k)
    kth = s_ref[want[-1]]
    band = np.abs(s_ref - kth) <= 2 * SCORE_RTOL * a_ref
    gw, ww = set(idx_gpu.tolist()), set(want.tolist())
    diff = gw.symmetric_difference(ww)
    assert all(band[i] for i in diff), sorted(diff)[:10]


@pytest.mark.parametrize("config,n,Hkv,Hq,B,k", [(1, 4096, 1, 1, 64, 64), (2, 9000, 2, 8, 92, 2048),
                                                 (2, 20000, 1, 4, 68, 1024), (2, 3000, 2, 8, 0, 16)])
def test_scan_topk_vs_fp64(ref, config, n, Hkv, Hq, B, k):
    inp = make(config, n=n, Hkv=Hkv, Hq=Hq)
    K, q = inp["K"], inp["q"]
    st = F.pack_bitplanes(dev(K))
    planes, scales = ref.pack(K)
    dep = host(F.alloc_depths(q_dev(inp), dev(inp["sigma2"]), B))
    assert np.array_equal(dep, ref.alloc_depths(q, inp["sigma2"], B))
    idx, top = F.scan_topk(st, q_dev(inp), dev(dep), k)
    idx, top = host(idx), host(top)
    s_ref, a_ref = ref.scores(planes, scales, n, q, dep, with_abs=True)
    for h in range(Hq):
        topk_sets_agree(ref, s_ref[h], a_ref[h], idx[h], k)
        assert np.all(np.diff(top[h]) <= 0)
        assert len(set(idx[h].tolist())) == k
    if B == 0:
        assert np.array_equal(idx, np.tile(np.arange(k), (Hq, 1)))


def test_scan_topk_consistent_with_own_scores(ref):
    """Given the scan's own fp32 scores, the top-k is exactly (score desc, index asc)."""
    inp = make(2, n=12345, Hkv=2, Hq=8)
    st = F.pack_bitplanes(dev(inp["K"]))
    dep = F.alloc_depths(q_dev(inp), dev(inp["sigma2"]), 92)
    ws = torch.empty(F.scan_workspace_bytes(st, 8, 512), dtype=torch.uint8, device=DEV)
    idx, top = F.scan_topk(st, q_dev(inp), dep, 512, workspace=ws)
    s = host(F.scan_scores_view(ws, 8, st.n_pad))[:, :12345]
    idx = host(idx)
    for h in range(8):
        order = np.lexsort((np.arange(12345), -s[h].astype(np.float64)))[:512]
        assert np.array_equal(idx[h], order)


# --------------------------------------------------------------------------
# a3: host-resident store gives the same scan
# --------------------------------------------------------------------------
def test_host_resident_store(ref):
    """Host-resident and device-resident stores give the same scan, both
    within the score tolerance of the oracle."""
    for Hq in (8, 4):   # GQA groups of 4 and of 2
        inp = make(2, n=7000, Hkv=2, Hq=Hq)
        st = F.pack_bitplanes(dev(inp["K"]))
        hst = st.to_host()
        dep = F.alloc_depths(q_dev(inp), dev(inp["sigma2"]), 92)
        s_dev = host(F.scan_scores(st, q_dev(inp), dep))
        s_host = host(F.scan_scores(hst, q_dev(inp), dep))
        planes, scales = ref.pack(inp["K"])
        s_ref, a_ref = check_scores(ref, planes, scales, 7000, inp["q"], host(dep), s_host)
        check_scores(ref, planes, scales, 7000, inp["q"], host(dep), s_dev)
        assert np.array_equal(s_dev, s_host)
        i_dev, _ = F.scan_topk(st, q_dev(inp), dep, 700)
        i_host, _ = F.scan_topk(hst, q_dev(inp), dep, 700)
        for h in range(Hq):
            topk_sets_agree(ref, s_ref[h], a_ref[h], host(i_dev)[h], 700)
            topk_sets_agree(ref, s_ref[h], a_ref[h], host(i_host)[h], 700)


def test_residency_mismatch_rejected():
    inp = make(1, n=300, Hkv=1, Hq=1, d=32)
    st = F.pack_bitplanes(dev(inp["K"]))
    dep = F.alloc_depths(dev(inp["q"]), dev(inp["sigma2"]), 10)
    pageable = F.Store(st.planes.cpu(), st.scales.cpu(), 300, host_resident=True)
    with pytest.raises(F.FathomError) as e:
        F.scan_scores(pageable, dev(inp["q"]), dep)
    assert e.value.status == F.EINVAL
    wrong = F.Store(st.planes, st.scales, 300, host_resident=True)
    with pytest.raises(F.FathomError):
        F.scan_scores(wrong, dev(inp["q"]), dep)
    with pytest.raises(F.FathomError) as e:
        F.scan_topk(st, dev(inp["q"]), dep, 301)
    assert e.value.status == F.EINVAL
    with pytest.raises(F.FathomError) as e:
        F.scan_topk(st, dev(inp["q"]), dep, 10, workspace=torch.empty(64, dtype=torch.uint8, device=DEV))
    assert e.value.status == F.ENOMEM


# --------------------------------------------------------------------------
# a6: exact sparse attention
# --------------------------------------------------------------------------
@pytest.mark.parametrize("d,k,host_rows,interleaved", [
    (128, 2048, False, False), (128, 5, False, False), (64, 300, False, False), (256, 64, False, False),
    (32, 1, False, False), (128, 1000, True, False), (128, 1000, True, True), (64, 777, False, True),
    (256, 300, True, True)])
def test_sparse_attend(ref, d, k, host_rows, interleaved):
    rng = np.random.default_rng(d + k)
    Hkv, G, n = 2, 4, 5000
    inp = make(2, n=n, Hkv=Hkv, Hq=Hkv * G, d=d, values=True)
    idx = np.stack([rng.choice(n, k, replace=False) for _ in range(Hkv * G)]).astype(np.int32)
    Kr, Vr = bf16(inp["K_rows"]), bf16(inp["V_rows"])
    if interleaved:   # one [Hkv][n][2][d] buffer, row stride 2d
        Ki, Vi = F.kv_rows(Hkv, n, d, device=None if host_rows else DEV, pin_memory=host_rows)
        Ki.copy_(Kr)
        Vi.copy_(Vr)
        assert Ki.stride(1) == 2 * d
        Kr, Vr = Ki, Vi
    elif host_rows:
        Kr, Vr = Kr.cpu().pin_memory(), Vr.cpu().pin_memory()
    out = host(F.sparse_attend(q_dev(inp), Kr, Vr, dev(idx)))
    want = ref.attend(inp["q"], inp["K_rows"], inp["V_rows"], idx)
    for h in range(Hkv * G):
        assert np.linalg.norm(out[h] - want[h]) <= 1e-3 * np.linalg.norm(want[h]), h
    assert F.last_device_status() == 0


@pytest.mark.parametrize("order", ["rising", "falling"])
@pytest.mark.parametrize("d", [32, 128, 256])
def test_sparse_attend_running_maximum_moves(ref, d, order):
    """Rows given in order of rising exact score make the running maximum of
    every lane group move again and again (the rescale branch on almost every
    row); falling order takes it once.  q is scaled up so the logits span a
    wide range (softmax weights from 1 down to far below fp32's epsilon)."""
    Hkv, G, n, k = 1, 4, 6000, 1500
    inp = make(2, n=n, Hkv=Hkv, Hq=Hkv * G, d=d, values=True)
    q = (inp["q"] * 12.0).astype(np.float32)
    Kf = synth.bf16_bits_to_f32(inp["K_rows"]).astype(np.float64)
    rng = np.random.default_rng(d)
    idx = np.empty((G, k), dtype=np.int32)
    for h in range(G):
        sel = rng.choice(n, k, replace=False)
        s = Kf[0][sel] @ q[h].astype(np.float64)
        sel = sel[np.argsort(s, kind="stable")]
        idx[h] = sel if order == "rising" else sel[::-1]
    out = host(F.sparse_attend(dev(q), bf16(inp["K_rows"]), bf16(inp["V_rows"]), dev(idx)))
    want = ref.attend(q, inp["K_rows"], inp["V_rows"], idx)
    for h in range(G):
        assert np.linalg.norm(out[h] - want[h]) <= 1e-4 * np.linalg.norm(want[h]), (h, order)
    assert F.last_device_status() == 0


def test_sparse_attend_rejects_bad_row_stride():
    inp = make(2, n=300, Hkv=1, Hq=4, d=128, values=True)
    Kr, Vr = bf16(inp["K_rows"]), bf16(inp["V_rows"])
    idx = dev(np.tile(np.arange(10, dtype=np.int32), (4, 1)))
    out = torch.empty((4, 128), dtype=torch.float32, device=DEV)
    q = q_dev(inp)
    s = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for stride in (127, 100, 0):   # below d, or not a multiple of 8
        rc = F.lib().fathom_sparse_attend(ctypes.c_void_p(q.data_ptr()), F.BF16, ctypes.c_void_p(Kr.data_ptr()),
                                          ctypes.c_void_p(Vr.data_ptr()), stride, 0, ctypes.c_void_p(idx.data_ptr()),
                                          4, 1, 300, 128, 10, ctypes.c_void_p(out.data_ptr()), s)
        assert rc == F.EINVAL, stride


def test_sparse_attend_bad_index_flagged(ref):
    inp = make(2, n=300, Hkv=1, Hq=4, d=128, values=True)
    idx = np.tile(np.arange(10, dtype=np.int32), (4, 1))
    idx[1, 3] = 300
    idx[2, 0] = -1
    F.last_device_status()
    out = host(F.sparse_attend(q_dev(inp), bf16(inp["K_rows"]), bf16(inp["V_rows"]), dev(idx)))
    assert F.last_device_status() & F.DEV_BAD_INDEX
    want = ref.attend(inp["q"][:1], inp["K_rows"], inp["V_rows"], idx[:1])
    assert np.linalg.norm(out[0] - want[0]) <= 1e-3 * np.linalg.norm(want[0])
    ok = np.delete(idx[1], 3)[None]
    want1 = ref.attend(inp["q"][1:2], inp["K_rows"], inp["V_rows"], ok)
    assert np.linalg.norm(out[1] - want1[0]) <= 1e-3 * np.linalg.norm(want1[0])


# --------------------------------------------------------------------------
# batched sessions (ragged lengths, per-session sigma, mixed residency)
# --------------------------------------------------------------------------
def test_scan_topk_batched_matches_single_sessions(ref):
    lengths = [3000, 777, 12345, 1024, 5000]
    Hkv, Hq, B, k = 2, 8, 68, 128
    stores, qs, s2s, inps = [], [], [], []
    for sidx, n in enumerate(lengths):
        inp = make(4, n=n, Hkv=Hkv, Hq=Hq, layer=sidx)
        st = F.pack_bitplanes(dev(inp["K"]))
        stores.append(st.to_host() if sidx % 2 else st)
        qs.append(inp["q_bf16"])
        s2s.append(inp["sigma2"])
        inps.append(inp)
    q = bf16(np.stack(qs))                                   # [S][Hq][d]
    s2 = dev(np.concatenate(s2s))                            # [S*Hkv][d]
    dep = F.alloc_depths(q.view(-1, 128), s2, B).view(len(lengths), Hq, 128)
    idx, top = F.scan_topk_batched(stores, q, dep, k)
    idx, top = host(idx), host(top)
    for sidx, n in enumerate(lengths):
        i1, t1 = F.scan_topk(stores[sidx], q[sidx], dep[sidx], k)
        assert np.array_equal(idx[sidx], host(i1)), sidx
        assert np.array_equal(top[sidx], host(t1)), sidx
        planes, scales = ref.pack(inps[sidx]["K"])
        d_h = host(dep[sidx])
        assert np.array_equal(d_h, ref.alloc_depths(inps[sidx]["q"], inps[sidx]["sigma2"], B))
        s_ref, a_ref = ref.scores(planes, scales, n, inps[sidx]["q"], d_h, with_abs=True)
        for h in range(Hq):
            topk_sets_agree(ref, s_ref[h], a_ref[h], idx[sidx, h], k)
            topk_sets_agree(ref, s_ref[h], a_ref[h], host(i1)[h], k)
            sel = idx[sidx, h]
            assert np.all(np.abs(top[sidx, h] - s_ref[h][sel]) <= SCORE_RTOL * a_ref[h][sel])
    assert F.last_device_status() == 0


def test_scan_topk_batched_rejects_bad_batches():
    a = F.pack_bitplanes(dev(make(4, n=500, Hkv=2, Hq=8)["K"]))
    b = F.pack_bitplanes(dev(make(4, n=600, Hkv=1, Hq=4)["K"]))
    q = torch.zeros((2, 8, 128), dtype=torch.bfloat16, device=DEV)
    dep = torch.zeros((2, 8, 128), dtype=torch.uint8, device=DEV)
    with pytest.raises(F.FathomError):          # mismatched KV heads
        F.scan_topk_batched([a, b], q, dep, 16)
    with pytest.raises(F.FathomError):          # k above a session's length
        F.scan_topk_batched([a, a], q, dep, 501)
