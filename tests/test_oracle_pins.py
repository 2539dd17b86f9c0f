"""Pins for the oracle: checks that do not go through the oracle's own formulas.

Each test fixes one part of the oracle against something independent:
  * a library routine (numpy's IEEE fp16 conversion, numpy sort, scipy softmax);
  * a closed form (powers-of-four importances, full-depth scores equal q . Q4(x),
    zero budget gives zero scores);
  * brute force on tiny inputs (every depth vector for d <= 4);
  * the textbook t-bit mid-rise quantizer (the prefix property the pages state);
  * a hand-worked example (tests/golden/six_key_example.json).
"""
import itertools
import json
import os

import numpy as np
import pytest
import scipy.special

import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def textbook_midrise(x, delta, t):
    """t-bit uniform mid-rise quantizer on [-8 delta, 8 delta): step 16 delta / 2^t,
    index floor(x/step) clamped to [-2^(t-1), 2^(t-1)-1], value (index + 1/2) step.
    Zero bits read give 0 (the quantizer's only level)."""
    x = np.asarray(x, np.float64)
    if t == 0:
        return np.zeros_like(x)
    step = 16.0 * delta / (1 << t)
    with np.errstate(divide="ignore", invalid="ignore"):
        idx = np.floor(x / step)
    idx = np.clip(idx, -(1 << (t - 1)), (1 << (t - 1)) - 1)
    idx = np.where(step == 0, 0.0, idx)
    return (idx + 0.5) * step


# --------------------------------------------------------------------------
# fp16 scale rounding vs numpy's IEEE binary16 conversion
# --------------------------------------------------------------------------
def test_fp16_rounding_matches_numpy(ref):
    rng = np.random.default_rng(0)
    x = np.concatenate([
        rng.standard_normal(20000).astype(np.float32) * np.float32(10.0) ** rng.integers(-9, 5, 20000),
        np.array([0.0, -0.0, 65504, 65519.99, 65520, 1e6, 2 ** -24, 2 ** -25, 3 * 2 ** -26, 2 ** -14,
                  2 ** -14 * 1.5, 1 + 2 ** -11, 1 + 3 * 2 ** -11, 1 + 2 ** -11 + 2 ** -20], np.float32),
    ]).astype(np.float32)
    with np.errstate(over="ignore"):
        want = x.astype(np.float16).view(np.uint16)
    got = ref.f32_to_f16_bits(x)
    assert np.array_equal(got, want)


# --------------------------------------------------------------------------
# Quantizer, planes and basis rule: a t-plane prefix IS the t-bit quantizer
# --------------------------------------------------------------------------
@pytest.mark.parametrize("n", [1, 63, 64, 200, 257])
def test_prefix_equals_textbook_quantizer(ref, n):
    rng = np.random.default_rng(n)
    d, H = 8, 2
    sig = np.exp(rng.uniform(-3, 2, size=(H, d)))
    K = (rng.standard_normal((H, n, d)) * sig[:, None, :]).astype(np.float32)
    K[0, :, 3] = 0.0                      # an all-zero channel: Delta = 0
    planes, scales = ref.pack(K)
    npad = ref.n_pad(n)
    assert planes.shape == (H, d, 4, npad // 32) and scales.shape == (H, d, npad // 64)
    # scales: fp16 of amax/8 per (head, channel, 64-key block), 0 for empty blocks
    for g in range(H):
        for c in range(d):
            for b in range(npad // 64):
                blk = K[g, b * 64:min(n, b * 64 + 64), c]
                amax = np.float32(np.max(np.abs(blk))) if blk.size else np.float32(0)
                assert scales[g, c, b] == np.float32(amax / np.float32(8)).astype(np.float16).view(np.uint16)
    delta = scales.view(np.float16).astype(np.float64)
    for g in range(H):
        blocks = np.arange(n) // 64
        dl = delta[g][:, blocks].T         # [n][d]
        for t in range(5):
            got = ref.reconstruct(planes, scales, n, g, np.full(d, t, np.uint8))
            want = textbook_midrise(K[g].astype(np.float64), dl, t)
            assert np.array_equal(got, want), (g, t)


def test_every_code_every_prefix(ref):
    """Exhaustive over the 16 codes: x at the centre of each code cell."""
    d = 16
    delta = 0.375  # exact in fp16 and fp32
    codes = np.arange(16)
    # one key per code in channel c = code, plus a key that pins amax = 8 delta
    n = 17
    K = np.zeros((1, n, d), np.float32)
    for c in range(d):
        K[0, c, c] = (codes[c] - 8 + 0.5) * delta
        K[0, 16, c] = 8 * delta
    planes, scales = ref.pack(K)
    assert np.all(scales[0, :, 0] == np.float16(delta).view(np.uint16))
    for t in range(5):
        kh = ref.reconstruct(planes, scales, n, 0, np.full(d, t, np.uint8))
        for c in range(d):
            assert kh[c, c] == textbook_midrise(K[0, c, c], delta, t)
            # bits of the code as written in the planes (plane 0 = MSB)
            bits = [(planes[0, c, j, 0] >> c) & 1 for j in range(4)]
            assert bits == [(codes[c] >> (3 - j)) & 1 for j in range(4)]
        # the key at +8 delta clamps to the top code 15
        assert np.all(kh[16] == textbook_midrise(np.full(d, 8 * delta), delta, t))


# --------------------------------------------------------------------------
# Hand-worked six-key example (builder's own; the pages print none)
# --------------------------------------------------------------------------
def _six():
    with open(os.path.join(GOLDEN, "six_key_example.json")) as f:
        return json.load(f)


def test_six_key_pack(ref):
    ex = _six()
    K = np.array(ex["keys_x"], np.float32)[None]
    scales, codes = ref.quantize(K)
    assert codes[0].tolist() == ex["expected_codes"]
    assert scales[0, :, 0].tolist() == ex["expected_scale_f16_bits"]
    assert np.all(scales[0, :, 1] == 0)     # block 1 is all padding
    planes = ref.pack_planes(codes)
    for c in range(4):
        assert planes[0, c, :, 0].tolist() == ex["expected_plane_words_block0"]["channel%d" % c]
        assert np.all(planes[0, c, :, 1:] == 0)


def test_six_key_depths_scores_topk(ref):
    ex = _six()
    q = np.array(ex["q"], np.float32)
    s2 = np.array(ex["sigma2"], np.float32)
    assert ref.importance(q, s2).tolist() == ex["expected_importance"]
    w = ref.importance(q, s2)
    for B, t in ex["expected_depths"].items():
        assert ref.depths(w, int(B)).tolist() == t, B
    K = np.array(ex["keys_x"], np.float32)[None]
    planes, scales = ref.pack(K)
    for B, want in ex["expected_scores"].items():
        t = ref.depths(w, int(B))
        s = ref.scores(planes, scales, 6, q[None], t[None])[0]
        assert s.tolist() == want, B
        assert ref.topk(s, 3).tolist() == ex["expected_top3"][B], B
    exact = K[0].astype(np.float64) @ q.astype(np.float64)
    assert int(np.argmax(exact)) == ex["exact_top1"]


# --------------------------------------------------------------------------
# Depths: invariants, brute-force optimum, closed form, tie rule
# --------------------------------------------------------------------------
def _objective(w, t):
    return float(np.sum(np.asarray(w, np.float64) * 4.0 ** (-np.asarray(t, np.float64))))


@pytest.mark.parametrize("d", [1, 2, 3, 4])
def test_depths_brute_force_optimum(ref, d):
    rng = np.random.default_rng(100 + d)
    for trial in range(30):
        w = (rng.exponential(1.0, d) * 10.0 ** rng.integers(-2, 3, d)).astype(np.float32)
        if trial % 7 == 0:
            w[rng.integers(0, d)] = 0.0
        for B in range(0, 4 * d + 3):
            t = ref.depths(w, B)
            N = min(B, 4 * d)
            assert int(t.sum()) == N and t.max(initial=0) <= 4
            best = min(_objective(w, tt) for tt in itertools.product(range(5), repeat=d) if sum(tt) == N)
            assert _objective(w, t) == pytest.approx(best, rel=1e-12, abs=0.0)


def test_depths_invariants_large(ref):
    rng = np.random.default_rng(7)
    d = 128
    for trial in range(20):
        q = rng.standard_normal(d).astype(np.float32)
        s2 = np.exp(rng.uniform(-5, 4, d)).astype(np.float32)
        w = ref.importance(q, s2)
        for B in (0, 1, 46, 64, 68, 92, 136, 511, 512, 600):
            t = ref.depths(w, B)
            assert int(t.sum()) == min(B, 4 * d) and t.max() <= 4
            # more important channels are read at least as deep
            order = np.argsort(-w.astype(np.float64), kind="stable")
            assert np.all(np.diff(t[order].astype(int)) <= 0)


def test_depths_powers_of_four_closed_form(ref):
    """w_c = 4^m_c: candidate (c,t) has value 4^(m_c - t), so the water level is a
    power of four and the depth of channel c at level 4^L is clip(m_c - L + 1, 0, 4)
    once every candidate at or above the level is taken."""
    m = np.array([3, 1, 0, 2, 5, 1], np.int64)
    w = (4.0 ** m).astype(np.float32)
    for L in range(-4, 7):
        t_closed = np.clip(m - L + 1, 0, 4)
        B = int(t_closed.sum())
        assert ref.depths(w, B).tolist() == t_closed.tolist()


# --------------------------------------------------------------------------
# Group-pooled depths (a variant for comparison): reductions to the per-query
# rule and optimality of the pooled objective
# --------------------------------------------------------------------------
def test_pooled_depths_reduce_to_per_query_rule(ref):
    rng = np.random.default_rng(11)
    d = 64
    s2 = np.exp(rng.uniform(-3, 2, (2, d))).astype(np.float32)
    q = rng.standard_normal((2, d)).astype(np.float32)
    for B in (0, 17, 92, 256, 300):
        # one query head per KV head: pooling changes nothing
        assert np.array_equal(ref.alloc_depths_pooled(q, s2, B), ref.alloc_depths(q, s2, B))
        # two identical query heads: the pooled weight is exactly 2w, which orders as w
        q2 = np.repeat(q, 2, axis=0)
        want = np.repeat(ref.alloc_depths(q, s2, B), 2, axis=0)
        assert np.array_equal(ref.alloc_depths_pooled(q2, s2, B), want)


@pytest.mark.parametrize("d", [1, 2, 3])
def test_pooled_depths_minimise_the_group_distortion(ref, d):
    """For G = 2 the pooled depths minimise sum_c (w_0c + w_1c) 4^-t_c over all
    depth vectors with sum t = min(B, 4d) (brute force), and both heads get them."""
    rng = np.random.default_rng(40 + d)
    for trial in range(20):
        q = rng.standard_normal((2, d)).astype(np.float32)
        s2 = np.exp(rng.uniform(-2, 2, (1, d))).astype(np.float32)
        wsum = np.asarray(q[0], np.float64) ** 2 * s2[0] + np.asarray(q[1], np.float64) ** 2 * s2[0]
        for B in range(0, 4 * d + 2):
            t = ref.alloc_depths_pooled(q, s2, B)
            assert np.array_equal(t[0], t[1])
            N = min(B, 4 * d)
            assert int(t[0].sum()) == N
            best = min(_objective(wsum, tt) for tt in itertools.product(range(5), repeat=d) if sum(tt) == N)
            assert _objective(wsum, t[0]) == pytest.approx(best, rel=1e-6, abs=0.0)


def test_pooled_depths_hand_example(ref):
    """Two heads that each care about a different channel: per query each reads
    its own channel; pooled, the group splits the budget by the summed weight."""
    q = np.array([[2.0, 0.0, 1.0, 0.0], [0.0, 2.0, 1.0, 0.0]], np.float32)
    s2 = np.ones((1, 4), np.float32)
    # pooled w = (4, 4, 2, 0): candidates 4,4,1,1,2,0.5,0.5,0.25,... in (v desc, c asc, t asc)
    # B = 3 takes (c0,t0), (c1,t0), (c2,t0)
    assert ref.alloc_depths_pooled(q, s2, 3).tolist() == [[1, 1, 1, 0], [1, 1, 1, 0]]
    # per query: head 0 w = (4, 0, 1, 0) takes (c0,t0), (c0,t1), (c2,t0)
    assert ref.alloc_depths(q, s2, 3).tolist() == [[2, 0, 1, 0], [0, 2, 1, 0]]


def test_depths_tie_rule(ref):
    w = np.ones(4, np.float32)
    assert ref.depths(w, 5).tolist() == [2, 1, 1, 1]
    assert ref.depths(w, 3).tolist() == [1, 1, 1, 0]
    w = np.zeros(4, np.float32)            # zero-weight channels fill in channel order
    assert ref.depths(w, 6).tolist() == [4, 2, 0, 0]
    with pytest.raises(ValueError):
        ref.depths(np.ones(4, np.float32), -1)


def test_importance_is_fp32(ref):
    rng = np.random.default_rng(3)
    q = rng.standard_normal(1000).astype(np.float32)
    s2 = np.exp(rng.uniform(-5, 5, 1000)).astype(np.float32)
    w = ref.importance(q, s2)
    assert np.array_equal(w, (q * q) * s2)   # numpy fp32 ops round each product once
    assert w.dtype == np.float32


def test_fixed_r_depths(ref):
    q = np.array([0.5, -3.0, 2.0, -2.0, 2.0, 0.1], np.float32)
    assert ref.fixed_depths(q, 2).tolist() == [0, 4, 4, 0, 0, 0]
    assert ref.fixed_depths(q, 3).tolist() == [0, 4, 4, 4, 0, 0]
    assert ref.fixed_depths(q, 4).tolist() == [0, 4, 4, 4, 4, 0]
    assert ref.fixed_depths(q, 10).tolist() == [4] * 6
    rng = np.random.default_rng(5)
    qq = rng.standard_normal(128).astype(np.float32)
    for r in (16, 32):
        t = ref.fixed_depths(qq, r)
        chosen = np.argsort(-np.abs(qq), kind="stable")[:r]
        assert sorted(np.nonzero(t)[0].tolist()) == sorted(chosen.tolist())
        assert int(t.sum()) == 4 * r       # 64 / 128 plane bits + 16-bit scale per 64 keys = 68 / 136


def test_alloc_depths_gqa(ref):
    rng = np.random.default_rng(9)
    Hkv, G, d = 2, 4, 32
    q = rng.standard_normal((Hkv * G, d)).astype(np.float32)
    s2 = np.exp(rng.uniform(-3, 3, (Hkv, d))).astype(np.float32)
    dep = ref.alloc_depths(q, s2, 40)
    for h in range(Hkv * G):
        assert dep[h].tolist() == ref.depths((q[h] * q[h]) * s2[h // G], 40).tolist()


# --------------------------------------------------------------------------
# Scores: full depth = q . Q4(x) (textbook 4-bit quantizer); zero budget
# --------------------------------------------------------------------------
def test_scores_full_depth_equal_dot_with_4bit_quantizer(ref):
    cfg_rng = synth.rng_for(1, 0, 0)
    Hkv, G, d, n = 2, 2, 32, 300
    sig = synth.channel_sigma(cfg_rng, Hkv, d)
    K = synth.keys(synth.rng_for(1, 0, 1), sig, n)
    q = synth.queries(synth.rng_for(1, 0, 2), Hkv * G, d)
    planes, scales = ref.pack(K)
    delta = scales.view(np.float16).astype(np.float64)
    dep = np.full((Hkv * G, d), 4, np.uint8)
    s = ref.scores(planes, scales, n, q, dep)
    for h in range(Hkv * G):
        g = h // G
        Q4 = textbook_midrise(K[g].astype(np.float64), delta[g][:, np.arange(n) // 64].T, 4)
        want = Q4 @ q[h].astype(np.float64)
        np.testing.assert_allclose(s[h], want, rtol=1e-12, atol=1e-12)
    # zero budget: nothing read, every score is 0, top-k is 0..k-1 by the tie rule
    s0 = ref.scores(planes, scales, n, q, np.zeros_like(dep))
    assert np.all(s0 == 0.0)
    assert ref.topk(s0[0], 5).tolist() == [0, 1, 2, 3, 4]


def test_scores_sub_range_and_absterm(ref):
    rng = np.random.default_rng(11)
    n, d = 500, 32
    K = rng.standard_normal((1, n, d)).astype(np.float32)
    planes, scales = ref.pack(K)
    q = rng.standard_normal((1, d)).astype(np.float32)
    t = rng.integers(0, 5, (1, d)).astype(np.uint8)
    full, a = ref.scores(planes, scales, n, q, t, with_abs=True)
    part = ref.scores(planes, scales, n, q, t, 123, 321)
    assert np.array_equal(part, full[:, 123:321])
    assert np.all(a >= np.abs(full))


def test_depth_one_channel(ref):
    """d = 1: the score is q times the channel's prefix value."""
    K = np.array([[[1.0], [-2.0], [3.9], [-4.0]]], np.float32)   # amax 4 -> Delta 0.5
    planes, scales = ref.pack(K)
    q = np.array([[2.0]], np.float32)
    for t in range(5):
        s = ref.scores(planes, scales, 4, q, np.array([[t]], np.uint8))[0]
        assert s.tolist() == (2.0 * textbook_midrise(K[0, :, 0], 0.5, t)).tolist()


# --------------------------------------------------------------------------
# Top-k vs numpy lexsort (library), with ties
# --------------------------------------------------------------------------
def test_topk_vs_lexsort(ref):
    rng = np.random.default_rng(2)
    for n, k in [(1, 1), (10, 10), (100, 7), (5000, 64), (4097, 2048)]:
        s = np.round(rng.standard_normal(n), 1)          # many exact ties
        for arr in (s.astype(np.float64), s.astype(np.float32)):
            want = np.lexsort((np.arange(n), -arr.astype(np.float64)))[:k]
            assert ref.topk(arr, k).tolist() == want.tolist()
    with pytest.raises(ValueError):
        ref.topk(np.zeros(3), 4)


# --------------------------------------------------------------------------
# Attention: k = 1, equal logits, scipy softmax
# --------------------------------------------------------------------------
def test_attend_special_cases_and_softmax(ref):
    rng = np.random.default_rng(4)
    Hkv, G, n, d, k = 2, 2, 50, 16, 8
    Kr = synth.f32_to_bf16_bits(rng.standard_normal((Hkv, n, d)).astype(np.float32))
    Vr = synth.f32_to_bf16_bits(rng.standard_normal((Hkv, n, d)).astype(np.float32))
    Kf = synth.bf16_bits_to_f32(Kr).astype(np.float64)
    Vf = synth.bf16_bits_to_f32(Vr).astype(np.float64)
    q = rng.standard_normal((Hkv * G, d)).astype(np.float32)
    idx = np.stack([rng.choice(n, k, replace=False) for _ in range(Hkv * G)]).astype(np.int32)
    out = ref.attend(q, Kr, Vr, idx)
    for h in range(Hkv * G):
        g = h // G
        p = scipy.special.softmax(Kf[g, idx[h]] @ q[h].astype(np.float64) / np.sqrt(d))
        np.testing.assert_allclose(out[h], p @ Vf[g, idx[h]], rtol=1e-12, atol=1e-12)
    # k = 1: the output is the selected value row
    o1 = ref.attend(q, Kr, Vr, idx[:, :1])
    for h in range(Hkv * G):
        assert np.array_equal(o1[h], Vf[h // G, idx[h, 0]])
    # q = 0: equal logits, the output is the mean of the selected rows
    o0 = ref.attend(np.zeros_like(q), Kr, Vr, idx)
    for h in range(Hkv * G):
        np.testing.assert_allclose(o0[h], Vf[h // G, idx[h]].mean(0), rtol=1e-13, atol=1e-15)
