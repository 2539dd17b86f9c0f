"""The multi-rank path of the benchmark on CPU: two gloo ranks.

Each rank scans its own layer (independent inputs, no collective on the data
path); the only collectives are the barriers around the timed region and the
max over ranks of the device time.  These tests run that bookkeeping as two
spawned processes with the gloo backend: the max must be the slowest rank's
time on every rank, the whole-job throughput must count every rank's keys
over that time, and the ranks' inputs must differ.
"""
import json
import os
import socket
import sys

import numpy as np
import pytest

torch = pytest.importorskip("torch")
import torch.multiprocessing as mp  # noqa: E402

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, outdir):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import synth
    from bit_plane_key_b200.ranks import Ranks, layer_of_rank, throughput
    ranks = Ranks("gloo", device=torch.device("cpu"), timeout_s=60)
    assert (ranks.rank, ranks.world) == (rank, world)
    inp = synth.layer_inputs(3, layer=layer_of_rank(rank), n=2048, n_kv_heads=2, n_q_heads=8, needles=0)
    ranks.barrier()
    step_ms = [1.0 + rank, 2.0 + 3 * rank, 1.5]        # a slower rank 1
    total = ranks.max(sum(step_ms))
    value, ms = throughput(2048 * 2, world, total, len(step_ms))
    e2e = ranks.max(10.0 * (world - rank))             # the slowest rank differs here
    ranks.barrier()
    ranks.close()
    with open(os.path.join(outdir, "rank%d.json" % rank), "w") as f:
        json.dump({"total": total, "value": value, "ms": ms, "e2e": e2e,
                   "k_sum": float(np.float64(inp["K"]).sum()), "q_sum": float(np.float64(inp["q"]).sum())}, f)


@pytest.mark.timeout(180)
def test_two_gloo_ranks_max_and_throughput(tmp_path):
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    r = [json.load(open(tmp_path / ("rank%d.json" % i))) for i in range(world)]
    slow = max(1.0 + 2.0 + 1.5, 2.0 + 5.0 + 1.5)
    for x in r:
        assert x["total"] == slow                      # every rank sees the slowest rank's time
        assert x["ms"] == pytest.approx(slow / 3)
        assert x["value"] == pytest.approx(2048 * 2 * world / (slow / 3 * 1e-3) / 1e9)
        assert x["e2e"] == 20.0
    assert r[0]["k_sum"] != r[1]["k_sum"]              # each rank scans its own layer
    assert r[0]["q_sum"] != r[1]["q_sum"]


def test_single_process_needs_no_group():
    from bit_plane_key_b200.ranks import Ranks, throughput
    env = {k: os.environ.pop(k) for k in ("WORLD_SIZE", "RANK") if k in os.environ}
    try:
        r = Ranks("gloo")
        assert (r.world, r.rank, r.dist) == (1, 0, None)
        assert r.max(3.5) == 3.5
        r.barrier()
        r.close()
    finally:
        os.environ.update(env)
    v, ms = throughput(1 << 20, 1, 50.0, 10)
    assert ms == 5.0 and v == pytest.approx((1 << 20) / 5e-3 / 1e9)


def _one_rank_group_main(outdir):
    os.environ.pop("MASTER_PORT", None)
    os.environ.pop("WORLD_SIZE", None)
    os.environ.pop("RANK", None)
    sys.path.insert(0, ROOT)
    import torch
    from bit_plane_key_b200.ranks import Ranks
    from bit_plane_key_b200.shard import gather_candidates
    r = Ranks("gloo", device=torch.device("cpu"), timeout_s=60, always_group=True)
    s, i = gather_candidates(torch.tensor([[3.0, 1.0]]), torch.tensor([[7, 2]], dtype=torch.int32))
    res = {"world": r.world, "group": r.dist is not None, "s": s.tolist(), "i": i.tolist(), "max": r.max(2.5)}
    r.close()
    with open(os.path.join(outdir, "one.json"), "w") as f:
        json.dump(res, f)


def test_single_process_group_on_request(tmp_path):
    """always_group makes a one-rank group, so a path that calls collectives
    (the key-range sharded step) runs unchanged without a launcher."""
    ctx = mp.get_context("spawn")
    p = ctx.Process(target=_one_rank_group_main, args=(str(tmp_path),))
    p.start()
    p.join(120)
    assert p.exitcode == 0
    with open(tmp_path / "one.json") as f:
        r = json.load(f)
    assert r == {"world": 1, "group": True, "s": [[3.0, 1.0]], "i": [[7, 2]], "max": 2.5}


def _shard_rank_main(rank, world, port, outdir, scores_path):
    """Key-range sharding on CPU: local top-k of the rank's range (the oracle),
    the gloo all-gather of (score, global index) lists, then a merge."""
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import oracle
    from bit_plane_key_b200.ranks import Ranks
    from bit_plane_key_b200.shard import gather_candidates, shard_range
    ranks = Ranks("gloo", device=torch.device("cpu"), timeout_s=60)
    s = np.load(scores_path)
    rows, n = s.shape
    k = 300
    k0, k1 = shard_range(n, world, rank)
    top = np.full((rows, k), -np.inf, np.float32)
    idx = np.full((rows, k), -1, np.int32)
    for r in range(rows):
        loc = oracle.topk(s[r, k0:k1], min(k, k1 - k0))
        top[r, :len(loc)] = s[r, k0 + loc]
        idx[r, :len(loc)] = loc + k0
    cs, ci = gather_candidates(torch.from_numpy(top), torch.from_numpy(idx))
    merged = []
    for r in range(rows):
        pos = oracle.topk(cs[r].numpy(), k)   # ties -> the candidate listed first
        merged.append(ci[r].numpy()[pos].tolist())
    ranks.close()
    with open(os.path.join(outdir, "shard%d.json" % rank), "w") as f:
        json.dump({"range": [k0, k1], "merged": merged}, f)


@pytest.mark.timeout(180)
def test_key_range_sharding_merge_on_two_gloo_ranks(tmp_path, ref):
    """Two ranks each take the top-k of their key range; after the all-gather
    and the merge both hold the top-k of the whole rows, ties (planted across
    the range boundary) resolved to the lower global index."""
    rng = np.random.default_rng(3)
    rows, n = 3, 5000
    s = np.round(rng.standard_normal((rows, n)), 1).astype(np.float32)   # many exact ties
    s[:, 2040:2060] = 9.0                                                 # equal top scores on both sides of 2048
    path = tmp_path / "scores.npy"
    np.save(path, s)
    world = 2
    mp.start_processes(_shard_rank_main, args=(world, _free_port(), str(tmp_path), str(path)), nprocs=world,
                       join=True, start_method="spawn")
    out = [json.load(open(tmp_path / ("shard%d.json" % i))) for i in range(world)]
    assert out[0]["range"] == [0, 3072] and out[1]["range"] == [3072, 5000]
    for r in range(rows):
        want = ref.topk(s[r], 300).tolist()
        assert out[0]["merged"][r] == want and out[1]["merged"][r] == want


def test_shard_ranges_cover_the_keys_on_aligned_cuts():
    from bit_plane_key_b200.shard import shard_range
    for n in (1, 1000, 1024, 5000, 1 << 20, (1 << 20) + 17):
        for world in (1, 2, 3, 8):
            cuts = [shard_range(n, world, r) for r in range(world)]
            assert cuts[0][0] == 0 and cuts[-1][1] == n
            for (a0, a1), (b0, b1) in zip(cuts, cuts[1:]):
                assert a1 == b0
            for a0, a1 in cuts:   # every non-empty range starts on a 1024-key cut; empty ones sit at n
                assert (a0 % 1024 == 0) if a0 < a1 else (a0 == n)


def _attn_rank_main(rank, world, port, outdir):
    """Attention over a key range split across two gloo ranks: each rank forms
    the (o, m, l) partials of the selected rows it holds (plain numpy here, the
    layout fathom_sparse_attend_partial writes), the partials are all-gathered
    rank by rank, and the log-sum-exp merge gives the full attention."""
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    from bit_plane_key_b200.ranks import Ranks
    from bit_plane_key_b200.shard import gather_partials, shard_range
    ranks = Ranks("gloo", device=torch.device("cpu"), timeout_s=60)
    rng = np.random.default_rng(11)
    Hq, d, n, k = 3, 16, 3000, 50
    q = rng.standard_normal((Hq, d))
    K = rng.standard_normal((n, d))
    V = rng.standard_normal((n, d))
    idx = np.stack([rng.choice(n, k, replace=False) for _ in range(Hq)])
    idx[2] = np.arange(k)                       # head 2: every row in rank 0's range
    k0, k1 = shard_range(n, world, rank)
    parts = np.zeros((Hq, d + 2), np.float32)
    for h in range(Hq):
        sel = [i for i in idx[h] if k0 <= i < k1]
        if not sel:
            parts[h, d] = -np.inf
            continue
        s = K[sel] @ q[h] * np.log2(np.e) / np.sqrt(d)
        m = s.max()
        p = np.exp2(s - m)
        parts[h, :d] = p @ V[sel]
        parts[h, d], parts[h, d + 1] = m, p.sum()
    allp = gather_partials(torch.from_numpy(parts)).numpy().astype(np.float64)
    ranks.close()
    M = allp[:, :, d].max(axis=0)
    f = np.where(np.isinf(allp[:, :, d]), 0.0, np.exp2(allp[:, :, d] - M))
    out = (allp[:, :, :d] * f[:, :, None]).sum(0) / (allp[:, :, d + 1] * f).sum(0)[:, None]
    want = np.zeros((Hq, d))
    for h in range(Hq):
        s = K[idx[h]] @ q[h] / np.sqrt(d)
        p = np.exp(s - s.max())
        want[h] = p @ V[idx[h]] / p.sum()
    with open(os.path.join(outdir, "attn%d.json" % rank), "w") as fh:
        json.dump({"shape": list(allp.shape), "err": float(np.abs(out - want).max()),
                   "m_rank1_head2": float(allp[1, 2, d]) if world > 1 else None}, fh)


@pytest.mark.timeout(180)
def test_sharded_attention_partials_on_two_gloo_ranks(tmp_path):
    world = 2
    mp.start_processes(_attn_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    for r in range(world):
        x = json.load(open(tmp_path / ("attn%d.json" % r)))
        assert x["shape"] == [world, 3, 18]
        assert x["err"] < 1e-5                  # fp32 partials, fp64 merge
        assert x["m_rank1_head2"] == float("-inf")   # rank 1 holds none of head 2's rows
