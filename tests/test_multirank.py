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
