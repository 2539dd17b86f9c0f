"""Rank bookkeeping of the multi-GPU decode-step benchmark.

One process per GPU.  The layers of a decode step are independent problems,
so every rank scans its own layer with its own store: there is no collective
on the data path (weak scaling).  Collectives appear only around the timing:
a barrier on both sides of the timed region and a max over ranks of each
rank's device time, taken by every rank in the same order.

The class works with NCCL on GPUs and with gloo on CPU (the multi-process
tests use the latter).
"""
import datetime
import os


class Ranks:
    """The process group of a run launched by torch.distributed.run (or a
    single process when WORLD_SIZE is unset or 1)."""

    def __init__(self, backend="nccl", device=None, sync=None, timeout_s=600, always_group=False):
        """always_group: make a process group also for a single process (a
        path that calls collectives itself then runs unchanged at world 1)."""
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.device = device
        self._sync = sync
        self.dist = None
        if self.world > 1 or always_group:
            import torch.distributed as dist
            os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
            if self.world == 1 and "MASTER_PORT" not in os.environ:
                os.environ.update(MASTER_PORT=str(_free_port()), RANK="0", WORLD_SIZE="1")
            kw = {"device_id": device} if backend == "nccl" and device is not None else {}
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s), **kw)
            self.dist = dist

    def barrier(self):
        """All ranks arrive, then the local device drains."""
        if self.dist:
            self.dist.barrier()
        if self._sync:
            self._sync()

    def max(self, x):
        """Max of a float over ranks (the slowest rank's time)."""
        if not self.dist:
            return float(x)
        import torch
        t = torch.tensor([float(x)], dtype=torch.float64, device=self.device)
        self.dist.all_reduce(t, op=self.dist.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.dist:
            self.dist.barrier()
            self.dist.destroy_process_group()
            self.dist = None


def _free_port():
    import socket
    with socket.socket() as so:
        so.bind(("127.0.0.1", 0))
        return so.getsockname()[1]


def layer_of_rank(rank):
    """The layer a rank scans: rank r takes layer r (independent inputs)."""
    return rank


def throughput(keys_per_rank_step, world, max_total_ms, steps):
    """Whole-job Gkeys/s and ms per step: the keys every rank scanned in
    `steps` steps over the slowest rank's total time."""
    ms_per_step = max_total_ms / steps
    return keys_per_rank_step * world / (ms_per_step * 1e-3) / 1e9, ms_per_step
