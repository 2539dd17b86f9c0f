"""Host-side helpers of bench.py that its JSON line depends on (CPU).

gpu_launches is a claim about how many of the library's kernels one decode
step launches; it follows the top-k path the library picks for the rows
(fathom_scan_topk / fathom_decode_step with block maxima).  The cases mirror
the launcher's rules: rows of at most 131072 keys, and longer rows of at
least k and at most 2^17 blocks of 64 keys, take one cluster kernel; longer
rows of at least 8k blocks the three-kernel block path; the rest the
nine-launch histogram path.
"""
import bench


def test_topk_launches_follow_the_paths():
    assert bench.topk_launches(4096, 64) == 1                     # config 1
    assert bench.topk_launches(131072, 2048) == 1                 # config 2
    assert bench.topk_launches(1 << 20, 2048) == 1                # config 3: block maxima, one kernel
    assert bench.topk_launches(65536, 1024, 524288) == 1          # config 4: ragged sessions
    assert bench.topk_launches(131073, 2048) == 1                 # 2049 blocks >= k
    assert bench.topk_launches(131073, 3000) == 9                 # fewer blocks than k
    assert bench.topk_launches(1 << 24, 64) == 3                  # beyond 2^17 blocks, >= 8k blocks
    assert bench.topk_launches(1 << 24, 4096) == 3


def test_decode_step_launch_count():
    # depths, then per KV-head group: scan, top-k, attention
    assert bench.Layer.launches_per_step(1, 1 << 20, 2048) == 4
    assert bench.Layer.launches_per_step(4, 1 << 20, 2048) == 13
