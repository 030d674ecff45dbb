"""The benchmark's algorithmic counts match the definitions they stand for:
the windowed attention FLOPs count exactly the (query, key) pairs the oracle's
window attention lets attend (the oracle's own window assignment of every
token), at 4 * D FLOPs a pair like the full attention's count."""
import numpy as np

import bench
import oracle
from mmdit_joint_attention_b200 import inputs as I


def _pairs(w: I.Workload, parts) -> int:
    win = oracle.window_of_tokens(w.grid, parts)
    sizes = np.bincount(win)
    total = 0
    for L in w.ctx_lengths():
        # visual rows: own window + valid cond keys; cond rows: every valid key
        total += int(sum(int(sizes[x]) + L for x in win)) + L * (w.Nv + L)
    return total


def test_window_flops_match_the_oracle_windows():
    for name in ("block", "ragged", "480p"):
        w = I.WORKLOADS[name]
        for parts in ((1, 2, 2), (4, 1, 1), (2, 3, 2)):
            want = 4.0 * w.D * w.H * _pairs(w, parts)
            assert bench.window_attention_flops(w, parts) == want, (name, parts)


def test_full_attention_flops_are_the_one_window_case():
    for name in ("block", "ragged", "480p"):
        w = I.WORKLOADS[name]
        assert bench.window_attention_flops(w, (1, 1, 1)) == w.attention_flops()
