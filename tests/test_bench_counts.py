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


def test_scores_are_the_attention_flops_over_4d():
    """One exponential per valid (query, key) score: 4 * D FLOPs of the two
    products per score, so the count is the FLOP count / (4 D); 480p holds
    2.66e10 of them (24 heads x 33,272^2)."""
    for name in ("tiny", "block", "ragged", "480p", "720p"):
        w = I.WORKLOADS[name]
        assert bench.attention_scores(w) * 4 * w.D == w.attention_flops(), name
    assert bench.attention_scores(I.WORKLOADS["480p"]) == 24 * 33272 ** 2


def test_l2_note_follows_the_workload():
    assert "201 MB each, above" in bench.l2_note(I.WORKLOADS["480p"])
    assert "464 MB each, above" in bench.l2_note(I.WORKLOADS["720p"])
    assert "249 MB each, above" in bench.l2_note(I.WORKLOADS["ragged"])
    assert "fit in the 126 MB L2" in bench.l2_note(I.WORKLOADS["block"])
    assert bench.config_of(I.WORKLOADS["480p"], 1)["l2"] == bench.l2_note(I.WORKLOADS["480p"])


def test_recorded_traffic_only_for_the_captured_workloads():
    """The committed ncu traffic covers the 480p and 720p launches; a workload
    without a capture (ragged) gets none."""
    assert bench.recorded_traffic(I.WORKLOADS["ragged"]) is None
    t = bench.recorded_traffic(I.WORKLOADS["480p"])
    assert t is None or t > 8.0e8      # 480p moves at least its 817.8 MB of Q, K, V and O
    t = bench.recorded_traffic(I.WORKLOADS["720p"])
    assert t is None or t > 1.8e9      # 720p: at least its 1870.5 MB of Q, K, V and O
