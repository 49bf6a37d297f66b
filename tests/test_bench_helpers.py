"""Host-side helpers of bench.py (CPU): the algorithmic byte and flop counts behind the roofline
fields, and the next-window lists of the incremental-fetch measurement."""
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402
import synth  # noqa: E402


def test_algorithmic_counts_of_the_1m_workload():
    wl = synth.workload("ctx1m_fp8_b32")
    T = 32 * 262144
    fetched = 994416
    a = bench.algorithmic(wl, fetched)
    # E4M3 key (128 B) + fp32 scale per entry and layer, the split queries and weights, one bit per entry
    assert a["score_bytes_per_entry_layer"] == 132
    assert a["score_bytes"] == 3 * T * 132 + 3 * 32 * (64 * 128 * 2 + 64 * 4) + T // 8 == 3324534784
    # bf16 weights read once per layer, plus the small activations
    weights = 3 * (2048 * 4096 + 64 * 128 * 2048 + 64 * 4096) * 2
    assert a["proj_bytes"] == weights + 3 * 32 * (4096 * 2 + 64 * 128 * 2 + 64 * 4)
    assert a["gather_host_bytes"] == fetched * 1024
    assert a["topk_flops"] == 2.0 * 64 * 64 * 128 * fetched


def test_throughput_counts_every_rank():
    assert bench.job_throughput(4, 1000, 10, 2.0) == 4 * 1000 * 10 / 2e-3


def test_drifted_lists_keep_and_replace_entries():
    rng = np.random.default_rng(0)
    S = [5000, 0, 300, 70000]
    offs = np.concatenate([[0], np.cumsum(S)]).astype(np.int64)
    idx = np.full(int(offs[-1]), -1, dtype=np.int32)
    cnt = np.zeros(len(S), dtype=np.int32)
    for b, s in enumerate(S):
        P = np.sort(rng.choice(s, int(0.12 * s), replace=False)) if s else np.zeros(0, dtype=np.int64)
        idx[offs[b]:offs[b] + P.size] = P
        cnt[b] = P.size
    new_idx, new_cnt = bench.drifted_lists(idx, cnt, offs, 0.1, seed=3)
    for b, s in enumerate(S):
        P = idx[offs[b]:offs[b] + cnt[b]]
        N = new_idx[offs[b]:offs[b] + new_cnt[b]]
        assert np.all(np.diff(N) > 0) and (N.size == 0 or (N[0] >= 0 and N[-1] < s))  # ascending, inside
        assert new_cnt[b] == cnt[b]                                                      # same size
        if P.size >= 1000:
            kept = np.intersect1d(P, N).size / P.size
            assert 0.85 < kept < 0.95, kept                                              # about 1 - drift kept
        assert np.all(new_idx[offs[b] + new_cnt[b]:offs[b + 1]] == -1)                    # tail untouched
