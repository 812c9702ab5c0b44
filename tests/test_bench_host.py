"""Host logic of bench.py that needs no GPU: the row sets the CPU baseline
times and their FLOP count."""
import numpy as np
import pytest

import bench
import workloads


@pytest.mark.parametrize("key", ["tiny", "qwen7b", "packed"])
def test_all_rows_cover_each_query_row_once(key):
    w = workloads.BY_KEY[key]
    rows = bench.all_rows(w)
    lens = workloads.seq_lengths(w)
    assert len(rows) == w.Hq * sum(lens)
    assert len({tuple(r) for r in rows.tolist()}) == len(rows)
    assert (rows[:, 0] >= 0).all() and (rows[:, 0] < w.B).all()
    assert (rows[:, 1] >= 0).all() and (rows[:, 1] < w.Hq).all()
    assert all(0 <= i < lens[b] for b, _, i in rows[:: max(1, len(rows) // 5000)].tolist())


@pytest.mark.parametrize("key", ["tiny", "qwen7b", "gqa8k", "packed"])
def test_flops_of_all_rows_match_the_causal_closed_form(key):
    # algorithmic FLOPs of causal attention: 4 D Hq sum_b S_b (S_b + 1) / 2
    w = workloads.BY_KEY[key]
    lens = workloads.seq_lengths(w)
    assert w.causal
    want = 4.0 * w.D * w.Hq * sum(L * (L + 1) // 2 for L in lens)
    assert bench.rows_flops(w, bench.all_rows(w)) == want


def test_row_sample_stays_inside_the_workload():
    w = workloads.BY_KEY["packed"]
    rows = bench.oracle_rows_sample(w, 2000, 3)
    lens = np.array(workloads.seq_lengths(w))
    assert (rows[:, 2] < lens[rows[:, 0]]).all() and (rows[:, 1] < w.Hq).all()


def test_group_sample_stays_in_one_kv_group():
    w = workloads.BY_KEY["gqa8k"]
    G = w.Hq // w.Hkv
    for seed in range(5):
        rows = bench.oracle_rows_sample_group(w, 500, seed)
        assert len(set(rows[:, 0].tolist())) == 1
        assert len(set((rows[:, 1] // G).tolist())) == 1
        assert (rows[:, 2] >= 0).all() and (rows[:, 2] < workloads.seq_lengths(w)[rows[0, 0]]).all()
