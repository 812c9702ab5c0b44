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


def test_reference_arm_prints_the_contract_line():
    import json
    import os
    import subprocess
    import sys

    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--workload", "tiny", "--steps", "2",
                        "--warmup", "1"], cwd=root, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["steps"] == 2 and d["warmup"] == 1 and d["value"] > 0
    assert d["higher_is_better"] is True and d["config"]["workload"]
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_default_workload_is_the_largest_single_gpu_config():
    import bench

    args = bench.parse_args([])
    assert args.workload == "ntk16k" and args.only is None
    flops = {k: bench.workload_flops(w) for k, w in workloads.BY_KEY.items()}
    assert max(flops, key=flops.get) == args.workload


def test_both_arms_print_the_same_config():
    """The reference arm's config dict is the one the GPU arm prints (same
    keys and values), so the two lines describe one workload."""
    import json
    import os
    import subprocess
    import sys

    import bench

    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--workload", "tiny", "--steps", "1",
                        "--warmup", "0"], cwd=root, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    d = json.loads([l for l in r.stdout.splitlines() if l.startswith("{")][0])
    assert d["config"] == json.loads(json.dumps(bench.config_of(workloads.TINY, 1)))
