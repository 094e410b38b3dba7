"""Host-side arithmetic of the benchmark: the units the metric counts, the
algorithmic bytes per cached row, and the oracle baseline's report.

The metric counts one key scored per (query token, layer, cached token)
evaluation.  A full-prefix layer scores its N valid tokens; with hierarchical
selection a group of m layers scores N + (m - 1) min(B, N) positions per
query instead of m N (LatentIndex summary, Sec. 3.4).  These tests fix those
counts on the workloads' own sizes, with no GPU.
"""
import numpy as np
import pytest

import bench
from workloads import construction_inputs, generate, workload


def test_keys_per_step_of_the_long_context_step():
    wl = workload(3)                      # 4 sequences x 131072 tokens, B 8192, G 4
    lengths = np.full(wl.batch, 131072)
    hs, dsa = bench.keys_per_step(wl, lengths)
    assert hs == 4 * (131072 + 3 * 8192)  # anchor: N; 3 followers: B each
    assert dsa == 4 * 4 * 131072          # 4 layers, each its own full key scan
    assert hs + dsa == 2_719_744


def test_keys_per_step_caps_the_followers_at_the_valid_prefix():
    wl = workload(2)                      # B 8192
    lengths = np.array([5000, 8192, 20000])
    hs, dsa = bench.keys_per_step(wl, lengths)
    assert hs == (5000 + 3 * 5000) + (8192 + 3 * 8192) + (20000 + 3 * 8192)
    assert dsa == 4 * (5000 + 8192 + 20000)


@pytest.mark.parametrize("idx,dim,want", [(3, 192, 196), (3, 128, 132), (1, 192, 384), (1, 128, 256),
                                          (0, 48, 192)])
def test_row_bytes_are_the_stored_row(idx, dim, want):
    """e4m3 rows carry one fp32 scale; bf16 and f32 rows are the elements alone."""
    assert bench.row_bytes(workload(idx), dim) == want


def test_oracle_sample_step_counts_what_the_step_scores():
    wl = workload(1)                      # the latent is generated directly, as in every bench workload
    inp = generate(wl)
    hnew, Wd, Wk = construction_inputs(wl)
    n = int(inp.lengths[0])
    got = bench.oracle_sample_step(inp, 0, hnew, Wd, Wk)
    hs, dsa = bench.keys_per_step(wl, inp.lengths[:1])
    assert got == hs + dsa == n + 3 * min(wl.B, n) + 4 * n


def test_cpu_baseline_reports_all_cores_and_one_thread():
    wl = workload(1)
    inp = generate(wl)
    hnew, Wd, Wk = construction_inputs(wl)
    r = bench.cpu_baseline(inp, hnew, Wd, Wk, budget_s=0.2, one_thread_s=0.1)
    assert r["kind"] == "oracle" and r["unit"] == "keys/s" and r["value"] > 0
    assert r["cores"] == bench.cpu_cores() >= 1
    assert r["one_thread"]["cores"] == 1 and r["one_thread"]["value"] > 0


def _reference_line(extra_env=None, workload_idx=1):
    import json
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, **(extra_env or {}))
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--workload", str(workload_idx),
                        "--steps", "1", "--warmup", "0"], cwd=root, env=env, capture_output=True, text=True,
                       timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [x for x in r.stdout.splitlines() if x.startswith("{")]
    return [json.loads(x) for x in lines]


def test_reference_arm_prints_one_oracle_line_with_its_own_figures():
    """The reference arm times the oracle on the host: its cpu_baseline and
    e2e figures are the line's own value, with nothing crossing PCIe."""
    lines = _reference_line()
    assert len(lines) == 1
    d = lines[0]
    assert d["impl"] == "reference" and d["unit"] == "keys/s" and d["higher_is_better"] is True
    assert d["value"] > 0 and d["dtype"] == "f64" and d["data"] == "synthetic"
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["cpu_baseline"]["cores"] >= 1 and d["cpu_baseline"]["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": "keys/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    assert d["config"]["workload"].startswith("v32-decode-bf16-n8k")


def test_reference_arm_prints_nothing_on_other_ranks():
    assert _reference_line({"RANK": "1", "WORLD_SIZE": "2"}) == []


def test_prefill_oracle_sample_counts_the_causal_prefixes():
    """Queries at positions 64512..65535 of a 65536-token prefix see
    p + 1 tokens each: 1024 * (64513 + 65536) / 2 pairs a layer.  A sample
    of two rows is the first and the last query, in each of the 4 layers."""
    r = bench.prefill_cpu_baseline(rows=2)
    assert r["keys_per_layer"] == 1024 * (64513 + 65536) // 2 == 66_585_088
    assert r["keys_sampled"] == 4 * (64513 + 65536)
    assert r["kind"] == "oracle" and r["unit"] == "keys/s" and r["value"] > 0
    assert r["extrapolated_layer_s"] == pytest.approx(r["keys_per_layer"] / r["value"])


def test_cpu_baseline_configs_time_whole_group_steps():
    """The oracle timed on the smaller decode workloads: every sequence of a
    step (tiny-f32 builds its latent from the hidden states first)."""
    r = bench.cpu_baseline_configs(indices=(0, 1), budget_s=0.05)
    for i in (0, 1):
        wl = workload(i)
        d = r[wl.name]
        hs, dsa = bench.keys_per_step(wl, generate(wl).lengths)
        assert d["keys_per_step"] == hs + dsa
        assert d["kind"] == "oracle" and d["unit"] == "keys/s" and d["value"] > 0
        assert d["cores"] == bench.cpu_cores()
