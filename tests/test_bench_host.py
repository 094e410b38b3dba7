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
