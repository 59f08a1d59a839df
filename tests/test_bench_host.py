"""Host-side logic of bench.py: the algorithmic work model, the traffic lookup and the clock
summary.  No GPU is used."""
import json
import os

import numpy as np
import pytest

import bench


def _brute_counts(B, Hq, Hkv, Nq, Nkv, d, S, K, W, q_pos0):
    sum_n = 0
    tokens = 0
    for i in range(Nq):
        p = q_pos0 + i
        n = max(0, p - W + 1) // S if p - W + 1 > 0 else 0
        sum_n += n
        tokens += min(n, K) * S + (p - S * n + 1)
    return sum_n, tokens


@pytest.mark.parametrize("Nq,Nkv,q_pos0", [(300, 300, 0), (4, 1000, 996), (1, 777, 776)])
def test_work_model_matches_brute_force(Nq, Nkv, q_pos0):
    B, Hq, Hkv, d, S, K, W = 2, 4, 2, 64, 16, 3, 40
    dims = dict(B=B, Hq=Hq, Hkv=Hkv, N_q=Nq, N_kv=Nkv, d=d)
    wm = bench.work_model(dims, S, K, W, q_pos0, 2)
    sum_n, tokens = _brute_counts(B, Hq, Hkv, Nq, Nkv, d, S, K, W, q_pos0)
    # each (query head, eligible chunk) pair is one d-long dot product (2d flops)
    assert wm["score_flops"] == 2.0 * d * Hq * B * sum_n
    # QK^T and PV over every attended token: 4d flops per (query head, token)
    assert wm["attn_flops"] == 4.0 * d * B * Hq * tokens
    assert wm["tokens"] == B * Nq


def test_phase_bounds():
    wm = {"score_flops": 1.0, "select_bytes": 2.0, "attn_bytes": 3.0, "attn_flops": 4.0}
    assert bench.phase_work("score_topk_tc", wm) == ("tensor", 1.0, "TFLOP/s")
    assert bench.phase_work("select_stream", wm) == ("hbm", 2.0, "GB/s")
    assert bench.phase_work("attn_units", wm) == ("hbm", 3.0, "GB/s")
    assert bench.phase_work("attn_tc", wm) == ("tensor", 4.0, "TFLOP/s")


def test_traffic_lookup_requires_current_source(tmp_path, monkeypatch):
    prof = tmp_path / "profiles"
    prof.mkdir()
    csrc = tmp_path / "hierarchical_chunk_sparse_scoring_b200" / "csrc"
    csrc.mkdir(parents=True)
    for f in ("attn_tc.cu", "common.cuh", "sm100.cuh"):
        (csrc / f).write_text("// " + f + "\nint x = 1;\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    sha = bench.source_sha("attn_tc")
    (prof / "traffic.json").write_text(json.dumps(
        {"attn_tc@small_mha_bf16": {"bytes_per_launch": 123.0, "source_sha": sha}}))
    assert bench.traffic_for("attn_tc", "small_mha_bf16") == 123.0
    assert bench.traffic_for("attn_tc", "gqa7b_prefill") is None
    # comments and layout do not count; code does
    (csrc / "attn_tc.cu").write_text("/* reworded\n comment */ int   x =\n 1; // note\n")
    assert bench.traffic_for("attn_tc", "small_mha_bf16") == 123.0
    (csrc / "attn_tc.cu").write_text("// attn_tc.cu\nint x = 2;\n")
    assert bench.traffic_for("attn_tc", "small_mha_bf16") is None


def test_clock_summary_decodes_reasons():
    c = bench.ClockSampler(0)
    c.max_mhz = 1965.0
    c.rows = [(1965.0, 0), (1800.0, 0x4), (1900.0, 0)]
    s = c.summary()
    assert s["sm_mhz"] == 1900.0 and s["sm_max_mhz"] == 1965.0
    assert s["reasons"] == ["sw_power_cap"]
    c.rows = [(1000.0, 0x8 | 0x40)]
    assert c.summary()["reasons"] == ["hw_slowdown", "hw_thermal_slowdown"]
    c.rows = []
    assert c.summary() is None


def test_union_stat_counts_distinct_chunks():
    import torch
    # one KV group, 4 queries, K = 2; tiles of 2 queries
    idx = torch.tensor([[[[0, 1], [1, 2], [5, -1], [5, 6]]]], dtype=torch.int32)
    # tile 0: {0, 1, 2} -> 3; tile 1: {5, 6} -> 2; mean 2.5 / K
    assert bench.union_stat(idx, 2, C=8) == 2.5 / 2
