"""Host-side pieces of the benchmark: percentiles, work counts, the clock
summary and the DRAM traffic record lookup (no GPU needed)."""
import os
import random

import numpy as np
import pytest

import bench
from block_sparse_attention_32_b200 import capi, pipeline, workloads as wl


def test_percentile_matches_numpy_linear_interpolation():
    rng = random.Random(3)
    for n in (1, 2, 5, 10, 37):
        xs = [rng.uniform(-5, 5) for _ in range(n)]
        for q in (0, 50, 95, 99, 100):
            assert bench.percentile(xs, q) == pytest.approx(np.percentile(xs, q), abs=1e-12)


def test_stage_percentiles_per_stage():
    steps = [{n: float(i + k) for k, n in enumerate(bench.Stages.NAMES)} for i in range(5)]
    pct = bench.stage_percentiles(steps)
    assert set(pct) == set(bench.Stages.NAMES)
    assert pct["index"]["p50"] == 2.0 and pct["index"]["min"] == 0.0
    assert pct["merge"]["max"] == 8.0


@pytest.mark.parametrize("w", [
    wl.small("counts_tiny", 1, 700, 700, 0, 8, 2, 64, seed=1),
    wl.small("counts_chunk", 2, 300, 5000, 4700, 16, 2, 128, seed=2),
    wl.P128,
], ids=lambda w: w.name)
def test_work_counts_match_a_direct_count_and_the_library(w):
    """Entries equal the library's count; selected-token FLOPs equal a direct
    loop over queries (own block up to the query, 15 earlier blocks whole)."""
    idx_flops, attn_flops, n_ent = bench.work_counts(w)
    assert n_ent == capi.msa_num_entries(pipeline.dims_for(w))
    if w.n_q <= 1000:
        toks = 0
        cand = 0
        for i in range(w.n_q):
            t = w.q_pos0 + i
            own = t // 128
            toks += min(15, own) * 128 + (t % 128) + 1
            cand += own * 128
        assert attn_flops == w.batch * w.h_q * 4 * 128 * toks
        assert idx_flops == w.batch * w.h_kv * 2 * w.d_idx * cand


def test_clock_summary(tmp_path):
    p = tmp_path / "clocks.csv"
    p.write_text("0, 1965, 1965, 900.0, 0x4, Not Active, Not Active, Not Active, Active\n"
                 "0, 1800, 1965, 950.0, 0x4, Not Active, Not Active, Not Active, Active\n"
                 "0, 1900, 1965, 940.0, 0x0, Not Active, Not Active, Not Active, Not Active\n"
                 "1, 500, 1965, 10.0, 0x0, Active, Not Active, Not Active, Not Active\n")
    c = bench.summarize_clocks(str(p), 0)
    assert c == {"sm_mhz": 1900.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"]}
    assert bench.summarize_clocks(str(tmp_path / "missing.csv"), 0)["reasons"] == ["unsampled"]


def test_traffic_record_is_used_only_for_matching_sources():
    rec = "sparse_attn_fwd_profile_8k_r8.md"
    kv = dict(line.split(":", 1) for line in open(os.path.join(bench.ROOT, "profiles", rec))
              if ":" in line)
    per_entry = float(kv["dram_bytes_per_entry"])
    got = bench.measured_traffic(["sparse_attn.cu", "common.cuh"], rec, 1000)
    digest = bench.source_digest([os.path.join(bench.ROOT, "block_sparse_attention_32_b200",
                                               "csrc", f) for f in ("sparse_attn.cu",
                                                                    "common.cuh")])
    if kv["source_sha256"].strip() == digest:
        assert got == pytest.approx(per_entry * 1000)
    else:
        assert got is None
    # another kernel's sources never match the record; a missing record gives None
    assert bench.measured_traffic(["merge.cu"], rec, 1000) is None
    assert bench.measured_traffic(["sparse_attn.cu", "common.cuh"], "no_such_record.md", 1) is None
