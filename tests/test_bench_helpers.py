"""The benchmark's host-side helpers (no GPU): launches per step, the
profile-traffic lookup and its staleness check, the measured-peak fall-back,
and the multi-process oracle runner."""
import json
import os

import pytest

import bench
import workloads


def test_launches_per_step_by_mode():
    assert bench.launches_per_step(workloads.make_case("batched", B=1, V=256)) == 2   # top-k
    assert bench.launches_per_step(workloads.make_case("greedy", B=1, V=256)) == 2
    assert bench.launches_per_step(workloads.make_case("large", B=1, V=256)) == 3     # softmax residuals
    assert bench.launches_per_step(workloads.make_case("tiny", B=1)) == 3


def test_profiled_traffic_only_for_the_current_source(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "PROFILE_DIR", str(tmp_path))
    path = tmp_path / "sv_rows_kernel_batched.md"
    path.write_text(f"- kernel_source_sha256_16: `{bench.kernel_source_hash()}`\n- dram_bytes_per_launch: 1234\n")
    assert bench.profiled_traffic("batched") == 1234.0
    path.write_text("- kernel_source_sha256_16: `0000000000000000`\n- dram_bytes_per_launch: 1234\n")
    assert bench.profiled_traffic("batched") is None
    assert bench.profiled_traffic("greedy") is None  # no summary for this workload


def test_committed_profile_matches_the_kernel_source():
    assert bench.profiled_traffic("batched") is not None
    assert bench.profiled_traffic("head_greedy", "sv_head_kernel", bench.HEAD_SOURCES) is not None


def test_measured_peak_fallback(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.measured_peak() == (bench.FALLBACK_HBM_GBS, "fallback")
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps({"hbm_gbs": 6000.5}))
    assert bench.measured_peak() == (6000.5, "measured")


def test_oracle_runner_two_processes():
    run = bench.OracleRunner("tiny", 2)
    try:
        run.step()
        run.step()
    finally:
        run.close()
    assert run.sequences_per_step() == 2 * bench.ORACLE_REPS["tiny"]
    assert all(not p.is_alive() for p in run.procs)


def test_nearest_rank_percentiles():
    xs = [5.0, 1.0, 3.0, 2.0, 4.0]
    assert bench.pctl(xs, 10) == 1.0 and bench.pctl(xs, 50) == 3.0 and bench.pctl(xs, 90) == 5.0
    assert bench.pctl([7.0], 10) == 7.0 == bench.pctl([7.0], 90)


def test_single_core_oracle_leg():
    import oracle

    case = workloads.make_case("tiny", seed=3, B=6)
    drafts = oracle.draft_tokens_for(case)
    out = bench.cpu_baseline_single("tiny", case, drafts, 0.5, "test")
    assert out["cores"] == 1 and out["kind"] == "oracle" and out["value"] > 0
    assert "single thread" in out["sample"]
