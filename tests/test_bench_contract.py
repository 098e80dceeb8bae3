"""The benchmark's JSON contract, checked on the host: the reference arm (the
fp64 oracle timed on the host cores) on the tiny workload, and the lookup of
recorded DRAM traffic, which must ignore a record whose source no longer
matches."""
import hashlib
import json
import os
import subprocess
import sys

import pytest

from conftest import ROOT

sys.path.insert(0, ROOT)
import bench  # noqa: E402


def test_reference_arm_prints_the_contract_line():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--config", "0",
                          "--steps", "1", "--warmup", "3"], capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    line = json.loads(out.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference"
    assert line["metric"] == bench.METRIC and line["unit"] == bench.UNIT
    assert line["value"] > 0 and line["higher_is_better"] is True
    assert line["steps"] == 1 and line["warmup"] == 3 and line["n_gpus"] == 1
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == line["value"] and cb["sample"]
    assert line["e2e"] == {"value": line["value"], "unit": line["unit"], "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}


def test_traffic_record_needs_the_current_source(tmp_path, monkeypatch):
    from sparse_long_context_03_b200 import build
    src = os.path.join(build.CSRC, "attention.cu")
    digest = hashlib.sha256(open(src, "rb").read()).hexdigest()
    rec = tmp_path / "traffic.txt"
    rec.write_text("# comment\n"
                   f"sparse_prefill_kernel prefill-128k 100 20 {digest} attention.cu cmd\n"
                   f"indexer_tc_kernel prefill-128k 7 8 {'0' * 64} indexer_tc.cu cmd\n")
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(rec))
    assert bench.measured_traffic("attention", "prefill-128k") == 120
    assert bench.measured_traffic("attention", "prefill-32k") is None   # other workload
    assert bench.measured_traffic("indexer", "prefill-128k") is None    # stale hash
    assert bench.measured_traffic("topk", "prefill-128k") is None       # no record


@pytest.mark.parametrize("world", [1, 4])
def test_weak_scaling_aggregate(world):
    # whole-job tokens per second: every rank prefills its own sequence
    assert bench.aggregate_tok_per_s(world, 131072, 5, 500.0) == pytest.approx(world * 131072 * 5 / 0.5)


def test_oracle_sample_rows_and_extrapolation():
    from sparse_long_context_03_b200 import inputs
    cfg = inputs.config(2)
    rows = bench.sample_rows(cfg, 256, seed=5)
    assert len(rows) == 256 and len(set(rows)) == 256 and rows == sorted(rows)
    for t in (0, cfg.k - 2, cfg.k - 1, cfg.k, cfg.L - 1):
        assert t in rows
    assert all(0 <= t < cfg.L for t in rows)
    # multimodal: frame/text boundary rows are sampled too
    mm = inputs.config(4)
    t0 = inputs.FRAME_TOKENS * inputs.FRAMES_PER_GROUP
    assert {t0 - 1, t0, t0 + inputs.TEXT_TOKENS - 1, t0 + inputs.TEXT_TOKENS} <= set(bench.sample_rows(mm, 64, 1))
    # a sample whose rows cost exactly the mean row cost extrapolates by L / n_rows
    tiny = inputs.config(0, L=9)
    tok_s, full = bench.extrapolate_tok_per_s(tiny, [4], 2.0)  # mean of t+1 over t<9 is 5
    assert full == pytest.approx(2.0 * 9) and tok_s == pytest.approx(9 / 18.0)


def test_omega_union_counts_distinct_selected_keys():
    # 16 adjacent query rows; row t selects {t, t+1, ..., t+k-1} clipped to
    # -1 padding past 40: the union of rows t0..t0+15 is t0..min(39, t0+15+k-1)
    import torch

    k, L = 4, 64

    class Plan:
        pass

    plan = Plan()
    idx = torch.full((L, k), -1, dtype=torch.int32)
    for t in range(L):
        for j in range(k):
            if t + j < 40:
                idx[t, j] = t + j
    plan.idx = idx
    res = bench.omega_union(plan, L, k, width=16, fracs=(0.0, 0.5), samples=1)
    first = res["t~0"]  # rows 0..15: keys 0..18
    assert first["mean_union"] == 19 and first["min"] == 19 and first["max"] == 19
    assert abs(first["of_width_k"] - 19 / 64) < 1e-12
    second = res["t~32"]  # rows 32..47: keys 32..39 only
    assert second["mean_union"] == 8


def test_profile_case_choices_are_accepted():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--help"], capture_output=True, text=True,
                         cwd=ROOT, timeout=300)
    assert out.returncode == 0
    for case in ("fused", "attention", "omega-union", "decode-indexer", "decode-topk"):
        assert case in out.stdout
