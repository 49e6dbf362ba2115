"""Host-side logic of bench.py (no GPU): the traffic counters are used only
while the kernel's sources are unchanged, the oracle sample is calibrated
without one-time costs, and the single-rank aggregation and config fields."""
from __future__ import annotations

import hashlib
import json
import os

import pytest

import bench
from block_sparse_long_landmark_b200 import inputs


def _fake_tree(root, sources):
    """A minimal tree with kernel sources and a traffic summary keyed on them."""
    h = hashlib.sha256()
    for rel, body in sources.items():
        dst = root / rel
        dst.parent.mkdir(parents=True, exist_ok=True)
        dst.write_bytes(body)
        h.update(body)
    (root / "profiles").mkdir(parents=True, exist_ok=True)
    entry = {"dram_bytes_per_launch": 123456, "sources": list(sources), "sources_sha256": h.hexdigest()}
    (root / "profiles" / "ncu_traffic.json").write_text(json.dumps({"prefill_x": entry}))
    return entry


def test_traffic_is_used_only_for_the_measured_sources(tmp_path, monkeypatch):
    root = tmp_path / "repo"
    srcs = {"pkg/csrc/a.cu": b"kernel a\n", "pkg/csrc/b.cuh": b"helpers\n"}
    entry = _fake_tree(root, srcs)
    monkeypatch.setattr(bench, "ROOT", str(root))
    assert bench.traffic_for("prefill_x") == entry["dram_bytes_per_launch"]
    assert bench.traffic_for("no_such_kernel") is None
    # any byte of any listed source changed: the counters no longer apply
    for rel in srcs:
        f = root / rel
        f.write_bytes(srcs[rel] + b"\n")
        assert bench.traffic_for("prefill_x") is None
        f.write_bytes(srcs[rel])
        assert bench.traffic_for("prefill_x") == entry["dram_bytes_per_launch"]
    # a listed source that disappeared, or an entry without its hash, gives no counter
    (root / "pkg/csrc/b.cuh").unlink()
    assert bench.traffic_for("prefill_x") is None


def test_committed_traffic_entries_name_existing_sources():
    d = json.load(open(os.path.join(bench.ROOT, "profiles", "ncu_traffic.json")))
    for name, entry in d.items():
        if not isinstance(entry, dict) or "sources" not in entry:
            continue
        assert entry["sources"], name
        for rel in entry["sources"]:
            assert os.path.exists(os.path.join(bench.ROOT, rel)), (name, rel)
        assert len(entry["sources_sha256"]) == 64


def test_calibration_ignores_one_time_costs(monkeypatch):
    """The first oracle call pays the build and first-touch costs; the sample
    size must come from the steady per-unit cost, not from that outlier."""
    calls = []

    def fake(wl, Q, K, V, n, seed=0):
        first = not calls
        calls.append(n)
        return (30.0 if first else 0.0) + 0.01 * n, n * wl.block / wl.Hkv, 8

    monkeypatch.setattr(bench, "oracle_prefill_sample", fake)
    wl = inputs.WORKLOADS["gated_prefill_32k"]
    n = bench.calibrate_units(wl, None, None, None, 15.0)
    assert 1000 <= n <= 1600            # 15 s at 10 ms per unit, within the fit's slack
    assert calls[0] < 16                # the warm-up call is a small one


def test_calibration_with_a_flat_slope_stays_bounded(monkeypatch):
    times = {4: 1.0, 16: 1.0, 64: 1.0}  # noise: no visible slope between the probes
    monkeypatch.setattr(bench, "oracle_prefill_sample", lambda wl, Q, K, V, n, seed=0: (times[n], 1.0, 8))
    n = bench.calibrate_units(inputs.WORKLOADS["gated_prefill_32k"], None, None, None, 15.0)
    assert n <= 2 * 15.0 / (1.0 / 64)   # never more than twice what the larger probe's mean implies


def test_single_rank_aggregation_and_config():
    r = bench.Ranks.single()
    value, t = bench.aggregate(r, 500.0, 1000.0)
    assert t == 500.0 and value == pytest.approx(2000.0)
    c = bench.workload_config(inputs.WORKLOADS["gated_prefill_32k"])
    for k in ("workload", "global_batch", "seq_len", "parallelism", "l2"):
        assert k in c
    assert bench.FP32_ALU_TFLOPS == pytest.approx(148 * 128 * 2 * 1.965e9 / 1e12)


def test_reference_arm_prints_its_contract_line():
    """``bench.py --impl reference`` times the oracle on the host and prints
    one JSON line with the reference arm's keys."""
    import subprocess
    import sys
    r = subprocess.run([sys.executable, os.path.join(bench.ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "3", "--workload", "tiny_fp32_prefill", "--cpu-seconds", "0.3"],
                       capture_output=True, text=True, timeout=600, cwd=bench.ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    line = json.loads([l for l in r.stdout.splitlines() if l.startswith("{")][-1])
    assert line["impl"] == "reference" and line["value"] > 0 and line["higher_is_better"] is True
    for k in ("metric", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "config", "cpu_baseline", "e2e"):
        assert k in line, k
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"
