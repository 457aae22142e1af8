"""Host logic of bench.py (CPU): the step's flop count and the rule that the
recorded DRAM traffic of the fused GEMM is reported only for the sources it
was captured from."""

import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_training_step_flops():
    # fwd 2MNK + 2Mr(K+N) = 69.26 GFLOP, bwd 2MNK + 4Mr(N+K) = 69.79 GFLOP at
    # x 2048 x 4096, W 4096 x 4096, rank 16
    f = bench.train_flops(2048, 4096, 4096, 16)
    assert f == 2 * 2 * 2048 * 4096 * 4096 + 6 * 2048 * 16 * (4096 + 4096)
    assert round(f / 1e9, 2) == 139.05


def test_traffic_is_null_once_the_kernel_changes(monkeypatch, tmp_path):
    import json
    rec = tmp_path / "traffic.json"
    rec.write_text(json.dumps({"dram_bytes_per_launch": 123, "note": "capture",
                               "sources_sha1": bench.sources_sha1(bench.GEMM_SOURCES)}))
    byts, note = bench.recorded_traffic(str(rec))
    assert byts == 123, note
    monkeypatch.setattr(bench, "sources_sha1", lambda paths: "0" * 40)
    byts, note = bench.recorded_traffic(str(rec))
    assert byts is None and "changed" in note


def test_adapter_count_of_the_7b_model():
    # rank 16 on q, k, v, o (4096 x 4096) and gate, up (11008 x 4096), down
    # (4096 x 11008) of 32 layers: r (d_in + d_out) values each
    assert bench.ADAPTERS_7B == 39976960


def test_cpu_baseline_reports_all_cores_and_one_thread():
    r = bench.cpu_baseline(steps=1, rows=64)
    assert r["kind"] == "oracle" and r["unit"] == "TFLOP/s" and r["value"] > 0 and r["cores"] >= 1
    assert r["single_thread"]["cores"] == 1 and r["single_thread"]["value"] > 0
