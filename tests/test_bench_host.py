"""bench.py's host side on the CPU: the reference arm's JSON line on a small workload, and the
algorithmic units and traffic bookkeeping the GPU arm reports (no GPU is involved)."""
import json
import os
import subprocess
import sys

import pytest

from deformable_slide_attention_b200 import inputs

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


@pytest.mark.parametrize("workload", ["tiny-f32"])
def test_reference_arm_prints_one_complete_line(workload):
    env = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0", OMP_NUM_THREADS="2")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", workload, "--steps", "2", "--warmup", "1"],
                       env=env, capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["value"] > 0 and d["steps"] == 2
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}
    assert d["config"]["workload"] == workload


def test_metric_names_the_headline_only_on_the_default_workload():
    assert bench.metric_of(inputs.BY_NAME[bench.DEFAULT_WORKLOAD]) == bench.METRIC
    m = bench.metric_of(inputs.BY_NAME["720p-train-taps-bf16"])
    assert m != bench.METRIC and "per-tap" in m and "720p-train-taps-bf16" in m


def test_algorithmic_units():
    w = inputs.BY_NAME["1080p-long-bf16"]
    # per (token, head): forward q, k, v, out (4 dh s) + offsets 12 + lse 4; backward 8 dh s + 28
    assert bench.alg_bytes_per_item(w, "fwd") == 4 * 128 * 2 + 16
    assert bench.alg_bytes_per_item(w, "bwd") == 8 * 128 * 2 + 28
    assert bench.alg_flop_per_item(w, "fwd") == 4 * 128 * 400  # B = 4 x 10 x 10 box tokens
    t = inputs.BY_NAME["720p-train-taps-bf16"]
    K = 243
    assert bench.alg_bytes_per_item(t, "dsa3d_fwd_taps_kernel") == 4 * 128 * 2 + 12 * K + 4
    assert bench.alg_bytes_per_item(t, "dsa3d_bwd_taps_kernel") == 8 * 128 * 2 + 24 * K + 4
    assert bench.alg_flop_per_item(t, "dsa3d_bwd_taps_kernel") == 64 * 128 * K
    assert bench.alg_bytes_per_item(t, "dsa3d_fwd_mma_kernel") == 0  # not a per-tap kernel


def test_traffic_is_reported_only_for_the_captured_sources(tmp_path, monkeypatch):
    # each capture's figures are reported exactly while its kernels' sources are unchanged, and
    # not at all once they have changed (bench.py then reports null traffic)
    for cap in bench.NCU_TRAFFIC:
        assert os.path.exists(os.path.join(ROOT, cap["capture"]))
        current = cap["sources"] == bench.sources_digest(cap["files"])
        for k in cap["bytes_per_item"]:
            want = cap["bytes_per_item"][k] if current else None
            assert bench.traffic_per_item(k)[0] == want
    # a changed source file voids its family's figures, not the other family's
    csrc = tmp_path / "deformable_slide_attention_b200" / "csrc"
    csrc.mkdir(parents=True)
    (tmp_path / "include").mkdir()
    real = os.path.join(ROOT, "deformable_slide_attention_b200", "csrc")
    for f in os.listdir(real):
        (csrc / f).write_bytes(open(os.path.join(real, f), "rb").read())
    (csrc / "dsa3d_taps.cuh").write_bytes((csrc / "dsa3d_taps.cuh").read_bytes() + b"\n")
    before = {k: bench.traffic_per_item(k)[0] for k in ("dsa3d_bwd_taps_kernel", "dsa3d_bwd_q_kernel")}
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.traffic_per_item("dsa3d_bwd_taps_kernel") == (None, None)
    assert bench.traffic_per_item("dsa3d_bwd_q_kernel")[0] == before["dsa3d_bwd_q_kernel"]


def test_dwconv_part_units_and_default():
    assert bench.parse_args([]).part == "attention"  # the default step is the operator's
    w = inputs.BY_NAME["1080p-long-bf16"]
    u = bench.dwconv_units(w)
    C, K = 32 * 128, 243
    assert u["fwd_bytes"] == u["bwd_bytes"] == 3 * C * 2
    assert u["fwd_flop"] == 2 * C * K and u["bwd_flop"] == 4 * C * K


def test_e2e_groups_option():
    """--e2e-groups picks the end-to-end leg's head groups; 0 (the default) keeps bench.py's own
    choice (the largest group with four groups or more that fits)."""
    assert bench.parse_args([]).e2e_groups == 0
    assert bench.parse_args(["--e2e-groups", "8"]).e2e_groups == 8
