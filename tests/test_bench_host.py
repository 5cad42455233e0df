"""Host-side logic of bench.py (CPU only): algorithmic bytes, the statistics
kernel the library picks, the committed-traffic lookup and the reference
leg's JSON line."""
import hashlib
import json
import os
import subprocess
import sys

import numpy as np
import pytest

import bench
from speculative_decoding_block_spec_b200 import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_window_and_step_bytes():
    w = synth.WORKLOADS[2]
    vl = np.full(w.B, w.L)
    # 8 requests x (16 target + 16 draft rows) x 151936 x 2 B
    assert bench.window_bytes(w, vl) == 256 * 151936 * 2 == 77791232
    acc = np.zeros(w.B, np.int32)  # every request rejects: no bonus row
    small = w.B * (w.L * 4 * 2 + 4 + (w.L + 1) * 4)
    assert bench.step_bytes(w, vl, acc) == 77791232 + w.B * w.V * 4 + small
    acc[:3] = w.L  # three requests accept everything: one bonus target row each
    assert bench.step_bytes(w, vl, acc) == 77791232 + w.B * w.V * 4 + 3 * w.V * 2 + small
    w4 = synth.WORKLOADS[4]
    vl4 = np.full(w4.B, 7)
    assert bench.window_bytes(w4, vl4) == w4.B * 7 * 2 * w4.V * 2


def test_stats_kernel_choice_mirrors_the_library():
    names = {cid: bench.stats_kernel_name(synth.WORKLOADS[cid], 148) for cid in synth.WORKLOADS}
    assert names[2] == "k_row_stats_dyn"  # 78 MB window, 1.7 rows per SM share
    assert names[1] == "k_row_stats"      # too small for a slice per warp
    assert names[3] == names[5] == "k_row_stats"  # windows above 256 MB
    assert names[4] == "k_row_stats"      # dense upper bound 311 MB
    odd = synth.Workload(99, "odd", 8, 16, 50257, 1, 1.0, "f32", 1.0, 0, 0.0, 1.0)
    assert bench.stats_kernel_name(odd, 148) == "k_row_stats"  # rows not 16-byte vectors


def test_headline_is_the_largest_workload_and_extras_follow():
    a = bench.parse_args([])
    assert a.workload == 5 and synth.WORKLOADS[a.workload].name == "stress B64 L16 V151936 K4 bf16 budget544"
    assert a.extra_ids == [1, 2, 3, 4]
    assert bench.parse_args(["--extras", ""]).extra_ids == []
    assert bench.parse_args(["--workload", "3", "--extras", "2,3"]).extra_ids == [2]


def test_both_arms_describe_the_workload_alike():
    w = synth.WORKLOADS[5]
    c = bench.config_of(w, 4, 1)
    assert c["workload"] == w.name and c["budget"] == 544 and c["parallelism"] == "dp1"
    assert "above the 126 MB L2" in c["l2"]
    # one input set: target 64x17 rows + packed 544 rows + draft 64x4x16 rows (bf16), Gumbel 64x17 rows (fp32)
    V = w.V
    expect = 64 * 17 * V * 2 + 544 * V * 2 + 64 * 4 * 16 * V * 2 + 64 * 17 * V * 4 + 64 * 16 * 8 + 64 * 4 * 4 \
        + 64 * 16 * 4
    assert bench.set_bytes(w) == expect
    assert "NOT above" in bench.l2_note(synth.WORKLOADS[1], 4)


def test_spread():
    s = bench.spread([3.0, 1.0, 2.0, 5.0, 4.0])
    assert s["median_ms"] == 3.0 and s["min_ms"] == 1.0 and s["max_ms"] == 5.0 and s["n"] == 5
    assert s["p10_ms"] <= s["median_ms"] <= s["p90_ms"]


def _ref(acc, out, margins, gaps, kappas):
    return {"accept_len": np.array(acc), "out_tokens": np.array(out), "accept_margin": np.array(margins),
            "argmax_gap": np.array(gaps), "argmax_kappa": np.array(kappas)}


def test_margin_report_counts_decisions_and_low_margins():
    # two requests, L = 3: request 0 rejects at 1 (2 accept tests + draw), request 1 accepts all (3 + draw)
    ref = _ref([1, 3], [[7, 9, -1, -1], [1, 2, 3, 4]], [[0.3, 0.2, 0.1], [0.5, 0.5, 0.5]], [1.0, 2.0], [1.0, 1.0])
    acc = np.array([1, 3])
    out = np.array([[7, 9, -1, -1], [1, 2, 3, 4]])
    r = bench.margin_report(acc, out, ref, None)
    assert r["decisions"] == 3 + 4 and r["low_margin"] == 0 and r["mismatches"] == 0
    out2 = out.copy()
    out2[1, 3] = 5
    assert bench.margin_report(acc, out2, ref, None)["mismatches"] == 1
    # the same difference under a low-margin terminal draw is exempt
    ref_low = dict(ref, argmax_gap=np.array([1.0, 1e-8]))
    r = bench.margin_report(acc, out2, ref_low, None)
    assert r["low_margin"] == 1 and r["exempted_differences"] == 1 and r["mismatches"] == 0
    # a low-margin accept test exempts the request's later outputs
    ref_acc = dict(ref, accept_margin=np.array([[0.3, 5e-7, 0.1], [0.5, 0.5, 0.5]]))
    acc3 = np.array([2, 3])
    out3 = np.array([[7, 8, 6, -1], [1, 2, 3, 4]])
    r = bench.margin_report(acc3, out3, ref_acc, None)
    assert r["low_margin"] == 1 and r["exempted_differences"] == 1 and r["mismatches"] == 0


def test_committed_traffic_needs_matching_source(tmp_path, monkeypatch):
    src = tmp_path / "k.cu"
    src.write_text("kernel source v1\n")
    (tmp_path / "profiles").mkdir()
    digest = hashlib.sha256(src.read_bytes()).hexdigest()
    (tmp_path / "profiles" / "k_w.md").write_text(
        "kernel: k_row_stats\nworkload: block B8\ntraffic_bytes_per_launch: 12345\n"
        "source_sha256: %s\nsource_files: k.cu\n" % digest)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.committed_traffic("k_row_stats", "block B8") == (12345, os.path.join("profiles", "k_w.md"))
    assert bench.committed_traffic("k_row_stats_dyn", "block B8") == (None, None)
    assert bench.committed_traffic("k_row_stats", "other") == (None, None)
    src.write_text("kernel source v2\n")  # the kernel changed after the capture
    assert bench.committed_traffic("k_row_stats", "block B8") == (None, None)


def test_committed_profiles_parse():
    """Every committed ncu summary that names a traffic figure also names its
    kernel, workload and the sources it was taken on."""
    pdir = os.path.join(ROOT, "profiles")
    for name in sorted(os.listdir(pdir)):
        text = open(os.path.join(pdir, name)).read()
        if "traffic_bytes_per_launch:" not in text:
            continue
        for key in ("kernel:", "workload:", "source_sha256:", "source_files:", "command:"):
            assert key in text, (name, key)
        files = text.split("source_files:")[1].split("\n")[0].split()
        assert files and all(os.path.exists(os.path.join(ROOT, f)) for f in files), name


def test_reference_leg_prints_one_json_line():
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--workload", "1", "--steps", "2",
                        "--warmup", "3"], cwd=ROOT, capture_output=True, text=True, env=env, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["metric"] == bench.METRIC and d["unit"] == bench.UNIT
    assert d["value"] > 0 and d["steps"] == 2 and d["warmup"] == 3
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    assert d["config"] == bench.config_of(synth.WORKLOADS[1], 4, 1)
