"""Host-side logic of bench.py (no GPU): the algorithmic bytes of each row of
the step, and the lookup of ncu traffic with its staleness check (a kernel's
captured DRAM bytes count only while the code of its source files is
unchanged; comment edits do not count as changes)."""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import workloads as W  # noqa: E402


def test_code_only_drops_comments_and_blank_lines():
    src = "int a; // one\n/* two\n   lines */ int b;\n\n   \nint c;  \n"
    assert bench._code_only(src) == "int a;\n int b;\nint c;"


def test_files_sha_ignores_comments_but_not_code(tmp_path):
    f = tmp_path / "k.cu"
    f.write_text("__global__ void k() { x = 1; }  // note\n")
    h0 = bench._files_sha([str(f)])
    f.write_text("// a new comment\n__global__ void k() { x = 1; }  /* other */\n")
    assert bench._files_sha([str(f)]) == h0
    f.write_text("__global__ void k() { x = 2; }\n")
    assert bench._files_sha([str(f)]) != h0


def test_traffic_scaled_by_units_and_dropped_when_the_code_changes(tmp_path, monkeypatch):
    src = tmp_path / "row.cu"
    src.write_text("__global__ void row_update() {}\n")
    entry = {"dram_bytes_per_launch": 1000.0, "units": 10, "l2_hit_pct": 42.0, "files": [str(src)],
             "sha256": bench._files_sha([str(src)]), "note": "captured"}
    tj = tmp_path / "traffic.json"
    tj.write_text(json.dumps({"large": {"row_update": entry}}))
    monkeypatch.setattr(bench, "TRAFFIC", str(tj))
    b, hit, note = bench._traffic("large", "row_update", 80)
    assert b == 8000.0 and hit == 42.0 and "scaled by 8.000" in note
    assert bench._traffic("large", "pool", 80)[0] is None
    assert bench._traffic("criteo26", "row_update", 80)[0] is None
    src.write_text("// only a comment more\n__global__ void row_update() {}\n")
    assert bench._traffic("large", "row_update", 10)[0] == 1000.0
    src.write_text("__global__ void row_update() { int x; }\n")
    b, hit, note = bench._traffic("large", "row_update", 10)
    assert b is None and "changed" in note


def test_algorithmic_bytes_of_each_row():
    # one table, D = 64, Adam (s = 2), pooled only: N = 1000 occurrences,
    # U = 300 unique keys, 50 new keys, F * B = 2 * 100 bags
    w = W.WORKLOADS["criteo26"].scaled(100)
    w.tables = [W.TableSpec("t", [0, 1], 64, "adam", 1e-3, "sum", init_seed=1)]
    a = bench._alg_bytes(w, [(1000, 300, 50)])
    D, s, N, U, n_new, bags = 64, 2, 1000, 300, 50, 200
    assert a["feature_hash"] == 16 * N
    assert a["dedup"] == 8 * N + 4 * N + 16 * U + 16 * U + 4 * D * (1 + s) * n_new
    assert a["gather_pool"] == 4 * D * U + 4 * D * bags + 8 * bags
    assert a["backward"] == 4 * D * bags + 2 * 4 * D * (1 + s) * U


def test_reference_arm_times_exactly_k_steps_after_w_warmups():
    # the reference arm (the CPU oracle) prints one line of exactly K timed
    # steps; the tiny workload keeps it to a second
    import subprocess
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--workload", "tiny", "--steps", "3", "--warmup", "2"],
                         capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    line = json.loads([ln for ln in out.stdout.splitlines() if ln.startswith("{")][-1])
    assert line["impl"] == "reference" and line["steps"] == 3 and line["warmup"] == 2
    assert line["value"] > 0 and line["cpu_baseline"]["sample"].startswith("3 ")
    assert line["e2e"] == {"value": line["value"], "unit": "IDs/s", "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}
