"""The bench's reference arm (the oracle on the host cores) prints one JSON line of the contract.

Runs on CPU: `bench.py --impl reference` times the oracle on a bounded sample of the 100M-token
workload (a process pool over the host cores) and never touches a GPU."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_prints_one_contract_line():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "0"], capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.strip().startswith("{")]
    assert len(lines) == 1, r.stdout
    d = json.loads(lines[0])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["value"] > 0 and d["higher_is_better"] is True
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["value"] == d["value"]
    # the same workload name and sizes as the GPU arm's line
    sys.path.insert(0, ROOT)
    import bench

    assert d["config"]["workload"] == bench.workload_label()


def test_traffic_record_follows_the_code_not_the_comments(tmp_path, monkeypatch):
    # the DRAM-traffic figure is used only while the scan's code hashes to the recorded digest;
    # comments and blank lines do not count
    sys.path.insert(0, ROOT)
    import bench

    csrc = tmp_path / "long_context_memory_b200" / "csrc"
    csrc.mkdir(parents=True)
    (tmp_path / "profiles").mkdir()
    (csrc / "k.cu").write_text("int f() {  // a comment\n  return 1;\n}\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    digest = bench.source_digest(["k.cu"])
    (tmp_path / "profiles" / "scan_traffic.txt").write_text(
        f"# capture notes\nsources: k.cu\ncode_sha256: {digest}\ndram_bytes_per_launch_full_size: 1234\n")
    assert bench.scan_traffic_record("scan") == 1234.0
    (csrc / "k.cu").write_text("int f() {  // another comment\n\n  return 1;\n}\n")
    assert bench.scan_traffic_record("scan") == 1234.0
    (csrc / "k.cu").write_text("int f() {\n  return 2;\n}\n")
    assert bench.scan_traffic_record("scan") is None
    assert bench.scan_traffic_record("no_such_kernel") is None


def test_profiles_are_short_text_summaries_with_their_commands():
    d = os.path.join(ROOT, "profiles")
    for f in sorted(os.listdir(d)):
        assert f.endswith((".md", ".txt")), f
        text = open(os.path.join(d, f), encoding="utf-8").read()
        assert len(text) < 16_000, f
        assert any(cmd in text for cmd in ("ncu ", "nvcc ")), f"{f} does not give the command that made it"
