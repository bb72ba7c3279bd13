"""The bench's reference arm (the oracle timed on the host) and its JSON line,
on CPU."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(args, env=None):
    e = dict(os.environ)
    e.update(env or {})
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], cwd=ROOT, env=e,
                          capture_output=True, text=True, timeout=600)


def test_reference_arm_prints_one_contract_line():
    r = _run(["--impl", "reference", "--steps", "1", "--warmup", "0", "--workload", "c1"])
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["value"] > 0 and d["unit"] == "scores/s"
    for key in ("metric", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling", "dtype", "data",
                "config"):
        assert key in d, key
    assert d["higher_is_better"] is True and d["vs_baseline"] is None
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] == 1 and cb["value"] == d["value"] and cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": "scores/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    assert "c1" in d["config"]["workload"]


def test_reference_arm_other_ranks_do_nothing():
    r = _run(["--impl", "reference", "--steps", "1", "--warmup", "0", "--workload", "c1"], env={"RANK": "1"})
    assert r.returncode == 0 and r.stdout.strip() == ""


def test_traffic_key_ignores_comments_only():
    sys.path.insert(0, ROOT)
    import bench

    src = "int a; // note\n/* block\n   comment */ int b;  \n\n  // only a comment\nint c;\n"
    assert bench.code_only(src) == "int a;\n int b;\nint c;"
    assert bench.code_only(src.replace("note", "another note")) == bench.code_only(src)
    assert bench.code_only(src.replace("int c;", "int d;")) != bench.code_only(src)
