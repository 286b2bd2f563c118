"""bench.py's JSONL log on CPU (the reference arm, which needs no GPU): the
line is appended with the commit and its key, and a rerun with --skip-logged
prints the logged line and runs nothing (a killed sweep resumes)."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench(*args):
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], capture_output=True, text=True,
                       timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    return json.loads(lines[0])


def test_log_appends_and_skip_logged_resumes(tmp_path):
    log = str(tmp_path / "bench.jsonl")
    common = ["--impl", "reference", "--workload", "tiny", "--steps", "1", "--warmup", "0", "--ref-rows", "4",
              "--log", log]
    first = _bench(*common)
    assert first["impl"] == "reference" and first["config"]["workload"] == "tiny"
    rows = [json.loads(x) for x in open(log)]
    assert len(rows) == 1
    key = rows[0]["log_key"]
    assert key["workload"] == "tiny" and key["impl"] == "reference" and key["steps"] == 1 and key["git_sha"]
    assert rows[0]["value"] == first["value"]
    # the same entry again: the logged line is printed, nothing runs or is appended
    again = _bench(*common, "--skip-logged")
    assert again == first
    assert len(open(log).read().splitlines()) == 1
    # another entry (more steps) runs and is appended
    _bench(*common[:-2], "--log", log, "--steps", "2", "--skip-logged")
    assert len(open(log).read().splitlines()) == 2
