"""bench.py's reference arm (the oracle timed on the host's cores) keeps the JSON-line contract:
one line with the metric, the workload, a cpu_baseline describing the run and an e2e object; and
under a multi-rank launch only rank 0 works and prints."""

import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(env_extra):
    env = dict(os.environ, **env_extra)
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1", "--warmup", "1"],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    return [ln for ln in r.stdout.splitlines() if ln.startswith("{")]


def test_reference_arm_line():
    lines = _run({"WORLD_SIZE": "1", "RANK": "0"})
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["value"] > 0 and d["unit"] == "us/step"
    assert d["higher_is_better"] is False and d["n_gpus"] == 1 and d["data"] == "synthetic"
    assert d["config"]["workload"] == "qwen3-8b-32k-decode-step"
    assert d["config"]["seq_len"] == 32768 and d["config"]["token_budget"] == 4096
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == d["value"] and cb["sample"]
    # the whole batch, dealt to one process per host core (as many as there are pairs at most)
    assert "every one of the 64" in cb["sample"] and f"to {cb['cores']} host processes" in cb["sample"]
    assert 1 <= cb["cores"] <= min(64, os.cpu_count())
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    assert abs(d["ms_per_step"] - d["value"] / 1e3) < 1e-9


def test_reference_arm_other_ranks_exit_quietly():
    assert _run({"WORLD_SIZE": "2", "RANK": "1", "LOCAL_RANK": "1"}) == []
