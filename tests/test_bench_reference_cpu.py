"""Host-side parts of the benchmark.  The reference arm (the oracle timed on
the host cores) keeps the benchmark line contract: one JSON line on rank 0
with the metric, unit, direction and workload of the CUDA arm, a
cpu_baseline describing the run and a zero-copy e2e; the other ranks of a
torchrun launch exit 0 without work.  The algorithmic byte count behind the
roofline's `achieved` matches a count by hand."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _run(env_extra):
    env = dict(os.environ, **env_extra)
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "2",
                           "--warmup", "1"], cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)


def test_reference_arm_line(monkeypatch):
    monkeypatch.setattr(sys, "argv", ["bench.py"])
    default_desc = bench.Workload(bench.parse(), 0).desc
    r = _run({})
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.strip().startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference"
    assert d["metric"] == bench.METRIC and d["unit"] == bench.UNIT
    assert d["higher_is_better"] is True and d["scaling"] == "weak"
    assert d["steps"] == 2 and d["warmup"] == 1 and d["n_gpus"] == 1
    assert d["value"] > 0 and d["ms_per_step"] > 0
    assert abs(d["value"] - d["config"]["batch"] * d["config"]["layers"] / (d["ms_per_step"] / 1e3)) < 1e-6 * d["value"]
    cfg = d["config"]
    assert (cfg["batch"], cfg["seq_len"], cfg["topk"], cfg["layers"]) == (8, 16384, 64, 1)
    assert cfg["workload"] == default_desc
    # the CUDA arm's config object, key for key
    assert cfg == bench.run_config(bench.Workload(bench.parse(), 0), bench.parse(), 1)
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == d["value"] and cb["cores"] >= 1 and cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_reference_arm_other_ranks_exit_quietly():
    r = _run({"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"})
    assert r.returncode == 0, r.stderr[-2000:]
    assert not [ln for ln in r.stdout.splitlines() if ln.strip().startswith("{")]


def test_algorithmic_bytes_of_the_default_step(monkeypatch):
    """The roofline numerator of the default workload (NOSA-1B, B=8, L=16384,
    16 q / 2 KV heads, top-k 64, 16 local blocks), counted by hand per
    (sequence, KV head): 1023 windows, 256 blocks, 240 candidates."""
    monkeypatch.setattr(sys, "argv", ["bench.py"])
    wl = bench.Workload(bench.parse(), 0)
    G = 8
    pool = 2 * 256 + 2 * 256 + 1 * (31 * 256 + 512)    # new K/V rows in and out; the window token 16383 completes
    select = 960 * 512 + G * 256 + 64 * 4 + 4           # windows of the 240 candidate blocks (fp32), q, selection
    decode = (64 * 64 + 16 * 64) * 2 * 256 + 2 * G * 256 + 64 * 4 + 4   # 80 tiles of K and V, q + out, selection
    per_pair = pool + select + decode
    m = wl.bytes_model()
    assert sum(m.values()) == 16 * per_pair == 50_065_536
