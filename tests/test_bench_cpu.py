"""bench.py's reference arm (the oracle, timed on the host cores) on CPU: one step of a
one-row sample prints one JSON line with the contract's keys, and the oracle-table mode
reports both builds for a config."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_json_line():
    env = dict(os.environ)
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        env.pop(k, None)
    out = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1", "--warmup", "1",
                          "--sample-rows", "1"], cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "impl", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["value"] > 0 and d["steps"] == 1
    assert d["config"]["workload"].startswith("llama3_8b_gate_up_prefill_4096x14336x4096 (sampled")
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["value"] == d["value"]


def test_oracle_table_one_config(monkeypatch, capsys):
    import bench
    orig = bench.oracle_configs
    monkeypatch.setattr(bench, "oracle_configs", lambda: [c for c in orig() if c[0] == "C1"])
    rows = bench.oracle_table(None)
    assert [r["mode"] for r in rows] == ["single-thread", "openmp"]
    for r in rows:
        assert r["oracle_table"] == "C1" and r["gemm_rows"] == "all" and r["gemm_mac_per_s"] > 0
        assert r["quantise_elems"] == 16 * 256 + 128 * 256
