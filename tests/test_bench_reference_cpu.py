"""The benchmark's reference arm (the oracle on the host cores) runs without a GPU: one JSON line
with the contract's keys on rank 0, nothing on the other ranks."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(extra_env=None):
    env = dict(os.environ)
    env.update(extra_env or {})
    res = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload", "tiny",
                          "--steps", "1", "--warmup", "1"], capture_output=True, text=True, env=env, timeout=600,
                         cwd=ROOT)
    assert res.returncode == 0, res.stderr[-2000:]
    return [l for l in res.stdout.splitlines() if l.strip()]


def test_reference_arm_prints_one_contract_line():
    lines = _run()
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["value"] > 0 and d["higher_is_better"] is True
    assert d["config"]["workload"] == "tiny"
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0


def test_reference_arm_is_silent_off_rank_zero():
    assert _run({"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"}) == []


def _bench_module():
    import importlib.util
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_roofline_arithmetic_and_committed_dram_summary():
    """The roofline object of the bench line on made-up stage times: the dominant stage, its
    algorithmic bytes over its time, the step's fraction over both directions' bytes, and the
    traffic read from the committed ncu summary of the med4b step (one figure per stage, and the
    stages add up to the step total written beside them)."""
    B = _bench_module()
    stages = {"forward": 2.0, "allocate": 0.1, "pack": 0.6, "decode_index": 0.03, "idct_hw": 1.4, "idct_s": 1.1}
    prof = {"stages": stages, "compress_ms": 2.7, "decompress_ms": 2.53}
    in_bytes, pay, bins = 2_000_000_000, 130_000_000, 1_000_000
    r = B.stage_roofline(prof, in_bytes, pay, bins, 5.5, 6500.0, "measured", "med4b")
    assert r["kernel"] == "forward" and r["algorithmic_bytes"] == in_bytes
    assert abs(r["achieved"] - in_bytes / 2.0e-3 / 1e9) < 0.1 and abs(r["frac"] - r["achieved"] / 6500.0) < 1e-4
    assert abs(r["step_achieved"] - 2 * (in_bytes + pay) / 5.5e-3 / 1e9) < 0.1
    assert abs(r["compress_frac"] - (in_bytes + pay) / 2.7e-3 / 1e9 / 6500.0) < 1e-4
    per_stage = {s: B.dram_traffic("med4b", s) for s in stages}
    assert all(v and v > 0 for v in per_stage.values()), per_stage
    assert r["traffic"] == per_stage["forward"]
    total = [int(l.split(":")[1]) for l in open(os.path.join(ROOT, "profiles", "med4b_dram_bytes.txt"))
             if l.startswith("dram_bytes_per_step:")]
    assert total and total[0] == sum(per_stage.values())
    assert B.dram_traffic("no_such_workload", "forward") is None
