"""Host-side rules of bench.py (CPU): the source hash behind the ncu traffic
figure ignores comments and blank space but not code, and the whole-job
throughput is all ranks' work over the slowest rank's time; the reference arm
(the oracle on host cores) prints the contract's JSON line on rank 0 only."""
import os

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_code_only_hash_ignores_comments_not_code():
    a = "int f(int x) {  // doubles x\n  return 2 * x;  /* twice */\n}\n"
    b = "// a comment line\nint f(int x) {\n\n  return 2 * x;\n}\n"
    c = "int f(int x) {\n  return 3 * x;\n}\n"
    assert bench._code_only(a) == bench._code_only(b)
    assert bench._code_only(a) != bench._code_only(c)


def test_aggregate_uses_the_slowest_rank():
    value, ms_per_step = bench.aggregate([90.0, 120.0, 100.0], [1e12] * 3, 10)
    assert ms_per_step == 12.0
    assert value == 3e12 / 0.120


def _run_reference(env_extra):
    import json
    import subprocess
    import sys
    env = dict(os.environ, **env_extra)
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "3"], capture_output=True, text=True, timeout=300, env=env, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    return [json.loads(ln) for ln in lines]


def test_reference_arm_json_line():
    """The oracle arm: one JSON line with the contract's keys, its own value repeated
    as cpu_baseline and e2e (no host-device copies)."""
    (line,) = _run_reference({"RANK": "0", "WORLD_SIZE": "1"})
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config"):
        assert key in line, key
    assert line["impl"] == "reference" and line["steps"] == 1 and line["warmup"] == 3
    assert line["value"] > 0 and line["unit"] == "TFLOP/s" and line["higher_is_better"] is True
    assert "workload" in line["config"]
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == line["value"] and cb["cores"] >= 1 and cb["sample"]
    e2e = line["e2e"]
    assert e2e["value"] == line["value"] and e2e["unit"] == line["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0


def test_reference_arm_other_ranks_print_nothing():
    assert _run_reference({"RANK": "1", "WORLD_SIZE": "2"}) == []


def test_cpu_baseline_leg_reports_all_and_single_thread_figures():
    from diffusion_transformer_denoising_dit_b200 import synth
    w = synth.WORKLOADS["tiny"]
    q, k, v = synth.qkv(w)
    pos = synth.positions(w.T, w.G).numpy()
    line = bench.cpu_baseline_leg(q, k, v, pos, w, seconds=0.0)
    assert line["kind"] == "oracle" and line["unit"] == "TFLOP/s" and line["value"] > 0 and line["cores"] >= 1
    assert "1 of 2 heads" in line["sample"]          # always one head, more only while the budget lasts
    assert "2 of 2 heads" in bench.cpu_baseline_leg(q, k, v, pos, w, seconds=60.0)["sample"]
    st = line["single_thread"]
    assert st["cores"] == 1 and st["value"] > 0 and "288 query rows" in st["sample"]
