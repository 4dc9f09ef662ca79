"""The bench's reference arm (the oracle timed on the host cores) runs without a
GPU and prints one JSON line with the contract's keys."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_json_line():
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--config", "35b_decode", "--steps", "2",
                        "--warmup", "1"], cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["steps"] == 2 and d["warmup"] == 1
    assert d["value"] > 0 and d["higher_is_better"] is True
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["value"] == d["value"]
    assert d["config"]["workload"] == "35b_decode T=64"
    assert d["cpu_baseline"]["cpu_model"]
    # the reference arm's config block is the one this arm prints for the same workload
    import bench
    import synth
    assert d["config"] == bench.workload_config(synth.CONFIGS["35b_decode"], 64, 1)


def test_default_workload_is_the_largest_layer():
    import bench
    import synth
    name, T = bench.HEADLINE
    cfg = synth.CONFIGS[name]
    # the 753B-class layer: the widest hidden size and the largest batch of the five configs
    assert cfg.d == max(c.d for c in synth.CONFIGS.values())
    assert T == max(t for c in synth.CONFIGS.values() for t in c.T)
    covered = {(n, t) for n, ts in bench.SUITE for t in ts} | {bench.HEADLINE}
    want = {(n, t) for n, c in synth.CONFIGS.items() if n != "tiny" for t in c.T}
    assert covered == want


def test_graph_plan_covers_exactly_the_steps():
    import bench
    r = bench.Runner.__new__(bench.Runner)
    r.chunk = 20
    for n in (1, 5, 20, 21, 47, 100):
        plan = r._plan(n)
        assert sum(k for k, _ in plan) == n
        assert [t for _, t in plan] == [i % 2 for i in range(len(plan))]


def test_reference_arm_other_ranks_exit_quietly():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1", "--warmup", "0"],
                       cwd=ROOT, capture_output=True, text=True, timeout=600, env=env)
    assert r.returncode == 0, r.stderr[-2000:]
    assert not [l for l in r.stdout.splitlines() if l.startswith("{")]
