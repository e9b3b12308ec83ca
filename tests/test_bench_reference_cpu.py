"""bench.py's reference arm (the CPU oracle) on this machine: the JSON line
carries the contract's keys, and under torchrun every rank but 0 exits 0
without work or output. Runs without a GPU."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(env_extra):
    env = dict(os.environ, **env_extra)
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl",
                           "reference", "--config", "tiny_fp32", "--steps", "2",
                           "--warmup", "3"],
                          cwd=ROOT, env=env, capture_output=True, text=True, timeout=300)


def test_reference_line_has_the_contract_keys():
    r = _run({"RANK": "0"})
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    j = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in j, key
    assert j["impl"] == "reference" and j["steps"] == 2 and j["warmup"] == 3
    assert j["value"] > 0 and j["cpu_baseline"]["value"] == j["value"]
    assert j["cpu_baseline"]["kind"] == "oracle" and j["cpu_baseline"]["cores"] >= 1
    assert j["e2e"]["h2d_bytes_per_step"] == 0 and j["e2e"]["d2h_bytes_per_step"] == 0
    # one sampled token per oracle thread (at most T)
    assert f"first {min(128, j['cpu_baseline']['cores'])} of 128 tokens" in \
        j["cpu_baseline"]["sample"]
    # the GPU arm builds its `config` with the same function, so the two arms'
    # lines name the same workload with the same keys
    sys.path.insert(0, ROOT)
    import bench
    from moe_synth import get_config
    assert j["config"] == bench.run_config(get_config("tiny_fp32"), 0, 1)


def test_default_workload_is_the_large_expert_layer():
    sys.path.insert(0, ROOT)
    import bench
    args = bench.make_parser().parse_args([])
    assert args.config == "large_e" and args.gpus == 1 and args.impl == "ours"


def test_reference_other_ranks_exit_quietly():
    r = _run({"RANK": "1"})
    assert r.returncode == 0, r.stderr[-2000:]
    assert not [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
