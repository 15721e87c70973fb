"""The benchmark's reference arm on CPU: `bench.py --impl reference` times the fp64 oracle
on a bounded prefix of the workload and prints one JSON line with the same keys as the
GPU arm, plus `impl`, a `cpu_baseline` describing the run and a zero-copy `e2e`.  Under
torchrun only rank 0 works and prints; the other ranks exit 0 silently."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(extra_env=None, args=("--steps", "1", "--warmup", "3")):
    env = dict(os.environ)
    env.update(extra_env or {})
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", *args],
                          cwd=ROOT, env=env, capture_output=True, text=True, timeout=300)


def test_reference_arm_prints_the_contract_line():
    p = _run()
    assert p.returncode == 0, p.stderr[-2000:]
    lines = [l for l in p.stdout.strip().splitlines() if l.startswith("{")]
    assert len(lines) == 1, p.stdout
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference"
    assert d["steps"] == 1 and d["warmup"] == 3 and d["n_gpus"] == 1
    assert d["value"] > 0 and d["ms_per_step"] > 0 and d["higher_is_better"] is True
    assert d["config"]["workload"] == "c3_causal_n4m_clusters" and d["config"]["N"] == 4194304
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"] and cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    # tokens per step x steps / time agrees with the reported rate
    n = d["config"]["sample_tokens_per_step"]
    assert abs(n / (d["ms_per_step"] / 1e3) - d["value"]) <= 1e-6 * d["value"]


def test_reference_arm_other_ranks_exit_quietly():
    p = _run({"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"})
    assert p.returncode == 0, p.stderr[-2000:]
    assert not [l for l in p.stdout.splitlines() if l.startswith("{")]


def test_reference_arm_forward_only_workload():
    """The forward-only workload (bidirectional fp32 forward at N = 1024) is timed as a forward
    pass alone, under its own metric name."""
    p = _run(args=("--workload", "c1_noncausal_fwd_f32", "--steps", "2", "--warmup", "3"))
    assert p.returncode == 0, p.stderr[-2000:]
    lines = [l for l in p.stdout.strip().splitlines() if l.startswith("{")]
    assert len(lines) == 1, p.stdout
    d = json.loads(lines[0])
    assert d["metric"].startswith("RACE attn forward tokens/s")
    assert d["config"]["workload"] == "c1_noncausal_fwd_f32" and d["config"]["N"] == 1024
    assert d["cpu_baseline"]["sample"].startswith("bidirectional forward of the first 1024 tokens")


def test_step_work_of_forward_only_and_full_steps():
    """Algorithmic bytes and flops per token: a forward reads q, k, v and writes out and den;
    forward + backward also reads dO, out and den twice over and writes dq, dk, dv."""
    sys.path.insert(0, ROOT)
    import bench
    import race_inputs
    c1 = race_inputs.WORKLOADS["c1_noncausal_fwd_f32"]
    M, D, LP, d = c1.L * c1.R, c1.d + 1, c1.L * c1.P, c1.d
    assert bench.step_work(c1) == (4 * d * 4 + 4, 4 * M * D + 4 * LP * d)
    c3 = race_inputs.WORKLOADS["c3_causal_n4m_clusters"]
    assert bench.step_work(c3) == (1544, 248832)
    # the general path's bidirectional pass named fwd_walk is a read-out
    assert bench.kernel_work("generic_fwd_walk", c1) == (2 * d * 4 + 4, 2 * M * D + 2 * LP * d)
