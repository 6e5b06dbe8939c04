"""bench.py without a GPU: the reference arm (the fp64 oracle on the host)
prints the contract's JSON line, its non-zero ranks exit quietly, and the
product arm refuses to run instead of falling back to the CPU."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench(args, env_extra=None, timeout=600):
    env = dict(os.environ)
    env.update(env_extra or {})
    env["CUDA_VISIBLE_DEVICES"] = ""          # no GPU, also on a GPU host
    return subprocess.run([sys.executable, "bench.py"] + args, cwd=ROOT, env=env, capture_output=True,
                          text=True, timeout=timeout)


def test_reference_arm_prints_the_contract_line():
    r = _bench(["--impl", "reference", "--steps", "1", "--warmup", "0", "--workload", "tinymlp"])
    assert r.returncode == 0, r.stderr[-2000:]
    line = json.loads(r.stdout.strip().splitlines()[-1])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline",
                "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["value"] > 0 and line["steps"] == 1
    assert line["unit"] == "TFLOP/s" and line["higher_is_better"] is True
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
    assert line["config"]["workload"] == "tinymlp"


def test_reference_arm_other_ranks_exit_quietly():
    r = _bench(["--impl", "reference", "--steps", "1", "--warmup", "0", "--workload", "tinymlp"],
               env_extra={"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"})
    assert r.returncode == 0 and r.stdout.strip() == ""


def test_product_arm_refuses_to_run_without_a_gpu():
    r = _bench(["--steps", "1", "--warmup", "3", "--workload", "tinymlp"], timeout=300)
    assert r.returncode != 0
    assert "{" not in r.stdout          # no JSON line: no CPU fallback number


def test_adamw_only_mode_refuses_to_run_without_a_gpu():
    r = _bench(["--adamw-only", "16", "--steps", "1"], timeout=300)
    assert r.returncode != 0
    assert "{" not in r.stdout
