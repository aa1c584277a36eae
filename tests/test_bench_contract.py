"""bench.py's reference arm (the CPU oracle timed on the host cores) prints the
contract's JSON line; runs on CPU."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_json_line():
    env = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1", "--warmup", "0"],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    d = json.loads(lines[0])
    for k in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
              "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert k in d, k
    assert d["impl"] == "reference" and d["higher_is_better"] is True and d["value"] > 0
    assert d["config"]["workload"] == "llama2_7b"
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_variant_helpers():
    """The timed kernel's name and the CPU baseline follow --variant: the
    oracle sample runs the variant's options (stochastic rounding with either
    draw width, clipping) and says so."""
    sys.path.insert(0, ROOT)
    import argparse

    import bench

    names = {v: bench.kernel_name(argparse.Namespace(variant=v, no_tma=False))
             for v in ("default", "sr", "sr16", "history", "clip", "jit")}
    assert names["default"] == "fp8adam_step_tma_kernel<E4M3,E5M2>"
    assert "SRK=1" in names["sr"] and "SRK=2" in names["sr16"] and "SRK=0" in names["history"]
    assert names["clip"].endswith("grad-norm pre-pass") and names["jit"].endswith("amax pre-pass")
    for v in ("sr16", "clip"):
        value, ms, threads, desc = bench.run_oracle_sample("llama2_100m", 1, 1, single_thread=True, variant=v)
        assert value > 0 and ms > 0 and threads == 1 and ("variant " + v) in desc
    assert bench.workload_config("llama2_7b", 1, "sr16")["variant"] == "sr16"
