"""The benchmark's contract, checked on CPU: the JSON line of the reference arm (the
fp64 oracle, the one arm that runs without a GPU), its torchrun behaviour (rank 0
prints, the other ranks exit 0 without work), and the algorithmic byte counts the
roofline divides by."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402

KEYS = ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
        "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config", "impl",
        "cpu_baseline", "e2e")


def run(args, env=None):
    out = subprocess.run([sys.executable, "bench.py", *args], cwd=ROOT, capture_output=True,
                         text=True, timeout=600, env=env)
    assert out.returncode == 0, out.stderr[-2000:]
    return [json.loads(l) for l in out.stdout.splitlines() if l.startswith("{")]


@pytest.mark.parametrize("family", ["wkv7", "gdn", "sane"])
def test_reference_arm_line(family):
    lines = run(["--impl", "reference", "--steps", "1", "--warmup", "1", "--family", family])
    assert len(lines) == 1
    d = lines[0]
    for k in KEYS:
        assert k in d, k
    assert d["impl"] == "reference" and d["unit"] == "tokens/s" and d["value"] > 0
    assert d["higher_is_better"] is True and d["scaling"] == "weak"
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}
    assert d["metric"] == {"gdn": bench.GDN_METRIC, "sane": bench.SANE_METRIC}.get(family,
                                                                                  bench.METRIC)
    assert d["config"]["workload"].endswith("fwd_bf16_b8_t4096_h64")


def test_reference_arm_under_torchrun():
    env = dict(os.environ, OMP_NUM_THREADS="2")
    out = subprocess.run([sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
                          "--nproc-per-node", "2", "--master-addr", "127.0.0.1",
                          "--master-port", "29531", "bench.py", "--impl", "reference",
                          "--gpus", "2", "--steps", "1", "--warmup", "1"],
                         cwd=ROOT, capture_output=True, text=True, timeout=600, env=env)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [json.loads(l) for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1 and lines[0]["n_gpus"] == 2


def test_algorithmic_bytes():
    # forward: 6 bf16 inputs + bf16 output per token-head, fp32 s0 and sT per unit
    assert bench.fwd_algorithmic_bytes(8, 4096, 64) == 8 * 4096 * 64 * 7 * 128 + 2 * 512 * 16384
    assert bench.fwd_algorithmic_bytes(8, 4096, 64) == 1_895_825_408
    # decode: the state read and written once, 6 inputs + 1 output vector per unit
    assert bench.step_algorithmic_bytes(1024, 32) == 1_103_101_952
    # Gated DeltaNet: q, k, v, o vectors + g, beta scalars (bf16)
    assert bench.gdn_fwd_algorithmic_bytes(8, 4096, 64) == 8 * 4096 * 64 * 516 + 2 * 512 * 16384
    assert bench.gdn_step_algorithmic_bytes(1024, 32) == 1024 * 32 * (2 * 16384 + 516)
    # head sizes scale the vectors by D and the states by D^2
    assert bench.fwd_algorithmic_bytes(8, 4096, 32, 128) == (8 * 4096 * 32 * 7 * 256
                                                             + 2 * 256 * 128 * 128 * 4)
