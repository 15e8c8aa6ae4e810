"""Host-side logic of bench.py: the algorithmic byte counts behind the
roofline, the step kind of each workload, and the oracle reference arm on a
tiny case (CPU only)."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from workloads import WORKLOADS, get_workload  # noqa: E402


def test_decode_bytes_per_layer_qwen05b():
    # per (sequence, layer): (28 + e) H + (4e + 8 + 2 k e) n_kv d; per layer 256 H of slots
    w = WORKLOADS["qwen05b"]
    dec, _ = bench.workload_bytes(w)
    assert dec == 24 * 266_496 == 6_395_904


def test_decode_bytes_batched_k16():
    # 152,064 B per (sequence, layer) with the 256 H slot bytes shared over the batch
    w = get_workload("batched_decode_k16_g0.9_a1.0")
    dec, _ = bench.workload_bytes(w)
    assert dec == 28 * 256 * 152_064


def test_decode_bytes_qwen7b():
    w = WORKLOADS["qwen7b_decode"]
    dec, _ = bench.workload_bytes(w)
    assert dec == 28 * 1_065_984


def test_prefill_bytes_qwen05b_512():
    # 5,888 B per token and layer, the state once per stream, slots once per layer
    w = WORKLOADS["qwen05b"]
    _, pre = bench.workload_bytes(w)
    state = 2 * 16 * 128 * 2 + 4 * 128 + 72 * 896
    assert pre == 24 * 512 * 5_888 + 24 * state + 24 * 256 * 896
    assert pre == 79_613_952


def test_prefill_bytes_follow_the_context():
    w = WORKLOADS["qwen7b_decode"]
    _, p1 = bench.workload_bytes(w, 1024)
    _, p8 = bench.workload_bytes(w, 8192)
    per_tok_layer = 2 * 3584 + 2 * 2 * 512 + 4 * 3584
    assert p8 - p1 == 28 * (8192 - 1024) * per_tok_layer


def test_step_kinds():
    assert bench.step_kind(WORKLOADS["qwen05b"]) == "step"
    assert bench.step_kind(WORKLOADS["tiny"]) == "step"
    assert bench.step_kind(WORKLOADS["qwen7b_decode"]) == "step"
    assert bench.step_kind(WORKLOADS["long_prefill"]) == "prefill"
    assert bench.step_kind(WORKLOADS["batched_decode"]) == "decode"
    assert bench.step_kind(get_workload("batched_decode_k256_g0.98_a10.0")) == "decode"


def test_reference_arm_prints_one_json_line():
    env = dict(os.environ, OMP_NUM_THREADS="2")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", "tiny", "--steps", "2", "--warmup", "0"],
                       capture_output=True, text=True, timeout=300, env=env, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference"
    assert d["value"] > 0 and d["unit"] == "tokens/s"
    assert d["cpu_baseline"]["kind"] == "oracle"
    assert d["e2e"]["h2d_bytes_per_step"] == 0
    assert d["config"]["step"] == "step"


def test_full_kv_bytes_per_token_7b():
    # K and V, 4 KV heads x 128 dims, bf16, 28 layers: 57,344 B per token
    w = WORKLOADS["qwen7b_decode"]
    assert bench.full_kv_bytes(w, 1) == 57_344
    assert bench.full_kv_bytes(w, 65536) == 65536 * 57_344


def test_enhancement_stats_closed_forms():
    import numpy as np
    rng = np.random.default_rng(0)
    x = rng.standard_normal((50, 64))
    # enh parallel to x with |enh| = 0.1 |x|: cos 1, share 0.1 / 1.1
    st = bench.enhancement_stats(x, 1.1 * x)
    assert abs(st["cos_median"] - 1.0) < 1e-12
    assert abs(st["share_median"] - 0.1 / 1.1) < 1e-12
    # enh orthogonal to x: cos 0, share = |e| / sqrt(|x|^2 + |e|^2)
    e = rng.standard_normal((50, 64))
    e -= (e * x).sum(1, keepdims=True) / (x * x).sum(1, keepdims=True) * x
    st = bench.enhancement_stats(x, x + e)
    assert st["abs_cos_p90"] < 1e-12
    share = np.linalg.norm(e, axis=1) / np.linalg.norm(x + e, axis=1)
    assert abs(st["share_median"] - np.median(share)) < 1e-12


def test_step_medians():
    m = bench.step_medians([1.0, 3.0, 2.0], [10.0, 30.0, 20.0])
    assert m == {"step_ms": 22.0, "prefill_ms": 2.0, "decode_ms": 20.0, "steps": 3}
    # medians are per part, so they need not add up to the step median
    m = bench.step_medians([1.0, 9.0, 2.0, 8.0], [9.0, 1.0, 8.0, 2.0])
    assert m["step_ms"] == 10.0 and m["prefill_ms"] == 5.0 and m["decode_ms"] == 5.0
