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


class _FakeEvent:
    def __init__(self, enable_timing=False):
        pass

    def record(self, stream=None):
        pass

    def elapsed_time(self, other):
        return 2.0


class _FakeStream:
    def __init__(self, device=None):
        pass

    def wait_event(self, e):
        pass

    def wait_stream(self, s):
        pass


class _RecordingOp:
    """Stands in for SfaOperator: records what every call received."""

    def __init__(self):
        self.calls = []

    def reset(self, stream=None):
        self.calls.append(("reset",))

    def prefill(self, q, k, v, out=None, stream=None):
        self.calls.append(("prefill", q.clone(), k.clone(), v.clone(), out))
        out.fill_(1.0)
        return out

    def decode(self, q, k, v, out=None, stream=None):
        self.calls.append(("decode", q.clone(), k.clone(), v.clone(), out))
        out.fill_(2.0)
        return out


def _fake_cuda(monkeypatch):
    import contextlib
    import torch
    monkeypatch.setattr(torch.cuda, "Event", _FakeEvent)
    monkeypatch.setattr(torch.cuda, "Stream", _FakeStream)
    monkeypatch.setattr(torch.cuda, "current_stream", lambda device=None: _FakeStream())
    monkeypatch.setattr(torch.cuda, "stream", lambda s: contextlib.nullcontext())
    monkeypatch.setattr(torch.cuda, "synchronize", lambda device=None: None)
    monkeypatch.setattr(torch.Tensor, "pin_memory", lambda self: self)


@pytest.mark.parametrize("n_dec", [0, 3])
def test_e2e_step_loop_feeds_every_call_its_own_inputs(monkeypatch, n_dec):
    """measure_e2e on CPU with fake streams and events: each step resets,
    prefills with that step's inputs and runs every decode call on its own
    token's q/k/v and output slice, alternating the two buffer sets."""
    import types
    import torch
    _fake_cuda(monkeypatch)
    w = types.SimpleNamespace(n_layers=2, batch=1, hidden=8)
    g = torch.Generator().manual_seed(0)
    mk = lambda *s: torch.randn(*s, generator=g).to(torch.bfloat16)
    n_pre = 5
    qp, kp, vp = mk(2, 1, n_pre, 2, 4), mk(2, 1, n_pre, 1, 4), mk(2, 1, n_pre, 1, 4)
    qd = [mk(2, 1, 2, 4) for _ in range(n_dec)]
    kd = [mk(2, 1, 1, 4) for _ in range(n_dec)]
    vd = [mk(2, 1, 1, 4) for _ in range(n_dec)]
    op = _RecordingOp()
    args = types.SimpleNamespace(steps=4)
    e2e = bench.measure_e2e(args, w, op, qp, kp, vp, qd, kd, vd, n_pre, n_dec, 1, "cpu")
    steps = 3 + max(3, min(args.steps, 200)) + 1  # run(3), the timed run, the host-cost run(1)
    per_step = 2 + n_dec
    assert len(op.calls) == steps * per_step
    outs = set()
    for s in range(steps):
        c = op.calls[s * per_step:(s + 1) * per_step]
        assert c[0] == ("reset",)
        assert c[1][0] == "prefill" and all(torch.equal(a, b) for a, b in zip(c[1][1:4], (qp, kp, vp)))
        for t in range(n_dec):
            name, q, k, v, out = c[2 + t]
            assert name == "decode"
            assert torch.equal(q, qd[t]) and torch.equal(k, kd[t]) and torch.equal(v, vd[t])
            assert out.shape == (2, 1, 8) and out.is_contiguous()
            outs.add(out.data_ptr())
    assert len(outs) == 2 * n_dec  # one output slice per token and buffer set
    dec_elems = sum(x.numel() for x in qd + kd + vd)
    assert e2e["h2d_bytes_per_step"] == 2 * (qp.numel() + kp.numel() + vp.numel() + dec_elems)
    assert e2e["d2h_bytes_per_step"] == 4 * 2 * 8 * (n_pre + n_dec)
    assert e2e["value"] == pytest.approx(1 * (n_pre + n_dec) * 4 / 2e-3)
    assert e2e["ms_per_step"] == pytest.approx(2.0 / 4) and e2e["host_issue_ms_per_step"] > 0


def test_e2e_decode_only_loop_copies_each_token(monkeypatch):
    """measure_e2e_decode on CPU with fake streams and events: every call
    copies in its token's inputs (cycling the input ring) and decodes them."""
    import types
    import torch
    _fake_cuda(monkeypatch)
    w = types.SimpleNamespace(n_layers=2, batch=3, hidden=8)
    g = torch.Generator().manual_seed(1)
    mk = lambda *s: torch.randn(*s, generator=g).to(torch.bfloat16)
    n_ring, n_dec = 2, 5
    qd = [mk(2, 3, 2, 4) for _ in range(n_ring)]
    kd = [mk(2, 3, 1, 4) for _ in range(n_ring)]
    vd = [mk(2, 3, 1, 4) for _ in range(n_ring)]
    op = _RecordingOp()
    args = types.SimpleNamespace(steps=3)
    e2e = bench.measure_e2e_decode(args, w, op, qd, kd, vd, n_dec, 1, "cpu")
    runs = 3 + 3  # three untimed, then max(3, min(steps, 5)) timed
    assert len(op.calls) == runs * n_dec
    for i, c in enumerate(op.calls):
        r = (i % n_dec) % n_ring
        assert c[0] == "decode" and torch.equal(c[1], qd[r]) and torch.equal(c[3], vd[r])
    assert e2e["h2d_bytes_per_step"] == n_dec * 2 * (qd[0].numel() + kd[0].numel() + vd[0].numel())
    assert e2e["d2h_bytes_per_step"] == n_dec * 2 * 3 * 8 * 4
    assert e2e["value"] == pytest.approx(3 * n_dec * 3 / 2e-3)


def test_nvtx_range_wraps_and_reraises():
    with bench.nvtx_range("test range"):
        pass
    with pytest.raises(KeyError):
        with bench.nvtx_range("test range"):
            raise KeyError("inside")
