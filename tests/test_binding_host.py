"""Argument marshalling of the Python binding, on CPU.

The C library is replaced by a recorder and the CUDA-tensor test by a plain
tensor test, so the binding's own logic (sizes, dtypes, contiguity, the
order of the C arguments) runs without a GPU.  SfaOperator.decode, the
per-token call of a serving loop, must pass exactly what the module-level
sfa_decode_step passes.
"""
import pytest
import torch

import kv_cache_compression_sfa_b200 as sfa


class _Recorder:
    """The C entry points the operator touches, recording their arguments."""

    def __init__(self, state_bytes):
        self.state_bytes = state_bytes
        self.calls = []

    def sfa_state_bytes(self, h, batch):
        return self.state_bytes

    def sfa_decode_step(self, *args):
        self.calls.append(("sfa_decode_step", args))
        return 0

    def sfa_destroy(self, h):
        return 0


@pytest.fixture
def fake(monkeypatch):
    rec = _Recorder(state_bytes=4096)
    handles = []

    def fake_init(cfg, slots):
        handles.append(sfa.Handle(0xABC, cfg))
        return handles[-1]

    monkeypatch.setattr(sfa, "_lib", rec)
    monkeypatch.setattr(sfa, "_is_cuda_tensor", lambda t: isinstance(t, torch.Tensor))
    monkeypatch.setattr(sfa, "_stream_ptr", lambda stream: 0x5151)
    monkeypatch.setattr(sfa, "sfa_init", fake_init)
    monkeypatch.setattr(sfa, "sfa_state_reset", lambda h, state, batch, stream=None: None)
    yield rec
    # The fake handles must never reach the real library (which would read
    # through their pointer): drop the pointers before the patches are undone.
    for h in handles:
        h.ptr = None


def _op(batch=3):
    cfg = sfa.SfaConfig(n_layers=2, n_q_heads=4, n_kv_heads=2, head_dim=64)
    slots = torch.zeros(2, 64, cfg.hidden)
    return sfa.SfaOperator(cfg, slots, batch, device="cpu"), cfg


def _inputs(cfg, batch, dtype=torch.bfloat16):
    q = torch.randn(cfg.n_layers, batch, cfg.n_q_heads, cfg.head_dim).to(dtype)
    k = torch.randn(cfg.n_layers, batch, cfg.n_kv_heads, cfg.head_dim).to(dtype)
    v = torch.randn(cfg.n_layers, batch, cfg.n_kv_heads, cfg.head_dim).to(dtype)
    out = torch.empty(cfg.n_layers, batch, cfg.hidden)
    return q, k, v, out


def test_operator_decode_passes_what_the_module_call_passes(fake):
    op, cfg = _op()
    q, k, v, out = _inputs(cfg, 3)
    assert op.decode(q, k, v, out=out) is out
    sfa.sfa_decode_step(op.handle, q, k, v, 3, op.state, out)
    (n0, a0), (n1, a1) = fake.calls
    assert n0 == n1 == "sfa_decode_step"
    assert a0 == a1 == (0xABC, q.data_ptr(), k.data_ptr(), v.data_ptr(), 3, op.state.data_ptr(),
                        out.data_ptr(), 0x5151)


def test_operator_decode_reads_the_current_state_tensor(fake):
    op, cfg = _op()
    q, k, v, out = _inputs(cfg, 3)
    op.state = torch.empty(4096, dtype=torch.uint8)  # a state swapped in after init
    op.decode(q, k, v, out=out)
    assert fake.calls[-1][1][5] == op.state.data_ptr()


@pytest.mark.parametrize("bad", ["q_dtype", "k_short", "v_strided", "out_dtype", "state_short"])
def test_operator_decode_rejects_bad_tensors_before_the_call(fake, bad):
    op, cfg = _op()
    q, k, v, out = _inputs(cfg, 3)
    if bad == "q_dtype":
        q = q.float()
    elif bad == "k_short":
        k = k[:, :2]
    elif bad == "v_strided":
        v = v.transpose(2, 3)
    elif bad == "out_dtype":
        out = out.double()
    elif bad == "state_short":
        op.state = torch.empty(100, dtype=torch.uint8)
    with pytest.raises(ValueError):
        op.decode(q, k, v, out=out)
    assert fake.calls == []


def test_operator_decode_allocates_out_when_none_is_given(fake):
    op, cfg = _op(batch=1)
    q, k, v, _ = _inputs(cfg, 1)
    out = op.decode(q, k, v)
    assert out.shape == (2, 1, cfg.hidden) and out.dtype == torch.float32
    assert fake.calls[-1][1][6] == out.data_ptr()
