"""Failure handling without faulting the GPU.

Host-side checks reject bad calls before any launch.  On the device, a state
built for another configuration is detected from its header and latched;
the prefill's waits are bounded, and a test hook makes one CTA wait on a
barrier that nothing completes so that its wait runs out: the kernel still
finishes, latches SFA_ERR_DEVICE_TIMEOUT, and the context stays usable.
"""
import ctypes

import pytest
import torch

import kv_cache_compression_sfa_b200 as sfa
from sfa_harness import sfa_config
from workloads import WORKLOADS, TokenSource, make_slots

pytestmark = pytest.mark.gpu


def _w(**kw):
    return WORKLOADS["qwen05b"].replace(name="faults", n_layers=2, batch=2, **kw)


def test_host_rejects_bad_arguments_without_launching():
    w = _w()
    op = sfa.SfaOperator(sfa_config(w), make_slots(w, "cuda"), w.batch, max_prefill=64)
    lib = sfa.load_library()
    q, k, v = TokenSource(w, "cuda").get(0, 8)
    out = torch.empty((2, 2, 8, w.hidden), device="cuda")
    h, st, ws = op.handle.ptr, op.state.data_ptr(), op.workspace.data_ptr()
    nbytes = op.workspace.numel()
    s = torch.cuda.current_stream().cuda_stream
    before = op.state.clone()
    args = [h, q.data_ptr(), k.data_ptr(), v.data_ptr(), 8, 2, st, out.data_ptr(), ws, nbytes, s]
    assert lib.sfa_prefill(*args) == 0
    torch.cuda.synchronize()
    before = op.state.clone()
    bad = list(args); bad[1] = None
    assert lib.sfa_prefill(*bad) == sfa.SFA_ERR_INVALID_ARG
    bad = list(args); bad[1] = q.data_ptr() + 4
    assert lib.sfa_prefill(*bad) == sfa.SFA_ERR_ALIGNMENT
    bad = list(args); bad[4] = -1
    assert lib.sfa_prefill(*bad) == sfa.SFA_ERR_INVALID_ARG
    bad = list(args); bad[9] = 16
    assert lib.sfa_prefill(*bad) == sfa.SFA_ERR_WORKSPACE
    bad = list(args); bad[0] = None
    assert lib.sfa_prefill(*bad) == sfa.SFA_ERR_INVALID_ARG
    # beyond the call limits: 2 layers x 40000 sequences > 65535 streams, and
    # n > 64 x (2^31 - 1) tokens; no workspace size, refused before any launch
    for n, b in [(8, 40000), (1 << 40, 2)]:
        assert lib.sfa_prefill_workspace_bytes(h, b, n) == 0
        bad = list(args); bad[4] = n; bad[5] = b
        assert lib.sfa_prefill(*bad) == sfa.SFA_ERR_UNSUPPORTED
        assert lib.sfa_prefill_static_ws(h, *args[1:4], n, b, st, out.data_ptr(), s) == \
            sfa.SFA_ERR_UNSUPPORTED
    assert lib.sfa_decode_step(h, q.data_ptr() + 2, k.data_ptr(), v.data_ptr(), 2, st,
                               out.data_ptr(), s) == sfa.SFA_ERR_ALIGNMENT
    torch.cuda.synchronize()
    assert torch.equal(before, op.state)
    assert op.check() == 0


def test_init_rejects_unsupported_config():
    w = _w()
    cfg = sfa_config(w)
    cfg.head_dim = 96
    with pytest.raises(sfa.SfaError) as e:
        sfa.sfa_init(cfg, torch.zeros(2 * 64 * cfg.hidden, device="cuda"))
    assert e.value.code == sfa.SFA_ERR_UNSUPPORTED


def test_state_of_another_config_is_detected_on_the_device():
    w = _w()
    slots = make_slots(w, "cuda")
    a = sfa.SfaOperator(sfa_config(w), slots, w.batch, max_prefill=64)
    other = sfa_config(w)
    other.alpha_base = 0.5
    b = sfa.SfaOperator(other, slots, w.batch, max_prefill=64)
    b.state = a.state  # a's state, b's handle: header hash differs
    before = a.state.clone()
    q, k, v = TokenSource(w, "cuda").get(0, 5)
    out = torch.full((2, 2, 5, w.hidden), 7.0, device="cuda")
    b.prefill(q, k, v, out=out)
    assert b.check() == sfa.SFA_ERR_STATE_MISMATCH
    qd, kd, vd = (x[:, :, 0].contiguous() for x in (q, k, v))
    out1 = torch.full((2, 2, w.hidden), 7.0, device="cuda")
    b.decode(qd, kd, vd, out=out1)
    assert b.check() == sfa.SFA_ERR_STATE_MISMATCH
    assert torch.equal(before, a.state)
    assert bool((out == 7.0).all()) and bool((out1 == 7.0).all())
    assert b.check() == 0  # the latch was cleared by the previous check
    a.prefill(q, k, v)
    assert a.check() == 0


def test_bounded_wait_runs_out_and_the_context_survives():
    w = _w()
    op = sfa.SfaOperator(sfa_config(w), make_slots(w, "cuda"), w.batch, max_prefill=256)
    n_streams = w.n_layers * w.batch
    # tile 1 of stream 0: index = tile * n_streams + stream
    sfa.sfa_debug_set_wait_limit(op.handle, spin_limit=2000, withhold_tile=1 * n_streams + 0)
    q, k, v = TokenSource(w, "cuda").get(0, 256)
    op.prefill(q, k, v)
    assert op.check() == sfa.SFA_ERR_DEVICE_TIMEOUT
    # back to normal: the same call on a fresh state succeeds and matches a
    # fresh operator
    sfa.sfa_debug_set_wait_limit(op.handle, 0, -1)
    op.reset()
    got = op.prefill(q, k, v)
    assert op.check() == 0
    ref_op = sfa.SfaOperator(sfa_config(w), make_slots(w, "cuda"), w.batch, max_prefill=256)
    ref = ref_op.prefill(q, k, v)
    assert torch.equal(got, ref)
