"""sfa_prefill_static_ws: prefill for callers that cannot allocate.

Such callers (an operator hook inside another engine that only receives its
input/output tensors, a serving loop that forbids cudaMalloc in steady state)
get the prefill's scratch from a fixed device array inside the library.  This
test calls that entry point through the C ABI twice in a row and checks both
calls against sfa_prefill with a caller-provided workspace, on its own state.
It must pass when run alone in a fresh process and after the other tests;
the file name makes pytest collect it last.
"""
import ctypes

import pytest
import torch

import kv_cache_compression_sfa_b200 as sfa
from sfa_harness import sfa_config
from workloads import WORKLOADS, TokenSource, make_slots

pytestmark = pytest.mark.gpu


def test_static_workspace_prefill_matches_the_workspace_entry_point_on_two_calls():
    w = WORKLOADS["qwen05b"]  # 24 layers, hidden 896, bf16
    slots = make_slots(w, "cuda")
    ref = sfa.SfaOperator(sfa_config(w), slots, w.batch, max_prefill=512, device="cuda")
    sut = sfa.SfaOperator(sfa_config(w), slots, w.batch, device="cuda")
    lib = sfa.load_library()
    src = TokenSource(w, "cuda")
    stream = torch.cuda.current_stream().cuda_stream
    t = 0
    for n in (512, 200):  # two calls in a row; the second continues the state
        q, k, v = src.get(t, t + n)
        t += n
        want = ref.prefill(q, k, v)
        got = torch.full_like(want, float("nan"))
        rc = lib.sfa_prefill_static_ws(sut.handle.ptr, q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                       n, w.batch, sut.state.data_ptr(), got.data_ptr(), stream)
        assert rc == sfa.SFA_OK, sfa.sfa_status_string(rc)
        torch.cuda.synchronize()
        assert sut.check() == 0 and ref.check() == 0
        # the same kernels on the same inputs: identical bits
        assert torch.equal(got, want), float((got - want).abs().max())
    s_sut, s_ref = sfa.read_state(sut), sfa.read_state(ref)
    for key in s_ref:
        assert torch.equal(s_sut[key], s_ref[key]), key


def test_static_workspace_rejects_a_call_larger_than_the_array():
    w = WORKLOADS["qwen05b"]
    slots = make_slots(w, "cuda")
    op = sfa.SfaOperator(sfa_config(w), slots, w.batch, device="cuda")
    n = 4096  # needs ~25 MB of scratch
    assert sfa.sfa_prefill_workspace_bytes(op.handle, w.batch, n) > sfa.SFA_STATIC_WORKSPACE_BYTES
    q, k, v = TokenSource(w, "cuda").get(0, 1)  # never read: the call is refused first
    out = torch.empty(1, device="cuda")
    lib = sfa.load_library()
    rc = lib.sfa_prefill_static_ws(op.handle.ptr, q.data_ptr(), k.data_ptr(), v.data_ptr(), n,
                                   w.batch, op.state.data_ptr(), out.data_ptr(),
                                   torch.cuda.current_stream().cuda_stream)
    assert rc == sfa.SFA_ERR_WORKSPACE


def test_static_workspace_checks_the_handle_like_sfa_prefill():
    """A bad handle is refused with the status sfa_prefill gives, n == 0 too."""
    lib = sfa.load_library()
    for n in (0, 16):
        assert lib.sfa_prefill_static_ws(None, None, None, None, n, 1, None, None, None) == \
            sfa.SFA_ERR_INVALID_ARG
        assert lib.sfa_prefill(None, None, None, None, n, 1, None, None, None, 0, None) == \
            sfa.SFA_ERR_INVALID_ARG
