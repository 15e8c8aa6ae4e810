"""GPU self-consistency: properties of the definition that hold at any size.

  * prefill(n) equals n decode steps (same recurrences, different kernels);
  * a prefill split into chunks equals one prefill;
  * n = 0 is a no-op;
  * sequences are independent: permuting the batch permutes the outputs
    bit for bit;
  * a state copied out and restored resumes exactly (checkpoint/resume);
  * the decode input-prefetch option does not change any bit.
"""
import numpy as np
import pytest
import torch

import kv_cache_compression_sfa_b200 as sfa
from sfa_harness import sfa_config
from workloads import WORKLOADS, TokenSource, make_slots

pytestmark = pytest.mark.gpu


def _w():
    return WORKLOADS["qwen05b"].replace(name="consistency", n_layers=3, batch=2)


def _op(w, slots):
    return sfa.SfaOperator(sfa_config(w), slots, w.batch, device="cuda")


def _rel(a, b):
    a, b = a.double(), b.double()
    return float(((a - b).abs() / (1 + b.abs())).max())


def test_prefill_equals_decode_steps():
    w = _w()
    slots = make_slots(w, "cuda")
    src = TokenSource(w, "cuda")
    n = 150
    q, k, v = src.get(0, n)
    a = _op(w, slots)
    out_p = a.prefill(q, k, v)
    b = _op(w, slots)
    out_d = torch.stack([b.decode(q[:, :, t].contiguous(), k[:, :, t].contiguous(),
                                  v[:, :, t].contiguous()) for t in range(n)], dim=2)
    assert a.check() == 0 and b.check() == 0
    assert _rel(out_p, out_d) < 2e-5
    sa, sb = sfa.read_state(a), sfa.read_state(b)
    for key in ("pos", "win_k", "win_v"):
        assert torch.equal(sa[key], sb[key]), key
    for key in ("far", "field", "ring", "ring_sum"):
        assert _rel(sa[key], sb[key]) < 2e-5, key


def test_decode_input_prefetch_gives_identical_results():
    """The input-prefetch option only moves the point where the decode kernel
    fetches q, k and v (before or after the previous kernel on the stream
    ends); outputs and state are bit-identical with and without it."""
    w = _w()
    slots = make_slots(w, "cuda")
    q, k, v = TokenSource(w, "cuda").get(0, 40)
    steps = [tuple(x[:, :, t].contiguous() for x in (q, k, v)) for t in range(40)]
    torch.cuda.synchronize()  # every input is complete before the calls
    runs = []
    for prefetch in (False, True):
        op = _op(w, slots)
        sfa.sfa_set_decode_input_prefetch(op.handle, prefetch)
        outs = [op.decode(*s) for s in steps]
        assert op.check() == 0
        runs.append((torch.stack(outs), op.state.clone()))
    assert torch.equal(runs[0][0], runs[1][0])
    assert torch.equal(runs[0][1], runs[1][1])


@pytest.mark.parametrize("cuts", [[64], [1, 63], [15, 16, 17], [100, 7, 43]])
def test_chunked_prefill_equals_one_prefill(cuts):
    w = _w()
    slots = make_slots(w, "cuda")
    src = TokenSource(w, "cuda")
    n = 150
    q, k, v = src.get(0, n)
    a = _op(w, slots)
    whole = a.prefill(q, k, v)
    b = _op(w, slots)
    bounds = [0] + list(np.cumsum(cuts)) + [n]  # cuts are chunk lengths
    parts = [b.prefill(q[:, :, s:e].contiguous(), k[:, :, s:e].contiguous(),
                       v[:, :, s:e].contiguous()) for s, e in zip(bounds[:-1], bounds[1:])]
    assert a.check() == 0 and b.check() == 0
    assert _rel(torch.cat(parts, dim=2), whole) < 2e-5


def test_zero_length_prefill_is_a_no_op():
    w = _w()
    op = _op(w, make_slots(w, "cuda"))
    q, k, v = TokenSource(w, "cuda").get(0, 20)
    op.prefill(q, k, v)
    before = op.state.clone()
    e = TokenSource(w, "cuda").get(0, 0)
    op.prefill(*e)
    torch.cuda.synchronize()
    assert torch.equal(before, op.state)


def test_batch_permutation_is_exact():
    w = WORKLOADS["qwen05b"].replace(name="perm", n_layers=2, batch=4)
    slots = make_slots(w, "cuda")
    q, k, v = TokenSource(w, "cuda").get(0, 90)
    perm = torch.tensor([2, 0, 3, 1], device="cuda")
    a, b = _op(w, slots), _op(w, slots)
    oa = a.prefill(q, k, v)
    ob = b.prefill(q[:, perm].contiguous(), k[:, perm].contiguous(), v[:, perm].contiguous())
    qd, kd, vd = (x[:, :, 0].contiguous() for x in TokenSource(w, "cuda", salt=1).get(0, 1))
    da = a.decode(qd, kd, vd)
    db = b.decode(qd[:, perm].contiguous(), kd[:, perm].contiguous(), vd[:, perm].contiguous())
    assert torch.equal(oa[:, perm], ob)
    assert torch.equal(da[:, perm], db)


def test_state_snapshot_resumes_exactly():
    """The state is one flat buffer: copying it out and back is a checkpoint."""
    w = _w()
    slots = make_slots(w, "cuda")
    src = TokenSource(w, "cuda")
    a = _op(w, slots)
    q, k, v = src.get(0, 70)
    a.prefill(q, k, v)
    snap = a.state.clone()
    q2, k2, v2 = src.get(70, 100)
    first = a.prefill(q2, k2, v2)
    a.state.copy_(snap)
    again = a.prefill(q2, k2, v2)
    assert torch.equal(first, again)


def test_prefill_is_deterministic_across_runs():
    """Every reduction and carry runs in a fixed order: repeated runs are
    bitwise equal, whatever the timing of the CTAs."""
    w = WORKLOADS["qwen05b"].replace(name="determinism", n_layers=2, batch=3)
    slots = make_slots(w, "cuda")
    q, k, v = TokenSource(w, "cuda").get(0, 2100)  # 33 tiles per stream, the last one ragged
    op = _op(w, slots)
    first = op.prefill(q, k, v)
    s1 = op.state.clone()
    for _ in range(3):
        op.reset()
        again = op.prefill(q, k, v)
        assert torch.equal(first, again)
        assert torch.equal(s1, op.state)
    assert op.check() == 0


def test_chunked_prefill_across_many_tiles():
    w = WORKLOADS["qwen05b"].replace(name="groups", n_layers=1, batch=2)
    slots = make_slots(w, "cuda")
    q, k, v = TokenSource(w, "cuda").get(0, 2300)
    a = _op(w, slots)
    whole = a.prefill(q, k, v)
    b = _op(w, slots)
    bounds = [0, 1030, 1031, 2200, 2300]
    parts = [b.prefill(q[:, :, s:e].contiguous(), k[:, :, s:e].contiguous(),
                       v[:, :, s:e].contiguous()) for s, e in zip(bounds[:-1], bounds[1:])]
    assert a.check() == 0 and b.check() == 0
    assert _rel(torch.cat(parts, dim=2), whole) < 2e-5
