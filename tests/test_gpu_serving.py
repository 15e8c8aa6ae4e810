"""Serving variants of the boundary: per-layer calls and decode of a subset
of the batch.  The arithmetic of a stream does not depend on which other
streams share the launch, so both must equal the full calls bit for bit;
sequences left out of a decode call keep their state.  The full calls are
checked against the fp64 oracle elsewhere."""
import pytest
import torch

import kv_cache_compression_sfa_b200 as sfa
from sfa_harness import Pair, TOL, assert_close, sfa_config
from workloads import WORKLOADS, TokenSource, make_slots

pytestmark = pytest.mark.gpu


def _w(**kw):
    base = dict(name="serving", n_layers=4, batch=3)
    base.update(kw)
    return WORKLOADS["qwen05b"].replace(**base)


def _op(w, slots, decode_tile=-1):
    op = sfa.SfaOperator(sfa_config(w), slots, w.batch, device="cuda")
    sfa.sfa_debug_set_paths(op.handle, decode_tile, True)
    return op


def _state_equal(a, b):
    sa, sb = sfa.read_state(a), sfa.read_state(b)
    for key in sa:
        assert torch.equal(sa[key], sb[key]), key


@pytest.mark.parametrize("split", [[1, 1, 1, 1], [3, 1], [2, 2]])
def test_layer_range_calls_equal_the_full_calls(split):
    w = _w()
    slots = make_slots(w, "cuda")
    src = TokenSource(w, "cuda")
    q, k, v = src.get(0, 130)
    full, part = _op(w, slots), _op(w, slots)
    out_full = full.prefill(q, k, v)
    outs = []
    l0 = 0
    for lc in split:
        outs.append(part.prefill_layers(l0, q[l0:l0 + lc].contiguous(), k[l0:l0 + lc].contiguous(),
                                        v[l0:l0 + lc].contiguous()))
        l0 += lc
    assert torch.equal(out_full, torch.cat(outs, dim=0))
    for t in range(130, 135):
        qd, kd, vd = (x[:, :, 0].contiguous() for x in src.get(t, t + 1))
        d_full = full.decode(qd, kd, vd)
        d_part = []
        l0 = 0
        for lc in split:
            d_part.append(part.decode_ex(l0, qd[l0:l0 + lc].contiguous(), kd[l0:l0 + lc].contiguous(),
                                         vd[l0:l0 + lc].contiguous()))
            l0 += lc
        assert torch.equal(d_full, torch.cat(d_part, dim=0))
    assert full.check() == 0 and part.check() == 0
    _state_equal(full, part)


@pytest.mark.parametrize("decode_tile", [0, 1], ids=["per_sequence", "batch_tiled"])
def test_decode_of_a_subset_of_the_batch(decode_tile):
    w = _w(n_layers=2, batch=4)
    slots = make_slots(w, "cuda")
    src = TokenSource(w, "cuda")
    q, k, v = src.get(0, 70)
    op = _op(w, slots, decode_tile)
    op.prefill(q, k, v)
    keep = [1, 3]
    before = sfa.read_state(op)
    # reference: a batch holding only sequences 2 and 0, in that order
    sel = torch.tensor([2, 0], device="cuda")
    wr = w.replace(batch=2)
    ref = _op(wr, slots, decode_tile)
    ref.prefill(*(x.index_select(1, sel).contiguous() for x in (q, k, v)))
    ids = torch.tensor([2, 0], dtype=torch.int32, device="cuda")
    for t in range(70, 75):
        qd, kd, vd = (x[:, :, 0].index_select(1, sel).contiguous() for x in src.get(t, t + 1))
        got = op.decode_ex(0, qd, kd, vd, seq_ids=ids)
        exp = ref.decode(qd, kd, vd)
        assert torch.equal(got, exp)
    assert op.check() == 0 and ref.check() == 0
    after = sfa.read_state(op)
    sr = sfa.read_state(ref)
    for key in after:
        for b in keep:  # untouched
            assert torch.equal(after[key][:, b], before[key][:, b]), key
        assert torch.equal(after[key][:, 2], sr[key][:, 0]), key
        assert torch.equal(after[key][:, 0], sr[key][:, 1]), key
    assert int(after["pos"][0, 2]) == 75 and int(after["pos"][0, 1]) == 70


def test_subset_decode_matches_the_oracle():
    w = _w(n_layers=2, batch=2)
    pair = Pair(w)
    got, ref = pair.prefill(40)
    assert_close(got, ref, TOL[w.in_dtype], "prefill")
    # decode every sequence through decode_ex with an explicit, permuted list
    ids = torch.tensor([1, 0], dtype=torch.int32, device="cuda")
    q, k, v = pair.src.get(pair.t, pair.t + 1)
    qd, kd, vd = (x[:, :, 0].contiguous() for x in (q, k, v))
    perm = torch.tensor([1, 0], device="cuda")
    out = pair.op.decode_ex(0, *(x.index_select(1, perm).contiguous() for x in (qd, kd, vd)),
                            seq_ids=ids)
    pair.t += 1
    ref = pair._oracle(q, k, v)[:, :, 0]
    assert_close(out.index_select(1, perm).cpu().numpy(), ref, TOL[w.in_dtype], "decode_ex")
    pair.compare_state(TOL[w.in_dtype])


@pytest.mark.parametrize("decode_tile", [0, 1], ids=["per_sequence", "batch_tiled"])
def test_out_of_range_sequence_is_skipped_and_latched(decode_tile):
    w = _w(n_layers=1, batch=2)
    slots = make_slots(w, "cuda")
    src = TokenSource(w, "cuda")
    op = _op(w, slots, decode_tile)
    op.prefill(*src.get(0, 20))
    assert op.check() == 0
    before = sfa.read_state(op)
    ids = torch.tensor([5], dtype=torch.int32, device="cuda")
    qd, kd, vd = (x[:, :1, 0].contiguous() for x in src.get(20, 21))
    op.decode_ex(0, qd, kd, vd, seq_ids=ids)
    assert op.check() == sfa.SFA_ERR_INVALID_ARG
    after = sfa.read_state(op)
    for key in after:
        assert torch.equal(after[key], before[key]), key
    assert op.check() == 0  # cleared by the previous check


def test_serving_calls_reject_bad_ranges_on_the_host():
    w = _w(n_layers=2, batch=2)
    slots = make_slots(w, "cuda")
    op = _op(w, slots)
    src = TokenSource(w, "cuda")
    q, k, v = src.get(0, 8)
    with pytest.raises(sfa.SfaError):
        op.prefill_layers(1, q, k, v)  # layers 1..2 of 2
    qd, kd, vd = (x[:, :, 0].contiguous() for x in (q, k, v))
    with pytest.raises(sfa.SfaError):
        op.decode_ex(-1, qd[:1], kd[:1], vd[:1])
    assert sfa.sfa_prefill_layers_workspace_bytes(op.handle, 3, 2, 8) == 0
    assert sfa.sfa_prefill_layers_workspace_bytes(op.handle, 1, 2, 8) > 0
