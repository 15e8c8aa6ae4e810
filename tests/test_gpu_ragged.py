"""Ragged prefill (sfa_prefill_ragged): in one call every sequence folds in
its own number of tokens from its own position.  Checked against the fp64
oracle stream by stream (each (layer, sequence) stream has its own oracle
state, advanced by its own count), together with the rows a call must leave
alone and a count outside 0 .. n_max, which is latched and changes nothing.

Tolerance per element: |gpu - oracle| <= tol * (1 + |oracle|), tol = 1e-4
for fp32 inputs and 2e-3 for bf16 inputs; window slots and positions exact.
"""
import numpy as np
import pytest
import torch

import kv_cache_compression_sfa_b200 as sfa
import oracle
from sfa_harness import TOL, assert_close, np32, oracle_alpha, oracle_params, sfa_config
from workloads import WORKLOADS, make_slots

pytestmark = pytest.mark.gpu


def _w(**kw):
    return WORKLOADS["tiny"].replace(**kw)


class Ragged:
    """One operator on the GPU and one oracle state per (layer, sequence)."""

    def __init__(self, w, seed=0, prefill_near=3):
        self.w = w
        self.dev = torch.device("cuda")
        slots = make_slots(w, "cpu")
        self.slots_np = np32(slots)
        self.op = sfa.SfaOperator(sfa_config(w), slots.to(self.dev), w.batch, device=self.dev)
        sfa.sfa_debug_set_paths(self.op.handle, -1, prefill_near)
        self.p = oracle_params(w)
        self.ost = [[oracle.OracleState(self.p, 1) for _ in range(w.batch)]
                    for _ in range(w.n_layers)]
        self.g = torch.Generator().manual_seed(seed)

    def _draw(self, shape_tokens):
        w = self.w
        mk = lambda heads: torch.randn((w.n_layers, w.batch, *shape_tokens, heads, w.head_dim),
                                       generator=self.g).to(w.torch_dtype)
        return mk(w.n_q_heads), mk(w.n_kv_heads), mk(w.n_kv_heads)

    def _oracle(self, l, b, q, k, v):
        ref, _ = oracle.run_streams(self.p, [oracle_alpha(self.w, l)], self.slots_np[l][None],
                                    np32(q)[None], np32(k)[None], np32(v)[None], self.ost[l][b])
        return ref[0]

    def prefill(self, lens, n_max=None):
        w = self.w
        n_max = max(max(lens), 1) if n_max is None else n_max
        q, k, v = self._draw((n_max,))
        lens_d = torch.tensor(lens, dtype=torch.int32, device=self.dev)
        out = self.op.prefill_ragged(q.to(self.dev), k.to(self.dev), v.to(self.dev), lens_d)
        got = out.cpu().numpy()
        tol = TOL[w.in_dtype]
        for l in range(w.n_layers):
            for b in range(w.batch):
                n = lens[b]
                if n < 0 or n > n_max:  # a bad count: nothing written
                    assert np.isnan(got[l, b]).all(), f"layer {l} seq {b}: bad count wrote rows"
                    continue
                assert np.isnan(got[l, b, n:]).all(), f"layer {l} seq {b}: rows past {n} written"
                if n == 0:
                    continue
                ref = self._oracle(l, b, q[l, b, :n], k[l, b, :n], v[l, b, :n])
                assert_close(got[l, b, :n], ref, tol, f"ragged prefill layer {l} seq {b} ({n} tokens)")

    def decode(self):
        w = self.w
        q, k, v = (x[:, :, 0] for x in self._draw((1,)))
        got = self.op.decode(q.contiguous().to(self.dev), k.contiguous().to(self.dev),
                             v.contiguous().to(self.dev)).cpu().numpy()
        for l in range(w.n_layers):
            for b in range(w.batch):
                ref = self._oracle(l, b, q[l, b][None], k[l, b][None], v[l, b][None])
                assert_close(got[l, b][None], ref, TOL[w.in_dtype], f"decode layer {l} seq {b}")

    def compare_state(self):
        st = sfa.read_state(self.op)
        tol = TOL[self.w.in_dtype]
        for l in range(self.w.n_layers):
            for b in range(self.w.batch):
                o = self.ost[l][b]
                assert int(st["pos"][l, b]) == int(o.pos[0]), (l, b)
                np.testing.assert_array_equal(np32(st["win_k"][l, b]).astype(np.float64), o.win_k[0])
                np.testing.assert_array_equal(np32(st["win_v"][l, b]).astype(np.float64), o.win_v[0])
                assert_close(np32(st["far"][l, b]), o.S[0], tol, f"S {l} {b}")
                assert_close(np32(st["field"][l, b]), o.field[0], tol, f"field {l} {b}")
                assert_close(np32(st["ring"][l, b]), o.ring[0], tol, f"ring {l} {b}")
                assert_close(np32(st["ring_sum"][l, b]), o.ring[0].sum(axis=0), tol, f"ring_sum {l} {b}")


CASES = [
    # bf16 with k <= 16: the tensor-core near field; counts of 0, 1, a tile
    # boundary and past it, two tiles and more
    ("bf16_k12", dict(name="ragged_bf16", n_layers=2, batch=6, n_q_heads=4, n_kv_heads=2,
                      head_dim=64, window_k=12, in_dtype="bf16"),
     [[0, 1, 15, 64, 65, 130], [5, 0, 70, 1, 64, 3]]),
    # fp32, window wider than a decode chunk: the CUDA-core near field
    ("f32_k20_d128", dict(name="ragged_f32", n_layers=1, batch=4, n_q_heads=4, n_kv_heads=1,
                          head_dim=128, window_k=20, in_dtype="f32"),
     [[3, 0, 129, 64], [17, 1, 0, 66]]),
    # seven query heads per KV head (the Qwen2.5-0.5B grouping)
    ("gqa7_bf16", dict(name="ragged_gqa7", n_layers=2, batch=3, n_q_heads=14, n_kv_heads=2,
                       head_dim=64, window_k=16, in_dtype="bf16"),
     [[100, 0, 33], [1, 64, 0]]),
]


@pytest.mark.parametrize("mode", [3, 2], ids=["default", "fused"])
@pytest.mark.parametrize("name,over,calls", CASES, ids=[c[0] for c in CASES])
def test_ragged_prefill_matches_the_oracle(name, over, calls, mode):
    """mode: the prefill near-field path (sfa_debug_set_paths); 2 pins the
    fused kernel, which these small calls would not take by default (fp32
    inputs keep the CUDA cores either way)."""
    r = Ragged(_w(**over), prefill_near=mode)
    r.prefill(calls[0])
    r.decode()  # every sequence one token on, from different positions
    r.prefill(calls[1])
    assert r.op.check() == 0
    r.compare_state()


def test_ragged_prefill_with_equal_counts_equals_prefill():
    """All counts equal to n: bit-identical to sfa_prefill."""
    w = _w(name="ragged_equal", n_layers=2, batch=3, n_q_heads=4, n_kv_heads=2, head_dim=64,
           window_k=16, in_dtype="bf16")
    g = torch.Generator().manual_seed(3)
    mk = lambda h: torch.randn((2, 3, 77, h, 64), generator=g).to(torch.bfloat16).cuda()
    q, k, v = mk(4), mk(2), mk(2)
    slots = make_slots(w, "cuda")
    a = sfa.SfaOperator(sfa_config(w), slots, 3, device="cuda")
    b = sfa.SfaOperator(sfa_config(w), slots, 3, device="cuda")
    out_a = a.prefill(q, k, v)
    out_b = b.prefill_ragged(q, k, v, torch.full((3,), 77, dtype=torch.int32, device="cuda"))
    assert torch.equal(out_a, out_b)
    sa, sb = sfa.read_state(a), sfa.read_state(b)
    for key in sa:
        assert torch.equal(sa[key], sb[key]), key


def test_ragged_prefill_latches_a_bad_count():
    """A count outside 0 .. n_max: latched as SFA_ERR_INVALID_ARG, that
    sequence's state and output untouched, the others served."""
    w = _w(name="ragged_bad", n_layers=1, batch=4, n_q_heads=4, n_kv_heads=2, head_dim=64,
           window_k=8, in_dtype="bf16")
    r = Ragged(w)
    r.prefill([3, 10, 2, 7])
    assert r.op.check() == 0
    before = sfa.read_state(r.op)
    r.prefill([2, -1, 12, 5], n_max=10)  # -1 and 12 (> n_max) are bad
    assert r.op.check() == sfa.SFA_ERR_INVALID_ARG
    after = sfa.read_state(r.op)
    for key in after:
        for b in (1, 2):
            assert torch.equal(after[key][:, b], before[key][:, b]), (key, b)
    assert r.op.check() == 0
    r.compare_state()
