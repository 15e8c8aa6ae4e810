"""Output modes (sfa_set_output_mode) against the fp64 oracle.

The pages add the enhancement to the attention output ([P3] §2.2 output =
attention_output + enhancement; [P2] llama.cpp bridge
compute_enhancement(layer, attn_output)).  The oracle gives out = x + enh; a
second oracle run with alpha_base = 0 gives x itself (the state never
depends on alpha_base), so enh = out - x.  Checked per element:

  * SFA_OUT_BF16:      out = x + enh rounded to bf16;
  * SFA_OUT_ADD_F32:   out = y + enh for the caller's fp32 y already in out;
  * SFA_OUT_ADD_BF16:  out = y + enh rounded to bf16, y bf16.

Bound: |gpu - ref| <= tol * (1 + |ref|), tol = 1e-4 (fp32 inputs) or 2e-3
(bf16 inputs), plus one bf16 unit in the last place, 2^-8 * |ref|, where the
result is rounded to bf16 (the final rounding of a value already within the
tolerance).  The state must match as in every parity test.
"""
import numpy as np
import pytest
import torch

import kv_cache_compression_sfa_b200 as sfa
import oracle
from sfa_harness import TOL, np32, oracle_alpha, oracle_params, sfa_config, violation
from workloads import WORKLOADS, make_slots

pytestmark = pytest.mark.gpu


def _check(got, ref, tol, bf16_out, what):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    bound = tol * (1.0 + np.abs(ref)) + (2.0 ** -8) * np.abs(ref) * bf16_out
    err = np.abs(got - ref)
    bad = int((err > bound).sum())
    if bad:
        i = np.unravel_index(np.argmax(err / bound), err.shape)
        raise AssertionError(f"{what}: {bad} of {err.size} outside the bound; worst at {i}: "
                             f"gpu {got[i]!r} ref {ref[i]!r}")


class Modes:
    def __init__(self, w, mode, seed=7, prefill_near=3):
        self.w, self.mode = w, mode
        self.dev = torch.device("cuda")
        slots = make_slots(w, "cpu")
        self.slots_np = np32(slots)
        self.op = sfa.SfaOperator(sfa_config(w), slots.to(self.dev), w.batch, device=self.dev)
        sfa.sfa_debug_set_paths(self.op.handle, -1, prefill_near)
        self.op.set_output_mode(mode)
        self.p = oracle_params(w)
        S = w.n_layers * w.batch
        self.ost, self.ost0 = oracle.OracleState(self.p, S), oracle.OracleState(self.p, S)
        self.g = torch.Generator().manual_seed(seed)
        self.bf16_out = mode in (sfa.SFA_OUT_BF16, sfa.SFA_OUT_ADD_BF16)
        self.add = mode in (sfa.SFA_OUT_ADD_F32, sfa.SFA_OUT_ADD_BF16)

    def _draw(self, n):
        w = self.w
        mk = lambda h: torch.randn((w.n_layers, w.batch, n, h, w.head_dim), generator=self.g).to(w.torch_dtype)
        return mk(w.n_q_heads), mk(w.n_kv_heads), mk(w.n_kv_heads)

    def _refs(self, q, k, v):
        w = self.w
        S, n = w.n_layers * w.batch, q.shape[2]
        alpha = [oracle_alpha(w, l) for l in range(w.n_layers) for _ in range(w.batch)]
        sl = np.stack([self.slots_np[l] for l in range(w.n_layers) for _ in range(w.batch)])
        qq = np32(q).reshape(S, n, *q.shape[3:])
        kk = np32(k).reshape(S, n, *k.shape[3:])
        vv = np32(v).reshape(S, n, *v.shape[3:])
        out, _ = oracle.run_streams(self.p, alpha, sl, qq, kk, vv, self.ost)
        x, _ = oracle.run_streams(self.p, [0.0] * S, sl, qq, kk, vv, self.ost0)
        shape = (w.n_layers, w.batch, n, self.p.hidden)
        return out.reshape(shape), x.reshape(shape)

    def _y(self, shape):
        y = torch.randn(shape, generator=self.g)
        return y.to(torch.bfloat16) if self.bf16_out else y

    def step(self, n):
        """A prefill of n tokens (n > 0) or a decode step (n == 0)."""
        w = self.w
        q, k, v = self._draw(max(n, 1))
        out_shape = (w.n_layers, w.batch, max(n, 1), w.hidden)
        y = self._y(out_shape) if self.add else None
        dq, dk, dv = (x.to(self.dev) for x in (q, k, v))
        if n > 0:
            out = y.to(self.dev) if self.add else None
            got = self.op.prefill(dq, dk, dv, out=out)
        else:
            out = y[:, :, 0].contiguous().to(self.dev) if self.add else None
            got = self.op.decode(dq[:, :, 0].contiguous(), dk[:, :, 0].contiguous(),
                                 dv[:, :, 0].contiguous(), out=out)[:, :, None]
        assert got.dtype == (torch.bfloat16 if self.bf16_out else torch.float32)
        ref_out, ref_x = self._refs(q, k, v)
        ref = (np32(y).astype(np.float64) + (ref_out - ref_x)) if self.add else ref_out
        _check(np32(got), ref, TOL[w.in_dtype], self.bf16_out, f"mode {self.mode} n={n}")

    def compare_state(self):
        st = sfa.read_state(self.op)
        w, o = self.w, self.ost
        tol = TOL[w.in_dtype]
        shape = (w.n_layers, w.batch)
        np.testing.assert_array_equal(st["pos"].numpy(), o.pos.reshape(shape))
        worst, bad = violation(np32(st["field"]), o.field.reshape(*shape, -1), tol)
        assert bad == 0, worst
        worst, bad = violation(np32(st["far"]), o.S.reshape(*shape, *o.S.shape[1:]), tol)
        assert bad == 0, worst


MODES = [sfa.SFA_OUT_BF16, sfa.SFA_OUT_ADD_F32, sfa.SFA_OUT_ADD_BF16]
CONFIGS = [
    # bf16 inputs, k <= 16: tensor-core prefill near field; 3 sequences
    ("bf16_b3", dict(name="modes_bf16", n_layers=2, batch=3, n_q_heads=14, n_kv_heads=2,
                     head_dim=64, window_k=16, in_dtype="bf16")),
    # 70 sequences: decode calls of this size take the per-sequence kernel in
    # these modes
    ("bf16_b70", dict(name="modes_b70", n_layers=1, batch=70, n_q_heads=4, n_kv_heads=2,
                      head_dim=64, window_k=8, in_dtype="bf16")),
    ("f32_d128", dict(name="modes_f32", n_layers=2, batch=2, n_q_heads=4, n_kv_heads=2,
                      head_dim=128, window_k=20, in_dtype="f32")),
]


@pytest.mark.parametrize("mode", MODES, ids=["bf16", "add_f32", "add_bf16"])
@pytest.mark.parametrize("name,over", CONFIGS, ids=[c[0] for c in CONFIGS])
def test_output_mode_matches_the_oracle(name, over, mode):
    m = Modes(WORKLOADS["tiny"].replace(**over), mode)
    for n in (70, 0, 0, 0, 20):
        m.step(n)
    assert m.op.check() == 0
    m.compare_state()


@pytest.mark.parametrize("mode", MODES, ids=["bf16", "add_f32", "add_bf16"])
def test_output_mode_with_the_fused_prefill(mode):
    """The fused prefill kernel (pinned; these calls are small) keeps x in the
    workspace for the output kernel in every mode."""
    m = Modes(WORKLOADS["tiny"].replace(**CONFIGS[0][1]), mode, prefill_near=2)
    for n in (70, 0, 20):
        m.step(n)
    assert m.op.check() == 0
    m.compare_state()


def test_output_mode_workspace_and_argument_checks():
    w = WORKLOADS["tiny"].replace(name="modes_ws", n_layers=2, batch=2, n_q_heads=4, n_kv_heads=2,
                                  head_dim=64, window_k=16, in_dtype="bf16")
    op = sfa.SfaOperator(sfa_config(w), make_slots(w, "cuda"), 2, device="cuda")
    base = sfa.sfa_prefill_workspace_bytes(op.handle, 2, 100)
    op.set_output_mode(sfa.SFA_OUT_BF16)
    # x between the prefill kernels moves into the workspace
    assert sfa.sfa_prefill_workspace_bytes(op.handle, 2, 100) >= base + 2 * 2 * 100 * w.hidden * 4
    with pytest.raises(sfa.SfaError):
        op.set_output_mode(4)
    op.set_output_mode(sfa.SFA_OUT_ADD_F32)
    q = torch.zeros((2, 2, 5, 4, 64), dtype=torch.bfloat16, device="cuda")
    kv = torch.zeros((2, 2, 5, 2, 64), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ValueError):
        op.prefill(q, kv, kv)  # the add modes need the caller's attention output
    with pytest.raises(ValueError):  # fp32 out expected
        op.prefill(q, kv, kv, out=torch.zeros((2, 2, 5, w.hidden), dtype=torch.bfloat16, device="cuda"))
