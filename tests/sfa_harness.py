"""Test helpers: run the CUDA library and the fp64 oracle on the same seeded
inputs and compare them element by element.

Tolerance (per element): |gpu - oracle| <= tol * (1 + |oracle|), with
tol = 1e-4 for fp32 inputs and 2e-3 for bf16 inputs.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, List, Optional, Sequence, Tuple

import numpy as np
import torch

import kv_cache_compression_sfa_b200 as sfa
import oracle
from workloads import TokenSource, Workload, make_slots

TOL = {"f32": 1e-4, "bf16": 2e-3}


def sfa_config(w: Workload) -> sfa.SfaConfig:
    v = w.values
    return sfa.SfaConfig(
        n_layers=w.n_layers, n_q_heads=w.n_q_heads, n_kv_heads=w.n_kv_heads,
        head_dim=w.head_dim, window_k=w.window_k, gamma_far=v.gamma_far,
        alpha_far=v.alpha_far, ring_size=v.ring_size, ema_gamma=v.ema_gamma,
        n_slots=v.n_slots, temperature=v.temperature, clip_eps=v.clip_eps,
        alpha_base=v.alpha_base, cross_decay=v.cross_decay,
        in_dtype=sfa.SFA_F32 if w.in_dtype == "f32" else sfa.SFA_BF16)


def oracle_params(w: Workload) -> oracle.OracleParams:
    v = w.values
    # The library stores the scalars as fp32; the oracle gets the same values.
    f = lambda x: float(np.float32(x))
    return oracle.OracleParams(
        n_q_heads=w.n_q_heads, n_kv_heads=w.n_kv_heads, head_dim=w.head_dim,
        window_k=w.window_k, gamma_far=f(v.gamma_far), alpha_far=f(v.alpha_far),
        ring_size=v.ring_size, ema_gamma=f(v.ema_gamma), n_slots=v.n_slots,
        temperature=f(v.temperature), clip_eps=f(v.clip_eps))


def oracle_alpha(w: Workload, layer: int) -> float:
    v = w.values
    return oracle.alpha_layer(float(np.float32(v.alpha_base)), float(np.float32(v.cross_decay)),
                              layer, w.n_layers)


def np32(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float32).numpy()


def violation(gpu: np.ndarray, ref: np.ndarray, tol: float) -> Tuple[float, int]:
    """Largest |gpu-ref| / (tol*(1+|ref|)) and the number of elements above 1."""
    gpu = np.asarray(gpu, np.float64)
    ref = np.asarray(ref, np.float64)
    if gpu.shape != ref.shape:
        raise AssertionError(f"shape {gpu.shape} vs {ref.shape}")
    if gpu.size == 0:
        return 0.0, 0
    r = np.abs(gpu - ref) / (tol * (1.0 + np.abs(ref)))
    r = np.where(np.isfinite(r), r, np.inf)
    return float(r.max()), int((r > 1.0).sum())


def assert_close(gpu, ref, tol: float, what: str):
    worst, bad = violation(gpu, ref, tol)
    if bad:
        g = np.asarray(gpu, np.float64)
        rf = np.asarray(ref, np.float64)
        idx = np.unravel_index(np.argmax(np.abs(g - rf) / (tol * (1 + np.abs(rf)))), g.shape)
        raise AssertionError(
            f"{what}: {bad} of {g.size} elements outside tol {tol}; worst ratio {worst:.3g} "
            f"at {idx}: gpu {g[idx]!r} oracle {rf[idx]!r}")


class Pair:
    """One workload on the GPU (all streams) and in the oracle (a subset).

    ``layers``/``seqs`` choose the oracle's streams (default: all).
    """

    def __init__(self, w: Workload, layers: Optional[Sequence[int]] = None,
                 seqs: Optional[Sequence[int]] = None, device="cuda", max_prefill: int = 0,
                 gen_device: Optional[str] = None):
        self.w = w
        self.device = torch.device(device)
        self.layers = list(range(w.n_layers)) if layers is None else list(layers)
        self.seqs = list(range(w.batch)) if seqs is None else list(seqs)
        self.src = TokenSource(w, device=gen_device or device)
        slots = make_slots(w, device=gen_device or device)
        self.slots_np = np32(slots)
        self.op = sfa.SfaOperator(sfa_config(w), slots.to(self.device), w.batch,
                                  max_prefill=max_prefill, device=self.device)
        self.p = oracle_params(w)
        self.ostate = oracle.OracleState(self.p, len(self.layers) * len(self.seqs))
        self.t = 0  # tokens folded in so far

    def _streams(self, x: torch.Tensor) -> torch.Tensor:
        """The oracle's (layer, sequence) streams of x, selected where x lives
        (a full-size batch is gigabytes; only the chosen streams go to the host)."""
        L, S = self.layers, self.seqs
        if len(L) != x.shape[0]:
            x = x.index_select(0, torch.tensor(L, device=x.device))
        if len(S) != x.shape[1]:
            x = x.index_select(1, torch.tensor(S, device=x.device))
        return x.cpu()

    def _oracle(self, q, k, v) -> np.ndarray:
        L, S = self.layers, self.seqs
        qs, ks, vs = self._streams(q), self._streams(k), self._streams(v)
        pairs = [(l, b) for l in L for b in S]
        alpha = [oracle_alpha(self.w, l) for (l, _) in pairs]
        sl = np.stack([self.slots_np[l] for (l, _) in pairs]).astype(np.float32)
        n = q.shape[2]
        qq = np32(qs).reshape(len(pairs), n, *q.shape[3:])
        kk = np32(ks).reshape(len(pairs), n, *k.shape[3:])
        vv = np32(vs).reshape(len(pairs), n, *v.shape[3:])
        out, _ = oracle.run_streams(self.p, alpha, sl, qq, kk, vv, self.ostate)
        return out.reshape(len(L), len(S), n, self.p.hidden)

    def _select(self, gpu_out: torch.Tensor) -> np.ndarray:
        L, S = self.layers, self.seqs
        sel = gpu_out[L] if len(L) != gpu_out.shape[0] else gpu_out
        sel = sel[:, S] if len(S) != gpu_out.shape[1] else sel
        return np32(sel)

    def prefill(self, n: int, check: bool = True):
        q, k, v = self.src.get(self.t, self.t + n)
        q, k, v = q.to(self.device), k.to(self.device), v.to(self.device)
        out = self.op.prefill(q, k, v)
        self.t += n
        if not check:
            return None
        ref = self._oracle(q, k, v)
        return self._select(out), ref

    def decode(self, check: bool = True):
        q, k, v = self.src.get(self.t, self.t + 1)
        q, k, v = (x.to(self.device)[:, :, 0].contiguous() for x in (q, k, v))
        out = self.op.decode(q, k, v)
        self.t += 1
        if not check:
            return None
        ref = self._oracle(q[:, :, None], k[:, :, None], v[:, :, None])
        return self._select(out)[:, :, None], ref

    def decode_many(self, steps: int) -> Tuple[np.ndarray, np.ndarray]:
        """`steps` decode calls; the oracle runs them as one token loop."""
        q, k, v = self.src.get(self.t, self.t + steps)
        outs = []
        for s in range(steps):
            qs, ks, vs = (x[:, :, s].to(self.device).contiguous() for x in (q, k, v))
            outs.append(self._select(self.op.decode(qs, ks, vs)))
        self.t += steps
        ref = self._oracle(q, k, v)
        return np.stack(outs, axis=2), ref

    def compare_state(self, tol: float):
        st = sfa.read_state(self.op)
        L, S = self.layers, self.seqs
        o = self.ostate
        shape = (len(L), len(S))

        def sel(x):
            x = x[L] if len(L) != x.shape[0] else x
            return x[:, S] if len(S) != x.shape[1] else x

        pos = sel(st["pos"]).numpy()
        np.testing.assert_array_equal(pos, o.pos.reshape(shape))
        # window slots are copies of input values: bit-exact
        np.testing.assert_array_equal(np32(sel(st["win_k"])).astype(np.float64),
                                      o.win_k.reshape(*shape, *o.win_k.shape[1:]))
        np.testing.assert_array_equal(np32(sel(st["win_v"])).astype(np.float64),
                                      o.win_v.reshape(*shape, *o.win_v.shape[1:]))
        assert_close(np32(sel(st["far"])), o.S.reshape(*shape, *o.S.shape[1:]), tol, "state S")
        assert_close(np32(sel(st["field"])), o.field.reshape(*shape, -1), tol, "state field")
        ring = o.ring.reshape(*shape, *o.ring.shape[1:])
        assert_close(np32(sel(st["ring"])), ring, tol, "state ring")
        assert_close(np32(sel(st["ring_sum"])), ring.sum(axis=2), tol, "state ring_sum")

    def status(self) -> int:
        return self.op.check()
