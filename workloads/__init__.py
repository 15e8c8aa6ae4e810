"""Seeded synthetic workloads for the Signal Field Attention (SFA) operator.

This module is shared by the fp64 oracle's tests, the CUDA path's tests,
``bench.py`` and ``__graft_entry__``.  It holds shapes, configuration values
and random-number recipes only: none of the operator's arithmetic lives here.

Shapes follow the models the source pages measure on:
  * "Signal Field Attention (SFA)：8KB代码实现4.16倍推理加速与248倍内存压缩"
    §3.1 (Qwen2.5-0.5B-Instruct and Qwen2.5-7B-Instruct) and §3.3/§3.4
    (contexts 128 / 1,024 / 4,096 / 8,192);
  * "Dalin Soma SFA基于信号场注意力机制的神经网络推理加速框架" §3.2
    (Qwen2.5-0.5B, 512-token prefill, 128 generated tokens).
The pages measure on text corpora with real checkpoints; here synthetic
Q/K/V activations of the same shapes stand in for them.

Value recipes:
  * ``normal``: N(0, 1), rounded to the input dtype.
  * ``normal_drift``: N(0, 1) times s_t = 1 + 3 t / (n - 1) on every Q, K and
    V row of token t (per-token norms drift x1 -> x4 over the sequence).
  * ``student_t3``: Student-t with 3 degrees of freedom, built as
    z * sqrt(3 / (n1^2 + n2^2 + n3^2)) from four independent normals.

Every token's values depend only on (workload seed, tensor, token block), so
any split of a sequence into prefill chunks and decode steps sees the same
numbers.  Generation happens on the device the caller names (CPU or CUDA);
the two devices give different but individually reproducible streams, so a
test draws once and hands copies to both sides.
"""
from __future__ import annotations

import dataclasses
from dataclasses import dataclass, field
from typing import Dict, List, Optional, Tuple

import torch

__all__ = [
    "SfaConfigValues",
    "Workload",
    "WORKLOADS",
    "get_workload",
    "TokenSource",
    "make_slots",
    "sweep_c5",
]

# Token values are generated in blocks of this many tokens; a block is the
# unit of seeding so that chunking never changes the numbers.
TOKEN_BLOCK = 64


@dataclass(frozen=True)
class SfaConfigValues:
    """Operator hyper-parameters (names follow the pages' ``SFA_Config``)."""

    gamma_far: float = 0.9
    alpha_far: float = 0.1
    ring_size: int = 16
    ema_gamma: float = 0.98
    n_slots: int = 64
    temperature: float = 0.07
    clip_eps: float = 0.5
    alpha_base: float = 0.1
    cross_decay: float = 0.8


@dataclass(frozen=True)
class Workload:
    name: str
    n_layers: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    window_k: int
    batch: int
    in_dtype: str  # "f32" or "bf16"
    values: SfaConfigValues
    prefill_n: Tuple[int, ...]
    decode_steps: int
    dist: str = "normal"  # normal | normal_drift | student_t3
    seed: int = 0
    drift_n: int = 0  # total sequence length the norm drift is spread over

    @property
    def hidden(self) -> int:
        return self.n_q_heads * self.head_dim

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.float32 if self.in_dtype == "f32" else torch.bfloat16

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


_V = SfaConfigValues

WORKLOADS: Dict[str, Workload] = {
    # Tiny parity case: 1 layer, no GQA.
    "tiny": Workload(
        name="tiny", n_layers=1, n_q_heads=2, n_kv_heads=2, head_dim=64,
        window_k=16, batch=1, in_dtype="f32",
        values=_V(gamma_far=0.9, alpha_far=0.1, alpha_base=0.1, cross_decay=0.8),
        prefill_n=(128,), decode_steps=32, seed=1000),
    # Qwen2.5-0.5B attention shape.
    "qwen05b": Workload(
        name="qwen05b", n_layers=24, n_q_heads=14, n_kv_heads=2, head_dim=64,
        window_k=16, batch=1, in_dtype="bf16",
        values=_V(gamma_far=0.9, alpha_far=0.1, alpha_base=0.1, cross_decay=0.8),
        prefill_n=(512,), decode_steps=128, seed=2000),
    # Qwen2.5-7B attention shape, decode after three context lengths.
    "qwen7b_decode": Workload(
        name="qwen7b_decode", n_layers=28, n_q_heads=28, n_kv_heads=4,
        head_dim=128, window_k=16, batch=1, in_dtype="bf16",
        values=_V(gamma_far=0.9, alpha_far=0.1, alpha_base=1.0, cross_decay=0.95),
        prefill_n=(1024, 4096, 8192), decode_steps=256, seed=3000),
    # Long prefill scan stress: one 7B-shaped layer, 4 x 65,536 tokens.
    "long_prefill": Workload(
        name="long_prefill", n_layers=1, n_q_heads=28, n_kv_heads=4,
        head_dim=128, window_k=16, batch=4, in_dtype="bf16",
        values=_V(gamma_far=0.98, alpha_far=0.1, alpha_base=0.1, cross_decay=0.8),
        prefill_n=(65536,), decode_steps=0, dist="normal_drift", seed=4000,
        drift_n=65536),
    # Batched decode / heavy tails: one point of the sweep (see sweep_c5).
    "batched_decode": Workload(
        name="batched_decode", n_layers=28, n_q_heads=28, n_kv_heads=4,
        head_dim=128, window_k=16, batch=256, in_dtype="bf16",
        values=_V(gamma_far=0.9, alpha_far=0.1, alpha_base=1.0, cross_decay=0.95),
        prefill_n=(1024,), decode_steps=512, dist="student_t3", seed=5000),
}

# alpha_base paired with the cross-layer decay of the pages' calibration
# table (conservative / moderate / aggressive presets).
ALPHA_PRESETS: Tuple[Tuple[float, float], ...] = ((0.04, 0.90), (1.0, 0.95), (10.0, 0.98))


def sweep_c5() -> List[Workload]:
    """The 18 points of the batched-decode sweep: k x gamma_far x alpha preset."""
    base = WORKLOADS["batched_decode"]
    out = []
    i = 0
    for k in (16, 64, 256):
        for gf in (0.9, 0.98):
            for ab, dec in ALPHA_PRESETS:
                out.append(base.replace(
                    name=f"batched_decode_k{k}_g{gf}_a{ab}", window_k=k,
                    values=dataclasses.replace(base.values, gamma_far=gf,
                                               alpha_base=ab, cross_decay=dec),
                    seed=base.seed + 100 * i))
                i += 1
    return out


def get_workload(name: str) -> Workload:
    if name in WORKLOADS:
        return WORKLOADS[name]
    for w in sweep_c5():
        if w.name == name:
            return w
    raise KeyError(name)


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed) & 0x7FFF_FFFF_FFFF_FFFF)
    return g


def _draw(shape, dist: str, g: torch.Generator, device) -> torch.Tensor:
    if dist in ("normal", "normal_drift"):
        return torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    if dist == "student_t3":
        z = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
        chi = torch.zeros(shape, device=device, dtype=torch.float32)
        for _ in range(3):
            n = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
            chi.addcmul_(n, n)
        return z * torch.sqrt(3.0 / chi)
    raise ValueError(dist)


_TENSOR_ID = {"q": 1, "k": 2, "v": 3}


class TokenSource:
    """Deterministic per-token Q/K/V for one workload on one device.

    ``get(t0, t1)`` returns q [L,B,n,n_q,d], k and v [L,B,n,n_kv,d] for
    tokens [t0, t1) in the workload's input dtype.
    """

    def __init__(self, w: Workload, device="cpu", salt: int = 0):
        self.w = w
        self.device = torch.device(device)
        self.salt = salt
        self._cache: Dict[int, Tuple[torch.Tensor, ...]] = {}

    def _block(self, blk: int):
        if blk in self._cache:
            return self._cache[blk]
        w = self.w
        L, B = w.n_layers, w.batch
        out = []
        for name, heads in (("q", w.n_q_heads), ("k", w.n_kv_heads), ("v", w.n_kv_heads)):
            seed = (w.seed * 1_000_003 + self.salt * 7919
                    + _TENSOR_ID[name] * 1_000_000_007 + blk * 97)
            g = _gen(seed, self.device)
            x = _draw((L, B, TOKEN_BLOCK, heads, w.head_dim), w.dist, g, self.device)
            if w.dist == "normal_drift":
                n_tot = max(w.drift_n, 2)
                t = torch.arange(blk * TOKEN_BLOCK, (blk + 1) * TOKEN_BLOCK,
                                 device=self.device, dtype=torch.float32)
                s = 1.0 + 3.0 * t / float(n_tot - 1)
                x = x * s.view(1, 1, TOKEN_BLOCK, 1, 1)
            out.append(x.to(w.torch_dtype))
        # keep at most two blocks resident
        if len(self._cache) >= 2:
            self._cache.pop(next(iter(self._cache)))
        self._cache[blk] = tuple(out)
        return self._cache[blk]

    def get(self, t0: int, t1: int):
        assert 0 <= t0 <= t1
        w = self.w
        if t1 == t0:
            e = lambda h: torch.empty((w.n_layers, w.batch, 0, h, w.head_dim),
                                      dtype=w.torch_dtype, device=self.device)
            return e(w.n_q_heads), e(w.n_kv_heads), e(w.n_kv_heads)
        parts = ([], [], [])
        t = t0
        while t < t1:
            blk = t // TOKEN_BLOCK
            lo = t - blk * TOKEN_BLOCK
            hi = min(t1 - blk * TOKEN_BLOCK, TOKEN_BLOCK)
            b = self._block(blk)
            for i in range(3):
                parts[i].append(b[i][:, :, lo:hi])
            t = blk * TOKEN_BLOCK + hi
        return tuple(torch.cat(p, dim=2).contiguous() if len(p) > 1 else p[0].contiguous()
                     for p in parts)


def make_slots(w: Workload, device="cpu", salt: int = 0) -> torch.Tensor:
    """Semantic-pool slots [L, n_slots, hidden] fp32 ~ N(0, 1), seeded per layer."""
    H = w.hidden
    P = w.values.n_slots
    out = torch.empty((w.n_layers, P, H), dtype=torch.float32, device=device)
    for layer in range(w.n_layers):
        g = _gen(w.seed * 31 + 17 + layer * 1009 + salt * 65537, device)
        out[layer] = torch.randn((P, H), generator=g, device=device, dtype=torch.float32)
    return out
