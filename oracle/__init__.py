"""fp64 CPU oracle of the Signal Field Attention (SFA) operator.

TEST INFRASTRUCTURE ONLY.  Its users are ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py``.  The CUDA library and its Python
binding never import it, and it imports nothing from them.

The arithmetic lives in ``sfa_oracle.c`` (plain C99, double precision, one
token at a time).  This module compiles it with gcc, marshals numpy arrays and
keeps the per-stream fp64 state.

Pinning: every step of the definition is checked by ``tests/test_oracle_pins.py``
against closed forms, textbook special cases (full causal attention, sliding
window attention via ``torch.nn.functional.scaled_dot_product_attention``), an
unrolled whole-path formulation and the pages' printed constants.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from dataclasses import dataclass
from typing import Optional, Sequence, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "sfa_oracle.c")
_HDR = os.path.join(_HERE, "sfa_oracle.h")
_SO = os.path.join(_HERE, "_build", "libsfa_oracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compiles the oracle into ``oracle/_build/libsfa_oracle.so``."""
    os.makedirs(os.path.dirname(_SO), exist_ok=True)
    fresh = (os.path.exists(_SO)
             and os.path.getmtime(_SO) >= max(os.path.getmtime(_SRC), os.path.getmtime(_HDR)))
    if fresh and not force:
        return _SO
    tmp = _SO + f".tmp{os.getpid()}"
    cmd = ["gcc", "-std=c99", "-O2", "-fno-fast-math", "-ffp-contract=off", "-fopenmp",
           "-shared", "-fPIC", "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _SO)
    return _SO


class _Params(ctypes.Structure):
    _fields_ = [
        ("n_q_heads", ctypes.c_int), ("n_kv_heads", ctypes.c_int), ("head_dim", ctypes.c_int),
        ("window_k", ctypes.c_int), ("ring_size", ctypes.c_int), ("n_slots", ctypes.c_int),
        ("gamma_far", ctypes.c_double), ("alpha_far", ctypes.c_double),
        ("ema_gamma", ctypes.c_double), ("temperature", ctypes.c_double),
        ("clip_eps", ctypes.c_double),
    ]


class _Stream(ctypes.Structure):
    _fields_ = [
        ("win_k", ctypes.POINTER(ctypes.c_double)), ("win_v", ctypes.POINTER(ctypes.c_double)),
        ("S", ctypes.POINTER(ctypes.c_double)), ("ring", ctypes.POINTER(ctypes.c_double)),
        ("field", ctypes.POINTER(ctypes.c_double)), ("pos", ctypes.c_longlong),
    ]


def _load():
    global _lib
    with _lock:
        if _lib is None:
            # SFA_ORACLE_LIB lets the mutation tests load a deliberately broken
            # copy of the oracle to show that the pins catch the mistake.
            path = os.environ.get("SFA_ORACLE_LIB") or build()
            lib = ctypes.CDLL(path)
            lib.sfa_oracle_alpha_layer.restype = ctypes.c_double
            lib.sfa_oracle_alpha_layer.argtypes = [ctypes.c_double, ctypes.c_double,
                                                   ctypes.c_int, ctypes.c_int]
            lib.sfa_oracle_run_streams.restype = ctypes.c_int
            _lib = lib
    return _lib


@dataclass(frozen=True)
class OracleParams:
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    window_k: int
    gamma_far: float
    alpha_far: float
    ring_size: int = 16
    ema_gamma: float = 0.98
    n_slots: int = 64
    temperature: float = 0.07
    clip_eps: float = 0.5

    @property
    def hidden(self) -> int:
        return self.n_q_heads * self.head_dim

    def _c(self) -> _Params:
        return _Params(self.n_q_heads, self.n_kv_heads, self.head_dim, self.window_k,
                       self.ring_size, self.n_slots, self.gamma_far, self.alpha_far,
                       self.ema_gamma, self.temperature, self.clip_eps)


def alpha_layer(alpha_base: float, cross_decay: float, layer: int, n_layers: int) -> float:
    return float(_load().sfa_oracle_alpha_layer(alpha_base, cross_decay, layer, n_layers))


class OracleState:
    """fp64 state of ``n_streams`` independent streams (zero, pos 0, at creation)."""

    def __init__(self, p: OracleParams, n_streams: int):
        self.p = p
        self.n_streams = n_streams
        d, K, nkv, H = p.head_dim, p.window_k, p.n_kv_heads, p.hidden
        self.win_k = np.zeros((n_streams, K, nkv, d))
        self.win_v = np.zeros((n_streams, K, nkv, d))
        self.S = np.zeros((n_streams, nkv, d))
        self.ring = np.zeros((n_streams, p.ring_size, H))
        self.field = np.zeros((n_streams, H))
        self.pos = np.zeros((n_streams,), dtype=np.int64)

    def copy(self) -> "OracleState":
        o = OracleState.__new__(OracleState)
        o.p, o.n_streams = self.p, self.n_streams
        for name in ("win_k", "win_v", "S", "ring", "field", "pos"):
            setattr(o, name, getattr(self, name).copy())
        return o

    def subset(self, idx: Sequence[int]) -> "OracleState":
        o = OracleState.__new__(OracleState)
        o.p, o.n_streams = self.p, len(idx)
        for name in ("win_k", "win_v", "S", "ring", "field", "pos"):
            setattr(o, name, np.ascontiguousarray(getattr(self, name)[list(idx)]))
        return o


def _f32(a) -> np.ndarray:
    a = np.asarray(a)
    if a.dtype != np.float32:
        raise TypeError("oracle inputs must be float32 (bf16 values widened exactly)")
    return np.ascontiguousarray(a)


def _dptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def run_streams(p: OracleParams, alpha: Sequence[float], slots, q, k, v,
                state: OracleState) -> Tuple[np.ndarray, int]:
    """Runs n tokens for each of S streams.

    alpha: [S] alpha_layer per stream; slots: [S, n_slots, H] float32;
    q: [S, n, n_q, d]; k, v: [S, n, n_kv, d] float32.  Returns (out [S, n, H]
    float64, threads used).  ``state`` is advanced in place.
    """
    lib = _load()
    slots, q, k, v = _f32(slots), _f32(q), _f32(k), _f32(v)
    S = state.n_streams
    n = q.shape[1]
    assert slots.shape == (S, p.n_slots, p.hidden), slots.shape
    assert q.shape == (S, n, p.n_q_heads, p.head_dim), q.shape
    assert k.shape == (S, n, p.n_kv_heads, p.head_dim) and v.shape == k.shape
    out = np.zeros((S, n, p.hidden))
    if S == 0 or n == 0:
        return out, 0
    streams = (_Stream * S)()
    for s in range(S):
        streams[s].win_k = _dptr(state.win_k[s])
        streams[s].win_v = _dptr(state.win_v[s])
        streams[s].S = _dptr(state.S[s])
        streams[s].ring = _dptr(state.ring[s])
        streams[s].field = _dptr(state.field[s])
        streams[s].pos = int(state.pos[s])
    sptrs = (ctypes.POINTER(_Stream) * S)(*[ctypes.pointer(streams[s]) for s in range(S)])
    FP = ctypes.POINTER(ctypes.c_float)
    mk = lambda arr: (FP * S)(*[arr[s].ctypes.data_as(FP) for s in range(S)])
    alpha_arr = (ctypes.c_double * S)(*[float(a) for a in alpha])
    outp = (ctypes.POINTER(ctypes.c_double) * S)(*[_dptr(out[s]) for s in range(S)])
    used = ctypes.c_int(0)
    params = p._c()
    rc = lib.sfa_oracle_run_streams(ctypes.byref(params), ctypes.c_int(S), alpha_arr, mk(slots),
                                    mk(q), mk(k), mk(v), ctypes.c_longlong(n), sptrs, outp,
                                    ctypes.byref(used))
    if rc != 0:
        raise ValueError("oracle rejected the parameters")
    for s in range(S):
        state.pos[s] = streams[s].pos
    return out, int(used.value)


def run_layers(p: OracleParams, alpha_base: float, cross_decay: float, slots, q, k, v,
               state: OracleState, layers: Optional[Sequence[int]] = None,
               seqs: Optional[Sequence[int]] = None, n_layers: Optional[int] = None):
    """Convenience form for [L, B, ...] tensors.

    slots [L, P, H]; q [L, B, n, n_q, d]; k, v [L, B, n, n_kv, d] (float32).
    Runs the streams (l, b) for l in ``layers`` and b in ``seqs`` (default: all);
    ``state`` holds exactly those streams in that (layer-major) order.  Returns
    out [len(layers), len(seqs), n, H].
    """
    q, k, v = np.asarray(q), np.asarray(k), np.asarray(v)
    L, B = q.shape[0], q.shape[1]
    n_layers = L if n_layers is None else n_layers
    layers = list(range(L)) if layers is None else list(layers)
    seqs = list(range(B)) if seqs is None else list(seqs)
    pairs = [(l, b) for l in layers for b in seqs]
    assert state.n_streams == len(pairs)
    alpha = [alpha_layer(alpha_base, cross_decay, l, n_layers) for (l, _) in pairs]
    sl = np.stack([np.asarray(slots)[l] for (l, _) in pairs]) if pairs else np.zeros((0,))
    qq = np.stack([q[l, b] for (l, b) in pairs])
    kk = np.stack([k[l, b] for (l, b) in pairs])
    vv = np.stack([v[l, b] for (l, b) in pairs])
    out, used = run_streams(p, alpha, sl.astype(np.float32), qq, kk, vv, state)
    return out.reshape(len(layers), len(seqs), q.shape[2], p.hidden), used
