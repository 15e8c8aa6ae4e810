"""Python binding of the SFA C ABI (``include/sfa.h``).

Argument marshalling only: every step of the operator runs in the CUDA
library ``libsfa.so`` built from ``csrc/``.  PyTorch supplies device memory
and streams.  There is no CPU fallback: if the library is missing the calls
raise.

The functions keep the C names (``sfa_init``, ``sfa_prefill``,
``sfa_decode_step``, ``sfa_state_reset``, ...).  ``SfaOperator`` bundles a
handle with its state and workspace buffers for convenience.

Sources (web pages):
  [P1] "Signal Field Attention (SFA)：8KB代码实现4.16倍推理加速与248倍内存压缩"
  [P2] "Signal Field Attention (SFA)" (project README page)
  [P3] "Dalin Soma SFA基于信号场注意力机制的神经网络推理加速框架"
"""
from __future__ import annotations

import ctypes
import os
import threading
from dataclasses import dataclass
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libsfa.so")

SFA_OK = 0
SFA_ERR_INVALID_ARG = -1
SFA_ERR_UNSUPPORTED = -2
SFA_ERR_ALIGNMENT = -3
SFA_ERR_STATE_MISMATCH = -4
SFA_ERR_CUDA = -5
SFA_ERR_DEVICE_TIMEOUT = -6
SFA_ERR_WORKSPACE = -7

SFA_F32 = 0
SFA_BF16 = 1

SFA_OUT_F32 = 0       # out fp32 = x + enhancement (default)
SFA_OUT_BF16 = 1      # out bf16 = x + enhancement
SFA_OUT_ADD_F32 = 2   # out fp32 += enhancement (out holds the caller's attention output)
SFA_OUT_ADD_BF16 = 3  # out bf16 += enhancement

EXPORTED = (
    "sfa_config_default", "sfa_config_validate", "sfa_state_layout_for", "sfa_init",
    "sfa_destroy", "sfa_state_bytes", "sfa_prefill_workspace_bytes", "sfa_state_reset",
    "sfa_prefill", "sfa_decode_step", "sfa_check_device_status", "sfa_status_string",
    "sfa_abi_version", "sfa_debug_set_wait_limit", "sfa_debug_set_paths", "sfa_prefill_static_ws",
    "sfa_prefill_layers_workspace_bytes", "sfa_prefill_layers", "sfa_decode_step_ex",
    "sfa_set_decode_input_prefetch", "sfa_prefill_ragged", "sfa_set_output_mode",
)


class SfaError(RuntimeError):
    def __init__(self, code: int, what: str = ""):
        self.code = code
        super().__init__(f"{what}: {sfa_status_string(code)} ({code})" if what else
                         f"{sfa_status_string(code)} ({code})")


class sfa_config(ctypes.Structure):
    _fields_ = [
        ("n_layers", ctypes.c_int), ("n_q_heads", ctypes.c_int), ("n_kv_heads", ctypes.c_int),
        ("head_dim", ctypes.c_int), ("window_k", ctypes.c_int), ("gamma_far", ctypes.c_float),
        ("alpha_far", ctypes.c_float), ("ring_size", ctypes.c_int), ("ema_gamma", ctypes.c_float),
        ("n_slots", ctypes.c_int), ("temperature", ctypes.c_float), ("clip_eps", ctypes.c_float),
        ("alpha_base", ctypes.c_float), ("cross_decay", ctypes.c_float),
        ("in_dtype", ctypes.c_int), ("slots", ctypes.c_void_p),
    ]


class sfa_state_layout(ctypes.Structure):
    _fields_ = [(name, ctypes.c_size_t) for name in (
        "header_bytes", "stream_stride", "total_bytes", "off_pos", "off_win_k", "off_win_v",
        "off_far", "off_field", "off_ring_sum", "off_ring")]


_lock = threading.Lock()
_lib = None


def load_library(path: Optional[str] = None) -> ctypes.CDLL:
    """Loads libsfa.so (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        path = path or LIB_PATH
        if not os.path.exists(path):
            raise RuntimeError(
                f"SFA CUDA library not found at {path}; build it with "
                "`python kv_cache_compression_sfa_b200/build.py` or __graft_entry__.build()")
        lib = ctypes.CDLL(path)
        vp, i, ll, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_longlong, ctypes.c_size_t
        P = ctypes.POINTER
        sigs = {
            "sfa_config_default": (None, [P(sfa_config)]),
            "sfa_config_validate": (i, [P(sfa_config)]),
            "sfa_state_layout_for": (i, [P(sfa_config), i, P(sfa_state_layout)]),
            "sfa_init": (i, [P(sfa_config), P(vp)]),
            "sfa_destroy": (i, [vp]),
            "sfa_state_bytes": (sz, [vp, i]),
            "sfa_prefill_workspace_bytes": (sz, [vp, i, ll]),
            "sfa_state_reset": (i, [vp, vp, i, vp]),
            "sfa_prefill": (i, [vp, vp, vp, vp, ll, i, vp, vp, vp, sz, vp]),
            "sfa_decode_step": (i, [vp, vp, vp, vp, i, vp, vp, vp]),
            "sfa_check_device_status": (i, [vp, vp]),
            "sfa_status_string": (ctypes.c_char_p, [i]),
            "sfa_abi_version": (i, []),
            "sfa_debug_set_wait_limit": (i, [vp, ctypes.c_uint, ll]),
            "sfa_debug_set_paths": (i, [vp, i, i]),
            "sfa_prefill_static_ws": (i, [vp, vp, vp, vp, ll, i, vp, vp, vp]),
            "sfa_prefill_layers_workspace_bytes": (sz, [vp, i, i, ll]),
            "sfa_prefill_layers": (i, [vp, i, i, vp, vp, vp, ll, i, vp, vp, vp, sz, vp]),
            "sfa_decode_step_ex": (i, [vp, i, i, vp, i, vp, vp, vp, i, vp, vp, vp]),
            "sfa_set_decode_input_prefetch": (i, [vp, i]),
            "sfa_prefill_ragged": (i, [vp, vp, vp, vp, ll, vp, i, vp, vp, vp, sz, vp]),
            "sfa_set_output_mode": (i, [vp, i]),
        }
        for name, (res, args) in sigs.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
        return lib


# --------------------------------------------------------------- host-only


@dataclass
class SfaConfig:
    """Python view of ``sfa_config``; defaults are the pages' SFA_Config."""

    n_layers: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    window_k: int = 16
    gamma_far: float = 0.9
    alpha_far: float = 0.1
    ring_size: int = 16
    ema_gamma: float = 0.98
    n_slots: int = 64
    temperature: float = 0.07
    clip_eps: float = 0.5
    alpha_base: float = 0.1
    cross_decay: float = 0.8
    in_dtype: int = SFA_BF16

    @property
    def hidden(self) -> int:
        return self.n_q_heads * self.head_dim

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.float32 if self.in_dtype == SFA_F32 else torch.bfloat16

    def to_c(self, slots_ptr: int = 0) -> sfa_config:
        c = sfa_config()
        for f, _ in sfa_config._fields_:
            if f != "slots":
                setattr(c, f, getattr(self, f))
        c.slots = slots_ptr
        return c


def sfa_config_default() -> sfa_config:
    c = sfa_config()
    load_library().sfa_config_default(ctypes.byref(c))
    return c


def sfa_config_validate(cfg: sfa_config) -> int:
    return int(load_library().sfa_config_validate(ctypes.byref(cfg)))


def sfa_state_layout_for(cfg: sfa_config, batch: int) -> sfa_state_layout:
    lay = sfa_state_layout()
    rc = load_library().sfa_state_layout_for(ctypes.byref(cfg), batch, ctypes.byref(lay))
    if rc != SFA_OK:
        raise SfaError(rc, "sfa_state_layout_for")
    return lay


def sfa_status_string(code: int) -> str:
    return load_library().sfa_status_string(int(code)).decode()


def sfa_abi_version() -> int:
    return int(load_library().sfa_abi_version())


# --------------------------------------------------------------- device


def _stream_ptr(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream) if hasattr(stream, "cuda_stream") else int(stream)


def _is_cuda_tensor(t) -> bool:
    return isinstance(t, torch.Tensor) and t.is_cuda


def _dev(t: torch.Tensor, name: str, dtype=None, min_numel: int = 0) -> int:
    if not _is_cuda_tensor(t):
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must have dtype {dtype}, got {t.dtype}")
    if t.numel() < min_numel:
        raise ValueError(f"{name} has {t.numel()} elements, needs {min_numel}")
    return t.data_ptr()


class Handle:
    """An initialised sfa_handle and the configuration it was built from."""

    def __init__(self, ptr: int, cfg: SfaConfig):
        self.ptr = ptr
        self.cfg = cfg
        self.out_mode = SFA_OUT_F32

    @property
    def out_dtype(self) -> torch.dtype:
        """dtype of `out` in the handle's output mode."""
        return torch.bfloat16 if self.out_mode in (SFA_OUT_BF16, SFA_OUT_ADD_BF16) else torch.float32

    def __del__(self):
        if getattr(self, "ptr", None):
            try:
                load_library().sfa_destroy(self.ptr)
            except Exception:
                pass
            self.ptr = None


def sfa_init(cfg: SfaConfig, slots: torch.Tensor) -> Handle:
    L, P, H = cfg.n_layers, cfg.n_slots, cfg.hidden
    _dev(slots, "slots", torch.float32, L * P * H)
    c = cfg.to_c(slots.data_ptr())
    h = ctypes.c_void_p()
    rc = load_library().sfa_init(ctypes.byref(c), ctypes.byref(h))
    if rc != SFA_OK:
        raise SfaError(rc, "sfa_init")
    return Handle(h.value, cfg)


def sfa_destroy(h: Handle) -> None:
    if h.ptr:
        rc = load_library().sfa_destroy(h.ptr)
        h.ptr = None
        if rc != SFA_OK:
            raise SfaError(rc, "sfa_destroy")


def sfa_state_bytes(h: Handle, batch: int) -> int:
    return int(load_library().sfa_state_bytes(h.ptr, batch))


def sfa_prefill_workspace_bytes(h: Handle, batch: int, n: int) -> int:
    return int(load_library().sfa_prefill_workspace_bytes(h.ptr, batch, n))


def sfa_state_reset(h: Handle, state: torch.Tensor, batch: int, stream=None) -> None:
    _dev(state, "state", torch.uint8, sfa_state_bytes(h, batch))
    rc = load_library().sfa_state_reset(h.ptr, state.data_ptr(), batch, _stream_ptr(stream))
    if rc != SFA_OK:
        raise SfaError(rc, "sfa_state_reset")


def _qkv_checks(h: Handle, q, k, v, tokens: int, batch: int, layers: Optional[int] = None):
    c = h.cfg
    rows = (c.n_layers if layers is None else layers) * batch * tokens
    return (_dev(q, "q", c.torch_dtype, rows * c.n_q_heads * c.head_dim),
            _dev(k, "k", c.torch_dtype, rows * c.n_kv_heads * c.head_dim),
            _dev(v, "v", c.torch_dtype, rows * c.n_kv_heads * c.head_dim))


def sfa_prefill(h: Handle, q, k, v, n: int, batch: int, state: torch.Tensor, out: torch.Tensor,
                workspace: Optional[torch.Tensor], stream=None) -> None:
    if n == 0:
        return
    qp, kp, vp = _qkv_checks(h, q, k, v, n, batch)
    sp = _dev(state, "state", torch.uint8, sfa_state_bytes(h, batch))
    op = _dev(out, "out", h.out_dtype, h.cfg.n_layers * batch * n * h.cfg.hidden)
    need = sfa_prefill_workspace_bytes(h, batch, n)
    if workspace is None or workspace.numel() < need:
        raise SfaError(SFA_ERR_WORKSPACE, "sfa_prefill")
    wp = _dev(workspace, "workspace", torch.uint8)
    rc = load_library().sfa_prefill(h.ptr, qp, kp, vp, n, batch, sp, op, wp,
                                    workspace.numel(), _stream_ptr(stream))
    if rc != SFA_OK:
        raise SfaError(rc, "sfa_prefill")


def sfa_prefill_ragged(h: Handle, q, k, v, n_max: int, lens: torch.Tensor, batch: int,
                       state: torch.Tensor, out: torch.Tensor, workspace: Optional[torch.Tensor],
                       stream=None) -> None:
    """sfa_prefill where sequence b folds in lens[b] (device int32) tokens of
    its rows 0 .. lens[b]-1 of the n_max-row inputs; out rows past lens[b]
    are left as they were."""
    if n_max == 0:
        return
    qp, kp, vp = _qkv_checks(h, q, k, v, n_max, batch)
    sp = _dev(state, "state", torch.uint8, sfa_state_bytes(h, batch))
    op = _dev(out, "out", h.out_dtype, h.cfg.n_layers * batch * n_max * h.cfg.hidden)
    lp = _dev(lens, "lens", torch.int32, batch)
    need = sfa_prefill_workspace_bytes(h, batch, n_max)
    if workspace is None or workspace.numel() < need:
        raise SfaError(SFA_ERR_WORKSPACE, "sfa_prefill_ragged")
    wp = _dev(workspace, "workspace", torch.uint8)
    rc = load_library().sfa_prefill_ragged(h.ptr, qp, kp, vp, n_max, lp, batch, sp, op, wp,
                                           workspace.numel(), _stream_ptr(stream))
    if rc != SFA_OK:
        raise SfaError(rc, "sfa_prefill_ragged")


def sfa_prefill_layers_workspace_bytes(h: Handle, layer_count: int, batch: int, n: int) -> int:
    return int(load_library().sfa_prefill_layers_workspace_bytes(h.ptr, layer_count, batch, n))


def sfa_prefill_layers(h: Handle, layer_begin: int, layer_count: int, q, k, v, n: int,
                       batch: int, state: torch.Tensor, out: torch.Tensor,
                       workspace: Optional[torch.Tensor], stream=None) -> None:
    """sfa_prefill for layers layer_begin .. layer_begin+layer_count-1 only;
    q/k/v/out hold those layers alone."""
    if n == 0:
        return
    qp, kp, vp = _qkv_checks(h, q, k, v, n, batch, layer_count)
    sp = _dev(state, "state", torch.uint8, sfa_state_bytes(h, batch))
    op = _dev(out, "out", h.out_dtype, layer_count * batch * n * h.cfg.hidden)
    need = sfa_prefill_layers_workspace_bytes(h, layer_count, batch, n)
    if workspace is None or workspace.numel() < need:
        raise SfaError(SFA_ERR_WORKSPACE, "sfa_prefill_layers")
    wp = _dev(workspace, "workspace", torch.uint8)
    rc = load_library().sfa_prefill_layers(h.ptr, layer_begin, layer_count, qp, kp, vp, n, batch,
                                           sp, op, wp, workspace.numel(), _stream_ptr(stream))
    if rc != SFA_OK:
        raise SfaError(rc, "sfa_prefill_layers")


def sfa_decode_step_ex(h: Handle, layer_begin: int, layer_count: int,
                       seq_ids: Optional[torch.Tensor], q, k, v, batch: int,
                       state: torch.Tensor, out: torch.Tensor, stream=None) -> None:
    """sfa_decode_step for a layer range and (optionally) a device int32
    tensor of distinct sequence indices; q/k/v/out rows follow seq_ids."""
    n_seq = batch if seq_ids is None else int(seq_ids.numel())
    qp, kp, vp = _qkv_checks(h, q, k, v, 1, n_seq, layer_count)
    sp = _dev(state, "state", torch.uint8, sfa_state_bytes(h, batch))
    op = _dev(out, "out", h.out_dtype, layer_count * n_seq * h.cfg.hidden)
    ip = None if seq_ids is None else _dev(seq_ids, "seq_ids", torch.int32, n_seq)
    rc = load_library().sfa_decode_step_ex(h.ptr, layer_begin, layer_count, ip, n_seq, qp, kp, vp,
                                           batch, sp, op, _stream_ptr(stream))
    if rc != SFA_OK:
        raise SfaError(rc, "sfa_decode_step_ex")


SFA_STATIC_WORKSPACE_BYTES = 16 << 20


def sfa_prefill_static_ws(h: Handle, q, k, v, n: int, batch: int, state: torch.Tensor,
                          out: torch.Tensor, stream=None) -> None:
    """sfa_prefill on the library's fixed device scratch (no workspace
    argument, nothing allocated); see include/sfa.h for the limits."""
    if n == 0:
        return
    qp, kp, vp = _qkv_checks(h, q, k, v, n, batch)
    sp = _dev(state, "state", torch.uint8, sfa_state_bytes(h, batch))
    op = _dev(out, "out", h.out_dtype, h.cfg.n_layers * batch * n * h.cfg.hidden)
    rc = load_library().sfa_prefill_static_ws(h.ptr, qp, kp, vp, n, batch, sp, op,
                                              _stream_ptr(stream))
    if rc != SFA_OK:
        raise SfaError(rc, "sfa_prefill_static_ws")


def sfa_decode_step(h: Handle, q, k, v, batch: int, state: torch.Tensor, out: torch.Tensor,
                    stream=None) -> None:
    """One token per sequence, all layers.  q, k and v are read once the
    previous kernel on the stream has finished, unless the handle's input
    prefetch is on (sfa_set_decode_input_prefetch)."""
    qp, kp, vp = _qkv_checks(h, q, k, v, 1, batch)
    sp = _dev(state, "state", torch.uint8, sfa_state_bytes(h, batch))
    op = _dev(out, "out", h.out_dtype, h.cfg.n_layers * batch * h.cfg.hidden)
    rc = load_library().sfa_decode_step(h.ptr, qp, kp, vp, batch, sp, op, _stream_ptr(stream))
    if rc != SFA_OK:
        raise SfaError(rc, "sfa_decode_step")


def sfa_set_decode_input_prefetch(h: Handle, enable: bool) -> None:
    """Declare (True) that every later decode call's q, k and v are complete
    when the call is enqueued and that nothing still running on the stream
    writes them; the decode kernel then fetches them before the previous
    kernel on the stream has finished.  False (the default) fetches them
    after it.  Results are identical either way."""
    rc = load_library().sfa_set_decode_input_prefetch(h.ptr, 1 if enable else 0)
    if rc != SFA_OK:
        raise SfaError(rc, "sfa_set_decode_input_prefetch")


def sfa_set_output_mode(h: Handle, mode: int) -> None:
    """What later compute calls write into out: SFA_OUT_F32 / SFA_OUT_BF16
    (x + enhancement) or SFA_OUT_ADD_F32 / SFA_OUT_ADD_BF16 (out, holding
    the caller's attention output, plus the enhancement in place)."""
    rc = load_library().sfa_set_output_mode(h.ptr, int(mode))
    if rc != SFA_OK:
        raise SfaError(rc, "sfa_set_output_mode")
    h.out_mode = int(mode)


def sfa_check_device_status(h: Handle, stream=None) -> int:
    return int(load_library().sfa_check_device_status(h.ptr, _stream_ptr(stream)))


def sfa_debug_set_wait_limit(h: Handle, spin_limit: int = 0, withhold_tile: int = -1) -> None:
    """Test hook of the prefill's bounded waits: the pool CTA of tile
    `withhold_tile` (tile * streams + stream) waits on a barrier that nothing
    completes, giving up after `spin_limit` polls (0: default); -1 disables."""
    rc = load_library().sfa_debug_set_wait_limit(h.ptr, spin_limit, withhold_tile)
    if rc != SFA_OK:
        raise SfaError(rc, "sfa_debug_set_wait_limit")


def sfa_debug_set_paths(h: Handle, decode_tile: int = -1, prefill_near=3) -> None:
    """Test hook that pins the kernel variants: decode_tile -1 (by batch
    size), 0 (per-sequence kernel) or 1 (batch-tiled kernel); prefill near
    field, where the tensor cores apply, 3 by call size (the default; also
    True), 2 fused with the pool scores, 1 tensor cores with a separate pool
    kernel, 0 CUDA cores (also False)."""
    mode = {True: 3, False: 0}[prefill_near] if isinstance(prefill_near, bool) else int(prefill_near)
    rc = load_library().sfa_debug_set_paths(h.ptr, int(decode_tile), mode)
    if rc != SFA_OK:
        raise SfaError(rc, "sfa_debug_set_paths")


class SfaOperator:
    """A handle plus the device buffers one batch of sequences needs.

    ``prefill(q, k, v)`` takes [L, B, n, heads, d] tensors and returns
    out [L, B, n, hidden] fp32; ``decode(q, k, v)`` takes [L, B, heads, d]
    and returns [L, B, hidden].
    """

    def __init__(self, cfg: SfaConfig, slots: torch.Tensor, batch: int,
                 max_prefill: int = 0, device=None):
        self.cfg = cfg
        self.batch = batch
        self.device = torch.device(device or slots.device)
        self.handle = sfa_init(cfg, slots)
        self._state_bytes = sfa_state_bytes(self.handle, batch)
        self.state = torch.empty(self._state_bytes, dtype=torch.uint8, device=self.device)
        # Per-call constants of decode(), which a serving loop calls once per
        # token: the C entry point, the element counts and the input dtype.
        rows = cfg.n_layers * batch
        self._dec_numel = (rows * cfg.n_q_heads * cfg.head_dim, rows * cfg.n_kv_heads * cfg.head_dim,
                           rows * cfg.hidden)
        self._in_dtype = cfg.torch_dtype
        self._decode_fn = load_library().sfa_decode_step
        self.workspace = None
        if max_prefill > 0:
            self._ensure_workspace(max_prefill)
        self.reset()

    def _grow_workspace(self, need: int, stream=None):
        """A workspace of at least `need` bytes.  The buffer it replaces may
        still be in use by work enqueued on `stream`: it is marked as used
        there, so the caching allocator hands it out again only after that
        work."""
        if self.workspace is None or self.workspace.numel() < need:
            if self.workspace is not None and isinstance(stream, torch.cuda.Stream):
                self.workspace.record_stream(stream)
            self.workspace = torch.empty(need, dtype=torch.uint8, device=self.device)

    def _ensure_workspace(self, n: int, stream=None):
        self._grow_workspace(sfa_prefill_workspace_bytes(self.handle, self.batch, n), stream)

    def reset(self, stream=None):
        sfa_state_reset(self.handle, self.state, self.batch, stream)

    def set_output_mode(self, mode: int) -> None:
        sfa_set_output_mode(self.handle, mode)

    def _new_out(self, shape, stream=None):
        """A result buffer allocated on the current stream; if the call runs
        on another stream it is marked as used there too."""
        if self.handle.out_mode in (SFA_OUT_ADD_F32, SFA_OUT_ADD_BF16):
            raise ValueError("the add output modes need out: it holds the attention output")
        out = torch.empty(shape, dtype=self.handle.out_dtype, device=self.device)
        if isinstance(stream, torch.cuda.Stream):
            out.record_stream(stream)
        return out

    def prefill(self, q, k, v, out: Optional[torch.Tensor] = None, stream=None):
        n = q.shape[2]
        c = self.cfg
        if out is None:
            out = self._new_out((c.n_layers, self.batch, n, c.hidden), stream)
        if n > 0:
            self._ensure_workspace(n, stream)
            sfa_prefill(self.handle, q, k, v, n, self.batch, self.state, out, self.workspace,
                        stream)
        return out

    def prefill_ragged(self, q, k, v, lens: torch.Tensor, out: Optional[torch.Tensor] = None,
                       stream=None):
        """Prefill where sequence b takes lens[b] (device int32) of the n_max
        rows of q, k, v ([L, B, n_max, heads, d]); out rows past lens[b] keep
        their contents (a new out starts as NaN there)."""
        n = q.shape[2]
        c = self.cfg
        if out is None:
            out = self._new_out((c.n_layers, self.batch, n, c.hidden), stream).fill_(float("nan"))
            if isinstance(stream, torch.cuda.Stream):
                stream.wait_stream(torch.cuda.current_stream())  # the fill comes first
        if n > 0:
            self._ensure_workspace(n, stream)
            sfa_prefill_ragged(self.handle, q, k, v, n, lens, self.batch, self.state, out,
                               self.workspace, stream)
        return out

    def decode(self, q, k, v, out: Optional[torch.Tensor] = None, stream=None):
        """One token per sequence, all layers: the checks and the call of
        sfa_decode_step, with the per-operator constants looked up once."""
        if out is None:
            c = self.cfg
            out = self._new_out((c.n_layers, self.batch, c.hidden), stream)
        nq, nkv, nout = self._dec_numel
        dt = self._in_dtype
        rc = self._decode_fn(self.handle.ptr, _dev(q, "q", dt, nq), _dev(k, "k", dt, nkv),
                             _dev(v, "v", dt, nkv),
                             self.batch, _dev(self.state, "state", torch.uint8, self._state_bytes),
                             _dev(out, "out", self.handle.out_dtype, nout), _stream_ptr(stream))
        if rc != SFA_OK:
            raise SfaError(rc, "sfa_decode_step")
        return out

    def prefill_layers(self, layer_begin: int, q, k, v, out: Optional[torch.Tensor] = None,
                       stream=None):
        """Prefill of layers layer_begin .. layer_begin + q.shape[0] - 1."""
        lc, n = q.shape[0], q.shape[2]
        if out is None:
            out = self._new_out((lc, self.batch, n, self.cfg.hidden), stream)
        if n > 0:
            self._grow_workspace(sfa_prefill_layers_workspace_bytes(self.handle, lc, self.batch, n),
                                 stream)
            sfa_prefill_layers(self.handle, layer_begin, lc, q, k, v, n, self.batch, self.state,
                               out, self.workspace, stream)
        return out

    def decode_ex(self, layer_begin: int, q, k, v, seq_ids: Optional[torch.Tensor] = None,
                  out: Optional[torch.Tensor] = None, stream=None):
        """Decode of layers layer_begin .. layer_begin + q.shape[0] - 1 for the
        sequences in seq_ids (int32, on the device; None = all)."""
        lc, ns = q.shape[0], q.shape[1]
        if out is None:
            out = self._new_out((lc, ns, self.cfg.hidden), stream)
        sfa_decode_step_ex(self.handle, layer_begin, lc, seq_ids, q, k, v, self.batch,
                           self.state, out, stream)
        return out

    def check(self, stream=None) -> int:
        return sfa_check_device_status(self.handle, stream)

    def layout(self) -> sfa_state_layout:
        return sfa_state_layout_for(_layout_cfg(self.cfg), self.batch)


def _layout_cfg(cfg: SfaConfig) -> sfa_config:
    # Layout arithmetic needs a non-null, aligned slots pointer only for the
    # validity check; 16 is a stand-in address that is never dereferenced.
    return cfg.to_c(16)


def read_state(op: SfaOperator) -> dict:
    """Copies the state of every stream to host tensors (for tests/inspection):
    pos [L,B], win_k/win_v [L,B,k,n_kv,d], far [L,B,n_kv,d], field, ring_sum
    [L,B,H], ring [L,B,16,H]."""
    c = op.cfg
    lay = sfa_state_layout_for(_layout_cfg(c), op.batch)
    raw = op.state.cpu()
    L, B = c.n_layers, op.batch
    body = raw[lay.header_bytes: lay.header_bytes + L * B * lay.stream_stride]
    body = body.view(L, B, lay.stream_stride)
    esz = 4 if c.in_dtype == SFA_F32 else 2
    wdt = torch.float32 if c.in_dtype == SFA_F32 else torch.bfloat16
    K, nkv, d, H = c.window_k, c.n_kv_heads, c.head_dim, c.hidden

    def grab(off, nbytes, dtype, shape):
        return body[:, :, off: off + nbytes].contiguous().view(dtype).view(L, B, *shape)

    return {
        "pos": grab(lay.off_pos, 8, torch.int64, ()),
        "win_k": grab(lay.off_win_k, K * nkv * d * esz, wdt, (K, nkv, d)),
        "win_v": grab(lay.off_win_v, K * nkv * d * esz, wdt, (K, nkv, d)),
        "far": grab(lay.off_far, nkv * d * 4, torch.float32, (nkv, d)),
        "field": grab(lay.off_field, H * 4, torch.float32, (H,)),
        "ring_sum": grab(lay.off_ring_sum, H * 4, torch.float32, (H,)),
        "ring": grab(lay.off_ring, 16 * H * 4, torch.float32, (16, H)),
    }
