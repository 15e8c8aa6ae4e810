"""C-ABI checks that need no GPU: the library loads, exports every symbol the
header declares, validates configurations and lays out the state as the
pages describe."""
import ctypes
import os
import re

import pytest

import kv_cache_compression_sfa_b200 as sfa
from kv_cache_compression_sfa_b200 import build as sfa_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "sfa.h")
GOLDEN = os.path.join(ROOT, "tests", "golden")


@pytest.fixture(scope="module")
def lib():
    sfa_build.build()
    return sfa.load_library()


def _declared():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^SFA_API\s+[\w\s\*]+?\b(sfa_\w+)\s*\(", text, re.M)))


def test_header_declares_the_binding_surface():
    assert _declared() == sorted(sfa.EXPORTED)


def test_library_exports_every_declared_symbol(lib):
    for name in _declared():
        assert hasattr(lib, name), name
    # and nothing else with the sfa_ prefix leaks (internals are hidden)
    out = os.popen(f"nm -D --defined-only {sfa.LIB_PATH}").read()
    exported = sorted(set(re.findall(r"\bT (sfa_\w+)", out)))
    assert exported == _declared()


def test_plain_c_client_compiles_links_and_runs(lib, tmp_path):
    """The header is plain C99 and the library is enough to link against: a C
    program that includes only sfa.h builds with gcc -std=c99 -Wall -Wextra
    -Werror, links libsfa.so and runs the host-only calls without a GPU."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("gcc not found")
    exe = str(tmp_path / "c_abi_client")
    libdir = os.path.dirname(sfa.LIB_PATH)
    subprocess.run([gcc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic",
                    "-I", os.path.join(ROOT, "include"),
                    os.path.join(ROOT, "tests", "c_abi_client.c"), "-o", exe,
                    "-L", libdir, "-lsfa", f"-Wl,-rpath,{libdir}"], check=True)
    r = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == "ok"


def test_abi_version(lib):
    assert sfa.sfa_abi_version() == 3


def _golden(name):
    vals = {}
    for line in open(os.path.join(GOLDEN, name)):
        line = line.split("--")[0].split("#")[0].strip()
        if "=" in line:
            a, b = line.split("=")
            vals[a.strip()] = float(b)
    return vals


def test_config_default_is_the_printed_config(lib):
    g = _golden("sfa_config_defaults.txt")
    c = sfa.sfa_config_default()
    assert c.alpha_base == pytest.approx(g["alpha_base"])
    assert c.cross_decay == pytest.approx(g["cross_decay"])
    assert c.ema_gamma == pytest.approx(g["ema_gamma"])
    assert c.ring_size == g["ring_size"]
    assert c.n_slots == g["n_slots"]
    assert c.clip_eps == pytest.approx(g["enhancement_clip"])
    assert c.temperature == pytest.approx(g["temperature"])
    assert c.window_k == g["window_k"]
    assert c.slots is None


def _cfg(**kw):
    base = dict(n_layers=2, n_q_heads=4, n_kv_heads=2, head_dim=64)
    base.update(kw)
    return sfa.SfaConfig(**base)


@pytest.mark.parametrize("kw,code", [
    ({}, sfa.SFA_OK),
    ({"n_layers": 0}, sfa.SFA_ERR_INVALID_ARG),
    ({"n_q_heads": 6, "n_kv_heads": 4}, sfa.SFA_ERR_INVALID_ARG),
    ({"head_dim": 96}, sfa.SFA_ERR_UNSUPPORTED),
    ({"window_k": 0}, sfa.SFA_ERR_INVALID_ARG),
    ({"window_k": 257}, sfa.SFA_ERR_UNSUPPORTED),
    ({"ring_size": 8}, sfa.SFA_ERR_UNSUPPORTED),
    ({"n_slots": 32}, sfa.SFA_ERR_UNSUPPORTED),
    ({"temperature": 0.0}, sfa.SFA_ERR_INVALID_ARG),
    ({"temperature": 1e-45}, sfa.SFA_ERR_INVALID_ARG),   # 1/T overflows to inf
    ({"gamma_far": 1.5}, sfa.SFA_ERR_INVALID_ARG),
    ({"ema_gamma": float("nan")}, sfa.SFA_ERR_INVALID_ARG),
    ({"clip_eps": -1.0}, sfa.SFA_ERR_INVALID_ARG),
    ({"in_dtype": 7}, sfa.SFA_ERR_INVALID_ARG),
    ({"n_q_heads": 128, "n_kv_heads": 8, "head_dim": 128}, sfa.SFA_ERR_UNSUPPORTED),
    ({"n_q_heads": 17, "n_kv_heads": 1}, sfa.SFA_ERR_UNSUPPORTED),   # no cluster split of 17 heads
    ({"gamma_far": 1.0}, sfa.SFA_OK),                                # S stays as it is
    ({"gamma_far": -0.1}, sfa.SFA_ERR_INVALID_ARG),
])
def test_config_validate_codes(lib, kw, code):
    assert sfa.sfa_config_validate(_cfg(**kw).to_c(256)) == code


def test_config_validate_slots_pointer(lib):
    assert sfa.sfa_config_validate(_cfg().to_c(0)) == sfa.SFA_ERR_INVALID_ARG
    assert sfa.sfa_config_validate(_cfg().to_c(260)) == sfa.SFA_ERR_ALIGNMENT


def test_state_layout_channel_sizes_match_the_pages(lib):
    """README architecture diagram at hidden 1024: ring ~64 KB, field ~4 KB,
    pool ~256 KB (fp32): 16*H*4, H*4 and 64*H*4 bytes."""
    g = _golden("channel_memory.txt")
    H = int(g["hidden"])
    cfg = _cfg(n_q_heads=16, n_kv_heads=2, head_dim=64)  # hidden 1024
    assert cfg.hidden == H
    lay = sfa.sfa_state_layout_for(cfg.to_c(256), 1)
    assert lay.off_ring_sum - lay.off_field == g["field_bytes"]     # field: H fp32
    assert lay.stream_stride - lay.off_ring == g["ring_bytes"]      # ring: 16 x H fp32
    assert cfg.n_slots * H * 4 == g["pool_bytes"]                   # slots: 64 x H fp32


def test_state_layout_is_constant_in_context_and_linear_in_batch(lib):
    """[P1 §2.2]: O(k·d) state; nothing grows with the sequence length."""
    cfg = _cfg(n_layers=28, n_q_heads=28, n_kv_heads=4, head_dim=128)
    l1 = sfa.sfa_state_layout_for(cfg.to_c(256), 1)
    l8 = sfa.sfa_state_layout_for(cfg.to_c(256), 8)
    assert l8.total_bytes - l8.header_bytes == 8 * (l1.total_bytes - l1.header_bytes)
    assert l1.header_bytes == 256 and l1.stream_stride % 256 == 0
    offs = [l1.off_pos, l1.off_win_k, l1.off_win_v, l1.off_far, l1.off_field, l1.off_ring_sum,
            l1.off_ring]
    assert offs == sorted(offs) and all(o % 256 == 0 for o in offs)
    # window bytes: k x n_kv x d x 2 (bf16)
    assert l1.off_win_v - l1.off_win_k == 16 * 4 * 128 * 2


def test_state_layout_rejects_bad_batch(lib):
    with pytest.raises(sfa.SfaError):
        sfa.sfa_state_layout_for(_cfg().to_c(256), 0)


def test_status_strings(lib):
    for code in range(-7, 1):
        assert sfa.sfa_status_string(code) != "unknown status"
    assert sfa.sfa_status_string(-99) == "unknown status"


def test_library_needs_no_gpu_to_load_and_init_fails_cleanly_without_one(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("GPU present")
    c = _cfg().to_c(256)
    h = ctypes.c_void_p()
    rc = lib.sfa_init(ctypes.byref(c), ctypes.byref(h))
    assert rc == sfa.SFA_ERR_CUDA and h.value is None
