"""GPU parity: the CUDA library against the fp64 oracle on seeded inputs.

Every output element and the final state are compared with
|gpu - oracle| <= tol * (1 + |oracle|), tol = 1e-4 (fp32 inputs) or 2e-3
(bf16 inputs); window slots (copies of inputs) and positions must match
exactly.  Full-size workloads compare a seeded subset of (layer, sequence)
streams, whose whole token sequence the oracle replays.
"""
import dataclasses

import numpy as np
import pytest
import torch

import kv_cache_compression_sfa_b200 as sfa
from sfa_harness import TOL, Pair, assert_close
from workloads import WORKLOADS, SfaConfigValues, Workload, sweep_c5

pytestmark = pytest.mark.gpu


def _tiny_variant(**kw) -> Workload:
    base = WORKLOADS["tiny"]
    vals = kw.pop("values", {})
    return base.replace(values=dataclasses.replace(base.values, **vals), **kw)


def _run_schedule(w: Workload, schedule, layers=None, seqs=None, check_state=True, paths=None):
    """schedule: list of ("p", n) prefill calls and ("d", steps) decode runs;
    paths: (decode_tile, prefill_near) for sfa_debug_set_paths."""
    pair = Pair(w, layers=layers, seqs=seqs)
    if paths is not None:
        sfa.sfa_debug_set_paths(pair.op.handle, *paths)
    tol = TOL[w.in_dtype]
    for kind, n in schedule:
        if kind == "p":
            got, ref = pair.prefill(n)
            assert_close(got, ref, tol, f"{w.name} prefill {n} at t={pair.t - n}")
        else:
            got, ref = pair.decode_many(n)
            assert_close(got, ref, tol, f"{w.name} decode x{n} at t={pair.t - n}")
    assert pair.status() == 0
    if check_state:
        pair.compare_state(tol)
    return pair


def test_tiny_workload_prefill_128_then_32_decode_steps():
    w = WORKLOADS["tiny"]
    _run_schedule(w, [("p", 128), ("d", 32)])


def test_qwen05b_workload_prefill_512_then_128_decode_steps():
    w = WORKLOADS["qwen05b"]
    _run_schedule(w, [("p", 512), ("d", 128)])


@pytest.mark.parametrize("context", [1024, 4096, 8192])
def test_qwen7b_decode_after_context(context):
    w = WORKLOADS["qwen7b_decode"]
    _run_schedule(w, [("p", context), ("d", 256)], layers=[0, 13, 27])


def test_long_prefill_65536_tokens_x4():
    w = WORKLOADS["long_prefill"]
    pair = Pair(w, seqs=[0, 3])
    tol = TOL[w.in_dtype]
    got, ref = pair.prefill(65536)
    assert_close(got, ref, tol, "long prefill")
    assert pair.status() == 0
    pair.compare_state(tol)


@pytest.mark.parametrize("w", sweep_c5(), ids=lambda w: w.name)
def test_batched_decode_sweep(w):
    """256 sequences x 28 layers: 1,024 prefilled tokens (in chunks of 128),
    then 512 decode steps; the oracle replays 9 streams."""
    pair = Pair(w, layers=[0, 14, 27], seqs=[0, 128, 255])
    tol = TOL[w.in_dtype]
    for c in range(8):
        got, ref = pair.prefill(128)
        assert_close(got, ref, tol, f"{w.name} prefill chunk {c}")
    for c in range(8):
        got, ref = pair.decode_many(64)
        assert_close(got, ref, tol, f"{w.name} decode steps {64 * c}..{64 * c + 63}")
    assert pair.status() == 0
    pair.compare_state(tol)


# ----------------------------------------------------------- edge cases

EDGE = [
    # name, workload overrides, schedule
    ("gqa_f32_d64", dict(n_q_heads=4, n_kv_heads=2, window_k=4),
     [("p", 1), ("p", 2), ("p", 15), ("p", 16), ("d", 3), ("p", 63), ("p", 65), ("d", 5)]),
    ("mha_k1", dict(n_q_heads=2, n_kv_heads=2, window_k=1), [("p", 70), ("d", 4), ("p", 3)]),
    ("k256_spans_tiles", dict(n_q_heads=4, n_kv_heads=1, window_k=256),
     [("p", 100), ("p", 200), ("d", 7), ("p", 130), ("d", 3)]),
    ("d128_f32_multilayer", dict(n_layers=3, batch=2, n_q_heads=4, n_kv_heads=2, head_dim=128,
                                 window_k=16), [("p", 130), ("d", 6), ("p", 1)]),
    ("gqa7_bf16", dict(n_layers=2, batch=3, n_q_heads=14, n_kv_heads=2, head_dim=64,
                       window_k=16, in_dtype="bf16"), [("p", 200), ("d", 10)]),
    ("decode_from_empty", dict(n_q_heads=4, n_kv_heads=2, window_k=8), [("d", 40), ("p", 9)]),
    ("gamma_zero_alpha_big", dict(n_q_heads=4, n_kv_heads=2, window_k=5,
                                  values=dict(gamma_far=0.0, alpha_far=1.0, alpha_base=10.0,
                                              cross_decay=0.98)),
     [("p", 77), ("d", 9)]),
    ("eight_heads_per_cta", dict(n_q_heads=16, n_kv_heads=16, head_dim=64, window_k=3),
     [("p", 66), ("d", 2)]),
    # bf16, k <= 16: the tensor-core near field with tensor copies; short and
    # ragged calls put a call's first tile (rows before the call from the
    # state window) next to stream boundaries
    ("bf16_small_chunks", dict(n_layers=2, batch=2, n_q_heads=4, n_kv_heads=2, head_dim=64,
                               window_k=12, in_dtype="bf16"),
     [("p", 3), ("p", 17), ("d", 2), ("p", 64), ("p", 1), ("p", 130), ("d", 3)]),
    ("bf16_d128_small_chunks", dict(n_layers=1, batch=3, n_q_heads=4, n_kv_heads=1, head_dim=128,
                                    window_k=16, in_dtype="bf16"),
     [("p", 15), ("p", 16), ("p", 65), ("d", 1), ("p", 2)]),
]


@pytest.mark.parametrize("name,over,schedule", EDGE, ids=[e[0] for e in EDGE])
def test_edge_schedules(name, over, schedule):
    w = _tiny_variant(name=name, **over)
    _run_schedule(w, schedule)


def test_cuda_core_near_field_on_bf16_inputs():
    """bf16 inputs with k <= 16 take the tensor-core near field; the handle's
    test hook keeps them on the CUDA cores, which must meet the same bar."""
    w = _tiny_variant(name="cuda_core_near_bf16", n_layers=2, batch=2, n_q_heads=14,
                      n_kv_heads=2, head_dim=64, window_k=16, in_dtype="bf16")
    _run_schedule(w, [("p", 130), ("d", 5), ("p", 70)], paths=(-1, False))


@pytest.mark.parametrize("mode", [1, 2], ids=["unfused", "fused"])
@pytest.mark.parametrize("name,over,schedule", [e for e in EDGE if e[1].get("in_dtype") == "bf16"],
                         ids=[e[0] for e in EDGE if e[1].get("in_dtype") == "bf16"])
def test_tensor_core_prefill_paths(name, over, schedule, mode):
    """Each tensor-core prefill path pinned by the handle's test hook (by
    default calls this small take the unfused one): the near field followed
    by the separate pool kernel (1), and the fused kernel (2)."""
    w = _tiny_variant(name=name + f"_tc{mode}", **over)
    _run_schedule(w, schedule, paths=(-1, mode))


@pytest.mark.parametrize("mode", [1, 2], ids=["unfused", "fused"])
def test_gqa7_bf16_chunked_prefill_and_decode(mode):
    """Seven query heads per KV head, bf16, prefill calls across a decode."""
    w = _tiny_variant(name=f"gqa7_bf16_chunks_tc{mode}", n_layers=2, batch=2, n_q_heads=14,
                      n_kv_heads=2, head_dim=64, window_k=16, in_dtype="bf16")
    _run_schedule(w, [("p", 130), ("d", 5), ("p", 70)], paths=(-1, mode))


@pytest.mark.parametrize("name,over,schedule", EDGE, ids=[e[0] for e in EDGE])
def test_batch_tiled_decode_on_edge_schedules(name, over, schedule):
    """The batch-tiled decode (64 sequences per cluster, pool on the tensor
    cores) serves every batch when the handle's test hook pins it; same bar
    as above."""
    w = _tiny_variant(name=name + "_tiled", **over)
    _run_schedule(w, schedule, paths=(1, True))


def test_batch_tiled_decode_partial_tile_and_sequence_list():
    """70 sequences (a full and a partial tile), then a permuted subset."""
    w = _tiny_variant(name="tiled_70", n_layers=2, batch=70, n_q_heads=14, n_kv_heads=2,
                      head_dim=64, window_k=16, in_dtype="bf16")
    pair = Pair(w, seqs=[0, 1, 63, 64, 69])
    tol = TOL[w.in_dtype]
    got, ref = pair.prefill(20)
    assert_close(got, ref, tol, "prefill")
    got, ref = pair.decode_many(6)  # 70 >= 64 sequences: the batch-tiled decode
    assert_close(got, ref, tol, "tiled decode")
    assert pair.status() == 0
    pair.compare_state(tol)
