"""The enhancement-share diagnostic computed from the CUDA path agrees with
the same statistics computed from the fp64 oracle's outputs."""
import dataclasses

import numpy as np
import pytest

import bench
from sfa_harness import Pair
from workloads import WORKLOADS

pytestmark = pytest.mark.gpu


def test_enhancement_share_matches_the_oracle():
    base = WORKLOADS["tiny"]
    got, ref = {}, {}
    for ab in (0.0, 10.0):
        w = base.replace(values=dataclasses.replace(base.values, alpha_base=ab))
        pair = Pair(w)
        g, r = pair.prefill(128)
        got[ab], ref[ab] = g, r
    sg = bench.enhancement_stats(got[0.0], got[10.0])
    sr = bench.enhancement_stats(ref[0.0], ref[10.0])
    for key in ("cos_median", "share_median", "share_p90"):
        assert abs(sg[key] - sr[key]) < 1e-3, (key, sg[key], sr[key])
    # the enhancement is bounded by eps * alpha_layer (0.5 * 0.3 * 10 at L = 1)
    assert np.abs(got[10.0] - got[0.0]).max() <= 0.5 * 0.3 * 10.0 + 1e-6


def test_context_flatness_rows_report_the_state_layout():
    """The context-flatness path of bench.py (state bytes per sequence and
    decode time after prompts of several lengths) on a small 7B-shaped
    model: the state bytes are the library's layout, constant in the
    context, and the full-K/V figure grows with it."""
    import torch

    import kv_cache_compression_sfa_b200 as sfa
    from sfa_harness import sfa_config
    w = WORKLOADS["qwen7b_decode"].replace(n_layers=2)
    rows = bench.context_rows(w, sfa, torch.device("cuda", 0), (64, 300, 1024), n_dec=4, reps=1)
    lay = sfa.sfa_state_layout_for(sfa_config(w).to_c(16), w.batch)
    assert [r["context"] for r in rows] == [64, 300, 1024]
    for r in rows:
        assert r["sfa_state_bytes_per_seq"] == lay.stream_stride * w.n_layers
        assert r["full_kv_bytes_per_seq"] == bench.full_kv_bytes(w, r["context"])
        assert r["compression"] == pytest.approx(r["full_kv_bytes_per_seq"] / r["sfa_state_bytes_per_seq"])
        assert r["decode_us_per_step"] > 0
    assert rows[2]["compression"] > rows[0]["compression"]
